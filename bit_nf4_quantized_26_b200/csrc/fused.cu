// fused.cu — dequantise-in-GEMM kernels of the QLoRA linear ("QLoRA"
// encyclopedia entry, tonho.wtf, section "a ideia": the 4-bit weight is
// dequantised to BFloat16 at the moment of use and discarded; the gradient
// crosses the frozen weight).
//
//   forward:  Y^T tile [128 n x BN m]  = W'[n, k] . X[m, k]^T      (+ B . (sU)^T)
//   dX:       dX^T tile [128 k x BN m] = W'[n, k]^T . dY[m, n]^T   (+ A^T . dU^T)
//
// The W side is the MMA's M = 128 dimension, tokens are its N = BN dimension,
// so one dequantised element feeds BN tokens.  Warp roles (64 + 32 DQW threads):
//   warp 0      TMA producer (token tile + packed codes; LoRA operands)
//   warp 1      TMEM owner and tcgen05.mma issuer (warp-uniform loop, elected lane)
//   warps 2..   dequantisers, DQW / 4 groups of four taking stages in turn: one
//               thread per 64-element NF4 block per stage, 16 lookups of bf16
//               pairs written straight into the 128-byte swizzled operand
//               layout; afterwards the epilogue (TMEM -> global)
// The LoRA up-projection is appended to the contraction as extra K steps over
// the interleaved hi/lo bf16 split of the fp32 down-projection, accumulated in
// the same TMEM accumulator (no second pass over Y).  No TMA multicast.
#include <cstdlib>

#include "kernels.h"

namespace qnf4 {

// Ring plan.  For a handful of tokens (BN <= 64) the kernel only streams the
// weight: two CTAs share an SM (3-4 stages each) so more dequantiser warps
// hide the lookup latency; larger tiles run one CTA per SM with a deep ring.
template <int BN>
struct FusedPlan {
  static constexpr uint32_t kB = BN * 128;  // token tile, 64 bf16 per row
  static constexpr uint32_t kA = 16384;     // W-side tile 128 x 64 bf16
  static constexpr uint32_t kC = 4096;      // packed codes of the stage
  static constexpr uint32_t kStage = kB + kA + kC;
  static constexpr uint32_t kCtasPerSm = BN <= 128 ? 2 : 1;
  static constexpr uint32_t kFit = (233472u / kCtasPerSm - 1024u - 2048u) / kStage;
  static constexpr uint32_t kStages = kFit > 8 ? 8 : kFit;
  static constexpr uint32_t kBarOff = kStages * kStage;
  static constexpr uint32_t kSmem = 1024 + kBarOff + 256;
  // Split contraction: the idle ring receives the slices of the partial tiles
  // this CTA reduces, rows padded by 4 floats so that row-wise accesses
  // spread over the banks.
  static constexpr uint32_t kPartLd = BN + 4;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kStages >= 3, "pipeline too shallow");
  // receive slots of a split reduction: S slots of ceil(128 / S) rows, S <= 8
  static_assert(136 * kPartLd * 4 <= kBarOff, "split-reduction slots must fit in the ring");
};

template <int BN, bool DX, int DQW>
__global__ void __launch_bounds__(64 + 32 * DQW, FusedPlan<BN>::kCtasPerSm)
    fused_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_codes,
                 const __grid_constant__ CUtensorMap tm_uc, const __grid_constant__ CUtensorMap tm_ext,
                 const FusedArgs a) {
  using P = FusedPlan<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::kBarOff);
  uint64_t* wfull = full + P::kStages;
  uint64_t* empty = wfull + P::kStages;
  uint64_t* accf = empty + P::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * 128;
  const int m0 = blockIdx.y * BN;
  const int z = blockIdx.z;
  const int kt0 = z * a.kt_per_split;
  const int kt1 = min(a.kt_total, kt0 + a.kt_per_split);
  const int nmain = kt1 - kt0;
  const int next = (z == 0) ? (2 * a.r + 63) / 64 : 0;
  const int T = nmain + next;

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < P::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&wfull[s], 4);  // one elected arrival per dequantiser warp of the stage
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_uc);
    tma_prefetch_desc(&tm_ext);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  const WaitCtx wc{abort_flag, a.status};
  // Programmatic dependent launch: of this kernel's inputs, only the hi/lo
  // of sU / dU (read by the extension stages) comes from the kernel launched
  // just before it; the rest comes from earlier kernels, complete when that
  // kernel let this one launch.  The producer waits just before the first
  // extension load; every other role passes the wait after its main loop,
  // before triggering the next kernel.

  bool acc_ok = false;  // dequantiser warps: the accumulators are final
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    bool waited = false;
    // Grouped forward: this tile's member reads its own columns of the hi/lo copy of s*U.
    const int uc0 = DX ? 0 : group_member(a.grp_end, a.groups, row0) * 2 * a.r;
    if (lane == 0) {
      // The codes are the part of a stage that streams from DRAM (each is
      // read by one CTA).  With one CTA per SM they are pulled into L2 ahead
      // (stages kStages .. kPfAhead - 1 now, stage t + kPfAhead with stage
      // t): 4-7% at 200-256 tokens.  With two CTAs per SM it measured
      // neutral to 2% slower, and is off.
      constexpr int kPfAhead = P::kCtasPerSm == 1 ? static_cast<int>(P::kStages) + 4 : 0;
      auto prefetch_codes = [&](int t) {
        if (kPfAhead == 0 || t >= nmain) return;
        const int kt = kt0 + t;
        if (!DX) tma_prefetch_l2_2d(&tm_codes, kt * 32, row0);
        else tma_prefetch_l2_2d(&tm_codes, row0 / 2, kt * 64);
      };
      for (int t = P::kStages; t < kPfAhead; ++t) prefetch_codes(t);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (t >= static_cast<int>(P::kStages) && !mbar_wait(&empty[s], (u - 1) & 1, wc)) break;
        prefetch_codes(t + kPfAhead);
        uint8_t* st = smem + s * P::kStage;
        if (t < nmain) {
          const int kt = kt0 + t;
          mbar_arrive_expect_tx(&full[s], P::kB + P::kC);
          tma_load_2d(st, &tm_b, &full[s], kt * 64, m0);
          if (!DX) tma_load_2d(st + P::kB + P::kA, &tm_codes, &full[s], kt * 32, row0);
          else tma_load_2d(st + P::kB + P::kA, &tm_codes, &full[s], row0 / 2, kt * 64);
        } else {
          if (!waited) {
            grid_dependency_wait();  // sU / dU of the preceding kernel are complete and visible
            grid_dependents_launch();
            waited = true;
          }
          const int e = t - nmain;
          if (!DX) {
            mbar_arrive_expect_tx(&full[s], P::kB + 16384);
            tma_load_2d(st, &tm_uc, &full[s], uc0 + 64 * e, m0);
            tma_load_2d(st + P::kB, &tm_ext, &full[s], 32 * e, row0);
          } else {
            const bool second = row0 + 64 < a.rows;
            mbar_arrive_expect_tx(&full[s], P::kB + (second ? 16384 : 8192));
            tma_load_2d(st, &tm_uc, &full[s], uc0 + 64 * e, m0);
            tma_load_2d(st + P::kB, &tm_ext, &full[s], row0, 32 * e);
            if (second) tma_load_2d(st + P::kB + 8192, &tm_ext, &full[s], row0 + 64, 32 * e);
          }
        }
        issued = t + 1;
      }
      // Do not leave the CTA while a copy into its shared memory is in flight.
      for (int t = max(0, issued - static_cast<int>(P::kStages)); t < issued; ++t)
        mbar_drain(&full[t % P::kStages], (t / P::kStages) & 1, a.status);
    }
    __syncwarp();  // the other lanes pass the wait only after lane 0 is through its loop
    if (!waited) {  // lanes 1..31, a split without extension stages, or a producer that gave up
      grid_dependency_wait();
      grid_dependents_launch();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (warp-uniform waits and descriptors); the
    // elected lane issues the MMAs and the commits.
    {
      const uint32_t idesc = idesc_bf16_f32(128, BN, DX ? 1 : 0, 0);
      const uint32_t a_step = DX ? (2048u >> 4) : (32u >> 4);  // one K=16 step, descriptor units
      bool aborted = false;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait_all(&full[s], u & 1, wc)) { aborted = true; break; }
        if (t < nmain && !mbar_wait_all(&wfull[s], u & 1, wc)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + s * P::kStage);
        const uint32_t sa = sb + P::kB;
        const uint64_t bdesc = sdesc_sw128(sb, 16, 1024);
        const uint64_t adesc = DX ? sdesc_sw128(sa, 8192, 1024) : sdesc_sw128(sa, 16, 1024);
        if (elect_one()) {
          if (t < nmain) {
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)
              umma_bf16(tmem_d, adesc + kk * a_step, bdesc + kk * 2, idesc, (t | kk) != 0 ? 1u : 0u);
          } else {
            const int e = t - nmain;
            const int nkk = min(64, 2 * a.r - 64 * e) / 16;
            for (int kk = 0; kk < nkk; ++kk)
              umma_bf16(tmem_d, adesc + static_cast<uint32_t>(kk >> 1) * a_step, bdesc + static_cast<uint32_t>(kk) * 2,
                        idesc, 1u);
          }
          umma_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (elect_one()) {
        umma_commit(accf);
        if (aborted) mbar_drain(accf, 0, a.status);
      }
    }
    __syncwarp();
    grid_dependency_wait();
    grid_dependents_launch();
  } else {
    // ------------------------------------------------------------ dequantisers
    // Thread dt owns tile row dt % 128 (one whole NF4 block per stage).
    // DQW == 8: two groups of four warps take alternate stages (two
    // independent instruction streams per SM sub-partition).
    const int dt = threadIdx.x - 64;
    const Nf4Mean wmean = nf4_load_mean(a.mean);  // from an earlier kernel: complete (see above)
    const int rl = dt & 127;
    constexpr int kStep = DQW / 4;  // stages between two of this group's
    const int grp = dt >> 7;
    const int64_t kbpr = a.k_in / 64;  // NF4 blocks per W row
    auto block_of = [&](int t, int64_t& b) -> bool {
      const int kt = kt0 + t;
      if (!DX) {
        const int n = row0 + rl;
        b = static_cast<int64_t>(n) * kbpr + kt;
        return n < a.n_out;
      } else {
        const int n = kt * 64 + (rl & 63);
        const int kb = row0 / 64 + (rl >> 6);
        b = static_cast<int64_t>(n) * kbpr + kb;
        return n < a.n_out && kb < kbpr;
      }
    };
    // register prefetch of the block constants, six stages ahead for a
    // handful of tokens (the weight streams through once: cover a DRAM miss),
    // four for 128 or more (two CTAs of 128 tokens per SM sit at the register
    // limit; each of their stages takes longer)
    constexpr int kPD = BN >= 128 ? 4 : 6;
    uint32_t pc[kPD];
    float ps[kPD];
    auto fetch = [&](int t, uint32_t& c, float& sv) {
      int64_t b;
      if (t < nmain && block_of(t, b)) {
        c = __ldg(a.c8 + b);
        sv = __ldg(a.s2 + (b >> 8));
      } else {
        c = 0;
        sv = 0.f;
      }
    };
#pragma unroll
    for (int i = 0; i < kPD; ++i) fetch(grp + kStep * i, pc[i], ps[i]);
    for (int t = grp; t < nmain; t += kStep) {
      const uint32_t c8b = pc[0];
      const float s2v = ps[0];
#pragma unroll
      for (int i = 0; i + 1 < kPD; ++i) {
        pc[i] = pc[i + 1];
        ps[i] = ps[i + 1];
      }
      fetch(t + kStep * kPD, pc[kPD - 1], ps[kPD - 1]);
      int64_t bdummy;
      const bool valid = block_of(t, bdummy);
      const uint32_t s = t % P::kStages, u = t / P::kStages;
      // When the ring is not a multiple of the group count the slot's
      // previous stage t - kStages belongs to another group, and this group
      // may get here before that stage's copy has landed; a parity wait on
      // full[s] would then see the older phase as this one.  Waiting first
      // for the MMA of stage t - kStages (which the refill needs anyway)
      // rules that out.
      if (P::kStages % kStep != 0 && u > 0 && !mbar_wait_all(&empty[s], (u - 1) & 1, wc)) break;
      if (!mbar_wait_all(&full[s], u & 1, wc)) break;
      uint8_t* st = smem + s * P::kStage;
      const uint8_t* src;
      uint8_t* dst;
      uint32_t swz;
      if (!DX) {
        src = st + P::kB + P::kA + rl * 32;
        dst = st + P::kB + rl * 128;
        swz = rl & 7;
      } else {
        const int nl = rl & 63, bs = rl >> 6;
        src = st + P::kB + P::kA + nl * 64 + bs * 32;
        dst = st + P::kB + bs * 8192 + (nl >> 3) * 1024 + (nl & 7) * 128;
        swz = nl & 7;
      }
      const float chat = valid ? nf4_block_scale(c8b, s2v, wmean) : 0.0f;
      if (valid) {
        nf4_block_to_swizzled_row(src, nf4_make_lut(a.tab, chat), dst, swz);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(dst + j * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();  // this lane's tile writes -> async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(&wfull[s]);
    }

    grid_dependency_wait();
    grid_dependents_launch();

    // ------------------------------------------------------------ epilogue
    // Warp w reads TMEM lane quadrant w % 4; the groups' warps of a quadrant
    // split the BN accumulator columns between them.
    acc_ok = mbar_wait_warp(accf, 0, wc);
    if (acc_ok && gridDim.z == 1) {
      tc_fence_after();
      const int q = warp & 3;
      const int erow = q * 32 + lane;
      const int cgrp = (warp - 2) / 4;
      constexpr int kAll = BN / 32;                              // 32-column chunks
      constexpr int kChunks = (kAll + DQW / 4 - 1) / (DQW / 4);  // per column group
      const int orow = row0 + erow;
      const bool rok = orow < a.rows;
      const uint32_t tq = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
      {
#pragma unroll 1
        for (int ci = 0; ci < kChunks; ++ci) {
          const int cb = cgrp * kChunks + ci;
          if (cb >= kAll) break;  // warp-uniform
          uint32_t v[32];
          tmem_ld_32x32b_x32(tq + cb * 32, v);
          tmem_ld_wait();
          if (rok) {
            const int mb = m0 + cb * 32;
            const int nv = min(32, a.M - mb);
            const int64_t ld = a.ld_out;
            if (a.out_f32) {
              float* o = reinterpret_cast<float*>(a.out) + orow + static_cast<int64_t>(mb) * ld;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (j < nv) *o = __uint_as_float(v[j]);
                o += ld;
              }
            } else {
              uint16_t* o = reinterpret_cast<uint16_t*>(a.out) + orow + static_cast<int64_t>(mb) * ld;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (j < nv) *o = bf16_bits(__uint_as_float(v[j]));
                o += ld;
              }
            }
          }
        }
      }
    }
  }

  if (gridDim.z > 1) {
    // Split contraction: the S CTAs of the cluster (one per slice of the
    // contraction, cluster rank = blockIdx.z) reduce the tile together; CTA o
    // owns rows [o R, o R + R) of it, R = ceil(128 / S).  Each CTA writes its
    // accumulator rows straight from tensor memory into the owners' receive
    // slots (slot = the writer's rank) with remote stores, which pipeline,
    // and then every owner sums its slots from its own shared memory in rank
    // order 0..S-1 (deterministic) and writes the outputs.
    __syncwarp();
    cluster_sync_all();  // every CTA's rings are idle: its dequantiser warps saw accf
    const int S = static_cast<int>(gridDim.z);
    const int R = (128 + S - 1) / S;
    const uint32_t slot_bytes = static_cast<uint32_t>(R * P::kPartLd * 4);
    if (acc_ok) {
      tc_fence_after();
      const int q = warp & 3;
      const int erow = q * 32 + lane;
      const int cgrp = (warp - 2) / 4;
      constexpr int kAll = BN / 32;
      constexpr int kChunks = (kAll + DQW / 4 - 1) / (DQW / 4);
      const uint32_t tq = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
      const int own = erow / R;
      const uint32_t dst0 = dsmem_addr(smem, static_cast<uint32_t>(own)) + static_cast<uint32_t>(z) * slot_bytes +
                            static_cast<uint32_t>((erow - own * R) * P::kPartLd * 4);
#pragma unroll 1
      for (int ci = 0; ci < kChunks; ++ci) {
        const int cb = cgrp * kChunks + ci;
        if (cb >= kAll) break;  // warp-uniform
        uint32_t v[32];
        tmem_ld_32x32b_x32(tq + cb * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          dsmem_st_f4(dst0 + static_cast<uint32_t>((cb * 32 + j) * 4), __uint_as_float(v[j]),
                      __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
      }
    }
    __syncwarp();
    cluster_sync_all();  // every slot is written
    const int r0 = z * R, nrow = min(128, r0 + R) - r0;
    const float* slots = reinterpret_cast<const float*>(smem);
    const int64_t ld = a.ld_out;
    constexpr int kC4 = BN / 4;
    for (int e = threadIdx.x; e < nrow * kC4; e += blockDim.x) {
      const int row = e % nrow, c4 = (e / nrow) * 4;
      const float* src = slots + row * P::kPartLd + c4;
      float4 acc = *reinterpret_cast<const float4*>(src);
      for (int k = 1; k < S; ++k) {
        const float4 v = *reinterpret_cast<const float4*>(src + k * R * P::kPartLd);
        acc.x = __fadd_rn(acc.x, v.x);
        acc.y = __fadd_rn(acc.y, v.y);
        acc.z = __fadd_rn(acc.z, v.z);
        acc.w = __fadd_rn(acc.w, v.w);
      }
      const int orow = row0 + r0 + row;
      const float o[4] = {acc.x, acc.y, acc.z, acc.w};
      if (orow < a.rows) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = m0 + c4 + i;
          if (m < a.M) {
            if (a.out_f32) reinterpret_cast<float*>(a.out)[orow + static_cast<int64_t>(m) * ld] = o[i];
            else reinterpret_cast<uint16_t*>(a.out)[orow + static_cast<int64_t>(m) * ld] = bf16_bits(o[i]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, BN);
  }
}

// ============================================================================
// fused2x: large-M variant.  One CTA owns 128 W-side rows and 512 tokens in two
// 128 x 256 fp32 TMEM accumulators (all 512 TMEM columns), so every
// dequantised weight feeds 512 tokens: half the integer-pipe work per MMA
// FLOP of the 256-token kernel.  Stages are 32 deep along the contraction
// (64-byte swizzled token tiles) so that five stages fit in shared memory.
//   forward: a thread owns one W row; an NF4 block spans two stages and its
//            table is built once and reused for the second half.
//   dX:      a stage covers 32 W rows x 128 columns = 64 blocks; a pair of
//            adjacent lanes shares a block (table built jointly).
// The LoRA extension adds r/16 stages, each one 16-wide j block as a hi and a
// lo MMA.
// ============================================================================

struct Plan2x {
  static constexpr uint32_t kBh = 256 * 64;   // 256 tokens x 32 bf16, one accumulator's operand
  static constexpr uint32_t kB = 2 * kBh;     // 32 KB
  static constexpr uint32_t kA = 8192;        // 128 x 32 bf16
  static constexpr uint32_t kC = 2048;        // packed codes of the stage
  static constexpr uint32_t kStage = kB + kA + kC;
  static constexpr uint32_t kStages = 5;
  static constexpr uint32_t kBarOff = kStages * kStage;
  static constexpr uint32_t kSmem = 1024 + kBarOff + 256;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kSmem <= 232448u, "too much shared memory");
};

template <bool DX>
__global__ void __launch_bounds__(192, 1)
    fused2x_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_uc, const __grid_constant__ CUtensorMap tm_ext,
                   const FusedArgs a) {
  using P = Plan2x;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::kBarOff);
  uint64_t* wfull = full + P::kStages;
  uint64_t* empty = wfull + P::kStages;
  uint64_t* accf = empty + P::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * 128;
  const int m0 = blockIdx.y * 512;
  const int nmain = a.kt_total;               // stages of 32
  const int next = a.r / 16;                  // one per 16-wide j block
  const int T = nmain + next;

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < P::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&wfull[s], 4);  // one elected arrival per dequantiser warp
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_uc);
    tma_prefetch_desc(&tm_ext);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  const WaitCtx wc{abort_flag, a.status};
  // Programmatic dependent launch: of this kernel's inputs, only the hi/lo
  // of sU / dU (read by the extension stages) comes from the kernel launched
  // just before it; the rest comes from earlier kernels, complete when that
  // kernel let this one launch.  The producer waits just before the first
  // extension load; every other role passes the wait after its main loop,
  // before triggering the next kernel.

  if (warp == 0) {
    bool waited = false;
    // Grouped forward: this tile's member reads its own columns of the hi/lo copy of s*U.
    const int uc0 = DX ? 0 : group_member(a.grp_end, a.groups, row0) * 2 * a.r;
    if (lane == 0) {
      int issued = 0;
      const bool a2 = !DX || row0 + 64 < a.rows;  // dX ext: second 64-column half inside K
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (t >= static_cast<int>(P::kStages) && !mbar_wait(&empty[s], (u - 1) & 1, wc)) break;
        uint8_t* st = smem + s * P::kStage;
        if (t < nmain) {
          mbar_arrive_expect_tx(&full[s], P::kB + P::kC);
          tma_load_2d(st, &tm_b, &full[s], t * 32, m0);
          tma_load_2d(st + P::kBh, &tm_b, &full[s], t * 32, m0 + 256);
          if (!DX) tma_load_2d(st + P::kB + P::kA, &tm_codes, &full[s], t * 16, row0);
          else tma_load_2d(st + P::kB + P::kA, &tm_codes, &full[s], row0 / 2, t * 32);
        } else {
          if (!waited) {
            grid_dependency_wait();  // sU / dU of the preceding kernel are complete and visible
            grid_dependents_launch();
            waited = true;
          }
          const int e = t - nmain;
          if (!DX) {
            mbar_arrive_expect_tx(&full[s], P::kB + P::kA);
            tma_load_2d(st + P::kB, &tm_ext, &full[s], 16 * e, row0);  // B_lora [128 n x 32 j]
          } else {
            mbar_arrive_expect_tx(&full[s], P::kB + (a2 ? 4096u : 2048u));
            tma_load_2d(st + P::kB, &tm_ext, &full[s], row0, 16 * e);  // A_lora [16 j x 64 k]
            if (a2) tma_load_2d(st + P::kB + 4096, &tm_ext, &full[s], row0 + 64, 16 * e);
          }
          tma_load_2d(st, &tm_uc, &full[s], uc0 + 32 * e, m0);
          tma_load_2d(st + P::kBh, &tm_uc, &full[s], uc0 + 32 * e, m0 + 256);
        }
        issued = t + 1;
      }
      for (int t = max(0, issued - static_cast<int>(P::kStages)); t < issued; ++t)
        mbar_drain(&full[t % P::kStages], (t / P::kStages) & 1, a.status);
    }
    __syncwarp();  // the other lanes pass the wait only after lane 0 is through its loop
    if (!waited) {  // lanes 1..31, or a producer that gave up
      grid_dependency_wait();
      grid_dependents_launch();
    }
  } else if (warp == 1) {
    // The whole warp runs the loop (warp-uniform waits and descriptors); the
    // elected lane issues the MMAs and the commits.
    {
      const uint32_t idesc = idesc_bf16_f32(128, 256, DX ? 1 : 0, 0);
      const uint32_t a_step = DX ? (2048u >> 4) : (32u >> 4);
      bool aborted = false;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait_all(&full[s], u & 1, wc)) { aborted = true; break; }
        if (t < nmain && !mbar_wait_all(&wfull[s], u & 1, wc)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + s * P::kStage);
        const uint32_t sa = sb + P::kB;
        const uint64_t b0 = sdesc_sw64(sb, 16, 512), b1 = sdesc_sw64(sb + P::kBh, 16, 512);
        const uint64_t ad = DX ? sdesc_sw128(sa, 4096, 1024) : sdesc_sw64(sa, 16, 512);
        if (elect_one()) {
          if (t < nmain) {
#pragma unroll
            for (uint32_t kk = 0; kk < 2; ++kk) {
              const uint32_t acc = (t | kk) != 0 ? 1u : 0u;
              umma_bf16(tmem_d, ad + kk * a_step, b0 + kk * 2, idesc, acc);
              umma_bf16(tmem_d + 256, ad + kk * a_step, b1 + kk * 2, idesc, acc);
            }
          } else {
#pragma unroll
            for (uint32_t part = 0; part < 2; ++part) {  // hi, lo
              umma_bf16(tmem_d, ad, b0 + part * 2, idesc, 1u);
              umma_bf16(tmem_d + 256, ad, b1 + part * 2, idesc, 1u);
            }
          }
          umma_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (elect_one()) {
        umma_commit(accf);
        if (aborted) mbar_drain(accf, 0, a.status);
      }
    }
    __syncwarp();
    grid_dependency_wait();
    grid_dependents_launch();
  } else {
    const int dt = threadIdx.x - 64;  // 0..127
    const Nf4Mean wmean = nf4_load_mean(a.mean);  // from an earlier kernel: complete (see above)
    const int64_t kbpr = a.k_in / 64;
    if (!DX) {
      // -------------------------------------------------- forward dequant
      const int rl = dt;
      const int n = row0 + rl;
      const bool valid = n < a.n_out;
      const int64_t rowb = static_cast<int64_t>(n) * kbpr;
      const uint32_t swz = (rl >> 1) & 3;
      constexpr int kPD = 4;  // blocks of prefetch (two stages each)
      uint32_t pc[kPD];
      float ps[kPD];
      auto fetch = [&](int blk, uint32_t& c, float& sv) {
        if (valid && 2 * blk < nmain) {
          c = __ldg(a.c8 + rowb + blk);
          sv = __ldg(a.s2 + ((rowb + blk) >> 8));
        } else {
          c = 0;
          sv = 0.f;
        }
      };
#pragma unroll
      for (int i = 0; i < kPD; ++i) fetch(i, pc[i], ps[i]);
      Nf4Lut lut{};
      for (int t = 0; t < nmain; ++t) {
        if ((t & 1) == 0) {
          const float chat = valid ? nf4_block_scale(pc[0], ps[0], wmean) : 0.0f;
#pragma unroll
          for (int i = 0; i + 1 < kPD; ++i) {
            pc[i] = pc[i + 1];
            ps[i] = ps[i + 1];
          }
          fetch(t / 2 + kPD, pc[kPD - 1], ps[kPD - 1]);
          lut = nf4_make_lut(a.tab, chat);
        }
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait_all(&full[s], u & 1, wc)) break;
        uint8_t* st = smem + s * P::kStage;
        uint8_t* dst = st + P::kB + rl * 64;
        if (valid) {
          const uint4 c = *reinterpret_cast<const uint4*>(st + P::kB + P::kA + rl * 16);
          const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
          for (uint32_t j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(dst + ((j ^ swz) << 4)) = nf4_lookup8(cw[j], lut);
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(dst + j * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();  // this lane's tile writes -> async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&wfull[s]);
      }
    } else {
      // -------------------------------------------------- dX dequant
      const uint32_t half = dt & 1;
      const int p = dt >> 1;          // block of the stage: 32 rows x 2 column blocks
      const int nl = p & 31, bs = p >> 5;
      const int kb = row0 / 64 + bs;
      const bool kok = kb < kbpr;
      constexpr int kPD = 6;
      uint32_t pc[kPD];
      float ps[kPD];
      auto fetch = [&](int t, uint32_t& c, float& sv) {
        const int n = t * 32 + nl;
        if (t < nmain && kok && n < a.n_out) {
          const int64_t b = static_cast<int64_t>(n) * kbpr + kb;
          c = __ldg(a.c8 + b);
          sv = __ldg(a.s2 + (b >> 8));
        } else {
          c = 0;
          sv = 0.f;
        }
      };
#pragma unroll
      for (int i = 0; i < kPD; ++i) fetch(i, pc[i], ps[i]);
      for (int t = 0; t < nmain; ++t) {
        const uint32_t c8b = pc[0];
        const float s2v = ps[0];
#pragma unroll
        for (int i = 0; i + 1 < kPD; ++i) {
          pc[i] = pc[i + 1];
          ps[i] = ps[i + 1];
        }
        fetch(t + kPD, pc[kPD - 1], ps[kPD - 1]);
        const bool valid = kok && (t * 32 + nl) < a.n_out;
        const float chat = valid ? nf4_block_scale(c8b, s2v, wmean) : 0.0f;
        const Nf4Lut lut = nf4_make_lut_pair(a.tab, chat, half);  // all lanes
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait_all(&full[s], u & 1, wc)) break;
        uint8_t* st = smem + s * P::kStage;
        uint8_t* dst = st + P::kB + bs * 4096 + (nl >> 3) * 1024 + (nl & 7) * 128;
        if (valid) {
          nf4_half_block_to_swizzled_row(st + P::kB + P::kA + nl * 64 + bs * 32 + 16 * half, lut, dst, nl & 7,
                                         half);
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(dst + (4 * half + j) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();  // this lane's tile writes -> async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&wfull[s]);
      }
    }

    grid_dependency_wait();
    grid_dependents_launch();

    // ------------------------------------------------------------ epilogue
    if (mbar_wait_warp(accf, 0, wc)) {
      tc_fence_after();
      const int q = warp & 3;
      const int orow = row0 + q * 32 + lane;
      const bool rok = orow < a.rows;
      const uint32_t tq = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int cb = 0; cb < 16; ++cb) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tq + cb * 32, v);
        tmem_ld_wait();
        const int mb = m0 + cb * 32;
        const int nv = min(32, a.M - mb);
        if (rok && nv > 0) {
          const int64_t ld = a.ld_out;
          if (a.out_f32) {
            float* o = reinterpret_cast<float*>(a.out) + orow + static_cast<int64_t>(mb) * ld;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nv) *o = __uint_as_float(v[j]);
              o += ld;
            }
          } else {
            uint16_t* o = reinterpret_cast<uint16_t*>(a.out) + orow + static_cast<int64_t>(mb) * ld;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nv) *o = bf16_bits(__uint_as_float(v[j]));
              o += ld;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, 512);
  }
}

template <bool DX>
static cudaError_t launch_fused2x_impl(const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& m2,
                                       const CUtensorMap& m3, const FusedArgs& a, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(fused2x_kernel<DX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Plan2x::kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((a.rows + 127) / 128, (a.M + 511) / 512, 1);
  return launch_kernel(fused2x_kernel<DX>, grid, dim3(192), Plan2x::kSmem, stream, dim3(1, 1, 1), m0, m1, m2, m3, a);
}

cudaError_t launch_fused2x(bool dx, const CUtensorMap& tm_b, const CUtensorMap& tm_codes, const CUtensorMap& tm_uc,
                           const CUtensorMap& tm_ext, const FusedArgs& a, cudaStream_t stream) {
  return dx ? launch_fused2x_impl<true>(tm_b, tm_codes, tm_uc, tm_ext, a, stream)
            : launch_fused2x_impl<false>(tm_b, tm_codes, tm_uc, tm_ext, a, stream);
}

template <int BN, bool DX, int DQW>
static cudaError_t launch_fused_impl(const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& m2,
                                     const CUtensorMap& m3, const FusedArgs& a, int splits, cudaStream_t stream) {
  using P = FusedPlan<BN>;
  static bool attr_set = false;  // benign race: setting the same value twice is harmless
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(fused_kernel<BN, DX, DQW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(P::kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (splits < 1 || splits > 8) return cudaErrorInvalidValue;
  dim3 grid((a.rows + 127) / 128, (a.M + BN - 1) / BN, splits);
  // A split contraction runs as a cluster of its slices (reduced in-cluster).
  return launch_kernel(fused_kernel<BN, DX, DQW>, grid, dim3(64 + 32 * DQW), P::kSmem, stream,
                       dim3(1, 1, static_cast<unsigned>(splits)), m0, m1, m2, m3, a);
}

// Dequantiser warps per CTA: eight (two groups of four taking alternate
// stages) measured 3-6% faster than four at 64 to 256 tokens on 22016 x 8192
// and 8192 x 22016 weights (200 tokens: 196 against 208 us); each stage's
// dequantisation is a chain of dependent byte permutes, and two groups give
// each SM sub-partition two of them to interleave (three groups of four, with
// one CTA per SM, measured within 2% of two).  QLORA_DEQUANT_WARPS=4 selects
// four.
static int dequant_warps(int bn) {
  static int forced = [] {
    const char* e = getenv("QLORA_DEQUANT_WARPS");
    return e ? atoi(e) : 0;
  }();
  (void)bn;
  return forced == 4 ? 4 : 8;
}

template <int BN, bool DX>
static cudaError_t launch_fused_dqw(const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& m2,
                                    const CUtensorMap& m3, const FusedArgs& a, int splits, cudaStream_t stream) {
  return dequant_warps(BN) == 4 ? launch_fused_impl<BN, DX, 4>(m0, m1, m2, m3, a, splits, stream)
                                : launch_fused_impl<BN, DX, 8>(m0, m1, m2, m3, a, splits, stream);
}

cudaError_t launch_fused_fwd(int bn, const CUtensorMap& tm_x, const CUtensorMap& tm_codes,
                             const CUtensorMap& tm_uc, const CUtensorMap& tm_bl, const FusedArgs& a,
                             int splits, cudaStream_t stream) {
  switch (bn) {
    case 32: return launch_fused_dqw<32, false>(tm_x, tm_codes, tm_uc, tm_bl, a, splits, stream);
    case 64: return launch_fused_dqw<64, false>(tm_x, tm_codes, tm_uc, tm_bl, a, splits, stream);
    case 128: return launch_fused_dqw<128, false>(tm_x, tm_codes, tm_uc, tm_bl, a, splits, stream);
    case 256: return launch_fused_dqw<256, false>(tm_x, tm_codes, tm_uc, tm_bl, a, splits, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fused_dx(int bn, const CUtensorMap& tm_dy, const CUtensorMap& tm_codes,
                            const CUtensorMap& tm_duc, const CUtensorMap& tm_al, const FusedArgs& a, int splits,
                            cudaStream_t stream) {
  switch (bn) {
    case 128: return launch_fused_dqw<128, true>(tm_dy, tm_codes, tm_duc, tm_al, a, splits, stream);
    case 256: return launch_fused_dqw<256, true>(tm_dy, tm_codes, tm_duc, tm_al, a, splits, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qnf4
