// fused_pair.cu — large-M dequantise-in-GEMM on CTA pairs (tcgen05 cta_group::2),
// the forward Y = X W'^T + (sU) B^T and the input gradient dX = dY W' + dU A of
// the QLoRA linear ("QLoRA" encyclopedia entry, tonho.wtf, section "a ideia":
// the 4-bit weight is dequantised to BFloat16 at the moment of use).
//
// A cluster of two CTAs computes 256 W-side rows x 512 tokens.  Each CTA
// dequantises its own 128 W rows; one thread of the leader CTA issues
// M = 256, N = 256 MMAs whose A rows come from both CTAs' shared memory and
// whose B (token) rows are split between them, into two TMEM accumulators
// per CTA (tokens 0-255 and 256-511 of the tile).  Every CTA therefore holds
// only 256 token rows per stage: a stage is 26 KB and eight stages fit, twice
// the pipeline depth (in MMA time) of a single-CTA tile of the same shape.
//
// Barriers (all bounded waits):
//   cfull[s]  this CTA's packed codes landed (local TMA)
//   full[s]   leader only: both CTAs' token / LoRA tiles landed (paired TMA)
//             and both CTAs' dequantised W tiles are written (one arrival per
//             dequantiser warp of the stage's group, after each lane fenced
//             its writes): one barrier, so the MMA warp checks one per stage
//   empty[s]  both CTAs: the pair's MMAs of the stage finished (multicast commit)
//   accf      both CTAs: the accumulators are final (multicast commit)
// No TMA multicast is used.
#include "kernels.h"

namespace qnf4 {

namespace {

struct PlanPair {
  static constexpr uint32_t kBq = 128 * 64;  // 128 tokens x 32 bf16, one accumulator's half
  static constexpr uint32_t kB = 2 * kBq;    // 16 KB
  static constexpr uint32_t kA = 8192;       // 128 W-side rows x 32
  static constexpr uint32_t kC = 2048;       // packed codes of the stage
  static constexpr uint32_t kStage = kB + kA + kC;
  static constexpr uint32_t kStages = 8;
  static constexpr uint32_t kBarOff = kStages * kStage;
  static constexpr uint32_t kSmem = 1024 + kBarOff + 512;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kSmem <= 232448u, "too much shared memory");
  // two dequantiser groups take alternate stages: with an even ring a slot's
  // previous stage is the same group's, so the parity waits cannot alias
  static_assert(kStages % 2 == 0, "two alternating dequantiser groups need an even ring");
};

}  // namespace

// Warp 0: copies; warp 1: MMAs (leader CTA); warps 2..9: two groups of four
// dequantiser warps taking alternate stages (two independent instruction
// streams per SM sub-partition: one warp per stage is latency-bound), which
// also split the epilogue's columns between them.
constexpr int kPairThreads = 320;

template <bool DX>
__global__ void __launch_bounds__(kPairThreads, 1)
    fused_pair_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_codes,
                      const __grid_constant__ CUtensorMap tm_uc, const __grid_constant__ CUtensorMap tm_ext,
                      const FusedArgs a) {
  using P = PlanPair;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::kBarOff);
  uint64_t* cfull = full + P::kStages;
  uint64_t* empty = cfull + P::kStages;
  uint64_t* accf = empty + P::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();            // 0 = leader
  const int row0 = (blockIdx.x >> 1) * 256 + static_cast<int>(rank) * 128;  // this CTA's W-side rows
  const int m0 = blockIdx.y * 512;                    // the pair's tokens
  const int mt = m0 + static_cast<int>(rank) * 128;   // this CTA's token rows (+256 for the second half)
  const int nmain = a.kt_total;                       // stages of 32
  const int next = a.r / 16;
  const int T = nmain + next;

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < P::kStages; ++s) {
      mbar_init(&full[s], 1 + 8);  // the producer's expect-tx arrival + 4 dequantiser warps per CTA
      mbar_init(&cfull[s], 1);
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
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // barrier inits and the TMEM allocation are visible to the pair
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  const WaitCtx wc{abort_flag, a.status};
  // Programmatic dependent launch: the only input produced by the kernel
  // launched just before this one is the bf16 hi/lo of sU / dU, read by the
  // extension stages at the end of the contraction; X or dY, the codes and
  // the block constants come from earlier kernels, which had completed when
  // that kernel let this one launch (every kernel here waits before it
  // triggers).  So the producer waits for the preceding grid just before the
  // first extension load, and every other role passes the wait (a no-op by
  // then) after its main loop, before triggering the next kernel.

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    bool waited = false;
    // Grouped forward: this tile's member reads its own columns of the hi/lo copy of s*U.
    const int uc0 = DX ? 0 : group_member(a.grp_end, a.groups, row0) * 2 * a.r;
    if (lane == 0) {
      int issued = 0;
      // Extension bytes of one CTA: token/U halves plus the LoRA tile.
      const uint32_t ext_a = DX ? 4096u : 8192u;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (t >= static_cast<int>(P::kStages) && !mbar_wait(&empty[s], (u - 1) & 1, wc)) break;
        uint8_t* st = smem + s * P::kStage;
        const uint32_t full0 = dsmem_addr(&full[s], 0);
        if (t < nmain) {
          mbar_arrive_expect_tx(&cfull[s], P::kC);
          if (!DX) tma_load_2d(st + P::kB + P::kA, &tm_codes, &cfull[s], t * 16, row0);
          else tma_load_2d(st + P::kB + P::kA, &tm_codes, &cfull[s], row0 / 2, t * 32);
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * P::kB);
          tma_load_2d_pair(st, &tm_b, full0, t * 32, mt);
          tma_load_2d_pair(st + P::kBq, &tm_b, full0, t * 32, mt + 256);
        } else {
          if (t == nmain) {
            grid_dependency_wait();  // sU / dU of the preceding kernel are complete and visible
            grid_dependents_launch();
            waited = true;
          }
          const int e = t - nmain;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (P::kB + ext_a));
          tma_load_2d_pair(st, &tm_uc, full0, uc0 + 32 * e, mt);
          tma_load_2d_pair(st + P::kBq, &tm_uc, full0, uc0 + 32 * e, mt + 256);
          if (!DX) {
            tma_load_2d_pair(st + P::kB, &tm_ext, full0, 16 * e, row0);  // B_lora [128 n x 32 j]
          } else {
            tma_load_2d_pair(st + P::kB, &tm_ext, full0, row0, 16 * e);  // A_lora [16 j x 64 k] x 2
            tma_load_2d_pair(st + P::kB + 4096, &tm_ext, full0, row0 + 64, 16 * e);
          }
        }
        issued = t + 1;
      }
      // Leave nothing in flight into this CTA's shared memory: codes land on the
      // local barrier; the leader also waits for the pair's tiles.
      // The full barriers also count the dequantisers' arrivals, which may
      // never come after an abort, so the drain then takes a short limit (the
      // copies themselves land in microseconds).
      const uint64_t lim = *abort_flag ? 1000000ull : kWaitTimeoutNs;
      for (int t = max(0, issued - static_cast<int>(P::kStages)); t < issued; ++t) {
        if (t < nmain) mbar_drain(&cfull[t % P::kStages], (t / P::kStages) & 1, a.status, lim);
        if (rank == 0) mbar_drain(&full[t % P::kStages], (t / P::kStages) & 1, a.status, lim);
      }
    }
    __syncwarp();  // the other lanes pass the wait only after lane 0 is through its loop
    if (!waited) {  // lanes 1..31, or a producer that gave up early
      grid_dependency_wait();
      grid_dependents_launch();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA (leader)
    // The whole warp runs the loop (warp-uniform waits and descriptors); the
    // elected lane issues the MMAs and the commits.
    if (rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(256, 256, DX ? 1 : 0, 0);
      const uint32_t a_step = DX ? (2048u >> 4) : (32u >> 4);
      bool aborted = false;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait_all(&full[s], u & 1, wc)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + s * P::kStage);
        const uint32_t sa = sb + P::kB;
        const uint64_t b0 = sdesc_sw64(sb, 16, 512), b1 = sdesc_sw64(sb + P::kBq, 16, 512);
        const uint64_t ad = DX ? sdesc_sw128(sa, 4096, 1024) : sdesc_sw64(sa, 16, 512);
        if (elect_one()) {
          if (t < nmain) {
#pragma unroll
            for (uint32_t kk = 0; kk < 2; ++kk) {
              const uint32_t acc = (t | kk) != 0 ? 1u : 0u;
              umma_bf16_pair(tmem_d, ad + kk * a_step, b0 + kk * 2, idesc, acc);
              umma_bf16_pair(tmem_d + 256, ad + kk * a_step, b1 + kk * 2, idesc, acc);
            }
          } else {
#pragma unroll
            for (uint32_t part = 0; part < 2; ++part) {  // hi, lo
              umma_bf16_pair(tmem_d, ad, b0 + part * 2, idesc, 1u);
              umma_bf16_pair(tmem_d + 256, ad, b1 + part * 2, idesc, 1u);
            }
          }
          umma_commit_pair(&empty[s], 0x3);
        }
        __syncwarp();
      }
      if (elect_one()) {
        umma_commit_pair(accf, 0x3);
        if (aborted) mbar_drain(accf, 0, a.status);
      }
    }
    __syncwarp();
    grid_dependency_wait();
    grid_dependents_launch();
  } else {
    const int dt = (threadIdx.x - 64) & 127;  // 0..127 within the group
    const int grp = (threadIdx.x - 64) >> 7;  // stages t with t % 2 == grp
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
      // Stage t covers half of block t / 2: each group builds that block's
      // table itself.
      for (int t = grp; t < nmain; t += 2) {
        const float chat = valid ? nf4_block_scale(pc[0], ps[0], wmean) : 0.0f;
#pragma unroll
        for (int i = 0; i + 1 < kPD; ++i) {
          pc[i] = pc[i + 1];
          ps[i] = ps[i + 1];
        }
        fetch(t / 2 + kPD, pc[kPD - 1], ps[kPD - 1]);
        const Nf4Lut lut = nf4_make_lut(a.tab, chat);
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait_all(&cfull[s], u & 1, wc)) break;
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
        if (lane == 0) mbar_arrive_remote(dsmem_addr(&full[s], 0));
      }
    } else {
      // -------------------------------------------------- dX dequant
      const uint32_t half = dt & 1;
      const int p = dt >> 1;  // block of the stage: 32 W rows x 2 column blocks
      const int nl = p & 31, bs = p >> 5;
      const int kb = row0 / 64 + bs;
      const bool kok = kb < kbpr;
      constexpr int kPD = 4;  // stages of prefetch (this group's: every other stage)
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
      for (int i = 0; i < kPD; ++i) fetch(grp + 2 * i, pc[i], ps[i]);
      for (int t = grp; t < nmain; t += 2) {
        const uint32_t c8b = pc[0];
        const float s2v = ps[0];
#pragma unroll
        for (int i = 0; i + 1 < kPD; ++i) {
          pc[i] = pc[i + 1];
          ps[i] = ps[i + 1];
        }
        fetch(t + 2 * kPD, pc[kPD - 1], ps[kPD - 1]);
        const bool valid = kok && (t * 32 + nl) < a.n_out;
        const float chat = valid ? nf4_block_scale(c8b, s2v, wmean) : 0.0f;
        const Nf4Lut lut = nf4_make_lut_pair(a.tab, chat, half);  // all lanes
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait_all(&cfull[s], u & 1, wc)) break;
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
        if (lane == 0) mbar_arrive_remote(dsmem_addr(&full[s], 0));
      }
    }
    // Adapter stages: nothing to dequantise, but the stage's group still
    // arrives on full[s].  It first waits until the slot's previous stage
    // (t - kStages, a main stage of this group) is retired, so the arrival
    // falls in the stage's own phase.
    for (int t = nmain + ((grp - nmain) & 1); t < T; t += 2) {
      const uint32_t s = t % P::kStages;
      if (t >= static_cast<int>(P::kStages) && !mbar_wait_all(&empty[s], ((t / P::kStages) - 1) & 1, wc)) break;
      if (lane == 0) mbar_arrive_remote(dsmem_addr(&full[s], 0));
    }

    grid_dependency_wait();
    grid_dependents_launch();

    // ------------------------------------------------------------ epilogue
    if (mbar_wait_warp(accf, 0, wc)) {
      tc_fence_after();
      // Warp w reads TMEM lanes 32 (w % 4) ..; the two groups take half of
      // the 16 column blocks each.
      const int q = warp & 3;
      const int orow = row0 + q * 32 + lane;
      const bool rok = orow < a.rows;
      const uint32_t tq = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int cb = 8 * grp; cb < 8 * grp + 8; ++cb) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tq + cb * 32, v);
        tmem_ld_wait();
        const int mb = m0 + cb * 32;  // columns 0..255: tokens m0.., 256..511: m0+256..
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
  __syncwarp();
  cluster_sync_all();  // both CTAs are done with TMEM and with each other's barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_d, 512);
  }
}

template <bool DX>
static cudaError_t launch_pair_impl(const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& m2,
                                    const CUtensorMap& m3, const FusedArgs& a, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(fused_pair_kernel<DX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(PlanPair::kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_kernel(fused_pair_kernel<DX>, dim3(2 * ((a.rows + 255) / 256), (a.M + 511) / 512, 1), dim3(kPairThreads),
                       PlanPair::kSmem, stream, dim3(2, 1, 1), m0, m1, m2, m3, a);
}

cudaError_t launch_fused_pair(bool dx, const CUtensorMap& tm_b, const CUtensorMap& tm_codes,
                              const CUtensorMap& tm_uc, const CUtensorMap& tm_ext, const FusedArgs& a,
                              cudaStream_t stream) {
  return dx ? launch_pair_impl<true>(tm_b, tm_codes, tm_uc, tm_ext, a, stream)
            : launch_pair_impl<false>(tm_b, tm_codes, tm_uc, tm_ext, a, stream);
}

}  // namespace qnf4
