// fused_pair_fwd.cu — large-M forward Y = X W'^T + (sU) B^T of the QLoRA linear
// on CTA pairs (tcgen05 cta_group::2) with the dequantised weight tile kept in
// tensor memory ("QLoRA" encyclopedia entry, tonho.wtf, section "a ideia": the
// 4-bit weight is dequantised to BFloat16 at the moment of use).
//
// The same pair tiling as fused_pair.cu (256 W rows per pair, each CTA
// dequantising its 128 rows), but the dequantiser warps store their rows of
// the bf16 tile straight into tensor memory (tcgen05.st) and the MMA takes its
// A operand from there.  The weight tile then never passes through shared
// memory: shared memory carries only the token tiles (TMA in, MMA out) and
// the packed codes, so a stage is 16 KB instead of 26 and the ring holds 12
// stages instead of 8 (the adapter stages' rows of B have buffers of their
// own).  The main loop is bound by the latency of the copies the ring must
// hide, so its depth in time is what counts.  Tensor memory holds two
// 128 x 224 fp32 accumulators (448 tokens per pair) and a ring of four
// 16-column A slots (one 32-deep stage each).
//
// Barriers (all bounded waits):
//   cfull[s]  this CTA's packed codes landed (local TMA)
//   full[s]   leader only: both CTAs' token / LoRA tiles landed (paired TMA)
//             and both CTAs' A rows are stored in tensor memory (one arrival
//             per dequantiser warp of the stage's group, after
//             tcgen05.wait::st and the tcgen05 fence before the thread
//             synchronisation): one barrier per stage for the MMA warp
//   empty[s]  both CTAs: the pair's MMAs of the stage finished (multicast
//             commit); the dequantisers also wait on it before reusing an A slot
//   accf      both CTAs: the accumulators are final (multicast commit)
// Warp 0 copies, warp 1 issues the MMAs (the whole warp runs the loop, an
// elected lane issues), warps 2..9 are two groups of four dequantiser warps
// taking alternate stages.
// The adapter stages (r/16 of them) take their A operand (the rows of B) from
// shared memory as in fused_pair.cu.  No TMA multicast is used.
#include "kernels.h"

namespace qnf4 {

namespace {

template <int ASLOTS>
struct PlanPairT {
  static constexpr int kN = (512 - 16 * ASLOTS) / 2;  // tokens per accumulator (MMA N)
  static constexpr uint32_t kBq = (kN / 2) * 64; // one accumulator's token rows in one CTA: kN/2 x 32 bf16
  static constexpr uint32_t kB = 2 * kBq;
  static constexpr uint32_t kC = 2048;           // packed codes of a main stage (128 rows x 16 B)
  static constexpr uint32_t kStage = (kB + kC + 1023) / 1024 * 1024;
  static constexpr uint32_t kExt = 8192;         // rows of B in an adapter stage (128 x 32 bf16)
  static constexpr uint32_t kExtBufs = 4;        // one per adapter stage: r / 16 <= 4
  static constexpr int kASlots = ASLOTS;
  static constexpr uint32_t kACol = 2 * kN;      // first tensor-memory column of the A ring
  // As many stages as shared memory holds beside the adapter buffers (the
  // ring's depth in time is what hides the copies' latency), rounded down to
  // an even count for the two alternating dequantiser groups.
  static constexpr uint32_t kStages = ((232448u - 1024u - 512u - kExtBufs * kExt) / kStage) & ~1u;
  static constexpr uint32_t kExtOff = kStages * kStage;
  static constexpr uint32_t kBarOff = kExtOff + kExtBufs * kExt;
  static constexpr uint32_t kSmem = 1024 + kBarOff + 512;
  static_assert(kStage % 1024 == 0 && kStage >= kB + kC, "stage layout");
  static_assert(kBq % 512 == 0, "64-byte swizzle atoms");
  static_assert(kACol + 16 * kASlots <= 512, "tensor memory");
  static_assert(kStages >= 8 && kStages <= 16, "ring depth");
  // two dequantiser groups take alternate stages: with an even ring a slot's
  // previous stage is the same group's, so the parity waits cannot alias
  static_assert(kStages % 2 == 0, "two alternating dequantiser groups need an even ring");
  static_assert(kSmem <= 232448u, "too much shared memory");
};

// D[tmem] (+)= A[tmem] * B[smem]^T on the CTA pair, bf16 in, fp32 accumulate.
__device__ __forceinline__ void umma_bf16_pair_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                  uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// This warp's 32 lanes x 16 consecutive 32-bit columns from registers.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

}  // namespace

// The dequantisers publish their rows with a plain remote arrival (release at
// CTA scope, as for any cross-CTA pair barrier); a cluster-scope release costs
// a memory barrier per warp and stage and measured 2.3-2.7x slower.
template <int ASLOTS>
__global__ void __launch_bounds__(320, 1)
    fused_pair_fwd_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_codes,
                          const __grid_constant__ CUtensorMap tm_uc, const __grid_constant__ CUtensorMap tm_ext,
                          const FusedArgs a) {
  using P = PlanPairT<ASLOTS>;
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
  const int row0 = (blockIdx.x >> 1) * 256 + static_cast<int>(rank) * 128;  // this CTA's W rows
  const int m0 = blockIdx.y * (2 * P::kN);            // the pair's tokens
  const int mt = m0 + static_cast<int>(rank) * (P::kN / 2);  // this CTA's token rows (+kN for the second half)
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
  // Programmatic dependent launch, as in fused_pair.cu: only the hi/lo of sU
  // (the adapter stages) comes from the kernel launched just before; the
  // producer waits for it right before the first adapter load, the other
  // roles after their main loop.

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    bool waited = false;
    if (lane == 0) {
      int issued = 0;
      const int uc0 = group_member(a.grp_end, a.groups, row0) * 2 * a.r;  // this tile's member's sU columns
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (t >= static_cast<int>(P::kStages) && !mbar_wait(&empty[s], (u - 1) & 1, wc)) break;
        uint8_t* st = smem + s * P::kStage;
        const uint32_t full0 = dsmem_addr(&full[s], 0);
        if (t < nmain) {
          mbar_arrive_expect_tx(&cfull[s], P::kC);
          tma_load_2d(st + P::kB, &tm_codes, &cfull[s], t * 16, row0);
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * P::kB);
          tma_load_2d_pair(st, &tm_b, full0, t * 32, mt);
          tma_load_2d_pair(st + P::kBq, &tm_b, full0, t * 32, mt + P::kN);
        } else {
          if (t == nmain) {
            grid_dependency_wait();  // sU of the preceding kernel is complete and visible
            grid_dependents_launch();
            waited = true;
          }
          const int e = t - nmain;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (P::kB + P::kExt));
          tma_load_2d_pair(st, &tm_uc, full0, uc0 + 32 * e, mt);
          tma_load_2d_pair(st + P::kBq, &tm_uc, full0, uc0 + 32 * e, mt + P::kN);
          tma_load_2d_pair(smem + P::kExtOff + e * P::kExt, &tm_ext, full0, 16 * e, row0);  // B_lora [128 n x 32 j]
        }
        issued = t + 1;
      }
      // Leave nothing in flight into this CTA's shared memory.
      // The full barriers also count the dequantisers' arrivals, which may
      // never come after an abort, so the drain then takes a short limit.
      const uint64_t lim = *abort_flag ? 1000000ull : kWaitTimeoutNs;
      for (int t = max(0, issued - static_cast<int>(P::kStages)); t < issued; ++t) {
        if (t < nmain) mbar_drain(&cfull[t % P::kStages], (t / P::kStages) & 1, a.status, lim);
        if (rank == 0) mbar_drain(&full[t % P::kStages], (t / P::kStages) & 1, a.status, lim);
      }
    }
    __syncwarp();
    if (!waited) {
      grid_dependency_wait();
      grid_dependents_launch();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA (leader)
    // The whole warp runs the loop (warp-uniform waits and descriptors); the
    // elected lane issues the MMAs and the commits.
    if (rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(256, P::kN, 0, 0);
      bool aborted = false;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait_all(&full[s], u & 1, wc)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + s * P::kStage);
        const uint64_t b0 = sdesc_sw64(sb, 16, 512), b1 = sdesc_sw64(sb + P::kBq, 16, 512);
        const uint32_t at = tmem_d + P::kACol + static_cast<uint32_t>(t % P::kASlots) * 16;
        const uint64_t ad = sdesc_sw64(smem_u32(smem + P::kExtOff + (t >= nmain ? t - nmain : 0) * P::kExt), 16, 512);
        if (elect_one()) {
          if (t < nmain) {
#pragma unroll
            for (uint32_t kk = 0; kk < 2; ++kk) {
              const uint32_t acc = (t | kk) != 0 ? 1u : 0u;
              umma_bf16_pair_ta(tmem_d, at + kk * 8, b0 + kk * 2, idesc, acc);
              umma_bf16_pair_ta(tmem_d + P::kN, at + kk * 8, b1 + kk * 2, idesc, acc);
            }
          } else {
#pragma unroll
            for (uint32_t part = 0; part < 2; ++part) {  // hi, lo
              umma_bf16_pair(tmem_d, ad, b0 + part * 2, idesc, 1u);
              umma_bf16_pair(tmem_d + P::kN, ad, b1 + part * 2, idesc, 1u);
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
    // ------------------------------------------------------------ dequantisers
    // Warp w may access tensor-memory lanes 32 (w % 4) .. + 31 only, so the
    // thread dequantises W row rl = its lane there (A row i = TMEM lane i).
    // Eight warps in two groups taking alternate stages; group g's four warps
    // cover the four lane quarters.
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    const int grp = (threadIdx.x - 64) >> 7;
    const Nf4Mean wmean = nf4_load_mean(a.mean);  // from an earlier kernel: complete (see above)
    const int64_t kbpr = a.k_in / 64;
    const int n = row0 + rl;
    const bool valid = n < a.n_out;
    const int64_t rowb = static_cast<int64_t>(n) * kbpr;
    const uint32_t tq = tmem_d + (static_cast<uint32_t>(q * 32) << 16) + P::kACol;
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
      // The A slot of stage t was last read by the MMAs of stage t - kASlots
      // (with as many slots as stages, the codes of stage t landing already
      // imply it: they were loaded after that stage's MMAs finished).
      if (P::kASlots < static_cast<int>(P::kStages) && t >= P::kASlots) {
        const int tp = t - P::kASlots;
        if (!mbar_wait_all(&empty[tp % P::kStages], (tp / P::kStages) & 1, wc)) break;
      }
      uint32_t w[16];
      if (valid) {
        const uint4 c = *reinterpret_cast<const uint4*>(smem + s * P::kStage + P::kB + rl * 16);
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 o = nf4_lookup8(cw[j], lut);
          w[4 * j] = o.x;
          w[4 * j + 1] = o.y;
          w[4 * j + 2] = o.z;
          w[4 * j + 3] = o.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) w[j] = 0u;
      }
      tmem_st_32x32b_x16(tq + static_cast<uint32_t>(t % P::kASlots) * 16, w);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(dsmem_addr(&full[s], 0));
    }
    // Adapter stages: nothing to dequantise, but the stage's group still
    // arrives on full[s], once the slot's previous stage (t - kStages, a main
    // stage of this group) is retired, so the arrival falls in its own phase.
    for (int t = nmain + ((grp - nmain) & 1); t < T; t += 2) {
      const uint32_t s = t % P::kStages;
      if (t >= static_cast<int>(P::kStages) && !mbar_wait_all(&empty[s], ((t / P::kStages) - 1) & 1, wc)) break;
      if (lane == 0) mbar_arrive_remote(dsmem_addr(&full[s], 0));
    }

    grid_dependency_wait();
    grid_dependents_launch();

    // ------------------------------------------------------------ epilogue
    // Accumulator column c holds token m0 + c (columns 0..kN-1: the first
    // accumulator, kN..2kN-1: the second).
    if (mbar_wait_warp(accf, 0, wc)) {
      tc_fence_after();
      const int orow = row0 + rl;
      const bool rok = orow < a.rows;
      const uint32_t tqd = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      // the two groups take half of the column blocks each
      constexpr int kCb = (2 * P::kN) / 32;
      for (int cb = grp * ((kCb + 1) / 2); cb < min(kCb, (grp + 1) * ((kCb + 1) / 2)); ++cb) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tqd + cb * 32, v);
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
  __syncwarp();
  cluster_sync_all();  // both CTAs are done with TMEM and with each other's barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_d, 512);
  }
}

template <int ASLOTS>
static cudaError_t launch_pair_fwd_impl(const CUtensorMap& tm_b, const CUtensorMap& tm_codes,
                                        const CUtensorMap& tm_uc, const CUtensorMap& tm_ext, const FusedArgs& a,
                                        cudaStream_t stream) {
  using P = PlanPairT<ASLOTS>;
  if (a.r / 16 > static_cast<int>(P::kExtBufs)) return cudaErrorInvalidValue;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(fused_pair_fwd_kernel<ASLOTS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(P::kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int tok = 2 * P::kN;
  return launch_kernel(fused_pair_fwd_kernel<ASLOTS>, dim3(2 * ((a.rows + 255) / 256), (a.M + tok - 1) / tok, 1),
                       dim3(320), P::kSmem, stream, dim3(2, 1, 1), tm_b, tm_codes, tm_uc, tm_ext, a);
}

int pair_fwd_tokens(int slots) { return 512 - 16 * slots; }

cudaError_t launch_fused_pair_fwd(const CUtensorMap& tm_b, const CUtensorMap& tm_codes, const CUtensorMap& tm_uc,
                                  const CUtensorMap& tm_ext, const FusedArgs& a, int slots,
                                  cudaStream_t stream) {
  return slots == 8 ? launch_pair_fwd_impl<8>(tm_b, tm_codes, tm_uc, tm_ext, a, stream)
                    : launch_pair_fwd_impl<4>(tm_b, tm_codes, tm_uc, tm_ext, a, stream);
}

}  // namespace qnf4
