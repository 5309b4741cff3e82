// fused.cu — dequantise-in-GEMM kernels of the QLoRA linear ("QLoRA"
// encyclopedia entry, tonho.wtf, section "a ideia": the 4-bit weight is
// dequantised to BFloat16 at the moment of use and discarded; the gradient
// crosses the frozen weight).
//
//   forward:  Y^T tile [128 n x BN m]  = W'[n, k] . X[m, k]^T      (+ B . (sU)^T)
//   dX:       dX^T tile [128 k x BN m] = W'[n, k]^T . dY[m, n]^T   (+ A^T . dU^T)
//
// The W side is the MMA's M = 128 dimension, tokens are its N = BN dimension,
// so one dequantised element feeds BN tokens.  Warp roles (192 threads):
//   warp 0      TMA producer (token tile + packed codes; LoRA operands)
//   warp 1      TMEM owner and single-thread tcgen05.mma issuer
//   warps 2..5  dequantisers: one thread per 64-element NF4 block per stage,
//               16 lookups of bf16 pairs written straight into the 128-byte
//               swizzled operand layout; afterwards the epilogue (TMEM -> global)
// The LoRA up-projection is appended to the contraction as extra K steps over
// the interleaved hi/lo bf16 split of the fp32 down-projection, accumulated in
// the same TMEM accumulator (no second pass over Y).  No TMA multicast.
#include "kernels.h"

namespace qnf4 {

__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitTimeoutNs) return;
  }
}

template <int BN>
struct FusedPlan {
  static constexpr uint32_t kB = BN * 128;  // token tile, 64 bf16 per row
  static constexpr uint32_t kA = 16384;     // W-side tile 128 x 64 bf16
  static constexpr uint32_t kC = 4096;      // packed codes of the stage
  static constexpr uint32_t kStage = kB + kA + kC;
  static constexpr uint32_t kFit = (232448u - 2048u) / kStage;
  static constexpr uint32_t kStages = kFit > 8 ? 8 : kFit;
  static constexpr uint32_t kBarOff = kStages * kStage;
  static constexpr uint32_t kSmem = 1024 + kBarOff + 256;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kStages >= 3, "pipeline too shallow");
};

template <int BN, bool DX>
__global__ void __launch_bounds__(192, 1)
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
      mbar_init(&wfull[s], 128);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (t >= static_cast<int>(P::kStages) && !mbar_wait(&empty[s], (u - 1) & 1, wc)) break;
        uint8_t* st = smem + s * P::kStage;
        if (t < nmain) {
          const int kt = kt0 + t;
          mbar_arrive_expect_tx(&full[s], P::kB + P::kC);
          tma_load_2d(st, &tm_b, &full[s], kt * 64, m0);
          if (!DX) tma_load_2d(st + P::kB + P::kA, &tm_codes, &full[s], kt * 32, row0);
          else tma_load_2d(st + P::kB + P::kA, &tm_codes, &full[s], row0 / 2, kt * 64);
        } else {
          const int e = t - nmain;
          if (!DX) {
            mbar_arrive_expect_tx(&full[s], P::kB + 16384);
            tma_load_2d(st, &tm_uc, &full[s], 64 * e, m0);
            tma_load_2d(st + P::kB, &tm_ext, &full[s], 32 * e, row0);
          } else {
            const bool second = row0 + 64 < a.rows;
            mbar_arrive_expect_tx(&full[s], P::kB + (second ? 16384 : 8192));
            tma_load_2d(st, &tm_uc, &full[s], 64 * e, m0);
            tma_load_2d(st + P::kB, &tm_ext, &full[s], row0, 32 * e);
            if (second) tma_load_2d(st + P::kB + 8192, &tm_ext, &full[s], row0 + 64, 32 * e);
          }
        }
        issued = t + 1;
      }
      // Do not leave the CTA while a copy into its shared memory is in flight.
      for (int t = max(0, issued - static_cast<int>(P::kStages)); t < issued; ++t)
        mbar_wait_drain(&full[t % P::kStages], (t / P::kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, BN, DX ? 1 : 0, 0);
      const uint32_t a_step = DX ? (2048u >> 4) : (32u >> 4);  // one K=16 step, descriptor units
      bool aborted = false;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait(&full[s], u & 1, wc)) { aborted = true; break; }
        if (t < nmain && !mbar_wait(&wfull[s], u & 1, wc)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + s * P::kStage);
        const uint32_t sa = sb + P::kB;
        const uint64_t bdesc = sdesc_sw128(sb, 16, 1024);
        const uint64_t adesc = DX ? sdesc_sw128(sa, 8192, 1024) : sdesc_sw128(sa, 16, 1024);
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
      umma_commit(accf);
      if (aborted) mbar_wait_drain(accf, 0);
    }
  } else {
    // ------------------------------------------------------------ dequantisers
    const int q = warp & 3;
    const int rl = q * 32 + lane;
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
    // three-deep register prefetch of the block constants
    uint32_t pc0 = 0, pc1 = 0, pc2 = 0;
    float ps0 = 0.f, ps1 = 0.f, ps2 = 0.f;
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
    fetch(0, pc0, ps0);
    fetch(1, pc1, ps1);
    fetch(2, pc2, ps2);
    for (int t = 0; t < nmain; ++t) {
      const uint32_t c8b = pc0;
      const float s2v = ps0;
      pc0 = pc1; ps0 = ps1;
      pc1 = pc2; ps1 = ps2;
      fetch(t + 3, pc2, ps2);
      int64_t bdummy;
      const bool valid = block_of(t, bdummy);
      const uint32_t s = t % P::kStages, u = t / P::kStages;
      if (!mbar_wait(&full[s], u & 1, wc)) break;
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
      if (valid) {
        const Nf4Lut lut = nf4_make_lut(a.tab, nf4_block_scale(c8b, s2v));
        nf4_block_to_swizzled_row(src, lut, dst, swz);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(dst + j * 16) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      mbar_arrive(&wfull[s]);
    }

    // ------------------------------------------------------------ epilogue
    if (mbar_wait(accf, 0, wc)) {
      tc_fence_after();
      const int orow = row0 + rl;
      const bool rok = orow < a.rows;
      const uint32_t tq = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tq + cb * 32, v);
        tmem_ld_wait();
        if (rok) {
          const int mb = m0 + cb * 32;
          const int nv = min(32, a.M - mb);
          if (a.split_stride || a.out_f32) {
            float* o = reinterpret_cast<float*>(a.out) + static_cast<int64_t>(z) * a.split_stride + orow +
                       static_cast<int64_t>(mb) * a.ld_out;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nv) o[static_cast<int64_t>(j) * a.ld_out] = __uint_as_float(v[j]);
          } else {
            uint16_t* o = reinterpret_cast<uint16_t*>(a.out) + orow + static_cast<int64_t>(mb) * a.ld_out;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nv) o[static_cast<int64_t>(j) * a.ld_out] = bf16_bits(__uint_as_float(v[j]));
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

template <int BN, bool DX>
static cudaError_t launch_fused_impl(const CUtensorMap& m0, const CUtensorMap& m1, const CUtensorMap& m2,
                                     const CUtensorMap& m3, const FusedArgs& a, int splits, cudaStream_t stream) {
  using P = FusedPlan<BN>;
  static bool attr_set = false;  // benign race: setting the same value twice is harmless
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(fused_kernel<BN, DX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(P::kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid((a.rows + 127) / 128, (a.M + BN - 1) / BN, splits);
  fused_kernel<BN, DX><<<grid, 192, P::kSmem, stream>>>(m0, m1, m2, m3, a);
  return cudaGetLastError();
}

cudaError_t launch_fused_fwd(int bn, const CUtensorMap& tm_x, const CUtensorMap& tm_codes,
                             const CUtensorMap& tm_uc, const CUtensorMap& tm_bl, const FusedArgs& a,
                             int splits, cudaStream_t stream) {
  switch (bn) {
    case 32: return launch_fused_impl<32, false>(tm_x, tm_codes, tm_uc, tm_bl, a, splits, stream);
    case 64: return launch_fused_impl<64, false>(tm_x, tm_codes, tm_uc, tm_bl, a, splits, stream);
    case 128: return launch_fused_impl<128, false>(tm_x, tm_codes, tm_uc, tm_bl, a, splits, stream);
    case 256: return launch_fused_impl<256, false>(tm_x, tm_codes, tm_uc, tm_bl, a, splits, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fused_dx(int bn, const CUtensorMap& tm_dy, const CUtensorMap& tm_codes,
                            const CUtensorMap& tm_duc, const CUtensorMap& tm_al, const FusedArgs& a,
                            cudaStream_t stream) {
  switch (bn) {
    case 128: return launch_fused_impl<128, true>(tm_dy, tm_codes, tm_duc, tm_al, a, 1, stream);
    case 256: return launch_fused_impl<256, true>(tm_dy, tm_codes, tm_duc, tm_al, a, 1, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qnf4
