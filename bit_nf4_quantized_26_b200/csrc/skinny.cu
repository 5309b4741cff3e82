// skinny.cu — the rank-r products of the LoRA adapter path ("QLoRA"
// encyclopedia entry, tonho.wtf, section "a ideia": the adapters stay in 16 bit
// and are the only parameters that receive gradients).
//
//   mode DOWN:  U[m, j]  = sum_k X[m,k]  A[j,k]        -> U (fp32), bf16 hi/lo of s*U
//   mode DU:    dU[m, j] = s * sum_n dY[m,n] B[n,j]    -> bf16 hi/lo of dU (and of s*U)
//   mode DB:    dB[n, j] = sum_m dY[m,n] sU[m,j]       -> dB (fp32)
//   mode DA:    dA[j, k] = sum_m dU[m,j] X[m,k]        -> dA (fp32)
//
// Each is a tcgen05 GEMM with M = 128 rows and a narrow N that streams its long
// operand through a TMA ring.  The contraction is split over the S CTAs of a
// thread-block cluster (S <= 8, along blockIdx.y): every CTA parks its fp32
// partial tile in its own shared memory, and after a cluster barrier each CTA
// sums a slice of the tile's rows over all S partials through distributed
// shared memory, in rank order 0..S-1, and writes the final outputs.  The
// result is deterministic and needs no partial buffers in global memory and
// no extra launch.  The fp32 operands (sU, dU) enter the tensor core as a
// bf16 hi/lo pair in the interleaved "hi/lo per 16" column layout: column c
// holds part (c/16)%2 (0 = hi, 1 = lo) of j = 16*(c/32) + c%16.  A single
// linear of rank above 64 runs as rank chunks of 64 in the members' place
// (SkinnyArgs::chunks), the same layout.
#include "kernels.h"

namespace qnf4 {

// Shared-memory ring per mode: about 97 KB, so two CTAs fit on an SM (each
// with three or four 24-32 KB stages in flight).
template <int MODE>
struct SkPlan {
  static constexpr uint32_t kA = 16384;
  static constexpr uint32_t kB = (MODE == kSkDA || MODE == kSkDB) ? 16384 : 8192;
  static constexpr uint32_t kStage = kA + kB;
  static constexpr uint32_t kStages = (MODE == kSkDA || MODE == kSkDB) ? 3 : 4;
  static constexpr uint32_t kCtasPerSm = 2;
  static constexpr uint32_t kBarOff = kStages * kStage;
  static constexpr uint32_t kSmem = 1024 + kBarOff + 256;
  static constexpr uint32_t kTmemCols = (MODE == kSkDA || MODE == kSkDB) ? 128 : 64;
  // Partial tile parked in the (then idle) ring: 128 rows x r (padded to 68
  // floats per row so the per-row float4 stores spread over the banks), or for
  // DA r rows x 128 columns (padded to 132).
  static constexpr int kLdRows = 68;
  static constexpr int kLdCols = 132;
  static_assert(kSmem * kCtasPerSm <= 232448u, "ring too large for the CTAs per SM");
  static_assert(128 * kLdRows * 4 <= kStages * kStage, "partial tile must fit in the ring");
  static_assert(64 * kLdCols * 4 <= kStages * kStage || MODE != kSkDA, "partial tile must fit in the ring");
};

__device__ __forceinline__ int hilo_col(int j) { return 32 * (j >> 4) + (j & 15); }

// v -> (bf16(v), bf16(v - bf16(v))) at the interleaved hi/lo columns of row m
// (row stride `ld` elements; the member's columns start at `col0`).
__device__ __forceinline__ void store_hilo(uint16_t* cat, int m, int ld, int col0, int j, float v) {
  const uint16_t hi = bf16_bits(v);
  const uint16_t lo = bf16_bits(__fsub_rn(v, bf16_bits_to_float(hi)));
  uint16_t* row = cat + static_cast<int64_t>(m) * ld + col0;
  row[hilo_col(j)] = hi;
  row[hilo_col(j) + 16] = lo;
}

template <int MODE>
__global__ void __launch_bounds__(192, SkPlan<MODE>::kCtasPerSm)
    skinny_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const SkinnyArgs a) {
  using P = SkPlan<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P::kBarOff);
  uint64_t* empty = full + P::kStages;
  uint64_t* accf = empty + P::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Tile origin: DOWN/DU rows are tokens, DB rows are output features, DA's
  // 128 rows are the hi/lo columns of dU and its tiles walk K in 128s.  The
  // member g: DOWN, DU and DA have G CTAs per tile; DB's rows lie in one member
  // (rank chunks of one linear: DB too has G CTAs per row tile).
  const int G = a.groups;
  const bool per_tile = MODE != kSkDB || a.chunks;
  const int tile = per_tile ? static_cast<int>(blockIdx.x) / G : static_cast<int>(blockIdx.x);
  const int row0 = tile * 128;
  int g = per_tile ? static_cast<int>(blockIdx.x) % G : 0;
  if (!per_tile)
    for (int i = 1; i < G; ++i) g += row0 >= a.grp_n[i] ? 1 : 0;
  const int ra = a.chunks ? a.r_total : G * a.r;  // U row stride
  const int ucol = g * 2 * a.r;                   // this member's first hi/lo column
  const int rw = a.chunks ? min(a.r, a.r_total - g * a.r) : a.r;  // this member's rank
  const int nbase = a.chunks ? 0 : a.grp_n[g];  // DU: this member's first output feature
  const int z = blockIdx.y;
  const int st0 = z * a.stages_per_split;
  const int st_all = MODE == kSkDU && !a.chunks ? (a.grp_n[g + 1] - nbase) / 64 : a.stages_total;
  const int T = min(st_all, st0 + a.stages_per_split) - st0;  // <= 0: no MMA, the partial is zero
  const int nc = (2 * rw > 64) ? 128 : 64;  // DB: width of the sU operand

  if (threadIdx.x == 0) {
    for (uint32_t s = 0; s < P::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, P::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  const WaitCtx wc{abort_flag, a.status};
  grid_dependency_wait();  // inputs of earlier kernels are complete and visible
  grid_dependents_launch();
  if (MODE == kSkDown && a.zero && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < a.zero_count; i += blockDim.x) a.zero[i] = 0u;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (t >= static_cast<int>(P::kStages) && !mbar_wait(&empty[s], (u - 1) & 1, wc)) break;
        uint8_t* sa = smem + s * P::kStage;
        uint8_t* sb = sa + P::kA;
        const int kt = st0 + t;
        if (MODE == kSkDown) {
          mbar_arrive_expect_tx(&full[s], 16384 + 8192);
          tma_load_2d(sa, &tmA, &full[s], kt * 64, row0);
          tma_load_2d(sb, &tmB, &full[s], kt * 64, g * a.r);       // this member's rows of A
        } else if (MODE == kSkDU) {
          mbar_arrive_expect_tx(&full[s], 16384 + 8192);
          tma_load_2d(sa, &tmA, &full[s], nbase + kt * 64, row0);  // this member's columns of dY
          tma_load_2d(sb, &tmB, &full[s], a.chunks ? g * a.r : 0, nbase + kt * 64);  // and rows of B
        } else if (MODE == kSkDB) {
          const bool a2 = row0 + 64 < a.N;
          mbar_arrive_expect_tx(&full[s], 8192u * ((a2 ? 2 : 1) + nc / 64));
          tma_load_2d(sa, &tmA, &full[s], row0, kt * 64);
          if (a2) tma_load_2d(sa + 8192, &tmA, &full[s], row0 + 64, kt * 64);
          tma_load_2d(sb, &tmB, &full[s], ucol, kt * 64);
          if (nc == 128) tma_load_2d(sb + 8192, &tmB, &full[s], ucol + 64, kt * 64);
        } else {  // DA
          int nb = 0;
          for (int i = 0; i < 2; ++i) nb += (row0 + 64 * i < a.K) ? 1 : 0;
          mbar_arrive_expect_tx(&full[s], 8192u * ((nc / 64) + nb));
          tma_load_2d(sa, &tmA, &full[s], ucol, kt * 64);
          if (nc == 128) tma_load_2d(sa + 8192, &tmA, &full[s], ucol + 64, kt * 64);
          for (int i = 0; i < nb; ++i) tma_load_2d(sb + 8192 * i, &tmB, &full[s], row0 + 64 * i, kt * 64);
        }
        issued = t + 1;
      }
      for (int t = max(0, issued - static_cast<int>(P::kStages)); t < issued; ++t)
        mbar_drain(&full[t % P::kStages], (t / P::kStages) & 1, a.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const bool a_mn = (MODE == kSkDB || MODE == kSkDA);
      const bool b_mn = (MODE != kSkDown);
      const int n = MODE == kSkDA ? 128 : (MODE == kSkDB ? nc : 64);
      const uint32_t idesc = idesc_bf16_f32(128, n, a_mn ? 1 : 0, b_mn ? 1 : 0);
      const uint32_t a_step = a_mn ? (2048u >> 4) : (32u >> 4);
      const uint32_t b_step = b_mn ? (2048u >> 4) : (32u >> 4);
      bool aborted = false;
      for (int t = 0; t < T; ++t) {
        const uint32_t s = t % P::kStages, u = t / P::kStages;
        if (!mbar_wait(&full[s], u & 1, wc)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * P::kStage), sb = sa + P::kA;
        const uint64_t adesc = a_mn ? sdesc_sw128(sa, 8192, 1024) : sdesc_sw128(sa, 16, 1024);
        const uint64_t bdesc = b_mn ? sdesc_sw128(sb, 8192, 1024) : sdesc_sw128(sb, 16, 1024);
#pragma unroll
        for (uint32_t kk = 0; kk < 4; ++kk)
          umma_bf16(tmem_d, adesc + kk * a_step, bdesc + kk * b_step, idesc, (t | kk) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(accf);
      if (aborted) mbar_drain(accf, 0, a.status);
    }
  } else {
    // ------------------------------------------------ TMEM -> own partial tile
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    float* part = reinterpret_cast<float*>(smem);  // ring is idle once accf completes
    if (mbar_wait_warp(accf, 0, wc)) {
      tc_fence_after();
      const uint32_t tq = tmem_d + (static_cast<uint32_t>(q * 32) << 16);
      if (MODE == kSkDown || MODE == kSkDU) {
        // rows = tokens, columns j < r
        for (int cb = 0; cb < (rw + 31) / 32; ++cb) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tq + cb * 32, v);
          tmem_ld_wait();
          if (T <= 0)
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          float* dst = part + rl * P::kLdRows + cb * 32;
          const int nv = min(32, rw - cb * 32);
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            if (j < nv)
              *reinterpret_cast<float4*>(dst + j) = make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                                                __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        }
      } else if (MODE == kSkDB) {
        // rows = output features, columns = hi/lo pairs of j -> combined
        for (int jb = 0; jb < rw / 16; ++jb) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tq + jb * 32, v);
          tmem_ld_wait();
          if (T <= 0)
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          float* dst = part + rl * P::kLdRows + jb * 16;
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(dst + j) = make_float4(
                __uint_as_float(v[j]) + __uint_as_float(v[j + 16]),
                __uint_as_float(v[j + 1]) + __uint_as_float(v[j + 17]),
                __uint_as_float(v[j + 2]) + __uint_as_float(v[j + 18]),
                __uint_as_float(v[j + 3]) + __uint_as_float(v[j + 19]));
        }
      } else {  // DA: TMEM rows c = 32q + lane; hi row (lane < 16) plus lo row (lane + 16)
        const int j = 16 * q + lane;
        const bool jok = lane < 16 && j < rw;
        for (int cb = 0; cb < 4; ++cb) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tq + cb * 32, v);
          tmem_ld_wait();
          if (T <= 0)
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          float sum[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            sum[i] = __uint_as_float(v[i]) + __shfl_down_sync(0xFFFFFFFFu, __uint_as_float(v[i]), 16);
          if (jok) {
            float* dst = part + j * P::kLdCols + cb * 32;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) = make_float4(sum[i], sum[i + 1], sum[i + 2], sum[i + 3]);
          }
        }
      }
    }
  }

  // -------------------------------------------- cluster-wide fixed-order sum
  __syncwarp();
  cluster_sync_all();
  {
    const float* part = reinterpret_cast<const float*>(smem);
    const uint32_t S = gridDim.y;      // splits; a cluster of S > 1 spans the split dimension
    const uint32_t rank = blockIdx.y;  // this CTA's slice of the tile's rows
    // Cluster rank of the CTA holding split z: z itself, or with S = 1 (a
    // cluster of two row tiles, or none) this CTA.
    const uint32_t self = cluster_ctarank();
    auto holder = [&](uint32_t z) { return S == 1 ? self : z; };
    const bool by_rows = (MODE != kSkDA);
    const int R = by_rows ? 128 : rw;                  // rows of the partial tile
    const int C = by_rows ? rw : 128;                  // columns
    const int ld = by_rows ? P::kLdRows : P::kLdCols;  // floats per smem row
    const int rows_per = (R + static_cast<int>(S) - 1) / static_cast<int>(S);
    const int r0 = static_cast<int>(rank) * rows_per;
    const int r1 = min(R, r0 + rows_per);
    const int c4 = C / 4;
    for (int e = threadIdx.x; e < (r1 - r0) * c4; e += blockDim.x) {
      const int row = r0 + e / c4;
      const int col = (e % c4) * 4;
      const float* loc = part + row * ld + col;
      float4 acc = dsmem_ld_f4(dsmem_addr(loc, holder(0)));
      for (uint32_t z = 1; z < S; ++z) {
        const float4 v = dsmem_ld_f4(dsmem_addr(loc, holder(z)));
        acc.x = __fadd_rn(acc.x, v.x);
        acc.y = __fadd_rn(acc.y, v.y);
        acc.z = __fadd_rn(acc.z, v.z);
        acc.w = __fadd_rn(acc.w, v.w);
      }
      const float vals[4] = {acc.x, acc.y, acc.z, acc.w};
      if (MODE == kSkDown || MODE == kSkDU) {
        const int m = row0 + row;
        if (m < a.M) {
          if (MODE == kSkDown)
            *reinterpret_cast<float4*>(a.out_f32 + static_cast<int64_t>(m) * ra + g * a.r + col) = acc;
#pragma unroll
          for (int i = 0; i < 4; ++i) store_hilo(a.out_cat, m, 2 * ra, ucol, col + i, __fmul_rn(a.s, vals[i]));
          if (MODE == kSkDU) {
            // The same rows of the saved U, as the bf16 hi/lo of s*U for dB.
            const float4 uv =
                __ldg(reinterpret_cast<const float4*>(a.in_u + static_cast<int64_t>(m) * ra + g * a.r + col));
            const float us[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) store_hilo(a.out_cat2, m, 2 * ra, ucol, col + i, __fmul_rn(a.s, us[i]));
          }
        }
      } else if (MODE == kSkDB) {
        const int n = row0 + row;
        if (n < a.N) {
          float* o = a.chunks ? a.out_f32 + static_cast<int64_t>(n) * ra + g * a.r
                              : a.out_f32 + static_cast<int64_t>(n) * a.r;
          *reinterpret_cast<float4*>(o + col) = acc;
        }
      } else {
        const int k = row0 + col;
        if (k < a.K) *reinterpret_cast<float4*>(a.out_f32 + static_cast<int64_t>(g * a.r + row) * a.K + k) = acc;
      }
    }
  }
  __syncwarp();
  cluster_sync_all();  // peers may still be reading this CTA's partial tile

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, P::kTmemCols);
  }
}

template <int MODE>
static cudaError_t launch_skinny_impl(const CUtensorMap& tmA, const CUtensorMap& tmB, const SkinnyArgs& a,
                                      int grid_rows, int splits, cudaStream_t stream) {
  using P = SkPlan<MODE>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(skinny_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(P::kSmem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  if (splits < 1 || splits > 8) return cudaErrorInvalidValue;
  // Unsplit products run beside a CTA-pair GEMM: launched as clusters of two
  // row tiles they sit on both SMs of a TPC, rather than on one SM of many
  // TPCs, each of which could then hold no GEMM pair.
  const dim3 cluster = (splits == 1 && grid_rows % 2 == 0) ? dim3(2, 1, 1) : dim3(1, static_cast<unsigned>(splits), 1);
  return launch_kernel(skinny_kernel<MODE>, dim3(grid_rows, splits, 1), dim3(192), P::kSmem, stream, cluster, tmA,
                       tmB, a);
}

cudaError_t launch_skinny(int mode, const CUtensorMap& tmA, const CUtensorMap& tmB, const SkinnyArgs& a,
                          int grid_rows, int splits, cudaStream_t stream) {
  switch (mode) {
    case kSkDown: return launch_skinny_impl<kSkDown>(tmA, tmB, a, grid_rows, splits, stream);
    case kSkDU: return launch_skinny_impl<kSkDU>(tmA, tmB, a, grid_rows, splits, stream);
    case kSkDB: return launch_skinny_impl<kSkDB>(tmA, tmB, a, grid_rows, splits, stream);
    case kSkDA: return launch_skinny_impl<kSkDA>(tmA, tmB, a, grid_rows, splits, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qnf4
