// quant.cu — NF4 blockwise quantisation with FP8 double quantisation, and the
// standalone dequantisation ("QLoRA" encyclopedia entry, tonho.wtf, sections
// "como funciona" and "a ideia").  Both kernels are HBM-bound streams.
#include "kernels.h"
#include "nf4_lut.cuh"

namespace qnf4 {

// ------------------------------------------------------------------ quantize
//
// One CTA (256 threads) owns one double-quantisation group: 256 blocks of 64
// elements = 32 KB of bf16 input.  Four threads share a block (16 elements,
// 32 bytes each, two 16-byte loads), so a warp reads 1 KB contiguous per
// pass and writes 256 contiguous bytes of codes; 4 passes cover the group.
// All 8 loads of a thread are issued before any arithmetic; five CTAs per SM
// keep 160 KB of loads in flight.  The block absmax is a max over the bf16
// magnitude bits (non-negative floats order like unsigned ints) reduced
// across the 4 lanes with two shuffles; each lane takes the block's
// reciprocal once for its 16 elements.  Per pair of elements the scaling and
// the bucket fma are one packed two-lane fp32 instruction each; the nearest
// code then costs one mask, a 4-byte threshold load and a 1-byte base load
// from shared memory (the 33 buckets' thresholds sit in distinct banks but
// for buckets 0 and 32, and all bases in 9 words, so a warp's loads rarely
// conflict), one compare and the nibble placement.

constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint32_t max_abs_bits(uint4 v) {
  // bf16 magnitudes of 8 elements, max over pairs with SIMD u16 max.
  uint32_t m = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return max(m & 0xFFFFu, m >> 16);
}

// x = RN32(e * rc) and t = RN32(16 x + C) for both elements of a bf16 pair,
// with packed two-lane fp32 instructions (each lane rounds as the scalar op).
// C = 1.5 * 2^23 + 16, so t's bits are 0x4B400000 + RNE(16 x + 16): the low
// six bits are the bucket b (b = 0..32 for |x| <= 1).
__device__ __forceinline__ void scale_pair(uint32_t word, uint64_t rc2, float& x0, float& x1, float& t0,
                                           float& t1) {
  uint64_t e2, x2, t2;
  asm("mov.b64 %0, {%1, %2};" : "=l"(e2) : "r"(word << 16), "r"(word & 0xFFFF0000u));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(x2) : "l"(e2), "l"(rc2));
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(t2)
      : "l"(x2), "l"(0x4180000041800000ull), "l"(0x4B4000104B400010ull));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x0), "=f"(x1) : "l"(x2));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(t0), "=f"(t1) : "l"(t2));
}

// Nearest-level code of x from its bucket: code = base[b] + (x > thr[b]).  The
// mask keeps the bucket inside the 64-entry tables whatever x is (a
// non-finite input gives an unspecified code, never a stray address).
__device__ __forceinline__ uint32_t quant_code(float x, float t, const float* thr, const uint8_t* base) {
  const uint32_t b = __float_as_uint(t) & 63u;
  return static_cast<uint32_t>(base[b]) + (x > thr[b] ? 1u : 0u);
}

// Packed codes of the 8 elements of v (element i in nibble i).
__device__ __forceinline__ uint32_t codes8(uint4 v, uint64_t rc2, const float* thr, const uint8_t* base) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float x0, x1, t0, t1;
    scale_pair(w[i], rc2, x0, x1, t0, t1);
    out = quant_code(x0, t0, thr, base) * (1u << (8 * i)) + out;
    out = quant_code(x1, t1, thr, base) * (1u << (8 * i + 4)) + out;  // disjoint nibbles: + == |
  }
  return out;
}

// Codes of 8 elements where 1/c is not finite (c = 0, or c so small that the
// reciprocal overflows): zero -> 7, positive -> 15, negative -> 0.
__device__ __forceinline__ uint32_t codes_degenerate(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t b = (w[i] >> (16 * h)) & 0xFFFFu;
      const uint32_t code = (b & 0x7FFFu) == 0 ? 7u : ((b & 0x8000u) ? 0u : 15u);
      out |= code << (4 * (2 * i + h));
    }
  }
  return out;
}

// CENTERED: instead of the FP8 step, the group's fp32 constants go to cbuf and
// their fp64 pairwise sum to gsum[group]; the mean and the centred encoding
// follow in more kernels.
template <bool CENTERED>
__global__ void __launch_bounds__(kQuantThreads, 5) nf4_quantize_kernel(const uint16_t* __restrict__ w,
                                                                         int64_t numel, uint8_t* __restrict__ codes,
                                                                         uint8_t* __restrict__ c8,
                                                                         float* __restrict__ s2, int32_t* status,
                                                                         Nf4Tables tab, float* __restrict__ cbuf,
                                                                         double* __restrict__ gsum) {
  __shared__ float thr[64];
  __shared__ uint8_t base[64];
  __shared__ uint32_t cblk[256];
  __shared__ uint32_t wmax[kQuantThreads / 32];

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, sub = lane & 3;
  if (tid < 64) {
    thr[tid] = tab.thr[tid];
    base[tid] = static_cast<uint8_t>(tab.base[tid]);
  }
  grid_dependency_wait();
  grid_dependents_launch();

  const int64_t nblocks = (numel + 63) / 64;
  const int64_t blk0 = static_cast<int64_t>(blockIdx.x) * 256;
  const bool full_group = (blk0 + 256) * 64 <= numel;

  // Pass p, lane: block p*64 + warp*8 + lane/4, elements sub*16 .. sub*16+15.
  uint4 v[4][2];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int64_t e0 = (blk0 + p * 64 + warp * 8 + (lane >> 2)) * 64 + sub * 16;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (full_group) {
        v[p][h] = __ldg(reinterpret_cast<const uint4*>(w + e0 + 8 * h));
      } else {
        uint32_t t[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t e = e0 + 8 * h + i;
          if (e < numel) t[i >> 1] |= static_cast<uint32_t>(w[e]) << (16 * (i & 1));
        }
        v[p][h] = make_uint4(t[0], t[1], t[2], t[3]);
      }
    }
  }
  __syncthreads();  // bucket tables ready

#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int lb = p * 64 + warp * 8 + (lane >> 2);
    uint32_t m = max(max_abs_bits(v[p][0]), max_abs_bits(v[p][1]));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    if (m > 0x7F7Fu && sub == 0 && status) atomicOr(status, QLORA_DEV_NONFINITE);
    const float c = __uint_as_float(m << 16);
    const float rc = __frcp_rn(c);
    uint2 out;
    if (rc < __int_as_float(0x7F800000)) {
      uint64_t rc2;
      asm("mov.b64 %0, {%1, %1};" : "=l"(rc2) : "f"(rc));
      out.x = codes8(v[p][0], rc2, thr, base);
      out.y = codes8(v[p][1], rc2, thr, base);
    } else {
      out.x = codes_degenerate(v[p][0]);
      out.y = codes_degenerate(v[p][1]);
    }
    const int64_t b = blk0 + lb;
    if (b < nblocks) *reinterpret_cast<uint2*>(codes + b * 32 + sub * 8) = out;
    if (sub == 0) cblk[lb] = m << 16;  // c as fp32 bits (0 for padding blocks)
  }
  __syncthreads();

  if (CENTERED) {
    const int64_t b = blk0 + tid;
    if (b < nblocks) cbuf[b] = __uint_as_float(cblk[tid]);
    // Pairwise sum of the group's 256 constants (padding blocks are +0):
    // neighbours by xor-shuffles within each warp (IEEE addition commutes, so
    // lane l and lane l ^ k form the same sum), then the 8 warp sums.
    double v = static_cast<double>(__uint_as_float(cblk[tid]));
#pragma unroll
    for (int k = 1; k < 32; k <<= 1) v = __dadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, k));
    __shared__ double wsum[kQuantThreads / 32];
    if (lane == 0) wsum[warp] = v;
    __syncthreads();
    if (tid == 0) {
      const double q0 = __dadd_rn(__dadd_rn(wsum[0], wsum[1]), __dadd_rn(wsum[2], wsum[3]));
      const double q1 = __dadd_rn(__dadd_rn(wsum[4], wsum[5]), __dadd_rn(wsum[6], wsum[7]));
      gsum[blockIdx.x] = __dadd_rn(q0, q1);
    }
    return;
  }

  // Double quantisation of the 256 constants of this group.
  const uint32_t cbits = cblk[tid];
  uint32_t amax = __reduce_max_sync(0xFFFFFFFFu, cbits);  // c >= 0: bit order = value order
  if (lane == 0) wmax[warp] = amax;
  __syncthreads();
  amax = wmax[0];
#pragma unroll
  for (int i = 1; i < kQuantThreads / 32; ++i) amax = max(amax, wmax[i]);
  const float scale = __fdiv_rn(__uint_as_float(amax), 448.0f);
  const float y = scale > 0.0f ? __fdiv_rn(__uint_as_float(cbits), scale) : 0.0f;
  const int64_t b = blk0 + tid;
  if (b < nblocks) c8[b] = static_cast<uint8_t>(float_to_e4m3_satfinite(y));
  if (tid == 0) s2[blockIdx.x] = scale;
}

// ------------------------------------------------ mean-centred constants
//
// The tensor mean of the block constants: their fp64 pairwise sum (zero-padded
// to a power of two, neighbours added level by level), divided by the number
// of blocks in fp64 and rounded once to fp32.  The group sums are the tree's
// nodes 256 constants up; each CTA of this kernel turns an aligned chunk of
// 2048 of the values below into their pairwise sum (values past `len` are
// +0, the padding), so repeated passes over 2048x fewer values reach the
// root, and the pass that runs as a single CTA writes the mean.
constexpr int kSumThreads = 1024;

__global__ void __launch_bounds__(kSumThreads) nf4_pairwise_kernel(const double* __restrict__ in, int64_t len,
                                                                   double* __restrict__ out, int64_t nblocks,
                                                                   float* mean) {
  __shared__ double wsum[32];
  grid_dependency_wait();
  grid_dependents_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * (2 * kSumThreads) + 2 * tid;
  const double x0 = i0 < len ? in[i0] : 0.0;
  const double x1 = i0 + 1 < len ? in[i0 + 1] : 0.0;
  double v = __dadd_rn(x0, x1);
#pragma unroll
  for (int k = 1; k < 32; k <<= 1) v = __dadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, k));
  if (lane == 0) wsum[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = wsum[lane];
#pragma unroll
    for (int k = 1; k < 32; k <<= 1) v = __dadd_rn(v, __shfl_xor_sync(0xFFFFFFFFu, v, k));
    if (lane == 0) {
      if (gridDim.x == 1) *mean = __double2float_rn(__ddiv_rn(v, static_cast<double>(nblocks)));
      else out[blockIdx.x] = v;
    }
  }
}

// Per group of 256 constants: c' = RN32(c - mean) (0 for padding blocks);
// s2 = RN32(max|c'| / 448); c8 = E4M3(RN32(c' / s2)), 0 when s2 = 0.
__global__ void __launch_bounds__(256) nf4_encode_centered_kernel(const float* __restrict__ cbuf, int64_t nblocks,
                                                                  const float* __restrict__ mean,
                                                                  uint8_t* __restrict__ c8, float* __restrict__ s2) {
  __shared__ uint32_t wmax[8];
  grid_dependency_wait();
  grid_dependents_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t b = static_cast<int64_t>(blockIdx.x) * 256 + tid;
  const float cc = b < nblocks ? __fsub_rn(cbuf[b], *mean) : 0.0f;
  // |c'| as bits: non-negative floats order like unsigned ints
  uint32_t amax = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(cc) & 0x7FFFFFFFu);
  if (lane == 0) wmax[warp] = amax;
  __syncthreads();
  amax = wmax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = max(amax, wmax[i]);
  const float scale = __fdiv_rn(__uint_as_float(amax), 448.0f);
  const float y = scale > 0.0f ? __fdiv_rn(cc, scale) : 0.0f;
  if (b < nblocks) c8[b] = static_cast<uint8_t>(float_to_e4m3_satfinite(y));
  if (tid == 0) s2[blockIdx.x] = scale;
}

// ---------------------------------------------------------------- dequantize
//
// One thread per 64-element block (its 32 bytes of codes in two 128-bit
// loads, a warp reading 1 KB contiguous; its table built once).  The 128
// bytes of bf16 it produces go to shared memory in the 128-byte-swizzled
// layout (row = block; conflict-free), and one lane per warp writes the
// warp's 32 rows (4 KB contiguous in HBM) with a single TMA store, so the
// global writes are whole lines.  A CTA covers one double-quantisation group,
// so all its blocks share one s2.  A trailing partial block (numel % 64) is
// written element by element.

constexpr int kDequantThreads = 256;

__global__ void __launch_bounds__(kDequantThreads) nf4_dequantize_kernel(const __grid_constant__ CUtensorMap tm_out,
                                                                          int has_map,
                                                                          const uint8_t* __restrict__ codes,
                                                                          const uint8_t* __restrict__ c8,
                                                                          const float* __restrict__ s2,
                                                                          const float* __restrict__ mean,
                                                                          int64_t numel, uint16_t* __restrict__ out,
                                                                          Nf4Tables tab) {
  __shared__ __align__(1024) uint8_t stage[kDequantThreads * 128];
  grid_dependency_wait();
  grid_dependents_launch();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t b = static_cast<int64_t>(blockIdx.x) * kDequantThreads + tid;
  const int64_t nblocks = (numel + 63) / 64, nfull = numel / 64;
  const bool valid = b < nblocks;
  const Nf4Mean wmean = nf4_load_mean(mean);
  const float chat = valid ? nf4_block_scale(__ldg(c8 + b), __ldg(s2 + (b >> 8)), wmean) : 0.0f;
  const Nf4Lut lut = nf4_make_lut(tab, chat);
  uint4 c0 = make_uint4(0x77777777u, 0x77777777u, 0x77777777u, 0x77777777u), c1 = c0;  // code 7 = +0
  if (valid) {
    c0 = __ldg(reinterpret_cast<const uint4*>(codes + b * 32));
    c1 = __ldg(reinterpret_cast<const uint4*>(codes + b * 32 + 16));
  }
  const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  uint8_t* row = stage + tid * 128;
  const uint32_t sw = static_cast<uint32_t>(tid) & 7u;
#pragma unroll
  for (uint32_t j = 0; j < 8; ++j) *reinterpret_cast<uint4*>(row + ((j ^ sw) << 4)) = nf4_lookup8(cw[j], lut);
  if (b == nfull && valid) {
    // partial last block: elements [b*64, numel)
    for (int e = 0; e < static_cast<int>(numel - b * 64); ++e) {
      const int j = e >> 3;
      out[b * 64 + e] = *reinterpret_cast<const uint16_t*>(row + ((j ^ sw) << 4) + (e & 7) * 2);
    }
  }
  fence_proxy_async_smem();  // this lane's rows -> async proxy
  __syncwarp();
  const int64_t wrow = static_cast<int64_t>(blockIdx.x) * kDequantThreads + warp * 32;
  if (lane == 0 && has_map && wrow < nfull) {
    tma_store_2d(&tm_out, stage + warp * 32 * 128, 0, static_cast<int>(wrow));  // rows >= nfull are clipped
    bulk_commit_group();
    bulk_wait_group_read0();  // shared memory stays valid until the store has read it
  }
}

// ------------------------------------------------------------------ launches

cudaError_t launch_nf4_quantize(const uint16_t* w, int64_t numel, uint8_t* codes, uint8_t* c8, float* s2,
                                int32_t* status, const Nf4Tables& tab, cudaStream_t stream) {
  const int64_t ngroups = (numel + 16383) / 16384;
  return launch_kernel(nf4_quantize_kernel<false>, dim3(static_cast<unsigned>(ngroups)), dim3(kQuantThreads), 0,
                       stream, dim3(1, 1, 1), w, numel, codes, c8, s2, status, tab, static_cast<float*>(nullptr),
                       static_cast<double*>(nullptr));
}

cudaError_t launch_nf4_quantize_centered(const uint16_t* w, int64_t numel, uint8_t* codes, uint8_t* c8, float* s2,
                                         float* mean, float* cbuf, double* gsum, double* lvl0, double* lvl1,
                                         int32_t* status, const Nf4Tables& tab, cudaStream_t stream) {
  const int64_t nblocks = (numel + 63) / 64;
  const int64_t ngroups = (numel + 16383) / 16384;
  const dim3 one(1, 1, 1);
  cudaError_t e = launch_kernel(nf4_quantize_kernel<true>, dim3(static_cast<unsigned>(ngroups)), dim3(kQuantThreads),
                                0, stream, one, w, numel, codes, c8, s2, status, tab, cbuf, gsum);
  if (e != cudaSuccess) return e;
  // Pairwise passes: gsum -> lvl0 -> lvl1 -> lvl0 ... until one CTA is left.
  const double* in = gsum;
  int64_t len = ngroups;
  for (int pass = 0;; ++pass) {
    const int64_t ctas = (len + 2 * kSumThreads - 1) / (2 * kSumThreads);
    double* out = (pass & 1) ? lvl1 : lvl0;
    e = launch_kernel(nf4_pairwise_kernel, dim3(static_cast<unsigned>(ctas)), dim3(kSumThreads), 0, stream, one, in,
                      len, out, nblocks, mean);
    if (e != cudaSuccess || ctas == 1) break;
    in = out;
    len = ctas;
  }
  if (e != cudaSuccess) return e;
  return launch_kernel(nf4_encode_centered_kernel, dim3(static_cast<unsigned>(ngroups)), dim3(256), 0, stream, one,
                       static_cast<const float*>(cbuf), nblocks, static_cast<const float*>(mean), c8, s2);
}

cudaError_t launch_nf4_dequantize(const uint8_t* codes, const uint8_t* c8, const float* s2, const float* mean,
                                  int64_t numel, uint16_t* out, const CUtensorMap* tm_out, const Nf4Tables& tab,
                                  cudaStream_t stream) {
  const int64_t nblocks = (numel + 63) / 64;
  const int64_t grid = (nblocks + kDequantThreads - 1) / kDequantThreads;
  CUtensorMap none{};
  return launch_kernel(nf4_dequantize_kernel, dim3(static_cast<unsigned>(grid)), dim3(kDequantThreads), 0, stream,
                       dim3(1, 1, 1), tm_out ? *tm_out : none, tm_out ? 1 : 0, codes, c8, s2, mean, numel, out, tab);
}

// ------------------------------------------------------- bounded-wait self-test
//
// Two warps wait on one shared-memory mbarrier that expects an arrival that
// never comes, through the same waits the kernels' roles use, with the
// kernels' WaitCtx (CTA abort flag, device status word) and a caller-chosen
// limit in place of the 2 s: warp 0 as a producer / MMA issuer does (lane 0
// polls, mbar_wait_warp), warp 1 as the dequantisers do (every lane polls,
// mbar_wait_all).  Whichever runs out first records QLORA_DEV_TIMEOUT and
// raises the abort flag; the other then gives up on the flag.  Each warp whose
// wait returned false adds 1 to status[1].
__global__ void selftest_timeout_kernel(int32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtx wc{&abort_flag, status};
  const int warp = threadIdx.x >> 5;
  const bool ok = warp == 0 ? mbar_wait_warp(&bar, 0, wc, limit_ns) : mbar_wait_all(&bar, 0, wc, limit_ns);
  if ((threadIdx.x & 31) == 0 && !ok) atomicAdd(status + 1, 1);
}

cudaError_t launch_selftest_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t stream) {
  selftest_timeout_kernel<<<1, 64, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace qnf4
