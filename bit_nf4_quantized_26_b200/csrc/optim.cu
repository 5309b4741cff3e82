// optim.cu — the adapter optimizer step: AdamW with 8-bit states ("QLoRA"
// encyclopedia entry, tonho.wtf, section "como funciona": optimizer states in
// paged unified memory; "Tutorial fine-tuning LLM LoRA/QLoRA 2026",
// nexusinovation, section "Mão na Massa": the trainer's paged 8-bit AdamW).
//
// State per parameter tensor: E4M3 codes of the first moment m and of the
// square root u = sqrt(v) of the second moment, with one fp32 absmax scale per
// 256 elements for each (the two-level FP8 scheme the pages use for the
// quantisation constants).  Every operation is a single IEEE fp32 operation
// rounded to nearest even, in a fixed order, so the result is bit-exact with
// the CPU oracle:
//
//   m  = RN(e4m3(m8) s_m)      u = RN(e4m3(u8) s_u)      v = RN(u u)
//   m1 = RN(RN(b1 m) + RN((1-b1) g))
//   v1 = RN(RN(b2 v) + RN((1-b2) RN(g g)))          u1 = sqrt_RN(v1)
//   d  = RN(RN(m1 bc1) / RN(RN(u1 bc2) + eps));      d = RN(d + RN(wd p))
//   p1 = RN(p - RN(lr d))  -> bf16
//
// then per 256-element block s_m = RN(max|m1| / 448), m8 = E4M3(RN(m1 / s_m))
// (zero when s_m = 0) and the same for u1.
//
// One warp per 256-element block, 8 consecutive elements per lane (16-byte
// parameter and 2 x 16-byte gradient loads, 8-byte state loads); the block
// maxima are warp reductions over the magnitude bits.  The kernel streams
// 12 bytes per parameter (bf16 p read + write, fp32 g, two state bytes read +
// write): an HBM-bound stream.
#include "kernels.h"

namespace qnf4 {

namespace {

constexpr int kOptThreads = 256;  // 8 warps, 8 state blocks per CTA

__device__ __forceinline__ uint32_t e4m3_state_code(float x, float scale) {
  if (scale == 0.0f) return 0u;
  const uint32_t c = float_to_e4m3_satfinite(__fdiv_rn(x, scale));
  return (c & 0x7Fu) == 0 ? 0u : c;  // a value that rounds to zero is stored as +0
}

__global__ void __launch_bounds__(kOptThreads) adamw8_kernel(const AdamW8Args a) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int lane = threadIdx.x & 31;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * (kOptThreads / 32) + (threadIdx.x >> 5);
  const int64_t nblk = (a.n + 255) / 256;
  if (blk >= nblk) return;  // warp-uniform
  const int64_t e0 = blk * 256 + lane * 8;
  const bool full = e0 + 8 <= a.n;

  float g[8], p[8], m[8], u[8];
  const float sm = a.m_scale[blk], su = a.u_scale[blk];
  if (full) {
    const float4 g0 = *reinterpret_cast<const float4*>(a.g + e0);
    const float4 g1 = *reinterpret_cast<const float4*>(a.g + e0 + 4);
    const uint4 pv = *reinterpret_cast<const uint4*>(a.p + e0);
    const uint2 mv = *reinterpret_cast<const uint2*>(a.m8 + e0);
    const uint2 uv = *reinterpret_cast<const uint2*>(a.u8 + e0);
    g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w;
    g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
    const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      p[i] = bf16_bits_to_float((pw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
      const uint32_t mb = ((i < 4 ? mv.x : mv.y) >> (8 * (i & 3))) & 0xFFu;
      const uint32_t ub = ((i < 4 ? uv.x : uv.y) >> (8 * (i & 3))) & 0xFFu;
      m[i] = __fmul_rn(e4m3_to_float(mb), sm);
      u[i] = __fmul_rn(e4m3_to_float(ub), su);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool in = e0 + i < a.n;
      g[i] = in ? a.g[e0 + i] : 0.0f;
      p[i] = in ? bf16_bits_to_float(a.p[e0 + i]) : 0.0f;
      m[i] = in ? __fmul_rn(e4m3_to_float(a.m8[e0 + i]), sm) : 0.0f;
      u[i] = in ? __fmul_rn(e4m3_to_float(a.u8[e0 + i]), su) : 0.0f;
    }
  }

  float m1[8], u1[8], p1[8];
  uint32_t mmax = 0, umax = 0;
  bool finite = true;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    finite = finite && isfinite(g[i]);
    const float v = __fmul_rn(u[i], u[i]);
    m1[i] = __fadd_rn(__fmul_rn(a.b1, m[i]), __fmul_rn(a.omb1, g[i]));
    const float v1 = __fadd_rn(__fmul_rn(a.b2, v), __fmul_rn(a.omb2, __fmul_rn(g[i], g[i])));
    u1[i] = __fsqrt_rn(v1);
    const float den = __fadd_rn(__fmul_rn(u1[i], a.bc2), a.eps);
    float d = __fdiv_rn(__fmul_rn(m1[i], a.bc1), den);
    d = __fadd_rn(d, __fmul_rn(a.wd, p[i]));
    p1[i] = __fsub_rn(p[i], __fmul_rn(a.lr, d));
    mmax = max(mmax, __float_as_uint(m1[i]) & 0x7FFFFFFFu);  // magnitudes order like their bits
    umax = max(umax, __float_as_uint(u1[i]));
  }
  if (!finite && a.status) atomicOr(a.status, QLORA_DEV_NONFINITE);
  mmax = __reduce_max_sync(0xFFFFFFFFu, mmax);
  umax = __reduce_max_sync(0xFFFFFFFFu, umax);
  const float sm1 = __fdiv_rn(__uint_as_float(mmax), 448.0f);
  const float su1 = __fdiv_rn(__uint_as_float(umax), 448.0f);

  uint32_t mc[2] = {0, 0}, uc[2] = {0, 0}, pw[4] = {0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    mc[i >> 2] |= e4m3_state_code(m1[i], sm1) << (8 * (i & 3));
    uc[i >> 2] |= e4m3_state_code(u1[i], su1) << (8 * (i & 3));
    pw[i >> 1] |= static_cast<uint32_t>(bf16_bits(p1[i])) << (16 * (i & 1));
  }
  if (full) {
    *reinterpret_cast<uint4*>(a.p + e0) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
    *reinterpret_cast<uint2*>(a.m8 + e0) = make_uint2(mc[0], mc[1]);
    *reinterpret_cast<uint2*>(a.u8 + e0) = make_uint2(uc[0], uc[1]);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (e0 + i < a.n) {
        a.p[e0 + i] = static_cast<uint16_t>(pw[i >> 1] >> (16 * (i & 1)));
        a.m8[e0 + i] = static_cast<uint8_t>(mc[i >> 2] >> (8 * (i & 3)));
        a.u8[e0 + i] = static_cast<uint8_t>(uc[i >> 2] >> (8 * (i & 3)));
      }
    }
  }
  if (lane == 0) {
    a.m_scale[blk] = sm1;
    a.u_scale[blk] = su1;
  }
}

}  // namespace

cudaError_t launch_adamw8(const AdamW8Args& a, cudaStream_t stream) {
  const int64_t nblk = (a.n + 255) / 256;
  const int64_t ctas = (nblk + kOptThreads / 32 - 1) / (kOptThreads / 32);
  if (ctas > 0x7FFFFFFF) return cudaErrorInvalidValue;
  return launch_kernel(adamw8_kernel, dim3(static_cast<unsigned>(ctas)), dim3(kOptThreads), 0, stream,
                       dim3(1, 1, 1), a);
}

}  // namespace qnf4
