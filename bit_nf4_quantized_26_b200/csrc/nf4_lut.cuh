// nf4_lut.cuh — NF4 level tables and the register lookups used by every kernel
// that turns 4-bit codes into bf16 weights ("QLoRA" encyclopedia entry,
// tonho.wtf, sections "a ideia" and "como funciona").
#pragma once

#include "sm100.cuh"

namespace qnf4 {

// Host-computed constants, passed to kernels by value (constant bank).
//   q[16]     NF4 levels, ascending, fp32 (code i -> q[i]; q[7] = 0)
//   thr/base  bucket table of the quantiser: bucket b = RNE(16 x + 16) covers
//             x in [-1 + (b - 0.5)/16, -1 + (b + 0.5)/16], b = 0..32 (entry 63
//             guards x < -1 - 1/32, which cannot occur); every bucket holds at
//             most one midpoint m_i and none lies on a bucket edge, so
//             code(x) = base[b] + (x > thr[b]).
struct Nf4Tables {
  float q[16];
  float thr[64];
  int base[64];
};

// Byte planes of a 16-entry bf16 table T[i] = bf16(RN32(q[i] * chat)):
// L[k] holds the low bytes of T[4k..4k+3], H[k] the high bytes.
struct Nf4Lut {
  uint32_t L[4];
  uint32_t H[4];
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Dequantised block constant chat = RN32(e4m3(c8) * s2).
__device__ __forceinline__ float nf4_block_scale(uint32_t c8_byte, float s2) {
  return __fmul_rn(e4m3_to_float(c8_byte), s2);
}

// Mean of the constants of a mean-centred weight (0 and unused otherwise):
// chat = RN32(RN32(e4m3(c8) * s2) + mean).
struct Nf4Mean {
  bool centered;
  float value;
};

__device__ __forceinline__ Nf4Mean nf4_load_mean(const float* mean) {
  return Nf4Mean{mean != nullptr, mean != nullptr ? __ldg(mean) : 0.0f};
}

__device__ __forceinline__ float nf4_block_scale(uint32_t c8_byte, float s2, const Nf4Mean& m) {
  const float c = nf4_block_scale(c8_byte, s2);
  return m.centered ? __fadd_rn(c, m.value) : c;
}

// The 16 dequantised values of one block, as byte planes.  Two separate
// roundings per value: RN32 product, then RNE to bf16.
__device__ __forceinline__ Nf4Lut nf4_make_lut(const Nf4Tables& tab, float chat) {
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    P[j] = pack_bf16x2(__fmul_rn(tab.q[2 * j], chat), __fmul_rn(tab.q[2 * j + 1], chat));
  }
  Nf4Lut t;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t.L[k] = prmt(P[2 * k], P[2 * k + 1], 0x6420u);
    t.H[k] = prmt(P[2 * k], P[2 * k + 1], 0x7531u);
  }
  return t;
}

// Four codes -> four bf16 values.  `idx` holds the low three bits of each
// code in nibbles 0..3 and `msk` is 0xFF in byte i where code i is >= 8; the
// result is two packed pairs (element 0 in the low half of o01).
__device__ __forceinline__ void nf4_lookup4(uint32_t idx, uint32_t msk, const Nf4Lut& t, uint32_t& o01,
                                            uint32_t& o23) {
  const uint32_t la = prmt(t.L[0], t.L[1], idx);
  const uint32_t lb = prmt(t.L[2], t.L[3], idx);
  const uint32_t ha = prmt(t.H[0], t.H[1], idx);
  const uint32_t hb = prmt(t.H[2], t.H[3], idx);
  const uint32_t lo = (lb & msk) | (la & ~msk);
  const uint32_t hi = (hb & msk) | (ha & ~msk);
  o01 = prmt(lo, hi, 0x5140u);
  o23 = prmt(lo, hi, 0x7362u);
}

// Eight codes (one 32-bit word of packed codes, element i in nibble i) ->
// eight bf16 values in a uint4.  The high-bit masks come from the byte
// permute's sign-replicate mode: the top bit of code 2j is the top bit of
// byte j of (w << 4), that of code 2j+1 the top bit of byte j of w, so one
// permute of (w << 4, w) spreads four of them into byte masks.
__device__ __forceinline__ uint4 nf4_lookup8(uint32_t w, const Nf4Lut& t) {
  const uint32_t idx = w & 0x77777777u;
  const uint32_t ws = w << 4;
  uint4 o;
  nf4_lookup4(idx, prmt(ws, w, 0xD9C8u), t, o.x, o.y);
  nf4_lookup4(idx >> 16, prmt(ws, w, 0xFBEAu), t, o.z, o.w);
  return o;
}

// Two threads (adjacent lanes, `half` = lane & 1) build one block's table
// together: each forms four of the eight bf16 pairs and the pairs are swapped
// with a shuffle.  Every lane of the warp must call this (full-mask shuffle).
__device__ __forceinline__ Nf4Lut nf4_make_lut_pair(const Nf4Tables& tab, float chat, uint32_t half) {
  uint32_t mine[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = 8 * static_cast<int>(half) + 2 * j;
    mine[j] = pack_bf16x2(__fmul_rn(tab.q[e], chat), __fmul_rn(tab.q[e + 1], chat));
  }
  uint32_t other[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) other[j] = __shfl_xor_sync(0xFFFFFFFFu, mine[j], 1);
  uint32_t P[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    P[j] = half ? other[j] : mine[j];
    P[4 + j] = half ? mine[j] : other[j];
  }
  Nf4Lut t;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    t.L[k] = prmt(P[2 * k], P[2 * k + 1], 0x6420u);
    t.H[k] = prmt(P[2 * k], P[2 * k + 1], 0x7531u);
  }
  return t;
}

// Half of a 64-element block (16 bytes of codes at `src`, elements
// 32*half .. 32*half+31) into the 16-byte chunks 4*half .. 4*half+3 of a
// 128-byte swizzled shared-memory row (chunk j at position j ^ swz).
__device__ __forceinline__ void nf4_half_block_to_swizzled_row(const uint8_t* src, const Nf4Lut& t,
                                                               uint8_t* dst_row, uint32_t swz, uint32_t half) {
  const uint4 c = *reinterpret_cast<const uint4*>(src);
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (uint32_t j = 0; j < 4; ++j) {
    *reinterpret_cast<uint4*>(dst_row + (((4 * half + j) ^ swz) << 4)) = nf4_lookup8(cw[j], t);
  }
}

// Dequantise one 64-element block (32 bytes of codes at `src`, 16-byte aligned)
// into one 128-byte row of a 128-byte-swizzled shared-memory tile: the 16-byte
// chunk j (elements 8j..8j+7) goes to position (j ^ swz).
__device__ __forceinline__ void nf4_block_to_swizzled_row(const uint8_t* src, const Nf4Lut& t, uint8_t* dst_row,
                                                          uint32_t swz) {
  const uint4 c0 = *reinterpret_cast<const uint4*>(src);
  const uint4 c1 = *reinterpret_cast<const uint4*>(src + 16);
  const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (uint32_t j = 0; j < 8; ++j) {
    *reinterpret_cast<uint4*>(dst_row + ((j ^ swz) << 4)) = nf4_lookup8(cw[j], t);
  }
}

}  // namespace qnf4
