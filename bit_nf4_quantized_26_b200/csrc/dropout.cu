// dropout.cu — LoRA dropout on the adapter input ("Tutorial fine-tuning LLM
// LoRA/QLoRA 2026", nexusinovation, section "Mão na Massa": the adapter
// configuration's lora_dropout).  The frozen path sees X, the adapter sees
// X_drop; the backward's dropout derivative is keep * c.
//
// Mask: Philox-4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel random
// numbers: as easy as 1, 2, 3", SC 2011), key (seed mod 2^32, seed div 2^32),
// counter (g mod 2^32, g div 2^32, 0, 0) for the group g of four consecutive
// elements of the flattened [M, K] tensor; word i of the call decides element
// 4g + i, kept when the word is below T = floor((1 - p) 2^32).  A kept element
// is bf16(RN32(x * c)) with c = fp32(1 / (1 - p)), a dropped one +0.
#include <algorithm>

#include "kernels.h"

namespace qnf4 {

namespace {

__device__ __forceinline__ uint4 philox4x32_10(uint4 ctr, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    const uint32_t lo0 = 0xD2511F53u * ctr.x, hi0 = __umulhi(0xD2511F53u, ctr.x);
    const uint32_t lo1 = 0xCD9E8D57u * ctr.z, hi1 = __umulhi(0xCD9E8D57u, ctr.z);
    ctr = make_uint4(hi1 ^ ctr.y ^ k0, lo1, hi0 ^ ctr.w ^ k1, lo0);
    k0 += 0x9E3779B9u;  // the bump after the last round is never used
    k1 += 0xBB67AE85u;
  }
  return ctr;
}

// Bit i set when element 4g + i is kept.
__device__ __forceinline__ uint32_t keep4(uint64_t g, const DropoutArgs& d) {
  if (d.keep_all) return 0xFu;
  const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), 0u, 0u),
                                static_cast<uint32_t>(d.seed), static_cast<uint32_t>(d.seed >> 32));
  return (w.x < d.threshold ? 1u : 0u) | (w.y < d.threshold ? 2u : 0u) | (w.z < d.threshold ? 4u : 0u) |
         (w.w < d.threshold ? 8u : 0u);
}

__device__ __forceinline__ uint32_t drop_pair(uint32_t xx, uint32_t keep2, float c) {
  const uint32_t lo = (keep2 & 1u) ? bf16_bits(__fmul_rn(bf16_bits_to_float(xx & 0xFFFFu), c)) : 0u;
  const uint32_t hi = (keep2 & 2u) ? bf16_bits(__fmul_rn(bf16_bits_to_float(xx >> 16), c)) : 0u;
  return lo | (hi << 16);
}

// X_drop = dropout(X): one Philox call per group of four elements, 8-byte
// loads and stores, grid-stride.
__global__ void __launch_bounds__(256) dropout_apply_kernel(const uint16_t* __restrict__ X, uint16_t* __restrict__ Xd,
                                                            int64_t groups, const DropoutArgs d) {
  grid_dependency_wait();
  grid_dependents_launch();
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < groups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint2 x = *reinterpret_cast<const uint2*>(X + 4 * g);
    const uint32_t k = keep4(static_cast<uint64_t>(g), d);
    *reinterpret_cast<uint2*>(Xd + 4 * g) = make_uint2(drop_pair(x.x, k, d.c), drop_pair(x.y, k >> 2, d.c));
  }
}

// dX = dX_main + keep * c * (dU A), dX_main fp32 [M, K] from the GEMM without
// its adapter stages, dU from the bf16 hi/lo pairs of the interleaved layout
// (column c holds part (c/16)%2 of j = 16 floor(c/32) + c%16), A bf16 [r, K].
// A CTA computes a 64 x 64 block of (m, k): dU A on the tensor cores
// (register-operand m16n8k16 MMAs, fp32 accumulate, the hi and the lo part of
// dU each once), over the rank in blocks of 64 staged in turn, then per
// element the mask and the add.  Warp w takes rows
// 16 (w % 4) .. + 15 and columns 32 (w / 4) .. + 31 of the block.
constexpr int kDxTile = 64;
constexpr int kDxLd = 64 + 8;  // bf16 per shared-memory row: 144 bytes, conflict-free fragment loads

__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256) dropout_dx_kernel(const float* __restrict__ dx32,
                                                         const uint16_t* __restrict__ ducat,
                                                         const uint16_t* __restrict__ A, void* __restrict__ out,
                                                         int out_f32, int M, int K, int r, const DropoutArgs d) {
  __shared__ __align__(16) uint16_t uh[kDxTile][kDxLd];  // [m][j] hi part of dU
  __shared__ __align__(16) uint16_t ul[kDxTile][kDxLd];  // [m][j] lo part
  __shared__ __align__(16) uint16_t at[kDxTile][kDxLd];  // [k][j] A transposed
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int m0 = blockIdx.y * kDxTile, k0 = blockIdx.x * kDxTile;
  grid_dependency_wait();
  grid_dependents_launch();
  const int mr = (warp & 3) * 16, kc = (warp >> 2) * 32;
  float acc[4][4] = {};
  // The rank in blocks of 64 staged one after the other (one for r <= 64).
  for (int j0 = 0; j0 < r; j0 += kDxTile) {
    if (j0 > 0) __syncthreads();  // the previous block's fragments are read
    for (int e = tid; e < kDxTile * kDxTile; e += 256) {
      const int mm = e / kDxTile, j = e % kDxTile;
      uint16_t hi = 0, lo = 0;
      if (m0 + mm < M && j0 + j < r) {
        const uint16_t* row = ducat + static_cast<int64_t>(m0 + mm) * 2 * r;
        const int col = 32 * ((j0 + j) >> 4) + ((j0 + j) & 15);
        hi = row[col];
        lo = row[col + 16];
      }
      uh[mm][j] = hi;
      ul[mm][j] = lo;
      const int jj = e / kDxTile, kk = e % kDxTile;
      at[kk][jj] = j0 + jj < r ? A[static_cast<int64_t>(j0 + jj) * K + k0 + kk] : uint16_t(0);
    }
    __syncthreads();
    for (int ks = 0; ks < min(kDxTile, r - j0); ks += 16) {
      const int jc = ks + 2 * t;
      const uint32_t ah0 = *reinterpret_cast<const uint32_t*>(&uh[mr + g][jc]);
      const uint32_t ah1 = *reinterpret_cast<const uint32_t*>(&uh[mr + g + 8][jc]);
      const uint32_t ah2 = *reinterpret_cast<const uint32_t*>(&uh[mr + g][jc + 8]);
      const uint32_t ah3 = *reinterpret_cast<const uint32_t*>(&uh[mr + g + 8][jc + 8]);
      const uint32_t al0 = *reinterpret_cast<const uint32_t*>(&ul[mr + g][jc]);
      const uint32_t al1 = *reinterpret_cast<const uint32_t*>(&ul[mr + g + 8][jc]);
      const uint32_t al2 = *reinterpret_cast<const uint32_t*>(&ul[mr + g][jc + 8]);
      const uint32_t al3 = *reinterpret_cast<const uint32_t*>(&ul[mr + g + 8][jc + 8]);
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int kk = kc + nt * 8 + g;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&at[kk][jc]);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&at[kk][jc + 8]);
        mma_16816_bf16(acc[nt], ah0, ah1, ah2, ah3, b0, b1);
        mma_16816_bf16(acc[nt], al0, al1, al2, al3, b0, b1);
      }
    }
  }
  // acc[nt]: (row g, columns 2t, 2t+1) and (row g + 8, the same columns) of
  // the 16 x 8 tile nt; the two columns lie in one group of four (one mask word).
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const int k = k0 + kc + nt * 8 + 2 * t;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = m0 + mr + g + 8 * h;
      if (m >= M) continue;
      const int64_t e = static_cast<int64_t>(m) * K + k;
      const uint32_t keep = keep4(static_cast<uint64_t>(e >> 2), d) >> (e & 3);
      const float2 base = *reinterpret_cast<const float2*>(dx32 + e);
      const float v0 = (keep & 1u) ? __fadd_rn(base.x, __fmul_rn(d.c, acc[nt][2 * h])) : base.x;
      const float v1 = (keep & 2u) ? __fadd_rn(base.y, __fmul_rn(d.c, acc[nt][2 * h + 1])) : base.y;
      if (out_f32) {
        *reinterpret_cast<float2*>(reinterpret_cast<float*>(out) + e) = make_float2(v0, v1);
      } else {
        *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(out) + e) =
            static_cast<uint32_t>(bf16_bits(v0)) | (static_cast<uint32_t>(bf16_bits(v1)) << 16);
      }
    }
  }
}

}  // namespace

cudaError_t launch_dropout_apply(const uint16_t* X, uint16_t* Xd, int64_t count, const DropoutArgs& d,
                                 cudaStream_t stream) {
  if (count % 4 != 0) return cudaErrorInvalidValue;
  const int64_t groups = count / 4;
  const int64_t ctas = std::min<int64_t>((groups + 255) / 256, 148 * 16);
  return launch_kernel(dropout_apply_kernel, dim3(static_cast<unsigned>(ctas)), dim3(256), 0, stream,
                       dim3(1, 1, 1), X, Xd, groups, d);
}

cudaError_t launch_dropout_dx(const float* dx32, const uint16_t* ducat, const uint16_t* A, void* out, int out_f32,
                              int M, int K, int r, const DropoutArgs& d, cudaStream_t stream) {
  if (K % kDxTile != 0 || r % 16 != 0 || r > 256) return cudaErrorInvalidValue;
  return launch_kernel(dropout_dx_kernel, dim3(K / kDxTile, (M + kDxTile - 1) / kDxTile), dim3(256), 0, stream,
                       dim3(1, 1, 1), dx32, ducat, A, out, out_f32, M, K, r, d);
}

}  // namespace qnf4
