// kernels.h — host-side launch functions of the CUDA kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <utility>

#include "nf4_lut.cuh"

namespace qnf4 {

// Whether launches use programmatic dependent launch (QLORA_PDL=0 disables).
bool pdl_enabled();

// Every check qlora_linear_fwd makes before it looks at the workspace, in the
// same order (shape, output dtype, M == 0 -> QLORA_OK, null pointers, weight
// pointers, alignment).  Xa is the adapter's input (X, or X after dropout).
qlora_status check_fwd_args(const uint16_t* X, const uint16_t* Xa, int64_t M, const nf4_weight& W,
                            const uint16_t* A, const uint16_t* B, int32_t r, const void* Y, int32_t y_dtype,
                            const float* U_out, const int32_t* d_status);

// cudaLaunchKernelEx with programmatic stream serialisation (when enabled)
// and an optional thread-block cluster shape.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 dim3 cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster.x * cluster.y * cluster.z > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster.x;
    attr[n].val.clusterDim.y = cluster.y;
    attr[n].val.clusterDim.z = cluster.z;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Arguments shared by the fused dequantise-in-GEMM kernels.  The W side of the
// product (dequantised NF4 rows: output features in the forward, input
// features in dX) is the MMA's M dimension; tokens are its N dimension.
struct FusedArgs {
  const uint8_t* c8;   // FP8 block constants of W [n_out * k_in / 64]
  const float* s2;     // group scales of W
  const float* mean;   // mean of W's constants (mean-centred scheme) or null
  void* out;           // out[m * ld_out + row]
  int out_f32;         // 1: fp32 output, 0: bf16 output
  int64_t ld_out;      // row stride of out (elements)
  int M;               // tokens
  int rows;            // extent of the W-side index (N for fwd, K for dX)
  int n_out, k_in;     // shape of W
  int r;               // LoRA rank
  int kt_total;        // main contraction stages (64 each)
  int kt_per_split;    // stages per blockIdx.z slice
  int32_t* status;
  Nf4Tables tab;
  // Grouped forward (several linears sharing X, stacked along W's rows): the
  // W-side rows where members 0..groups-2 end.  A tile of member g reads its
  // adapter operand from columns g * 2r of the stacked hi/lo copy of s*U.
  int groups;          // 1 for a single linear
  int grp_end[3];
};

// Member of a stacked group that W-side row `row` belongs to.
__host__ __device__ __forceinline__ int group_member(const int* ends, int groups, int row) {
  int g = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) g += (i < groups - 1 && row >= ends[i]) ? 1 : 0;
  return g;
}

enum SkinnyMode { kSkDown = 0, kSkDU = 1, kSkDB = 2, kSkDA = 3 };

// A group of G linears sharing one input, stacked along the output dimension:
// member g owns output rows grp_n[g] .. grp_n[g+1]-1 of the stacked W, B and
// dB, rows g*r .. g*r+r-1 of the stacked A and dA, and columns g*r .. of U
// (row stride G*r) and g*2r .. of the hi/lo copies (row stride 2*G*r).  A
// single linear is the group of one.  DOWN, DU and DA grids hold G CTAs per
// row tile (blockIdx.x = tile * G + g); DB finds g from its output rows.
struct SkinnyArgs {
  int M, N, K, r;       // N: all members' outputs; r: one member's rank
  int stages_total;     // contraction stages (64 each); DU: those of the longest member
  int stages_per_split; // stages per CTA of a cluster (the cluster spans the splits)
  float s;              // DOWN: scale of the hi/lo copy of U; DU: the LoRA scale
  float* out_f32;       // DOWN: U [M, G r]; DB: dB [N, r]; DA: dA [G r, K]
  uint16_t* out_cat;    // DOWN: hi/lo of s*U [M, 2 G r]; DU: hi/lo of dU [M, 2 G r]
  const float* in_u;    // DU: the saved U [M, G r]
  uint16_t* out_cat2;   // DU: hi/lo of s*U [M, 2 G r] (the dB operand)
  int32_t* status;
  int groups;           // G (1..4)
  int grp_n[5];         // member offsets along N (grp_n[0] = 0, grp_n[G] = N)
  uint32_t* zero;       // DOWN: words cleared by the first CTA (the few-token forward's tile counters)
  int zero_count;
  // 1: the "members" are rank chunks of one linear of rank r_total: chunk g
  // holds ranks g r .. g r + rw - 1, rw = min(r, r_total - g r) (r = 64);
  // DU reads all N outputs of dY and those columns of B [N, r_total]; DB runs
  // G CTAs per row tile and writes those columns of dB [N, r_total].
  int chunks;
  int r_total;
};

// One CTA waits on an mbarrier nothing completes, with a `limit_ns` bound,
// then reports QLORA_DEV_TIMEOUT (quant.cu; diagnostics).
cudaError_t launch_selftest_timeout(int32_t* status, uint64_t limit_ns, cudaStream_t stream);

// LoRA dropout on the adapter input (dropout.cu).
struct DropoutArgs {
  uint64_t seed;        // Philox key: (seed mod 2^32, seed div 2^32)
  uint32_t threshold;   // keep when the 32-bit word is below this
  int keep_all;         // p = 0: every element kept
  float c;              // fp32(1 / (1 - p))
};
//   X_drop = dropout(X) over `count` elements (a multiple of 4).
cudaError_t launch_dropout_apply(const uint16_t* X, uint16_t* Xd, int64_t count, const DropoutArgs& d,
                                 cudaStream_t stream);
//   out = dx32 + keep * c * (dU A): dx32 fp32 [M, K], dU as the bf16 hi/lo pairs
//   of the interleaved [M, 2r] layout, A bf16 [r, K]; K % 64 == 0, r <= 64.
cudaError_t launch_dropout_dx(const float* dx32, const uint16_t* ducat, const uint16_t* A, void* out, int out_f32,
                              int M, int K, int r, const DropoutArgs& d, cudaStream_t stream);

// AdamW step with 8-bit states (optim.cu).
struct AdamW8Args {
  uint16_t* p;       // [n] bf16 parameters, in place
  const float* g;    // [n] fp32 gradients
  uint8_t* m8;       // [n] E4M3 codes of m
  uint8_t* u8;       // [n] E4M3 codes of sqrt(v)
  float* m_scale;    // [ceil(n/256)]
  float* u_scale;    // [ceil(n/256)]
  int64_t n;
  float lr, b1, b2, omb1, omb2, eps, wd, bc1, bc2;
  int32_t* status;
};
cudaError_t launch_adamw8(const AdamW8Args& a, cudaStream_t stream);

cudaError_t launch_nf4_quantize(const uint16_t* w, int64_t numel, uint8_t* codes, uint8_t* c8, float* s2,
                                int32_t* status, const Nf4Tables& tab, cudaStream_t stream);
// Mean-centred constants: codes plus the fp32 constants (cbuf [nblocks]) and
// fp64 group sums (gsum [ngroups]); then the mean; then the centred FP8 encoding.
cudaError_t launch_nf4_quantize_centered(const uint16_t* w, int64_t numel, uint8_t* codes, uint8_t* c8, float* s2,
                                         float* mean, float* cbuf, double* gsum, double* lvl0, double* lvl1,
                                         int32_t* status, const Nf4Tables& tab, cudaStream_t stream);
//   tm_out: out viewed as [numel / 64, 64] bf16, box {64, 32} SW128 (null when numel < 64);
//   mean: null for the plain scheme.
cudaError_t launch_nf4_dequantize(const uint8_t* codes, const uint8_t* c8, const float* s2, const float* mean,
                                  int64_t numel, uint16_t* out, const CUtensorMap* tm_out, const Nf4Tables& tab,
                                  cudaStream_t stream);

// Forward: Y[m, n] (+)= sum_k X[m,k] W'[n,k]  (+ LoRA extension in split 0).
//   tm_x: X [M,K] box {64, BN} SW128; tm_codes: codes [N, K/2] box {32, 128};
//   tm_uc: Ucat [M, 2r] box {64, BN} SW128; tm_bl: B [N, r] box {64, 128} SW128.
cudaError_t launch_fused_fwd(int bn, const CUtensorMap& tm_x, const CUtensorMap& tm_codes,
                             const CUtensorMap& tm_uc, const CUtensorMap& tm_bl, const FusedArgs& a,
                             int splits, cudaStream_t stream);

// dX: dX[m, k] = sum_n dY[m,n] W'[n,k] + LoRA extension.
//   tm_dy: dY [M,N] box {64, BN} SW128; tm_codes: codes [N, K/2] box {64, 64};
//   tm_duc: dUcat [M, 2r] box {64, BN} SW128; tm_al: A [r, K] box {64, 64} SW128.
cudaError_t launch_fused_dx(int bn, const CUtensorMap& tm_dy, const CUtensorMap& tm_codes,
                            const CUtensorMap& tm_duc, const CUtensorMap& tm_al, const FusedArgs& a, int splits,
                            cudaStream_t stream);

// Large-M forward / dX: 128 W-side rows x 512 tokens per CTA, 32-deep stages.
//   tm_b: X or dY [M, *] box {32, 256} SW64; tm_codes: fwd [N, K/2] box {16, 128},
//   dX [N, K/2] box {64, 32}; tm_uc: Ucat/dUcat [M, 2r] box {32, 256} SW64;
//   tm_ext: fwd B [N, r] box {32, 128} SW64, dX A [r, K] box {64, 16} SW128.
//   a.kt_total counts stages of 32.
cudaError_t launch_fused2x(bool dx, const CUtensorMap& tm_b, const CUtensorMap& tm_codes, const CUtensorMap& tm_uc,
                           const CUtensorMap& tm_ext, const FusedArgs& a, cudaStream_t stream);

// Same products on CTA pairs (tcgen05 cta_group::2): 256 W-side rows x 512
// tokens per cluster of two CTAs, 8-stage rings.  Needs rows % 256 == 0.
//   tm_b / tm_uc: boxes {32, 128} SW64; other maps as for launch_fused2x.
cudaError_t launch_fused_pair(bool dx, const CUtensorMap& tm_b, const CUtensorMap& tm_codes,
                              const CUtensorMap& tm_uc, const CUtensorMap& tm_ext, const FusedArgs& a,
                              cudaStream_t stream);

// Large-M forward on CTA pairs with the dequantised tile in tensor memory:
// 256 W rows x pair_fwd_tokens(slots) tokens per cluster of two CTAs (`slots`
// A slots of 16 columns: 4 or 8).  Needs rows % 256 == 0.
//   tm_b: X [M, K] box {32, tokens/4} SW64; tm_codes: codes [N, K/2] box {16, 128};
//   tm_uc: Ucat [M, 2r] box {32, tokens/4} SW64; tm_ext: B [N, r] box {32, 128} SW64.
int pair_fwd_tokens(int slots);
cudaError_t launch_fused_pair_fwd(const CUtensorMap& tm_b, const CUtensorMap& tm_codes, const CUtensorMap& tm_uc,
                                  const CUtensorMap& tm_ext, const FusedArgs& a, int slots,
                                  cudaStream_t stream);

// Skinny LoRA products; the contraction is split over a cluster of `splits`
// (1..8) CTAs along y and reduced in-cluster.  See skinny.cu for the maps.
cudaError_t launch_skinny(int mode, const CUtensorMap& tmA, const CUtensorMap& tmB, const SkinnyArgs& a,
                          int grid_rows, int splits, cudaStream_t stream);

// Few-token forward (M <= 32): register-operand MMAs on in-register
// dequantised tiles, persistent CTAs over (128-row tile, 256-wide K chunk)
// units; the last CTA to finish a row tile adds its partials in CTA order and
// s U B^T (U from the rank-r kernel launched just before).  See lowm.cu.
constexpr int kLowmThreads = 256;
constexpr int kLowmRows = 128;
constexpr int kLowmMaxM = 16;  // token rows the few-token kernel takes (8 or 16 per MMA column block)

struct LowmArgs {
  const uint8_t* codes;  // [N, K/2]
  const uint8_t* c8;     // [N * K / 64]
  const float* s2;
  const float* mean;     // mean of W's constants (mean-centred scheme) or null
  const uint16_t* B;     // [N, r] bf16
  float* part;           // [ctas][2][128][mpad] fp32 partials
  void* Y;               // [M, N]
  int y_f32;
  const float* U;        // [M, ra] fp32, from the rank-r kernel launched before
  uint32_t* tile_count;  // [tiles] partials counted in, cleared by that kernel
  float s;
  int M, N, K, r;
  int tiles;             // ceil(N / 128)
  int atiles;            // 0 (U comes from the rank-r kernel)
  int kc;                // ceil(K / 256)
  int ctas;              // CTAs of the main kernel (>= tiles + atiles)
  int mpad;              // tokens per partial row: 8 * n8 token tiles (8, 16 or 32)
  int32_t* status;
  Nf4Tables tab;
  // Grouped forward: A holds the G members' adapters stacked ([ra = G r, K]),
  // U is [M, ra], B and Y are stacked along N; members end at grp_end.
  int ra;
  int groups;
  int grp_end[3];
};

//   tm_codes: codes [N, K/2] u8 box {128, 128} SW128; tm_x: X [M, K] bf16
//   box {64, mpad} SW128.
cudaError_t launch_lowm_fwd(const CUtensorMap& tm_codes, const CUtensorMap& tm_x, const LowmArgs& a,
                            cudaStream_t stream);

}  // namespace qnf4
