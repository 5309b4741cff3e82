/*
 * qlora_nf4.h — C ABI of the NF4 / QLoRA linear-layer library for sm_100a (B200).
 *
 * What the library computes (sources are web pages, cited by title and section):
 *
 *  - "QLoRA" encyclopedia entry (tonho.wtf), section "como funciona": a 4-bit
 *    storage type (NF4) built from standard-normal quantiles, asymmetric so that
 *    zero is exact; blockwise absmax quantisation with one constant per 64
 *    elements; the constants themselves quantised to FP8 in blocks of 256.
 *  - same entry, section "a ideia": weights are stored in 4 bit and dequantised
 *    to BFloat16 only when used in a matmul; the gradient crosses the frozen
 *    weight and lands in the 16-bit LoRA adapters, the only trainable parameters.
 *  - "Tutorial fine-tuning LLM LoRA/QLoRA 2026" (nexusinovation), section
 *    "LoRA: O Padrão Ouro de Eficiência": the adapter adds a scaled low-rank
 *    product to the frozen weight; "Mão na Massa" shows the knobs
 *    (r, lora_alpha, nf4, bf16 compute, double quant).
 *
 * Notation: W is [N = out, K = in] row-major (PyTorch Linear layout); X is
 * [M, K]; Y is [M, N]; the adapters are A [r, K] and B [N, r], all row-major;
 * s = alpha / r.  bf16 tensors are passed as uint16_t bit patterns.
 *
 *   forward:   U = X A^T (fp32)           Y = X W'^T + s U B^T
 *   backward:  dU = s dY B                dX = dY W' + dU A
 *              dA = dU^T X                dB = s dY^T U
 *
 * where W' = dequantize(NF4(W)) in bf16.  There is no dW (the base is frozen).
 * The same calls with LoRA dropout on the adapter input are declared below
 * (qlora_linear_{fwd,bwd}_dropout); the adapter optimizer step is in
 * qlora_optim.h.
 *
 * NF4 storage of a tensor of `numel` elements (flattened row-major):
 *   codes  uint8[ceil(numel/64)*32]  two 4-bit codes per byte; element 2j in
 *                                    the low nibble of byte j; code i is the
 *                                    i-th NF4 level in ascending order
 *                                    (code 7 is the exact zero)
 *   c8     uint8[ceil(numel/64)]     FP8 E4M3 absmax constant per 64 elements
 *   s2     float[ceil(numel/16384)]  fp32 scale per group of 256 constants
 *
 * Conventions common to every entry point:
 *  - Ownership: the caller allocates and owns every buffer (device memory
 *    unless stated).  The library never allocates or frees device memory and
 *    keeps no state beyond host-side constant tables and cached device
 *    attributes.
 *  - Asynchrony: every compute call only enqueues work on `stream` (a
 *    cudaStream_t; NULL = legacy default stream) and returns.  The returned
 *    status covers the synchronous argument checks and launch errors only.
 *  - Device-side conditions (non-finite input, a bounded wait that ran out)
 *    are OR-ed into the optional device word `d_status` (int32, caller
 *    zeroes it; NULL = not reported): bit 0 = QLORA_DEV_NONFINITE,
 *    bit 1 = QLORA_DEV_TIMEOUT.
 *  - Alignment: every pointer must be 16-byte aligned (QLORA_ERR_ALIGN).
 *  - Errors are reported before any work is enqueued; on error nothing runs.
 *  - Only sm_100 devices are supported (QLORA_ERR_ARCH); there is no fallback.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_API __attribute__((visibility("default")))
#else
#define QLORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_NULL = 1,       /* a required pointer is NULL                       */
  QLORA_ERR_SHAPE = 2,      /* a size violates the documented constraints      */
  QLORA_ERR_ALIGN = 3,      /* a pointer is not 16-byte aligned                */
  QLORA_ERR_WORKSPACE = 4,  /* workspace NULL or smaller than the size query   */
  QLORA_ERR_NONFINITE = 5,  /* (reserved for host-visible non-finite reports)  */
  QLORA_ERR_TIMEOUT = 6,    /* (reserved for host-visible timeout reports)     */
  QLORA_ERR_CUDA = 7,       /* a CUDA runtime/driver call failed               */
  QLORA_ERR_ARCH = 8,       /* current device is not sm_100                    */
  QLORA_ERR_DTYPE = 9,      /* unknown output dtype code                       */
  QLORA_ERR_INTERNAL = 10   /* the library's constant tables failed a check    */
} qlora_status;

/* Device status bits OR-ed into d_status by the kernels. */
#define QLORA_DEV_NONFINITE 1
#define QLORA_DEV_TIMEOUT 2

/* Output dtype codes for Y and dX. */
#define QLORA_DTYPE_BF16 0
#define QLORA_DTYPE_F32 1

/* A quantised weight [n_out, k_in]: views into caller-owned device memory.
 * mean: NULL for the plain double quantisation; for a weight quantised with
 * nf4_quantize_centered, the device address of its fp32 constants' mean
 * (every dequantiser then adds it to the block constant, see below). */
typedef struct {
  const uint8_t* codes; /* uint8[n_out*k_in/2]           */
  const uint8_t* c8;    /* uint8[n_out*k_in/64]          */
  const float* s2;      /* float[ceil(n_out*k_in/16384)] */
  int64_t n_out;
  int64_t k_in;
  const float* mean;    /* NULL, or float[1] (mean-centred constants) */
} nf4_weight;

/*
 * nf4_quantize — NF4 blockwise quantisation with FP8 double quantisation
 * ("QLoRA" entry, "como funciona").
 *
 *  w_bf16  [numel] bf16 input (device)
 *  numel   > 0, any value; the last 64-block is padded with +0 (code 7) and
 *          the last 256-constant group with zero constants
 *  codes   [ceil(numel/64)*32] out; c8 [ceil(numel/64)] out; s2 [ceil(numel/16384)] out
 *  d_status optional device word (see above); a non-finite input sets
 *          QLORA_DEV_NONFINITE and leaves the affected outputs unspecified
 *
 * Per block of 64: c = max|w|; x = RN32(w * RN32(1/c)); code = #{i: x > m_i}
 * with m_i the fp32 midpoints of adjacent levels (ties go to the lower code;
 * zero is always code 7).  Per group of 256 constants: s2 = RN32(amax/448);
 * c8 = E4M3 round-to-nearest-even, saturating (RN32(c/s2)).  Bit-exact with
 * the CPU oracle.  numel == 0 is a no-op.
 */
QLORA_API qlora_status nf4_quantize(const uint16_t* w_bf16, int64_t numel, uint8_t* codes, uint8_t* c8,
                          float* s2, int32_t* d_status, void* stream);

/*
 * nf4_dequantize — bf16 weights from NF4 storage ("a ideia": dequantised to
 * BFloat16 at use).  w' = bf16(RN32(q[code] * RN32(e4m3(c8) * s2))), two
 * separate roundings.  Writes exactly numel bf16 values.  numel == 0 is a
 * no-op; numel >= 2^37 returns QLORA_ERR_SHAPE (the output is written
 * through a 2-D tensor map of numel/64 rows).  All pointers 16-byte aligned.
 */
QLORA_API qlora_status nf4_dequantize(const uint8_t* codes, const uint8_t* c8, const float* s2,
                            int64_t numel, uint16_t* w_bf16, void* stream);

/*
 * Mean-centred double quantisation (a variant of "como funciona"'s FP8
 * encoding of the block constants; the pages do not centre, the original
 * NF4 scheme does).  The codes are those of nf4_quantize; the constants are
 * centred on their tensor mean before the FP8 step, which spends the FP8
 * sign bit on them and cuts the constants' error (about 2.8% -> 0.4% RMS on
 * N(0, 0.02) weights):
 *
 *   mean = fp32(S / nblocks), S = fp64 pairwise sum of the block constants
 *          c (zero-padded to a power of two, neighbouring pairs added level
 *          by level until one value is left);
 *   per group: c' = RN32(c - mean); s2 = RN32(max|c'| / 448);
 *          c8 = E4M3 round-to-nearest-even, saturating (RN32(c' / s2));
 *   dequantised constant: c_hat = RN32(RN32(e4m3(c8) * s2) + mean).
 *
 * nf4_quantize_centered writes codes, c8, s2 as nf4_quantize does plus the
 * fp32 `mean` (device float[1]); it runs the codes-and-constants kernel,
 * one or more pairwise-sum passes (one per factor of 2048 groups) and the
 * centred FP8 encoding, and needs a device workspace of
 * nf4_centered_workspace_size(numel) bytes (about 4 per block + 8 per group).
 * nf4_dequantize_centered is nf4_dequantize with c_hat as above.  Pass the
 * mean in nf4_weight.mean to run the GEMMs on such a weight.  Bit-exact with
 * the CPU oracle.  Other conventions as for nf4_quantize / nf4_dequantize.
 */
QLORA_API size_t nf4_centered_workspace_size(int64_t numel);
QLORA_API qlora_status nf4_quantize_centered(const uint16_t* w_bf16, int64_t numel, uint8_t* codes, uint8_t* c8,
                                             float* s2, float* mean, void* ws, size_t ws_bytes, int32_t* d_status,
                                             void* stream);
QLORA_API qlora_status nf4_dequantize_centered(const uint8_t* codes, const uint8_t* c8, const float* s2,
                                               const float* mean, int64_t numel, uint16_t* w_bf16, void* stream);

/*
 * qlora_linear_fwd — Y = X W'^T + s (X A^T) B^T with W' dequantised inside the
 * tensor-core GEMM (the bf16 weight never reaches global memory).
 *
 *  X      [M, K] bf16;  W: NF4 weight with n_out = N, k_in = K
 *  A      [r, K] bf16;  B [N, r] bf16;  s scalar (alpha / r)
 *  Y      [M, N] out, bf16 or fp32 per y_dtype
 *  U_out  [M, r] fp32 out: U = X A^T, to be passed back to qlora_linear_bwd
 *  ws     device workspace of at least qlora_fwd_workspace_size(M, N, K, r) bytes
 *
 * Constraints: M >= 0 (0 = no-op), K % 64 == 0, N % 64 == 0, K >= 64,
 * N >= 64, M < 2^31, N*K < 2^40, r % 16 == 0 and 16 <= r <= 256 (ranks
 * above 64 run their rank-r products as chunks of 64).  The grouped calls
 * with more than one member take r <= 64.
 * Accuracy: fp32 accumulation over exact bf16 inputs; relative Frobenius
 * error of Y within 2e-3 of the fp64 product on the same dequantised weights.
 */
QLORA_API qlora_status qlora_linear_fwd(const uint16_t* X, int64_t M, nf4_weight W, const uint16_t* A,
                              const uint16_t* B, int32_t r, float s, void* Y, int32_t y_dtype,
                              float* U_out, void* ws, size_t ws_bytes, int32_t* d_status,
                              void* stream);

/*
 * qlora_linear_bwd — gradients through the frozen NF4 weight into the adapters.
 *
 *  dY [M, N] bf16; X [M, K] bf16; U [M, r] fp32 (from qlora_linear_fwd)
 *  dX [M, K] out (bf16 or fp32 per dx_dtype) = dY W' + (s dY B) A
 *  dA [r, K] fp32 out = (s dY B)^T X;  dB [N, r] fp32 out = s dY^T U
 *  ws device workspace of at least qlora_bwd_workspace_size(M, N, K, r) bytes
 *
 * Same constraints as the forward.  dA and dB are overwritten (not
 * accumulated); their reductions over tokens run in a fixed order, so repeated
 * calls give bitwise-identical results.
 */
QLORA_API qlora_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, const float* U, int64_t M,
                              nf4_weight W, const uint16_t* A, const uint16_t* B, int32_t r,
                              float s, void* dX, int32_t dx_dtype, float* dA, float* dB, void* ws,
                              size_t ws_bytes, int32_t* d_status, void* stream);

/* Workspace sizes in bytes (0 when M == 0).  Pure host functions. */
QLORA_API size_t qlora_fwd_workspace_size(int64_t M, int64_t N, int64_t K, int32_t r);
QLORA_API size_t qlora_bwd_workspace_size(int64_t M, int64_t N, int64_t K, int32_t r);

/*
 * Grouped projections: several linears that read the same input X — the q, k
 * and v projections of an attention layer, or the gate and up projections of
 * its MLP — run as one forward and one backward call ("QLoRA" entry, "como
 * funciona": adapters on every linear layer; grouping the ones that share an
 * input reads X once and gives its gradient summed).  The G members (1..4)
 * are stacked along the output dimension:
 *
 *   W        one NF4 weight [N, K], N = sum of the members' n_member[g]: the
 *            NF4 storage of the members' rows one after another (each
 *            n_member[g] a multiple of 128, of 64 when G = 1).  nf4_quantize
 *            of the stacked bf16 weight produces it; when every member holds
 *            a whole number of double-quantisation groups (n_member[g] * K a
 *            multiple of 16384) it is also the members' own storages back to
 *            back;
 *   A        [G r, K] bf16: member g's adapter A_g in rows g r .. g r + r - 1;
 *   B        [N, r]   bf16: member g's B_g in the member's rows;
 *   Y, dY    [M, N]: member g's outputs in its columns;
 *   U        [M, G r] fp32: U_g = X A_g^T in columns g r .. g r + r - 1;
 *   dA, dB   [G r, K] and [N, r] fp32, stacked like A and B;
 *   dX       [M, K] = sum over the members of (dY_g W_g' + s (dY_g B_g) A_g),
 *            the gradient of the shared input.
 *
 * Every member uses the same r and s.  Per member the results are those of
 * qlora_linear_fwd / qlora_linear_bwd on that member alone (same accuracy);
 * dX is accumulated over all members in one fp32 accumulator.  n_member is a
 * host array of G sizes.  Constraints as for the single linear, plus
 * 1 <= G <= 4 and the member sizes above (QLORA_ERR_SHAPE; a NULL n_member is
 * QLORA_ERR_NULL).  Workspaces: qlora_group_{fwd,bwd}_workspace_size(M, N,
 * K, G, r) bytes (with G = 1 the same as the single linear's).
 */
QLORA_API size_t qlora_group_fwd_workspace_size(int64_t M, int64_t N, int64_t K, int32_t members, int32_t r);
QLORA_API size_t qlora_group_bwd_workspace_size(int64_t M, int64_t N, int64_t K, int32_t members, int32_t r);
QLORA_API qlora_status qlora_group_fwd(const uint16_t* X, int64_t M, nf4_weight W, int32_t members,
                                       const int64_t* n_member, const uint16_t* A, const uint16_t* B, int32_t r,
                                       float s, void* Y, int32_t y_dtype, float* U_out, void* ws, size_t ws_bytes,
                                       int32_t* d_status, void* stream);
QLORA_API qlora_status qlora_group_bwd(const uint16_t* dY, const uint16_t* X, const float* U, int64_t M,
                                       nf4_weight W, int32_t members, const int64_t* n_member, const uint16_t* A,
                                       const uint16_t* B, int32_t r, float s, void* dX, int32_t dx_dtype, float* dA,
                                       float* dB, void* ws, size_t ws_bytes, int32_t* d_status, void* stream);

/*
 * LoRA dropout on the adapter input ("Tutorial fine-tuning LLM LoRA/QLoRA
 * 2026", "Mão na Massa": the adapter configuration's lora_dropout; where it
 * acts is this library's reading).  The frozen path sees X, the adapter sees
 * X_drop:
 *
 *   forward:   X_drop = dropout(X);  U = X_drop A^T;  Y = X W'^T + s U B^T
 *   backward:  dU = s dY B;  dX = dY W' + keep * c * (dU A);
 *              dA = dU^T X_drop;  dB = s dY^T U
 *
 * Mask: Philox-4x32-10 (Salmon et al., SC 2011) with key (seed mod 2^32,
 * seed div 2^32) and counter (g mod 2^32, g div 2^32, 0, 0) for the group g of
 * four consecutive elements of the flattened [M, K] X; word i decides element
 * 4g + i, kept when below T = floor((1 - p) 2^32) (all kept for p = 0).  A kept
 * element is bf16(RN32(x * c)) with c = fp32(1 / (1 - p)), a dropped one +0.
 *
 * qlora_linear_fwd_dropout writes X_drop [M, K] bf16 (caller-owned; keep it for
 * the backward) and then runs the forward with X_drop as the adapter's input;
 * its workspace is qlora_fwd_workspace_size.  qlora_linear_bwd_dropout takes
 * X_drop (X itself is not needed) and the same p and seed, and needs
 * qlora_bwd_dropout_workspace_size bytes (the plain backward's plus an fp32
 * [M, K] buffer for dX's frozen-path term).  0 <= p < 1, else QLORA_ERR_SHAPE;
 * everything else as for qlora_linear_fwd / qlora_linear_bwd.
 */
QLORA_API size_t qlora_bwd_dropout_workspace_size(int64_t M, int64_t N, int64_t K, int32_t r);
QLORA_API qlora_status qlora_linear_fwd_dropout(const uint16_t* X, int64_t M, nf4_weight W, const uint16_t* A,
                                                const uint16_t* B, int32_t r, float s, float p, uint64_t seed,
                                                uint16_t* X_drop, void* Y, int32_t y_dtype, float* U_out, void* ws,
                                                size_t ws_bytes, int32_t* d_status, void* stream);
QLORA_API qlora_status qlora_linear_bwd_dropout(const uint16_t* dY, const uint16_t* X_drop, const float* U,
                                                int64_t M, nf4_weight W, const uint16_t* A, const uint16_t* B,
                                                int32_t r, float s, float p, uint64_t seed, void* dX,
                                                int32_t dx_dtype, float* dA, float* dB, void* ws, size_t ws_bytes,
                                                int32_t* d_status, void* stream);

/*
 * qlora_linear_fwd_noalloc — the forward of qlora_linear_fwd for callers that
 * cannot provide a workspace.  The pages have no counterpart; it exists for
 * callers that may not allocate device memory at call time: a plugin that a
 * host framework hands only its input and output buffers (the framework owns
 * the device memory pool), or a latency-critical loop that must not call
 * cudaMalloc/cudaFree because they can synchronise the device.
 *
 * Same arguments, constraints, results and accuracy as qlora_linear_fwd
 * (Y and U_out are caller-owned device buffers), minus the workspace: the
 * scratch lives in a 16 MiB array of device memory declared statically by
 * the library, which every GPU that loads the library holds until the process
 * exits.  The library allocates nothing here.
 *  - Limit: problems whose qlora_fwd_workspace_size(M, N, K, r) exceeds
 *    16 MiB (16777216 bytes) are rejected with QLORA_ERR_WORKSPACE before any
 *    work is enqueued (e.g. 4096 tokens on 4096x4096 with r=64 fits).
 *  - Set-up: the first call on each device (with that device current) looks
 *    up the array's device address with cudaGetSymbolAddress and caches it;
 *    make that first call before any stream capture.
 *  - Sharing: every call on a device uses the same array and leaves its last
 *    contents behind (nothing in it needs to start at zero).  Calls whose
 *    executions overlap on the GPU (different streams, or concurrent host
 *    threads) race on the array and give undefined results; serialise them.
 */
QLORA_API qlora_status qlora_linear_fwd_noalloc(const uint16_t* X, int64_t M, nf4_weight W,
                                                const uint16_t* A, const uint16_t* B, int32_t r,
                                                float s, void* Y, int32_t y_dtype, float* U_out,
                                                int32_t* d_status, void* stream);

/*
 * nf4_levels — the 16 fp32 NF4 levels the kernels use, ascending (code i ->
 * out[i]; out[7] == 0).  Host-only, needs no device.  The library derives
 * them itself from the standard-normal quantile construction of "como
 * funciona" (outermost probability (1-1/30 + 1-1/32)/2, the reading also used
 * by the CPU oracle), by bisection on the normal CDF in double precision.
 */
QLORA_API void nf4_levels(float out[16]);

/*
 * Kernel timing (diagnostics).  While enabled, every kernel this library
 * launches is bracketed by a pair of CUDA events recorded on the launch
 * stream (the events are library-owned host objects; no device memory is
 * allocated).  qlora_profile_collect waits for the recorded events, writes up
 * to `capacity` (kernel id, milliseconds) pairs in launch order, clears the
 * record list and returns the number of records (or -1 on a CUDA error).
 * qlora_kernel_name maps an id to a static name.  While enabled, the
 * backward's dB and dA kernels run on the caller's stream instead of beside
 * the dX GEMM, so each event pair times one kernel alone.  Not thread-safe
 * with respect to concurrent launches from several host threads.
 */
QLORA_API void qlora_profile_enable(int32_t enable);
QLORA_API int32_t qlora_profile_collect(int32_t* kernel_ids, float* ms, int32_t capacity);
QLORA_API const char* qlora_kernel_name(int32_t kernel_id);

/*
 * qlora_selftest_timeout — exercises the bounded waits every kernel uses
 * (diagnostics).  Launches one CTA of two warps that wait on a shared-memory
 * mbarrier that nothing completes, through the kernels' own wait functions
 * and their CTA abort flag, with a time limit of `limit_ns` nanoseconds
 * (1e3 .. 2e9) in place of the kernels' 2 s: warp 0 the way a producer or
 * MMA issuer waits (lane 0 polls), warp 1 the way the dequantiser warps wait
 * (every lane polls).  The first to run out ORs QLORA_DEV_TIMEOUT into
 * d_status[0] and raises the abort flag, on which the other gives up; each
 * warp whose wait gave up adds 1 to d_status[1] (so 2 is expected).
 * d_status is required: int32[2], zeroed by the caller.  The kernel returns
 * and the context stays usable; nothing faults, traps or hangs.  limit_ns out
 * of range returns QLORA_ERR_SHAPE.
 */
QLORA_API qlora_status qlora_selftest_timeout(int32_t* d_status, int64_t limit_ns, void* stream);

/*
 * qlora_set_few_token_threshold — which forward kernel runs for few tokens
 * (a performance setting; results are the same within the GEMM tolerances,
 * and the dequantised weight is bit-exact either way).  A forward (or a
 * group's) with M <= 16 token rows and a weight of at least
 * `min_weight_elems` elements (N x K, stacked outputs for a group) runs the
 * register-path few-token kernel; anything else with M <= 256 runs the
 * mid-size tensor-core kernel.  Default 2^26 elements, the measured
 * crossover on B200 (the few-token kernel streams large weights faster; on
 * smaller ones its fixed costs dominate).  0 selects the few-token kernel
 * for every M <= 16; INT64_MAX never.  Negative values count as 0.
 * Process-wide and thread-safe; it changes the workspace sizes of later
 * queries, so set it before querying (a call given a workspace smaller than
 * the current setting needs returns QLORA_ERR_WORKSPACE before anything is
 * enqueued).  Returns the previous value.
 */
QLORA_API int64_t qlora_set_few_token_threshold(int64_t min_weight_elems);

/* Static, NUL-terminated description of a status code. */
QLORA_API const char* qlora_strerror(qlora_status status);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
