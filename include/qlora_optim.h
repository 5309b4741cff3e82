/*
 * qlora_optim.h — C ABI of the adapter optimizer step: AdamW with 8-bit
 * states kept in paged (CUDA managed) memory.
 *
 * Sources (web pages, cited by title and section):
 *  - "QLoRA" encyclopedia entry (tonho.wtf), section "como funciona", third
 *    piece: the optimizer states live in NVIDIA unified memory; when the GPU
 *    runs short they are evicted to CPU RAM and brought back for the update.
 *  - "Tutorial fine-tuning LLM LoRA/QLoRA 2026" (nexusinovation), section
 *    "Mão na Massa": the trainer's optimizer is a paged 8-bit AdamW
 *    (learning rate 2e-4 in the listing).
 *
 * The pages fix neither the update nor the 8-bit format.  This library's
 * reading: AdamW (decoupled weight decay) with bias correction; the state of
 * each parameter tensor is the E4M3 code of the first moment m and of the
 * square root u = sqrt(v) of the second moment, with one fp32 absmax scale per
 * 256 elements for each — the same two-level FP8 scheme as the NF4 constants.
 * Every operation is one fp32 operation rounded to nearest even, in this
 * order (bit-exact with the library's CPU reference):
 *
 *   m  = RN(e4m3(m8) s_m)      u = RN(e4m3(u8) s_u)      v = RN(u u)
 *   m1 = RN(RN(b1 m) + RN((1-b1) g))
 *   v1 = RN(RN(b2 v) + RN((1-b2) RN(g g)))          u1 = sqrt_RN(v1)
 *   d  = RN(RN(m1 bc1) / RN(RN(u1 bc2) + eps));      d = RN(d + RN(wd p))
 *   p1 = RN(p - RN(lr d)), stored as bf16 (RNE)
 *
 * with 1-b computed in fp32 and bc1 = fp32(1/(1-b1^t)), bc2 =
 * fp32(1/sqrt(1-b2^t)) computed in fp64 (t = step).  Per 256-element block the
 * new state is s_m = RN(max|m1| / 448), m8 = E4M3_RNE_satfinite(RN(m1 / s_m))
 * (0 when s_m = 0; a code that rounds to zero is +0), and the same for u1.
 *
 * Conventions as in qlora_nf4.h: asynchronous on `stream`; 16-byte aligned
 * pointers (QLORA_ERR_ALIGN); d_status bit QLORA_DEV_NONFINITE for a
 * non-finite gradient (the affected outputs are then unspecified); errors are
 * reported before any work is enqueued.
 */
#ifndef QLORA_OPTIM_H
#define QLORA_OPTIM_H

#include "qlora_nf4.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * qlora_adamw8_step — one AdamW step over n parameters, in place.
 *
 *  p        [n] bf16 parameters (device or managed memory), updated
 *  grad     [n] fp32 gradients (e.g. dA or dB of qlora_linear_bwd)
 *  m8, u8   [n] uint8 E4M3 state codes, updated (all zero before step 1)
 *  m_scale, u_scale  [ceil(n/256)] fp32 state scales, updated (zero before step 1)
 *  lr, beta1, beta2, eps, weight_decay   hyper-parameters (finite; 0 <= beta < 1,
 *           eps >= 0)
 *  step     1-based step count t used by the bias corrections
 *
 * n == 0 is a no-op.  n < 0, n >= 2^40, step < 1 or a hyper-parameter outside
 * its range returns QLORA_ERR_SHAPE.  State buffers may live in memory from
 * qlora_paged_alloc; the kernel reads and writes them in place wherever they
 * currently reside (pages evicted to the host migrate back on access).
 */
QLORA_API qlora_status qlora_adamw8_step(uint16_t* p, const float* grad, uint8_t* m8, uint8_t* u8,
                                         float* m_scale, float* u_scale, int64_t n, float lr, float beta1,
                                         float beta2, float eps, float weight_decay, int64_t step,
                                         int32_t* d_status, void* stream);

/*
 * Paged memory for optimizer states: CUDA managed memory whose preferred
 * location is the current device, so it stays in HBM until the device runs
 * short and is then evicted to host RAM and migrated back when touched.
 * These are the only library calls that allocate; the caller owns the
 * allocation and releases it with qlora_paged_free (after the work that uses
 * it has completed).
 *
 *  qlora_paged_alloc     *ptr = managed allocation of `bytes` (> 0), zero-filled
 *  qlora_paged_prefetch  asynchronously migrates [ptr, ptr+bytes) to the
 *                        current device (to_host = 0) or to host RAM
 *                        (to_host != 0) on `stream`; a hint, not required
 *                        for correctness
 *  qlora_paged_free      releases an allocation from qlora_paged_alloc
 */
QLORA_API qlora_status qlora_paged_alloc(void** ptr, size_t bytes);
QLORA_API qlora_status qlora_paged_prefetch(const void* ptr, size_t bytes, int32_t to_host, void* stream);
QLORA_API qlora_status qlora_paged_free(void* ptr);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_OPTIM_H */
