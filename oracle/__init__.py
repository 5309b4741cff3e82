"""CPU oracle for the QLoRA NF4 linear layer — TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct statement of what the
GPU library computes.  It exists so that tests can check the CUDA path
against it.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import it; the product path (the C-ABI library and
its Python binding) never imports, links or executes anything here, and this
package never imports the product.  The two share no code: the only module
both sides use is ``synth`` (seeded random inputs, no method arithmetic).

Sources (web pages; cited by title and section):

* "QLoRA" encyclopedia entry (tonho.wtf), sections "a ideia" and
  "como funciona": 4-bit storage type built from standard-normal quantiles,
  made asymmetric so that zero is exact; absmax normalisation to [-1, 1];
  blocks of 64 elements with one constant each; the constants double-quantised
  to FP8 in blocks of 256; BF16 compute with dequantisation at use; LoRA
  adapters in 16 bit receive the only gradients.
* "Tutorial fine-tuning LLM LoRA/QLoRA 2026" (nexusinovation), section
  "LoRA: O Padrão Ouro de Eficiência": W' = W + alpha*A*B, and the
  ``LoraConfig``/``BitsAndBytesConfig`` knobs and the ``paged_adamw_8bit``
  trainer in "Mão na Massa".
* "QLoRA" encyclopedia entry, section "como funciona", third piece: optimizer
  states paged between GPU and CPU memory (unified memory).

Modules:

* :mod:`oracle.numerics` — bf16 and FP8 E4M3 encodings from their definitions.
* :mod:`oracle.nf4` — codebook, blockwise quantisation, double quantisation,
  dequantisation (encodings: the GPU must match these bit for bit).
* :mod:`oracle.linear` — forward / backward of the adapter-augmented linear in
  fp64 (the GPU must match within a relative Frobenius error).
* :mod:`oracle.optim` — the adapter optimizer step, AdamW with 8-bit blockwise
  FP8 states (every operation one fp32 rounding: the GPU must match bit for
  bit).
* :mod:`oracle.dropout` — LoRA dropout on the adapter input with a
  Philox-4x32-10 mask (the GPU must match X_drop bit for bit and the
  products within the GEMM tolerances).
* :mod:`oracle.dq_centered` — double quantisation with mean centring, for an
  error ablation against the plain scheme (no CUDA path).

Parity status per function is listed in each module header.  Every function
here is pinned by ``tests/test_oracle_*.py`` to facts the pages or
mathematics fix; functions whose pin is partial say so.
"""

from . import numerics, nf4, linear, optim, dropout, dq_centered  # noqa: F401
