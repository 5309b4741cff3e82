"""Seeded synthetic inputs for the QLoRA NF4 linear layer.

This module only draws random numbers and names workload shapes; it holds
none of the method's arithmetic.  It is the one module shared by the CPU
oracle's tests and the GPU path's tests and benchmark.

Every tensor is drawn in fp32 from a seeded ``torch.Generator`` and rounded
to bf16 (torch's round-to-nearest-even cast).  ``N(0, sigma)`` means standard
deviation ``sigma``.  The pages' own workloads (LLaMA-7B and 65B finetuning on
public datasets) are stood in for by these synthetic tensors of the same
shapes; no dataset or trained weight is used.

Workloads (one linear = W [out, in], LoRA A [r, in], B [out, r]):

* ``c1``: one 512x512 linear, 64 tokens, r=16, alpha=16 (s=1);
  W ~ N(0, 0.02), A ~ N(0, 1/512), B ~ N(0, 0.01), X, dY ~ N(0, 1); seed 0.
* ``c2``: LLaMA-7B attention projection 4096x4096, 4 x 1024 tokens, r=64,
  alpha=16 (s=0.25); A ~ N(0, 1/in).
* ``c3``: LLaMA-7B MLP gate/up 4096->11008 and down 11008->4096, 8192
  tokens, r=64, alpha=16; W has 0.1% of its elements (each independently)
  replaced by +-10 sigma with the sign of the draw.
* ``c4``: the seven linears of a LLaMA-7B decoder layer (q, k, v, o
  4096x4096; gate, up 4096->11008; down 11008->4096), 8 x 2048 tokens.
* ``c5``: 65B-shaped sweep, 80 layers of hidden 8192 / intermediate 22016;
  forward over M in {1, 16, 128, 2048, 16384} on the 8192->22016 and
  22016->8192 shapes, r=64.
"""

from dataclasses import dataclass

import torch

W_STD = 0.02
B_STD = 0.01
OUTLIER_P = 0.001
OUTLIER_SIGMAS = 10.0


@dataclass(frozen=True)
class Linear:
    name: str
    n_out: int
    k_in: int


@dataclass(frozen=True)
class Workload:
    name: str
    linears: tuple
    m_tokens: int
    r: int
    alpha: float
    outliers: bool = False

    @property
    def s(self):
        return self.alpha / self.r


LLAMA7B_LAYER = (
    Linear("q", 4096, 4096), Linear("k", 4096, 4096), Linear("v", 4096, 4096),
    Linear("o", 4096, 4096), Linear("gate", 11008, 4096),
    Linear("up", 11008, 4096), Linear("down", 4096, 11008),
)

WORKLOADS = {
    "c1": Workload("c1", (Linear("proj", 512, 512),), 64, 16, 16.0),
    "c2": Workload("c2", (Linear("q", 4096, 4096),), 4 * 1024, 64, 16.0),
    "c3": Workload("c3", (Linear("gate", 11008, 4096), Linear("up", 11008, 4096),
                          Linear("down", 4096, 11008)), 8192, 64, 16.0, True),
    "c4": Workload("c4", LLAMA7B_LAYER, 8 * 2048, 64, 16.0),
}

C5_HIDDEN = 8192
C5_INTER = 22016
C5_LAYERS = 80
C5_M = (1, 16, 128, 2048, 16384)
C5_SHAPES = (Linear("up", C5_INTER, C5_HIDDEN), Linear("down", C5_HIDDEN, C5_INTER))


def c5_layer_linears():
    """The seven linear shapes of one 65B-shaped decoder layer."""
    h, i = C5_HIDDEN, C5_INTER
    return (Linear("q", h, h), Linear("k", h, h), Linear("v", h, h), Linear("o", h, h),
            Linear("gate", i, h), Linear("up", i, h), Linear("down", h, i))


def _gen(seed, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std, seed, device="cpu"):
    """bf16 tensor of N(0, std) draws from a generator seeded with ``seed``."""
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (x * std).to(torch.bfloat16)


def weight_bf16(n_out, k_in, seed, outliers=False, device="cpu", std=W_STD):
    """Frozen base weight [n_out, k_in] ~ N(0, std), optionally with outliers."""
    g = _gen(seed, device)
    w = torch.randn((n_out, k_in), generator=g, device=device, dtype=torch.float32) * std
    if outliers:
        hit = torch.rand((n_out, k_in), generator=g, device=device) < OUTLIER_P
        w = torch.where(hit, torch.sign(w) * (OUTLIER_SIGMAS * std), w)
    return w.to(torch.bfloat16)


def linear_inputs(lin, m_tokens, r, seed, outliers=False, device="cpu"):
    """All inputs of one adapter-augmented linear: W, X, dY, A, B (bf16).

    Each tensor gets its own seed derived from ``seed`` so that the draws do
    not depend on the order in which tensors are requested.
    """
    base = int(seed) * 1000
    return {
        "W": weight_bf16(lin.n_out, lin.k_in, base + 1, outliers, device),
        "X": normal_bf16((m_tokens, lin.k_in), 1.0, base + 2, device),
        "dY": normal_bf16((m_tokens, lin.n_out), 1.0, base + 3, device),
        "A": normal_bf16((r, lin.k_in), 1.0 / lin.k_in, base + 4, device),
        "B": normal_bf16((lin.n_out, r), B_STD, base + 5, device),
    }


def dp_shard_inputs(lin, m_per_rank, r, rank, seed=0, outliers=False, device="cpu"):
    """Data-parallel inputs: every rank holds the same frozen weight and
    adapters (drawn with ``seed``) and its own batch of tokens (drawn with a
    seed derived from ``rank``)."""
    shared = linear_inputs(lin, 1, r, seed, outliers, device)
    own = linear_inputs(lin, m_per_rank, r, seed + 1 + rank, outliers, device)
    return {"W": shared["W"], "A": shared["A"], "B": shared["B"], "X": own["X"], "dY": own["dY"]}


def workload_inputs(name, index=0, seed=0, device="cpu", m_tokens=None):
    """Inputs of linear ``index`` of workload ``name`` (seed offset per linear)."""
    wl = WORKLOADS[name]
    lin = wl.linears[index]
    m = wl.m_tokens if m_tokens is None else m_tokens
    d = linear_inputs(lin, m, wl.r, seed * 100 + index, wl.outliers, device)
    d.update(r=wl.r, s=wl.s, n_out=lin.n_out, k_in=lin.k_in, m=m)
    return d


def bf16_bits(t):
    """bf16 torch tensor -> numpy uint16 bit patterns (host copy)."""
    import numpy as np
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def random_bf16_bits(shape, seed, std=1.0):
    """Convenience: seeded N(0, std) draws as numpy bf16 bit patterns."""
    return bf16_bits(normal_bf16(shape, std, seed))


# Which input each linear of the decoder layer reads: q, k and v read the
# same normalised hidden state, gate and up the same MLP input; o reads the
# attention output and down the MLP activation.
LAYER_INPUT_OF = ("attn", "attn", "attn", "o", "mlp", "mlp", "down")
LAYER_INPUT_WIDTH = {"attn": 4096, "o": 4096, "mlp": 4096, "down": 11008}


def decoder_layer_params(r, seed=0, device="cpu", linears=LLAMA7B_LAYER):
    """Frozen weights and adapters of one decoder layer's linears, the same on
    every data-parallel rank: a list of {"W", "A", "B"} (bf16), in layer
    order.  W ~ N(0, 0.02), A ~ N(0, 1/in) (std), B ~ N(0, 0.01)."""
    base = int(seed) * 1000
    out = []
    for i, lin in enumerate(linears):
        out.append({"W": weight_bf16(lin.n_out, lin.k_in, base + 10 * i + 1, device=device),
                    "A": normal_bf16((r, lin.k_in), 1.0 / lin.k_in, base + 10 * i + 2, device),
                    "B": normal_bf16((lin.n_out, r), B_STD, base + 10 * i + 3, device)})
    return out


def decoder_layer_activations(m_tokens, rank=0, seed=0, device="cpu", linears=LLAMA7B_LAYER):
    """One rank's batch for the layer's linears: the four distinct inputs
    {"attn", "o", "mlp", "down"} [m, in] and one upstream gradient per
    linear [m, out], all N(0, 1) bf16, drawn from seeds derived from ``rank``."""
    base = (int(seed) + 1 + int(rank)) * 100000
    X = {name: normal_bf16((m_tokens, width), 1.0, base + j, device)
         for j, (name, width) in enumerate(LAYER_INPUT_WIDTH.items())}
    dY = [normal_bf16((m_tokens, lin.n_out), 1.0, base + 100 + i, device) for i, lin in enumerate(linears)]
    return X, dY
