"""The optional CTA-pair forward that keeps the dequantised weight tile in
tensor memory (selected with QLORA_TMEM_A=1, read once per process, so it
runs here in a child process): the dequantisation inside it bit-exact (one-hot
tokens, B = 0: Y is exactly W'^T) and the forward within the usual
tolerances, for plain and mean-centred constants, with 4 and 8 A slots."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import numpy as np, torch, synth
import bit_nf4_quantized_26_b200 as lib
from oracle import nf4, dq_centered as dqc, linear as ol
from tests._util import bits
N, K, M = 1024, 2048, 2048
for centred in (False, True):
    w = synth.weight_bf16(N, K, seed=11, outliers=True)
    wb = bits(w).reshape(-1)
    if centred:
        rc, r8, rs2, rm = dqc.quantize_centered(wb)
        ref = dqc.dequantize_centered(rc, r8, rs2, rm, N * K).reshape(N, K)
        W = lib.quantize_weight_centered(w.cuda())
    else:
        rc, r8, rs2 = nf4.quantize(wb)
        ref = nf4.dequantize(rc, r8, rs2, N * K).reshape(N, K)
        W = lib.quantize_weight(w.cuda())
    A = synth.normal_bf16((64, K), 1.0 / K, seed=2).cuda()
    B0 = torch.zeros((N, 64), dtype=torch.bfloat16, device="cuda")
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    X[torch.arange(M, device="cuda"), torch.arange(M, device="cuda") % K] = 1.0
    Y, _ = lib.qlora_linear_fwd(X, W, A, B0, 0.25, y_dtype=1)
    torch.cuda.synchronize()
    want = (ref[:, np.arange(M) % K].T.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(Y.cpu().numpy(), want), "dequantised tile differs"
    d = synth.linear_inputs(synth.Linear("t", N, K), 700, 64, 3)
    g = {k: v.cuda() for k, v in d.items()}
    Y, U = lib.qlora_linear_fwd(g["X"], W, g["A"], g["B"], 0.25)
    torch.cuda.synchronize()
    _, Yr = ol.linear_fwd(bits(d["X"]), ref, bits(d["A"]), bits(d["B"]), 0.25)
    assert ol.rel_frobenius(Y.float().cpu().numpy(), Yr) <= 2e-3
print("ok")
'''


@pytest.mark.parametrize("slots", ["4", "8"])
def test_tensor_memory_forward(slots):
    env = dict(os.environ, QLORA_TMEM_A="1", QLORA_TMEM_A_SLOTS=slots, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-2000:]
