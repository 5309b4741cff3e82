"""Failure detection without a GPU fault: the bounded waits every kernel uses
(lane 0 polling for a warp, and every lane polling) run out against a barrier
that nothing completes; the first reports QLORA_DEV_TIMEOUT in the device
status word and raises the CTA's abort flag, the other gives up on the flag,
and the context stays usable."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_26_b200 as q
import synth
from oracle import nf4

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    q.qlora_selftest_timeout(status, 5_000_000)  # 5 ms limit
    torch.cuda.synchronize()
    assert int(status[0]) & q.DEV_TIMEOUT
    assert int(status[1]) == 2  # both waiting warps gave up
    # the same context still runs kernels correctly
    w = synth.weight_bf16(64, 512, seed=2).cuda()
    W = q.quantize_weight(w)
    torch.cuda.synchronize()
    codes, c8, s2 = nf4.quantize(synth.bf16_bits(w.cpu()).reshape(-1))
    assert np.array_equal(W.codes.cpu().numpy(), codes)
    assert np.array_equal(W.c8.cpu().numpy(), c8)


def test_status_untouched_without_timeout():
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    w = synth.weight_bf16(64, 512, seed=3).cuda()
    q.nf4_quantize(w.reshape(-1), status=status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
