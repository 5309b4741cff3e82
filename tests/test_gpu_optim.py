"""GPU parity of the adapter optimizer step (AdamW with 8-bit states in paged
memory) against the CPU oracle: parameters, state codes and state scales
bit for bit over several steps, for paged and device-resident states, with
states evicted to host RAM between steps, on ragged sizes."""

import numpy as np
import pytest
import torch

import bit_nf4_quantized_26_b200 as q
from oracle import numerics as nm
from oracle import optim

pytestmark = pytest.mark.gpu

HP = dict(lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _inputs(n, seed):
    g = torch.Generator().manual_seed(seed)
    p = (torch.randn(n, generator=g) * 0.02).to(torch.bfloat16)
    grads = [(torch.randn(n, generator=g) * 1e-3 * (1 + t)).float() for t in range(4)]
    return p, grads


def _run_both(n, paged, evict, seed=0, hp=HP, steps=4):
    p, grads = _inputs(n, seed)
    pd = p.cuda()
    st = q.AdamW8State(n, paged=paged)
    ref_p = p.view(torch.int16).numpy().view(np.uint16)
    ref_st = optim.init_state(n)
    for t in range(1, steps + 1):
        if evict:
            st.prefetch(to_host=True)
        q.qlora_adamw8_step(pd, grads[t - 1].cuda(), st, step=t, **hp)
        ref_p, ref_st = optim.adamw8_step(ref_p, grads[t - 1].numpy(), ref_st, hp["lr"], hp["beta1"], hp["beta2"],
                                          hp["eps"], hp["weight_decay"], t)
    torch.cuda.synchronize()
    got_p = pd.cpu().view(torch.int16).numpy().view(np.uint16)
    got_st = st.host_arrays()
    st.close()
    return got_p, got_st, ref_p, ref_st


@pytest.mark.parametrize("n", [1, 7, 255, 256, 257, 8 * 256 + 77, 3 * 65536 + 5])
@pytest.mark.parametrize("paged", [True, False])
def test_adamw8_matches_oracle(n, paged):
    got_p, got_st, ref_p, ref_st = _run_both(n, paged, evict=False)
    assert np.array_equal(got_p, ref_p)
    for g, r in zip(got_st, ref_st):
        assert np.array_equal(np.asarray(g).view(np.uint8), np.asarray(r).view(np.uint8))


@pytest.mark.parametrize("n", [4096 + 33, 1 << 20])
def test_adamw8_evicted_state_matches(n):
    """Paged states migrated to host RAM before every step give the same bits."""
    got_p, got_st, ref_p, ref_st = _run_both(n, paged=True, evict=True, seed=3)
    assert np.array_equal(got_p, ref_p)
    for g, r in zip(got_st, ref_st):
        assert np.array_equal(np.asarray(g).view(np.uint8), np.asarray(r).view(np.uint8))


def test_adamw8_hyperparameter_edges():
    """No weight decay and eps = 0; beta1 = 0 (no momentum)."""
    for hp in (dict(HP, weight_decay=0.0, eps=0.0), dict(HP, beta1=0.0), dict(HP, lr=1e-2, beta2=0.95)):
        got_p, got_st, ref_p, ref_st = _run_both(1000, paged=False, evict=False, seed=5, hp=hp)
        assert np.array_equal(got_p, ref_p)
        for g, r in zip(got_st, ref_st):
            assert np.array_equal(np.asarray(g).view(np.uint8), np.asarray(r).view(np.uint8))


def test_adamw8_nonfinite_gradient_sets_status():
    n = 1000
    p, grads = _inputs(n, 7)
    g = grads[0].clone()
    g[123] = float("inf")
    st = q.AdamW8State(n, paged=False)
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    q.qlora_adamw8_step(p.cuda(), g.cuda(), st, step=1, status=status, **HP)
    torch.cuda.synchronize()
    assert int(status[0]) & q.DEV_NONFINITE


def test_adamw8_on_linear_gradients():
    """The optimizer consumes dA / dB of the backward pass directly."""
    import synth
    d = {k: v.cuda() for k, v in synth.linear_inputs(synth.Linear("c1", 512, 512), 64, 16, 0).items()}
    W = q.quantize_weight(d["W"])
    Y, U = q.qlora_linear_fwd(d["X"], W, d["A"], d["B"], 1.0)
    dX, dA, dB = q.qlora_linear_bwd(d["dY"], d["X"], U, W, d["A"], d["B"], 1.0)
    for param, grad in ((d["A"], dA), (d["B"], dB)):
        n = param.numel()
        ref_p = param.cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1)
        ref_p, ref_st = optim.adamw8_step(ref_p, grad.cpu().numpy().reshape(-1), optim.init_state(n), HP["lr"],
                                          HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], 1)
        st = q.AdamW8State(n)
        pc = param.contiguous().view(-1)
        q.qlora_adamw8_step(pc, grad.contiguous().view(-1), st, step=1, **HP)
        torch.cuda.synchronize()
        assert np.array_equal(pc.cpu().view(torch.int16).numpy().view(np.uint16), ref_p)
        st.close()
