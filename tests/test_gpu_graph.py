"""The library's calls can be captured in one CUDA graph (no allocation, no
host synchronisation, programmatic launches and the side-stream fork/join
included); a replay reproduces an eager step bit for bit."""

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("M,N,K,r", [(64, 512, 512, 16), (12, 1024, 2048, 64), (700, 512, 1024, 32)])
def test_graph_replay_matches_eager(M, N, K, r, few_token_kernel):
    import bit_nf4_quantized_26_b200 as lib
    dev = torch.device("cuda")
    g = {k: v.to(dev) for k, v in synth.linear_inputs(synth.Linear("g", N, K), M, r, 3).items()}
    s = 16.0 / r
    nc, nb, ns = lib.nf4_sizes(N * K)
    codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    c8 = torch.empty(nb, dtype=torch.uint8, device=dev)
    s2 = torch.empty(ns, dtype=torch.float32, device=dev)
    W = lib.NF4Weight(codes, c8, s2, N, K)
    out = {"Y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
           "U": torch.empty((M, r), dtype=torch.float32, device=dev),
           "dX": torch.empty((M, K), dtype=torch.bfloat16, device=dev),
           "dA": torch.empty((r, K), dtype=torch.float32, device=dev),
           "dB": torch.empty((N, r), dtype=torch.float32, device=dev)}
    ws_f = torch.empty(max(lib.qlora_fwd_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(max(lib.qlora_bwd_workspace_size(M, N, K, r), 16), dtype=torch.uint8, device=dev)

    def step():
        lib.nf4_quantize(g["W"].reshape(-1), codes, c8, s2)
        lib.qlora_linear_fwd(g["X"], W, g["A"], g["B"], s, Y=out["Y"], U=out["U"], ws=ws_f)
        lib.qlora_linear_bwd(g["dY"], g["X"], out["U"], W, g["A"], g["B"], s, dX=out["dX"], dA=out["dA"],
                             dB=out["dB"], ws=ws_b)

    cs = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(cs):
        step()
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in out.items()}
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cs):
        step()
    for v in out.values():
        v.fill_(0)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    for k in out:
        assert torch.equal(_bits(out[k]), _bits(ref[k])), k
    del graph
