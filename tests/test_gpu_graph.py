"""The layer's forward (prologue + GEMM, two C-ABI calls) in a CUDA graph and in interleaved
streams of calls.

A captured forward replays the same two launches with the same tensor maps, so a replay
on new inputs written into the captured input buffer must give the eager call's output
bit for bit, with a clean device error word.  The prologue -> GEMM launch keeps its
programmatic dependency inside the graph.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")


def _layer(fmt, M, K, N, rank, seed):
    from bit_w4a4_quantized_group_b200 import prepare as P
    from bit_w4a4_quantized_group_b200.layer import W4A4LowRankLinear
    rng = np.random.default_rng(seed)
    prep = {"lam": rng.uniform(0.5, 4.0, K).astype(np.float32),
            "R_nk": (rng.standard_normal((N, K)) * 0.02).astype(np.float32),
            "L1_rk": (rng.standard_normal((rank, K)) * 0.05).astype(np.float32),
            "L2_nr": (rng.standard_normal((N, rank)) * 0.05).astype(np.float32),
            "act_gscale": 1.0}
    bias = (rng.standard_normal(N) * 0.1).astype(np.float32)
    dev = torch.device("cuda", 0)
    return W4A4LowRankLinear(fmt, N, K, P.pack(fmt, prep), prep["lam"], 1.0, bias, device=dev)


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "int4", "w8a8"])
@pytest.mark.parametrize("M,K,N,rank", [(256, 3072, 1024, 32), (300, 640, 640, 16), (1024, 2048, 512, 0)])
def test_forward_replays_from_a_cuda_graph(fmt, M, K, N, rank):
    from bit_w4a4_quantized_group_b200 import binding as B
    lin = _layer(fmt, M, K, N, rank, seed=M + K + N + rank)
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev).manual_seed(M * 31 + K)
    X = (torch.randn(M, K, device=dev, generator=gen) * 3).to(torch.bfloat16)
    Y = torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev)
    # warm-up outside the capture (workspace allocation, launch-configuration caches)
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        lin.forward(X, Y)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lin.forward(X, Y)
    for i in range(3):
        Xn = (torch.randn(M, K, device=dev, generator=gen) * (1.0 + i)).to(torch.bfloat16)
        X.copy_(Xn)
        g.replay()
        Y_eager = lin.forward(Xn.clone())
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), Y_eager.view(torch.int16)), f"replay {i}"
    st, site = B.svdq_get_last_device_error(None)
    assert st == B.SVDQ_OK, (st, site)
    del g


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "w8a8"])
def test_interleaved_calls_of_two_layers_keep_stream_order(fmt):
    """Prologue A, prologue B, GEMM A, GEMM B on one stream.  Each GEMM may start its set-up
    under the kernel just before it (here the other layer's prologue) and must still read
    its own, completed prologue outputs: Y equals the plain sequential calls bit for bit."""
    from bit_w4a4_quantized_group_b200 import binding as B
    dev = torch.device("cuda", 0)
    la = _layer(fmt, 512, 2048, 1024, 32, seed=11)
    lb = _layer(fmt, 256, 2048, 1024, 16, seed=12)
    gen = torch.Generator(device=dev).manual_seed(5)
    Xa = (torch.randn(512, 2048, device=dev, generator=gen) * 2).to(torch.bfloat16)
    Xb = (torch.randn(256, 2048, device=dev, generator=gen) * 2).to(torch.bfloat16)
    Ya_ref = la.forward(Xa)
    Yb_ref = lb.forward(Xb)
    torch.cuda.synchronize()
    Ya = torch.empty_like(Ya_ref)
    Yb = torch.empty_like(Yb_ref)
    for _ in range(3):
        la.prologue_only(Xa)
        lb.prologue_only(Xb)
        la.gemm_only(512, Ya)
        lb.gemm_only(256, Yb)
    torch.cuda.synchronize()
    assert torch.equal(Ya.view(torch.int16), Ya_ref.view(torch.int16))
    assert torch.equal(Yb.view(torch.int16), Yb_ref.view(torch.int16))
    st, site = B.svdq_get_last_device_error(None)
    assert st == B.SVDQ_OK, (st, site)
