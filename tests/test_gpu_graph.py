"""The forward captured in a CUDA graph (the way a model's step is often
replayed) gives bit-identical results to the eager call, for the tcgen05 and
SIMT kernel families, gated and closed, including the programmatic
dependent launches between its kernels."""
import pytest
import torch

from rank_latent_attention_mixer_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,path", [("bf16", 0), ("f16", 0), ("f32", 0), ("bf16", 1)])
@pytest.mark.parametrize("gated", [True, False])
def test_graph_replay_matches_eager(dtype, path, gated):
    from rank_latent_attention_mixer_b200 import binding as b
    x = W.random_inputs(2, 4, 3000, 128, 32, dtype=dtype, seed=21)
    d = {k: t.cuda() for k, t in x.items()}
    dt = b._dtype_code(d["k"])
    ws = torch.empty(b.workspace_bytes(2, 4, 3000, 128, 32, dt, gated, path), dtype=torch.uint8, device="cuda")
    y_eager = b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"] if gated else None, d["k0"], d["k"], d["v"],
                          path=path, workspace=ws)
    y = torch.empty_like(y_eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):          # warm-up outside capture, on the capture stream
        b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"] if gated else None, d["k0"], d["k"], d["v"], y,
                    path=path, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    y.zero_()
    with torch.cuda.graph(g):
        b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"] if gated else None, d["k0"], d["k"], d["v"], y,
                    path=path, workspace=ws)
    for _ in range(3):
        y.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    assert torch.equal(y, y_eager)
    # new inputs in the same buffers flow through the replay
    d["v"].mul_(-1.0)
    g.replay()
    y2 = b.mixer_fwd(d["q0"], d["q_fixed"], d["gate"] if gated else None, d["k0"], d["k"], d["v"], path=path,
                     workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


@pytest.mark.parametrize("dtype,path", [("bf16", 0), ("f32", 0), ("bf16", 1)])
def test_backward_graph_replay_matches_eager(dtype, path):
    """The backward, and a training step (forward with saved state, then the
    backward from it), captured in one CUDA graph each, replay bit-identically
    to the eager calls."""
    from rank_latent_attention_mixer_b200 import binding as b
    x = W.random_inputs(2, 2, 2000, 96, 64, dtype=dtype, seed=23)
    dy = W.random_cotangent((2, 2, 2000, 64), dtype, seed=123).cuda()
    d = {k: t.cuda() for k, t in x.items()}
    args = (d["q0"], d["q_fixed"], d["gate"], d["k0"], d["k"], d["v"], dy)
    dt = b._dtype_code(d["k"])
    ws = torch.empty(b.bwd_workspace_bytes(2, 2, 2000, 96, 64, dt, path), dtype=torch.uint8, device="cuda")
    g_eager = b.mixer_bwd(*args, path=path, workspace=ws)
    y_eager, ctx = b.mixer_fwd_train(*args[:6], path=path)
    g_ctx_eager = b.mixer_bwd(*args, path=path, workspace=ws, ctx=ctx, y=y_eager)
    out = {k: torch.empty_like(t) for k, t in g_eager.items()}
    out_ctx = {k: torch.empty_like(t) for k, t in g_eager.items()}
    y = torch.empty_like(y_eager)
    ctx2 = torch.empty_like(ctx)
    fws = torch.empty(b.workspace_bytes(2, 2, 2000, 96, 64, dt, True, path), dtype=torch.uint8, device="cuda")

    def step():
        b.mixer_bwd(*args, path=path, workspace=ws, out=out)
        b.mixer_fwd_train(*args[:6], y, ctx=ctx2, path=path, workspace=fws)
        b.mixer_bwd(*args, path=path, workspace=ws, out=out_ctx, ctx=ctx2, y=y)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):          # warm-up outside capture, on the capture stream
        step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        for t in list(out.values()) + list(out_ctx.values()):
            t.zero_()
        graph.replay()
    torch.cuda.synchronize()
    assert b.check_device_status() == 0
    for name in g_eager:
        assert torch.equal(out[name], g_eager[name]), name
        assert torch.equal(out_ctx[name], g_ctx_eager[name]), name + " (saved state)"
    assert torch.equal(y, y_eager)
