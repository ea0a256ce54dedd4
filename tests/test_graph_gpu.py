"""The C ABI under CUDA-graph capture: after one eager call has set up the
per-device state (RoPE table, kernel attributes), the training step (the
saving forward and the context backward) and a decode step can be captured
in a CUDA graph and replayed, with results equal to the eager calls."""
import pytest
import torch

import structured_sparse_attention_fibonacci_b200 as sa

DEV = "cuda"


@pytest.mark.gpu
def test_training_step_and_decode_replay_from_a_cuda_graph():
    shape = (2, 2, 2, 512, 64)
    g = torch.Generator(device="cpu").manual_seed(21)
    q, k, v, do = (torch.randn(shape, generator=g).to(torch.bfloat16).to(DEV) for _ in range(4))
    alpha = torch.tensor([0.8, 1.3], device=DEV)
    kw = dict(window=12)
    ctx = torch.empty(sa.context_size(shape, torch.bfloat16, **kw), dtype=torch.uint8, device=DEV)
    ws = torch.empty(sa.workspace_size(shape, torch.bfloat16, backward=True, **kw),
                     dtype=torch.uint8, device=DEV)
    o, lse = torch.empty_like(q), torch.empty(shape[:4], dtype=torch.float32, device=DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    dal = torch.empty(2, dtype=torch.float32, device=DEV)
    od = torch.empty(shape[:3] + shape[4:], dtype=torch.bfloat16, device=DEV)
    q1 = q[:, :, :, 400].contiguous()

    def step():
        sa.fwd(q, k, v, alpha, out=o, lse=lse, context=ctx, **kw)
        sa.bwd(q, k, v, o, lse, do, alpha, dq=dq, dk=dk, dv=dv, dalpha=dal, workspace=ws,
               context=ctx, **kw)
        sa.decode(q1, k, v, alpha, 400, out=od, lse=None, want_lse=False, **kw)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()                                  # eager: sets up the device state
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    eager = [t.clone() for t in (o, lse, dq, dk, dv, dal, od)]
    for t in (o, lse, dq, dk, dv, dal, od):
        t.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip((o, lse, dq, dk, dv, dal, od), eager):
        assert torch.equal(a, b)
    assert sa.device_error() == 0
