"""The decode steps under CUDA-graph capture: a captured sequence of steps,
replayed, gives bit for bit what the same calls give eagerly (the library
launches only on the stream it is given and does nothing else a capture
forbids)."""
import pytest
import torch

import rwkv_wkv_recurrence_b200 as rw
import wkv_inputs as wi

pytestmark = pytest.mark.gpu


def _replay_equals_eager(cuda_device, run):
    # run(state) issues the steps on the current stream and returns the outputs
    s_eager, s_graph = run.init(), run.init()
    y_eager = run(s_eager)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run(run.init())  # warm-up on a side stream, as capture requires
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        y_graph = run(s_graph)
    s_graph.copy_(run.init())
    g.replay()
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(y_eager, y_graph))
    assert torch.equal(s_eager, s_graph)


def test_wkv4_step_graph(cuda_device):
    B, C, T = 64, 256, 8
    p = {k: v.to(cuda_device) for k, v in wi.wkv4_problem(B, T, C, 61).items()}
    ks = [p["k"][:, t].contiguous() for t in range(T)]
    vs = [p["v"][:, t].contiguous() for t in range(T)]
    _, s0 = rw.rwkv_wkv4_forward(p["w"], p["u"], p["k"], p["v"], return_state=True)

    def run(state):
        return [rw.rwkv_wkv4_step(p["w"], p["u"], ks[t], vs[t], state, stream=torch.cuda.current_stream())
                for t in range(T)]

    run.init = lambda: s0.clone()
    _replay_equals_eager(cuda_device, run)


@pytest.mark.parametrize("finch", [False, True])
def test_matrix_state_step_graph(cuda_device, finch):
    B, H, T = 8, 4, 8
    gen = wi.wkv6_problem if finch else wi.wkv5_problem
    p = {k: v.to(cuda_device) for k, v in gen(B, T, H, 64, seed=62).items()}
    names = ("r", "k", "v", "omega") if finch else ("r", "k", "v")
    toks = [{n: p[n][:, t].contiguous() for n in names} for t in range(T)]
    fwd = rw.rwkv_wkv6_forward if finch else rw.rwkv_wkv5_forward
    _, s0 = fwd(**p, return_state=True)

    def run(state):
        out = []
        for t in range(T):
            if finch:
                y, _ = rw.rwkv_wkv6_step(**toks[t], u=p["u"], state=state, state_out=state,
                                         stream=torch.cuda.current_stream())
            else:
                y, _ = rw.rwkv_wkv5_step(**toks[t], omega=p["omega"], u=p["u"], state=state, state_out=state,
                                         stream=torch.cuda.current_stream())
            out.append(y)
        return out

    run.init = lambda: s0.clone()
    _replay_equals_eager(cuda_device, run)


@pytest.mark.parametrize("finch", [False, True])
@pytest.mark.parametrize("with_state", [False, True])
def test_matrix_state_forward_and_backward_graph(cuda_device, with_state, finch):
    # the Eagle forward and backward (whose reversed forward pass runs on a side stream, forked
    # and joined with events), or the Finch forward and backward (four launches), captured in one
    # graph, replayed: bit for bit the eager results
    B, T, H = 2, 150, 3
    gen = wi.wkv6_problem if finch else wi.wkv5_problem
    p = {k: v.to(cuda_device) for k, v in gen(B, T, H, 64, seed=63).items()}
    g = {k: v.to(cuda_device) for k, v in wi.wkv5_grads(B, T, H, 64, seed=64, states=with_state).items()}
    fwd = rw.rwkv_wkv6_forward if finch else rw.rwkv_wkv5_forward
    bwd = rw.rwkv_wkv6_backward if finch else rw.rwkv_wkv5_backward

    def run():
        y = fwd(p["r"], p["k"], p["v"], p["omega"], p["u"], g.get("s_in"), stream=torch.cuda.current_stream())
        grads = bwd(p["r"], p["k"], p["v"], p["omega"], p["u"], g["gy"], g.get("s_in"), g.get("gs_out"),
                    want_gs_in=True, stream=torch.cuda.current_stream())
        return (y,) + tuple(grads)

    eager = run()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()  # warm-up on a side stream, as capture requires
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        captured = run()
    graph.replay()
    torch.cuda.synchronize()
    rw.rwkv_check_device_error()
    for a, b in zip(eager, captured):
        assert torch.equal(a, b)
