"""The library's calls under CUDA-graph capture (torch.cuda.graph, which captures on its own stream;
the binding launches on the current stream): captured decode steps and a captured chunk forward,
replayed, give results bit-identical to the same calls made eagerly, and a second replay from the
same starting state repeats them.  Each entry is called once eagerly before capture, so that
one-time setup happens outside it."""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _dev(x):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}


def test_decode_steps_replayed_from_a_graph():
    import linear_attention_sequence_rule_b200 as gdn
    N, H, d, steps = 16, 8, 128, 6
    xs = [_dev(workloads.make_decode_step_inputs(N, H, d, d, "bf16", seed=7, step=s)) for s in range(steps)]
    S0 = workloads.make_decode_state(N, H, d, d, seed=7).cuda()
    S_e = S0.clone()
    outs_e = [gdn.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_e).clone() for x in xs]
    S_g = S0.clone()
    outs_g = [torch.empty_like(o) for o in outs_e]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for x, o in zip(xs, outs_g):
            gdn.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S_g, out=o)
    for _ in range(2):
        S_g.copy_(S0)
        graph.replay()
        torch.cuda.synchronize()
        for a, b in zip(outs_g, outs_e):
            assert torch.equal(a, b)
        assert torch.equal(S_g, S_e)
    gdn.device_status()


def test_chunk_forward_replayed_from_a_graph():
    import linear_attention_sequence_rule_b200 as gdn
    inp = _dev(workloads.make_chunk_inputs(B=2, T=300, H=4, dk=64, dv=64, dtype="bf16", seed=8, s0_std=0.05))
    out_e, S_e = gdn.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=inp["S0"])
    out_g = torch.empty_like(out_e)
    S_g = torch.empty_like(S_e)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        gdn.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S0=inp["S0"], out=out_g,
                      S_final=S_g)
    for _ in range(2):
        out_g.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_g, out_e)
        assert torch.equal(S_g, S_e)
    gdn.device_status()
