"""GPU parity of gdn_chunk_fwd against the fp64 oracle (element by element, same seeded inputs).

Small cases span several 64-token chunks, a ragged tail, both head sizes, both dtypes, varlen
packs with empty / 1-token / boundary-length sequences, exact resets (log_alpha = -inf) and the
extreme gates beta = 0 and beta = 2.  The named workloads run at full size in the launch
configuration the benchmark times, with every (sequence, head) chain compared.
"""
import numpy as np
import pytest
import torch

import workloads
from tests.parity import TOL, compare_chunk, run_gpu_chunk, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def small(dtype, dk, dv, B=2, T=300, H=3, seed=0, s0=0.1, **kw):
    return workloads.make_chunk_inputs(B=B, T=T, H=H, dk=dk, dv=dv, dtype=dtype, seed=seed,
                                       s0_std=s0, **kw)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_small_dense(dtype, dk, dv):
    inp = small(dtype, dk, dv, seed=dk + dv)
    out, Sf = run_gpu_chunk(inp)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL[dtype] and e_s <= TOL[dtype], (e_o, e_s)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
def test_small_varlen_ragged(dtype, d):
    lengths = [1, 63, 64, 65, 0, 200, 129, 7]
    inp = workloads.make_chunk_inputs(H=2, dk=d, dv=d, dtype=dtype, seed=7, s0_std=0.05,
                                      lengths=lengths)
    out, Sf = run_gpu_chunk(inp)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL[dtype] and e_s <= TOL[dtype], (e_o, e_s)
    # the empty sequence keeps its initial state exactly
    assert torch.equal(Sf[4].cpu(), inp["S0"][4])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_resets_and_extreme_gates(dtype):
    inp = small(dtype, 64, 64, B=1, T=257, H=2, seed=11, beta_scale=2.0, la_std=2.0)
    la, be = inp["log_alpha"], inp["beta"]
    la[0, 5, 0] = -float("inf")
    la[0, 64, 1] = -float("inf")  # first token of a chunk
    la[0, 127, 0] = -float("inf")  # last token of a chunk
    la[0, 200:203, 1] = -float("inf")
    be[0, 10:20, 0] = 0.0
    be[0, 30:40, 1] = 2.0
    be[0, 256, :] = 2.0
    out, Sf = run_gpu_chunk(inp)
    assert torch.isfinite(out).all() and torch.isfinite(Sf).all()
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL[dtype] and e_s <= TOL[dtype], (e_o, e_s)


def test_zero_initial_state_and_no_final_state():
    inp = small("bf16", 64, 64, s0=0.0, seed=3)
    out, Sf = run_gpu_chunk(inp, S_final=False)
    assert Sf is None
    e_o, _ = compare_chunk(inp, out, None)
    assert e_o <= TOL["bf16"]


def test_in_place_state_carry():
    """S_final == S0 (same buffer) is allowed and equals the out-of-place result."""
    import linear_attention_sequence_rule_b200 as gdn
    inp = small("bf16", 128, 128, seed=5)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    S = d["S0"].clone()
    out1, Sf1 = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    out2, Sf2 = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=S, S_final=S)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(Sf1, S)


def test_split_with_carry_equals_single_call():
    import linear_attention_sequence_rule_b200 as gdn
    inp = small("bf16", 64, 64, B=2, T=320, seed=9)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    cut = 128
    sl = lambda t, a, b: t[:, a:b].contiguous()
    o1, s1 = gdn.chunk_fwd(sl(d["q"], 0, cut), sl(d["k"], 0, cut), sl(d["v"], 0, cut),
                           sl(d["log_alpha"], 0, cut), sl(d["beta"], 0, cut), S0=d["S0"])
    o2, s2 = gdn.chunk_fwd(sl(d["q"], cut, 320), sl(d["k"], cut, 320), sl(d["v"], cut, 320),
                           sl(d["log_alpha"], cut, 320), sl(d["beta"], cut, 320), S0=s1)
    torch.cuda.synchronize()
    assert max_abs(f64(torch.cat([o1, o2], 1)), f64(out)) <= 1e-2
    assert max_abs(f64(s2), f64(Sf)) <= 1e-2


def test_dense_equals_varlen_pack():
    import linear_attention_sequence_rule_b200 as gdn
    inp = small("bf16", 128, 128, B=3, T=200, seed=13)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    flat = lambda t: t.reshape(-1, *t.shape[2:]).contiguous()
    cu = torch.tensor([0, 200, 400, 600], dtype=torch.int32, device="cuda")
    out2, Sf2 = gdn.chunk_fwd(flat(d["q"]), flat(d["k"]), flat(d["v"]), flat(d["log_alpha"]),
                              flat(d["beta"]), S0=d["S0"], cu_seqlens=cu)
    torch.cuda.synchronize()
    assert torch.equal(flat(out), out2) and torch.equal(Sf, Sf2)


def test_decode_steps_equal_chunk_forward():
    import linear_attention_sequence_rule_b200 as gdn
    inp = small("f32", 64, 64, B=2, T=70, H=2, seed=17)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    S = d["S0"].clone()
    outs = []
    for t in range(70):
        outs.append(gdn.decode_step(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(),
                                    d["v"][:, t].contiguous(), d["log_alpha"][:, t].contiguous(),
                                    d["beta"][:, t].contiguous(), S))
    torch.cuda.synchronize()
    assert max_abs(f64(torch.stack(outs, 1)), f64(out)) <= 1e-4
    assert max_abs(f64(S), f64(Sf)) <= 1e-4


# ---- named workloads at full size ------------------------------------------------------------

def sample_units(n_units, k, seed):
    g = np.random.default_rng(seed)
    return sorted(g.choice(n_units, size=min(k, n_units), replace=False).tolist())


def test_tiny_full():
    inp = workloads.config_inputs("tiny")
    out, Sf = run_gpu_chunk(inp)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL["f32"] and e_s <= TOL["f32"], (e_o, e_s)


def test_hybrid_lm_full():
    inp = workloads.config_inputs("hybrid_lm")
    out, Sf = run_gpu_chunk(inp)
    e_o, e_s = compare_chunk(inp, out, Sf)  # all 96 chains
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_long_context_full_all_heads():
    """The long-context workload in full (segment scan, five launches): every head's outputs and
    final state against the oracle."""
    inp = workloads.config_inputs("long_context")
    out, Sf = run_gpu_chunk(inp)
    assert torch.isfinite(out).all() and torch.isfinite(Sf).all()
    e_o, e_s = compare_chunk(inp, out, Sf)  # all 16 heads
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_varlen_full_all_chains():
    """The varlen workload in full: all 512 (sequence, head) chains against the oracle."""
    inp = workloads.config_inputs("varlen")
    out, Sf = run_gpu_chunk(inp)
    assert torch.isfinite(out).all() and torch.isfinite(Sf).all()
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)
