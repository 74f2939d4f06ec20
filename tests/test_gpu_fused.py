"""GPU parity of gdn_chunk_fwd_fused (q/k normalisation and gate activations inside the kernel)
against the fp64 oracle applied to the same raw projections: oracle.prologue.forward_fused.
Cases cover both head sizes, varlen packs with ragged and empty sequences, exact resets
(a_raw = +inf), the beta range ends, the segment-scan path and the hybrid-LM workload at full size.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle import prologue
from tests.parity import TOL, f64, max_abs, unit_slices

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def run_fused(inp, S_final=True):
    import linear_attention_sequence_rule_b200 as gdn
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd_fused(d["q_raw"], d["k_raw"], d["v"], d["a_raw"], d["b_raw"], inp["a_scale"],
                                  inp["b_scale"], S0=d["S0"], cu_seqlens=d["cu_seqlens"],
                                  output_final_state=S_final)
    gdn.device_status()
    return out, Sf


def compare(inp, out, Sf, units=None):
    o_ref, s_ref = prologue.forward_fused(inp["q_raw"], inp["k_raw"], inp["v"], inp["a_raw"], inp["b_raw"],
                                          inp["S0"], inp["a_scale"], inp["b_scale"],
                                          cu_seqlens=inp["cu_seqlens"], units=units)
    og = f64(out)
    sg = f64(Sf) if Sf is not None else None
    if units is None:
        return max_abs(og, o_ref), (max_abs(sg, s_ref) if sg is not None else 0.0)
    e_o = e_s = 0.0
    for s, h, idx in unit_slices(inp, units):
        e_o = max(e_o, max_abs(og[idx], o_ref[idx]))
        if sg is not None:
            e_s = max(e_s, max_abs(sg[s, h], s_ref[s, h]))
    return e_o, e_s


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_small_dense(dk, dv):
    inp = workloads.make_raw_chunk_inputs(B=2, T=300, H=3, dk=dk, dv=dv, dtype="bf16", seed=dk + 3 * dv,
                                          s0_std=0.1, la_scale=0.3)
    e_o, e_s = compare(inp, *run_fused(inp))
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


@pytest.mark.parametrize("d", [64, 128])
def test_varlen_ragged_and_empty(d):
    inp = workloads.make_raw_chunk_inputs(H=2, dk=d, dv=d, dtype="bf16", seed=21, s0_std=0.05,
                                          lengths=[1, 63, 64, 65, 0, 200, 129, 7], beta_scale=2.0,
                                          la_std=2.0)
    out, Sf = run_fused(inp)
    e_o, e_s = compare(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)
    assert torch.equal(Sf[4].cpu(), inp["S0"][4])


def test_resets_and_beta_range_ends():
    inp = workloads.make_raw_chunk_inputs(B=1, T=257, H=2, dk=64, dv=64, dtype="bf16", seed=31,
                                          beta_scale=2.0, la_std=2.0)
    a, b = inp["a_raw"], inp["b_raw"]
    a[0, 5, 0] = float("inf")
    a[0, 64, 1] = float("inf")
    a[0, 200:203, 1] = float("inf")
    b[0, 10:20, 0] = -60.0   # beta -> 0
    b[0, 30:40, 1] = 60.0    # beta -> b_scale = 2
    out, Sf = run_fused(inp)
    assert torch.isfinite(out).all() and torch.isfinite(Sf).all()
    e_o, e_s = compare(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_segment_scan_path():
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_raw_chunk_inputs(B=1, T=81 * 64 - 45, H=2, dk=128, dv=128, dtype="bf16", seed=41,
                                          s0_std=0.05, la_scale=0.1)
    assert gdn.workspace_bytes(1, inp["T"], 2, 128, 128) > 0
    e_o, e_s = compare(inp, *run_fused(inp))
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_hybrid_lm_raw_full():
    inp = workloads.config_raw_inputs("hybrid_lm")
    e_o, e_s = compare(inp, *run_fused(inp))  # all 96 chains
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_varlen_raw_sampled_chains():
    inp = workloads.config_raw_inputs("varlen")
    out, Sf = run_fused(inp)
    units = sorted(np.random.default_rng(3).choice(inp["B"] * inp["H"], size=12, replace=False).tolist())
    e_o, e_s = compare(inp, out, Sf, units)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)
