"""GPU parity of the grouped-value-head entries (gdn_chunk_fwd_gva, gdn_decode_step_gva) against
the fp64 oracle oracle.grouped: both head sizes, both dtypes (bf16 runs on the tensor cores, fp32
on the CUDA-core chunk kernel), varlen, the segment-scan path, and decode steps."""
import numpy as np
import pytest
import torch

import workloads
from oracle import grouped
from tests.parity import TOL, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def run_check(inp, tol):
    import linear_attention_sequence_rule_b200 as gdn
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd_gva(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"],
                                cu_seqlens=d["cu_seqlens"])
    gdn.device_status()
    o_ref, s_ref = grouped.forward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                                       cu_seqlens=inp["cu_seqlens"])
    e_o, e_s = max_abs(f64(out), o_ref), max_abs(f64(Sf), s_ref)
    assert e_o <= tol and e_s <= tol, (e_o, e_s)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Hk,Hv", [(1, 2), (2, 8)])
def test_dense(dtype, d, Hk, Hv):
    inp = workloads.make_gva_chunk_inputs(B=2, T=200, Hk=Hk, Hv=Hv, dk=d, dv=d, dtype=dtype, seed=Hv + d,
                                          s0_std=0.1, la_scale=0.3)
    run_check(inp, TOL[dtype])


def test_varlen_ragged():
    inp = workloads.make_gva_chunk_inputs(Hk=2, Hv=6, dk=64, dv=128, dtype="bf16", seed=5, s0_std=0.05,
                                          lengths=[1, 63, 64, 65, 0, 200, 7], beta_scale=2.0, la_std=2.0)
    run_check(inp, TOL["bf16"])


def test_segment_scan_path():
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_gva_chunk_inputs(B=1, T=64 * 64 + 17, Hk=1, Hv=2, dk=128, dv=128, dtype="bf16",
                                          seed=6, s0_std=0.05, la_scale=0.1)
    assert gdn.workspace_bytes(1, inp["T"], 2, 128, 128) > 0
    run_check(inp, TOL["bf16"])


def test_hybrid_lm_shape_with_groups_of_two():
    inp = workloads.make_gva_chunk_inputs(B=8, T=4096, Hk=6, Hv=12, dk=64, dv=64, dtype="bf16", seed=7,
                                          la_scale=0.1)
    run_check(inp, TOL["bf16"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_steps(dtype):
    import linear_attention_sequence_rule_b200 as gdn
    N, Hk, Hv, dk, dv = 3, 2, 6, 128, 64
    g = torch.Generator().manual_seed(8)
    S = (0.05 * torch.randn(N, Hv, dk, dv, generator=g)).float()
    S_dev = S.cuda()
    S_ref = S.double().numpy()
    e_o = 0.0
    for step in range(30):
        inp = workloads.make_gva_chunk_inputs(B=N, T=1, Hk=Hk, Hv=Hv, dk=dk, dv=dv, dtype=dtype,
                                              seed=100 + step, la_scale=0.3)
        one = {k: inp[k][:, 0] for k in ("q", "k", "v", "log_alpha", "beta")}
        d = {k: v.cuda() for k, v in one.items()}
        out = gdn.decode_step_gva(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S_dev)
        o_ref, S_ref = grouped.decode_step_gva(one["q"], one["k"], one["v"], one["log_alpha"], one["beta"], S_ref)
        e_o = max(e_o, max_abs(f64(out), o_ref))
    gdn.device_status()
    e_s = max_abs(f64(S_dev), S_ref)
    assert e_o <= TOL[dtype] and e_s <= TOL[dtype], (e_o, e_s)
