"""GPU parity of gdn_chunk_bwd_gva (grouped value heads: Hv value heads reading Hk q/k heads)
against the fp64 oracle (oracle/grouped.py backward_gva, pinned by finite differences in
tests/test_oracle_grouped_backward.py): dense and varlen, G = 2 and 3, with and without S0 and
dS_final, value head sizes 64 and 128.  Bound as the plain backward: max |g - g_ref| <= 1e-5 * (1 + max |g_ref|) per tensor."""
import numpy as np
import pytest
import torch

import workloads
from oracle import grouped
from tests.parity import f64

pytestmark = pytest.mark.gpu
RTOL = 1e-5


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def check(inp, seed, with_dsf=True):
    import linear_attention_sequence_rule_b200 as gdn
    g = torch.Generator().manual_seed(seed)
    lead = inp["v"].shape[:-1]
    dout = torch.randn(*lead, inp["dv"], generator=g).to(inp["v"].dtype)
    dsf = torch.randn(inp["B"], inp["H"], inp["dk"], inp["dv"], generator=g).float() if with_dsf else None
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    got = gdn.chunk_bwd_gva(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dout.cuda(), S0=d["S0"],
                            dS_final=None if dsf is None else dsf.cuda(), cu_seqlens=d["cu_seqlens"])
    gdn.device_status()
    ref = grouped.backward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], dout, dsf,
                               cu_seqlens=inp["cu_seqlens"])
    errs = {}
    for name, a, b in zip(("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"), got, ref):
        a = f64(a)
        errs[name] = float(np.max(np.abs(a - b)) / (1.0 + np.max(np.abs(b)))) if a.size else 0.0
    assert max(errs.values()) <= RTOL, errs


def test_dense_groups_of_three():
    check(workloads.make_gva_chunk_inputs(B=2, T=300, Hk=2, Hv=6, dk=64, dv=64, dtype="bf16", seed=81, s0_std=0.1,
                                          la_scale=0.3), 1)


def test_varlen_groups_of_two_fp32():
    check(workloads.make_gva_chunk_inputs(Hk=2, Hv=4, dk=64, dv=64, dtype="f32", seed=82,
                                          lengths=[1, 64, 0, 130, 7]), 2, with_dsf=False)


def test_dense_groups_of_two_value_head_128():
    check(workloads.make_gva_chunk_inputs(B=2, T=150, Hk=1, Hv=2, dk=64, dv=128, dtype="bf16", seed=83, s0_std=0.1,
                                          la_scale=0.3), 3)
