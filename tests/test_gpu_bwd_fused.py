"""GPU parity of gdn_chunk_bwd_fused (gradients of the fused-prologue forward with respect to the
raw projections) against the fp64 oracle (oracle/prologue.py backward_fused, pinned by finite
differences in tests/test_oracle_prologue_backward.py), on the same seeded raw inputs: dense and
varlen, bf16 and fp32 inputs, an exact reset (a = +inf), b_scale 1 and 2, with and without S0 and
dS_final, value head sizes 64, 128 and 256.

The prologue and the recurrence's backward run in fp32 on the stored input values (the oracle
reads the same values in fp64), so the bound is the plain backward's: max |g - g_ref| <= 1e-5 *
(1 + max |g_ref|) per tensor."""
import numpy as np
import pytest
import torch

import workloads
from oracle import prologue
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
    got = gdn.chunk_bwd_fused(d["q_raw"], d["k_raw"], d["v"], d["a_raw"], d["b_raw"], dout.cuda(), inp["a_scale"],
                              inp["b_scale"], S0=d["S0"], dS_final=None if dsf is None else dsf.cuda(),
                              cu_seqlens=d["cu_seqlens"])
    gdn.device_status()
    ref = prologue.backward_fused(inp["q_raw"], inp["k_raw"], inp["v"], inp["a_raw"], inp["b_raw"], inp["S0"], dout,
                                  inp["a_scale"], inp["b_scale"], dS_final=dsf, cu_seqlens=inp["cu_seqlens"])
    errs = {}
    for name, a, b in zip(("dq_raw", "dk_raw", "dv", "da_raw", "db_raw", "dS0"), got, ref):
        a = f64(a)
        errs[name] = float(np.max(np.abs(a - b)) / (1.0 + np.max(np.abs(b)))) if a.size else 0.0
    assert max(errs.values()) <= RTOL, errs
    return errs


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense(dtype):
    inp = workloads.make_raw_chunk_inputs(B=2, T=300, H=3, dk=64, dv=64, dtype=dtype, seed=61, s0_std=0.1,
                                          la_scale=0.3)
    check(inp, 1)


def test_varlen_reset_and_beta_scale_two():
    inp = workloads.make_raw_chunk_inputs(H=2, dk=64, dv=64, dtype="bf16", seed=62, beta_scale=2.0, la_std=2.0,
                                          lengths=[1, 63, 64, 65, 0, 200, 7])
    inp["a_raw"][70, 1] = float("inf")  # log alpha = -inf: an exact reset
    errs = check(inp, 2, with_dsf=False)
    assert errs["da_raw"] <= RTOL


@pytest.mark.parametrize("dv,lengths", [(128, None), (256, [70, 0, 129])])
def test_value_heads_128_and_256(dv, lengths):
    kw = dict(lengths=lengths) if lengths else dict(B=2, T=150)
    inp = workloads.make_raw_chunk_inputs(H=2, dk=64, dv=dv, dtype="bf16", seed=63 + dv, s0_std=0.1, la_scale=0.3,
                                          **kw)
    check(inp, 3)
