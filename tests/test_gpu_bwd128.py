"""GPU parity of gdn_chunk_bwd at key head size 128 (two 64-column key blocks) against the fp64
backward oracle (oracle.backward, pinned by finite differences): dense and varlen (ragged, empty
and one-token sequences), exact resets on chunk boundaries, beta up to 2, with and without S0 and
dS_final, bf16 and fp32 inputs, value head sizes 64 and 128, and grouped value heads.  Bound as the
dk = 64 backward: max |g - g_ref| <= 1e-5 * (1 + max |g_ref|) per tensor."""
import numpy as np
import pytest
import torch

import workloads
from oracle import grouped
from tests.test_gpu_bwd import RTOL, check

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


@pytest.mark.parametrize("dtype,dv", [("bf16", 128), ("f32", 64)])
def test_dense(dtype, dv):
    inp = workloads.make_chunk_inputs(B=2, T=200, H=2, dk=128, dv=dv, dtype=dtype, seed=41 + dv, s0_std=0.1,
                                      la_scale=0.3)
    check(inp, 11)


def test_varlen_ragged_resets_beta_two():
    inp = workloads.make_chunk_inputs(H=2, dk=128, dv=64, dtype="bf16", seed=42, s0_std=0.05,
                                      lengths=[1, 65, 0, 130, 64, 7], beta_scale=2.0, la_std=2.0)
    inp["log_alpha"][66 + 64, 1] = -float("inf")  # first token of a chunk
    inp["log_alpha"][66 + 63, 0] = -float("inf")  # last token of a chunk
    check(inp, 12)
    check(inp, 13, with_dsf=False)


def test_grouped_value_heads():
    import linear_attention_sequence_rule_b200 as gdn
    from tests.parity import f64
    inp = workloads.make_gva_chunk_inputs(B=2, T=150, Hk=1, Hv=2, dk=128, dv=64, dtype="bf16", seed=43,
                                          s0_std=0.1, la_scale=0.3)
    g = torch.Generator().manual_seed(14)
    dout = torch.randn(*inp["v"].shape, generator=g).to(inp["v"].dtype)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    got = gdn.chunk_bwd_gva(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dout.cuda(), S0=d["S0"])
    gdn.device_status()
    ref = grouped.backward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], dout)
    for a, b in zip(got, ref):
        a = f64(a)
        assert float(np.max(np.abs(a - b)) / (1.0 + np.max(np.abs(b)))) <= RTOL
