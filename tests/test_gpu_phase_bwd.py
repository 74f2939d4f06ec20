"""GPU parity of gdn_phase_bwd (gradients of the complex-phase delta memory, dk = 32 complex,
dv = 64, 128 and 256) against the fp64 phase backward oracle (oracle/phase.py backward, pinned by finite
differences of the complex definition in tests/test_oracle_phase.py): dense and varlen, bf16 and
fp32 values, unit and Laplace keys, with and without M0 and dM_final.  The backward runs in fp32
on the stored inputs, so the bound is the plain backward's: max |g - g_ref| <= 1e-5 *
(1 + max |g_ref|) per tensor (real and imaginary parts separately)."""
import numpy as np
import pytest
import torch

import workloads
from oracle import phase
from tests.parity import f64

pytestmark = pytest.mark.gpu
RTOL = 1e-5


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _parts(x):
    x = x.detach().cpu()
    if x.is_complex():
        x = x.to(torch.complex128).numpy()
        return [x.real, x.imag]
    return [f64(x)]


def check(inp, seed, with_dm=True):
    import linear_attention_sequence_rule_b200 as gdn
    g = torch.Generator().manual_seed(seed)
    lead = inp["v"].shape[:-1]
    dout = torch.randn(*lead, inp["dv"], generator=g).to(inp["v"].dtype)
    dMf = None
    if with_dm:
        dMf = torch.complex(torch.randn(inp["B"], inp["H"], inp["dv"], inp["dk"], generator=g),
                            torch.randn(inp["B"], inp["H"], inp["dv"], inp["dk"], generator=g))
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    got = gdn.phase_bwd(d["K"], d["Q"], d["v"], d["log_lam"], d["beta"], dout.cuda(), M0=d["M0"],
                        dM_final=None if dMf is None else dMf.cuda(), cu_seqlens=d["cu_seqlens"])
    gdn.device_status()
    ref = phase.backward(inp["K"], inp["Q"], inp["v"], inp["log_lam"], inp["beta"], inp["M0"], dout, dMf,
                         cu_seqlens=inp["cu_seqlens"])
    errs = {}
    for name, a, b in zip(("dK", "dQ", "dv", "dlog_lam", "dbeta", "dM0"), got, ref):
        b = [b.real, b.imag] if np.iscomplexobj(b) else [b]
        for i, (x, y) in enumerate(zip(_parts(a), b)):
            errs[f"{name}{i}"] = float(np.max(np.abs(x - y)) / (1.0 + np.max(np.abs(y)))) if x.size else 0.0
    assert max(errs.values()) <= RTOL, errs


def test_dense_bf16_with_states():
    check(workloads.make_phase_inputs(B=2, T=300, H=3, dk=32, dv=64, dtype="bf16", seed=601, m0_std=0.05), 1)


def test_dense_fp32_laplace_keys():
    check(workloads.make_phase_inputs(B=2, T=200, H=2, dk=32, dv=64, dtype="f32", seed=602, m0_std=0.05,
                                      laplace=True, la_scale=1.0), 2)


def test_varlen_ragged_beta_two():
    check(workloads.make_phase_inputs(H=2, dk=32, dv=64, dtype="bf16", seed=603, beta_scale=2.0,
                                      lengths=[0, 1, 63, 64, 65, 200, 7]), 3, with_dm=False)


def test_value_head_128_varlen():
    check(workloads.make_phase_inputs(H=2, dk=32, dv=128, dtype="bf16", seed=604, m0_std=0.05,
                                      lengths=[70, 0, 129, 1]), 4)


def test_value_head_256_dense_fp32():
    check(workloads.make_phase_inputs(B=1, T=150, H=2, dk=32, dv=256, dtype="f32", seed=605, m0_std=0.05), 5)
