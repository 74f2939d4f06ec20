"""GPU parity of gdn_phase_rowdecay_fwd (the complex-phase memory with one decay per value
channel, the Laplace core's diag(r_t)) against the fp64 oracle ``oracle.phase.forward_rowdecay``
(pinned in tests/test_oracle_phase.py), on the same seeded inputs: dense and varlen (empty,
one-token and chunk-boundary sequences), unit and Laplace keys, beta up to 2, strong per-channel
decays, with and without M0, in-place carry, both key sizes, channel counts that do not fill a
warp's channel groups, bf16 and fp32 values.

Bounds as the scalar phase memory's (max-abs per tensor against max(1, max |ref|)): fp32 1e-4,
bf16 2e-2.  The arithmetic is fp32 on both paths; the bf16 path rounds only the values read and
the outputs written."""
import numpy as np
import pytest
import torch

import workloads
from oracle import phase
from tests.parity import TOL, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def check(inp, in_place=False):
    import linear_attention_sequence_rule_b200 as gdn
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    if in_place and d["M0"] is not None:
        M = torch.view_as_real(d["M0"]).contiguous()
        out, Mf = gdn.phase_rowdecay_fwd(d["K"], d["Q"], d["v"], d["log_r"], d["beta"], M0=M,
                                         cu_seqlens=d["cu_seqlens"], M_final=M)
    else:
        out, Mf = gdn.phase_rowdecay_fwd(d["K"], d["Q"], d["v"], d["log_r"], d["beta"], M0=d["M0"],
                                         cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    o_ref, M_ref = phase.forward_rowdecay(inp["K"], inp["Q"], inp["v"], inp["log_r"], inp["beta"], inp["M0"],
                                          cu_seqlens=inp["cu_seqlens"])
    tol = TOL[inp["dtype"]]
    Mf = Mf.cpu().to(torch.complex128).numpy()
    pairs = ((f64(out), o_ref), (Mf.real, M_ref.real), (Mf.imag, M_ref.imag))
    errs = tuple(max_abs(a, b) / max(1.0, float(np.abs(b).max())) for a, b in pairs)
    assert max(errs) <= tol, errs
    assert np.abs(o_ref).max() > 0.1  # the check is not vacuous
    return errs


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(32, 64), (64, 64), (32, 6), (64, 130)])
def test_dense_with_initial_state(dtype, dk, dv):
    check(workloads.make_phase_rowdecay_inputs(B=2, T=300, H=3, dk=dk, dv=dv, dtype=dtype, seed=600 + dk + dv,
                                               m0_std=0.05, beta_scale=2.0, la_scale=0.5))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_varlen_laplace_strong_decays(dtype):
    inp = workloads.make_phase_rowdecay_inputs(H=2, dk=32, dv=64, dtype=dtype, seed=610, beta_scale=2.0,
                                               la_scale=1.0, lr_std=2.0, m0_std=0.1, laplace=True,
                                               lengths=[0, 1, 63, 64, 65, 200, 7, 130])
    inp["log_r"][3, 1, 5] = -30.0   # a near-reset of one channel
    check(inp)


def test_channels_differ_and_scalar_case_agrees():
    # with equal decays on every channel the per-channel kernel equals the scalar phase memory
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_phase_rowdecay_inputs(B=2, T=150, H=2, dk=32, dv=64, dtype="f32", seed=620, m0_std=0.05)
    inp["log_r"] = inp["log_lam"][..., None].expand(*inp["log_lam"].shape, 64).contiguous()
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    o1, M1 = gdn.phase_rowdecay_fwd(d["K"], d["Q"], d["v"], d["log_r"], d["beta"], M0=d["M0"])
    o2, M2 = gdn.phase_fwd(d["K"], d["Q"], d["v"], d["log_lam"], d["beta"], M0=d["M0"])
    torch.cuda.synchronize()
    scale = max(1.0, float(o2.abs().max()))
    assert float((o1 - o2).abs().max()) <= 1e-4 * scale
    assert float((M1 - M2).abs().max()) <= 1e-4 * max(1.0, float(M2.abs().max()))


def test_in_place_carry():
    check(workloads.make_phase_rowdecay_inputs(B=2, T=100, H=2, dk=64, dv=64, dtype="bf16", seed=630, m0_std=0.1),
          in_place=True)


def test_hybrid_lm_size():
    # the benchmark's per-channel-decay workload: B=8, T=4096, H=12, dk=32 complex, dv=64
    check(workloads.make_phase_rowdecay_inputs(B=8, T=4096, H=12, dk=32, dv=64, dtype="bf16", seed=640))
