"""GPU parity of gdn_phase_fwd (the complex-phase delta memory on the chunk kernels) against the
fp64 phase oracle (oracle/phase.py, pinned in tests/test_oracle_phase.py), on the same seeded
inputs: dense and varlen (ragged, empty and one-token sequences), unit and Laplace (|K| < 1)
keys, beta up to 2, with and without M0, both key sizes and both value sizes, bf16 and fp32.

Bounds (max-abs on outputs and on the final state's real and imaginary parts, each tensor against
its own scale): fp32 1e-4 * max(1, max |ref|), as the real fp32 path; bf16 2e-2 * max(1, max |ref|),
the real bf16 path's 2e-2 taken relative.  bf16 rounding errors scale with the values rounded:
the real workloads' states stay near 1, while the state here is M itself, whose entries reach
5-10 (values enter the real recurrence as lam sqrt(dk) V), so an absolute 2e-2 would ask the
phase state for several times the real path's relative accuracy.  The bf16 path also rounds the
rescaled keys, queries and values to bf16 (relative 2^-9 each) while the oracle reads the fp32
phasors.  Observed: outputs 0.5-1.3e-2 at |o| <= 1.7; states 0.4-0.6 % of max |M|."""
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


def check(inp):
    import linear_attention_sequence_rule_b200 as gdn
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Mf = gdn.phase_fwd(d["K"], d["Q"], d["v"], d["log_lam"], d["beta"], M0=d["M0"], cu_seqlens=d["cu_seqlens"])
    gdn.device_status()
    o_ref, M_ref = phase.forward(inp["K"], inp["Q"], inp["v"], inp["log_lam"], inp["beta"], inp["M0"],
                                 cu_seqlens=inp["cu_seqlens"])
    tol = TOL[inp["dtype"]]
    Mf = Mf.cpu().to(torch.complex128).numpy()
    pairs = ((f64(out), o_ref), (Mf.real, M_ref.real), (Mf.imag, M_ref.imag))
    errs = tuple(max_abs(a, b) / max(1.0, float(np.abs(b).max())) for a, b in pairs)
    assert max(errs) <= tol, errs
    assert np.abs(o_ref).max() > 0.1  # the check is not vacuous
    return errs


@pytest.mark.parametrize("dk,dv", [(32, 64), (64, 64), (64, 128), (32, 128), (32, 256), (64, 256)])
def test_dense_bf16_with_initial_state(dk, dv):
    check(workloads.make_phase_inputs(B=2, T=300, H=3, dk=dk, dv=dv, dtype="bf16", seed=500 + dk + dv, m0_std=0.05))


@pytest.mark.parametrize("dk", [32, 64])
def test_dense_fp32_laplace_keys(dk):
    check(workloads.make_phase_inputs(B=2, T=200, H=2, dk=dk, dv=64, dtype="f32", seed=510 + dk, m0_std=0.05,
                                      laplace=True, la_scale=1.0))


def test_varlen_ragged_beta_two():
    check(workloads.make_phase_inputs(H=2, dk=64, dv=64, dtype="bf16", seed=520, beta_scale=2.0,
                                      lengths=[0, 1, 63, 64, 65, 200, 7, 130]))


def test_hybrid_lm_size():
    # the benchmark's phase workload: B=8, T=4096, H=12, dk=32 complex (64 real), dv=64
    check(workloads.make_phase_inputs(B=8, T=4096, H=12, dk=32, dv=64, dtype="bf16", seed=530))
