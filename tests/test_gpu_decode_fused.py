"""GPU parity of gdn_decode_step_fused (a decode step from raw projections: q/k normalisation and
the gate activations inside the step) against the fp64 oracle: oracle.prologue's l2_normalize and
gates (pinned in tests/test_oracle_prologue.py) followed by oracle.decode_step, step after step
with the state carried on each side.  Cases: both dtypes, dv 64 / 128 / 256, b_scale 1 and 2, an
exact reset (a = +inf), a zero key row, and agreement with the fused chunk forward over the same
raw tokens."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from oracle import prologue
from tests.parity import TOL, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def run(N, H, dk, dv, dtype, steps, seed, beta_scale=1.0, la_scale=0.3, hook=None):
    import linear_attention_sequence_rule_b200 as gdn
    S0 = workloads.make_decode_state(N, H, dk, dv, seed)
    S_dev = S0.cuda()
    S_ref = S0.double().numpy().reshape(N * H, 1, dk, dv)
    e_o = 0.0
    flat = lambda x: np.asarray(x).reshape(N * H, 1, *np.asarray(x).shape[2:])
    for step in range(steps):
        x = workloads.make_raw_decode_step_inputs(N, H, dk, dv, dtype, seed=seed, step=step, beta_scale=beta_scale,
                                                  la_scale=la_scale)
        if hook:
            hook(step, x)
        d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
        out = gdn.decode_step_fused(d["q_raw"], d["k_raw"], d["v"], d["a_raw"], d["b_raw"], x["a_scale"],
                                    x["b_scale"], S_dev)
        q = prologue.l2_normalize(x["q_raw"])
        k = prologue.l2_normalize(x["k_raw"])
        la, be = prologue.gates(x["a_raw"], x["b_raw"], x["a_scale"], x["b_scale"])
        o_ref, S_ref = oracle.decode_step(flat(q), flat(k), flat(f64(x["v"])), flat(la), flat(be), S_ref)
        e_o = max(e_o, max_abs(f64(out).reshape(N * H, dv), o_ref[:, 0]))
    gdn.device_status()
    e_s = max_abs(f64(S_dev).reshape(N * H, dk, dv), S_ref[:, 0])
    return e_o, e_s


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 256)])
def test_steps(dtype, dk, dv):
    e_o, e_s = run(3, 4, dk, dv, dtype, steps=30, seed=dk + dv)
    assert e_o <= TOL[dtype] and e_s <= TOL[dtype], (e_o, e_s)


def test_reset_beta_scale_two_and_zero_key():
    def hook(step, x):
        if step == 5:
            x["a_raw"][1, 2] = float("inf")  # log alpha = -inf: the state restarts from zero
        if step == 7:
            x["k_raw"][0, 1] = 0.0  # a zero key row normalises to zero (the epsilon keeps it finite)
    e_o, e_s = run(2, 3, 128, 128, "bf16", steps=12, seed=5, beta_scale=2.0, hook=hook)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_steps_equal_fused_chunk_forward():
    # T decode steps on raw tokens = the fused chunk forward over the same T raw tokens
    import linear_attention_sequence_rule_b200 as gdn
    N, H, dk, dv, T = 2, 3, 128, 128, 40
    xs = [workloads.make_raw_decode_step_inputs(N, H, dk, dv, "bf16", seed=9, step=t, la_scale=0.3)
          for t in range(T)]
    S0 = workloads.make_decode_state(N, H, dk, dv, 9)
    S = S0.cuda()
    outs = []
    for x in xs:
        d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
        outs.append(gdn.decode_step_fused(d["q_raw"], d["k_raw"], d["v"], d["a_raw"], d["b_raw"], x["a_scale"],
                                          x["b_scale"], S))
    stack = lambda key: torch.stack([x[key] for x in xs], dim=1).contiguous().cuda()  # [N, T, ...]
    out_c, S_c = gdn.chunk_fwd_fused(stack("q_raw"), stack("k_raw"), stack("v"), stack("a_raw"), stack("b_raw"),
                                     xs[0]["a_scale"], xs[0]["b_scale"], S0=S0.cuda())
    gdn.device_status()
    assert max_abs(f64(torch.stack(outs, dim=1)), f64(out_c)) <= TOL["bf16"]
    assert max_abs(f64(S), f64(S_c)) <= TOL["bf16"]
