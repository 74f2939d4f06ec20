"""GPU parity of gdn_decode_step against the fp64 oracle, step after step with the state carried
on the device (the oracle carries its own fp64 state)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import TOL, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def run_steps(N, H, dk, dv, dtype, steps, seed, units=None, la_scale=0.1, beta_scale=1.0,
              hook=None):
    import linear_attention_sequence_rule_b200 as gdn
    S0 = workloads.make_decode_state(N, H, dk, dv, seed)
    S_dev = S0.cuda()
    S_ref = S0.double().numpy().reshape(N * H, dk, dv)
    sel = np.arange(N * H) if units is None else np.asarray(units)
    S_ref = S_ref[sel][:, None]  # [n_sel, 1, dk, dv]
    e_o = 0.0
    for step in range(steps):
        inp = workloads.make_decode_step_inputs(N, H, dk, dv, dtype, seed=seed, step=step,
                                                la_scale=la_scale, beta_scale=beta_scale)
        if hook:
            hook(step, inp)
        d = {k: v.cuda() for k, v in inp.items()}
        out = gdn.decode_step(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S_dev)
        flat = lambda t: t.reshape(N * H, *t.shape[2:])[sel][:, None]
        o_ref, S_ref = oracle.decode_step(flat(inp["q"]), flat(inp["k"]), flat(inp["v"]),
                                          flat(inp["log_alpha"]), flat(inp["beta"]), S_ref)
        e_o = max(e_o, max_abs(f64(out).reshape(N * H, dv)[sel], o_ref[:, 0]))
    torch.cuda.synchronize()
    e_s = max_abs(f64(S_dev).reshape(N * H, dk, dv)[sel], S_ref[:, 0])
    return e_o, e_s


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64), (128, 256), (64, 256), (256, 64),
                                   (256, 128), (256, 256)])
def test_small(dtype, dk, dv):
    e_o, e_s = run_steps(3, 5, dk, dv, dtype, steps=40, seed=dk * 7 + dv)
    assert e_o <= TOL[dtype] and e_s <= TOL[dtype], (e_o, e_s)


def test_extreme_gates():
    def hook(step, inp):
        if step % 3 == 0:
            inp["log_alpha"][0, :] = -float("inf")
        if step % 4 == 1:
            inp["beta"][1, :] = 2.0
        if step % 5 == 2:
            inp["beta"][2, :] = 0.0
    e_o, e_s = run_steps(3, 4, 128, 128, "f32", steps=30, seed=3, hook=hook, la_scale=1.0)
    assert e_o <= TOL["f32"] and e_s <= TOL["f32"], (e_o, e_s)


def test_decode_full_size_sampled_states():
    """The decode workload at full size (N=256, H=32, d=128, 1000 steps); every state runs on
    the GPU, the oracle follows a seeded sample of 24 states through all 1000 steps."""
    cfg = workloads.CONFIGS["decode"]
    N, H, d = cfg["N"], cfg["H"], cfg["dk"]
    units = sorted(np.random.default_rng(0).choice(N * H, 24, replace=False).tolist())
    e_o, e_s = run_steps(N, H, d, d, "bf16", steps=cfg["steps"], seed=cfg["seed"], units=units,
                         la_scale=cfg["la_scale"])
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)
