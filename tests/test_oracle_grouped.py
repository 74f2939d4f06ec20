"""Pins of the grouped-value-head oracle: it reduces to the plain oracle when every value head has
its own q/k head, each value head equals a single-head run on its group's q/k, heads that share
q/k and everything else agree exactly, and decode steps reproduce the forward."""
import numpy as np

import oracle
import workloads
from oracle import grouped


def test_one_value_head_per_qk_head_is_the_plain_oracle():
    inp = workloads.make_gva_chunk_inputs(B=2, T=50, Hk=3, Hv=3, dk=16, dv=8, dtype="f32", seed=1, s0_std=0.3)
    o1, s1 = grouped.forward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    o2, s2 = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    assert np.array_equal(o1, o2) and np.array_equal(s1, s2)


def test_each_value_head_is_a_single_head_run_on_its_group():
    inp = workloads.make_gva_chunk_inputs(B=2, T=70, Hk=2, Hv=6, dk=16, dv=8, dtype="f32", seed=2, s0_std=0.3)
    out, Sf = grouped.forward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    G = 3
    for h in range(6):
        sl = slice(h, h + 1)
        g = slice(h // G, h // G + 1)
        o, s = oracle.forward(inp["q"][:, :, g], inp["k"][:, :, g], inp["v"][:, :, sl],
                              inp["log_alpha"][:, :, sl], inp["beta"][:, :, sl], inp["S0"][:, sl])
        np.testing.assert_array_equal(out[:, :, sl], o)
        np.testing.assert_array_equal(Sf[:, sl], s)


def test_heads_sharing_everything_agree_and_groups_differ():
    inp = workloads.make_gva_chunk_inputs(B=1, T=40, Hk=2, Hv=4, dk=16, dv=8, dtype="f32", seed=3)
    for key in ("v", "log_alpha", "beta"):
        t = inp[key]
        t[:, :, 1] = t[:, :, 0]  # heads 0 and 1 share q/k (group 0): make the rest equal too
        t[:, :, 2] = t[:, :, 0]  # head 2 is in group 1: same v and gates, other q/k
    out, Sf = grouped.forward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None)
    assert np.array_equal(out[:, :, 0], out[:, :, 1]) and np.array_equal(Sf[:, 0], Sf[:, 1])
    assert np.abs(out[:, :, 0] - out[:, :, 2]).max() > 1e-3


def test_decode_steps_reproduce_the_forward():
    inp = workloads.make_gva_chunk_inputs(B=2, T=12, Hk=2, Hv=4, dk=16, dv=8, dtype="f32", seed=4, s0_std=0.2)
    out, Sf = grouped.forward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    S = inp["S0"].double().numpy()
    for t in range(12):
        o, S = grouped.decode_step_gva(inp["q"][:, t], inp["k"][:, t], inp["v"][:, t], inp["log_alpha"][:, t],
                                       inp["beta"][:, t], S)
        np.testing.assert_allclose(o, out[:, t], atol=1e-13)
    np.testing.assert_allclose(S, Sf, atol=1e-13)
