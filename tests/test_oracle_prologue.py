"""Pins of the fp64 prologue (raw projections -> normalised q, k and gates) against closed forms
and identities of the functions it is made of."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from oracle import prologue as P


def test_softplus_and_sigmoid_closed_forms():
    assert P.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert P.sigmoid(0.0) == 0.5
    x = np.linspace(-30, 30, 601)
    # softplus(x) - softplus(-x) = x and sigmoid(x) + sigmoid(-x) = 1, for every x
    np.testing.assert_allclose(P.softplus(x) - P.softplus(-x), x, atol=1e-12)
    np.testing.assert_allclose(P.sigmoid(x) + P.sigmoid(-x), 1.0, atol=1e-15)
    # the derivative of softplus is sigmoid (central difference)
    h = 1e-5
    np.testing.assert_allclose((P.softplus(x + h) - P.softplus(x - h)) / (2 * h), P.sigmoid(x), atol=1e-9)
    # tails: no overflow, the asymptotes
    assert P.softplus(1000.0) == 1000.0 and P.softplus(-1000.0) == 0.0
    assert P.sigmoid(1000.0) == 1.0 and P.sigmoid(-1000.0) == 0.0


def test_gate_forms():
    a = np.array([0.0, 1.0, -2.0, np.inf])
    b = np.array([0.0, 3.0, -3.0, 0.0])
    la, be = P.gates(a, b, a_scale=0.1, b_scale=2.0)
    np.testing.assert_allclose(la[:3], -0.1 * np.log1p(np.exp(a[:3])), rtol=1e-14)
    assert la[3] == -np.inf  # an exact reset
    np.testing.assert_allclose(be, 2.0 / (1.0 + np.exp(-b)), rtol=1e-14)
    assert np.all(be > 0) and np.all(be < 2)


def test_l2_normalize():
    g = np.random.default_rng(0)
    x = g.normal(size=(7, 5, 64)) * 3.0
    y = P.l2_normalize(x, eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-14)
    np.testing.assert_allclose(y * np.linalg.norm(x, axis=-1, keepdims=True), x, atol=1e-12)
    z = P.l2_normalize(np.zeros((2, 64)))
    assert np.all(z == 0.0)
    # with the default eps the norm is 1 - eps / (2 |x|^2) to first order
    n = np.linalg.norm(P.l2_normalize(x), axis=-1)
    np.testing.assert_allclose(n, 1.0 - P.EPS / (2 * np.sum(x * x, axis=-1)), atol=1e-12)


def test_fused_forward_without_gating_is_a_readout_of_s0():
    """a_scale = 0 (alpha = 1) and b_scale = 0 (beta = 0): the state stays S0 and every output is
    S0^T q_hat with the normalised query."""
    inp = workloads.make_raw_chunk_inputs(B=2, T=70, H=3, dk=16, dv=8, dtype="f32", seed=3, s0_std=0.5)
    out, Sf = P.forward_fused(inp["q_raw"], inp["k_raw"], inp["v"], inp["a_raw"], inp["b_raw"],
                              inp["S0"], a_scale=0.0, b_scale=0.0)
    S0 = inp["S0"].double().numpy()
    q = inp["q_raw"].double().numpy()
    qh = q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + P.EPS)
    expect = np.einsum("bhkv,bthk->bthv", S0, qh)
    np.testing.assert_allclose(out, expect, atol=1e-13)
    np.testing.assert_allclose(Sf, S0, atol=0)


def test_raw_inputs_match_the_plain_workload_draws():
    """The raw generator draws what the plain generator draws, before normalising/activating."""
    raw = workloads.make_raw_chunk_inputs(B=1, T=40, H=2, dk=16, dv=16, dtype="f32", seed=9,
                                          beta_scale=2.0, la_std=2.0, la_scale=0.5, s0_std=0.1)
    ref = workloads.make_chunk_inputs(B=1, T=40, H=2, dk=16, dv=16, dtype="f32", seed=9,
                                      beta_scale=2.0, la_std=2.0, la_scale=0.5, s0_std=0.1)
    la, be = P.gates(raw["a_raw"], raw["b_raw"], raw["a_scale"], raw["b_scale"])
    np.testing.assert_allclose(la, ref["log_alpha"].double().numpy(), rtol=1e-6)
    np.testing.assert_allclose(be, ref["beta"].double().numpy(), rtol=1e-6)
    np.testing.assert_allclose(P.l2_normalize(raw["k_raw"], eps=0.0), ref["k"].double().numpy(), atol=1e-6)
    assert torch.equal(raw["v"], ref["v"]) and torch.equal(raw["S0"], ref["S0"])
