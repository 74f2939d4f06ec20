"""Pins of the fp64 oracle to facts the definition fixes (CPU only).

Each test checks the sequential oracle (and, where marked, the chunkwise form) against something
other than itself: closed forms, invariants, a hand-worked example, brute-force agreement of two
independently written algorithms, and a textbook triangular solve.  The shapes use dk != dv
wherever possible, so a transposed operand fails on shape as well as on value.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import chunkwise

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(rng, B, T, H, dk, dv, beta_scale=1.0, la_std=1.0, s0=True, unit=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    beta = beta_scale / (1 + np.exp(-rng.standard_normal((B, T, H))))
    la = -np.log1p(np.exp(la_std * rng.standard_normal((B, T, H))))
    S0 = 0.5 * rng.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, la, beta, S0


def test_hand_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_2x2.json")))
    a = np.array(g["alpha"])
    with np.errstate(divide="ignore"):
        la = np.log(a)
    q = np.array(g["q"])[None, :, None, :]
    k = np.array(g["k"])[None, :, None, :]
    v = np.array(g["v"])[None, :, None, :]
    beta = np.array(g["beta"])[None, :, None]
    S0 = np.array(g["S0"])[None, None]
    out, Sf = oracle.forward(q, k, v, la[None, :, None], beta, S0)
    np.testing.assert_allclose(out[0, :, 0], np.array(g["out"]), atol=1e-14)
    np.testing.assert_allclose(Sf[0, 0], np.array(g["S_final"]), atol=1e-14)
    # the chunkwise form and the decode oracle reach the same values
    out_c, Sf_c = chunkwise.forward_chunkwise(q, k, v, la[None, :, None], beta, S0, chunk=2)
    np.testing.assert_allclose(out_c[0, :, 0], np.array(g["out"]), atol=1e-14)
    np.testing.assert_allclose(Sf_c[0, 0], np.array(g["S_final"]), atol=1e-14)
    S = S0[0][None]
    for t in range(3):
        o, S = oracle.decode_step(q[0, t][None], k[0, t][None], v[0, t][None],
                                  la[t].reshape(1, 1), beta[0, t][None], S)
        np.testing.assert_allclose(o[0, 0], np.array(g["out"][t]), atol=1e-14)
    np.testing.assert_allclose(S[0, 0], np.array(g["S_final"]), atol=1e-14)


def test_beta_zero_is_pure_decay():
    """beta = 0: S_t = a_t S_{t-1}, so S_T = (prod a) S0 and o_t = gamma_t S0^T q_t."""
    rng = np.random.default_rng(1)
    B, T, H, dk, dv = 2, 37, 3, 7, 5
    q, k, v, la, beta, S0 = rand_inputs(rng, B, T, H, dk, dv)
    beta[:] = 0.0
    out, Sf = oracle.forward(q, k, v, la, beta, S0)
    G = np.cumsum(la, axis=1)  # [B,T,H]
    expect_out = np.exp(G)[..., None] * np.einsum("bhij,bthi->bthj", S0, q)
    np.testing.assert_allclose(out, expect_out, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(Sf, np.exp(G[:, -1])[..., None, None] * S0, rtol=1e-12)


def test_alpha_zero_resets_state():
    """log_alpha = -inf at token t0: S_{t0} = b k v^T and the suffix equals a fresh run."""
    rng = np.random.default_rng(2)
    B, T, H, dk, dv = 1, 40, 2, 6, 4
    q, k, v, la, beta, S0 = rand_inputs(rng, B, T, H, dk, dv)
    t0 = 17
    la[:, t0] = -np.inf
    out, Sf = oracle.forward(q, k, v, la, beta, S0)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(Sf))
    out2, Sf2 = oracle.forward(q[:, t0:], k[:, t0:], v[:, t0:], la[:, t0:], beta[:, t0:], None)
    np.testing.assert_allclose(out[:, t0:], out2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Sf, Sf2, rtol=1e-13, atol=1e-14)
    # o_{t0} = (b k v^T)^T q = b (k . q) v
    kq = np.einsum("bhi,bhi->bh", k[:, t0], q[:, t0])
    np.testing.assert_allclose(out[:, t0], (beta[:, t0] * kq)[..., None] * v[:, t0],
                               rtol=1e-13, atol=1e-14)


def test_orthonormal_keys_store_and_overwrite():
    """a = b = 1, orthonormal keys, S0 = 0: querying k_j returns v_j; rewriting k_j replaces it."""
    rng = np.random.default_rng(3)
    dk, dv, n = 8, 5, 6
    Kq, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Kq[:, :n].T  # n orthonormal rows
    vals = rng.standard_normal((n, dv))
    vnew = rng.standard_normal(dv)
    # tokens: n writes, n reads, one overwrite of key 2, n reads
    ks, vs, qs, bs = [], [], [], []
    for j in range(n):
        ks.append(keys[j]); vs.append(vals[j]); qs.append(np.zeros(dk)); bs.append(1.0)
    for j in range(n):
        ks.append(np.zeros(dk)); vs.append(np.zeros(dv)); qs.append(keys[j]); bs.append(0.0)
    ks.append(keys[2]); vs.append(vnew); qs.append(np.zeros(dk)); bs.append(1.0)
    for j in range(n):
        ks.append(np.zeros(dk)); vs.append(np.zeros(dv)); qs.append(keys[j]); bs.append(0.0)
    T = len(ks)
    q = np.array(qs)[None, :, None]
    k = np.array(ks)[None, :, None]
    v = np.array(vs)[None, :, None]
    beta = np.array(bs)[None, :, None]
    la = np.zeros((1, T, 1))
    out, _ = oracle.forward(q, k, v, la, beta, None)
    np.testing.assert_allclose(out[0, n:2 * n, 0], vals, atol=1e-13)
    expect = vals.copy()
    expect[2] = vnew
    np.testing.assert_allclose(out[0, 2 * n + 1:, 0], expect, atol=1e-13)


def test_beta_two_is_householder_reflection():
    """a = 1, b = 2, unit k: S_t - 2 k v^T = (I - 2 k k^T) S_{t-1}; with v = 0 the Frobenius
    norm is kept, det flips sign (dk = dv), and the same key twice restores S."""
    rng = np.random.default_rng(4)
    d = 6
    S = rng.standard_normal((1, 1, d, d))
    for _ in range(5):
        k = rng.standard_normal(d)
        k /= np.linalg.norm(k)
        z = np.zeros((1, 1, d))
        one = np.zeros((1, 1))
        two = np.full((1, 1), 2.0)
        _, S1 = oracle.decode_step(z, k[None, None], z, one, two, S)
        np.testing.assert_allclose(np.linalg.norm(S1), np.linalg.norm(S), rtol=1e-13)
        np.testing.assert_allclose(np.linalg.det(S1[0, 0]), -np.linalg.det(S[0, 0]), rtol=1e-10)
        _, S2 = oracle.decode_step(z, k[None, None], z, one, two, S1)
        np.testing.assert_allclose(S2, S, atol=1e-13)
        v = rng.standard_normal(d)
        _, S3 = oracle.decode_step(z, k[None, None], v[None, None], one, two, S)
        Hh = np.eye(d) - 2 * np.outer(k, k)
        np.testing.assert_allclose(S3[0, 0] - 2 * np.outer(k, v), Hh @ S[0, 0], atol=1e-13)
        S = S1


def test_linear_in_values_and_initial_state():
    rng = np.random.default_rng(5)
    B, T, H, dk, dv = 2, 30, 2, 5, 7
    q, k, v1, la, beta, S01 = rand_inputs(rng, B, T, H, dk, dv)
    v2 = rng.standard_normal(v1.shape)
    S02 = rng.standard_normal(S01.shape)
    a, b = 0.7, -1.3
    o1, s1 = oracle.forward(q, k, v1, la, beta, S01)
    o2, s2 = oracle.forward(q, k, v2, la, beta, S02)
    o3, s3 = oracle.forward(q, k, a * v1 + b * v2, la, beta, a * S01 + b * S02)
    np.testing.assert_allclose(o3, a * o1 + b * o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s3, a * s1 + b * s2, rtol=1e-11, atol=1e-12)


def test_value_columns_are_separable():
    rng = np.random.default_rng(6)
    B, T, H, dk, dv = 1, 25, 2, 6, 5
    q, k, v, la, beta, S0 = rand_inputs(rng, B, T, H, dk, dv)
    o1, s1 = oracle.forward(q, k, v, la, beta, S0)
    j = 3
    v2 = v.copy()
    v2[..., j] += rng.standard_normal(v2[..., j].shape)
    o2, s2 = oracle.forward(q, k, v2, la, beta, S0)
    others = [c for c in range(dv) if c != j]
    np.testing.assert_array_equal(o1[..., others], o2[..., others])
    np.testing.assert_array_equal(s1[..., others], s2[..., others])
    assert np.abs(o1[..., j] - o2[..., j]).max() > 1e-3


def test_non_expansive_for_beta_in_closed_range():
    """Unit keys, b in [0, 2]: ||S_t||_2 <= a_t ||S_{t-1}||_2 + b_t ||v_t||."""
    rng = np.random.default_rng(7)
    dk, dv = 6, 4
    S = rng.standard_normal((1, 1, dk, dv))
    for t in range(200):
        k = rng.standard_normal(dk)
        k /= np.linalg.norm(k)
        v = rng.standard_normal(dv)
        b = [0.0, 2.0, rng.uniform(0, 2)][t % 3]
        la = -abs(rng.standard_normal())
        _, S1 = oracle.decode_step(np.zeros((1, 1, dk)), k[None, None], v[None, None],
                                   np.full((1, 1), la), np.full((1, 1), b), S)
        lhs = np.linalg.norm(S1[0, 0], 2)
        rhs = np.exp(la) * np.linalg.norm(S[0, 0], 2) + b * np.linalg.norm(v)
        assert lhs <= rhs * (1 + 1e-12) + 1e-12
        S = S1


def test_single_token_in_error_form():
    """T = 1, written in the read-out/error form: S1 = a S0 + k u^T, u = b (v - a S0^T k)."""
    rng = np.random.default_rng(8)
    B, T, H, dk, dv = 3, 1, 2, 5, 3
    q, k, v, la, beta, S0 = rand_inputs(rng, B, T, H, dk, dv, unit=False)
    out, Sf = oracle.forward(q, k, v, la, beta, S0)
    a = np.exp(la[:, 0])[..., None]
    b = beta[:, 0][..., None]
    u = b * (v[:, 0] - a * np.einsum("bhij,bhi->bhj", S0, k[:, 0]))
    S1 = a[..., None] * S0 + np.einsum("bhi,bhj->bhij", k[:, 0], u)
    np.testing.assert_allclose(Sf, S1, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(out[:, 0], np.einsum("bhij,bhi->bhj", S1, q[:, 0]),
                               rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
def test_chunkwise_form_matches_sequential(chunk):
    """Two independently written algorithms agree: the WY / UT chunk form and the definition."""
    rng = np.random.default_rng(10 + chunk)
    B, T, H, dk, dv = 2, 150, 2, 8, 6
    q, k, v, la, beta, S0 = rand_inputs(rng, B, T, H, dk, dv, beta_scale=2.0, la_std=2.0)
    la[0, 77, 1] = -np.inf  # an exact reset inside a chunk
    la[1, 64, 0] = -np.inf  # and one on a chunk boundary
    o_s, s_s = oracle.forward(q, k, v, la, beta, S0)
    o_c, s_c = chunkwise.forward_chunkwise(q, k, v, la, beta, S0, chunk=chunk)
    np.testing.assert_allclose(o_c, o_s, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s_c, s_s, rtol=0, atol=1e-12)


def test_chunkwise_form_matches_sequential_varlen():
    rng = np.random.default_rng(20)
    lengths = [1, 63, 64, 65, 130, 0, 200]
    Ttot = sum(lengths)
    H, dk, dv = 3, 8, 5
    q, k, v, la, beta, _ = rand_inputs(rng, 1, Ttot, H, dk, dv)
    q, k, v, la, beta = q[0], k[0], v[0], la[0], beta[0]
    S0 = rng.standard_normal((len(lengths), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    o_s, s_s = oracle.forward(q, k, v, la, beta, S0, cu_seqlens=cu)
    o_c, s_c = chunkwise.forward_chunkwise(q, k, v, la, beta, S0, chunk=64, cu_seqlens=cu)
    np.testing.assert_allclose(o_c, o_s, atol=1e-12)
    np.testing.assert_allclose(s_c, s_s, atol=1e-12)
    # the empty sequence keeps its initial state
    np.testing.assert_array_equal(s_s[5], S0[5])
    # each sequence of the pack equals its own dense run
    for s, L in enumerate(lengths):
        if L == 0:
            continue
        a, b_ = cu[s], cu[s + 1]
        o1, s1 = oracle.forward(q[None, a:b_], k[None, a:b_], v[None, a:b_], la[None, a:b_],
                                beta[None, a:b_], S0[s][None])
        np.testing.assert_allclose(o_s[a:b_], o1[0], atol=1e-13)
        np.testing.assert_allclose(s_s[s], s1[0], atol=1e-13)


def test_unit_lower_inverse_is_exact():
    rng = np.random.default_rng(30)
    C = 64
    A = np.tril(0.2 * rng.standard_normal((C, C)), k=-1)
    T = chunkwise.unit_lower_inverse(A)
    np.testing.assert_allclose((np.eye(C) + A) @ T, np.eye(C), atol=1e-12)
    np.testing.assert_allclose(T, np.linalg.solve(np.eye(C) + A, np.eye(C)), atol=1e-12)
    assert np.allclose(np.triu(T, 1), 0) and np.allclose(np.diag(T), 1)


def test_decode_steps_equal_forward():
    rng = np.random.default_rng(40)
    N, T, H, dk, dv = 3, 12, 2, 5, 4
    q, k, v, la, beta, S0 = rand_inputs(rng, N, T, H, dk, dv)
    out, Sf = oracle.forward(q, k, v, la, beta, S0)
    S = S0
    for t in range(T):
        o, S = oracle.decode_step(q[:, t], k[:, t], v[:, t], la[:, t], beta[:, t], S)
        np.testing.assert_allclose(o, out[:, t], atol=1e-13)
    np.testing.assert_allclose(S, Sf, atol=1e-13)


def test_state_carry_equals_single_call():
    rng = np.random.default_rng(41)
    B, T, H, dk, dv = 2, 50, 2, 6, 6
    q, k, v, la, beta, S0 = rand_inputs(rng, B, T, H, dk, dv)
    out, Sf = oracle.forward(q, k, v, la, beta, S0)
    o1, s1 = oracle.forward(q[:, :21], k[:, :21], v[:, :21], la[:, :21], beta[:, :21], S0)
    o2, s2 = oracle.forward(q[:, 21:], k[:, 21:], v[:, 21:], la[:, 21:], beta[:, 21:], s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), out, atol=1e-13)
    np.testing.assert_allclose(s2, Sf, atol=1e-13)


def test_unit_subset_matches_full():
    rng = np.random.default_rng(42)
    B, T, H, dk, dv = 3, 20, 4, 5, 3
    q, k, v, la, beta, S0 = rand_inputs(rng, B, T, H, dk, dv)
    out, Sf = oracle.forward(q, k, v, la, beta, S0)
    units = [1, 6, 11]
    o2, s2 = oracle.forward(q, k, v, la, beta, S0, units=units)
    for u in units:
        b, h = divmod(u, H)
        np.testing.assert_array_equal(o2[b, :, h], out[b, :, h])
        np.testing.assert_array_equal(s2[b, h], Sf[b, h])
    assert np.isnan(o2[0, :, 0]).all()
