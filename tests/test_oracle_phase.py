"""Pins of the complex-phase delta-memory oracle (oracle/phase.py), CPU only.

* a hand-worked example from the page's three steps (tests/golden/phase_hand_worked.json): store,
  decayed overwrite read before the decay, recall through an orthogonal key, a beta = 0 token and
  a non-real phasor key;
* exact store and overwrite through orthogonal (DFT) phasor keys;
* beta = 0: pure decay in closed form;
* joint real-linearity in (V, M0) and value-channel separability;
* the chunk form (its own derivation, a triangular solve per chunk) equals the definition to
  1e-12 for several chunk sizes, dense and varlen, Laplace keys |K| < 1, beta up to 2, M0 != 0;
* the reduction to the real gated delta rule that the CUDA path runs on: with S = [Re M | Im M]^T,
  k = (Re K, Im K) / sqrt(dk), q = (Re Q, Im Q) / dk, v = lam sqrt(dk) V, alpha = lam and
  beta' = beta / lam, the (separately pinned) real oracle returns the same outputs and state;
* the per-row decay form (one decay per value channel): with equal rows it is the scalar memory,
  each channel is the scalar memory with that channel's decay, beta = 0 is pure per-row decay in
  closed form, and its chunk form (a triangular solve per channel) equals the definition.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import phase

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "phase_hand_worked.json")


def rand_case(rng, B=2, T=37, H=2, dk=8, dv=5, lengths=None, laplace=False, beta_max=1.0, m0=True):
    lead = (int(sum(lengths)),) if lengths is not None else (B, T)
    nseq = len(lengths) if lengths is not None else B
    th_k = rng.uniform(0, 2 * np.pi, size=(*lead, H, dk))
    th_q = rng.uniform(0, 2 * np.pi, size=(*lead, H, dk))
    mag = np.exp(-rng.uniform(0, 0.5, size=th_k.shape)) if laplace else 1.0
    K = mag * np.exp(1j * th_k)
    Q = np.exp(1j * th_q)
    V = rng.normal(size=(*lead, H, dv))
    la = -np.log1p(np.exp(rng.normal(size=(*lead, H)))) * 0.3
    be = beta_max / (1.0 + np.exp(-rng.normal(size=(*lead, H))))
    M0 = (rng.normal(size=(nseq, H, dv, dk)) + 1j * rng.normal(size=(nseq, H, dv, dk))) * 0.3 if m0 else None
    cu = None if lengths is None else np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return dict(K=K, Q=Q, V=V, log_lam=la, beta=be, M0=M0, cu_seqlens=cu)


def run(c, fn=phase.forward, **kw):
    return fn(c["K"], c["Q"], c["V"], c["log_lam"], c["beta"], c["M0"], cu_seqlens=c["cu_seqlens"], **kw)


def test_hand_worked_example():
    g = json.load(open(GOLDEN))
    K = (np.array(g["K_re"]) + 1j * np.array(g["K_im"]))[None, :, None, :]
    Q = (np.array(g["Q_re"]) + 1j * np.array(g["Q_im"]))[None, :, None, :]
    V = np.array(g["V"], float)[None, :, None, None]
    la = np.log(np.array(g["lam"], float))[None, :, None]
    be = np.array(g["beta"], float)[None, :, None]
    M_ref = np.array(g["M_final_re"]) + 1j * np.array(g["M_final_im"])
    for fn, kw in ((phase.forward, {}), (phase.forward_chunkwise, dict(chunk=2)),
                   (phase.forward_chunkwise, dict(chunk=64))):
        o, M = fn(K, Q, V, la, be, **kw)
        np.testing.assert_allclose(o.ravel(), g["out"], atol=1e-12)
        np.testing.assert_allclose(M[0, 0], M_ref, atol=1e-12)


def dft_keys(dk):
    i = np.arange(dk)
    return np.exp(2j * np.pi * np.outer(np.arange(dk), i) / dk)  # row s: key s


def test_orthogonal_phasor_keys_store_and_overwrite():
    dk, dv = 8, 3
    rng = np.random.default_rng(1)
    keys = dft_keys(dk)
    Vs = rng.normal(size=(dk, dv))
    # tokens 0..7 write V_s with key s; token 8 rewrites key 2 with V'; queries read key t (t < 8),
    # then key 2 and key 5 at tokens 8 and 9 (token 9 writes nothing)
    V_new = rng.normal(size=dv)
    K = np.concatenate([keys, keys[[2, 0]]])[None, :, None, :]
    Q = np.concatenate([keys, keys[[2, 5]]])[None, :, None, :]
    V = np.concatenate([Vs, V_new[None], np.zeros((1, dv))])[None, :, None, :]
    la = np.zeros((1, 10, 1))
    be = np.ones((1, 10, 1))
    be[0, 9, 0] = 0.0
    o, M = phase.forward(K, Q, V, la, be)
    np.testing.assert_allclose(o[0, :8, 0], Vs, atol=1e-12)   # exact store: each key reads its value
    np.testing.assert_allclose(o[0, 8, 0], V_new, atol=1e-12)  # the delta rule overwrites
    np.testing.assert_allclose(o[0, 9, 0], Vs[5], atol=1e-12)  # the other keys are untouched


def test_beta_zero_is_pure_decay():
    rng = np.random.default_rng(2)
    c = rand_case(rng, B=1, T=20, H=3)
    c["beta"] = np.zeros_like(c["beta"])
    o, M = run(c)
    g = np.cumsum(c["log_lam"][0], axis=0)  # [T, H]
    dk = c["K"].shape[-1]
    for t in range(20):
        for h in range(3):
            ref = np.exp(g[t, h]) * (c["M0"][0, h] @ np.conj(c["Q"][0, t, h])).real / dk
            np.testing.assert_allclose(o[0, t, h], ref, atol=1e-12)
    np.testing.assert_allclose(M[0], np.exp(g[-1])[:, None, None] * c["M0"][0], atol=1e-12)


def test_joint_real_linearity_and_channel_separability():
    rng = np.random.default_rng(3)
    c1, c2 = rand_case(rng), rand_case(rng)
    c2.update(K=c1["K"], Q=c1["Q"], log_lam=c1["log_lam"], beta=c1["beta"])
    a, b = 0.7, -1.3
    mix = dict(c1, V=a * c1["V"] + b * c2["V"], M0=a * c1["M0"] + b * c2["M0"])
    o1, M1 = run(c1)
    o2, M2 = run(c2)
    o, M = run(mix)
    np.testing.assert_allclose(o, a * o1 + b * o2, atol=1e-11)
    np.testing.assert_allclose(M, a * M1 + b * M2, atol=1e-11)
    # perturbing value channel 2 moves only output channel 2 and state row 2
    pert = dict(c1, V=c1["V"].copy())
    pert["V"][..., 2] += 1.0
    o3, M3 = run(pert)
    others = [j for j in range(c1["V"].shape[-1]) if j != 2]
    np.testing.assert_allclose(o3[..., others], o1[..., others], atol=1e-12)
    np.testing.assert_allclose(M3[:, :, others], M1[:, :, others], atol=1e-12)
    assert np.abs(o3[..., 2] - o1[..., 2]).max() > 1e-3


@pytest.mark.parametrize("chunk", [1, 4, 16, 64])
def test_chunk_form_equals_definition_dense(chunk):
    rng = np.random.default_rng(10 + chunk)
    c = rand_case(rng, B=2, T=150, H=2, dk=8, dv=6, laplace=True, beta_max=2.0)
    o, M = run(c)
    o2, M2 = run(c, phase.forward_chunkwise, chunk=chunk)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(M2, M, atol=1e-12)


def test_chunk_form_equals_definition_varlen():
    rng = np.random.default_rng(20)
    c = rand_case(rng, H=3, dk=6, dv=4, lengths=[0, 1, 63, 64, 65, 130, 7])
    o, M = run(c)
    o2, M2 = run(c, phase.forward_chunkwise, chunk=64)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(M2, M, atol=1e-12)
    assert np.all(M[0] == c["M0"][0])  # the empty sequence keeps its initial state


def to_real_recurrence(c):
    """The real gated delta rule's inputs that reproduce the phase memory (see the module doc)."""
    K, Q = c["K"], c["Q"]
    dk = K.shape[-1]
    lam = np.exp(c["log_lam"])
    k = np.concatenate([K.real, K.imag], axis=-1) / np.sqrt(dk)
    q = np.concatenate([Q.real, Q.imag], axis=-1) / dk
    v = lam[..., None] * np.sqrt(dk) * c["V"]
    S0 = None
    if c["M0"] is not None:
        S0 = np.concatenate([c["M0"].real, c["M0"].imag], axis=-1).transpose(0, 1, 3, 2)
    return k, q, v, c["log_lam"], c["beta"] / lam, S0


def test_reduces_to_the_real_gated_delta_rule():
    rng = np.random.default_rng(30)
    for c in (rand_case(rng, B=2, T=90, H=2, dk=8, dv=5, laplace=True, beta_max=2.0),
              rand_case(rng, H=2, dk=4, dv=3, lengths=[5, 0, 70, 1])):
        o, M = run(c)
        k, q, v, la, be, S0 = to_real_recurrence(c)
        o_r, S_r = oracle.forward(q, k, v, la, be, S0, cu_seqlens=c["cu_seqlens"])
        dk = c["K"].shape[-1]
        np.testing.assert_allclose(o_r, o, atol=1e-10)
        np.testing.assert_allclose(S_r[:, :, :dk, :].transpose(0, 1, 3, 2), M.real, atol=1e-10)
        np.testing.assert_allclose(S_r[:, :, dk:, :].transpose(0, 1, 3, 2), M.imag, atol=1e-10)


def test_backward_matches_finite_differences():
    # the backward oracle (through the real form) against central differences of the complex
    # definition, for every real input component: Re / Im of K, Q, M0; V; log_lam; beta
    rng = np.random.default_rng(40)
    for lengths in (None, [3, 0, 6]):
        c = rand_case(rng, B=2, T=7, H=2, dk=3, dv=2, laplace=True, beta_max=2.0, lengths=lengths)
        Go = rng.normal(size=c["V"].shape)
        Wm = rng.normal(size=c["M0"].shape) + 1j * rng.normal(size=c["M0"].shape)

        def loss():
            o, M = run(c)
            return float(np.sum(o * Go) + np.sum(M.real * Wm.real + M.imag * Wm.imag))
        got = dict(zip(("K", "Q", "V", "log_lam", "beta", "M0"),
                       phase.backward(c["K"], c["Q"], c["V"], c["log_lam"], c["beta"], c["M0"], Go, Wm,
                                      cu_seqlens=c["cu_seqlens"])))
        h = 1e-6
        for name in ("K", "Q", "V", "log_lam", "beta", "M0"):
            x = c[name]
            parts = (1.0, 1j) if np.iscomplexobj(x) else (1.0,)
            for part in parts:
                fd = np.zeros(x.shape)
                for i in np.ndindex(x.shape):
                    old = x[i]
                    x[i] = old + h * part
                    lp = loss()
                    x[i] = old - h * part
                    lm = loss()
                    x[i] = old
                    fd[i] = (lp - lm) / (2 * h)
                g = got[name].real if part == 1.0 else got[name].imag
                if not np.iscomplexobj(x):
                    g = got[name]
                assert np.max(np.abs(fd - g)) / (1.0 + np.max(np.abs(fd))) < 1e-6, (name, part)


# ---- the per-row decay (the Laplace core's diag(r_t) on the output rows of M) ------------------

def with_row_decays(c, rng, spread=0.4):
    """The case with one finite log-decay per (token, head, value channel); some decays are strong
    (r down to about 1e-3), as finite as the phase memory requires (r > 0, like lam)."""
    dv = c["V"].shape[-1]
    lr = -np.log1p(np.exp(rng.normal(size=(*c["log_lam"].shape, dv)))) * spread
    lr.reshape(-1)[5] = -7.0
    return dict(c, log_r=lr)


def run_rd(c, fn=phase.forward_rowdecay, **kw):
    return fn(c["K"], c["Q"], c["V"], c["log_r"], c["beta"], c["M0"], cu_seqlens=c["cu_seqlens"], **kw)


def test_rowdecay_with_equal_rows_is_the_scalar_memory():
    rng = np.random.default_rng(50)
    for c in (rand_case(rng, B=2, T=40, H=2, dk=6, dv=4, laplace=True, beta_max=2.0),
              rand_case(rng, H=2, dk=5, dv=3, lengths=[7, 0, 30, 1])):
        c = dict(c, log_r=np.repeat(c["log_lam"][..., None], c["V"].shape[-1], axis=-1))
        o, M = run_rd(c)
        o2, M2 = run(c)
        np.testing.assert_allclose(o, o2, atol=1e-13)
        np.testing.assert_allclose(M, M2, atol=1e-13)


def test_rowdecay_is_one_scalar_memory_per_channel():
    # channel j of the per-row memory is the scalar-decay memory with value V[..., j], decay
    # log_r[..., j] and initial rows M0[:, :, j] (the separately pinned ``forward``)
    rng = np.random.default_rng(51)
    for lengths in (None, [9, 0, 33, 2]):
        c = with_row_decays(rand_case(rng, B=2, T=37, H=2, dk=6, dv=4, laplace=True, beta_max=2.0,
                                      lengths=lengths), rng)
        o, M = run_rd(c)
        assert np.abs(np.diff(c["log_r"], axis=-1)).max() > 0.1  # the channels' decays do differ
        for j in range(c["V"].shape[-1]):
            cj = dict(c, V=c["V"][..., j:j + 1], log_lam=c["log_r"][..., j], M0=c["M0"][:, :, j:j + 1])
            oj, Mj = run(cj)
            np.testing.assert_allclose(o[..., j], oj[..., 0], atol=1e-12)
            np.testing.assert_allclose(M[:, :, j], Mj[:, :, 0], atol=1e-12)


def test_rowdecay_beta_zero_is_pure_row_decay():
    rng = np.random.default_rng(52)
    c = with_row_decays(rand_case(rng, B=1, T=15, H=2, dk=4, dv=3), rng)
    c["beta"] = np.zeros_like(c["beta"])
    o, M = run_rd(c)
    G = np.cumsum(c["log_r"][0], axis=0)  # [T, H, dv]
    dk = c["K"].shape[-1]
    for t in range(15):
        for h in range(2):
            Mt = np.exp(G[t, h])[:, None] * c["M0"][0, h]
            np.testing.assert_allclose(o[0, t, h], (Mt @ np.conj(c["Q"][0, t, h])).real / dk, atol=1e-12)
    np.testing.assert_allclose(M[0], np.exp(G[-1])[:, :, None] * c["M0"][0], atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 5, 16, 64])
def test_rowdecay_chunk_form_equals_definition(chunk):
    rng = np.random.default_rng(60 + chunk)
    for lengths in (None, [0, 1, 63, 64, 65, 20]):
        c = with_row_decays(rand_case(rng, B=2, T=90, H=2, dk=6, dv=5, laplace=True, beta_max=2.0,
                                      lengths=lengths), rng)
        o, M = run_rd(c)
        o2, M2 = run_rd(c, phase.forward_rowdecay_chunkwise, chunk=chunk)
        np.testing.assert_allclose(o2, o, atol=1e-12)
        np.testing.assert_allclose(M2, M, atol=1e-12)
