"""Pins of the oracles' behaviour over value columns, the property the value-split kernels rest on.

S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T acts on S from the left, so column j of S,
of the outputs and of dL/dS follows from column j of V, S0, dout and dS_final alone.  Hence:
* forward and decode: a call on all columns equals the calls on column blocks, side by side;
* backward: dv and dS0 of the whole call are the blocks' dv and dS0 side by side, and dq, dk,
  dlog_alpha, dbeta are the sums of the blocks' (the loss is a sum over the blocks' outputs).
The oracles are the sequential fp64 definitions (pinned separately against closed forms and finite
differences); these tests check that nothing in them couples value columns, on dense and varlen
inputs with exact resets and beta = 2.  CPU only."""
import numpy as np

import oracle


def case(rng, dv, lengths=None, B=2, T=23, H=2, dk=5):
    lead = (int(sum(lengths)),) if lengths is not None else (B, T)
    nseq = len(lengths) if lengths is not None else B
    k = rng.normal(size=(*lead, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    c = dict(q=rng.normal(size=(*lead, H, dk)), k=k, v=rng.normal(size=(*lead, H, dv)),
             log_alpha=-np.log1p(np.exp(rng.normal(size=(*lead, H)))),
             beta=2.0 / (1.0 + np.exp(-rng.normal(size=(*lead, H)))),
             S0=0.5 * rng.normal(size=(nseq, H, dk, dv)),
             cu_seqlens=None if lengths is None else np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))
    c["log_alpha"].reshape(-1)[3] = -np.inf  # an exact reset
    return c


BLOCKS = (slice(0, 3), slice(3, 4), slice(4, 9))  # uneven blocks of a 9-column value head


def test_forward_splits_over_value_blocks():
    rng = np.random.default_rng(70)
    for lengths in (None, [4, 0, 11, 1]):
        c = case(rng, 9, lengths)
        o, S = oracle.forward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["S0"], cu_seqlens=c["cu_seqlens"])
        parts = [oracle.forward(c["q"], c["k"], c["v"][..., b], c["log_alpha"], c["beta"], c["S0"][..., b],
                                cu_seqlens=c["cu_seqlens"]) for b in BLOCKS]
        np.testing.assert_allclose(o, np.concatenate([p[0] for p in parts], axis=-1), rtol=0, atol=1e-13)
        np.testing.assert_allclose(S, np.concatenate([p[1] for p in parts], axis=-1), rtol=0, atol=1e-13)
        # and the blocks are not trivially equal: the whole and a block differ in the columns outside it
        assert np.abs(o[..., 4:]).max() > 1e-3


def test_decode_splits_over_value_blocks():
    rng = np.random.default_rng(71)
    N, H, dk, dv = 3, 2, 5, 9
    S = rng.normal(size=(N, H, dk, dv))
    k = rng.normal(size=(N, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q, v = rng.normal(size=(N, H, dk)), rng.normal(size=(N, H, dv))
    la, be = -np.abs(rng.normal(size=(N, H))), 2.0 / (1.0 + np.exp(-rng.normal(size=(N, H))))
    o, S1 = oracle.decode_step(q, k, v, la, be, S)
    parts = [oracle.decode_step(q, k, v[..., b], la, be, S[..., b]) for b in BLOCKS]
    np.testing.assert_allclose(o, np.concatenate([p[0] for p in parts], axis=-1), rtol=0, atol=1e-13)
    np.testing.assert_allclose(S1, np.concatenate([p[1] for p in parts], axis=-1), rtol=0, atol=1e-13)


def test_backward_splits_over_value_blocks():
    rng = np.random.default_rng(72)
    for lengths in (None, [4, 0, 11, 1]):
        c = case(rng, 9, lengths)
        dout = rng.normal(size=c["v"].shape)
        dSf = rng.normal(size=c["S0"].shape)
        whole = oracle.backward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["S0"], dout, dSf,
                                cu_seqlens=c["cu_seqlens"])
        parts = [oracle.backward(c["q"], c["k"], c["v"][..., b], c["log_alpha"], c["beta"], c["S0"][..., b],
                                 dout[..., b], dSf[..., b], cu_seqlens=c["cu_seqlens"]) for b in BLOCKS]
        for i in (0, 1, 3, 4):  # dq, dk, dlog_alpha, dbeta: sums over the blocks
            np.testing.assert_allclose(whole[i], sum(p[i] for p in parts), rtol=0, atol=1e-11)
        for i in (2, 5):  # dv, dS0: the blocks side by side
            np.testing.assert_allclose(whole[i], np.concatenate([p[i] for p in parts], axis=-1), rtol=0,
                                       atol=1e-12)
        assert np.abs(whole[0]).max() > 1e-3 and np.abs(parts[0][0]).max() > 1e-3
