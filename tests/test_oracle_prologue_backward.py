"""Pin of the fused-prologue backward oracle (oracle/prologue.py, backward_fused): every gradient
element against central finite differences of the fused forward oracle (prologue + recurrence,
fp64), on dense and varlen inputs with unnormalised q/k rows of different norms, one exact reset
(a = +inf), and gate projections spread over both tails.  CPU only."""
import numpy as np

from oracle import prologue

H_FD = 1e-6


def loss(c, G, W):
    out, S = prologue.forward_fused(c["q"], c["k"], c["v"], c["a"], c["b"], c["S0"], c["a_scale"], c["b_scale"],
                                    cu_seqlens=c["cu"])
    return float(np.sum(out * G) + np.sum(S * W))


def case(rng, lengths=None, B=2, T=9, H=2, dk=4, dv=3):
    lead = (int(sum(lengths)),) if lengths is not None else (B, T)
    nseq = len(lengths) if lengths is not None else B
    c = dict(q=rng.normal(size=(*lead, H, dk)) * rng.uniform(0.3, 3.0, size=(*lead, H, 1)),
             k=rng.normal(size=(*lead, H, dk)) * rng.uniform(0.3, 3.0, size=(*lead, H, 1)),
             v=rng.normal(size=(*lead, H, dv)), a=rng.normal(size=(*lead, H)) * 2.0,
             b=rng.normal(size=(*lead, H)) * 2.0, S0=0.5 * rng.normal(size=(nseq, H, dk, dv)),
             a_scale=0.7, b_scale=1.6,
             cu=None if lengths is None else np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32))
    return c


def check(c, rng):
    G = rng.normal(size=c["v"].shape)
    W = rng.normal(size=c["S0"].shape)
    got = prologue.backward_fused(c["q"], c["k"], c["v"], c["a"], c["b"], c["S0"], G, c["a_scale"], c["b_scale"],
                                  dS_final=W, cu_seqlens=c["cu"])
    for name, g in zip(("q", "k", "v", "a", "b", "S0"), got):
        x = c[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            if np.isinf(x[i]):
                continue
            old = x[i]
            x[i] = old + H_FD
            lp = loss(c, G, W)
            x[i] = old - H_FD
            lm = loss(c, G, W)
            x[i] = old
            fd[i] = (lp - lm) / (2 * H_FD)
        err = np.max(np.abs(fd - g)) / (1.0 + np.max(np.abs(fd)))
        assert err < 1e-6, (name, err)
    return got


def test_dense_matches_finite_differences():
    rng = np.random.default_rng(41)
    check(case(rng), rng)


def test_varlen_with_reset_matches_finite_differences():
    rng = np.random.default_rng(42)
    c = case(rng, lengths=[3, 0, 7, 1])
    c["a"][4, 1] = np.inf  # an exact reset: log alpha = -inf, its own gradient is 0
    got = check(c, rng)
    assert got[3][4, 1] == 0.0
