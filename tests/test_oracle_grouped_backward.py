"""Pin of the grouped-value-head backward oracle (oracle/grouped.py, backward_gva): every gradient
element against central finite differences of forward_gva, dense and varlen, G = 3.  CPU only."""
import numpy as np

from oracle import grouped

H_FD = 1e-6


def test_matches_finite_differences():
    rng = np.random.default_rng(71)
    for lengths in (None, [4, 0, 6]):
        lead = (2, 5) if lengths is None else (int(sum(lengths)),)
        nseq = 2 if lengths is None else len(lengths)
        Hk, G, dk, dv = 2, 3, 3, 2
        Hv = Hk * G
        c = dict(q=rng.normal(size=(*lead, Hk, dk)), k=rng.normal(size=(*lead, Hk, dk)),
                 v=rng.normal(size=(*lead, Hv, dv)), la=-np.log1p(np.exp(rng.normal(size=(*lead, Hv)))),
                 be=1.8 / (1.0 + np.exp(-rng.normal(size=(*lead, Hv)))), S0=rng.normal(size=(nseq, Hv, dk, dv)))
        c["k"] /= np.linalg.norm(c["k"], axis=-1, keepdims=True)
        cu = None if lengths is None else np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        Go = rng.normal(size=c["v"].shape)
        W = rng.normal(size=c["S0"].shape)

        def loss():
            o, S = grouped.forward_gva(c["q"], c["k"], c["v"], c["la"], c["be"], c["S0"], cu_seqlens=cu)
            return float(np.sum(o * Go) + np.sum(S * W))
        got = grouped.backward_gva(c["q"], c["k"], c["v"], c["la"], c["be"], c["S0"], Go, W, cu_seqlens=cu)
        for name, g in zip(("q", "k", "v", "la", "be", "S0"), got):
            x = c[name]
            fd = np.zeros_like(x)
            for i in np.ndindex(x.shape):
                old = x[i]
                x[i] = old + H_FD
                lp = loss()
                x[i] = old - H_FD
                lm = loss()
                x[i] = old
                fd[i] = (lp - lm) / (2 * H_FD)
            assert np.max(np.abs(fd - g)) / (1.0 + np.max(np.abs(fd))) < 1e-6, name
