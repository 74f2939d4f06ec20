"""Pins of the fp64 backward oracle: every gradient element against central finite differences of
the (separately pinned) forward oracle, on dense and varlen inputs with exact resets, beta = 2
and a nonzero initial state; plus mutants of the backward, each caught by the finite-difference
check.  CPU only."""
import os
import subprocess

import numpy as np
import pytest

import oracle

H_FD = 1e-5


def rand_case(rng, B=2, T=7, H=2, dk=4, dv=3, lengths=None):
    lead = (int(sum(lengths)),) if lengths is not None else (B, T)
    nseq = len(lengths) if lengths is not None else B
    q = rng.normal(size=(*lead, H, dk))
    k = rng.normal(size=(*lead, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.normal(size=(*lead, H, dv))
    la = -np.log1p(np.exp(rng.normal(size=(*lead, H))))
    be = 2.0 / (1.0 + np.exp(-rng.normal(size=(*lead, H))))
    S0 = 0.5 * rng.normal(size=(nseq, H, dk, dv))
    cu = None
    if lengths is not None:
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=be, S0=S0, cu_seqlens=cu)


def loss(c, Go, Gs):
    out, Sf = oracle.forward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["S0"],
                             cu_seqlens=c["cu_seqlens"], nthreads=1)
    return float(np.sum(out * Go) + np.sum(Sf * Gs))


def fd_check(c, rng, skip=()):
    """Max relative error of the analytic gradients against central differences, per input."""
    out, Sf = oracle.forward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["S0"], cu_seqlens=c["cu_seqlens"])
    Go, Gs = rng.normal(size=out.shape), rng.normal(size=Sf.shape)
    grads = dict(zip(("q", "k", "v", "log_alpha", "beta", "S0"),
                     oracle.backward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["S0"], Go, Gs,
                                     cu_seqlens=c["cu_seqlens"])))
    errs = {}
    for name, g in grads.items():
        x = c[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            if (name, idx) in skip or not np.isfinite(x[idx]):
                fd[idx] = g[idx]
                continue
            x0 = x[idx]
            x[idx] = x0 + H_FD
            lp = loss(c, Go, Gs)
            x[idx] = x0 - H_FD
            lm = loss(c, Go, Gs)
            x[idx] = x0
            fd[idx] = (lp - lm) / (2 * H_FD)
        errs[name] = float(np.max(np.abs(fd - g) / (1.0 + np.abs(fd))))
    return errs, grads


def test_dense_gradients_match_finite_differences():
    rng = np.random.default_rng(1)
    c = rand_case(rng)
    errs, _ = fd_check(c, rng)
    assert max(errs.values()) < 1e-7, errs


def test_varlen_resets_and_householder_gradients():
    rng = np.random.default_rng(2)
    c = rand_case(rng, H=1, lengths=[5, 0, 6])
    c["log_alpha"][2, 0] = -np.inf   # exact reset inside the first sequence
    c["log_alpha"][7, 0] = 0.0       # alpha = 1 ...
    c["beta"][7, 0] = 2.0            # ... with beta = 2: a Householder reflection
    errs, grads = fd_check(c, rng)
    assert max(errs.values()) < 1e-7, errs
    assert grads["log_alpha"][2, 0] == 0.0
    # the reset makes everything before it irrelevant to the outputs after it; the gradient of
    # the first sequence's tokens 0-1 comes only from their own outputs
    assert np.all(np.isfinite(grads["q"])) and np.all(np.isfinite(grads["S0"]))


SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")
MUTANTS = {
    "dk_correction_sign": ("- a * b * Sp[(size_t)i * dv + j] * r[j]", "+ a * b * Sp[(size_t)i * dv + j] * r[j]"),
    "dbeta_without_gate": ("db += r[j] * (vt[j] - a * u[j]);", "db += r[j] * (vt[j] - u[j]);"),
    "state_grad_missing_beta": ("a * (G[(size_t)i * dv + j] - b * kt[i] * r[j])", "a * (G[(size_t)i * dv + j] - kt[i] * r[j])"),
    "readout_grad_with_previous_state": ("acc += S_t[(size_t)i * dv + j] * dot[j];", "acc += Sp[(size_t)i * dv + j] * dot[j];"),
    "dalpha_not_times_alpha": ("0.0 : a * da;", "0.0 : da;"),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_backward_mutants_are_caught(tmp_path, name, monkeypatch):
    src = open(SRC).read()
    a, b = MUTANTS[name]
    assert src.count(a) == 1, name
    c_file = tmp_path / "m.c"
    so = tmp_path / "libm.so"
    c_file.write_text(src.replace(a, b))
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c_file), "-lm"],
                   check=True)
    import ctypes
    monkeypatch.setattr(oracle, "_lib", None)
    monkeypatch.setattr(oracle, "_LIB", str(so))
    monkeypatch.setattr(oracle, "build", lambda force=False: str(so))
    rng = np.random.default_rng(3)
    errs, _ = fd_check(rand_case(rng, B=1, T=5, H=1), rng)
    assert max(errs.values()) > 1e-4, (name, errs)
