"""fp64 prologue of the fused chunk forward: raw projections -> the recurrence's inputs.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Plain numpy, fp64, elementwise; the
recurrence itself is the sequential oracle ``oracle.forward``.

Forms (each a reading recorded with the library's design notes):
* beta_t = b_scale * sigmoid(b_t): DeltaPhase README, section 1 "Extended Householder Beta
  Range", writes beta_t = 2 sigmoid(W_beta x_t) for beta in (0, 2); b_scale = 1 gives (0, 1).
* log alpha_t = -a_scale * softplus(a_t): Sykra README, "Architectural Highlights", names a
  data-dependent forget gate alpha_t in (0, 1] without fixing its parametrisation; this is the
  plainest form with that range (a = +inf gives an exact reset).
* q_t, k_t divided by sqrt(|x|^2 + EPS): unit-norm keys and queries, as the workloads feed the
  plain entry point; EPS keeps an all-zero row at zero.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def softplus(x):
    """log(1 + e^x), written so that neither tail overflows."""
    x = _f64(x)
    with np.errstate(over="ignore", invalid="ignore"):
        return np.where(x > 0, x + np.log1p(np.exp(-np.abs(x))), np.log1p(np.exp(np.minimum(x, 0.0))))


def sigmoid(x):
    """1 / (1 + e^-x), written so that neither tail overflows."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def l2_normalize(x, eps=EPS):
    """Rows of the last axis divided by sqrt(sum of squares + eps)."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def gates(a_raw, b_raw, a_scale, b_scale):
    """(log_alpha, beta) from the raw gate projections."""
    a = _f64(a_raw)
    with np.errstate(invalid="ignore"):
        log_alpha = np.where(np.isposinf(a), -np.inf, -float(a_scale) * softplus(a))
    return log_alpha, float(b_scale) * sigmoid(b_raw)


def forward_fused(q_raw, k_raw, v, a_raw, b_raw, S0, a_scale, b_scale, cu_seqlens=None, units=None):
    """The sequential fp64 forward on the prologue's outputs (same layouts as ``oracle.forward``)."""
    import oracle
    log_alpha, beta = gates(a_raw, b_raw, a_scale, b_scale)
    return oracle.forward(l2_normalize(q_raw), l2_normalize(k_raw), v, log_alpha, beta, S0,
                          cu_seqlens=cu_seqlens, units=units)


def backward_fused(q_raw, k_raw, v, a_raw, b_raw, S0, dout, a_scale, b_scale, dS_final=None, cu_seqlens=None):
    """fp64 gradients of ``forward_fused`` with respect to its raw inputs: the backward oracle on the
    prologue's outputs, then the chain rule through the prologue, elementwise:
      q = x / n with n = sqrt(|x|^2 + EPS):   dx = (dq - q (q . dq)) / n   (the same for k);
      log alpha = -a_scale softplus(a):       da = -a_scale sigmoid(a) dlog_alpha;
      beta = b_scale sigmoid(b):              db = b_scale sigmoid(b) (1 - sigmoid(b)) dbeta.
    Returns (dq_raw, dk_raw, dv, da_raw, db_raw, dS0)."""
    import oracle
    xq, xk = _f64(q_raw), _f64(k_raw)
    q, k = l2_normalize(xq), l2_normalize(xk)
    log_alpha, beta = gates(a_raw, b_raw, a_scale, b_scale)
    dq, dk, dv, dla, dbe, dS0 = oracle.backward(q, k, v, log_alpha, beta, S0, dout, dS_final,
                                                cu_seqlens=cu_seqlens)

    def through_norm(x, y, dy):
        n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + EPS)
        return (dy - y * np.sum(y * dy, axis=-1, keepdims=True)) / n

    a = _f64(a_raw)
    sa = sigmoid(a)
    sb = sigmoid(b_raw)
    with np.errstate(invalid="ignore"):
        da = np.where(np.isposinf(a), 0.0, -float(a_scale) * sa * dla)
    db = float(b_scale) * sb * (1.0 - sb) * dbe
    return through_norm(xq, q, dq), through_norm(xk, k, dk), dv, da, db, dS0
