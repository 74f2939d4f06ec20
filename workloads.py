"""Seeded synthetic inputs for the gated delta-rule workloads.

This module holds input recipes only -- none of the recurrence's arithmetic.  Both the CUDA path's
tests/benchmark and the fp64 oracle take their inputs from here, so each side sees the exact same
stored values (bf16 inputs are rounded once, here, and the oracle reads those rounded values).

Recipe (every draw from one CPU ``torch.Generator`` seeded per workload, in this order):
  varlen lengths  : integers uniform in [len_lo, len_hi]                        (varlen only)
  q, k            : N(0, 1) in fp32, L2-normalised per (token, head), then cast to the dtype
  v               : N(0, 1) in fp32, cast to the dtype
  beta            : beta_scale * sigmoid(N(0, 1))                                 fp32
  log_alpha       : -softplus(N(0, la_std)) * la_scale                            fp32 (<= 0)
  S0              : N(0, s0_std) fp32, or None when s0_std == 0
"N(0, s)" is read with s as the standard deviation.

Named workloads (sizes as the pages' hybrid-LM setting and the benchmark configurations fix them):
  tiny          B=1  T=256    H=2  d=64   fp32  (oracle-sized parity case)
  hybrid_lm     B=8  T=4096   H=12 d=64   bf16  log_alpha scaled by 0.1
  long_context  B=1  T=65536  H=16 d=128  bf16  log_alpha scaled by 0.1, S0 ~ N(0, 0.02)
  varlen        32 sequences, lengths U[128, 8192], H=16 d=128 bf16, beta in (0,2),
                log_alpha = -softplus(N(0, 2))
  decode        N=256 H=32 d=128 bf16, 1000 one-token steps, S0 ~ N(0, 0.02), log_alpha x 0.1
"""
from __future__ import annotations

import torch

DTYPES = {"bf16": torch.bfloat16, "f32": torch.float32}

CONFIGS = {
    "tiny": dict(kind="chunk", B=1, T=256, H=2, dk=64, dv=64, chunk=64, dtype="f32",
                 beta_scale=1.0, la_std=1.0, la_scale=1.0, s0_std=0.0, seed=1001),
    "hybrid_lm": dict(kind="chunk", B=8, T=4096, H=12, dk=64, dv=64, chunk=64, dtype="bf16",
                      beta_scale=1.0, la_std=1.0, la_scale=0.1, s0_std=0.0, seed=1002),
    "long_context": dict(kind="chunk", B=1, T=65536, H=16, dk=128, dv=128, chunk=64,
                         dtype="bf16", beta_scale=1.0, la_std=1.0, la_scale=0.1, s0_std=0.02,
                         seed=1003),
    "varlen": dict(kind="chunk", n_seqs=32, len_lo=128, len_hi=8192, H=16, dk=128, dv=128,
                   chunk=64, dtype="bf16", beta_scale=2.0, la_std=2.0, la_scale=1.0,
                   s0_std=0.0, seed=1004),
    # a smaller pack of the varlen workload's kind (for profiler captures of a few GB at most)
    "varlen_profile": dict(kind="chunk", n_seqs=32, len_lo=128, len_hi=2048, H=16, dk=128, dv=128,
                           chunk=64, dtype="bf16", beta_scale=2.0, la_std=2.0, la_scale=1.0,
                           s0_std=0.0, seed=1006),
    "decode": dict(kind="decode", N=256, H=32, dk=128, dv=128, steps=1000, dtype="bf16",
                   beta_scale=1.0, la_std=1.0, la_scale=0.1, s0_std=0.02, seed=1005),
}


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_chunk_inputs(B=None, T=None, H=2, dk=64, dv=64, dtype="bf16", seed=0, beta_scale=1.0,
                      la_std=1.0, la_scale=1.0, s0_std=0.0, lengths=None, n_seqs=None,
                      len_lo=None, len_hi=None, **_ignored):
    """Inputs for one chunk-forward call, as CPU tensors.

    Dense when ``lengths`` and ``n_seqs`` are None: q,k [B,T,H,dk], v [B,T,H,dv], gates [B,T,H].
    Varlen when ``lengths`` (list of ints) is given, or ``n_seqs`` with ``len_lo``/``len_hi``
    (drawn here): packed q,k [Ttot,H,dk] ..., ``cu_seqlens`` int32 [n+1].
    """
    g = torch.Generator().manual_seed(int(seed))
    dt = DTYPES[dtype]
    if n_seqs is not None and lengths is None:
        lengths = torch.randint(int(len_lo), int(len_hi) + 1, (int(n_seqs),), generator=g).tolist()
    if lengths is not None:
        lengths = [int(x) for x in lengths]
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
        lead = (int(cu[-1]),)
        nseq = len(lengths)
    else:
        cu = None
        lead = (int(B), int(T))
        nseq = int(B)
    q = _unit_rows(torch.randn(*lead, H, dk, generator=g)).to(dt)
    k = _unit_rows(torch.randn(*lead, H, dk, generator=g)).to(dt)
    v = torch.randn(*lead, H, dv, generator=g).to(dt)
    beta = (beta_scale * torch.sigmoid(torch.randn(*lead, H, generator=g))).float()
    log_alpha = (-torch.nn.functional.softplus(la_std * torch.randn(*lead, H, generator=g))
                 * la_scale).float()
    S0 = None
    if s0_std:
        S0 = (s0_std * torch.randn(nseq, H, dk, dv, generator=g)).float()
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S0=S0, cu_seqlens=cu,
                B=nseq, T=(lead[0] if cu is not None else int(T)), H=H, dk=dk, dv=dv,
                dtype=dtype, lengths=lengths)


def make_raw_chunk_inputs(B=None, T=None, H=2, dk=64, dv=64, dtype="bf16", seed=0, beta_scale=1.0,
                          la_std=1.0, la_scale=1.0, s0_std=0.0, lengths=None, n_seqs=None,
                          len_lo=None, len_hi=None, **_ignored):
    """Raw-projection inputs for the fused-prologue chunk forward: the same draws, in the same
    order and shapes, as ``make_chunk_inputs`` before any normalisation or gate activation.

    q_raw, k_raw ~ N(0, 1) cast to dtype (not normalised); v ~ N(0, 1) in dtype; b_raw ~ N(0, 1)
    and a_raw ~ N(0, la_std) in fp32; a_scale = la_scale and b_scale = beta_scale are the scales
    of the prologue's gate forms.
    """
    g = torch.Generator().manual_seed(int(seed))
    dt = DTYPES[dtype]
    if n_seqs is not None and lengths is None:
        lengths = torch.randint(int(len_lo), int(len_hi) + 1, (int(n_seqs),), generator=g).tolist()
    if lengths is not None:
        lengths = [int(x) for x in lengths]
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
        lead = (int(cu[-1]),)
        nseq = len(lengths)
    else:
        cu = None
        lead = (int(B), int(T))
        nseq = int(B)
    q_raw = torch.randn(*lead, H, dk, generator=g).to(dt)
    k_raw = torch.randn(*lead, H, dk, generator=g).to(dt)
    v = torch.randn(*lead, H, dv, generator=g).to(dt)
    b_raw = torch.randn(*lead, H, generator=g).float()
    a_raw = (la_std * torch.randn(*lead, H, generator=g)).float()
    S0 = None
    if s0_std:
        S0 = (s0_std * torch.randn(nseq, H, dk, dv, generator=g)).float()
    return dict(q_raw=q_raw, k_raw=k_raw, v=v, a_raw=a_raw, b_raw=b_raw, S0=S0, cu_seqlens=cu,
                a_scale=float(la_scale), b_scale=float(beta_scale), B=nseq,
                T=(lead[0] if cu is not None else int(T)), H=H, dk=dk, dv=dv, dtype=dtype,
                lengths=lengths)


def config_raw_inputs(name: str, **overrides):
    """Raw-projection inputs of a named chunk workload (see ``make_raw_chunk_inputs``)."""
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    assert cfg["kind"] == "chunk"
    return make_raw_chunk_inputs(**cfg)


def make_gva_chunk_inputs(B=None, T=None, Hk=2, Hv=4, dk=64, dv=64, dtype="bf16", seed=0,
                          beta_scale=1.0, la_std=1.0, la_scale=1.0, s0_std=0.0, lengths=None, **_ignored):
    """Inputs for a grouped-value-head chunk forward: q,k [..., Hk, dk] L2-normalised as in
    ``make_chunk_inputs``; v [..., Hv, dv]; gates [..., Hv]; S0 [B, Hv, dk, dv]."""
    g = torch.Generator().manual_seed(int(seed))
    dt = DTYPES[dtype]
    if lengths is not None:
        lengths = [int(x) for x in lengths]
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
        lead = (int(cu[-1]),)
        nseq = len(lengths)
    else:
        cu = None
        lead = (int(B), int(T))
        nseq = int(B)
    q = _unit_rows(torch.randn(*lead, Hk, dk, generator=g)).to(dt)
    k = _unit_rows(torch.randn(*lead, Hk, dk, generator=g)).to(dt)
    v = torch.randn(*lead, Hv, dv, generator=g).to(dt)
    beta = (beta_scale * torch.sigmoid(torch.randn(*lead, Hv, generator=g))).float()
    log_alpha = (-torch.nn.functional.softplus(la_std * torch.randn(*lead, Hv, generator=g))
                 * la_scale).float()
    S0 = (s0_std * torch.randn(nseq, Hv, dk, dv, generator=g)).float() if s0_std else None
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta, S0=S0, cu_seqlens=cu, B=nseq,
                T=(lead[0] if cu is not None else int(T)), Hk=Hk, H=Hv, dk=dk, dv=dv, dtype=dtype,
                lengths=lengths)


def make_phase_inputs(B=None, T=None, H=2, dk=32, dv=64, dtype="bf16", seed=0, beta_scale=1.0, la_scale=0.1,
                      m0_std=0.0, laplace=False, lengths=None, **_ignored):
    """Inputs of the complex-phase delta memory: K, Q complex64 [..., H, dk] unit phasors e^{i theta},
    theta ~ U[0, 2 pi) (K scaled by e^{sigma}, sigma ~ U[-0.5, 0] when ``laplace``); v [..., H, dv]
    N(0, 1) in dtype; beta = beta_scale * sigmoid(N(0, 1)); log_lam = -softplus(N(0, 1)) * la_scale
    (finite: lam > 0); M0 complex64 [B, H, dv, dk] with N(0, m0_std) parts, or None."""
    g = torch.Generator().manual_seed(int(seed))
    dt = DTYPES[dtype]
    if lengths is not None:
        lengths = [int(x) for x in lengths]
        cu = torch.zeros(len(lengths) + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0).to(torch.int32)
        lead = (int(cu[-1]),)
        nseq = len(lengths)
    else:
        cu = None
        lead = (int(B), int(T))
        nseq = int(B)
    two_pi = 6.283185307179586
    th_k = two_pi * torch.rand(*lead, H, dk, generator=g)
    th_q = two_pi * torch.rand(*lead, H, dk, generator=g)
    mag = torch.exp(-0.5 * torch.rand(*lead, H, dk, generator=g)) if laplace else torch.ones(*lead, H, dk)
    K = torch.polar(mag, th_k).to(torch.complex64)
    Q = torch.polar(torch.ones_like(th_q), th_q).to(torch.complex64)
    v = torch.randn(*lead, H, dv, generator=g).to(dt)
    beta = (beta_scale * torch.sigmoid(torch.randn(*lead, H, generator=g))).float()
    log_lam = (-torch.nn.functional.softplus(torch.randn(*lead, H, generator=g)) * la_scale).float()
    M0 = None
    if m0_std:
        M0 = torch.complex(m0_std * torch.randn(nseq, H, dv, dk, generator=g),
                           m0_std * torch.randn(nseq, H, dv, dk, generator=g)).to(torch.complex64)
    return dict(K=K, Q=Q, v=v, log_lam=log_lam, beta=beta, M0=M0, cu_seqlens=cu, B=nseq,
                T=(lead[0] if cu is not None else int(T)), H=H, dk=dk, dv=dv, dtype=dtype, lengths=lengths)


def make_phase_rowdecay_inputs(B=None, T=None, H=2, dk=32, dv=64, dtype="bf16", seed=0, beta_scale=1.0,
                               la_scale=0.1, lr_std=1.0, m0_std=0.0, laplace=False, lengths=None, **_ignored):
    """Inputs of the phase memory with one decay per value channel: the draws of
    ``make_phase_inputs`` (same seed, same order), then log_r [..., H, dv] =
    -softplus(N(0, lr_std)) * la_scale from the same generator (finite: r > 0).  The scalar
    log_lam is kept in the dict but unused by the per-channel form."""
    d = make_phase_inputs(B=B, T=T, H=H, dk=dk, dv=dv, dtype=dtype, seed=seed, beta_scale=beta_scale,
                          la_scale=la_scale, m0_std=m0_std, laplace=laplace, lengths=lengths)
    g = torch.Generator().manual_seed(int(seed) * 7 + 3)
    lead = tuple(d["v"].shape[:-2])
    d["log_r"] = (-torch.nn.functional.softplus(lr_std * torch.randn(*lead, H, dv, generator=g))
                  * la_scale).float()
    return d


def config_inputs(name: str, **overrides):
    """Inputs of a named chunk workload (``tiny``, ``hybrid_lm``, ``long_context``, ``varlen``)."""
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    assert cfg["kind"] == "chunk"
    return make_chunk_inputs(**cfg)


def make_decode_state(N, H, dk, dv, seed, s0_std=0.02):
    """Initial decode states [N,H,dk,dv] fp32 ~ N(0, s0_std)."""
    g = torch.Generator().manual_seed(int(seed))
    return (s0_std * torch.randn(N, H, dk, dv, generator=g)).float()


def make_decode_step_inputs(N, H, dk, dv, dtype="bf16", seed=0, step=0, beta_scale=1.0,
                            la_std=1.0, la_scale=1.0, **_ignored):
    """Inputs of decode step ``step``: q,k [N,H,dk], v [N,H,dv] in dtype; gates [N,H] fp32.

    Each step has its own generator (seeded from ``seed`` and ``step``), so any step can be
    regenerated without drawing the ones before it.
    """
    g = torch.Generator().manual_seed(int(seed) * 1_000_003 + int(step) + 1)
    dt = DTYPES[dtype]
    q = _unit_rows(torch.randn(N, H, dk, generator=g)).to(dt)
    k = _unit_rows(torch.randn(N, H, dk, generator=g)).to(dt)
    v = torch.randn(N, H, dv, generator=g).to(dt)
    beta = (beta_scale * torch.sigmoid(torch.randn(N, H, generator=g))).float()
    log_alpha = (-torch.nn.functional.softplus(la_std * torch.randn(N, H, generator=g))
                 * la_scale).float()
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta)


def make_raw_decode_step_inputs(N, H, dk, dv, dtype="bf16", seed=0, step=0, beta_scale=1.0, la_std=1.0,
                                la_scale=1.0, **_ignored):
    """Raw-projection inputs of decode step ``step`` for the fused decode entry: q_raw, k_raw
    ~ N(0, 1) [N,H,dk] and v ~ N(0, 1) [N,H,dv] in dtype; b_raw ~ N(0, 1) and a_raw ~ N(0, la_std)
    [N,H] fp32; a_scale = la_scale, b_scale = beta_scale.  One generator per step, as
    ``make_decode_step_inputs``."""
    g = torch.Generator().manual_seed(int(seed) * 1_000_003 + int(step) + 1)
    dt = DTYPES[dtype]
    q_raw = torch.randn(N, H, dk, generator=g).to(dt)
    k_raw = torch.randn(N, H, dk, generator=g).to(dt)
    v = torch.randn(N, H, dv, generator=g).to(dt)
    b_raw = torch.randn(N, H, generator=g).float()
    a_raw = (la_std * torch.randn(N, H, generator=g)).float()
    return dict(q_raw=q_raw, k_raw=k_raw, v=v, a_raw=a_raw, b_raw=b_raw, a_scale=float(la_scale),
                b_scale=float(beta_scale))
