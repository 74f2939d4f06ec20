"""Helpers for the GPU parity tests: run the CUDA path through the binding and the oracle on the
same seeded inputs, and measure max-abs differences.  Tolerances (max-abs on outputs and final
states): 2e-2 for bf16 inputs with fp32 accumulation, 1e-4 for fp32 inputs."""
import numpy as np
import torch

import oracle

TOL = {"bf16": 2e-2, "f32": 1e-4}


def to_dev(inp, device="cuda"):
    d = {}
    for key in ("q", "k", "v", "log_alpha", "beta", "S0", "cu_seqlens"):
        t = inp.get(key)
        d[key] = None if t is None else t.to(device).contiguous()
    return d


def run_gpu_chunk(inp, S_final=True, **kw):
    import linear_attention_sequence_rule_b200 as gdn
    d = to_dev(inp)
    out, Sf = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"],
                            cu_seqlens=d["cu_seqlens"], output_final_state=S_final, **kw)
    gdn.device_status()  # synchronises; raises if a device-side wait ran out
    return out, Sf


def run_oracle_chunk(inp, units=None):
    return oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                          cu_seqlens=inp["cu_seqlens"], units=units)


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def max_abs(a, b):
    a = np.asarray(a)
    b = np.asarray(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    if a.size == 0:
        return 0.0
    return float(np.max(np.abs(a - b)))


def unit_slices(inp, units):
    """Index helpers to pull the outputs of (sequence, head) units out of dense/varlen layouts."""
    H = inp["H"]
    cu = inp["cu_seqlens"]
    res = []
    for u in units:
        s, h = divmod(int(u), H)
        if cu is None:
            res.append((s, h, (s, slice(None), h)))
        else:
            res.append((s, h, (slice(int(cu[s]), int(cu[s + 1])), h)))
    return res


def compare_chunk(inp, out_gpu, Sf_gpu, units=None):
    """Max-abs errors (out, S_final) of the GPU result against the oracle on `units` (all if None)."""
    o_ref, s_ref = run_oracle_chunk(inp, units)
    og, sg = f64(out_gpu), (f64(Sf_gpu) if Sf_gpu is not None else None)
    if units is None:
        e_o = max_abs(og, o_ref)
        e_s = max_abs(sg, s_ref) if sg is not None else 0.0
        return e_o, e_s
    e_o = e_s = 0.0
    for s, h, idx in unit_slices(inp, units):
        e_o = max(e_o, max_abs(og[idx], o_ref[idx]))
        if sg is not None:
            e_s = max(e_s, max_abs(sg[s, h], s_ref[s, h]))
    return e_o, e_s
