"""Per-workload parity report: max-abs errors of the CUDA path against the fp64 oracle on the
named workloads at full size, and the oracle's own wall time on the host cores.

Run on a machine with a GPU:  python -m tests.parity_report
Prints a markdown table.  The chunk workloads compare every (sequence, head) chain; the decode
workload compares a seeded sample of 64 of its 8,192 states over all 1,000 steps (the oracle
would take minutes for all of them).
"""
import time

import numpy as np
import torch

import oracle
import workloads
from tests.parity import compare_chunk, f64, max_abs, run_gpu_chunk
from tests.test_gpu_decode import run_steps


def chunk_row(name):
    inp = workloads.config_inputs(name)
    out, Sf = run_gpu_chunk(inp)
    t0 = time.perf_counter()
    o_ref, s_ref = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                  inp["S0"], cu_seqlens=inp["cu_seqlens"])
    dt = time.perf_counter() - t0
    e_o = max_abs(f64(out), o_ref)
    e_s = max_abs(f64(Sf), s_ref)
    tokens = int(inp["cu_seqlens"][-1]) if inp["cu_seqlens"] is not None else inp["B"] * inp["T"]
    return dict(name=name, e_o=e_o, e_s=e_s, cpu_s=dt, units=f"{inp['B'] * inp['H']} of "
                f"{inp['B'] * inp['H']} chains", cpu_rate=tokens / dt, rate_unit="tokens/s")


def decode_row():
    cfg = workloads.CONFIGS["decode"]
    N, H, dk, dv, steps = cfg["N"], cfg["H"], cfg["dk"], cfg["dv"], cfg["steps"]
    units = sorted(np.random.default_rng(5).choice(N * H, size=64, replace=False).tolist())
    t0 = time.perf_counter()
    e_o, e_s = run_steps(N, H, dk, dv, cfg["dtype"], steps, cfg["seed"], units=units)
    dt = time.perf_counter() - t0  # GPU steps and the oracle on 64 states; the oracle dominates
    return dict(name="decode", e_o=e_o, e_s=e_s, cpu_s=dt, units=f"64 of {N * H} states, {steps} steps",
                cpu_rate=64 * steps / dt, rate_unit="state-updates/s")


def main():
    torch.cuda.init()
    rows = [chunk_row(n) for n in ("tiny", "hybrid_lm", "long_context", "varlen")] + [decode_row()]
    print(f"oracle threads: {oracle.max_threads()}")
    print("| workload | max-abs err out | max-abs err final state | compared | oracle wall time | oracle rate |")
    print("|---|---|---|---|---|---|")
    for r in rows:
        print(f"| {r['name']} | {r['e_o']:.2e} | {r['e_s']:.2e} | {r['units']} | {r['cpu_s']:.2f} s | "
              f"{r['cpu_rate']:.3g} {r['rate_unit']} |")


if __name__ == "__main__":
    main()
