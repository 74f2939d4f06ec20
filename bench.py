"""Benchmark of the gated delta-rule library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick]

One step = one gdn_chunk_fwd over the varlen packed prefill batch (32 sequences with lengths
uniform in [128, 8192], H=16, dk=dv=128, chunk 64, bf16 q/k/v, beta in (0, 2), strong decays
log_alpha = -softplus(N(0, 2)) with some alpha near 0, fp32 gates and state), the largest of the single-GPU prefill
workloads: the whole chunkwise path (gates, intra-chunk products, triangular inverse, state
chain, outputs, final states) in the library's kernels.  Inputs are synthetic (seeded, see
workloads.py) and resident in HBM before timing; the inputs are larger than L2 and L2 is flushed
(a 256 MB device write) between timed steps as well.  Rank 0 prints one JSON line.  The line
also reports, each with its own roofline and CPU baseline, the hybrid-LM prefill batch (B=8,
T=4096, H=12, d=64), the long-context prefill (B=1, T=65536, H=16, d=128) and the decode workload
(N=256, H=32, d=128, 1000 steps; state-updates/s, HBM fraction by algorithmic and by DRAM bytes).

With --gpus N (under torchrun) every rank runs its own batch (independent sequences need no
exchange): weak scaling, time = max over ranks.  --impl reference times the fp64 CPU oracle on
the host cores on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "gated-delta chunk-fwd tokens/s & % roofline; decode state-updates/s & HBM %"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "chunk": "linear_attention_sequence_rule_b200/csrc/gdn_chunk_tc.cu",
    "decode": "linear_attention_sequence_rule_b200/csrc/gdn_decode.cu",
}


# ---- algorithmic work (per token-head, chunk C = 64; a multiply-add counts 2 flops) -----------

def algo_bytes(token_heads, n_states, dk, dv, elem, has_s0, has_sfinal):
    b = token_heads * (elem * (2 * dk + 2 * dv) + 8)
    b += n_states * 4 * dk * dv * (int(has_s0) + int(has_sfinal))
    return b


def algo_flops(token_heads, dk, dv, C=64):
    return token_heads * ((3 * C - 1) * dk + 2 * C * dv + C * C / 3 + 6 * dk * dv)


DECODE_BYTES_PER_STATE = lambda dk, dv, e: 8 * dk * dv + e * (2 * dk + 2 * dv) + 8


# dense tf32 : bf16 tensor throughput, nominal (1.1 and 2.25 PFLOP/s per GPU): the tf32 peak is the
# measured bf16 peak scaled by it
TF32_PER_BF16 = 1.1 / 2.25


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    sha = source_sha(KERNEL_SOURCES[kernel_key])
    for line in open(p):
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("kernel") == kernel_key and f.get("workload") == workload and f.get("sha") == sha:
            return float(f["dram_bytes_per_launch"])
    return None


# ---- clocks during the timed region (NVML reads only) -------------------------------------

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, index, period=0.005):
        self.ok = False
        self.samples, self.reasons = [], set()
        self.period = period
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def result(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---- distributed plumbing ------------------------------------------------------------------

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device=None):
    """Max of a per-rank number over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed, rank):
    """Every rank runs its own independent batch (weak scaling), drawn with its own seed."""
    return int(base_seed) + 7919 * int(rank)


def aggregate_tokens_per_s(tokens_per_rank, world, ms_max):
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)


# ---- our arm -------------------------------------------------------------------------------

def to_dev(inp):
    return {k: (v.cuda().contiguous() if torch.is_tensor(v) else v) for k, v in inp.items()}


def chunk_workspace(gdn, d):
    """The workspace a chunk call needs (the segment scan of long dense sequences), or None."""
    n = gdn.workspace_bytes(d["B"], d["T"], d["H"], d["dk"], d["dv"], d["cu_seqlens"] is not None,
                            d["q"].dtype)
    return torch.empty(n, dtype=torch.uint8, device="cuda") if n else None


def chunk_launches(gdn, d):
    """Kernels one chunk call launches: one chunk kernel, or with the segment scan a segment table,
    two local passes, the combine and the output pass."""
    return 5 if chunk_workspace(gdn, d) is not None else 1


def time_chunk(gdn, d, steps, warmup, flush, stream):
    """Per-step CUDA-event time (ms) of gdn.chunk_fwd, L2 flushed before every step."""
    out = torch.empty_like(d["v"])
    Sf = torch.empty((d["B"], d["H"], d["dk"], d["dv"]), dtype=torch.float32, device="cuda")
    ws = chunk_workspace(gdn, d)
    call = lambda: gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"],
                                 cu_seqlens=d["cu_seqlens"], out=out, S_final=Sf, workspace=ws,
                                 stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush.zero_()
            call()
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for s, e in ev:
            flush.zero_()
            s.record(stream)
            call()
            e.record(stream)
        stream.synchronize()
    return [s.elapsed_time(e) for s, e in ev]


def gdn_mod():
    import linear_attention_sequence_rule_b200 as gdn
    return gdn


def time_prologue(gdn, d, steps, warmup, flush, stream, fused):
    """Per-step CUDA-event time (ms) from raw projections to outputs: the fused entry, or PyTorch
    normalisation and activations (separate kernels, one more HBM pass over q, k and the gates)
    followed by the plain entry."""
    out = torch.empty_like(d["v"])
    Sf = torch.empty((d["B"], d["H"], d["dk"], d["dv"]), dtype=torch.float32, device="cuda")
    ws = chunk_workspace(gdn, d | {"q": d["q_raw"]})

    def unfused_prologue():
        qf, kf = d["q_raw"].float(), d["k_raw"].float()
        q = (qf * torch.rsqrt((qf * qf).sum(-1, keepdim=True) + 1e-6)).to(d["q_raw"].dtype)
        k = (kf * torch.rsqrt((kf * kf).sum(-1, keepdim=True) + 1e-6)).to(d["k_raw"].dtype)
        la = -d["a_scale"] * torch.nn.functional.softplus(d["a_raw"])
        be = d["b_scale"] * torch.sigmoid(d["b_raw"])
        return q, k, la, be

    def call():
        if fused:
            gdn.chunk_fwd_fused(d["q_raw"], d["k_raw"], d["v"], d["a_raw"], d["b_raw"], d["a_scale"],
                                d["b_scale"], S0=d["S0"], cu_seqlens=d["cu_seqlens"], out=out, S_final=Sf,
                                workspace=ws, stream=stream)
        else:
            q, k, la, be = unfused_prologue()
            gdn.chunk_fwd(q, k, d["v"], la, be, S0=d["S0"], cu_seqlens=d["cu_seqlens"], out=out,
                          S_final=Sf, workspace=ws, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush.zero_()
            call()
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for s0, e in ev:
            flush.zero_()
            s0.record(stream)
            call()
            e.record(stream)
        stream.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def chunk_numbers(name, d, times_ms, peaks):
    ms = statistics.mean(times_ms)
    th = d["q"].shape[0] * (d["q"].shape[1] if d["cu_seqlens"] is None else 1) * d["H"]
    tokens = th // d["H"]
    elem = d["q"].element_size()
    by = algo_bytes(th, d["B"] * d["H"], d["dk"], d["dv"], elem, d["S0"] is not None, True)
    fl = algo_flops(th, d["dk"], d["dv"])
    gbs = by / (ms * 1e-3) / 1e9
    tfs = fl / (ms * 1e-3) / 1e12
    return dict(workload=name, ms=ms, tokens=tokens, tokens_per_s=tokens / (ms * 1e-3),
                launches_per_call=chunk_launches(gdn_mod(), d),
                algo_bytes=by, algo_flops=fl, gbs=gbs, hbm_frac=gbs / peaks["hbm_gbs"],
                tflops=tfs, tensor_frac=tfs / peaks["bf16_tflops"])


WIDE_VALUE = "hybrid_lm tokens and heads (B=8 T=4096 H=12) at dk=128, dv=256: two 128-column CTAs per chain"


def wide_value_inputs(seed=0):
    """The hybrid-LM token and head counts at head sizes dk=128, dv=256 (bf16), on the device."""
    return to_dev(workloads.make_chunk_inputs(B=8, T=4096, H=12, dk=128, dv=256, dtype="bf16", seed=seed,
                                              la_scale=0.1))


def time_decode(gdn, steps, warmup, stream, pool=32, fused=False):
    """The decode workload's steps (CUDA events per step); fused: from raw projections through
    gdn_decode_step_fused (same bytes: raw q/k and gates replace the prepared ones)."""
    cfg = workloads.CONFIGS["decode"]
    N, H, dk, dv = cfg["N"], cfg["H"], cfg["dk"], cfg["dv"]
    S = workloads.make_decode_state(N, H, dk, dv, cfg["seed"]).cuda()
    make = workloads.make_raw_decode_step_inputs if fused else workloads.make_decode_step_inputs
    xs = [{k: (v.cuda() if torch.is_tensor(v) else v)
           for k, v in make(N, H, dk, dv, cfg["dtype"], seed=cfg["seed"], step=i, la_scale=cfg["la_scale"]).items()}
          for i in range(pool)]
    out = torch.empty((N, H, dv), dtype=torch.bfloat16, device="cuda")
    if fused:
        call = lambda x: gdn.decode_step_fused(x["q_raw"], x["k_raw"], x["v"], x["a_raw"], x["b_raw"], x["a_scale"],
                                               x["b_scale"], S, out=out, stream=stream)
    else:
        call = lambda x: gdn.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S,
                                         out=out, stream=stream)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            call(xs[i % pool])
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i, (s, e) in enumerate(ev):
            s.record(stream)
            call(xs[i % pool])
            e.record(stream)
        stream.synchronize()
    t = [s.elapsed_time(e) for s, e in ev]
    ms = statistics.mean(t)
    by = N * H * DECODE_BYTES_PER_STATE(dk, dv, 2)
    name = f"decode N={N} H={H} dk=dv={dk} bf16, fp32 state" + (", from raw projections (fused entry)" if fused else "")
    return dict(workload=name, steps=steps,
                input_pool=pool, ms_per_step=ms, state_updates_per_s=N * H / (ms * 1e-3),
                tokens_per_s=N / (ms * 1e-3), algo_bytes_per_step=by,
                gbs=by / (ms * 1e-3) / 1e9)


def e2e_chunk(gdn, inp, steps, warmup, stream):
    """Same workload through the public host-memory call (gdn_chunk_fwd_host): every step copies
    the inputs up from page-locked host memory, runs the forward and copies out and S_final back
    down, all inside the timed region (the library overlaps the copies of one part of the batch
    with the compute and the opposite-direction copies of the others)."""
    host = {k: (v.contiguous().pin_memory() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out_h = torch.empty(inp["v"].shape, dtype=inp["v"].dtype).pin_memory()
    sf_h = torch.empty((inp["B"], inp["H"], inp["dk"], inp["dv"]), dtype=torch.float32).pin_memory()
    keys = [k for k in ("q", "k", "v", "log_alpha", "beta", "S0", "cu_seqlens") if host.get(k) is not None]
    h2d = sum(host[k].numel() * host[k].element_size() for k in keys)
    d2h = out_h.numel() * out_h.element_size() + sf_h.numel() * 4
    B, T = (inp["B"], inp["T"]) if host.get("cu_seqlens") is None else (inp["B"], int(inp["cu_seqlens"][-1]))
    need = gdn.gdn_chunk_fwd_host_workspace_bytes(B, T, inp["H"], inp["dk"], inp["dv"], 64,
                                                  int(host.get("cu_seqlens") is not None), gdn._DT[inp["v"].dtype])
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")

    def step():
        gdn.chunk_fwd_host(host["q"], host["k"], host["v"], host["log_alpha"], host["beta"], S0=host.get("S0"),
                           cu_seqlens=host.get("cu_seqlens"), out=out_h, S_final=sf_h, workspace=ws,
                           stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
        stream.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(steps):
            step()
        e.record(stream)
        stream.synchronize()
    ms = s.elapsed_time(e) / steps
    del ws
    return ms, h2d, d2h


def oracle_subproblem(inp, seqs):
    """fp64 host copies of the given sequences of a workload (all their heads), packed as a varlen
    batch: (q, k, v, log_alpha, beta, S0, cu_seqlens) and the token-heads they hold.  Built
    outside the timed regions, so that the CPU legs time the recurrence rather than a conversion
    of the whole workload to fp64 on every call."""
    import numpy as np
    H = inp["H"]
    seqs = list(seqs)
    f64 = lambda x: x.detach().to("cpu", torch.float64).numpy()
    if inp["cu_seqlens"] is None:
        T = inp["T"]
        pick = lambda x: f64(x[seqs].reshape(len(seqs) * T, *x.shape[2:]))
        lengths = [T] * len(seqs)
    else:
        cu = inp["cu_seqlens"]
        spans = [(int(cu[b]), int(cu[b + 1])) for b in seqs]
        pick = lambda x: f64(torch.cat([x[a:e] for a, e in spans]))
        lengths = [e - a for a, e in spans]
    cu_sub = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    S0 = None if inp["S0"] is None else f64(inp["S0"][seqs])
    args = (pick(inp["q"]), pick(inp["k"]), pick(inp["v"]), pick(inp["log_alpha"]), pick(inp["beta"]), S0,
            cu_sub)
    return args, H * int(sum(lengths))


def cpu_oracle_baseline(inp, budget_s=12.0):
    """Time the fp64 oracle, as it stands, on the host cores over whole sequences (every head of
    each: H independent chains per sequence) of the workload until about budget_s seconds of work;
    returns tokens/s and the sample."""
    import oracle
    H = inp["H"]
    threads = oracle.max_threads()
    # first a small probe (the first sequence) to size the sample
    sub, th = oracle_subproblem(inp, [0])
    t0 = time.perf_counter()
    oracle.forward(*sub[:6], cu_seqlens=sub[6])
    dt = time.perf_counter() - t0
    per_th = dt / th
    cu = inp["cu_seqlens"]
    lengths = [inp["T"]] * inp["B"] if cu is None else [int(cu[b + 1] - cu[b]) for b in range(inp["B"])]
    m, acc = 0, 0.0
    while m < inp["B"] and (m == 0 or acc + H * lengths[m] * per_th <= budget_s):
        acc += H * lengths[m] * per_th
        m += 1
    if m > 1:  # else the probe was the sample
        sub, th = oracle_subproblem(inp, range(m))
        t0 = time.perf_counter()
        oracle.forward(*sub[:6], cu_seqlens=sub[6])
        dt = time.perf_counter() - t0
    return dict(value=(th / H) / dt, unit="tokens/s", cores=threads, kind="oracle",
                sample=f"{m} of {inp['B']} sequences, every head of each ({m * H} of {inp['B'] * H} "
                       f"(sequence, head) chains, {th} token-heads = {th / H:.0f} tokens, {dt:.2f} s, "
                       f"fp64 sequential recurrence; inputs converted to fp64 before the timing)")


def cpu_decode_baseline(states=512, steps=200):
    """The fp64 decode oracle, as it stands, on the host cores: `steps` steps of a sample of
    `states` of the decode workload's states; returns state-updates/s and the sample."""
    import oracle
    cfg = workloads.CONFIGS["decode"]
    N, H, dk, dv = cfg["N"], cfg["H"], cfg["dk"], cfg["dv"]
    sel = list(range(states))
    S = workloads.make_decode_state(N, H, dk, dv, cfg["seed"]).double().numpy().reshape(N * H, dk, dv)
    S = S[sel][:, None]
    xs = []
    for step in range(steps):
        x = workloads.make_decode_step_inputs(N, H, dk, dv, cfg["dtype"], seed=cfg["seed"], step=step,
                                              la_scale=cfg["la_scale"])
        xs.append({k: v.reshape(N * H, *v.shape[2:])[sel][:, None] for k, v in x.items()})
    t0 = time.perf_counter()
    for x in xs:
        _, S = oracle.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
    dt = time.perf_counter() - t0
    return dict(value=states * steps / dt, unit="state-updates/s", cores=oracle.max_threads(), kind="oracle",
                sample=f"{states} of {N * H} states x {steps} of {cfg['steps']} steps "
                       f"({dt:.2f} s, fp64 sequential update)")


HEADLINE = "varlen"
WORKLOAD_TEXT = {
    "varlen": "varlen packed prefill chunk forward: 32 sequences, lengths U[128,8192] (seeded draw), "
              "H=16 dk=dv=128 chunk=64, bf16 q/k/v/out, fp32 gates and state, beta=2 sigmoid(N(0,1)), "
              "log_alpha=-softplus(N(0,2)), S0=0",
    "hybrid_lm": "hybrid_lm prefill chunk forward: B=8 T=4096 H=12 dk=dv=64 chunk=64, bf16 q/k/v/out, "
                 "fp32 gates and state, beta=sigmoid(N(0,1)), log_alpha=-0.1 softplus(N(0,1)), S0=0",
    "long_context": "long-context prefill chunk forward: B=1 T=65536 H=16 dk=dv=128 chunk=64, bf16 q/k/v/out, "
                    "fp32 gates and state, beta=sigmoid(N(0,1)), log_alpha=-0.1 softplus(N(0,1)), "
                    "S0~N(0,0.02), final state returned",
}


def headline_config(world):
    """The `config` object of the JSON line, identical in both arms."""
    cfg = workloads.CONFIGS[HEADLINE]
    return {"workload": WORKLOAD_TEXT[HEADLINE],
            "global_batch": cfg["n_seqs"] * world, "seq_len": f"U[{cfg['len_lo']},{cfg['len_hi']}]",
            "heads": cfg["H"], "head_dim": cfg["dk"],
            "parallelism": f"dp{world} (independent sequences per rank)",
            "l2": "inputs larger than L2 (126 MB); the GPU arm also flushes L2 (256 MB device write) "
                  "between timed steps"}


def roofline_obj(nums, peaks, peak_kind, traffic):
    return {"bound": "hbm", "achieved": nums["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": nums["gbs"] / peaks["hbm_gbs"], "traffic": traffic,
            "peak_source": f"{peak_kind} hbm_gbs", "algo_bytes_per_launch": nums["algo_bytes"]}


def tensor_obj(nums, peaks):
    return {"achieved_tflops": nums["tflops"], "peak_tflops": peaks["bf16_tflops"],
            "frac": nums["tensor_frac"], "algo_flops_per_launch": nums["algo_flops"]}


def run_ours(args, world, rank, local):
    import linear_attention_sequence_rule_b200 as gdn
    peaks, peak_kind = load_peaks()
    stream = torch.cuda.Stream()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    name = HEADLINE
    cfg = workloads.CONFIGS[name]
    inp = workloads.config_inputs(name, seed=rank_seed(cfg["seed"], rank))
    d = to_dev(inp)

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        times = time_chunk(gdn, d, args.steps, args.warmup, flush, stream)
    torch.cuda.synchronize()
    barrier(world)
    ms_local = statistics.mean(times)
    ms = max_over_ranks(ms_local, world)
    main = chunk_numbers(name, d, times, peaks)
    tokens_all = main["tokens"] * world
    value = aggregate_tokens_per_s(main["tokens"], world, ms)
    del d

    e2e_ms, h2d, d2h = e2e_chunk(gdn, inp, max(3, args.steps // 10), 3, stream)
    e2e_ms = max_over_ranks(e2e_ms, world)

    others = {}
    decode = None
    extra = {}
    if not args.quick:
        # the other prefill workloads, each with its own roofline (CPU baselines below)
        for w in ("hybrid_lm", "long_context"):
            cw = workloads.CONFIGS[w]
            dw = to_dev(workloads.config_inputs(w, seed=rank_seed(cw["seed"], rank)))
            tw = time_chunk(gdn, dw, max(3, args.steps // 2 if w == "hybrid_lm" else args.steps // 4), 3,
                            flush, stream)
            nums = chunk_numbers(w, dw, tw, peaks)
            nums["workload"] = WORKLOAD_TEXT[w]
            nums["roofline"] = roofline_obj(nums, peaks, peak_kind, ncu_traffic("chunk", w))
            nums["tensor"] = tensor_obj(nums, peaks)
            others[w] = {k: (round(v, 6) if isinstance(v, float) else v) for k, v in nums.items()}
            del dw
        decode = time_decode(gdn, 1000, 10, stream)
        decode["hbm_frac"] = decode["gbs"] / peaks["hbm_gbs"]
        # DRAM bytes per step from the ncu record of the current decode source (null once it
        # changed): part of the state stream is served by L2, so the DRAM-side fraction is lower
        decode["traffic"] = ncu_traffic("decode", "decode")
        if decode["traffic"]:
            decode["dram_gbs"] = decode["traffic"] / (decode["ms_per_step"] * 1e-3) / 1e9
            decode["dram_hbm_frac"] = decode["dram_gbs"] / peaks["hbm_gbs"]
        decode["roofline"] = {"bound": "hbm", "achieved": decode["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": decode["hbm_frac"], "traffic": decode["traffic"],
                              "peak_source": f"{peak_kind} hbm_gbs",
                              "algo_bytes_per_launch": decode["algo_bytes_per_step"],
                              "frac_by_dram_bytes": decode.get("dram_hbm_frac")}
        dfu = time_decode(gdn, 300, 10, stream, fused=True)
        extra["decode_fused"] = {k: (round(v, 6) if isinstance(v, float) else v) for k, v in dfu.items()}
        extra["decode_fused"]["hbm_frac"] = round(dfu["gbs"] / peaks["hbm_gbs"], 5)
        hl = workloads.CONFIGS["hybrid_lm"]
        dw = wide_value_inputs(rank_seed(hl["seed"], rank))
        nums = chunk_numbers(WIDE_VALUE, dw, time_chunk(gdn, dw, max(3, args.steps // 2), 3, flush, stream), peaks)
        extra["hybrid_lm_dv256"] = {k: (round(v, 6) if isinstance(v, float) else v) for k, v in nums.items()}
        del dw
        # the hybrid-LM step from raw projections: fused prologue vs PyTorch prologue + call
        dr = to_dev(workloads.config_raw_inputs("hybrid_lm", seed=rank_seed(hl["seed"], rank)))
        for key, fused in (("hybrid_lm_fused_prologue", True), ("hybrid_lm_pytorch_prologue", False)):
            tw = time_prologue(gdn, dr, max(3, args.steps // 2), 3, flush, stream, fused)
            ms_w = statistics.mean(tw)
            extra[key] = {"workload": f"hybrid_lm from raw projections ({'fused entry' if fused else 'PyTorch normalisation and activations, then the plain entry'})",
                          "ms": round(ms_w, 6), "tokens_per_s": round(8 * 4096 / (ms_w * 1e-3), 1),
                          "launches_per_call": 1 if fused else None}
        del dr
        # grouped value heads: the hybrid-LM shape with 6 q/k heads for its 12 value heads
        dg = to_dev(workloads.make_gva_chunk_inputs(B=8, T=4096, Hk=6, Hv=12, dk=64, dv=64, dtype="bf16",
                                                    seed=rank_seed(hl["seed"], rank), la_scale=0.1))
        outg = torch.empty_like(dg["v"])
        Sg = torch.empty((8, 12, 64, 64), dtype=torch.float32, device="cuda")

        def call_gva():
            gdn.chunk_fwd_gva(dg["q"], dg["k"], dg["v"], dg["log_alpha"], dg["beta"], out=outg, S_final=Sg,
                              stream=stream)
        ms_g = _time_loop(call_gva, max(3, args.steps // 2), 3, flush, stream)
        extra["hybrid_lm_gva"] = {"workload": "hybrid_lm shape, grouped value heads: Hk=6 q/k heads, Hv=12 value heads",
                                  "ms": round(ms_g, 6), "tokens_per_s": round(8 * 4096 / (ms_g * 1e-3), 1),
                                  "launches_per_call": 1}
        del dg, outg, Sg
        dh = to_dev(workloads.config_inputs("hybrid_lm", seed=rank_seed(hl["seed"], rank)))
        extra["hybrid_lm_backward"] = backward_numbers(gdn, dh, 5, 3, flush, stream, peaks)
        del dh
        dw = to_dev(workloads.make_chunk_inputs(B=8, T=4096, H=12, dk=64, dv=128, dtype="bf16",
                                                seed=rank_seed(hl["seed"], rank), la_scale=0.1))
        extra["hybrid_lm_backward_dv128"] = backward_numbers(gdn, dw, 3, 3, flush, stream, peaks)
        del dw
        extra["phase_memory"] = phase_numbers(gdn, 5, 3, flush, stream, peaks)
        extra["phase_memory_rowdecay"] = rowdecay_numbers(gdn, 5, 3, flush, stream, peaks)
        extra["decode_small_batch_graph"] = decode_graph_numbers(gdn)
        # key head size 128 (two key blocks), the hybrid-LM token and head counts at dk = dv = 128;
        # last of the device work and guarded, so that a failure here is reported in the line
        # rather than losing it
        try:
            dw = to_dev(workloads.make_chunk_inputs(B=8, T=4096, H=12, dk=128, dv=128, dtype="bf16",
                                                    seed=rank_seed(hl["seed"], rank), la_scale=0.1))
            extra["hybrid_lm_backward_dk128"] = backward_numbers(gdn, dw, 3, 3, flush, stream, peaks)
            del dw
        except Exception as exc:  # noqa: BLE001  (reported, not hidden)
            extra["hybrid_lm_backward_dk128"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    cpu = None
    if rank == 0 and world == 1:
        cpu = cpu_oracle_baseline(inp)
        if not args.quick:
            for w in ("hybrid_lm", "long_context"):
                cw = workloads.CONFIGS[w]
                others[w]["cpu_baseline"] = cpu_oracle_baseline(
                    workloads.config_inputs(w, seed=rank_seed(cw["seed"], rank)), budget_s=6.0)
            decode["cpu_baseline"] = cpu_decode_baseline()

    if rank != 0:
        return
    traffic = ncu_traffic("chunk", name)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; varlen lengths U[128,8192]; q,k L2-normalised N(0,1), v N(0,1), "
                "beta=2 sigmoid(N(0,1)), log_alpha=-softplus(N(0,2)), S0=0)",
        "config": headline_config(world),
        "roofline": roofline_obj(main, peaks, peak_kind, traffic),
        "tensor": tensor_obj(main, peaks),
        "e2e": {"value": tokens_all / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": args.steps * main["launches_per_call"],
        "clocks": clk.result(),
        "cpu_baseline": cpu,
        "tokens_per_step": main["tokens"],
    }
    if others:
        line.update(others)
    if decode is not None:
        line["decode"] = decode
    if extra:
        line["workloads"] = extra
    print(json.dumps(line), flush=True)


def _time_loop(call, steps, warmup, flush, stream):
    """Mean CUDA-event time (ms) of `call` on `stream` over `steps` calls after `warmup`, L2 flushed
    before each."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            flush.zero_()
            call()
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a0, b0 in ev:
            flush.zero_()
            a0.record(stream)
            call()
            b0.record(stream)
        stream.synchronize()
    return statistics.mean(a0.elapsed_time(b0) for a0, b0 in ev)


def bwd_products(KB, VS):
    """Distinct 64 x 64 x 64 products of the chunk-form backward per (chunk, head) at dk = 64 KB,
    dv = 64 VS, each counted once: forming T, W, U~, M, Bm, R (4 KB + VS + KB^2 + 2 KB VS, with
    K K^T, Q K^T, W and P W per key block), the two scans (2 KB^2 VS), and the gradients
    (5 KB VS + 4 VS + 5 KB + 2: K dS', W S, U dS'^T, dO S^T, dU S^T per key and value block;
    P^T dO, dO U^T, T^T dU, dU (b V)^T per value block; T^T dW, dW (b gam K)^T, (D + D^T) K, D2^T Q,
    D2 K per key block; dT T^T and T^T Z).  The gradient kernel's recomputed K K^T and Q K^T are
    not counted."""
    return (4 * KB + VS + KB * KB + 2 * KB * VS) + 2 * KB * KB * VS + (5 * KB * VS + 4 * VS + 5 * KB + 2)


def backward_numbers(gdn, d, steps, warmup, flush, stream, peaks):
    """The backward of the hybrid-LM step (dq, dk, dv, gate and state gradients; fp32-accurate
    products on the tensor cores as three tf32 terms) from a seeded dout; `d` holds inputs of the
    hybrid-LM token and head counts (B=8 T=4096 H=12) on the device, dk = 64 KB, dv = 64 VS."""
    dk, dv = d["q"].shape[-1], d["v"].shape[-1]
    KB, VS = dk // 64, dv // 64
    dout = torch.randn(d["v"].shape, device="cuda", generator=torch.Generator("cuda").manual_seed(7)).to(d["v"].dtype)
    wsb = torch.empty(gdn.gdn_chunk_bwd_workspace_bytes(8, 4096, 12, dk, dv, 64, 0), dtype=torch.uint8,
                      device="cuda")

    def call():
        gdn.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dout, workspace=wsb, stream=stream)
    ms_b = _time_loop(call, steps, warmup, flush, stream)
    # bytes per token-head: q, k, v, dout (bf16) and gates in; dq, dk, dv (fp32) and two gate grads out
    by_b = 393216 * (2 * dk * 2 + 2 * dv * 2 + 8 + 2 * dk * 4 + dv * 4 + 8)
    # algorithmic work: the distinct 64 x 64 x 64 products per (chunk, head) (bwd_products: 26 at
    # dk = dv = 64), at 2 * 64^3 fp32 flops each; the tensor cores execute three tf32 products for
    # each.  Value splits recompute the value-independent ones per 64-column block; those are
    # counted once here
    fl_b = 6144 * bwd_products(KB, VS) * 2 * 64 ** 3
    launches = 3 + (2 if VS > 1 else 0)
    tf32_peak = peaks["bf16_tflops"] * TF32_PER_BF16
    return {"workload": f"hybrid_lm backward: dq, dk, dv, dlog_alpha, dbeta (fp32) from dout; dk={dk}, dv={dv}",
            "ms": round(ms_b, 6), "tokens_per_s": round(32768 / (ms_b * 1e-3), 1),
            "launches_per_call": launches, "algo_bytes": by_b,
            "gbs": round(by_b / (ms_b * 1e-3) / 1e9, 3),
            "hbm_frac": round(by_b / (ms_b * 1e-3) / 1e9 / peaks["hbm_gbs"], 5),
            "algo_flops_fp32": fl_b,
            "fp32_tflops": round(fl_b / (ms_b * 1e-3) / 1e12, 3),
            "tf32_mma_tflops": round(3 * fl_b / (ms_b * 1e-3) / 1e12, 3),
            "tf32_peak_tflops": round(tf32_peak, 1),
            "tensor_frac": round(3 * fl_b / (ms_b * 1e-3) / 1e12 / tf32_peak, 5)}


def phase_numbers(gdn, steps, warmup, flush, stream, peaks):
    """The complex-phase delta memory at the hybrid-LM shape (dk = 32 complex = 64 real, dv = 64)."""
    ph = workloads.make_phase_inputs(B=8, T=4096, H=12, dk=32, dv=64, dtype="bf16", seed=530)
    dph = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in ph.items()}
    Kp, Qp = torch.view_as_real(dph["K"]).contiguous(), torch.view_as_real(dph["Q"]).contiguous()
    out_p = torch.empty_like(dph["v"])
    Mf_p = torch.empty(8, 12, 64, 32, 2, device="cuda")
    wsp = torch.empty(gdn.gdn_phase_fwd_workspace_bytes(8, 4096, 12, 32, 64, 0, gdn.GDN_DTYPE_BF16),
                      dtype=torch.uint8, device="cuda")

    def call():
        gdn.phase_fwd(Kp, Qp, dph["v"], dph["log_lam"], dph["beta"], out=out_p, M_final=Mf_p, workspace=wsp,
                      stream=stream)
    ms_p = _time_loop(call, steps, warmup, flush, stream)
    # bytes per token-head: K, Q (complex fp32), v and out (bf16), log_lam and beta; plus M_final
    by_p = 393216 * (2 * 32 * 8 + 2 * 64 * 2 + 8) + 96 * 64 * 32 * 8
    return {"workload": "complex-phase delta memory, hybrid_lm shape: B=8 T=4096 H=12, "
                        "dk=32 complex (64 real), dv=64, bf16 values, fp32 phasors",
            "ms": round(ms_p, 6), "tokens_per_s": round(32768 / (ms_p * 1e-3), 1),
            "launches_per_call": 2, "algo_bytes": by_p,
            "gbs": round(by_p / (ms_p * 1e-3) / 1e9, 3),
            "hbm_frac": round(by_p / (ms_p * 1e-3) / 1e9 / peaks["hbm_gbs"], 5)}


def rowdecay_numbers(gdn, steps, warmup, flush, stream, peaks):
    """The complex-phase memory with one decay per value channel (the Laplace core's diag(r_t)) at
    the hybrid-LM shape (dk = 32 complex, dv = 64): gdn_phase_rowdecay_fwd."""
    ph = workloads.make_phase_rowdecay_inputs(B=8, T=4096, H=12, dk=32, dv=64, dtype="bf16", seed=640)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in ph.items()}
    Kp, Qp = torch.view_as_real(d["K"]).contiguous(), torch.view_as_real(d["Q"]).contiguous()
    out = torch.empty_like(d["v"])
    Mf = torch.empty(8, 12, 64, 32, 2, device="cuda")

    def call():
        gdn.phase_rowdecay_fwd(Kp, Qp, d["v"], d["log_r"], d["beta"], out=out, M_final=Mf, stream=stream)
    ms = _time_loop(call, steps, warmup, flush, stream)
    # bytes per token-head: K, Q (complex fp32), v and out (bf16), log_r (fp32 per channel), beta;
    # plus M_final
    by = 393216 * (2 * 32 * 8 + 2 * 64 * 2 + 64 * 4 + 4) + 96 * 64 * 32 * 8
    return {"workload": "complex-phase memory with per-channel decays, hybrid_lm shape: B=8 T=4096 H=12, "
                        "dk=32 complex, dv=64, bf16 values, fp32 phasors and decays",
            "ms": round(ms, 6), "tokens_per_s": round(32768 / (ms * 1e-3), 1),
            "launches_per_call": 1, "algo_bytes": by,
            "gbs": round(by / (ms * 1e-3) / 1e9, 3),
            "hbm_frac": round(by / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 5)}


def decode_graph_numbers(gdn, steps=100):
    """Small-batch decode (16 sequences x 8 heads, d = 128), where launch overhead rivals the
    kernel: 100 steps launched one by one from Python versus the same steps captured once in a
    CUDA graph and replayed; per-step time from CUDA events around the 100 steps."""
    N, H, d = 16, 8, 128
    xs = [to_dev(workloads.make_decode_step_inputs(N, H, d, d, "bf16", seed=9, step=i)) for i in range(steps)]
    S = workloads.make_decode_state(N, H, d, d, seed=9).cuda()
    outs = [torch.empty(N, H, d, dtype=torch.bfloat16, device="cuda") for _ in range(steps)]

    def run_steps():
        for x, o in zip(xs, outs):
            gdn.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S, out=o)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        run_steps()  # first calls outside the capture
        side.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(side)
        run_steps()
        e1.record(side)
        side.synchronize()
    eager = e0.elapsed_time(e1) / steps
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_steps()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    graph.replay()
    torch.cuda.synchronize()
    g0.record()
    graph.replay()
    g1.record()
    torch.cuda.synchronize()
    replay = g0.elapsed_time(g1) / steps
    del graph
    return {"workload": "decode, 16 x 8 states of 128 x 128, 100 steps per measurement",
            "eager_us_per_step": round(eager * 1e3, 3), "graph_us_per_step": round(replay * 1e3, 3),
            "launches_per_step": 1}


def run_only(args):
    """One workload's timing loop, no e2e / CPU baseline; prints that workload's numbers."""
    import linear_attention_sequence_rule_b200 as gdn
    peaks, _ = load_peaks()
    stream = torch.cuda.Stream()
    if args.only in ("decode", "decode_fused"):
        r = time_decode(gdn, args.steps, args.warmup, stream, fused=args.only == "decode_fused")
        r["hbm_frac"] = r["gbs"] / peaks["hbm_gbs"]
    elif args.only == "hybrid_lm_backward":
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        r = backward_numbers(gdn, to_dev(workloads.config_inputs("hybrid_lm")), args.steps, args.warmup, flush,
                             stream, peaks)
    elif args.only in ("hybrid_lm_backward_dv128", "hybrid_lm_backward_dk128"):
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        dk = 128 if args.only.endswith("dk128") else 64
        d = to_dev(workloads.make_chunk_inputs(B=8, T=4096, H=12, dk=dk, dv=128, dtype="bf16", seed=0, la_scale=0.1))
        r = backward_numbers(gdn, d, args.steps, args.warmup, flush, stream, peaks)
    elif args.only == "phase_memory":
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        r = phase_numbers(gdn, args.steps, args.warmup, flush, stream, peaks)
    elif args.only == "phase_memory_rowdecay":
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        r = rowdecay_numbers(gdn, args.steps, args.warmup, flush, stream, peaks)
    elif args.only == "hybrid_lm_dv256":
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        d = wide_value_inputs()
        r = chunk_numbers(WIDE_VALUE, d, time_chunk(gdn, d, args.steps, args.warmup, flush, stream), peaks)
    elif args.only in ("hybrid_lm_fused", "hybrid_lm_unfused"):
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        d = to_dev(workloads.config_raw_inputs("hybrid_lm"))
        tw = time_prologue(gdn, d, args.steps, args.warmup, flush, stream, args.only.endswith("_fused"))
        ms = statistics.mean(tw)
        r = {"workload": args.only, "ms": ms, "tokens_per_s": 8 * 4096 / (ms * 1e-3)}
    else:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        d = to_dev(workloads.config_inputs(args.only))
        r = chunk_numbers(args.only, d, time_chunk(gdn, d, args.steps, args.warmup, flush, stream),
                          peaks)
    print(json.dumps({"only": args.only, **r}), flush=True)


# ---- reference arm: the fp64 oracle on the host cores ----------------------------------------

def run_reference(args, world, rank, inp=None):
    """The reference arm: the fp64 oracle on the host cores over a bounded sample of the headline
    workload's chains per step; returns the JSON line (rank 0) or None."""
    if rank != 0:
        return None
    import oracle
    if inp is None:
        inp = workloads.config_inputs(HEADLINE)
    H = inp["H"]
    threads = oracle.max_threads()
    # each step: enough whole sequences (every head: H independent chains each) to give every host
    # thread a chain, taken in turn, their inputs converted to fp64 before the step's timing; the
    # whole run takes a few minutes
    per_step = min(inp["B"], max(1, -(-threads // H)))
    times, token_heads = [], []
    for i in range(args.warmup + args.steps):
        sub, th = oracle_subproblem(inp, [(i * per_step + j) % inp["B"] for j in range(per_step)])
        t0 = time.perf_counter()
        oracle.forward(*sub[:6], cu_seqlens=sub[6])
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            token_heads.append(th)
    s = statistics.mean(times)
    # tokens, not token-heads: a token of the workload is all H of its heads
    value = (sum(token_heads) / H) / sum(times)
    sample = (f"{per_step} of {inp['B']} sequences per step, every head of each ({per_step * H} chains, "
              f"{sum(token_heads) // len(token_heads)} token-heads per step on average, counted as "
              f"token-heads / {H} tokens), fp64 sequential recurrence, inputs converted to fp64 "
              f"before each step's timing")
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": s * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded, same inputs as the GPU arm)",
        "config": headline_config(world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "token_heads_timed": sum(token_heads), "seconds_timed": sum(times),
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="main workload only")
    ap.add_argument("--only", choices=["hybrid_lm", "long_context", "varlen", "varlen_profile", "tiny", "decode",
                                       "hybrid_lm_fused",
                                             "hybrid_lm_unfused", "hybrid_lm_backward", "phase_memory",
                                             "hybrid_lm_dv256", "hybrid_lm_backward_dv128", "decode_fused",
                                             "hybrid_lm_backward_dk128", "phase_memory_rowdecay"],
                    help="time one workload's kernel loop only (for profiler runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.only:
            run_only(args)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
