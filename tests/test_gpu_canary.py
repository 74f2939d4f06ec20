"""Out-of-bounds write checks by guard bands (the stand-in for a memory sanitizer).

Every output buffer -- and the workspace where a call takes one -- is cut from the middle of a
larger allocation filled with NaN.  After the call the bands on both sides must still hold the
exact NaN bits they were filled with (nothing was written outside the tensor), and the tensor
itself must hold no NaN (every element it owns was written).  The cases are the ones where an
index slip would land outside a row: ragged last chunks, varlen packs with empty, 1-token and
chunk-boundary sequences, value head size 256 as two column blocks, the segment scan of a long
sequence, the backward's value splits and key blocks, decode with in-place states, grouped value
heads, the complex-phase memory and the host-memory entry.
"""
import math

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

BAND = 4096  # elements on each side; a multiple of 16 bytes for every element size used here
BITS = {torch.bfloat16: torch.int16, torch.float32: torch.int32, torch.uint8: torch.uint8}


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


class Guarded:
    """A tensor of `shape` inside NaN guard bands (uint8 buffers are banded with 0xA5 bytes)."""

    def __init__(self, shape, dtype, device="cuda", fill=None, pin=False):
        n = math.prod(shape)
        fillv = 0xA5 if dtype == torch.uint8 else float("nan")
        self.buf = torch.full((n + 2 * BAND,), fillv, dtype=dtype, device=device)
        if pin:
            self.buf = self.buf.pin_memory()
        self.t = self.buf[BAND:BAND + n].view(shape)
        if fill is not None:
            self.t.copy_(fill)
        self.ref = self.buf.view(BITS[dtype]).clone()

    def bands_intact(self):
        b = self.buf.view(BITS[self.buf.dtype])
        return torch.equal(b[:BAND], self.ref[:BAND]) and torch.equal(b[-BAND:], self.ref[-BAND:])

    def check(self, name, full=True):
        if self.buf.is_cuda:
            torch.cuda.synchronize()
        assert self.bands_intact(), f"{name}: a write landed outside the tensor"
        if full:
            assert not torch.isnan(self.t.float()).any(), f"{name}: an element was never written"


def dev(inp):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}


def chunk_call(inp, S_final=True, ws_guard=True):
    import linear_attention_sequence_rule_b200 as gdn
    d = dev(inp)
    B, H, dk, dv = inp["B"], inp["H"], inp["dk"], inp["dv"]
    varlen = d["cu_seqlens"] is not None
    T = inp["T"]
    out = Guarded(tuple(d["v"].shape), d["v"].dtype)
    Sf = Guarded((B, H, dk, dv), torch.float32) if S_final else None
    need = gdn.workspace_bytes(B, T, H, dk, dv, varlen, d["q"].dtype)
    ws = Guarded((need,), torch.uint8) if need else None
    gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], cu_seqlens=d["cu_seqlens"],
                  out=out.t, S_final=None if Sf is None else Sf.t, workspace=None if ws is None else ws.t)
    gdn.device_status()
    out.check("out")
    if Sf is not None:
        Sf.check("S_final")
    if ws is not None:
        ws.check("workspace", full=False)
    return out.t, None if Sf is None else Sf.t


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
def test_dense_ragged_tail(dtype, dk, dv):
    inp = workloads.make_chunk_inputs(B=2, T=300, H=3, dk=dk, dv=dv, dtype=dtype, seed=dk + dv, s0_std=0.1)
    chunk_call(inp)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
def test_varlen_ragged_pack(dtype, d):
    lengths = [1, 63, 64, 65, 0, 200, 129, 7]
    inp = workloads.make_chunk_inputs(H=2, dk=d, dv=d, dtype=dtype, seed=7, s0_std=0.05, lengths=lengths)
    chunk_call(inp)


@pytest.mark.parametrize("dk", [64, 128])
def test_value_head_256(dk):
    lengths = [1, 65, 0, 300, 128]
    inp = workloads.make_chunk_inputs(H=3, dk=dk, dv=256, dtype="bf16", seed=31, s0_std=0.05, lengths=lengths)
    chunk_call(inp)
    inp = workloads.make_chunk_inputs(B=2, T=190, H=2, dk=dk, dv=256, dtype="bf16", seed=32, s0_std=0.05)
    chunk_call(inp)


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 256)])
def test_segment_scan(dk, dv):
    import linear_attention_sequence_rule_b200 as gdn
    T = 81 * 64 - 45
    assert gdn.workspace_bytes(1, T, 2, dk, dv) > 0  # the segment scan runs
    inp = workloads.make_chunk_inputs(B=1, T=T, H=2, dk=dk, dv=dv, dtype="bf16", seed=41, s0_std=0.05,
                                      la_scale=0.1)
    chunk_call(inp)


def test_no_final_state():
    inp = workloads.make_chunk_inputs(B=2, T=130, H=2, dk=64, dv=64, dtype="bf16", seed=5)
    chunk_call(inp, S_final=False)


def test_fused_and_grouped_forward():
    import linear_attention_sequence_rule_b200 as gdn
    lengths = [3, 64, 0, 150]
    raw = dev(workloads.make_raw_chunk_inputs(H=2, dk=128, dv=128, dtype="bf16", seed=51, lengths=lengths,
                                              la_scale=0.5, beta_scale=2.0))
    out = Guarded(tuple(raw["v"].shape), torch.bfloat16)
    Sf = Guarded((4, 2, 128, 128), torch.float32)
    gdn.chunk_fwd_fused(raw["q_raw"], raw["k_raw"], raw["v"], raw["a_raw"], raw["b_raw"], raw["a_scale"],
                        raw["b_scale"], cu_seqlens=raw["cu_seqlens"], out=out.t, S_final=Sf.t)
    out.check("fused out")
    Sf.check("fused S_final")
    g = dev(workloads.make_gva_chunk_inputs(Hk=2, Hv=6, dk=64, dv=128, dtype="bf16", seed=52, s0_std=0.05,
                                            lengths=lengths))
    out = Guarded(tuple(g["v"].shape), torch.bfloat16)
    Sf = Guarded((4, 6, 64, 128), torch.float32)
    gdn.chunk_fwd_gva(g["q"], g["k"], g["v"], g["log_alpha"], g["beta"], S0=g["S0"], cu_seqlens=g["cu_seqlens"],
                      out=out.t, S_final=Sf.t)
    out.check("gva out")
    Sf.check("gva S_final")


@pytest.mark.parametrize("dk,dv,lengths", [(64, 128, [1, 63, 64, 65, 0, 200]), (128, 256, [70, 0, 129]),
                                           (128, 64, [5, 191])])
def test_backward_splits_and_blocks(dk, dv, lengths):
    import linear_attention_sequence_rule_b200 as gdn
    inp = dev(workloads.make_chunk_inputs(H=2, dk=dk, dv=dv, dtype="bf16", seed=61, s0_std=0.05,
                                          lengths=lengths, beta_scale=2.0))
    B, T, H = inp["B"], inp["T"], 2
    dout = torch.randn(inp["v"].shape, device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    dout = dout.to(torch.bfloat16)
    dSf = 0.1 * torch.randn(B, H, dk, dv, device="cuda")
    g = {"dq": Guarded((T, H, dk), torch.float32), "dk": Guarded((T, H, dk), torch.float32),
         "dv": Guarded((T, H, dv), torch.float32), "dla": Guarded((T, H), torch.float32),
         "dbe": Guarded((T, H), torch.float32), "dS0": Guarded((B, H, dk, dv), torch.float32)}
    need = gdn.gdn_chunk_bwd_workspace_bytes(B, T, H, dk, dv, 64, 1)
    ws = Guarded((need,), torch.uint8)
    p = lambda t: None if t is None else t.data_ptr()
    rc = gdn.gdn_chunk_bwd(p(inp["q"]), p(inp["k"]), p(inp["v"]), p(inp["log_alpha"]), p(inp["beta"]),
                           p(inp["S0"]), p(dout), p(dSf), p(g["dq"].t), p(g["dk"].t), p(g["dv"].t),
                           p(g["dla"].t), p(g["dbe"].t), p(g["dS0"].t), B, T, H, dk, dv, 64,
                           p(inp["cu_seqlens"]), gdn.GDN_DTYPE_BF16, p(ws.t), need, None)
    assert rc == gdn.GDN_OK, gdn.gdn_last_error()
    gdn.device_status()
    for name, x in g.items():
        x.check(name)
    ws.check("workspace", full=False)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 256), (128, 64)])
def test_decode_in_place(dtype, dk, dv):
    import linear_attention_sequence_rule_b200 as gdn
    N, H = 5, 3
    S = Guarded((N, H, dk, dv), torch.float32, fill=workloads.make_decode_state(N, H, dk, dv, seed=8).cuda())
    for step in range(3):
        x = dev(workloads.make_decode_step_inputs(N, H, dk, dv, dtype, seed=8, step=step))
        out = Guarded((N, H, dv), x["v"].dtype)
        gdn.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S.t, out=out.t)
        out.check("decode out")
        S.check("decode state")
    Hk = 1
    x = dev(workloads.make_decode_step_inputs(N, H, dk, dv, dtype, seed=9, step=0))
    out = Guarded((N, H, dv), x["v"].dtype)
    gdn.decode_step_gva(x["q"][:, :Hk].contiguous(), x["k"][:, :Hk].contiguous(), x["v"], x["log_alpha"],
                        x["beta"], S.t, out=out.t)
    out.check("decode gva out")
    S.check("decode gva state")


def test_phase_memory():
    import linear_attention_sequence_rule_b200 as gdn
    ph = workloads.make_phase_inputs(H=2, dk=32, dv=128, dtype="bf16", seed=71, m0_std=0.1,
                                     lengths=[1, 64, 0, 130])
    d = dev(ph)
    Kp, Qp = torch.view_as_real(d["K"]).contiguous(), torch.view_as_real(d["Q"]).contiguous()
    out = Guarded(tuple(d["v"].shape), torch.bfloat16)
    Mf = Guarded((4, 2, 128, 32, 2), torch.float32)
    gdn.phase_fwd(Kp, Qp, d["v"], d["log_lam"], d["beta"], M0=d["M0"], cu_seqlens=d["cu_seqlens"], out=out.t,
                  M_final=Mf.t)
    out.check("phase out")
    Mf.check("phase M_final")


def test_host_entry():
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_chunk_inputs(H=2, dk=128, dv=128, dtype="bf16", seed=81, s0_std=0.05,
                                      lengths=[1, 300, 0, 64, 65, 700])
    out = Guarded(tuple(inp["v"].shape), torch.bfloat16, device="cpu", pin=True)
    Sf = Guarded((6, 2, 128, 128), torch.float32, device="cpu", pin=True)
    host = {k: (v.pin_memory() if torch.is_tensor(v) else v) for k, v in inp.items()}
    gdn.chunk_fwd_host(host["q"], host["k"], host["v"], host["log_alpha"], host["beta"], S0=host["S0"],
                       cu_seqlens=host["cu_seqlens"], out=out.t, S_final=Sf.t)
    torch.cuda.synchronize()
    out.check("host out")
    Sf.check("host S_final")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(32, 6), (64, 130), (32, 64)])
def test_phase_rowdecay(dtype, dk, dv):
    # channel blocks with a ragged last block, ragged chunk tails, empty and one-token sequences
    import linear_attention_sequence_rule_b200 as gdn
    ph = workloads.make_phase_rowdecay_inputs(H=2, dk=dk, dv=dv, dtype=dtype, seed=91 + dv, m0_std=0.1,
                                              lengths=[1, 31, 0, 33, 70])
    d = dev(ph)
    tv = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = Guarded(tuple(d["v"].shape), tv)
    Mf = Guarded((5, 2, dv, dk, 2), torch.float32)
    gdn.phase_rowdecay_fwd(d["K"], d["Q"], d["v"], d["log_r"], d["beta"], M0=d["M0"], cu_seqlens=d["cu_seqlens"],
                           out=out.t, M_final=Mf.t)
    gdn.device_status()
    out.check("rowdecay out")
    Mf.check("rowdecay M_final")
