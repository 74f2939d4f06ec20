"""GPU parity of the chunk forward's general path (key head size 256, chunk length 128, fp32 at
value head size 256: gdn_chunk_general.cu, fp32 arithmetic on CUDA cores) against the fp64
oracle, element by element on the same seeded inputs: dense with a ragged tail and an initial
state, varlen packs with empty, one-token and chunk-boundary sequences, exact resets on and
inside chunk boundaries, beta = 0 and beta = 2, grouped value heads, guard bands around every
output and the workspace.  Bounds as every chunk-forward test: max-abs 2e-2 (bf16 inputs) and
1e-4 (fp32 inputs) on outputs and final states."""
import math

import pytest
import torch

import workloads
from tests.parity import TOL, compare_chunk

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def run(inp, chunk, guard=False):
    import linear_attention_sequence_rule_b200 as gdn
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    B, H, dk, dv = inp["B"], inp["H"], inp["dk"], inp["dv"]
    varlen = d["cu_seqlens"] is not None
    need = gdn.workspace_bytes(B, inp["T"], H, dk, dv, varlen, d["q"].dtype, chunk=chunk)
    # the general path passes its chunk factors through the workspace (bf16 at dk <= 128, dv = 256,
    # chunk 64 is the fused kernel's column-block case and needs none)
    assert (need > 0) == (dk == 256 or chunk == 128 or d["q"].dtype == torch.float32 and dv == 256)
    need = max(need, 16)
    band = 4096
    nout = math.prod(d["v"].shape)
    ob = torch.full((nout + 2 * band,), float("nan"), dtype=d["v"].dtype, device="cuda")
    sb = torch.full((B * H * dk * dv + 2 * band,), float("nan"), device="cuda")
    wb = torch.full((need + 2 * band,), 0xA5, dtype=torch.uint8, device="cuda")
    out = ob[band:band + nout].view(d["v"].shape)
    Sf = sb[band:band + B * H * dk * dv].view(B, H, dk, dv)
    ws = wb[band:band + need]
    bits = lambda t: t.view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32) if t.dtype != torch.uint8 else t
    refs = [bits(x).clone() for x in (ob, sb, wb)]
    gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"], cu_seqlens=d["cu_seqlens"],
                  out=out, S_final=Sf, workspace=ws, chunk=chunk)
    gdn.device_status()
    for x, r in zip((ob, sb, wb), refs):
        b = bits(x)
        assert torch.equal(b[:band], r[:band]) and torch.equal(b[-band:], r[-band:]), "write outside a buffer"
    assert not torch.isnan(out.float()).any() and not torch.isnan(Sf).any()
    return out, Sf


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv,chunk", [(256, 64, 64), (256, 128, 64), (256, 256, 64), (64, 64, 128),
                                         (128, 128, 128), (256, 128, 128), (128, 256, 64)])
def test_dense_ragged(dtype, dk, dv, chunk):
    inp = workloads.make_chunk_inputs(B=2, T=300, H=2, dk=dk, dv=dv, dtype=dtype, seed=dk + dv + chunk, s0_std=0.1,
                                      beta_scale=2.0, la_scale=0.5)
    out, Sf = run(inp, chunk)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL[dtype] and e_s <= TOL[dtype], (e_o, e_s)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,chunk", [(256, 64), (128, 128), (256, 128)])
def test_varlen_resets_extreme_gates(dtype, dk, chunk):
    lengths = [1, 127, 128, 129, 0, 300, 64, 7]
    inp = workloads.make_chunk_inputs(H=2, dk=dk, dv=64, dtype=dtype, seed=11 + dk + chunk, s0_std=0.05,
                                      lengths=lengths, beta_scale=2.0, la_std=2.0)
    la, be = inp["log_alpha"], inp["beta"]
    cu = inp["cu_seqlens"]
    s5 = int(cu[5])
    la[s5 + 5, 0] = -float("inf")
    la[s5 + 128, 1] = -float("inf")   # first token of a 128-chunk
    la[s5 + 127, 0] = -float("inf")   # last token of a 128-chunk
    be[s5 + 10:s5 + 20, 0] = 0.0
    be[s5 + 30:s5 + 40, 1] = 2.0
    out, Sf = run(inp, chunk)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL[dtype] and e_s <= TOL[dtype], (e_o, e_s)
    assert torch.equal(Sf[4].cpu(), inp["S0"][4])  # the empty sequence keeps its state


def test_grouped_value_heads_dk256():
    import linear_attention_sequence_rule_b200 as gdn
    from oracle import grouped
    inp = workloads.make_gva_chunk_inputs(B=2, T=200, Hk=1, Hv=3, dk=256, dv=64, dtype="bf16", seed=77,
                                          s0_std=0.05)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd_gva(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    gdn.device_status()
    o_ref, s_ref = grouped.forward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    e_o = float((out.double().cpu() - torch.from_numpy(o_ref)).abs().max())
    e_s = float((Sf.double().cpu() - torch.from_numpy(s_ref)).abs().max())
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_chunk_invariance_on_the_gpu():
    # the same inputs through chunk 64 and chunk 128 give the same results (the chunk form is an
    # exact refactoring of the recurrence)
    inp = workloads.make_chunk_inputs(B=1, T=500, H=2, dk=128, dv=128, dtype="f32", seed=5, s0_std=0.1)
    o1, s1 = run(inp, 64)
    o2, s2 = run(inp, 128)
    assert float((o1 - o2).abs().max()) <= 1e-4 and float((s1 - s2).abs().max()) <= 1e-4


@pytest.mark.parametrize("dk,chunk,lengths", [(256, 64, None), (128, 128, [0, 1, 130, 300, 64, 7])])
def test_host_entry_on_the_general_path(dk, chunk, lengths):
    # host buffers in and out, the batch cut into parts: each part runs the general path with the
    # same per-sequence arithmetic as the device entry, so the results are bit-identical
    import linear_attention_sequence_rule_b200 as gdn
    if lengths is None:
        inp = workloads.make_chunk_inputs(B=3, T=200, H=2, dk=dk, dv=128, dtype="bf16", seed=90, s0_std=0.05)
    else:
        inp = workloads.make_chunk_inputs(H=2, dk=dk, dv=128, dtype="bf16", seed=91, s0_std=0.05, lengths=lengths)
    host = {k: (v.contiguous().pin_memory() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out_h, sf_h = gdn.chunk_fwd_host(host["q"], host["k"], host["v"], host["log_alpha"], host["beta"], S0=host["S0"],
                                     cu_seqlens=host["cu_seqlens"], chunk=chunk)
    torch.cuda.synchronize()
    out_d, sf_d = run(inp, chunk)
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(sf_h, sf_d.cpu())


def test_noalloc_entry_on_the_general_path():
    # the general path's factors fit the fixed scratch array at these sizes; results bit-identical
    import ctypes
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_chunk_inputs(B=2, T=150, H=2, dk=256, dv=64, dtype="bf16", seed=92, s0_std=0.05)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    need = gdn.gdn_chunk_fwd_workspace_bytes(2, 150, 2, 256, 64, 64, 0, gdn.GDN_DTYPE_BF16)
    assert 0 < need <= 32 * 2 ** 20
    out = torch.empty_like(d["v"])
    Sf = torch.empty(2, 2, 256, 64, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = gdn.gdn_chunk_fwd_noalloc(p(d["q"]), p(d["k"]), p(d["v"]), p(d["log_alpha"]), p(d["beta"]), p(d["S0"]),
                                   p(out), p(Sf), 2, 150, 2, 256, 64, 64, None, gdn.GDN_DTYPE_BF16, stream)
    assert rc == gdn.GDN_OK, gdn.gdn_last_error()
    assert gdn.gdn_device_status(stream) == gdn.GDN_OK
    out_d, sf_d = run(inp, 64)
    assert torch.equal(out, out_d) and torch.equal(Sf, sf_d)
