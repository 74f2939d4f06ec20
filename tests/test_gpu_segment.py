"""GPU parity of the segment scan that gdn_chunk_fwd runs for long dense bf16 sequences with few
(sequence, head) chains: the sequence is cut into segments whose local states (from zero) and
transitions (from the identity, values zero) are computed in parallel, scanned per chain, and
the outputs then recomputed per segment from its entry state.  The affine form of the chunk state
map this rests on is the one in "Gated Delta Networks", section 3 (chunkwise form); the oracle
is the plain token-by-token recurrence, so any segment bookkeeping error shows up here.

The cases are sized so that the scan splits each sequence into several segments on a GPU with
100+ SMs, with a ragged last chunk and a short last segment.
"""
import ctypes

import pytest
import torch

import workloads
from tests.parity import TOL, compare_chunk, run_gpu_chunk

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _inputs(B, T, H, d, seed, s0=0.05, **kw):
    return workloads.make_chunk_inputs(B=B, T=T, H=H, dk=d, dv=d, dtype="bf16", seed=seed,
                                       s0_std=s0, **kw)


def _uses_segments(inp):
    import linear_attention_sequence_rule_b200 as gdn
    return gdn.workspace_bytes(inp["B"], inp["T"], inp["H"], inp["dk"], inp["dv"]) > 0


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("s0", [0.0, 0.05])
def test_segment_scan_single_sequence(d, s0):
    inp = _inputs(1, 81 * 64 - 45, 2, d, seed=100 + d, s0=s0, la_scale=0.1)
    assert _uses_segments(inp)
    out, Sf = run_gpu_chunk(inp)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


@pytest.mark.parametrize("d", [64, 128])
def test_segment_scan_several_sequences(d):
    inp = _inputs(2, 2100, 3, d, seed=200 + d, la_scale=0.1)
    assert _uses_segments(inp)
    out, Sf = run_gpu_chunk(inp)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_segment_scan_resets_and_extreme_gates():
    inp = _inputs(1, 81 * 64 - 45, 2, 64, seed=300, beta_scale=2.0, la_std=2.0)
    assert _uses_segments(inp)
    la, be = inp["log_alpha"], inp["beta"]
    # exact resets on and around chunk boundaries all along the sequence, so that some fall on
    # segment boundaries whatever the segment length
    for c in range(1, 81, 4):
        la[0, 64 * c, 0] = -float("inf")
        la[0, 64 * c - 1, 1] = -float("inf")
    la[0, 3000:3003, 0] = -float("inf")
    be[0, 100:180, 1] = 0.0
    be[0, 2000:2100, 0] = 2.0
    out, Sf = run_gpu_chunk(inp)
    assert torch.isfinite(out).all() and torch.isfinite(Sf).all()
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_segment_scan_without_final_state():
    inp = _inputs(1, 64 * 64, 2, 128, seed=400, la_scale=0.1)
    assert _uses_segments(inp)
    out, Sf = run_gpu_chunk(inp, S_final=False)
    assert Sf is None
    e_o, _ = compare_chunk(inp, out, None)
    assert e_o <= TOL["bf16"], e_o


def test_segment_scan_matches_single_chain_run():
    """The same sequence packed as a one-sequence varlen call runs as a single chain (the scan is
    for dense inputs only); the two results agree to rounding."""
    import linear_attention_sequence_rule_b200 as gdn
    inp = _inputs(1, 50 * 64 + 7, 4, 128, seed=500, la_scale=0.1)
    assert _uses_segments(inp)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out_s, Sf_s = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    cu = torch.tensor([0, inp["T"]], dtype=torch.int32, device="cuda")
    out_c, Sf_c = gdn.chunk_fwd(d["q"][0], d["k"][0], d["v"][0], d["log_alpha"][0], d["beta"][0],
                                S0=d["S0"], cu_seqlens=cu)
    gdn.device_status()
    assert (out_s[0].float() - out_c.float()).abs().max().item() <= TOL["bf16"]
    assert (Sf_s - Sf_c).abs().max().item() <= TOL["bf16"]


def test_segment_scan_rejects_short_workspace():
    import linear_attention_sequence_rule_b200 as gdn
    inp = _inputs(1, 40 * 64, 2, 64, seed=600)
    need = gdn.workspace_bytes(1, inp["T"], 2, 64, 64)
    assert need > 0
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out = torch.empty_like(d["v"])
    Sf = torch.empty(1, 2, 64, 64, device="cuda")
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    args = (p(d["q"]), p(d["k"]), p(d["v"]), p(d["log_alpha"]), p(d["beta"]), p(d["S0"]), p(out),
            p(Sf), 1, inp["T"], 2, 64, 64, 64, None, gdn.GDN_DTYPE_BF16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert gdn.gdn_chunk_fwd(*args, p(ws), need - 1, stream) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_chunk_fwd(*args, None, 0, stream) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_chunk_fwd(*args, p(ws), need, stream) == gdn.GDN_OK
    gdn.device_status()
