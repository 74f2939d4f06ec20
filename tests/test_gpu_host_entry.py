"""gdn_chunk_fwd_host (host buffers in and out, the batch cut into parts whose copies overlap the
compute) against gdn_chunk_fwd on device buffers and against the fp64 oracle.

Where every part runs the same kernel plan as the whole call (no segment scan on either side:
varlen inputs, fp32 inputs, short dense sequences) each (sequence, head) chain goes through the
same arithmetic, so the outputs must be bit-identical.  At the hybrid-LM size the two-sequence
parts take the segment scan while the whole batch does not, so that case is held to the oracle's
bf16 bound instead."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import TOL, f64, max_abs, run_gpu_chunk

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def host_inputs(inp, pinned=True):
    h = {}
    for key in ("q", "k", "v", "log_alpha", "beta", "S0", "cu_seqlens"):
        t = inp.get(key)
        if t is not None:
            t = t.contiguous()
            h[key] = t.pin_memory() if pinned else t.clone()
        else:
            h[key] = None
    return h


def run_host(inp, pinned=True, stream=None, workspace=None):
    import linear_attention_sequence_rule_b200 as gdn
    h = host_inputs(inp, pinned)
    out, Sf = gdn.chunk_fwd_host(h["q"], h["k"], h["v"], h["log_alpha"], h["beta"], S0=h["S0"],
                                 cu_seqlens=h["cu_seqlens"], stream=stream, workspace=workspace)
    gdn.device_status(stream)  # synchronises the stream the outputs were joined into
    return out, Sf


def assert_identical(inp, **kw):
    out_h, sf_h = run_host(inp, **kw)
    out_d, sf_d = run_gpu_chunk(inp)
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(sf_h, sf_d.cpu())
    return out_h, sf_h


def test_dense_bf16_identical_to_device_entry():
    inp = workloads.make_chunk_inputs(B=3, T=300, H=2, dk=64, dv=64, dtype="bf16", seed=401, s0_std=0.05)
    assert_identical(inp)


def test_dense_fp32_identical_and_within_oracle_bound():
    inp = workloads.make_chunk_inputs(B=2, T=200, H=2, dk=64, dv=64, dtype="f32", seed=402)
    out, sf = assert_identical(inp)
    o_ref, s_ref = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    assert max_abs(f64(out), o_ref) <= TOL["f32"]
    assert max_abs(f64(sf), s_ref) <= TOL["f32"]


def test_varlen_ragged_identical_to_device_entry():
    # empty and one-token sequences, more sequences than parts, head size 128
    inp = workloads.make_chunk_inputs(H=3, dk=128, dv=128, dtype="bf16", seed=403, s0_std=0.05,
                                      lengths=[0, 1, 63, 64, 65, 0, 200, 130, 7, 1, 300, 2])
    assert_identical(inp)


def test_pageable_buffers_and_a_side_stream_with_reused_workspace():
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_chunk_inputs(B=5, T=129, H=2, dk=64, dv=128, dtype="bf16", seed=404, s0_std=0.05)
    need = gdn.gdn_chunk_fwd_host_workspace_bytes(5, 129, 2, 64, 128, 64, 0, gdn.GDN_DTYPE_BF16)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    st = torch.cuda.Stream()
    first = run_host(inp, pinned=False, stream=st, workspace=ws)
    second = run_host(inp, pinned=True, stream=st, workspace=ws)
    out_d, sf_d = run_gpu_chunk(inp)
    for out, sf in (first, second):
        assert torch.equal(out, out_d.cpu())
        assert torch.equal(sf, sf_d.cpu())


def test_hybrid_lm_size_against_the_oracle():
    # the bench's end-to-end workload: four two-sequence parts, each through the segment scan
    inp = workloads.config_inputs("hybrid_lm")
    out, sf = run_host(inp)
    o_ref, s_ref = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    assert max_abs(f64(out), o_ref) <= TOL["bf16"]
    assert max_abs(f64(sf), s_ref) <= TOL["bf16"]
    assert np.isfinite(f64(out)).all()
