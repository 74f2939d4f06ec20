"""GPU parity of the value head size 256 against the fp64 oracles.

The recurrence never mixes value columns: column j of S and of the outputs follows from column j
of V and of S0 alone (S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T acts on S from the
left).  So dv = 256 runs as two 128-column blocks, and besides parity against the oracle these
tests check that property on the device: a dv = 256 call equals, bit for bit, two dv = 128 calls
on the column halves.  Entries covered: gdn_chunk_fwd (dense, varlen with ragged and empty
sequences, resets and beta range ends), gdn_chunk_fwd_gva, gdn_chunk_fwd_fused,
gdn_chunk_fwd_host, and gdn_decode_step (whose oracle parity at dv = 256 is in test_gpu_decode.py).
"""
import pytest
import torch

import workloads
from oracle import grouped, prologue
from tests.parity import TOL, compare_chunk, f64, max_abs, run_gpu_chunk

pytestmark = pytest.mark.gpu

DV = 256


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


@pytest.mark.parametrize("dk", [64, 128])
def test_dense(dk):
    inp = workloads.make_chunk_inputs(B=2, T=300, H=3, dk=dk, dv=DV, dtype="bf16", seed=5 + dk, s0_std=0.1)
    out, Sf = run_gpu_chunk(inp)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_varlen_ragged_empty_resets():
    lengths = [1, 63, 64, 65, 0, 200, 129, 7]
    inp = workloads.make_chunk_inputs(H=2, dk=128, dv=DV, dtype="bf16", seed=9, s0_std=0.05, lengths=lengths,
                                      beta_scale=2.0)
    inp["log_alpha"][70, 0] = -float("inf")  # an exact reset inside the 200-token sequence
    inp["beta"][200:210, 1] = 0.0
    out, Sf = run_gpu_chunk(inp)
    assert torch.isfinite(out).all() and torch.isfinite(Sf).all()
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)
    assert torch.equal(Sf[4].cpu(), inp["S0"][4])  # the empty sequence keeps its initial state


@pytest.mark.parametrize("varlen", [False, True])
def test_equals_two_column_halves_bitwise(varlen):
    import linear_attention_sequence_rule_b200 as gdn
    kw = dict(lengths=[130, 0, 64, 257]) if varlen else dict(B=2, T=200)
    inp = workloads.make_chunk_inputs(H=2, dk=128, dv=DV, dtype="bf16", seed=13, s0_std=0.1, **kw)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"],
                            cu_seqlens=d["cu_seqlens"])
    halves = []
    for c in (slice(0, 128), slice(128, 256)):
        halves.append(gdn.chunk_fwd(d["q"], d["k"], d["v"][..., c].contiguous(), d["log_alpha"], d["beta"],
                                    S0=d["S0"][..., c].contiguous(), cu_seqlens=d["cu_seqlens"]))
    gdn.device_status()
    assert torch.equal(out, torch.cat([h[0] for h in halves], dim=-1))
    assert torch.equal(Sf, torch.cat([h[1] for h in halves], dim=-1))


def test_grouped_value_heads():
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_gva_chunk_inputs(B=2, T=200, Hk=1, Hv=3, dk=128, dv=DV, dtype="bf16", seed=17,
                                          s0_std=0.1, la_scale=0.3)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd_gva(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], S0=d["S0"])
    gdn.device_status()
    o_ref, s_ref = grouped.forward_gva(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"])
    e_o, e_s = max_abs(f64(out), o_ref), max_abs(f64(Sf), s_ref)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


@pytest.mark.parametrize("dk", [64, 128])
def test_fused_prologue(dk):
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_raw_chunk_inputs(B=2, T=150, H=2, dk=dk, dv=DV, dtype="bf16", seed=19 + dk,
                                          s0_std=0.1, la_scale=0.3)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd_fused(d["q_raw"], d["k_raw"], d["v"], d["a_raw"], d["b_raw"], inp["a_scale"],
                                  inp["b_scale"], S0=d["S0"])
    gdn.device_status()
    o_ref, s_ref = prologue.forward_fused(inp["q_raw"], inp["k_raw"], inp["v"], inp["a_raw"], inp["b_raw"],
                                          inp["S0"], inp["a_scale"], inp["b_scale"])
    e_o, e_s = max_abs(f64(out), o_ref), max_abs(f64(Sf), s_ref)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)


def test_host_entry_equals_device_entry():
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_chunk_inputs(lengths=[300, 5, 0, 190], H=2, dk=128, dv=DV, dtype="bf16", seed=23,
                                      s0_std=0.1)
    out_d, Sf_d = run_gpu_chunk(inp)
    pin = {k: (v.pin_memory() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out_h, Sf_h = gdn.chunk_fwd_host(pin["q"], pin["k"], pin["v"], pin["log_alpha"], pin["beta"], S0=pin["S0"],
                                     cu_seqlens=pin["cu_seqlens"])
    torch.cuda.synchronize()
    gdn.device_status()
    assert torch.equal(out_h, out_d.cpu()) and torch.equal(Sf_h, Sf_d.cpu())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_equals_two_column_halves_bitwise(dtype):
    import linear_attention_sequence_rule_b200 as gdn
    N, H, dk = 3, 4, 128
    S = workloads.make_decode_state(N, H, dk, DV, seed=29).cuda()
    S_halves = [S[..., :128].contiguous(), S[..., 128:].contiguous()]
    for step in range(5):
        x = {k: v.cuda() for k, v in workloads.make_decode_step_inputs(N, H, dk, DV, dtype, seed=29,
                                                                        step=step).items()}
        o = gdn.decode_step(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], S)
        o_h = [gdn.decode_step(x["q"], x["k"], x["v"][..., c].contiguous(), x["log_alpha"], x["beta"], Sh)
               for c, Sh in zip((slice(0, 128), slice(128, 256)), S_halves)]
        assert torch.equal(o, torch.cat(o_h, dim=-1)), step
    gdn.device_status()
    assert torch.equal(S, torch.cat(S_halves, dim=-1))


def test_decode_grouped_value_heads():
    import linear_attention_sequence_rule_b200 as gdn
    from tests.parity import TOL
    N, Hk, Hv, dk = 2, 1, 3, 128
    S = workloads.make_decode_state(N, Hv, dk, DV, seed=31)
    S_dev, S_ref = S.cuda(), S.double().numpy()
    g = torch.Generator().manual_seed(31)
    for step in range(6):
        q = torch.nn.functional.normalize(torch.randn(N, Hk, dk, generator=g), dim=-1).to(torch.bfloat16)
        k = torch.nn.functional.normalize(torch.randn(N, Hk, dk, generator=g), dim=-1).to(torch.bfloat16)
        v = torch.randn(N, Hv, DV, generator=g).to(torch.bfloat16)
        la = (-0.3 * torch.nn.functional.softplus(torch.randn(N, Hv, generator=g))).float()
        be = torch.sigmoid(torch.randn(N, Hv, generator=g)).float()
        o = gdn.decode_step_gva(q.cuda(), k.cuda(), v.cuda(), la.cuda(), be.cuda(), S_dev)
        o_ref, S_ref = grouped.decode_step_gva(q, k, v, la, be, S_ref)
        assert max_abs(f64(o), o_ref) <= TOL["bf16"], step
    gdn.device_status()
    assert max_abs(f64(S_dev), S_ref) <= TOL["bf16"]


def test_segment_scan_path():
    # one sequence, two heads, 40 chunks: 4 column-block chains, so the long sequence is cut into
    # segments (a workspace is needed); parity against the oracle, and bit identity with two
    # 128-column calls, which cut the sequence the same way
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.make_chunk_inputs(B=1, T=40 * 64, H=2, dk=128, dv=DV, dtype="bf16", seed=37, s0_std=0.1,
                                      la_scale=0.1)
    assert gdn.workspace_bytes(1, 40 * 64, 2, 128, DV) > 0
    out, Sf = run_gpu_chunk(inp)
    e_o, e_s = compare_chunk(inp, out, Sf)
    assert e_o <= TOL["bf16"] and e_s <= TOL["bf16"], (e_o, e_s)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    halves = [gdn.chunk_fwd(d["q"], d["k"], d["v"][..., c].contiguous(), d["log_alpha"], d["beta"],
                            S0=d["S0"][..., c].contiguous()) for c in (slice(0, 128), slice(128, 256))]
    gdn.device_status()
    assert torch.equal(out, torch.cat([h[0] for h in halves], dim=-1))
    assert torch.equal(Sf, torch.cat([h[1] for h in halves], dim=-1))
