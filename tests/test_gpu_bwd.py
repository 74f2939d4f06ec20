"""GPU parity of gdn_chunk_bwd against the fp64 backward oracle (oracle.backward, itself pinned by
finite differences) on the same inputs: dense and varlen (ragged, empty and one-token sequences),
exact resets, beta in (0, 2], with and without S0 and dS_final, bf16 and fp32 inputs, value head
sizes 64, 128 and 256 (the larger ones as 64-column value splits, also checked bit for bit against
separate 64-column calls whose q/k and gate gradients are summed).

The kernels compute with fp32-level accuracy from the stored input values (fp32 on the CUDA
cores, products as three tf32 tensor-core terms with a relative error below 2^-21; the oracle
reads the same values in fp64), so the bound is relative to each gradient's scale:
max |g - g_ref| <= 1e-5 * (1 + max |g_ref|) per tensor (a few 1e-7 is what these sizes give)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import f64

pytestmark = pytest.mark.gpu
RTOL = 1e-5


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def check(inp, seed, with_dsf=True):
    import linear_attention_sequence_rule_b200 as gdn
    g = torch.Generator().manual_seed(seed)
    lead = inp["v"].shape[:-1]
    dout = torch.randn(*lead, inp["dv"], generator=g).to(inp["v"].dtype)
    dsf = torch.randn(inp["B"], inp["H"], inp["dk"], inp["dv"], generator=g).float() if with_dsf else None
    d = {k2: (v2.cuda() if torch.is_tensor(v2) else v2) for k2, v2 in inp.items()}
    got = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dout.cuda(), S0=d["S0"],
                        dS_final=None if dsf is None else dsf.cuda(), cu_seqlens=d["cu_seqlens"])
    gdn.device_status()
    ref = oracle.backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"], dout,
                          dsf, cu_seqlens=inp["cu_seqlens"])
    errs = {}
    for name, a, b in zip(("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"), got, ref):
        a = f64(a)
        errs[name] = float(np.max(np.abs(a - b)) / (1.0 + np.max(np.abs(b)))) if a.size else 0.0
    assert max(errs.values()) <= RTOL, errs
    return errs


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense(dtype):
    inp = workloads.make_chunk_inputs(B=2, T=300, H=3, dk=64, dv=64, dtype=dtype, seed=11, s0_std=0.1,
                                      la_scale=0.3)
    check(inp, 1)


def test_dense_without_initial_state_or_final_gradient():
    inp = workloads.make_chunk_inputs(B=1, T=129, H=2, dk=64, dv=64, dtype="bf16", seed=12)
    check(inp, 2, with_dsf=False)


def test_varlen_ragged_with_resets_and_beta_two():
    inp = workloads.make_chunk_inputs(H=2, dk=64, dv=64, dtype="bf16", seed=13, s0_std=0.05,
                                      lengths=[1, 63, 64, 65, 0, 200, 130, 7], beta_scale=2.0, la_std=2.0)
    la, be = inp["log_alpha"], inp["beta"]
    la[5, 0] = -float("inf")
    la[64 + 63, 1] = -float("inf")     # the last token of a chunk
    la[193 + 64, 0] = -float("inf")    # the first token of a chunk
    be[300:320, 1] = 2.0
    check(inp, 3)


def test_hybrid_lm_heads_on_a_short_sequence():
    inp = workloads.make_chunk_inputs(B=2, T=512, H=12, dk=64, dv=64, dtype="bf16", seed=14, la_scale=0.1)
    check(inp, 4)


def test_hybrid_lm_full_size_sampled_sequences():
    # the benchmark's launch: all 8 x 4096 tokens x 12 heads on the GPU; the oracle checks two of
    # the eight sequences (every head), which depend on nothing outside themselves
    import linear_attention_sequence_rule_b200 as gdn
    inp = workloads.config_inputs("hybrid_lm")
    g = torch.Generator().manual_seed(15)
    dout = torch.randn(inp["v"].shape, generator=g).to(inp["v"].dtype)
    d = {k2: (v2.cuda() if torch.is_tensor(v2) else v2) for k2, v2 in inp.items()}
    got = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dout.cuda())
    gdn.device_status()
    for s in (0, 7):
        sl = slice(s, s + 1)
        ref = oracle.backward(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["log_alpha"][sl], inp["beta"][sl], None,
                              dout[sl], None)
        for name, a, b in zip(("dq", "dk", "dv", "dlog_alpha", "dbeta"), got, ref):
            a = f64(a[sl])
            err = float(np.max(np.abs(a - b)) / (1.0 + np.max(np.abs(b))))
            assert err <= RTOL, (s, name, err)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dv", [128, 256])
def test_value_splits_dense(dtype, dv):
    inp = workloads.make_chunk_inputs(B=2, T=200, H=2, dk=64, dv=dv, dtype=dtype, seed=15 + dv, s0_std=0.1,
                                      la_scale=0.3)
    check(inp, 5)


def test_value_splits_varlen_ragged_with_resets():
    inp = workloads.make_chunk_inputs(H=3, dk=64, dv=128, dtype="bf16", seed=16, s0_std=0.05,
                                      lengths=[1, 65, 0, 130, 64, 7], beta_scale=2.0, la_std=2.0)
    inp["log_alpha"][66 + 64, 2] = -float("inf")  # the first token of the 130-token sequence's second chunk
    check(inp, 6)
    check(inp, 7, with_dsf=False)


@pytest.mark.parametrize("varlen", [False, True])
def test_value_split_equals_64_column_calls_bitwise(varlen):
    import linear_attention_sequence_rule_b200 as gdn
    kw = dict(lengths=[70, 0, 129]) if varlen else dict(B=2, T=150)
    inp = workloads.make_chunk_inputs(H=2, dk=64, dv=128, dtype="bf16", seed=17, s0_std=0.1, **kw)
    g = torch.Generator().manual_seed(8)
    d = {k2: (v2.cuda() if torch.is_tensor(v2) else v2) for k2, v2 in inp.items()}
    dout = torch.randn(*inp["v"].shape, generator=g).to(inp["v"].dtype).cuda()
    dsf = torch.randn(inp["B"], inp["H"], 64, 128, generator=g).float().cuda()
    whole = gdn.chunk_bwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], dout, S0=d["S0"], dS_final=dsf,
                          cu_seqlens=d["cu_seqlens"])
    parts = [gdn.chunk_bwd(d["q"], d["k"], d["v"][..., c].contiguous(), d["log_alpha"], d["beta"],
                           dout[..., c].contiguous(), S0=d["S0"][..., c].contiguous(), dS_final=dsf[..., c].contiguous(),
                           cu_seqlens=d["cu_seqlens"]) for c in (slice(0, 64), slice(64, 128))]
    gdn.device_status()
    for i in (0, 1, 3, 4):  # dq, dk, dlog_alpha, dbeta: sums over the value blocks
        assert torch.equal(whole[i], parts[0][i] + parts[1][i]), i
    for i in (2, 5):  # dv, dS0: the value blocks side by side
        assert torch.equal(whole[i], torch.cat([parts[0][i], parts[1][i]], dim=-1)), i
