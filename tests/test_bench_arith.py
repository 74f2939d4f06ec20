"""The benchmark's roofline arithmetic against counts made from first principles (CPU only).

The algorithmic flops of the chunk forward are counted here product by product over one chunk of
C tokens -- the multiply-adds of each triangular product enumerated row by row, the dense products
as 2 C dk dv each, the unit-lower inverse at its standard C^3/3 -- and compared with
``bench.algo_flops`` per token-head. Bytes are the tensors each call must move once. The figures
quoted with the results (46,357 and 140,501 flops per token-head; 132,104 bytes per decode state
at d = 128) are checked as well."""
import bench


def macs_lower(C, inclusive):
    """Multiply-adds of one output column of a (strictly or inclusively) lower C x C product."""
    return sum(r + 1 if inclusive else r for r in range(C))


def chunk_flops_per_token(C, dk, dv):
    f = 0
    f += 2 * dk * macs_lower(C, False)        # K K^T, strictly lower
    f += 2 * dk * macs_lower(C, True)         # Q K^T, lower inclusive
    f += 2 * dk * macs_lower(C, False)        # W = T diag(b gam) K with T unit lower
    f += 2 * dv * macs_lower(C, False)        # U~ = T diag(b) V
    f += 2 * dv * macs_lower(C, True)         # P U, P lower inclusive
    f += C ** 3 / 3                           # T = (I + A)^{-1}
    f += 3 * 2 * C * dk * dv                  # W S, (gam Q) S, K^T diag(lam) U
    return f / C


def test_chunk_flops_match_the_product_count():
    for dk, dv in ((64, 64), (128, 128), (64, 128), (128, 64), (128, 256)):
        assert abs(bench.algo_flops(1, dk, dv) - chunk_flops_per_token(64, dk, dv)) < 1e-9, (dk, dv)
    assert round(bench.algo_flops(1, 64, 64)) == 46357
    assert round(bench.algo_flops(1, 128, 128)) == 140501
    assert bench.algo_flops(7, 64, 64) == 7 * bench.algo_flops(1, 64, 64)


def test_chunk_bytes_are_each_tensor_once():
    th, n_states = 1000, 10
    for dk, dv, e in ((64, 64, 2), (128, 256, 2), (64, 64, 4)):
        q = k = th * dk * e
        v = out = th * dv * e
        gates = th * 2 * 4
        state = n_states * dk * dv * 4
        assert bench.algo_bytes(th, n_states, dk, dv, e, False, False) == q + k + v + out + gates
        assert bench.algo_bytes(th, n_states, dk, dv, e, True, True) == q + k + v + out + gates + 2 * state
        assert bench.algo_bytes(th, n_states, dk, dv, e, True, False) == q + k + v + out + gates + state


def test_decode_bytes_per_state():
    dk = dv = 128
    state_read_and_write = 2 * dk * dv * 4
    q_k_v_out = (dk + dk + dv + dv) * 2
    assert bench.DECODE_BYTES_PER_STATE(dk, dv, 2) == state_read_and_write + q_k_v_out + 8 == 132104


def test_backward_product_count():
    # 26 distinct products at dk = dv = 64 (8 forming the chunk maps, 1 per scan, 16 for the
    # gradients); 14 of them carry a value dimension, so dv = 128 adds 14; every product of the
    # chunk form grows with each key or value block it contracts over or produces
    assert bench.bwd_products(1, 1) == 26
    assert bench.bwd_products(1, 2) == 26 + 14
    assert bench.bwd_products(1, 4) == 26 + 3 * 14
    assert bench.bwd_products(2, 2) > bench.bwd_products(1, 2) + 26


def test_reference_arm_counts_tokens_not_token_heads(monkeypatch):
    """The reference arm's tokens/s is token-heads / H over the timed seconds, on a varlen pack
    whose chains differ in length; the per-sequence sub-problems both CPU legs time are the
    workload's own sequences in full."""
    import argparse
    import workloads
    inp = workloads.make_chunk_inputs(H=3, dk=64, dv=64, dtype="bf16", seed=5, lengths=[70, 5, 130])
    args = argparse.Namespace(steps=2, warmup=3)
    import oracle
    # 4 host threads over 3 heads: 2 whole sequences per step, taken in turn
    monkeypatch.setattr(oracle, "max_threads", lambda: 4)
    line = bench.run_reference(args, 1, 0, inp=inp)
    th, s = line["token_heads_timed"], line["seconds_timed"]
    assert line["unit"] == "tokens/s"
    assert abs(line["value"] - th / 3 / s) <= 1e-9 * line["value"]
    # warm-up steps take sequences {0, 1}, {2, 0}, {1, 2}; the timed ones {0, 1} and {2, 0}, all
    # 3 heads of each
    assert th == 3 * (70 + 5) + 3 * (130 + 70)
    # a sub-problem holds its sequences in full, and the oracle on it gives the same numbers as
    # the oracle on the whole pack
    import numpy as np
    sub, th2 = bench.oracle_subproblem(inp, [2, 0])
    assert th2 == 3 * (130 + 70)
    o_sub, s_sub = oracle.forward(*sub[:6], cu_seqlens=sub[6])
    o_all, s_all = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                                  inp["S0"], cu_seqlens=inp["cu_seqlens"])
    assert np.array_equal(o_sub, np.concatenate([o_all[75:205], o_all[0:70]]))
    assert np.array_equal(s_sub, s_all[[2, 0]])
    dense = workloads.make_chunk_inputs(B=2, T=40, H=3, dk=64, dv=64, dtype="bf16", seed=5)
    sub, th3 = bench.oracle_subproblem(dense, [1])
    assert th3 == 3 * 40
    o_sub, _ = oracle.forward(*sub[:6], cu_seqlens=sub[6])
    o_all, _ = oracle.forward(dense["q"], dense["k"], dense["v"], dense["log_alpha"], dense["beta"],
                              dense["S0"])
    assert np.array_equal(o_sub, o_all[1])
    assert bench.run_reference(args, 1, 1, inp=inp) is None
    assert line["config"] == bench.headline_config(1)
