"""Failure detection without faulting the GPU: a kernel's bounded wait on an mbarrier that nothing
arrives on runs out (gdn_selftest_wait_timeout, 100 ms), the kernel records it in the library's
device error word and returns; gdn_device_status then reports GDN_ERR_TIMEOUT and clears the
record, and the context stays usable -- a chunk forward right after matches the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.parity import TOL, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def test_bounded_wait_runs_out_and_is_reported():
    import linear_attention_sequence_rule_b200 as gdn
    st = torch.cuda.current_stream().cuda_stream
    assert gdn.gdn_device_status(st) == gdn.GDN_OK
    assert gdn.gdn_selftest_wait_timeout(100, st) == gdn.GDN_OK
    assert gdn.gdn_device_status(st) == gdn.GDN_ERR_TIMEOUT
    assert "ran out" in gdn.gdn_last_error()
    assert gdn.gdn_device_status(st) == gdn.GDN_OK  # the record was cleared
    # the context is still usable
    inp = workloads.make_chunk_inputs(B=1, T=200, H=2, dk=64, dv=64, dtype="bf16", seed=91)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out, Sf = gdn.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"])
    gdn.device_status()
    o_ref, s_ref = oracle.forward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], None)
    assert max_abs(f64(out), o_ref) <= TOL["bf16"]
    assert max_abs(f64(Sf), s_ref) <= TOL["bf16"]


def test_selftest_rejects_unbounded_limits():
    import linear_attention_sequence_rule_b200 as gdn
    assert gdn.gdn_selftest_wait_timeout(0, None) == gdn.GDN_ERR_INVALID_ARGUMENT
    assert gdn.gdn_selftest_wait_timeout(5000, None) == gdn.GDN_ERR_INVALID_ARGUMENT
