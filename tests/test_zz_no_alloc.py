"""gdn_chunk_fwd_noalloc (scratch from the library's fixed device array) against gdn_chunk_fwd
(scratch from a workspace the caller allocates), both through the C-ABI on the same inputs, two
no-alloc calls in a row each time.  The file is named to be collected last, so that it also runs
after every other test has used the library in the same process; it passes on its own as well.
"""
import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.init()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


CASES = {
    # the segment scan runs (scratch in use): one long sequence, both head sizes
    "segmented_d128": dict(B=1, T=81 * 64 - 45, H=2, dk=128, dv=128, seed=901),
    "segmented_d64_two_seqs": dict(B=2, T=2100, H=3, dk=64, dv=64, seed=902),
    # plans near the array's limit: 74 segments x 2 chains fill 148 SMs (29.1 MB at dk = dv = 128;
    # 24.2 MB at dv = 256, whose two column blocks count as the chains)
    "segmented_d128_full": dict(B=1, T=74 * 16 * 64 - 17, H=2, dk=128, dv=128, seed=904, min_mb=28),
    "segmented_dv256_full": dict(B=1, T=74 * 16 * 64, H=1, dk=128, dv=256, seed=905, min_mb=23),
    # no scratch needed: many chains
    "single_pass": dict(B=4, T=300, H=8, dk=64, dv=64, seed=903),
}


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry(name):
    import linear_attention_sequence_rule_b200 as gdn
    c = CASES[name]
    inp = workloads.make_chunk_inputs(B=c["B"], T=c["T"], H=c["H"], dk=c["dk"], dv=c["dv"],
                                      dtype="bf16", seed=c["seed"], s0_std=0.05, la_scale=0.1)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    B, T, H, dk, dv = c["B"], c["T"], c["H"], c["dk"], c["dv"]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    head = (_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["log_alpha"]), _p(d["beta"]), _p(d["S0"]))
    dims = (B, T, H, dk, dv, 64, None, gdn.GDN_DTYPE_BF16)

    need = gdn.gdn_chunk_fwd_workspace_bytes(B, T, H, dk, dv, 64, 0, gdn.GDN_DTYPE_BF16)
    assert (need > 0) == name.startswith("segmented")
    if "min_mb" in c and torch.cuda.get_device_properties(0).multi_processor_count == 148:
        assert c["min_mb"] * 1e6 <= need <= 32 * 2 ** 20, need
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    out_ref = torch.empty_like(d["v"])
    Sf_ref = torch.empty(B, H, dk, dv, device="cuda")
    rc = gdn.gdn_chunk_fwd(*head, _p(out_ref), _p(Sf_ref), *dims, _p(ws) if need else None, need,
                           stream)
    assert rc == gdn.GDN_OK, gdn.gdn_last_error()

    for _ in range(2):  # two calls in a row share the one scratch array
        out = torch.full_like(d["v"], float("nan"))
        Sf = torch.full((B, H, dk, dv), float("nan"), device="cuda")
        rc = gdn.gdn_chunk_fwd_noalloc(*head, _p(out), _p(Sf), *dims, stream)
        assert rc == gdn.GDN_OK, gdn.gdn_last_error()
        assert gdn.gdn_device_status(stream) == gdn.GDN_OK
        # the same kernels on the same segment plan: identical bits, so a partly overwritten or
        # stale scratch array would show here
        assert torch.equal(out, out_ref)
        assert torch.equal(Sf, Sf_ref)
