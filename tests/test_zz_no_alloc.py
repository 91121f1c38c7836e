"""ssa_decode_noalloc (the entry point that uses the library's built-in
scratch instead of a workspace) against the oracle and against ssa_decode,
through the C ABI, on two calls in a row; and its size limit.  Collected last on purpose: it must pass
alone in a fresh process and after every other test."""
import ctypes

import pytest
import torch

from gist_token_chunk_b200.inputs import Workload, make_inputs
from parity import check_single

pytestmark = pytest.mark.gpu

W = Workload("noalloc", B=2, Hq=32, Hkv=8, d=64, n_max=8192, C=128, g=8, topk=16,
             seq_lens=(8192, 5000), planted=16)


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gist_token_chunk_b200 import ssa as mod

    return mod


def test_noalloc_matches_oracle_twice_in_a_row(ssa, orc):
    for seed in (5, 6):  # two calls in a row; the second finds the first's leftovers
        h = make_inputs(W, seed=seed)
        x = {k: v.cuda() for k, v in h.items() if k != "planted_idx"}
        o_ref, s_ref = ssa.ssa_decode(x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"],
                                      x["seq_lens"], W.C, W.g, W.topk)
        out = torch.empty(W.B, W.Hq, W.d, dtype=torch.float32, device="cuda")
        sel = torch.empty(W.B, W.Hkv, W.topk, dtype=torch.int32, device="cuda")
        ssa.ssa_decode_noalloc(x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"],
                               x["seq_lens"], W.C, W.g, W.topk, out, sel)
        torch.cuda.synchronize()
        assert ssa.ssa_get_device_status() == 0
        check_single(orc, h, W.C, W.g, W.topk, out, sel)
        assert torch.equal(sel, s_ref)
        assert (out - o_ref).abs().max().item() <= 1e-5


def test_noalloc_rejects_sizes_beyond_its_scratch(ssa):
    # 16 sequences x 8 KV heads at 64K with C=64, g=8 take the two-kernel path,
    # whose kept logits alone need ~16.8 MB, more than the built-in 16 MiB:
    # the call must fail on the host, before anything is enqueued.  The
    # tensors are real, full-size allocations, so the call would stay in
    # bounds even if the host check were wrong.
    B, Hq, Hkv, d, n_max, C, g, topk = 16, 32, 8, 64, 65536, 64, 8, 16
    sh = ssa.make_shape(B, Hq, Hkv, d, n_max, ssa.SSA_BF16)
    assert ssa.ssa_decode_path(sh, C, g, topk) == ssa.SSA_PATH_PIPELINE
    assert ssa.ssa_workspace_size(sh, C, g, topk) > 16 << 20
    bf = torch.bfloat16
    q = torch.zeros(B, Hq, d, dtype=bf, device="cuda")
    k_raw = torch.empty(B, Hkv, n_max, d, dtype=bf, device="cuda")
    v_raw = torch.empty_like(k_raw)
    k_gist = torch.zeros(B, Hkv, n_max // C, g, d, dtype=bf, device="cuda")
    v_gist = torch.zeros_like(k_gist)
    lens = torch.full((B,), n_max, dtype=torch.int32, device="cuda")
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    sel = torch.empty(B, Hkv, topk, dtype=torch.int32, device="cuda")
    st = ssa.lib.ssa_decode_noalloc(ctypes.byref(sh), q.data_ptr(), k_raw.data_ptr(),
                                    v_raw.data_ptr(), k_gist.data_ptr(), v_gist.data_ptr(),
                                    lens.data_ptr(), C, g, topk, out.data_ptr(), sel.data_ptr(),
                                    None)
    assert st == 3  # SSA_ERR_WORKSPACE
    assert b"built-in" in ssa.lib.ssa_last_error()
    del k_raw, v_raw, k_gist, v_gist
    torch.cuda.empty_cache()
