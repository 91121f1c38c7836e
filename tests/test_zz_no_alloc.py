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
    # 128 sequences x 8 KV heads at 128K need far more than the built-in 8 MiB:
    # the call must fail on the host, before anything is enqueued.
    sh = ssa.make_shape(128, 32, 8, 64, 131072, 0)
    buf = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    st = ssa.lib.ssa_decode_noalloc(ctypes.byref(sh), p, p, p, p, p, p, 128, 8, 32, p, p, None)
    assert st == 3  # SSA_ERR_WORKSPACE
    assert b"built-in" in ssa.lib.ssa_last_error()
