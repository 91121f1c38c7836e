"""Device-side behaviour of the C ABI: status words for bad inputs, bounded
waits that time out with a status instead of hanging, determinism, workspace
reuse, and invariance to the split-K decomposition."""
import numpy as np
import pytest
import torch

from gist_token_chunk_b200.inputs import Workload, make_inputs
from parity import host

pytestmark = pytest.mark.gpu

W1 = Workload("abi", B=2, Hq=32, Hkv=8, d=64, n_max=4096, C=64, g=8, topk=16,
              seq_lens=(4096, 2500), planted=16)


@pytest.fixture(scope="module")
def ssa():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gist_token_chunk_b200 import ssa as mod

    yield mod
    mod.ssa_set_tuning(0, 0)
    mod.ssa_set_debug_flags(0)
    mod.ssa_set_wait_limit(0)


@pytest.fixture(scope="module")
def inp():
    i = make_inputs(W1, seed=31)
    return {k: v.cuda() if k != "planted_idx" else v for k, v in i.items()}


def run(ssa, inp, ws=None, w=W1):
    return ssa.ssa_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"],
                          inp["seq_lens"], w.C, w.g, w.topk, ws=ws)


def test_bitwise_deterministic(ssa, inp):
    o1, s1 = run(ssa, inp)
    o2, s2 = run(ssa, inp)
    assert torch.equal(s1, s2) and torch.equal(o1, o2)


def test_workspace_reuse_stays_clean(ssa, inp):
    sh = ssa.shape_of(inp["q"], inp["k_raw"])
    ws = ssa.workspace(ssa.ssa_workspace_size(sh, W1.C, W1.g, W1.topk))
    o0, s0 = run(ssa, inp)  # library-allocated workspace
    for _ in range(3):
        o, s = run(ssa, inp, ws=ws)
        assert torch.equal(s, s0) and torch.equal(o, o0)
    # the same workspace serves another problem size, then the first again
    other = Workload("abi2", B=1, Hq=32, Hkv=8, d=64, n_max=2048, C=64, g=8, topk=4,
                     seq_lens=(1500,))
    oi = {k: v.cuda() if k != "planted_idx" else v for k, v in make_inputs(other, 3).items()}
    run(ssa, oi, ws=ws, w=other)
    o, s = run(ssa, inp, ws=ws)
    assert torch.equal(s, s0) and torch.equal(o, o0)
    assert ssa.ssa_get_device_status() == 0


@pytest.mark.parametrize("blocks", [1, 3, 37])
def test_split_invariance(ssa, inp, blocks):
    o0, s0 = run(ssa, inp)
    ssa.ssa_set_tuning(blocks, 128)
    try:
        o, s = run(ssa, inp)
    finally:
        ssa.ssa_set_tuning(0, 0)
    assert torch.equal(s, s0)
    assert (o - o0).abs().max().item() <= 1e-6


W_ODD = Workload("odd_g", B=2, Hq=8, Hkv=2, d=64, n_max=4800, C=48, g=3, topk=7,
                 seq_lens=(4799, 3001), planted=4)


@pytest.mark.parametrize("blocks,rows", [(5, 128), (23, 0), (61, 64)])
def test_split_invariance_odd_rows(ssa, blocks, rows):
    """g = 3: a block's kept scoring rows of a second pair (or sub-item)
    start at an odd row, so the gist pass reads them from any offset."""
    i = {k: v.cuda() if k != "planted_idx" else v for k, v in make_inputs(W_ODD, seed=5).items()}
    o0, s0 = run(ssa, i, w=W_ODD)
    ssa.ssa_set_tuning(blocks, rows)
    try:
        o, s = run(ssa, i, w=W_ODD)
    finally:
        ssa.ssa_set_tuning(0, 0)
    assert ssa.ssa_get_device_status() == 0
    assert torch.equal(s, s0)
    assert (o - o0).abs().max().item() <= 1e-5


W_TIE = Workload("ties", B=2, Hq=8, Hkv=2, d=64, n_max=8192, C=64, g=8, topk=16,
                 seq_lens=(8192, 5000), planted=0)


@pytest.mark.parametrize("blocks,rows", [(0, 0), (37, 0), (5, 128)])
def test_equal_scores_select_lowest_chunks(ssa, blocks, rows):
    """Every gist key of a pair equal: every chunk scores the same, so the
    selection is chunks 0..k-1 (ties to the lower index), however the chunks
    are split into scoring segments and sub-items."""
    i = {k: v.cuda() if k != "planted_idx" else v for k, v in make_inputs(W_TIE, seed=9).items()}
    kg = i["k_gist"]
    i["k_gist"] = kg[:, :, :1, :1, :].expand_as(kg).contiguous()
    ssa.ssa_set_tuning(blocks, rows)
    try:
        out, sel = run(ssa, i, w=W_TIE)
    finally:
        ssa.ssa_set_tuning(0, 0)
    assert ssa.ssa_get_device_status() == 0
    s = sel.cpu()
    for b, n in enumerate(W_TIE.seq_lens):
        k = min(W_TIE.topk, n // W_TIE.C)
        want = list(range(k)) + [-1] * (W_TIE.topk - k)
        for j in range(W_TIE.Hkv):
            assert s[b, j].tolist() == want, (b, j)


def test_bad_length_sets_status_and_zeroes(ssa, inp):
    bad = dict(inp)
    bad["seq_lens"] = torch.tensor([4096, 5000], dtype=torch.int32, device="cuda")  # > n_max
    out, sel = run(ssa, bad)
    assert ssa.ssa_get_device_status() == ssa.SSA_ERR_DEVICE_STATUS
    assert (out[1] == 0).all() and (sel[1] == -1).all()
    good, _ = run(ssa, inp)
    # the other sequence is unaffected; the split of the work over blocks
    # depends on the whole batch, so only fp32 summation order may differ
    assert (out[0] - good[0]).abs().max().item() <= 1e-5
    assert ssa.ssa_get_device_status() == 0


def test_bad_selection_sets_status_and_zeroes(ssa, inp):
    _, sel = run(ssa, inp)
    bad = sel.clone()
    bad[0, 3, 0], bad[0, 3, 1] = bad[0, 3, 1], bad[0, 3, 0]  # not ascending
    bad[1, 5, 0] = 10_000                                     # out of range
    out = ssa.ssa_sparse_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                                inp["v_gist"], inp["seq_lens"], W1.C, W1.g, W1.topk, bad)
    assert ssa.ssa_get_device_status() == ssa.SSA_ERR_DEVICE_STATUS
    G = W1.Hq // W1.Hkv
    assert (out[0, 3 * G:4 * G] == 0).all() and (out[1, 5 * G:6 * G] == 0).all()
    ref = ssa.ssa_sparse_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                                inp["v_gist"], inp["seq_lens"], W1.C, W1.g, W1.topk, sel)
    keep = torch.ones(W1.B, W1.Hq, dtype=torch.bool, device="cuda")
    keep[0, 3 * G:4 * G] = False
    keep[1, 5 * G:6 * G] = False
    assert torch.equal(out[keep], ref[keep])
    assert ssa.ssa_get_device_status() == 0


def test_wait_that_never_ends_times_out_with_status(ssa, inp):
    """A selection flag that nothing sets: the bounded waits run out, the
    call reports SSA_ERR_DEVICE_TIMEOUT, and the context stays usable."""
    _, sel = run(ssa, inp)
    sh = ssa.shape_of(inp["q"], inp["k_raw"])
    ws = ssa.workspace(ssa.ssa_workspace_size(sh, W1.C, W1.g, W1.topk))
    ssa.ssa_set_wait_limit(2_000_000)  # 2 ms
    ssa.ssa_set_debug_flags(ssa.SSA_DEBUG_SKIP_PUBLISH)
    try:
        ssa.ssa_sparse_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                              inp["v_gist"], inp["seq_lens"], W1.C, W1.g, W1.topk, sel, ws=ws)
        assert ssa.ssa_get_device_status() == ssa.SSA_ERR_DEVICE_TIMEOUT
    finally:
        ssa.ssa_set_debug_flags(0)
        ssa.ssa_set_wait_limit(0)
    ssa.ssa_workspace_init(ws)
    out = ssa.ssa_sparse_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                                inp["v_gist"], inp["seq_lens"], W1.C, W1.g, W1.topk, sel, ws=ws)
    ref, _ = run(ssa, inp)
    assert ssa.ssa_get_device_status() == 0
    assert (out - ref).abs().max().item() <= 1e-6


def test_fused_equals_components(ssa, inp):
    out, sel = run(ssa, inp)
    scores = ssa.ssa_score_gists(inp["q"], inp["k_gist"], inp["seq_lens"], W1.C, W1.g, W1.n_max)
    sel2 = ssa.ssa_topk_chunks(scores, inp["seq_lens"], W1.C, W1.topk, W1.n_max)
    assert torch.equal(sel, sel2)
    out2 = ssa.ssa_sparse_decode(inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"],
                                 inp["v_gist"], inp["seq_lens"], W1.C, W1.g, W1.topk, sel2)
    assert (out - out2).abs().max().item() <= 1e-6


def test_decode_host_buffers_equal_device_call(ssa, inp):
    """ssa_decode_host (pinned and pageable host buffers) gives ssa_decode's
    results."""
    out_d, sel_d = run(ssa, inp)
    sh = ssa.shape_of(inp["q"], inp["k_raw"])
    ws = ssa.workspace(ssa.ssa_workspace_size_host(sh, W1.C, W1.g, W1.topk))
    for pin in (True, False):
        q = inp["q"].cpu()
        lens = inp["seq_lens"].cpu()
        out = torch.empty(out_d.shape, dtype=torch.float32)
        sel = torch.empty(sel_d.shape, dtype=torch.int32)
        if pin:
            q, lens, out, sel = q.pin_memory(), lens.pin_memory(), out.pin_memory(), sel.pin_memory()
        ssa.ssa_decode_host(q, inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"], lens,
                            W1.C, W1.g, W1.topk, out, sel, ws)
        torch.cuda.synchronize()
        assert ssa.ssa_get_device_status() == 0
        assert torch.equal(sel, sel_d.cpu())
        assert (out - out_d.cpu()).abs().max().item() <= 1e-6
