"""GPU-vs-oracle comparison rules shared by the GPU tests.

Criteria (written in the tests, applied here):
  * selected chunk (superchunk) indices are bit-exact wherever the oracle's
    k-th and (k+1)-th largest scores differ by more than NEAR_TIE;
  * at a near tie the GPU's selection must still be a valid top-k of the
    oracle's scores up to NEAR_TIE, and the oracle is re-run on the GPU's
    selection before outputs are compared;
  * outputs within MAX_ABS (max abs error) and MEAN_ABS (mean abs error) of the
    fp64 oracle.
"""
from __future__ import annotations

import numpy as np
import torch

NEAR_TIE = 1e-4
MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").float().numpy() if t.is_floating_point() else t.cpu().numpy()


def kth_gap(scores: np.ndarray, cand, k: int) -> float:
    """Gap between the k-th and (k+1)-th largest scores among `cand`."""
    vals = np.sort(np.asarray([scores[c] for c in cand], np.float64))[::-1]
    if k <= 0 or k >= len(vals):
        return np.inf
    return float(vals[k - 1] - vals[k])


def selection_is_valid_topk(scores: np.ndarray, cand, sel_row: np.ndarray, k: int) -> bool:
    """`sel_row` holds k ascending distinct entries of `cand` then only -1, and
    is a top-k of `scores` up to NEAR_TIE: min(selected) >= max(rest) - NEAR_TIE."""
    sel_row = np.asarray(sel_row)
    if len(sel_row) < k or not (sel_row[k:] == -1).all():
        return False
    chosen = [int(x) for x in sel_row[:k]]
    if any(x < 0 for x in chosen) or chosen != sorted(chosen) or len(set(chosen)) != k:
        return False
    cset = set(int(c) for c in cand)
    if any(c not in cset for c in chosen):
        return False
    taken = set(chosen)
    rest = [c for c in cand if c not in taken]
    if not chosen or not rest:
        return True
    return min(scores[c] for c in chosen) >= max(scores[c] for c in rest) - NEAR_TIE


def assert_outputs_close(gpu_out: np.ndarray, ref_out: np.ndarray, what: str = "out"):
    err = np.abs(gpu_out.astype(np.float64) - ref_out)
    assert np.isfinite(gpu_out).all(), f"{what}: non-finite GPU output"
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS, f"{what}: max abs err {mx:.3g} > {MAX_ABS}"
    assert mean <= MEAN_ABS, f"{what}: mean abs err {mean:.3g} > {MEAN_ABS}"
    return mx, mean


def check_single(orc, inp: dict, C: int, g: int, topk: int, gpu_out, gpu_sel) -> dict:
    """Compare a single-level decode step with the oracle; returns stats."""
    args = (inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"], inp["seq_lens"])
    ref = orc.decode(*args, C=C, g=g, topk=topk)
    sel = host(gpu_sel).astype(np.int32)
    out = host(gpu_out)
    B, Hkv = sel.shape[:2]
    lens = host(inp["seq_lens"])
    near = np.zeros((B, Hkv), bool)
    for b in range(B):
        M = int(lens[b]) // C
        k = min(topk, M)
        for j in range(Hkv):
            sc = ref["scores"][b, j]
            gap = kth_gap(sc, range(M), k)
            if gap > NEAR_TIE:
                assert np.array_equal(sel[b, j], ref["sel_idx"][b, j]), (
                    f"selection differs at (b={b}, j={j}) with gap {gap:.3g}: "
                    f"gpu {sel[b, j]} vs oracle {ref['sel_idx'][b, j]}")
            else:
                near[b, j] = True
                assert selection_is_valid_topk(sc, range(M), sel[b, j], k), (
                    f"near-tie selection at (b={b}, j={j}) is not a valid top-k: {sel[b, j]}")
    if near.any():
        ref = orc.decode(*args, C=C, g=g, topk=topk, sel=sel)
    mx, mean = assert_outputs_close(out, ref["out"])
    return {"max_abs": mx, "mean_abs": mean, "near_ties": int(near.sum())}


def check_h2(orc, inp: dict, C, g, J, gm, topk_super, topk_chunk, gpu_out, gpu_sup, gpu_sel):
    args = (inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"], inp["k_meta"],
            inp["v_meta"], inp["seq_lens"])
    kw = dict(C=C, g=g, J=J, gm=gm, topk_super=topk_super, topk_chunk=topk_chunk)
    ref = orc.decode_h2(*args, **kw)
    sup = host(gpu_sup).astype(np.int32)
    sel = host(gpu_sel).astype(np.int32)
    out = host(gpu_out)
    B, Hkv = sel.shape[:2]
    lens = host(inp["seq_lens"])
    near_s = False
    for b in range(B):
        S = (int(lens[b]) // C) // J
        ks = min(topk_super, S)
        for j in range(Hkv):
            gap = kth_gap(ref["super_scores"][b, j], range(S), ks)
            if gap > NEAR_TIE:
                assert np.array_equal(sup[b, j], ref["sel_super"][b, j]), (b, j, sup[b, j],
                                                                          ref["sel_super"][b, j])
            else:
                near_s = True
                assert selection_is_valid_topk(ref["super_scores"][b, j], range(S), sup[b, j], ks)
    if near_s:
        ref = orc.decode_h2(*args, sel_super=sup, **kw)
    near_c = False
    for b in range(B):
        M = int(lens[b]) // C
        S = M // J
        ks = min(topk_super, S)
        for j in range(Hkv):
            cand = [int(x) * J + i for x in ref["sel_super"][b, j][:ks] for i in range(J)]
            cand += list(range(S * J, M))
            kc = min(topk_chunk, len(cand))
            gap = kth_gap(ref["scores"][b, j], cand, kc)
            if gap > NEAR_TIE:
                assert np.array_equal(sel[b, j], ref["sel_idx"][b, j]), (b, j, sel[b, j],
                                                                        ref["sel_idx"][b, j])
            else:
                near_c = True
                assert selection_is_valid_topk(ref["scores"][b, j], cand, sel[b, j], kc)
    if near_c:
        ref = orc.decode_h2(*args, sel_super=ref["sel_super"], sel=sel, **kw)
    mx, mean = assert_outputs_close(out, ref["out"])
    return {"max_abs": mx, "mean_abs": mean, "near_ties": int(near_s) + int(near_c)}


def check_variant(orc, inp: dict, C: int, g: int, topk: int, context: int, select: int,
                  gpu_out, gpu_sel) -> dict:
    """Compare a decode step under a context / selection reading with the
    oracle.  Under the head-union selection every query head's own top-k is
    checked: away from near ties the union must equal the oracle's exactly;
    at a near tie of some head the GPU's union must contain that head's sure
    chunks (score > k-th + NEAR_TIE) and only chunks within NEAR_TIE of its
    k-th, and the oracle is re-run on the GPU's selection."""
    args = (inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"], inp["seq_lens"])
    ref = orc.decode(*args, C=C, g=g, topk=topk, context=context, select=select)
    sel = host(gpu_sel).astype(np.int32)
    out = host(gpu_out)
    B, Hkv = sel.shape[:2]
    G = ref["out"].shape[1] // Hkv
    lens = host(inp["seq_lens"])
    near = 0
    for b in range(B):
        M = int(lens[b]) // C
        k = min(topk, M)
        for j in range(Hkv):
            rows = [ref["scores"][b, j * G + r] for r in range(G)] if select else [ref["scores"][b, j]]
            gaps = [kth_gap(sc, range(M), k) for sc in rows]
            if min(gaps) > NEAR_TIE:
                assert np.array_equal(sel[b, j], ref["sel_idx"][b, j]), (
                    f"selection differs at (b={b}, j={j}): gpu {sel[b, j]} vs oracle "
                    f"{ref['sel_idx'][b, j]}")
                continue
            near += 1
            chosen = set(int(x) for x in sel[b, j] if x >= 0)
            assert list(sel[b, j][:len(chosen)]) == sorted(chosen)
            for sc in rows:
                if k == 0:
                    continue
                kth = np.sort(sc[:M])[::-1][k - 1]
                sure = {m for m in range(M) if sc[m] > kth + NEAR_TIE}
                assert sure <= chosen, (b, j, sure - chosen)
            allowed = set()
            for sc in rows:
                if k:
                    kth = np.sort(sc[:M])[::-1][k - 1]
                    allowed |= {m for m in range(M) if sc[m] >= kth - NEAR_TIE}
            assert chosen <= allowed, (b, j, chosen - allowed)
    if near:
        ref = orc.decode(*args, C=C, g=g, topk=topk, context=context, select=select, sel=sel)
    mx, mean = assert_outputs_close(out, ref["out"])
    return {"max_abs": mx, "mean_abs": mean, "near_ties": near}


def check_hier(orc, inp: dict, k_sum, v_sum, C: int, g: int, J: int, topks, gpu_out,
               gpu_sels) -> dict:
    """Compare a t-level step with the oracle: every level's selection
    bit-exact away from near ties (there the GPU's choice must be a valid
    top-k of the oracle's candidate scores, and the oracle is re-run on the
    GPU's selections of every level); outputs within the bars."""
    args = (inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"])
    ref = orc.decode_hier(*args, k_sum, v_sum, inp["seq_lens"], C=C, g=g, J=J, topks=topks)
    sels = [host(s).astype(np.int32) for s in gpu_sels]
    out = host(gpu_out)
    t = len(topks)
    near = 0
    B, Hkv = sels[0].shape[:2]
    for b in range(B):
        for j in range(Hkv):
            for l in range(t - 1, -1, -1):
                sc = ref["scores"][l][b, j]
                cand = [x for x in range(sc.shape[0]) if np.isfinite(sc[x])]
                k = min(topks[l], len(cand))
                if np.array_equal(sels[l][b, j], ref["sels"][l][b, j]):
                    continue
                # a different choice is allowed only at a near tie; the levels
                # below then see other candidates, so stop comparing this pair
                assert kth_gap(sc, cand, k) <= NEAR_TIE, (
                    f"level {l + 1} selection differs at (b={b}, j={j}): gpu {sels[l][b, j]} vs "
                    f"oracle {ref['sels'][l][b, j]}")
                assert selection_is_valid_topk(sc, cand, sels[l][b, j], k)
                near += 1
                break
    if near:
        ref = orc.decode_hier(*args, k_sum, v_sum, inp["seq_lens"], C=C, g=g, J=J, topks=topks,
                              sels=sels)
    mx, mean = assert_outputs_close(out, ref["out"])
    return {"max_abs": mx, "mean_abs": mean, "near_ties": near}
