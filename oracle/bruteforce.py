"""Brute-force restatement of the SSA decode step for tiny inputs (numpy, fp64).

TEST INFRASTRUCTURE ONLY.  An independent second formulation used to pin the
C oracle: instead of streaming over chunks it

* scores every chunk with one dense matrix product (all heads x all gists),
* finds the top-k set by enumerating every k-subset and keeping the one whose
  members all outrank every non-member under (score desc, index asc) -- the
  definition of "the k largest" with the lower-index tie rule,
* materialises the unfolded context as an explicit token list and runs one
  dense softmax over it.

Follows "Simplified Sparse Attention via Gist Tokens" sec. 3.2 / 3.3 (and
sec. 3.5 / App. B.2 for the two-level variant) under the same readings as the
C oracle.  Only for small M (subset enumeration is exponential).
"""
from __future__ import annotations

import itertools

import numpy as np


def _rank_key(scores: np.ndarray, i: int):
    v = scores[i]
    if np.isnan(v):
        v = -np.inf
    return (v, -i)


def _score_max(x: np.ndarray, axis=None):
    """Maximum over logits in which a NaN never wins: the largest non-NaN
    value, -inf when there is none (the NaN reading of the chunk score)."""
    return np.where(np.isnan(x), -np.inf, x).max(axis=axis)


def topk_subsets(scores: np.ndarray, cand, k: int):
    """Return the unique k-subset of ``cand`` that outranks its complement."""
    cand = list(cand)
    k = max(0, min(k, len(cand)))
    found = []
    for sub in itertools.combinations(cand, k):
        inside = set(sub)
        outside = [c for c in cand if c not in inside]
        if not sub or not outside:
            ok = True
        else:
            worst_in = min(_rank_key(scores, c) for c in sub)
            best_out = max(_rank_key(scores, c) for c in outside)
            ok = worst_in > best_out
        if ok:
            found.append(sorted(sub))
    assert len(found) == 1, f"top-k set not unique: {found}"
    return found[0]


def _softmax_attend(qh: np.ndarray, K: np.ndarray, V: np.ndarray):
    d = qh.shape[-1]
    if K.shape[0] == 0:  # an empty context attends to nothing
        return np.zeros(d), -np.inf
    logits = K @ qh / np.sqrt(d)
    mx = logits.max()
    w = np.exp(logits - mx)
    return (w[:, None] * V).sum(0) / w.sum(), mx + np.log(w.sum())


def decode(q, k_raw, v_raw, k_gist, v_gist, seq_lens, C, g, topk, sel=None, context=0, select=0):
    """context 0: unselected gists + selected raw + tail; 1: selected gists +
    selected raw + tail.  select 0: one top-k per KV head over the group's
    maximum; 1: each query head's own top-k (its own query only), union over
    the group (scores then per query head, sel_idx of G*topk entries)."""
    q = np.asarray(q, np.float64)
    k_raw, v_raw = np.asarray(k_raw, np.float64), np.asarray(v_raw, np.float64)
    k_gist, v_gist = np.asarray(k_gist, np.float64), np.asarray(v_gist, np.float64)
    B, Hq, d = q.shape
    Hkv, n_max = k_raw.shape[1], k_raw.shape[2]
    G = Hq // Hkv
    M_max = n_max // C
    cap = G * topk if select else topk
    scores = np.full((B, Hq if select else Hkv, M_max), -np.inf)
    sel_out = np.full((B, Hkv, cap), -1, np.int32)
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    ctx = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        n = int(seq_lens[b])
        M = n // C
        for j in range(Hkv):
            qg = q[b, j * G:(j + 1) * G]                       # [G, d]
            if M:
                gk = k_gist[b, j, :M].reshape(M * g, d)        # [M*g, d]
                s = (qg @ gk.T / np.sqrt(d)).reshape(G, M, g)  # [G, M, g]
                if select:
                    scores[b, j * G:(j + 1) * G, :M] = _score_max(s, axis=2)
                else:
                    scores[b, j, :M] = _score_max(s, axis=(0, 2))
            if sel is not None:
                chosen = [int(c) for c in sel[b, j] if c >= 0]
            elif select:
                chosen = sorted(set().union(*[topk_subsets(scores[b, j * G + r], range(M), topk)
                                              for r in range(G)]))
            else:
                chosen = topk_subsets(scores[b, j], range(M), topk)
            sel_out[b, j, :len(chosen)] = chosen
            keys, vals = [], []
            for m in range(M):
                picked = m in chosen
                if context == 0 and not picked or context == 1 and picked:
                    keys.append(k_gist[b, j, m])
                    vals.append(v_gist[b, j, m])
                if picked:
                    keys.append(k_raw[b, j, m * C:(m + 1) * C])
                    vals.append(v_raw[b, j, m * C:(m + 1) * C])
            keys.append(k_raw[b, j, M * C:n])
            vals.append(v_raw[b, j, M * C:n])
            K = np.concatenate(keys, 0)
            V = np.concatenate(vals, 0)
            ctx[b, j] = K.shape[0]
            for gh in range(G):
                h = j * G + gh
                out[b, h], lse[b, h] = _softmax_attend(q[b, h], K, V)
    return {"scores": scores, "sel_idx": sel_out, "out": out, "lse": lse, "ctx": ctx}


def decode_h2(q, k_raw, v_raw, k_gist, v_gist, k_meta, v_meta, seq_lens, C, g, J, gm,
              topk_super, topk_chunk):
    q = np.asarray(q, np.float64)
    k_raw, v_raw = np.asarray(k_raw, np.float64), np.asarray(v_raw, np.float64)
    k_gist, v_gist = np.asarray(k_gist, np.float64), np.asarray(v_gist, np.float64)
    k_meta, v_meta = np.asarray(k_meta, np.float64), np.asarray(v_meta, np.float64)
    B, Hq, d = q.shape
    Hkv, n_max = k_raw.shape[1], k_raw.shape[2]
    G = Hq // Hkv
    M_max = n_max // C
    S_max = M_max // J
    s2 = np.full((B, Hkv, S_max), -np.inf)
    s1 = np.full((B, Hkv, M_max), -np.inf)
    ss_out = np.full((B, Hkv, topk_super), -1, np.int32)
    sl_out = np.full((B, Hkv, topk_chunk), -1, np.int32)
    out = np.zeros((B, Hq, d))
    lse = np.full((B, Hq), -np.inf)
    ctx = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        n = int(seq_lens[b])
        M = n // C
        S = M // J
        for j in range(Hkv):
            qg = q[b, j * G:(j + 1) * G]
            if S:
                mk = k_meta[b, j, :S].reshape(S * gm, d)
                s2[b, j, :S] = _score_max((qg @ mk.T / np.sqrt(d)).reshape(G, S, gm), axis=(0, 2))
            sup = topk_subsets(s2[b, j], range(S), topk_super)
            ss_out[b, j, :len(sup)] = sup
            cand = [x * J + i for x in sup for i in range(J)] + list(range(S * J, M))
            for m in cand:
                s1[b, j, m] = _score_max(qg @ k_gist[b, j, m].T / np.sqrt(d))
            chosen = topk_subsets(s1[b, j], cand, topk_chunk)
            sl_out[b, j, :len(chosen)] = chosen
            keys, vals = [], []
            for x in range(S):
                if x not in sup:
                    keys.append(k_meta[b, j, x])
                    vals.append(v_meta[b, j, x])
            for m in cand:
                if m in chosen:
                    keys.append(k_raw[b, j, m * C:(m + 1) * C])
                    vals.append(v_raw[b, j, m * C:(m + 1) * C])
                else:
                    keys.append(k_gist[b, j, m])
                    vals.append(v_gist[b, j, m])
            keys.append(k_raw[b, j, M * C:n])
            vals.append(v_raw[b, j, M * C:n])
            K = np.concatenate(keys, 0)
            V = np.concatenate(vals, 0)
            ctx[b, j] = K.shape[0]
            for gh in range(G):
                h = j * G + gh
                out[b, h], lse[b, h] = _softmax_attend(q[b, h], K, V)
    return {"super_scores": s2, "scores": s1, "sel_super": ss_out, "sel_idx": sl_out,
            "out": out, "lse": lse, "ctx": ctx}


def decode_hier(q, k_raw, v_raw, k_gist, v_gist, k_sum, v_sum, seq_lens, C, g, J, topks):
    """t-level coarse-to-fine step, written as a recursion over kept units:
    a unit is scored when its parent was kept (or it is a top-level unit, or
    a remainder unit that lies in no complete parent), each level keeps its
    top-k by subset enumeration, and the context is built as an explicit
    token list (summaries of unkept candidates, gists of unkept candidate
    chunks, raw tokens of kept chunks, the tail)."""
    q = np.asarray(q, np.float64)
    k_raw, v_raw = np.asarray(k_raw, np.float64), np.asarray(v_raw, np.float64)
    k_gist, v_gist = np.asarray(k_gist, np.float64), np.asarray(v_gist, np.float64)
    k_sum = [np.asarray(x, np.float64) for x in k_sum]
    v_sum = [np.asarray(x, np.float64) for x in v_sum]
    t = len(topks)
    B, Hq, d = q.shape
    Hkv, n_max = k_raw.shape[1], k_raw.shape[2]
    G = Hq // Hkv
    sels = [np.full((B, Hkv, k), -1, np.int32) for k in topks]
    out = np.zeros((B, Hq, d))
    ctx = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        n = int(seq_lens[b])
        M = n // C
        U = [M]
        for _ in range(1, t):
            U.append(U[-1] // J)
        for j in range(Hkv):
            qg = q[b, j * G:(j + 1) * G]

            def keys_of(level, x):  # level 1-based
                return k_gist[b, j, x] if level == 1 else k_sum[level - 2][b, j, x]

            def vals_of(level, x):
                return v_gist[b, j, x] if level == 1 else v_sum[level - 2][b, j, x]

            keys, vals = [], []
            kept = []
            for level in range(t, 0, -1):
                if level == t:
                    cand = list(range(U[level - 1]))
                else:
                    cand = [x * J + i for x in kept for i in range(J)]
                    cand += list(range(U[level] * J, U[level - 1]))
                sc = np.full(max(U[level - 1], 1), -np.inf)
                for x in cand:
                    sc[x] = _score_max(qg @ keys_of(level, x).T / np.sqrt(d))
                keep = topk_subsets(sc, cand, topks[level - 1])
                sels[level - 1][b, j, :len(keep)] = keep
                for x in cand:
                    if level == 1 and x in keep:
                        keys.append(k_raw[b, j, x * C:(x + 1) * C])
                        vals.append(v_raw[b, j, x * C:(x + 1) * C])
                    elif x not in keep:
                        keys.append(keys_of(level, x))
                        vals.append(vals_of(level, x))
                kept = keep
            keys.append(k_raw[b, j, M * C:n])
            vals.append(v_raw[b, j, M * C:n])
            K = np.concatenate(keys, 0)
            V = np.concatenate(vals, 0)
            ctx[b, j] = K.shape[0]
            for gh in range(G):
                out[b, j * G + gh] = _softmax_attend(q[b, j * G + gh], K, V)[0]
    return {"sels": sels, "out": out, "ctx": ctx}
