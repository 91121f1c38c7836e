"""ctypes wrapper and build step for the fp64 C oracle (``ssa_oracle.c``).

TEST INFRASTRUCTURE ONLY: used by ``tests/``, the package smoke check and the
bench's CPU-baseline leg.  The product library never imports this module.

The oracle follows "Simplified Sparse Attention via Gist Tokens", sec. 3.2
(scoring against gist keys), sec. 3.3 (top-k, hybrid attention over the
unfolded context), sec. 3.5 / App. B.2 (coarse-to-fine selection) in
``ssa_oracle.c``, and sec. 3.1 / 3.6 (prefill under the gist mask, its block
mask) and App. A (adaptive top-k) in ``prefill_oracle.c``; the readings each
takes where the pages are open are listed in the C files' headers.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ssa_oracle.c")
SOURCES = [SRC, os.path.join(HERE, "prefill_oracle.c")]


def lib_path(mutant: int = 0, out_dir: Optional[str] = None) -> str:
    out_dir = out_dir or HERE
    name = "libssa_oracle.so" if mutant == 0 else f"libssa_oracle_mut{mutant}.so"
    return os.path.join(out_dir, name)


def build(mutant: int = 0, out_dir: Optional[str] = None, force: bool = False) -> str:
    """Compile the oracle (optionally with one planted mutant) with gcc."""
    out = lib_path(mutant, out_dir)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= max(os.path.getmtime(f) for f in SOURCES)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", f"-DORACLE_MUTANT={mutant}", *SOURCES,
           "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


_F = ctypes.POINTER(ctypes.c_float)
_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int32)


def _f32(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _i32(x) -> np.ndarray:
    try:
        import torch

        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


class Oracle:
    """Loaded oracle library (default build, or a mutant for the pin tests)."""

    def __init__(self, path: Optional[str] = None, mutant: int = 0):
        self.path = path or build(mutant)
        self.lib = ctypes.CDLL(self.path)
        self.lib.oracle_decode.restype = ctypes.c_int
        self.lib.oracle_decode_v.restype = ctypes.c_int
        self.lib.oracle_decode_hier.restype = ctypes.c_int
        self.lib.oracle_decode_h2.restype = ctypes.c_int
        self.lib.oracle_mutant_id.restype = ctypes.c_int
        self.lib.oracle_adaptive_topk.restype = ctypes.c_int64
        self.lib.oracle_adaptive_topk.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_int]
        self.lib.oracle_prefill.restype = ctypes.c_int
        self.lib.oracle_prefill_rows.restype = ctypes.c_int
        self.lib.oracle_prefill_blocks.restype = ctypes.c_int64
        self.lib.oracle_prefill_blocks.argtypes = [
            ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _I,
            ctypes.c_int64, _I, ctypes.c_int64]

    @property
    def mutant(self) -> int:
        return int(self.lib.oracle_mutant_id())

    def decode(self, q, k_raw, v_raw, k_gist, v_gist, seq_lens, C: int, g: int, topk: int,
               sel: Optional[np.ndarray] = None, context: int = 0, select: int = 0) -> dict:
        """Single-level decode step.  ``sel`` given => attend on that selection.

        context 0: unselected gists + selected raw + tail; 1: selected gists +
        selected raw + tail (sec. 3.3 wording).  select 0: one selection per KV
        head (max over the group's heads); 1: per-head top-k, union over the
        group (App. A) -- then scores are per query head [B,Hq,M_max] and
        sel_idx has G*topk entries per KV head."""
        q, k_raw, v_raw = _f32(q), _f32(k_raw), _f32(v_raw)
        k_gist, v_gist = _f32(k_gist), _f32(v_gist)
        lens = _i32(seq_lens)
        B, Hq, d = q.shape
        Hkv, n_max = k_raw.shape[1], k_raw.shape[2]
        M_max = n_max // C
        G = Hq // Hkv
        assert k_gist.shape == (B, Hkv, M_max, g, d), (k_gist.shape, (B, Hkv, M_max, g, d))
        scores = np.empty((B, Hq if select else Hkv, M_max), np.float64)
        out = np.empty((B, Hq, d), np.float64)
        lse = np.empty((B, Hq), np.float64)
        ctx = np.empty((B, Hkv), np.int32)
        cap = G * topk if select else topk
        force = sel is not None
        sel_arr = (_i32(sel).copy() if force else np.empty((B, Hkv, cap), np.int32))
        assert sel_arr.shape == (B, Hkv, cap), (sel_arr.shape, (B, Hkv, cap))
        rc = self.lib.oracle_decode_v(
            B, Hq, Hkv, d, n_max, C, g, topk, int(context), int(select), _p(q, _F),
            _p(k_raw, _F), _p(v_raw, _F), _p(k_gist, _F), _p(v_gist, _F), _p(lens, _I),
            int(force), _p(scores, _D), _p(sel_arr, _I), _p(out, _D), _p(lse, _D), _p(ctx, _I))
        if rc < 0:
            raise ValueError("oracle_decode_v: bad shape, topk or mode")
        return {"scores": scores, "sel_idx": sel_arr, "out": out, "lse": lse, "ctx": ctx,
                "bad_seq": rc}

    def decode_h2(self, q, k_raw, v_raw, k_gist, v_gist, k_meta, v_meta, seq_lens, C: int,
                  g: int, J: int, gm: int, topk_super: int, topk_chunk: int,
                  sel_super: Optional[np.ndarray] = None,
                  sel: Optional[np.ndarray] = None) -> dict:
        """Two-level decode step; given selections are used instead of top-k."""
        q, k_raw, v_raw = _f32(q), _f32(k_raw), _f32(v_raw)
        k_gist, v_gist = _f32(k_gist), _f32(v_gist)
        k_meta, v_meta = _f32(k_meta), _f32(v_meta)
        lens = _i32(seq_lens)
        B, Hq, d = q.shape
        Hkv, n_max = k_raw.shape[1], k_raw.shape[2]
        M_max = n_max // C
        S_max = M_max // J
        assert k_meta.shape == (B, Hkv, S_max, gm, d)
        force = 0
        if sel_super is not None:
            ss = _i32(sel_super).copy()
            force |= 1
        else:
            ss = np.empty((B, Hkv, topk_super), np.int32)
        if sel is not None:
            sl = _i32(sel).copy()
            force |= 2
        else:
            sl = np.empty((B, Hkv, topk_chunk), np.int32)
        s2 = np.empty((B, Hkv, max(S_max, 1)), np.float64)
        s1 = np.empty((B, Hkv, M_max), np.float64)
        out = np.empty((B, Hq, d), np.float64)
        lse = np.empty((B, Hq), np.float64)
        ctx = np.empty((B, Hkv), np.int32)
        rc = self.lib.oracle_decode_h2(
            B, Hq, Hkv, d, n_max, C, g, J, gm, topk_super, topk_chunk, _p(q, _F),
            _p(k_raw, _F), _p(v_raw, _F), _p(k_gist, _F), _p(v_gist, _F), _p(k_meta, _F),
            _p(v_meta, _F), _p(lens, _I), force, _p(s2, _D), _p(s1, _D), _p(ss, _I),
            _p(sl, _I), _p(out, _D), _p(lse, _D), _p(ctx, _I))
        if rc < 0:
            raise ValueError("oracle_decode_h2: bad shape or topk")
        return {"super_scores": s2[:, :, :S_max], "scores": s1, "sel_super": ss, "sel_idx": sl,
                "out": out, "lse": lse, "ctx": ctx, "bad_seq": rc}


    def decode_hier(self, q, k_raw, v_raw, k_gist, v_gist, k_sum, v_sum, seq_lens, C: int,
                    g: int, J: int, topks, sels=None) -> dict:
        """t-level coarse-to-fine decode step, t = len(topks): level 1 = chunks
        (gists), level l >= 2 = units of J level-(l-1) units with summaries
        k_sum[l-2], v_sum[l-2] [B,Hkv,Umax(l),gs,d]; topks[l-1] kept at level
        l.  ``sels`` (one array per level) given => attend on those."""
        q, k_raw, v_raw = _f32(q), _f32(k_raw), _f32(v_raw)
        k_gist, v_gist = _f32(k_gist), _f32(v_gist)
        k_sum = [_f32(x) for x in k_sum]
        v_sum = [_f32(x) for x in v_sum]
        lens = _i32(seq_lens)
        t = len(topks)
        assert len(k_sum) == len(v_sum) == t - 1
        B, Hq, d = q.shape
        Hkv, n_max = k_raw.shape[1], k_raw.shape[2]
        umax = [n_max // C]
        for _ in range(1, t):
            umax.append(umax[-1] // J)
        gs = np.asarray([x.shape[3] for x in k_sum] or [0], np.int32)
        for l in range(1, t):
            assert k_sum[l - 1].shape == (B, Hkv, umax[l], int(gs[l - 1]), d), (l, k_sum[l - 1].shape)
        tk = np.asarray(list(topks), np.int32)
        scores = [np.empty((B, Hkv, max(u, 1)), np.float64) for u in umax]
        force = sels is not None
        sel_arr = ([_i32(x).copy() for x in sels] if force
                   else [np.empty((B, Hkv, max(int(k), 1)), np.int32) for k in topks])
        out = np.empty((B, Hq, d), np.float64)
        lse = np.empty((B, Hq), np.float64)
        ctx = np.empty((B, Hkv), np.int32)
        FP = ctypes.POINTER(ctypes.c_float)
        ksp = (FP * max(t - 1, 1))(*[_p(x, _F) for x in k_sum])
        vsp = (FP * max(t - 1, 1))(*[_p(x, _F) for x in v_sum])
        scp = (_D * t)(*[_p(x, _D) for x in scores])
        slp = (_I * t)(*[_p(x, _I) for x in sel_arr])
        rc = self.lib.oracle_decode_hier(
            B, Hq, Hkv, d, n_max, C, g, J, t, _p(gs, _I), _p(tk, _I), _p(q, _F), _p(k_raw, _F),
            _p(v_raw, _F), _p(k_gist, _F), _p(v_gist, _F), ksp, vsp, _p(lens, _I), int(force),
            scp, slp, _p(out, _D), _p(lse, _D), _p(ctx, _I))
        if rc < 0:
            raise ValueError("oracle_decode_hier: bad arguments")
        return {"scores": [sc[:, :, :u] for sc, u in zip(scores, umax)],
                "sels": [x[:, :, :int(k)] for x, k in zip(sel_arr, topks)],
                "out": out, "lse": lse, "ctx": ctx, "bad_seq": rc}

    def adaptive_topk(self, n_kv: int, L: int, G: int, J: int = 1) -> int:
        """App. A budget: chunks each query head keeps at every level (J = 1:
        SSA, J > 1: H-SSA with J chunks per meta-gist group)."""
        k = int(self.lib.oracle_adaptive_topk(int(n_kv), int(L), int(G), int(J)))
        if k < 0:
            raise ValueError("oracle_adaptive_topk: bad arguments")
        return k

    def prefill(self, q_raw, q_gist, k_raw, k_gist, v_raw, v_gist, seq_lens, C: int,
                g: int) -> dict:
        """Prefill attention under the gist mask (sec. 3.1), dense, fp64.
        Rows past each sequence's length are NaN in the result."""
        q_raw, q_gist = _f32(q_raw), _f32(q_gist)
        k_raw, k_gist, v_raw, v_gist = _f32(k_raw), _f32(k_gist), _f32(v_raw), _f32(v_gist)
        lens = _i32(seq_lens)
        B, Hq, n_max, d = q_raw.shape
        Hkv = k_raw.shape[1]
        M_max = n_max // C
        assert q_gist.shape == (B, Hq, M_max, g, d), (q_gist.shape, (B, Hq, M_max, g, d))
        assert k_gist.shape == v_gist.shape == (B, Hkv, M_max, g, d)
        assert k_raw.shape == v_raw.shape == (B, Hkv, n_max, d)
        o_raw = np.full((B, Hq, n_max, d), np.nan, np.float64)
        o_gist = np.full((B, Hq, M_max, g, d), np.nan, np.float64)
        rc = self.lib.oracle_prefill(
            B, Hq, Hkv, d, n_max, C, g, _p(lens, _I), _p(q_raw, _F), _p(q_gist, _F),
            _p(k_raw, _F), _p(k_gist, _F), _p(v_raw, _F), _p(v_gist, _F), _p(o_raw, _D),
            _p(o_gist, _D))
        if rc < 0:
            raise ValueError("oracle_prefill: bad shape")
        return {"o_raw": o_raw, "o_gist": o_gist, "bad_seq": rc}

    def prefill_rows(self, q_raw, q_gist, k_raw, k_gist, v_raw, v_gist, seq_lens, C: int,
                     g: int, rows) -> np.ndarray:
        """The prefill output of the listed rows only: rows = [(b, h, part,
        r), ...] with part 0 raw, 1 gist (r = m g + t); returns [len(rows), d]."""
        q_raw, q_gist = _f32(q_raw), _f32(q_gist)
        k_raw, k_gist, v_raw, v_gist = _f32(k_raw), _f32(k_gist), _f32(v_raw), _f32(v_gist)
        lens = _i32(seq_lens)
        B, Hq, n_max, d = q_raw.shape
        Hkv = k_raw.shape[1]
        rr = np.ascontiguousarray(np.asarray(rows, np.int32).reshape(-1, 4))
        out = np.empty((len(rr), d), np.float64)
        rc = self.lib.oracle_prefill_rows(
            B, Hq, Hkv, d, n_max, C, g, _p(lens, _I), _p(q_raw, _F), _p(q_gist, _F),
            _p(k_raw, _F), _p(k_gist, _F), _p(v_raw, _F), _p(v_gist, _F),
            ctypes.c_int64(len(rr)), _p(rr, _I), _p(out, _D))
        if rc < 0:
            raise ValueError("oracle_prefill_rows: bad shape or row")
        return out

    def prefill_blocks(self, n: int, C: int, g: int, BM: int, BN: int) -> list:
        """Block mask of one sequence (sec. 3.6) from the dense gist mask: a
        list of ((kind, r0, rows), [entries]) in the order raw tiles, gist
        tiles; entry = (block << 2) | (part << 1) | full, part 0 = gist
        columns (listed first), 1 = raw columns."""
        M = n // C
        nt = -(-n // BM) + -(-(M * g) // BM)
        cap = max(1, nt * (-(-n // BN) + -(-(M * g) // BN)))
        tiles = np.zeros((max(nt, 1), 4), np.int32)
        ents = np.zeros(cap, np.int32)
        ne = int(self.lib.oracle_prefill_blocks(int(n), C, g, BM, BN, _p(tiles, _I), nt,
                                                _p(ents, _I), cap))
        if ne < 0:
            raise ValueError("oracle_prefill_blocks: bad arguments")
        res, off = [], 0
        for i in range(nt):
            kind, r0, rows, cnt = (int(x) for x in tiles[i])
            res.append(((kind, r0, rows), [int(e) for e in ents[off:off + cnt]]))
            off += cnt
        assert off == ne
        return res


_default: Optional[Oracle] = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
