"""Python binding of libssa (argument marshalling only).

Every step of the decode path runs in the library's CUDA kernels; this module
only turns torch tensors into pointers, allocates outputs with torch (device
memory is plumbing) and maps status codes to exceptions.  Importing it raises
``ImportError`` when ``libssa.so`` has not been built -- there is no fallback.

The functions carry the C ABI's names (see ``include/ssa.h``):
``ssa_score_gists``, ``ssa_topk_chunks``, ``ssa_sparse_decode``, ``ssa_decode``,
``ssa_decode_h2``, ``ssa_workspace_size``, ``ssa_workspace_size_h2``,
``ssa_workspace_init``, ``ssa_get_device_status``, and for the prefill and the
budget ``ssa_adaptive_topk``, ``ssa_prefill_plan_size``, ``ssa_prefill_plan``,
``ssa_prefill``, ``ssa_prefill_get_status``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SSA_LIB_PATH selects another build of the same library (e.g. one compiled
# with the SSA_TRACE timeline instrumentation); default: the in-tree build.
LIB_PATH = os.environ.get("SSA_LIB_PATH") or os.path.join(_HERE, "libssa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libssa.so not found at {LIB_PATH}: build it with gist_token_chunk_b200/build.py "
        "(or __graft_entry__.build()); there is no non-CUDA fallback")
lib = ctypes.CDLL(LIB_PATH)

SSA_OK = 0
SSA_ERR_INVALID_ARG = 1
SSA_ERR_UNSUPPORTED = 2
SSA_ERR_WORKSPACE = 3
SSA_ERR_CUDA = 4
SSA_ERR_DEVICE_STATUS = 5
SSA_ERR_DEVICE_TIMEOUT = 6
SSA_BF16 = 0
SSA_FP32 = 1
SSA_DEBUG_SKIP_PUBLISH = 1
SSA_DEBUG_FUSED_PATH = 2
SSA_PATH_GENERIC = 0
SSA_PATH_FUSED = 1
SSA_PATH_PIPELINE = 2
SSA_CONTEXT_UNSELECTED_GISTS = 0
SSA_CONTEXT_SELECTED_ONLY = 1
SSA_SELECT_GROUP_MAX = 0
SSA_SELECT_HEAD_UNION = 1
SSA_PREFILL_BM = 64
SSA_PREFILL_BN = 64
SSA_PREFILL_TILE_INTS = 8


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("n_max", ctypes.c_int32), ("dtype", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.c_size_t
_SH = ctypes.POINTER(Shape)

lib.ssa_score_gists.argtypes = [_SH, _P, _P, _P, _I, _I, _P, _P]
lib.ssa_topk_chunks.argtypes = [_SH, _P, _P, _I, _I, _P, _P]
lib.ssa_sparse_decode.argtypes = [_SH, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _S, _P]
lib.ssa_decode.argtypes = [_SH, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _S, _P]
lib.ssa_decode_noalloc.argtypes = [_SH, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P]
lib.ssa_decode_h2.argtypes = [_SH, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P,
                              _P, _P, _P, _S, _P]
lib.ssa_workspace_size.argtypes = [_SH, _I, _I, _I, ctypes.POINTER(_S)]
lib.ssa_decode_path.argtypes = [_SH, _I, _I, _I, ctypes.POINTER(_I)]
lib.ssa_decode_variant.argtypes = [_SH, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P,
                                   _S, _P]
lib.ssa_workspace_size_variant.argtypes = [_SH, _I, _I, _I, _I, _I, ctypes.POINTER(_S)]
_PP = ctypes.POINTER(ctypes.c_void_p)
_IP = ctypes.POINTER(ctypes.c_int32)
lib.ssa_decode_host.argtypes = [_SH, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _S, _P]
lib.ssa_workspace_size_host.argtypes = [_SH, _I, _I, _I, ctypes.POINTER(_S)]
lib.ssa_decode_hier.argtypes = [_SH, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _PP, _PP, _IP, _IP,
                                _P, _PP, _P, _S, _P]
lib.ssa_workspace_size_hier.argtypes = [_SH, _I, _I, _I, _I, _IP, _IP, ctypes.POINTER(_S)]
lib.ssa_workspace_size_h2.argtypes = [_SH, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_S)]
lib.ssa_workspace_init.argtypes = [_P, _S, _P]
lib.ssa_get_device_status.argtypes = [ctypes.POINTER(_I), _P]
lib.ssa_set_wait_limit.argtypes = [ctypes.c_int64]
lib.ssa_set_wait_limit.restype = None
lib.ssa_set_debug_flags.argtypes = [_I]
lib.ssa_set_debug_flags.restype = None
lib.ssa_set_tuning.argtypes = [_I, _I]
lib.ssa_set_tuning.restype = None
lib.ssa_status_string.argtypes = [_I]
lib.ssa_status_string.restype = ctypes.c_char_p
lib.ssa_last_error.argtypes = []
lib.ssa_last_error.restype = ctypes.c_char_p
lib.ssa_version.restype = _I
_I64 = ctypes.c_int64
lib.ssa_adaptive_topk.argtypes = [_I64, _I, _I, _I, ctypes.POINTER(_I)]
lib.ssa_prefill_plan_size.argtypes = [_I, _P, _I, _I, _I, ctypes.POINTER(_I64),
                                      ctypes.POINTER(_I64)]
lib.ssa_prefill_plan.argtypes = [_I, _P, _I, _I, _I, _P, _I64, _P, _I64]
lib.ssa_prefill.argtypes = [_SH, _P, _P, _P, _P, _P, _P, _I, _I, _P, _I64, _P, _I64, _P, _P, _P]
lib.ssa_prefill_get_status.argtypes = [ctypes.POINTER(_I), _P]
lib.ssa_prefill_last_error.argtypes = []
lib.ssa_prefill_last_error.restype = ctypes.c_char_p
for _f in ("ssa_adaptive_topk", "ssa_prefill_plan_size", "ssa_prefill_plan", "ssa_prefill",
           "ssa_prefill_get_status"):
    getattr(lib, _f).restype = _I
for _f in ("ssa_score_gists", "ssa_topk_chunks", "ssa_sparse_decode", "ssa_decode",
           "ssa_decode_path", "ssa_decode_variant", "ssa_workspace_size_variant",
           "ssa_decode_hier", "ssa_workspace_size_hier", "ssa_decode_host",
           "ssa_workspace_size_host",
           "ssa_decode_noalloc", "ssa_decode_h2", "ssa_workspace_size",
           "ssa_workspace_size_h2", "ssa_workspace_init", "ssa_get_device_status"):
    getattr(lib, _f).restype = _I


class SSAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: Optional[str] = None):
        self.status = status
        msg = lib.ssa_status_string(status).decode()
        if detail is None:
            detail = lib.ssa_last_error().decode()
        super().__init__(f"{where}: {msg} ({status}){': ' + detail if detail else ''}")


def _check(status: int, where: str) -> None:
    if status != SSA_OK:
        raise SSAError(status, where)


def _check_pf(status: int, where: str) -> None:
    """Status of a budget or prefill call (their detail text is kept apart)."""
    if status != SSA_OK:
        raise SSAError(status, where, lib.ssa_prefill_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SSA_BF16
    if t.dtype == torch.float32:
        return SSA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_shape(B, Hq, Hkv, d, n_max, dtype) -> Shape:
    return Shape(int(B), int(Hq), int(Hkv), int(d), int(n_max), int(dtype))


def shape_of(q: torch.Tensor, k_raw: torch.Tensor) -> Shape:
    B, Hq, d = q.shape
    Hkv, n_max = k_raw.shape[1], k_raw.shape[2]
    return make_shape(B, Hq, Hkv, d, n_max, _dtype_code(q))


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def ssa_decode_path(shape: Shape, C: int, g: int, topk: int) -> int:
    """SSA_PATH_PIPELINE, SSA_PATH_FUSED or SSA_PATH_GENERIC: the kernels
    ssa_decode runs for these sizes on the current device."""
    v = _I(0)
    _check(lib.ssa_decode_path(ctypes.byref(shape), C, g, topk, ctypes.byref(v)),
           "ssa_decode_path")
    return int(v.value)


def ssa_workspace_size(shape: Shape, C: int, g: int, topk: int) -> int:
    n = _S(0)
    _check(lib.ssa_workspace_size(ctypes.byref(shape), C, g, topk, ctypes.byref(n)),
           "ssa_workspace_size")
    return int(n.value)


def ssa_workspace_size_h2(shape: Shape, C, g, J, gm, topk_super, topk_chunk) -> int:
    n = _S(0)
    _check(lib.ssa_workspace_size_h2(ctypes.byref(shape), C, g, J, gm, topk_super, topk_chunk,
                                     ctypes.byref(n)), "ssa_workspace_size_h2")
    return int(n.value)


def ssa_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(lib.ssa_workspace_init(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "ssa_workspace_init")


def workspace(nbytes: int, device="cuda", stream=None) -> torch.Tensor:
    """A caller-owned workspace of ``nbytes``, initialised for first use."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    ssa_workspace_init(ws, stream)
    return ws


def ssa_score_gists(q, k_gist, seq_lens, C: int, g: int, n_max: int, scores=None, stream=None):
    B, Hq, d = q.shape
    Hkv, M_max = k_gist.shape[1], k_gist.shape[2]
    shape = make_shape(B, Hq, Hkv, d, n_max, _dtype_code(q))
    if scores is None:
        scores = torch.empty((B, Hkv, M_max), dtype=torch.float32, device=q.device)
    _check(lib.ssa_score_gists(ctypes.byref(shape), _ptr(q), _ptr(k_gist), _ptr(seq_lens), C, g,
                               _ptr(scores), _stream(stream)), "ssa_score_gists")
    return scores


def ssa_topk_chunks(scores, seq_lens, C: int, topk: int, n_max: int, sel_idx=None, stream=None):
    B, Hkv, _ = scores.shape
    shape = make_shape(B, Hkv, Hkv, 64, n_max, SSA_FP32)
    if sel_idx is None:
        sel_idx = torch.empty((B, Hkv, topk), dtype=torch.int32, device=scores.device)
    _check(lib.ssa_topk_chunks(ctypes.byref(shape), _ptr(scores), _ptr(seq_lens), C, topk,
                               _ptr(sel_idx), _stream(stream)), "ssa_topk_chunks")
    return sel_idx


def ssa_sparse_decode(q, k_raw, v_raw, k_gist, v_gist, seq_lens, C: int, g: int, topk: int,
                      sel_idx, out=None, ws=None, stream=None):
    shape = shape_of(q, k_raw)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.ssa_sparse_decode(ctypes.byref(shape), _ptr(q), _ptr(k_raw), _ptr(v_raw),
                                 _ptr(k_gist), _ptr(v_gist), _ptr(seq_lens), C, g, topk,
                                 _ptr(sel_idx), _ptr(out), _ptr(ws), nbytes, _stream(stream)),
           "ssa_sparse_decode")
    return out


def ssa_decode(q, k_raw, v_raw, k_gist, v_gist, seq_lens, C: int, g: int, topk: int, out=None,
               sel_idx=None, ws=None, stream=None):
    shape = shape_of(q, k_raw)
    B, Hkv = q.shape[0], k_raw.shape[1]
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if sel_idx is None:
        sel_idx = torch.empty((B, Hkv, topk), dtype=torch.int32, device=q.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.ssa_decode(ctypes.byref(shape), _ptr(q), _ptr(k_raw), _ptr(v_raw), _ptr(k_gist),
                          _ptr(v_gist), _ptr(seq_lens), C, g, topk, _ptr(out), _ptr(sel_idx),
                          _ptr(ws), nbytes, _stream(stream)), "ssa_decode")
    return out, sel_idx


def ssa_workspace_size_variant(shape: Shape, C: int, g: int, topk: int, context: int,
                               select: int) -> int:
    n = _S(0)
    _check(lib.ssa_workspace_size_variant(ctypes.byref(shape), C, g, topk, context, select,
                                          ctypes.byref(n)), "ssa_workspace_size_variant")
    return int(n.value)


def ssa_decode_variant(q, k_raw, v_raw, k_gist, v_gist, seq_lens, C: int, g: int, topk: int,
                       context: int = SSA_CONTEXT_UNSELECTED_GISTS,
                       select: int = SSA_SELECT_GROUP_MAX, out=None, sel_idx=None, ws=None,
                       stream=None):
    """The decode step under another context or selection reading (see
    include/ssa.h); sel_idx holds G * topk entries per KV head under the
    head-union selection."""
    shape = shape_of(q, k_raw)
    B, Hq, Hkv = q.shape[0], q.shape[1], k_raw.shape[1]
    cap = (Hq // Hkv) * topk if select == SSA_SELECT_HEAD_UNION else topk
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if sel_idx is None:
        sel_idx = torch.empty((B, Hkv, cap), dtype=torch.int32, device=q.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.ssa_decode_variant(ctypes.byref(shape), _ptr(q), _ptr(k_raw), _ptr(v_raw),
                                  _ptr(k_gist), _ptr(v_gist), _ptr(seq_lens), C, g, topk,
                                  context, select, _ptr(out), _ptr(sel_idx), _ptr(ws), nbytes,
                                  _stream(stream)), "ssa_decode_variant")
    return out, sel_idx


def _i32_array(xs):
    return (ctypes.c_int32 * max(len(xs), 1))(*[int(x) for x in xs])


def ssa_workspace_size_hier(shape: Shape, C: int, g: int, J: int, g_sum, topk) -> int:
    n = _S(0)
    _check(lib.ssa_workspace_size_hier(ctypes.byref(shape), C, g, J, len(topk), _i32_array(g_sum),
                                       _i32_array(topk), ctypes.byref(n)),
           "ssa_workspace_size_hier")
    return int(n.value)


def ssa_decode_hier(q, k_raw, v_raw, k_gist, v_gist, seq_lens, C: int, g: int, J: int, k_sum,
                    v_sum, topk, out=None, sels=None, ws=None, stream=None):
    """Coarse-to-fine decode step over t = len(topk) levels (see include/ssa.h):
    k_sum, v_sum are the t-1 summary tensors of levels 2..t [B,Hkv,Umax,g_l,d];
    returns out and one selection tensor per level [B,Hkv,topk[l]]."""
    shape = shape_of(q, k_raw)
    B, Hkv = q.shape[0], k_raw.shape[1]
    t = len(topk)
    assert len(k_sum) == len(v_sum) == t - 1
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if sels is None:
        sels = [torch.empty((B, Hkv, max(int(k), 1)), dtype=torch.int32, device=q.device)
                for k in topk]
    g_sum = [int(x.shape[3]) for x in k_sum]
    kp = (ctypes.c_void_p * max(t - 1, 1))(*[_ptr(x) for x in k_sum])
    vp = (ctypes.c_void_p * max(t - 1, 1))(*[_ptr(x) for x in v_sum])
    sp = (ctypes.c_void_p * t)(*[_ptr(x) for x in sels])
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.ssa_decode_hier(ctypes.byref(shape), _ptr(q), _ptr(k_raw), _ptr(v_raw),
                               _ptr(k_gist), _ptr(v_gist), _ptr(seq_lens), C, g, J, t, kp, vp,
                               _i32_array(g_sum), _i32_array(topk), _ptr(out), sp, _ptr(ws),
                               nbytes, _stream(stream)), "ssa_decode_hier")
    return out, [s[:, :, :int(k)] for s, k in zip(sels, topk)]


def ssa_workspace_size_host(shape: Shape, C: int, g: int, topk: int) -> int:
    n = _S(0)
    _check(lib.ssa_workspace_size_host(ctypes.byref(shape), C, g, topk, ctypes.byref(n)),
           "ssa_workspace_size_host")
    return int(n.value)


def ssa_decode_host(q_host, k_raw, v_raw, k_gist, v_gist, seq_lens_host, C: int, g: int,
                    topk: int, out_host, sel_idx_host, ws, stream=None):
    """ssa_decode with q, seq_lens, out and sel_idx in (pinned) host memory;
    the copies and the step are stream-ordered (see include/ssa.h)."""
    B, Hq, d = q_host.shape
    shape = make_shape(B, Hq, k_raw.shape[1], d, k_raw.shape[2], _dtype_code(q_host))
    _check(lib.ssa_decode_host(ctypes.byref(shape), _ptr(q_host), _ptr(k_raw), _ptr(v_raw),
                               _ptr(k_gist), _ptr(v_gist), _ptr(seq_lens_host), C, g, topk,
                               _ptr(out_host), _ptr(sel_idx_host), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)),
           "ssa_decode_host")
    return out_host, sel_idx_host


def ssa_decode_noalloc(q, k_raw, v_raw, k_gist, v_gist, seq_lens, C: int, g: int, topk: int,
                       out, sel_idx, stream=None):
    """ssa_decode without a workspace, for callers that cannot allocate:
    the library's built-in scratch is used (see include/ssa.h).  The caller
    passes the outputs; nothing is allocated here either."""
    shape = shape_of(q, k_raw)
    _check(lib.ssa_decode_noalloc(ctypes.byref(shape), _ptr(q), _ptr(k_raw), _ptr(v_raw),
                                  _ptr(k_gist), _ptr(v_gist), _ptr(seq_lens), C, g, topk,
                                  _ptr(out), _ptr(sel_idx), _stream(stream)),
           "ssa_decode_noalloc")
    return out, sel_idx


def ssa_decode_h2(q, k_raw, v_raw, k_gist, v_gist, k_meta, v_meta, seq_lens, C: int, g: int,
                  J: int, gm: int, topk_super: int, topk_chunk: int, out=None, sel_super=None,
                  sel_idx=None, ws=None, stream=None):
    shape = shape_of(q, k_raw)
    B, Hkv = q.shape[0], k_raw.shape[1]
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    if sel_super is None:
        sel_super = torch.empty((B, Hkv, topk_super), dtype=torch.int32, device=q.device)
    if sel_idx is None:
        sel_idx = torch.empty((B, Hkv, topk_chunk), dtype=torch.int32, device=q.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.ssa_decode_h2(ctypes.byref(shape), _ptr(q), _ptr(k_raw), _ptr(v_raw),
                             _ptr(k_gist), _ptr(v_gist), _ptr(k_meta), _ptr(v_meta),
                             _ptr(seq_lens), C, g, J, gm, topk_super, topk_chunk, _ptr(out),
                             _ptr(sel_super), _ptr(sel_idx), _ptr(ws), nbytes, _stream(stream)),
           "ssa_decode_h2")
    return out, sel_super, sel_idx


def ssa_get_device_status(stream=None) -> int:
    code = _I(0)
    _check(lib.ssa_get_device_status(ctypes.byref(code), _stream(stream)),
           "ssa_get_device_status")
    return int(code.value)


def ssa_set_wait_limit(ns: int) -> None:
    lib.ssa_set_wait_limit(int(ns))


def ssa_set_debug_flags(flags: int) -> None:
    lib.ssa_set_debug_flags(int(flags))


def ssa_set_tuning(max_blocks: int = 0, rows_per_score_item: int = 0) -> None:
    lib.ssa_set_tuning(int(max_blocks), int(rows_per_score_item))


# ------------------------------------------------------- budget, prefill ---

def ssa_adaptive_topk(n_kv: int, L: int, G: int, J: int = 1) -> int:
    """App. A selection budget: floor(n_kv / (L J G L)) + 1 (see include/ssa.h)."""
    k = _I(0)
    _check_pf(lib.ssa_adaptive_topk(int(n_kv), int(L), int(G), int(J), ctypes.byref(k)),
              "ssa_adaptive_topk")
    return int(k.value)


def _host_lens(seq_lens):
    import numpy as np

    if isinstance(seq_lens, torch.Tensor):
        seq_lens = seq_lens.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))


def ssa_prefill_plan_size(seq_lens, n_max: int, C: int, g: int):
    lens = _host_lens(seq_lens)
    nt, ne = ctypes.c_int64(0), ctypes.c_int64(0)
    _check_pf(lib.ssa_prefill_plan_size(len(lens), lens.ctypes.data, int(n_max), int(C), int(g),
                                        ctypes.byref(nt), ctypes.byref(ne)),
              "ssa_prefill_plan_size")
    return int(nt.value), int(ne.value)


def ssa_prefill_plan(seq_lens, n_max: int, C: int, g: int):
    """The block plan in host memory: (tiles int32 [n_tiles, 8], entries
    int32 [n_entries]) as torch CPU tensors; copy them to the device once and
    pass them to every layer's ssa_prefill."""
    lens = _host_lens(seq_lens)
    nt, ne = ssa_prefill_plan_size(lens, n_max, C, g)
    tiles = torch.zeros((max(nt, 1), SSA_PREFILL_TILE_INTS), dtype=torch.int32)
    entries = torch.zeros(max(ne, 1), dtype=torch.int32)
    _check_pf(lib.ssa_prefill_plan(len(lens), lens.ctypes.data, int(n_max), int(C), int(g),
                                   tiles.data_ptr(), nt, entries.data_ptr(), ne),
              "ssa_prefill_plan")
    return tiles[:nt], entries[:ne]


def ssa_prefill(q_raw, q_gist, k_raw, k_gist, v_raw, v_gist, C: int, g: int, plan_tiles,
                plan_entries, o_raw=None, o_gist=None, stream=None):
    """Prefill attention under the gist mask over the plan's blocks; the plan
    tensors live on the device.  Returns (o_raw, o_gist), fp32."""
    B, Hq, n_max, d = q_raw.shape
    shape = make_shape(B, Hq, k_raw.shape[1], d, n_max, _dtype_code(q_raw))
    if o_raw is None:
        o_raw = torch.zeros((B, Hq, n_max, d), dtype=torch.float32, device=q_raw.device)
    if o_gist is None:
        o_gist = torch.zeros(tuple(q_gist.shape), dtype=torch.float32, device=q_raw.device)
    gp = (lambda t: _ptr(t) if t.numel() else None)
    _check_pf(lib.ssa_prefill(ctypes.byref(shape), _ptr(q_raw), gp(q_gist), _ptr(k_raw),
                              gp(k_gist), _ptr(v_raw), gp(v_gist), int(C), int(g),
                              _ptr(plan_tiles), plan_tiles.shape[0], gp(plan_entries),
                              plan_entries.numel(), _ptr(o_raw), gp(o_gist), _stream(stream)),
              "ssa_prefill")
    return o_raw, o_gist


def ssa_prefill_get_status(stream=None) -> int:
    code = _I(0)
    _check_pf(lib.ssa_prefill_get_status(ctypes.byref(code), _stream(stream)),
              "ssa_prefill_get_status")
    return int(code.value)
