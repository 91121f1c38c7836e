"""Seeded synthetic decode workloads for Simplified Sparse Attention (gist tokens).

This module only *draws inputs*; it holds none of the method's arithmetic (no
scoring, no selection, no attention).  Both the CUDA path and the CPU oracle
receive the tensors it returns, so it is the one piece the two sides share.

Recipe (stated once, used everywhere):

* ``torch.Generator`` seeded with ``seed`` on the device the tensors are made
  on.  Draw order: q, k_raw, v_raw, k_gist, v_gist, (k_meta, v_meta),
  seq_lens, planted chunk indices, planted directions.
* q and every K/V entry ~ N(0, 1), drawn in fp32, then cast to the storage
  dtype (bf16 with round-to-nearest-even, or kept fp32).  The oracle reads the
  cast values, so both sides see bit-identical inputs.
* Planted chunks stand in for "query-relevant" chunks of the pages'
  long-context workloads (Simplified Sparse Attention via Gist Tokens, sec. 3.2
  and 4.1): per (sequence, KV head) a set of complete chunks is drawn without
  replacement, and each of their gist keys is replaced by
  ``|z| * (0.3 u + sqrt(0.91) w)`` where ``u`` is the unit mean direction of
  the group's query heads, ``z ~ N(0, I)`` and ``w`` the unit part of ``z``
  orthogonal to ``u`` -- a key with cosine 0.3 to the group's query direction.
  For the two-level variant the meta-gist keys of the superchunks holding a
  planted chunk get the same treatment.
* ``seq_lens`` is either fixed or uniform on an integer interval (drawn from a
  CPU generator with the same seed, so it does not depend on the device).

Layouts (row-major, contiguous): q [B,Hq,d]; k_raw, v_raw [B,Hkv,n_max,d];
k_gist, v_gist [B,Hkv,M_max,g,d] with M_max = n_max // C;
k_meta, v_meta [B,Hkv,S_max,gm,d] with S_max = M_max // J; seq_lens int32 [B].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import torch


@dataclass(frozen=True)
class Workload:
    """Shape and selection parameters of one decode workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    n_max: int
    C: int
    g: int
    topk: int
    dtype: str = "bf16"  # "bf16" or "fp32"
    # sequence lengths: explicit tuple, or (lo, hi) drawn uniformly (inclusive)
    seq_lens: Optional[Sequence[int]] = None
    seq_range: Optional[tuple] = None
    # planted relevant chunks per (b, kv head): a count, or a fraction of M_b
    planted: int = 0
    planted_frac: float = 0.0
    # two-level (gist-of-gist) parameters; J == 0 means single level
    J: int = 0
    gm: int = 0
    topk_super: int = 0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def M_max(self) -> int:
        return self.n_max // self.C

    @property
    def S_max(self) -> int:
        return self.M_max // self.J if self.J else 0

    @property
    def two_level(self) -> bool:
        return self.J > 0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the decode study (tiny parity case, then the 32K-512K
# single-level cases, then the two-level gist-of-gist case).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", B=1, Hq=1, Hkv=1, d=64, n_max=261 + 11, C=16, g=2,
                          topk=4, dtype="fp32", seq_lens=(261,)),
    "llama1b_32k": Workload("llama1b_32k", B=8, Hq=32, Hkv=8, d=64, n_max=32768, C=64, g=8,
                            topk=16, seq_lens=(32768,) * 8, planted=16),
    "llama1b_128k_var": Workload("llama1b_128k_var", B=4, Hq=32, Hkv=8, d=64, n_max=131072,
                                 C=128, g=8, topk=32, seq_range=(65536, 131072), planted=16),
    "llama1b_512k": Workload("llama1b_512k", B=2, Hq=32, Hkv=8, d=64, n_max=524288, C=256,
                             g=8, topk=64, seq_lens=(524288,) * 2, planted_frac=0.05),
    "hssa_128k": Workload("hssa_128k", B=8, Hq=32, Hkv=8, d=64, n_max=131072, C=64, g=8,
                          topk=16, seq_lens=(131072,) * 8, planted=16, J=16, gm=8,
                          topk_super=8),
}


def _torch_dtype(name: str) -> torch.dtype:
    if name == "bf16":
        return torch.bfloat16
    if name == "fp32":
        return torch.float32
    raise ValueError(f"unknown dtype {name!r}")


def _normal(gen: torch.Generator, shape, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)


def make_inputs(w: Workload, seed: int, device="cpu", planted_scale: float = 0.3) -> dict:
    """Draw one seeded instance of workload ``w`` on ``device``.

    Returns a dict of tensors in the storage dtype (plus int32 seq_lens and the
    planted chunk indices as an int64 [B,Hkv,P] tensor, -1 padded).
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    B, Hq, Hkv, d, C, g = w.B, w.Hq, w.Hkv, w.d, w.C, w.g
    M_max = w.M_max
    q = _normal(gen, (B, Hq, d), device)
    k_raw = _normal(gen, (B, Hkv, w.n_max, d), device)
    v_raw = _normal(gen, (B, Hkv, w.n_max, d), device)
    k_gist = _normal(gen, (B, Hkv, M_max, g, d), device)
    v_gist = _normal(gen, (B, Hkv, M_max, g, d), device)
    k_meta = v_meta = None
    if w.two_level:
        k_meta = _normal(gen, (B, Hkv, w.S_max, w.gm, d), device)
        v_meta = _normal(gen, (B, Hkv, w.S_max, w.gm, d), device)

    if w.seq_lens is not None:
        lens = torch.tensor(list(w.seq_lens), dtype=torch.int64)
        assert lens.numel() == B
    elif w.seq_range is not None:
        # drawn on a CPU generator so the lengths (hence the work per query)
        # are the same whichever device the tensors are made on
        lo, hi = w.seq_range
        cpu_gen = torch.Generator()
        cpu_gen.manual_seed(int(seed))
        lens = torch.randint(lo, hi + 1, (B,), generator=cpu_gen)
    else:
        lens = torch.full((B,), w.n_max, dtype=torch.int64)
    seq_lens = lens.to(torch.int32)

    # planted chunks (input synthesis only)
    n_plant_max = 0
    plants = []
    for b in range(B):
        M_b = int(lens[b]) // C
        if w.planted_frac > 0:
            n_p = int(round(w.planted_frac * M_b))
        else:
            n_p = min(w.planted, M_b)
        n_plant_max = max(n_plant_max, n_p)
        plants.append((M_b, n_p))
    planted_idx = torch.full((B, Hkv, max(n_plant_max, 1)), -1, dtype=torch.int64)
    if n_plant_max > 0:
        group_dir = q.view(B, Hkv, w.G, d).sum(dim=2)
        group_dir = group_dir / group_dir.norm(dim=-1, keepdim=True).clamp_min(1e-30)
        ortho = math.sqrt(1.0 - planted_scale * planted_scale)
        for b in range(B):
            M_b, n_p = plants[b]
            if n_p == 0:
                continue
            for j in range(Hkv):
                perm = torch.randperm(M_b, generator=gen, device=device)[:n_p]
                idx = torch.sort(perm).values
                planted_idx[b, j, :n_p] = idx.cpu()
                u = group_dir[b, j]
                z = _normal(gen, (n_p, g, d), device)
                zpar = (z @ u)[..., None] * u
                wv = z - zpar
                wv = wv / wv.norm(dim=-1, keepdim=True).clamp_min(1e-30)
                keys = z.norm(dim=-1, keepdim=True) * (planted_scale * u + ortho * wv)
                k_gist[b, j, idx] = keys
                if w.two_level:
                    sup = torch.unique(idx // w.J)
                    sup = sup[sup < w.S_max]
                    if sup.numel():
                        zm = _normal(gen, (sup.numel(), w.gm, d), device)
                        wm = zm - (zm @ u)[..., None] * u
                        wm = wm / wm.norm(dim=-1, keepdim=True).clamp_min(1e-30)
                        k_meta[b, j, sup] = zm.norm(dim=-1, keepdim=True) * (
                            planted_scale * u + ortho * wm)

    dt = _torch_dtype(w.dtype)
    out = {
        "q": q.to(dt),
        "k_raw": k_raw.to(dt),
        "v_raw": v_raw.to(dt),
        "k_gist": k_gist.to(dt),
        "v_gist": v_gist.to(dt),
        "seq_lens": seq_lens.to(device),
        "planted_idx": planted_idx,
    }
    if w.two_level:
        out["k_meta"] = k_meta.to(dt)
        out["v_meta"] = v_meta.to(dt)
    return out


def small_variant(w: Workload, n_max: int, B: Optional[int] = None, seq_lens=None,
                  **kw) -> Workload:
    """A reduced copy of ``w`` (same heads, d, C, g, dtype) for oracle-sized runs."""
    B = w.B if B is None else B
    if seq_lens is None:
        seq_lens = (n_max,) * B
    return w.with_(name=w.name + f"_n{n_max}", B=B, n_max=n_max, seq_lens=tuple(seq_lens),
                   seq_range=None, **kw)


def make_level_summaries(w: Workload, J: int, g_sum, seed: int, device="cpu"):
    """Summary K/V of levels 2 .. len(g_sum) + 1 for a t-level step: level l's
    tensors are [B,Hkv,Umax(l),g_sum[l-2],d] with Umax(l) = (n_max / C) /
    J^(l-1), N(0, 1) in the workload's storage dtype (seeded; input
    synthesis only).  Returns (k_sum, v_sum) lists."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    dt = _torch_dtype(w.dtype)
    umax = w.M_max
    k_sum, v_sum = [], []
    for gl in g_sum:
        umax //= J
        shape = (w.B, w.Hkv, umax, int(gl), w.d)
        k_sum.append(_normal(gen, shape, device).to(dt))
        v_sum.append(_normal(gen, shape, device).to(dt))
    return k_sum, v_sum
