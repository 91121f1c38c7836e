"""Host logic of the prefill and the budget (no GPU compute): the library's
block plan against the oracle's plan, derived from the dense gist mask
(bit-exact), its ordering and sizes, the adaptive top-k against the oracle,
and the argument checks of every new call."""
import ctypes

import numpy as np
import pytest
import torch

from gist_token_chunk_b200 import ssa

BM, BN = ssa.SSA_PREFILL_BM, ssa.SSA_PREFILL_BN


def _by_sequence(tiles, entries):
    """The library's plan regrouped as the oracle lists it: per sequence, raw
    tiles then gist tiles, each with its entry list."""
    out = {}
    t = tiles.numpy()
    e = entries.numpy()
    for row in t:
        b, kind, r0, rows, n, begin, cnt, pad = (int(x) for x in row)
        assert pad == 0
        out.setdefault(b, []).append(((kind, r0, rows), [int(x) for x in e[begin:begin + cnt]], n))
    for b in out:
        out[b].sort(key=lambda x: (x[0][0], x[0][1]))
    return out


# (seq_lens, n_max, C, g): ragged lengths, empty and chunk-less sequences,
# chunks shorter and longer than a tile, C not a multiple of the block, g > 1
# tile of gists, long sequences
PLAN_CASES = [
    ([300, 5, 0, 128], 384, 128, 8),
    ([1000, 999, 64], 1024, 64, 8),
    ([517], 544, 32, 3),
    ([700, 33], 800, 100, 7),
    ([4096, 4000], 4096, 16, 1),
    ([130, 129], 192, 64, 80),
    ([1], 8, 8, 2),
    ([8], 8, 8, 2),
    ([20000, 12345], 20480, 128, 8),
]


@pytest.mark.parametrize("lens, n_max, C, g", PLAN_CASES)
def test_plan_matches_oracle(orc, lens, n_max, C, g):
    tiles, entries = ssa.ssa_prefill_plan(lens, n_max, C, g)
    nt, ne = ssa.ssa_prefill_plan_size(lens, n_max, C, g)
    assert tiles.shape == (nt, ssa.SSA_PREFILL_TILE_INTS) and entries.shape == (ne,)
    got = _by_sequence(tiles, entries)
    for b, n in enumerate(lens):
        want = orc.prefill_blocks(n, C, g, BM, BN)
        mine = got.get(b, [])
        assert [(t, e) for t, e, _ in mine] == want, (b, n)
        assert all(nn == n for _, _, nn in mine)
    # every entry belongs to exactly one tile, in one contiguous run
    t = tiles.numpy()
    spans = sorted((int(r[5]), int(r[6])) for r in t)
    pos = 0
    for begin, cnt in spans:
        assert begin == pos and cnt >= 1
        pos += cnt
    assert pos == ne


def test_plan_orders_longest_tiles_first():
    tiles, _ = ssa.ssa_prefill_plan([5000, 300, 4096], 5120, 128, 8)
    t = tiles.numpy()
    counts = t[:, 6]
    assert np.all(counts[:-1] >= counts[1:])
    # ties keep (b, part, r0) order
    for i in range(len(t) - 1):
        if counts[i] == counts[i + 1]:
            assert tuple(t[i, [0, 1, 2]]) < tuple(t[i + 1, [0, 1, 2]])


def test_plan_of_empty_batch():
    assert ssa.ssa_prefill_plan_size([], 128, 64, 8) == (0, 0)
    assert ssa.ssa_prefill_plan_size([0, 0], 128, 64, 8) == (0, 0)


@pytest.mark.parametrize("lens, n_max, C, g", [
    ([10], 64, 0, 8), ([10], 64, 16, 0), ([10], 60, 16, 8), ([70], 64, 16, 8), ([-1], 64, 16, 8),
])
def test_plan_rejects(lens, n_max, C, g):
    with pytest.raises(ssa.SSAError) as e:
        ssa.ssa_prefill_plan_size(lens, n_max, C, g)
    assert e.value.status == ssa.SSA_ERR_INVALID_ARG


def test_plan_rejects_small_buffers():
    lens = np.asarray([300], np.int32)
    nt, ne = ssa.ssa_prefill_plan_size(lens, 384, 128, 8)
    tiles = torch.zeros((nt, 8), dtype=torch.int32)
    ents = torch.zeros(ne, dtype=torch.int32)
    rc = ssa.lib.ssa_prefill_plan(1, lens.ctypes.data, 384, 128, 8, tiles.data_ptr(), nt,
                                  ents.data_ptr(), ne - 1)
    assert rc == ssa.SSA_ERR_INVALID_ARG
    assert not ents.any() and not tiles.any()
    assert b"entries" in ssa.lib.ssa_prefill_last_error()


def test_adaptive_topk_matches_oracle(orc):
    for n_kv in (0, 1, 2047, 2048, 65536, 131072, 10 ** 6, 2 ** 40):
        for L in (16, 64, 128):
            for G in (1, 4, 8, 16):
                for J in (1, 4, 8):
                    want = orc.adaptive_topk(n_kv, L, G, J)
                    if want > 2 ** 31 - 1:
                        with pytest.raises(ssa.SSAError) as e:
                            ssa.ssa_adaptive_topk(n_kv, L, G, J)
                        assert e.value.status == ssa.SSA_ERR_UNSUPPORTED
                    else:
                        assert ssa.ssa_adaptive_topk(n_kv, L, G, J) == want


@pytest.mark.parametrize("args, code", [
    ((-1, 128, 4, 1), ssa.SSA_ERR_INVALID_ARG), ((10, 0, 4, 1), ssa.SSA_ERR_INVALID_ARG),
    ((10, 128, 0, 1), ssa.SSA_ERR_INVALID_ARG), ((10, 128, 4, 0), ssa.SSA_ERR_INVALID_ARG),
    ((2 ** 62, 1, 1, 1), ssa.SSA_ERR_UNSUPPORTED),
])
def test_adaptive_topk_rejects(args, code):
    with pytest.raises(ssa.SSAError) as e:
        ssa.ssa_adaptive_topk(*args)
    assert e.value.status == code


def test_prefill_argument_checks_before_cuda():
    """Host-checkable errors return before any CUDA call (no GPU here)."""
    sh = ssa.make_shape(1, 4, 2, 64, 128, ssa.SSA_BF16)
    buf = ctypes.c_void_p(4096)  # never dereferenced: every case fails its checks first
    tiles = ctypes.c_void_p(4096)

    def call(shape=sh, C=64, g=8, nt=1, ne=1, q=buf, o=buf, t=tiles):
        return ssa.lib.ssa_prefill(ctypes.byref(shape), q, buf, buf, buf, buf, buf, C, g, t, nt,
                                   buf, ne, o, buf, None)

    assert call(C=0) == ssa.SSA_ERR_INVALID_ARG
    assert call(g=0) == ssa.SSA_ERR_INVALID_ARG
    assert call(C=48) == ssa.SSA_ERR_INVALID_ARG            # n_max not a multiple of C
    assert call(nt=-1) == ssa.SSA_ERR_INVALID_ARG
    assert call(q=None) == ssa.SSA_ERR_INVALID_ARG
    assert call(t=None) == ssa.SSA_ERR_INVALID_ARG
    assert call(o=ctypes.c_void_p(4100)) == ssa.SSA_ERR_INVALID_ARG  # misaligned
    assert call(shape=ssa.make_shape(1, 4, 3, 64, 128, ssa.SSA_BF16)) == ssa.SSA_ERR_INVALID_ARG
    assert call(shape=ssa.make_shape(1, 4, 2, 64, 128, ssa.SSA_FP32)) == ssa.SSA_ERR_UNSUPPORTED
    assert call(shape=ssa.make_shape(1, 4, 2, 96, 128, ssa.SSA_BF16)) == ssa.SSA_ERR_UNSUPPORTED
    assert call(nt=0) == ssa.SSA_OK                          # nothing to do
    assert ssa.lib.ssa_prefill(None, buf, buf, buf, buf, buf, buf, 64, 8, tiles, 1, buf, 1, buf,
                               buf, None) == ssa.SSA_ERR_INVALID_ARG


def test_header_intervals_are_the_mask():
    """The per-row column intervals include/ssa.h states (and the kernel's
    element mask evaluates) give exactly the visible sets listed from the
    sentence of sec. 3.1, for every shape the GPU tests use."""
    from oracle_pins import _visible_sets

    def intervals(kind, r, C, g):
        if kind == 0:
            m = r // C
            return (0, m * g), (m * C, r + 1)
        m = r // g
        return (0, r + 1), (m * C, m * C + C)

    for n, C, g in ((1024, 128, 8), (777, 128, 8), (768, 16, 2), (1000, 100, 7), (450, 100, 7),
                    (256, 64, 80), (100, 128, 8), (5, 128, 8), (2047, 32, 3), (3000, 64, 4)):
        raw_rows, gist_rows, pos_raw, pos_gist = _visible_sets(n, C, g)
        for kind, rows in ((0, raw_rows), (1, gist_rows)):
            for r, (own, gists) in enumerate(rows):
                (gl, gh), (rl, rh) = intervals(kind, r, C, g)
                got = ({pos_gist(c // g, c % g) for c in range(gl, gh)}
                       | {pos_raw(c) for c in range(rl, rh)})
                assert got == set(own) | set(gists), (n, C, g, kind, r)


def test_plan_random_sizes_match_oracle(orc):
    """Seeded random (n, C, g): the library's plan equals the oracle's,
    derived pair by pair from the dense mask (the kernel trusts the full
    flags, so a wrong one would go unmasked)."""
    rng = np.random.default_rng(2024)
    done = 0
    while done < 40:
        C = int(rng.choice([1, 2, 3, 7, 16, 33, 64, 100, 128, 200, 256]))
        g = int(rng.integers(1, 90))
        n = int(rng.integers(0, 3000))
        if n + (n // C) * g > 3000:
            continue
        n_max = -(-max(n, 1) // C) * C
        tiles, entries = ssa.ssa_prefill_plan([n], n_max, C, g)
        got = _by_sequence(tiles, entries).get(0, [])
        assert [(t, e) for t, e, _ in got] == orc.prefill_blocks(n, C, g, BM, BN), (n, C, g)
        done += 1
