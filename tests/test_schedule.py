"""Host logic of the tensor-core work schedule, checked without a GPU.

The plan comes from the C-ABI plan query; the enumeration below restates how
each CTA walks its segments (whole tiles first, then its share of the tail
units) and which partial slot it writes, and how the merge kernel finds the
segments of a split tile.  Every (tile, unit) must be computed exactly once,
every split tile merged from exactly the slots its CTAs wrote, and no slot
may fall outside the workspace's two partial rows per CTA."""

import numpy as np

import pytest

import attention_cascade_b200 as jev


def _walk(p):
    n, fw, tail0, tc, U, P = (p[k] for k in ("n_ctas", "full_waves", "tail0", "tail_ctas", "tail_units",
                                             "units_per_tile"))
    begin = lambda c: c * U // tc
    cover, writes = {}, {}
    for c in range(n):
        has_tail = U > 0 and c < tc
        u, u_end = (begin(c), begin(c + 1)) if has_tail else (0, 0)
        k, slots = 0, []
        while True:
            if k < fw:
                w, ua, ub, tail = c + k * n, 0, P, False
            elif u < u_end:
                wt = u // P
                w, ua, ub, tail = tail0 + wt, u - wt * P, min(u_end, wt * P + P) - wt * P, True
                u = wt * P + ub
            else:
                break
            assert 0 <= w < p["n_tiles"]
            for x in range(ua, ub):
                assert (w, x) not in cover, "unit computed twice"
                cover[(w, x)] = c
            if not (ua == 0 and ub == P):
                slot = 2 * c if begin(c) >= (w - tail0) * P else 2 * c + 1
                slots.append(slot)
                writes.setdefault(w, []).append(slot)
            k += 1
        assert len(slots) == len(set(slots)) <= 2
    return cover, writes


def _merged(p):
    tc, U, P, tail0 = p["tail_ctas"], p["tail_units"], p["units_per_tile"], p["tail0"]
    out = {}
    if tc < 2 or p["n_tiles"] <= tail0:
        return out
    begin = lambda c: c * U // tc
    cta_of = lambda u: ((u + 1) * tc - 1) // U
    for bx in range(p["n_tiles"] - tail0):
        t0 = bx * P
        lo, hi = cta_of(t0), cta_of(t0 + P - 1)
        if lo == hi:
            continue
        slot_lo = 2 * lo if begin(lo) >= t0 else 2 * lo + 1
        out[tail0 + bx] = [slot_lo] + [2 * (lo + s) for s in range(1, hi - lo + 1)]
    return out


def _check(p):
    cover, writes = _walk(p)
    assert len(cover) == p["n_tiles"] * p["units_per_tile"]
    merged = _merged(p)
    assert set(merged) == set(writes)
    for w, slots in merged.items():
        assert sorted(slots) == sorted(writes[w])
        assert max(slots) < 2 * p["n_ctas"]
    assert bool(p["split"]) == bool(writes)


SHAPES = [  # (B, T, Lp, Hq, Hkv)
    (1, 1, 0, 4, 4), (3, 18, 128, 14, 2), (8, 138, 1024, 12, 2), (32, 700, 2048, 28, 4),
    (128, 3072, 4096, 28, 4), (5, 333, 300, 8, 1), (64, 1500, 6000, 32, 8), (2, 40000, 128, 8, 8),
]


@pytest.fixture
def tile_rows():
    """Forces the rows per tensor-core work tile for the test's plans (0: the
    plan chooses) and restores the automatic choice afterwards."""
    def force(rows):
        jev.jev_debug_set_tc_tile_rows(rows)
    yield force
    jev.jev_debug_set_tc_tile_rows(0)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("num_splits", [0, 1, 2, 3, 7])
@pytest.mark.parametrize("sms", [148, 132, 7, 1])
@pytest.mark.parametrize("rows", [0, 128, 256])
def test_schedule_covers_every_unit_once(shape, num_splits, sms, rows, tile_rows):
    B, T, Lp, Hq, Hkv = shape
    tile_rows(rows)
    desc = jev.make_attn_desc(B, Lp, Hq, Hkv, 128, T, jev.JEV_BF16, num_splits=num_splits)
    p = jev.jev_prefix_suffix_attn_plan(desc, kernel=1, num_sms=sms)
    assert p["kernel"] == 1
    assert p["tile_rows"] == (rows or p["tile_rows"]) and p["tile_rows"] in (128, 256)
    assert p["n_tiles"] == -(-T * (Hq // Hkv) // p["tile_rows"]) * Hkv
    assert p["units_per_tile"] == -(-Lp // 128) + 1
    if num_splits == 1:
        assert p["split"] == 0 and p["n_ctas"] <= sms
    if num_splits in (0, 1):
        assert p["n_ctas"] <= sms  # persistent: at most one CTA per SM
    _check(p)


def test_tile_rows_choice():
    """128-row work tiles (the one-Q-tile kernel) when 256-row tiles would be
    fewer than the SMs and their units fewer than 20 a CTA, else 256-row tiles
    (the two-Q-tile kernel); 0 for the CUDA-core plan."""
    def rows(B, Lp, Hq, Hkv, T, sms=148, kernel=1):
        return jev.jev_prefix_suffix_attn_plan(jev.make_attn_desc(B, Lp, Hq, Hkv, 128, T, jev.JEV_BF16), kernel,
                                               sms)["tile_rows"]
    assert rows(128, 4096, 28, 4, 3202) == 256     # 352 tiles of 256 rows
    assert rows(32, 2048, 28, 4, 707) == 128       # 80 tiles of 256 rows on 148 SMs
    assert rows(32, 2048, 28, 4, 707, sms=80) == 256   # 80 tiles: a whole wave of 80 SMs
    assert rows(32, 2048, 28, 4, 707, sms=81) == 128   # 1360 units < 20 x 81
    assert rows(32, 2048, 28, 4, 707, sms=68) == 256   # 1360 units = 20 x 68, and a wave
    assert rows(48, 8192, 28, 4, 1233) == 256      # 136 tiles of 65 units: 59.7 units a CTA
    assert rows(80, 2048, 28, 4, 896) == 128       # 100 tiles of 17 units: 11.5 a CTA
    assert rows(8, 1024, 12, 2, 128) == 128
    assert rows(8, 1024, 12, 2, 128, kernel=0) == 0
    with pytest.raises(jev.JevError):
        jev.jev_debug_set_tc_tile_rows(64)


def test_auto_schedule_choices():
    # fewer tiles than SMs and a long prefix: every tile is spread over several CTAs
    p = jev.jev_prefix_suffix_attn_plan(jev.make_attn_desc(8, 1024, 12, 2, 128, 138, jev.JEV_BF16), 1, 148)
    assert p["tile_rows"] == 128
    assert p["full_waves"] == 0 and p["split"] == 1 and p["n_ctas"] > p["n_tiles"]
    # 352 tiles on 148 SMs: two whole waves, only the 56 tail tiles are shared
    p = jev.jev_prefix_suffix_attn_plan(jev.make_attn_desc(128, 4096, 28, 4, 128, 3072, jev.JEV_BF16), 1, 148)
    assert p["tile_rows"] == 256 and (p["n_tiles"] == 336 or p["n_tiles"] == 352)
    assert p["full_waves"] == 2 and p["tail0"] == 296 and p["n_ctas"] == 148
    # as many tiles as SMs: one whole tile each, nothing to merge
    p = jev.jev_prefix_suffix_attn_plan(jev.make_attn_desc(1, 512, 4, 4, 128, 9472, jev.JEV_BF16), 1, 148)
    assert p["n_tiles"] == 148 and p["split"] == 0 and p["full_waves"] == 1


def test_plan_query_rejects_bad_arguments():
    desc = jev.make_attn_desc(2, 128, 8, 2, 128, 10, jev.JEV_BF16)
    with pytest.raises(jev.JevError):
        jev.jev_prefix_suffix_attn_plan(desc, kernel=2)
    with pytest.raises(jev.JevError):
        jev.jev_prefix_suffix_attn_plan(jev.make_attn_desc(2, 128, 8, 3, 128, 10, jev.JEV_BF16))
    # the CUDA-core plan: prefix splits of whole 32-key tiles covering Lp exactly once
    for Lp, ns in ((1000, 3), (1000, 0), (256, 0), (33, 0), (20, 5)):
        p = jev.jev_prefix_suffix_attn_plan(jev.make_attn_desc(2, Lp, 8, 2, 128, 10, jev.JEV_F32, num_splits=ns), 0)
        L, S = p["split_len"], p["simt_splits"]
        assert p["kernel"] == 0 and L % 32 == 0 and S >= 1
        assert S * L >= Lp and (S - 1) * L < Lp  # every split holds keys
    # a small problem gets several splits (two 32-key tiles each at least)
    p = jev.jev_prefix_suffix_attn_plan(jev.make_attn_desc(4, 256, 2, 1, 64, 64, jev.JEV_F32), 0)
    assert p["simt_splits"] == 4 and p["split_len"] == 64


def test_tree_schedule_study_inputs():
    """The tree schedule study's synthetic candidate sets (bench.py diag_tree_schedule) have the
    properties the study is about: 75% of each two-level candidate's tokens lie in its question,
    the two-level and flat tries pack the same number of unique tokens, and the multi-image
    tree has one first-level node per image with an empty root."""
    import synth
    import oracle
    BF = synth.CONFIGS["qwen25vl_7b"]
    two = synth.tree_case(synth.TreeConfig("two_level", synth.BF16, BF.Lp, 16, 24, 4, 4, 8, 8, BF.Hq, BF.Hkv,
                                           BF.d, BF.H, BF.V, seed=31), with_lm_head=False)
    flat = synth.tree_case(synth.TreeConfig("flat_trie", synth.BF16, BF.Lp, 64, 13, 1, 1, 1, 1, BF.Hq, BF.Hkv,
                                            BF.d, BF.H, BF.V, seed=32), with_lm_head=False)
    mi = synth.tree_case(synth.TreeConfig("multi_image", synth.BF16, 0, 8, 416, 3, 3, 1, 1, BF.Hq, BF.Hkv,
                                          BF.d, BF.H, BF.V, seed=33), with_lm_head=False)
    t2 = oracle.trie_build(two.seq_off, two.toks, BF.Lp)
    tf = oracle.trie_build(flat.seq_off, flat.toks, BF.Lp)
    tm = oracle.trie_build(mi.seq_off, mi.toks, 0)
    lens = np.diff(two.seq_off)
    assert two.seq_off.size - 1 == 64 and np.all(lens == 32) and np.all(two.score_from == 24)  # 24 of 32 shared
    assert int(t2["tok_off"][-1]) == int(tf["tok_off"][-1]) == 896
    assert int(two.seq_off[-1]) == 2048 and int(flat.seq_off[-1]) == 896
    assert t2["n_nodes"] == 1 + 16 + 64 and np.all(tf["parent"][1:] == 0) and tf["n_nodes"] == 65
    first = np.nonzero(tm["parent"] == 0)[0]
    assert first.size == 8 and np.all(tm["pos0"][first] == 0)
    assert np.all(np.diff(tm["tok_off"])[first] == 416) and int(tm["tok_off"][-1]) == 3352


@pytest.mark.parametrize("V", [1, 15, 16, 17, 255, 257, 5000, 59200, 151936, 152064])
@pytest.mark.parametrize("R", [1, 128, 129, 256, 300, 1024])
def test_vocab_lse_partition_and_workspace(R, V):
    """The full-vocabulary LSE kernel's work split, as its CTAs derive it: CTA c of n owns
    vocabulary rows [c*n16/n*16, min(V, (c+1)*n16/n*16)) (n16 = 16-row granules), walked in
    256-row tiles whose MMA width is the tile's rows rounded up to 16.  Every row is owned once,
    every MMA width is a legal N (16..256, step 16), and every (max, sum) partial the CTAs write,
    [row block][CTA][column half][256 rows], fits the workspace the library asks for after its
    256-byte status word."""
    # the SM count the library plans for (the device's, or 148 without one): a problem with
    # many whole-tile waves gets one persistent CTA per SM
    big = jev.make_attn_desc(1024, 4096, 28, 4, 128, 24000, jev.JEV_BF16)
    sms = jev.jev_prefix_suffix_attn_plan(big, 1, 0)["n_ctas"]
    n16 = -(-V // 16)
    n = max(1, min(n16, sms))
    owned = np.zeros(V, np.int32)
    for c in range(n):
        lo = c * n16 // n * 16
        hi = min(V, (c + 1) * n16 // n * 16)
        assert hi > lo
        owned[lo:hi] += 1
        for v0 in range(lo, hi, 256):
            width = -(-min(256, hi - v0) // 16) * 16
            assert 16 <= width <= 256 and width % 16 == 0
    assert np.all(owned == 1)
    n_mb = -(-R // 256)
    last = (((n_mb - 1) * n + (n - 1)) * 2 + 1) * 256 + 255  # largest partial index
    assert 256 + (last + 1) * 8 <= jev.jev_vocab_lse_workspace(R, V)
