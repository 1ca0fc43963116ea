"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs, element by element.

* tiny_f32 and qwen2vl_2b are compared on every output element (the qwen2vl_2b readout against the
  oracle's full-vocabulary logits, the pages' plain definition).
* qwen25vl_7b and wide_7b run at full size in the launch configuration bench.py times
  (automatic split count, default kernel) and are compared on sampled rows the
  oracle forms one by one: every branch's first and last token at every head
  plus random rows; the readout is compared on every set.
* Small cases cover the edges: ragged prefix tails, Lp = 0, empty and
  one-token branches, a suffix longer than a key tile, MHA (G = 1), G = 7,
  d = 64 and 128, explicit head maps, forced split counts, a position offset.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, check_attn, check_readout, compact_lm_head, dev, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def jev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import attention_cascade_b200 as m
    return m


def run_flat(jev, c, **kw):
    q, kp, vp, ks, vs = (dev(x) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf))
    cu = dev(c.cu_seqlens)
    ws_kw = {}
    if "head_map" in kw and kw["head_map"] is not None:
        kw["head_map"] = dev(np.asarray(kw["head_map"], np.int32))
    out, lse = jev.jev_prefix_suffix_attn(q, kp, vp, ks, vs, cu, **kw, **ws_kw)
    torch.cuda.synchronize()
    return host_f64(out), host_f64(lse)


def run_readout(jev, hidden, W_dev, so, toks, **kw):
    extra = {k: (dev(np.asarray(v, np.int32)) if v is not None else None) for k, v in kw.items()}
    lp, ch = jev.jev_candidate_readout(dev(hidden), W_dev, dev(so), dev(toks.astype(np.int32)), **extra)
    torch.cuda.synchronize()
    return lp.cpu().numpy().astype(np.float64), ch.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny_f32", "qwen2vl_2b"])
def test_flat_config_every_element(jev, name):
    cfg = synth.CONFIGS[name]
    c = synth.flat_case(cfg)
    out, lse = run_flat(jev, c, rope_theta=cfg.theta)
    ref_o, ref_l = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens, theta=cfg.theta)
    check_attn(out, lse, ref_o, ref_l, cfg.dtype, name)
    ref = oracle.candidate_readout(c.hidden, c.W, c.set_offsets, c.pair_tok, full_vocab=True)
    lp, ch = run_readout(jev, c.hidden, dev(c.W), c.set_offsets, c.pair_tok)
    check_readout(lp, ch, ref, cfg.dtype, name)


def _sample_rows(c, n_random, seed):
    rng = np.random.default_rng(seed)
    cu = c.cu_seqlens
    Hq = c.cfg.Hq
    toks = []
    for b in range(cu.size - 1):
        if cu[b + 1] > cu[b]:
            toks += [cu[b], cu[b + 1] - 1]
    rows = [(t, h) for t in sorted(set(toks)) for h in range(Hq)]
    rows += [(int(rng.integers(0, c.T)), int(rng.integers(0, Hq))) for _ in range(n_random)]
    return np.array(rows, np.int32)


@pytest.mark.parametrize("name", ["qwen25vl_7b", "wide_7b"])
def test_flat_config_full_size_sampled(jev, name):
    cfg = synth.CONFIGS[name]
    c = synth.flat_case(cfg, with_lm_head=False)
    out, lse = run_flat(jev, c, rope_theta=cfg.theta)
    rows = _sample_rows(c, 300, seed=7)
    ref_o, ref_l = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens,
                                             theta=cfg.theta, rows=rows)
    check_attn(out[rows[:, 0], rows[:, 1]], lse[rows[:, 0], rows[:, 1]], ref_o, ref_l, cfg.dtype, name)
    Wd, Wrows, inv = compact_lm_head(cfg, c.pair_tok)
    ref = oracle.candidate_readout(c.hidden, Wrows, c.set_offsets, inv, full_vocab=False)
    lp, ch = run_readout(jev, c.hidden, Wd, c.set_offsets, c.pair_tok)
    check_readout(lp, ch, ref, cfg.dtype, name)


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
def test_many_tokens_at_d64_sampled(jev, dtype):
    """About 9000 suffix tokens at d = 64: the RoPE pack's grid is deep enough
    for its sixteen-heads-a-warp form (more than 8192 warps at eight), which
    the other shapes reach only in bf16 at d = 128.  Sampled rows (first and
    last token of every branch plus random ones) against the oracle."""
    cfg = synth.FlatConfig("many_d64", dtype, 64, 600, 8, 22, 8, 2, 64, 64, 256, 2, 2, seed=31)
    c = synth.flat_case(cfg, with_lm_head=False)
    assert c.T > 8192
    out, lse = run_flat(jev, c)
    rows = _sample_rows(c, 300, seed=8)
    ref_o, ref_l = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens, rows=rows)
    check_attn(out[rows[:, 0], rows[:, 1]], lse[rows[:, 0], rows[:, 1]], ref_o, ref_l, dtype, "many tokens d64")


def _scale_rows(a, lo, hi, f, dtype):
    """a[lo:hi] *= f, on the host arrays both sides read (bf16 as its bits)."""
    a = a.copy()
    if dtype == synth.BF16:
        a[lo:hi] = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(a[lo:hi]) * np.float32(f))
    else:
        a[lo:hi] *= np.float32(f)
    return a


@pytest.mark.parametrize("rows", [0, 256])
@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
@pytest.mark.parametrize("splits", [0, 1])
def test_running_max_jumps_between_key_tiles(jev, dtype, splits, rows, force_tile_rows):
    """Scores that grow from key tile to key tile: prefix keys 128..383 scaled
    by 3, keys from 384 on and every suffix key by 6, so that in about half of
    the rows the maximum jumps past the softmax's lazy threshold (8 in log2
    units) at a tile boundary, some rows twice.  The running max must move and
    O be rescaled, and tiles whose scores fall back must not move it.  Every
    element against the oracle, split and unsplit.  The bf16 path stores the
    rotated queries and keys in bf16, and a score's rounding error grows with
    the size of its key: with keys up to 6 times those of the N(0, 1) cases
    the bf16 tolerances here are 4 times theirs (a rescale that went wrong
    would be off by a factor of 2^8 or more)."""
    force_tile_rows(rows)
    cfg = synth.FlatConfig("jump", dtype, 520, 5, 1, 1, 8, 2, 128, 16, 32, 2, 3, seed=41)
    c = synth.flat_case(cfg, with_lm_head=False, lengths=np.array([3, 40, 1, 150, 9], np.int32))
    c.k_pre = _scale_rows(_scale_rows(c.k_pre, 128, 384, 3.0, dtype), 384, 520, 6.0, dtype)
    c.k_suf = _scale_rows(c.k_suf, 0, c.T, 6.0, dtype)
    out, lse = run_flat(jev, c, num_splits=splits)
    ref_o, ref_l = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens)
    assert ref_l.max() > 10.0  # the later tiles dominate: far above the first tile's scores
    tol = TOL[dtype] if dtype == synth.F32 else {k: 4 * v for k, v in TOL[dtype].items()}
    err = np.abs(out - ref_o)
    assert np.all(np.isfinite(out))
    assert err.max() <= tol["max_abs"] and err.mean() <= tol["mean_abs"], (err.max(), err.mean())
    assert np.abs(lse - ref_l).max() <= tol["lse"], np.abs(lse - ref_l).max()


EDGE = [
    # dtype, Lp, lens, Hq, Hkv, d, splits, pos_offset, head_map
    (synth.BF16, 300, [1, 7, 0, 33, 130], 8, 2, 128, 0, -1, None),
    (synth.BF16, 0, [5, 17], 4, 4, 64, 0, -1, None),
    (synth.BF16, 1000, [200], 14, 2, 128, 3, -1, None),
    (synth.F32, 129, [3, 1, 2], 6, 3, 64, 0, 500, None),
    (synth.BF16, 256, [9, 4, 12], 8, 2, 128, 2, -1, [1, 0, 0, 1, 1, 0, 1, 0]),
    (synth.BF16, 2048, [40] * 12, 28, 4, 128, 1, -1, None),
    (synth.BF16, 2048, [40] * 12, 28, 4, 128, 5, -1, None),
    (synth.BF16, 384, [1] * 37, 12, 2, 64, 0, -1, None),
    (synth.F32, 200, [70, 1, 15], 4, 2, 128, 2, -1, None),
    # more branches than the RoPE pack's shared-memory offset table (4096): offsets searched in global memory
    (synth.BF16, 512, [1, 2] * 2100, 8, 2, 64, 0, 700, None),
]


@pytest.mark.parametrize("rows", [0, 256])
@pytest.mark.parametrize("case", EDGE, ids=[f"e{i}" for i in range(len(EDGE))])
def test_flat_edge_shapes(jev, case, rows, force_tile_rows):
    # rows 0: the plan's choice (128-row tiles, the one-Q-tile kernel, at these
    # sizes); 256: the two-Q-tile kernel on the same shapes
    force_tile_rows(rows)
    dtype, Lp, lens, Hq, Hkv, d, splits, pos_off, hm = case
    cfg = synth.FlatConfig("edge", dtype, Lp, len(lens), 1, 1, Hq, Hkv, d, 16, 32, 2, 3, seed=sum(lens) + Lp)
    c = synth.flat_case(cfg, with_lm_head=False, lengths=np.array(lens, np.int32))
    out, lse = run_flat(jev, c, num_splits=splits, pos_offset=pos_off, head_map=hm)
    ref_o, ref_l = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens,
                                             pos_offset=pos_off, head_map=hm)
    check_attn(out, lse, ref_o, ref_l, dtype, str(case[:3]))


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
def test_readout_multi_token_invalid_and_empty(jev, dtype):
    rng = np.random.default_rng(3)
    R, H, V = 9, 256, 3000
    hidden = rng.standard_normal((R, H)).astype(np.float32)
    W = (0.05 * rng.standard_normal((V, H))).astype(np.float32)
    if dtype == synth.BF16:
        hidden, W = synth.f32_to_bf16_bits(hidden), synth.f32_to_bf16_bits(W)
    # 5 sets: multi-token candidates, an empty set, a set with an invalid token, a 40-candidate set
    so = np.array([0, 3, 3, 5, 6, 46], np.int32)
    npair = np.array([1, 2, 4, 1, 3, 1] + [1] * 40)
    co = np.concatenate([[0], np.cumsum(npair)]).astype(np.int32)
    P = int(co[-1])
    prow = rng.integers(0, R, P).astype(np.int32)
    ptok = rng.integers(0, V, P).astype(np.int32)
    ptok[co[4]] = V + 5  # candidate 4 (set 2) invalid
    ref = oracle.candidate_readout(hidden, W, so, ptok, cand_offsets=co, pair_row=prow)
    lp, ch = run_readout(jev, hidden, dev(W), so, ptok, cand_offsets=co, pair_row=prow)
    check_readout(lp, ch, ref, dtype, "multi")
    assert ch[1] == -1 and ch[2] == -1 and np.all(np.isnan(lp[3:5]))


@pytest.mark.parametrize("H", [256, 1544, 4096, 4104])
def test_readout_many_one_pair_candidates(jev, H):
    # 2000 sets of one-token options (mostly 9; set 3 has 1, set 5 has 40): at H <= 4096 one warp
    # per set takes the scores and the set softmax (H = 1544 leaves a ragged last vector per lane
    # group); at H = 4104 a warp per candidate, then the set kernel.  An invalid token in set 7,
    # an empty set 11.
    rng = np.random.default_rng(5)
    n_sets, opts, V = 2000, 9, 4096
    hidden = synth.f32_to_bf16_bits(rng.standard_normal((n_sets, H)).astype(np.float32))
    W = synth.f32_to_bf16_bits((0.05 * rng.standard_normal((V, H))).astype(np.float32))
    sizes = np.full(n_sets, opts)
    sizes[3], sizes[5], sizes[11] = 1, 40, 0
    so = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    toks = rng.integers(0, V, int(so[-1])).astype(np.int32)
    toks[so[7] + 2] = -3
    ref = oracle.candidate_readout(hidden, W, so, toks)
    n0 = jev.jev_launch_count()
    lp, ch = run_readout(jev, hidden, dev(W), so, toks)
    assert jev.jev_launch_count() - n0 == (1 if H <= 4096 else 2)  # fused, or scores then set softmax
    check_readout(lp, ch, ref, synth.BF16, f"one-pair readout H={H}")
    assert ch[7] == -1 and ch[11] == -1 and np.all(np.isnan(lp[so[7]:so[8]]))
    assert ch[3] == 0 and lp[so[3]] == 0.0


def test_readout_tie_goes_to_first(jev):
    hidden = np.ones((2, 8), np.float32)
    W = np.zeros((4, 8), np.float32)
    W[1] = W[3] = 0.5
    lp, ch = run_readout(jev, hidden, dev(W), np.array([0, 2, 4], np.int32), np.array([1, 3, 3, 1], np.int32))
    assert ch.tolist() == [0, 0]
    np.testing.assert_allclose(lp, np.log(0.5), atol=1e-6)


def _tree_inputs(tc, jev):
    t = jev.jev_tree_build(tc.seq_off, tc.toks, tc.cfg.Lp)
    return t, dict(parent=dev(t["parent"]), tok_off=dev(t["tok_off"]), pos0=dev(t["pos0"]))


@pytest.mark.parametrize("rows", [0, 256])
@pytest.mark.parametrize("seed,d,dtype", [(0, 64, synth.BF16), (1, 128, synth.BF16), (2, 64, synth.F32)])
def test_tree_small_every_element(jev, seed, d, dtype, rows, force_tile_rows):
    force_tile_rows(rows)
    cfg = synth.TreeConfig("t", dtype, 300, 5, 9, 2, 6, 1, 5, 8, 2, d, 64, 500, seed=seed)
    tc = synth.tree_case(cfg, with_lm_head=True)
    t, td = _tree_inputs(tc, jev)
    out, lse = jev.jev_tree_attn(td["parent"], td["tok_off"], td["pos0"], dev(tc.q), dev(tc.k_root), dev(tc.v_root),
                                 dev(tc.k), dev(tc.v))
    ref_o, ref_l = oracle.tree_attn(oracle.trie_build(tc.seq_off, tc.toks, cfg.Lp), tc.q, tc.k, tc.v,
                                    tc.k_root, tc.v_root)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, cfg.dtype, "tree")
    plan = jev.jev_tree_readout_plan(tc.seq_off, tc.toks, tc.score_from, t["path_row"])
    ref = oracle.candidate_readout(tc.hidden, tc.W, tc.set_offsets, plan["pair_tok"],
                                   cand_offsets=plan["cand_offsets"], pair_row=plan["pair_row"])
    lp, ch = run_readout(jev, tc.hidden, dev(tc.W), tc.set_offsets, plan["pair_tok"],
                         cand_offsets=plan["cand_offsets"], pair_row=plan["pair_row"])
    check_readout(lp, ch, ref, cfg.dtype, "tree readout")


@pytest.mark.parametrize("rows", [0, 256])
@pytest.mark.parametrize("shape", ["chain", "zigzag"])
def test_deep_token_tries_every_element(jev, shape, rows, force_tile_rows):
    force_tile_rows(rows)
    """Tries 12 levels deep and more: a chain of one-token nodes each ending a
    candidate, and a zigzag whose path always continues through the second
    child, so a token's ancestors' keys are not one contiguous range."""
    if shape == "chain":
        cands = [list(range(1, k + 1)) for k in range(1, 15)]
    else:
        cands = [[100 + i for i in range(k)] + [200 + k] for k in range(13)] + [[100 + i for i in range(13)]]
    so = np.concatenate([[0], np.cumsum([len(x) for x in cands])]).astype(np.int32)
    toks = np.array([t for x in cands for t in x], np.int32)
    Lp, Hq, Hkv, d = 130, 8, 2, 64
    t = jev.jev_tree_build(so, toks, Lp)
    depth = np.zeros(t["n_nodes"], np.int32)
    for n in range(1, t["n_nodes"]):
        depth[n] = depth[t["parent"][n]] + 1
    assert depth.max() >= 12
    N = int(t["tok_off"][-1])
    rng = np.random.default_rng(4)
    mk = lambda *s: synth.f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32))
    q, k, v, kr, vr = mk(N, Hq, d), mk(N, Hkv, d), mk(N, Hkv, d), mk(Lp, Hkv, d), mk(Lp, Hkv, d)
    desc = jev.make_attn_desc(t["n_nodes"] - 1, Lp, Hq, Hkv, d, N, jev.JEV_BF16)
    ws = jev.new_workspace(jev.jev_tree_attn_workspace(desc, t["n_nodes"]), "cuda")
    out, lse = jev.jev_tree_attn(dev(t["parent"]), dev(t["tok_off"]), dev(t["pos0"]), dev(q), dev(kr), dev(vr),
                                 dev(k), dev(v), workspace=ws)
    assert jev.jev_check_device_status(ws) == 0
    ref_o, ref_l = oracle.tree_attn(oracle.trie_build(so, toks, Lp), q, k, v, kr, vr)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, synth.BF16, f"deep tree ({shape})")


def test_tree_more_nodes_than_the_shared_table(jev):
    # more nodes than the RoPE pack's shared-memory offset table (4096): node offsets searched in global memory
    cfg = synth.TreeConfig("tn", synth.BF16, 96, 560, 3, 5, 8, 1, 2, 4, 2, 64, 64, 5000, seed=11)
    tc = synth.tree_case(cfg, with_lm_head=False)
    t, td = _tree_inputs(tc, jev)
    assert t["n_nodes"] > 4096
    out, lse = jev.jev_tree_attn(td["parent"], td["tok_off"], td["pos0"], dev(tc.q), dev(tc.k_root), dev(tc.v_root),
                                 dev(tc.k), dev(tc.v))
    ref_o, ref_l = oracle.tree_attn(oracle.trie_build(tc.seq_off, tc.toks, cfg.Lp), tc.q, tc.k, tc.v,
                                    tc.k_root, tc.v_root)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, cfg.dtype, "tree, many nodes")


def test_multi_image_tree(jev):
    # one question over four images (Ochevid, "One question, multiple images"): an empty root, one
    # first-level node per image + question (300 tokens, positions 0..299), three one- or two-token
    # options under each.  Every image row is its own causal problem: against the oracle on every
    # element, and the first image run alone matches the same oracle rows.
    cfg = synth.TreeConfig("mi", synth.BF16, 0, 4, 300, 3, 3, 1, 2, 8, 2, 128, 64, 500, seed=21)
    tc = synth.tree_case(cfg, with_lm_head=False)
    t, td = _tree_inputs(tc, jev)
    assert t["n_nodes"] == 1 + 4 + 12 and np.all(t["pos0"][t["parent"] == 0][1:] == 0)
    out, lse = jev.jev_tree_attn(td["parent"], td["tok_off"], td["pos0"], dev(tc.q), dev(tc.k_root), dev(tc.v_root),
                                 dev(tc.k), dev(tc.v))
    ref_o, ref_l = oracle.tree_attn(oracle.trie_build(tc.seq_off, tc.toks, 0), tc.q, tc.k, tc.v, tc.k_root, tc.v_root)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, cfg.dtype, "multi-image tree")
    # the first image alone: its candidates are the first set
    c1 = int(tc.set_offsets[1])
    so1 = tc.seq_off[:c1 + 1]
    t1 = jev.jev_tree_build(so1, tc.toks[:so1[-1]], 0)
    n1 = int(t1["tok_off"][-1])
    o1, l1 = jev.jev_tree_attn(dev(t1["parent"]), dev(t1["tok_off"]), dev(t1["pos0"]), dev(tc.q[:n1]),
                               dev(tc.k_root), dev(tc.v_root), dev(tc.k[:n1]), dev(tc.v[:n1]))
    check_attn(host_f64(o1), host_f64(l1), ref_o[:n1], ref_l[:n1], cfg.dtype, "first image alone")


@pytest.mark.parametrize("rows", [128, 256])
def test_single_key_tile_segments_keep_the_pipeline_in_step(jev, rows, force_tile_rows):
    # Schedules whose CTAs run a segment of one key tile followed by more segments: 64 branches
    # of 32 tokens over a 2048-token prefix at the 7B heads (a one-unit tail segment), and a
    # multi-image tree (empty root, 8 nodes of 416 tokens: many one-tile windows).  The MMA warp
    # may release the Q buffer for the next segment only after every softmax thread has passed
    # this segment's q_full wait; otherwise a softmax thread still in the previous epilogue waits
    # on an aliased phase.  Five back-to-back calls on one workspace must leave the status word
    # clear, and sampled rows match the oracle.
    import dataclasses
    force_tile_rows(rows)
    cfg = dataclasses.replace(synth.CONFIGS["qwen25vl_7b"], B=64)
    c = synth.flat_case(cfg, with_lm_head=False, lengths=np.full(64, 32, np.int32))
    desc = jev.make_attn_desc(64, cfg.Lp, cfg.Hq, cfg.Hkv, cfg.d, c.T, jev.JEV_BF16, cfg.theta)
    plan = jev.jev_prefix_suffix_attn_plan(desc, 1, 148)
    assert plan["full_waves"] >= 1 and plan["tail_ctas"] < plan["n_ctas"]
    ws = jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(desc), "cuda")
    q, kp, vp, ks, vs = (dev(x) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf))
    cu = dev(c.cu_seqlens)
    for _ in range(5):
        out, lse = jev.jev_prefix_suffix_attn(q, kp, vp, ks, vs, cu, workspace=ws, rope_theta=cfg.theta)
    assert jev.jev_check_device_status(ws) == 0
    rows = _sample_rows(c, 256, 17)
    ref_o, ref_l = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens, rows=rows)
    o, l = host_f64(out), host_f64(lse)
    check_attn(o[rows[:, 0], rows[:, 1]], l[rows[:, 0], rows[:, 1]], ref_o, ref_l, cfg.dtype, "64 x 32 branches")

    BF = synth.CONFIGS["qwen25vl_7b"]
    mi = synth.TreeConfig("mi8", synth.BF16, 0, 8, 416, 3, 3, 1, 1, BF.Hq, BF.Hkv, BF.d, 64, 500, seed=33)
    tc = synth.tree_case(mi, with_lm_head=False)
    t, td = _tree_inputs(tc, jev)
    N = int(t["tok_off"][-1])
    tdesc = jev.make_attn_desc(t["n_nodes"] - 1, 0, BF.Hq, BF.Hkv, BF.d, N, jev.JEV_BF16, 1e4)
    tws = jev.new_workspace(jev.jev_tree_attn_workspace(tdesc, t["n_nodes"]), "cuda")
    tq, tkr, tvr, tk, tv = (dev(x) for x in (tc.q, tc.k_root, tc.v_root, tc.k, tc.v))
    for _ in range(5):
        out, lse = jev.jev_tree_attn(td["parent"], td["tok_off"], td["pos0"], tq, tkr, tvr, tk, tv, workspace=tws)
    assert jev.jev_check_device_status(tws) == 0
    ref_o, ref_l = oracle.tree_attn(oracle.trie_build(tc.seq_off, tc.toks, 0), tc.q, tc.k, tc.v, tc.k_root, tc.v_root)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, mi.dtype, "8-image tree")


def test_tree_config_tree_7b(jev):
    cfg = synth.CONFIGS["tree_7b"]
    tc = synth.tree_case(cfg, with_lm_head=False)
    t, td = _tree_inputs(tc, jev)
    out, lse = jev.jev_tree_attn(td["parent"], td["tok_off"], td["pos0"], dev(tc.q), dev(tc.k_root), dev(tc.v_root),
                                 dev(tc.k), dev(tc.v))
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.tree_attn(oracle.trie_build(tc.seq_off, tc.toks, cfg.Lp), tc.q, tc.k, tc.v,
                                    tc.k_root, tc.v_root)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, cfg.dtype, "tree_7b")
    plan = jev.jev_tree_readout_plan(tc.seq_off, tc.toks, tc.score_from, t["path_row"])
    Wd, Wrows, inv = compact_lm_head(cfg, plan["pair_tok"])
    ref = oracle.candidate_readout(tc.hidden, Wrows, tc.set_offsets, inv, cand_offsets=plan["cand_offsets"],
                                   pair_row=plan["pair_row"], full_vocab=False)
    lp, ch = run_readout(jev, tc.hidden, Wd, tc.set_offsets, plan["pair_tok"], cand_offsets=plan["cand_offsets"],
                         pair_row=plan["pair_row"])
    check_readout(lp, ch, ref, cfg.dtype, "tree_7b readout")


@pytest.mark.parametrize("lens,S,d,dtype", [([50, 1, 130, 77, 200], 128, 128, synth.BF16),
                                             ([256] * 16, 256, 128, synth.BF16), ([33, 0, 70], 64, 64, synth.BF16),
                                             ([20, 7, 41], 48, 64, synth.F32)])
def test_sink_block_parallel_encoding(jev, lens, S, d, dtype):
    """Blocks over a shared sink at their unsplit positions (PEVLM; the flat
    kernels with sequential positions), every element against the per-block oracle."""
    rng = np.random.default_rng(sum(lens) + S)
    Hq, Hkv = 8, 2
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    mk = lambda *sh: (synth.f32_to_bf16_bits(rng.standard_normal(sh).astype(np.float32)) if dtype == synth.BF16
                      else rng.standard_normal(sh).astype(np.float32))
    q, k, v, k_sink, v_sink = mk(T, Hq, d), mk(T, Hkv, d), mk(T, Hkv, d), mk(S, Hkv, d), mk(S, Hkv, d)
    out, lse = jev.jev_sink_block_attn(dev(q), dev(k_sink), dev(v_sink), dev(k), dev(v), dev(cu))
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.sink_block_attn(q, k, v, k_sink, v_sink, cu)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, dtype, f"sink-block {lens[:3]}")
