"""Pins for the fp64 oracle: each test checks it against something other than
itself — hand-derived closed forms (tests/golden), PyTorch's fp64
scaled-dot-product attention and numpy matrix products on the special cases
that reduce to them, invariants the pages state, and a brute-force trie.

Every function of ``oracle`` has at least one pin that a dropped term, a wrong
sign, a wrong index or a transposed operand would fail.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _rope_complex(x, pos, theta):
    """RoPE through complex multiplication (independent of oracle.rope):
    (x_i + i x_{i+d/2}) * exp(i * pos * theta^(-2i/d))."""
    x = np.asarray(x, np.float64)
    d = x.shape[-1]
    h = d // 2
    inv = theta ** (-2.0 * np.arange(h) / d)
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * np.multiply.outer(np.asarray(pos, np.float64), inv))
    return np.concatenate([z.real, z.imag], axis=-1)


def _f64(a):
    return synth.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _sdpa_branch(q_raw, k_raw, v, pos, Hkv, head_map, theta, scale):
    """Causal attention over a full sequence with torch's fp64 SDPA (library
    routine); q_raw [L, Hq, d], k_raw/v [L, Hkv, d] with k already rotated
    where pos is None for those rows.  Returns out [L, Hq, d] and lse [L, Hq]."""
    L, Hq, d = q_raw.shape
    qh = torch.from_numpy(q_raw).permute(1, 0, 2)          # [Hq, L, d]
    kh = torch.from_numpy(k_raw).permute(1, 0, 2)[head_map]  # [Hq, L, d]
    vh = torch.from_numpy(v).permute(1, 0, 2)[head_map]
    out = torch.nn.functional.scaled_dot_product_attention(qh[None], kh[None], vh[None], is_causal=True,
                                                           scale=scale)[0]
    s = (qh @ kh.transpose(1, 2)) * scale
    s = s.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf"))
    lse = torch.logsumexp(s, dim=-1)
    return out.permute(1, 0, 2).numpy(), lse.permute(1, 0).numpy()


# --------------------------------------------------------------------------- RoPE


def test_rope_hand_values():
    g = _gold("rope_d4.json")
    for c in g["cases"]:
        y = oracle.rope(np.array(c["x"], np.float64), c["pos"], g["theta"])
        np.testing.assert_allclose(y, c["y"], atol=g["tolerance"])


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(11)
    for d in (2, 8, 64, 128):
        for pos in (0, 1, 7, 1023, 4135):
            x = rng.standard_normal(d)
            np.testing.assert_allclose(oracle.rope(x, pos, 1e4), _rope_complex(x, pos, 1e4), atol=1e-11)


# --------------------------------------------------------------------------- attention


def test_hand_two_token_case():
    g = _gold("hand_2token.json")
    i = g["inputs"]
    arr = lambda v: np.array(v, np.float32).reshape(1, 1, 2)
    out, lse = oracle.prefix_suffix_attn(arr(i["q"]), arr(i["k_pre"]), arr(i["v_pre"]), arr(i["k_suf"]),
                                         arr(i["v_suf"]), np.array([0, 1]), theta=i["theta"])
    e = g["expected"]
    np.testing.assert_allclose(out[0, 0], e["out"], atol=g["tolerance"])
    assert abs(lse[0, 0] - e["lse"]) < g["tolerance"]
    # the same numbers by the two-key logistic closed form
    s0, s1 = math.cos(1.0) / math.sqrt(2.0), 1.0 / math.sqrt(2.0)
    p1 = 1.0 / (1.0 + math.exp(s0 - s1))
    assert abs(out[0, 0, 1] - p1) < 1e-12 and abs(out[0, 0, 0] - (1 - p1)) < 1e-12
    assert abs(lse[0, 0] - (s1 + math.log1p(math.exp(s0 - s1)))) < 1e-12


def test_sink_block_matches_sdpa_per_block():
    """Sink-block parallel encoding ("PEVLM", abstract): block b's rows equal
    the last rows of causal fp64 SDPA over [sink; block b] with the block's
    tokens at their positions in the unsplit sequence, S + cu[b] + j."""
    theta, S, Hq, Hkv, d = 1e4, 7, 4, 2, 16
    rng = np.random.default_rng(17)
    lens = np.array([3, 1, 6, 4], np.int32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    k_sink_raw = rng.standard_normal((S, Hkv, d))
    k_sink = _rope_complex(k_sink_raw.transpose(1, 0, 2), np.arange(S), theta).transpose(1, 0, 2).astype(np.float32)
    v_sink, q, k, v = (rng.standard_normal(s).astype(np.float32)
                       for s in ((S, Hkv, d), (T, Hq, d), (T, Hkv, d), (T, Hkv, d)))
    out, lse = oracle.sink_block_attn(q, k, v, k_sink, v_sink, cu, theta=theta)
    scale = 1.0 / math.sqrt(d)
    hm = torch.from_numpy(np.arange(Hq) // (Hq // Hkv)).long()
    for b in range(lens.size):
        a, e = cu[b], cu[b + 1]
        pos = S + a + np.arange(e - a)
        q_b = _rope_complex(_f64(q)[a:e].transpose(1, 0, 2), pos, theta).transpose(1, 0, 2)
        k_b = _rope_complex(_f64(k)[a:e].transpose(1, 0, 2), pos, theta).transpose(1, 0, 2)
        o_ref, l_ref = _sdpa_branch(np.concatenate([np.zeros((S, Hq, d)), q_b]),
                                    np.concatenate([_f64(k_sink), k_b]),
                                    np.concatenate([_f64(v_sink), _f64(v)[a:e]]), None, Hkv, hm, theta, scale)
        np.testing.assert_allclose(out[a:e], o_ref[S:], atol=1e-12)
        np.testing.assert_allclose(lse[a:e], l_ref[S:], atol=1e-12)


def test_sink_block_first_block_is_full_attention():
    """The first block sees exactly what full causal attention over the unsplit
    sequence gives it (the pages' alignment with Full-Attention is exact there);
    later blocks, which no longer see earlier blocks, differ."""
    rng = np.random.default_rng(23)
    S, Hq, Hkv, d = 5, 2, 1, 8
    lens = np.array([4, 3], np.int32)
    cu = np.array([0, 4, 7], np.int32)
    f32 = lambda *sh: rng.standard_normal(sh).astype(np.float32)
    k_sink, v_sink = f32(S, Hkv, d), f32(S, Hkv, d)
    q, k, v = f32(7, Hq, d), f32(7, Hkv, d), f32(7, Hkv, d)
    out, lse = oracle.sink_block_attn(q, k, v, k_sink, v_sink, cu)
    full_o, full_l = oracle.prefix_suffix_attn(q, k_sink, v_sink, k, v, np.array([0, 7], np.int32), pos_offset=S)
    np.testing.assert_allclose(out[:4], full_o[:4], atol=1e-13)
    np.testing.assert_allclose(lse[:4], full_l[:4], atol=1e-13)
    assert np.abs(out[4:] - full_o[4:]).max() > 1e-3


def _small_case(B=3, Lp=9, lens=(1, 4, 6), Hq=4, Hkv=2, d=8, seed=5, dtype=synth.F32):
    cfg = synth.FlatConfig("t", dtype, Lp, B, 1, 1, Hq, Hkv, d, 16, 32, 2, 3, seed=seed)
    return synth.flat_case(cfg, with_lm_head=False, lengths=np.array(lens, np.int32))


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
@pytest.mark.parametrize("head_map", [None, "perm"])
def test_matches_sdpa_per_branch(dtype, head_map):
    """Each branch's rows equal the last Ls rows of causal fp64 SDPA over the
    whole sequence [prefix; suffix] (prefix keys rotated at 0..Lp-1)."""
    theta, Lp, Hq, Hkv, d = 1e4, 9, 6, 2, 16
    rng = np.random.default_rng(3)
    lens = np.array([1, 5, 3, 7], np.int32)
    B = lens.size
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    k_pre_raw = rng.standard_normal((Lp, Hkv, d)).astype(np.float32)
    k_pre = _rope_complex(k_pre_raw.astype(np.float64).transpose(1, 0, 2), np.arange(Lp), theta).transpose(1, 0, 2)
    k_pre = k_pre.astype(np.float32)
    if dtype == synth.BF16:
        k_pre = synth.f32_to_bf16_bits(k_pre)
    mk = lambda *s: (synth.f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32)) if dtype == synth.BF16
                     else rng.standard_normal(s).astype(np.float32))
    v_pre, q, k_suf, v_suf = mk(Lp, Hkv, d), mk(T, Hq, d), mk(T, Hkv, d), mk(T, Hkv, d)
    hm = None if head_map is None else np.array([1, 0, 1, 0, 0, 1], np.int32)
    hm_eff = hm if hm is not None else np.arange(Hq) // (Hq // Hkv)
    out, lse = oracle.prefix_suffix_attn(q, k_pre, v_pre, k_suf, v_suf, cu, theta=theta, head_map=hm)
    scale = 1.0 / math.sqrt(d)
    for b in range(B):
        a, e = cu[b], cu[b + 1]
        Ls = e - a
        pos = Lp + np.arange(Ls)
        q_b = _rope_complex(_f64(q)[a:e].transpose(1, 0, 2), pos, theta).transpose(1, 0, 2)
        k_b = _rope_complex(_f64(k_suf)[a:e].transpose(1, 0, 2), pos, theta).transpose(1, 0, 2)
        qfull = np.concatenate([np.zeros((Lp, Hq, d)), q_b])
        kfull = np.concatenate([_f64(k_pre), k_b])
        vfull = np.concatenate([_f64(v_pre), _f64(v_suf)[a:e]])
        o_ref, l_ref = _sdpa_branch(qfull, kfull, vfull, None, Hkv, torch.from_numpy(hm_eff).long(), theta, scale)
        np.testing.assert_allclose(out[a:e], o_ref[Lp:], atol=1e-12)
        np.testing.assert_allclose(lse[a:e], l_ref[Lp:], atol=1e-12)


def test_lp_zero_is_plain_causal_attention():
    rng = np.random.default_rng(4)
    L, Hq, Hkv, d, theta = 11, 2, 1, 8, 500.0
    q = rng.standard_normal((L, Hq, d)).astype(np.float32)
    k = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    empty = np.zeros((0, Hkv, d), np.float32)
    out, lse = oracle.prefix_suffix_attn(q, empty, empty, k, v, np.array([0, L]), theta=theta)
    qr = _rope_complex(q.astype(np.float64).transpose(1, 0, 2), np.arange(L), theta).transpose(1, 0, 2)
    kr = _rope_complex(k.astype(np.float64).transpose(1, 0, 2), np.arange(L), theta).transpose(1, 0, 2)
    o_ref, l_ref = _sdpa_branch(qr, kr, v.astype(np.float64), None, Hkv, torch.zeros(Hq, dtype=torch.long),
                                theta, 1 / math.sqrt(d))
    np.testing.assert_allclose(out, o_ref, atol=1e-12)
    np.testing.assert_allclose(lse, l_ref, atol=1e-12)


def test_zero_query_averages_visible_values():
    c = _small_case()
    q = np.zeros_like(c.q)
    out, lse = oracle.prefix_suffix_attn(q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens)
    G = c.cfg.Hq // c.cfg.Hkv
    for b in range(c.cu_seqlens.size - 1):
        for j in range(c.cu_seqlens[b + 1] - c.cu_seqlens[b]):
            t = c.cu_seqlens[b] + j
            vis = np.concatenate([c.v_pre, c.v_suf[c.cu_seqlens[b]:t + 1]]).astype(np.float64)
            for h in range(c.cfg.Hq):
                np.testing.assert_allclose(out[t, h], vis[:, h // G].mean(0), atol=1e-12)
                assert abs(lse[t, h] - math.log(vis.shape[0])) < 1e-12


def test_dominant_own_key_selects_own_value():
    c = _small_case(d=64)
    G = c.cfg.Hq // c.cfg.Hkv
    q = np.repeat(c.k_suf, G, axis=1) * np.float32(50.0)  # q_raw = 50 * own k_raw, same rotation
    out, _ = oracle.prefix_suffix_attn(q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens)
    np.testing.assert_allclose(out, np.repeat(c.v_suf, G, axis=1), atol=1e-9)


def test_split_point_invariance_and_empty_suffix():
    """prefix[0, L-k) + a k-token suffix at positions L-k.. gives the last k
    rows of full causal attention over L tokens; k=1 is the prefix's own
    last-position attention (a branch with an empty question reproduces it)."""
    rng = np.random.default_rng(8)
    L, Hq, Hkv, d, theta = 13, 4, 2, 16, 1e4
    q = rng.standard_normal((L, Hq, d)).astype(np.float32)
    k = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    empty = np.zeros((0, Hkv, d), np.float32)
    full, full_lse = oracle.prefix_suffix_attn(q, empty, empty, k, v, np.array([0, L]), theta=theta)
    for kk in (1, 2, 5, L - 1):
        Lp = L - kk
        # the cache holds fp32 keys rotated at positions 0..Lp-1
        kp32 = np.stack([np.stack([oracle.rope(k[t, g].astype(np.float64), t, theta) for g in range(Hkv)])
                         for t in range(Lp)]).astype(np.float32)
        out, lse = oracle.prefix_suffix_attn(q[Lp:], kp32, v[:Lp], k[Lp:], v[Lp:], np.array([0, kk]), theta=theta)
        # only the fp32 rounding of the cached keys separates the two runs
        np.testing.assert_allclose(out, full[Lp:], atol=1e-5)
        np.testing.assert_allclose(lse, full_lse[Lp:], atol=1e-5)


def test_split_point_exact_with_fp64_keys():
    """Exact form of the split-point identity: with keys that are exactly
    representable after rotation (rotation at position 0 is the identity),
    a one-token prefix plus suffix equals the unsplit run to rounding."""
    rng = np.random.default_rng(9)
    L, Hq, Hkv, d, theta = 6, 2, 1, 8, 1e4
    q = rng.standard_normal((L, Hq, d)).astype(np.float32)
    k = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((L, Hkv, d)).astype(np.float32)
    empty = np.zeros((0, Hkv, d), np.float32)
    full, full_lse = oracle.prefix_suffix_attn(q, empty, empty, k, v, np.array([0, L]), theta=theta)
    out, lse = oracle.prefix_suffix_attn(q[1:], k[:1], v[:1], k[1:], v[1:], np.array([0, L - 1]), theta=theta)
    np.testing.assert_allclose(out, full[1:], atol=1e-13)
    np.testing.assert_allclose(lse, full_lse[1:], atol=1e-13)


def test_relative_position_invariance():
    """Shifting every position by D (prefix cache rotated from D, suffix from
    Lp + D) leaves scores, and so the outputs, unchanged."""
    rng = np.random.default_rng(10)
    Lp, Hq, Hkv, d, theta = 7, 2, 1, 16, 1e4
    lens = np.array([3, 4], np.int32)
    cu = np.array([0, 3, 7], np.int32)
    k_raw = rng.standard_normal((Lp, Hkv, d))
    q = rng.standard_normal((7, Hq, d)).astype(np.float32)
    ks = rng.standard_normal((7, Hkv, d)).astype(np.float32)
    vs = rng.standard_normal((7, Hkv, d)).astype(np.float32)
    vp = rng.standard_normal((Lp, Hkv, d)).astype(np.float32)
    res = []
    for D in (0, 37):
        kp = np.stack([[oracle.rope(k_raw[t, g], t + D, theta) for g in range(Hkv)] for t in range(Lp)])
        res.append(oracle.prefix_suffix_attn(q, kp.astype(np.float32), vp, ks, vs, cu, theta=theta,
                                             pos_offset=Lp + D))
    # the fp32 cache rounds the two rotations differently; scores agree to that rounding
    np.testing.assert_allclose(res[0][0], res[1][0], atol=2e-6)
    np.testing.assert_allclose(res[0][1], res[1][1], atol=2e-6)


def test_permutation_and_insertion_are_exact():
    c = _small_case(B=4, lens=(2, 5, 1, 3))
    cu = c.cu_seqlens
    out, lse = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, cu)
    perm = [2, 0, 3, 1]
    idx = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in perm])
    lens = np.diff(cu)[perm]
    cu2 = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o2, l2 = oracle.prefix_suffix_attn(c.q[idx], c.k_pre, c.v_pre, c.k_suf[idx], c.v_suf[idx], cu2)
    assert np.array_equal(o2, out[idx]) and np.array_equal(l2, lse[idx])
    # insert a new branch of 4 tokens in front: every old row is unchanged bit for bit
    rng = np.random.default_rng(1)
    ins = lambda a: np.concatenate([rng.standard_normal((4,) + a.shape[1:]).astype(a.dtype), a])
    cu3 = np.concatenate([[0], 4 + cu]).astype(np.int32)
    o3, l3 = oracle.prefix_suffix_attn(ins(c.q), c.k_pre, c.v_pre, ins(c.k_suf), ins(c.v_suf), cu3)
    assert np.array_equal(o3[4:], out) and np.array_equal(l3[4:], lse)


def test_merge_identity_of_partials():
    """Attention over [A; B] equals the log-sum-exp merge of the attentions
    over A and over B — the identity that lets the prefix be shared."""
    rng = np.random.default_rng(12)
    d = 32
    q = rng.standard_normal(d)
    K = rng.standard_normal((40, d)); V = rng.standard_normal((40, d))
    o, l = oracle.attend(q, K, V, 0.3)
    oa, la = oracle.attend(q, K[:29], V[:29], 0.3)
    ob, lb = oracle.attend(q, K[29:], V[29:], 0.3)
    m = max(la, lb)
    wa, wb = math.exp(la - m), math.exp(lb - m)
    np.testing.assert_allclose((wa * oa + wb * ob) / (wa + wb), o, atol=1e-12)
    assert abs(m + math.log(wa + wb) - l) < 1e-12
    # and against numpy's direct softmax form
    s = 0.3 * K @ q
    w = np.exp(s - s.max())
    np.testing.assert_allclose(o, w @ V / w.sum(), atol=1e-12)


def test_row_subset_matches_full():
    c = _small_case(dtype=synth.BF16)
    out, lse = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens)
    rows = np.array([[0, 0], [5, 3], [10, 1], [3, 2]], np.int32)
    o2, l2 = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens, rows=rows)
    for i, (t, h) in enumerate(rows):
        assert np.array_equal(o2[i], out[t, h]) and l2[i] == lse[t, h]


def test_bad_arguments_rejected():
    c = _small_case()
    with pytest.raises(ValueError):
        oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, np.array([0, 5, 3, 11]))


# --------------------------------------------------------------------------- readout


def test_readout_two_options_is_log_sigmoid():
    g = _gold("readout_pair.json")
    for z, lp_e, ch_e in ((g["logits"], g["expected_logprob"], g["expected_choice"]),
                          (g["tie_logits"], g["tie_expected_logprob"], g["tie_expected_choice"])):
        hidden = np.array([[1.0]], np.float32)
        W = np.array([[z[0]], [z[1]]], np.float32)
        r = oracle.candidate_readout(hidden, W, np.array([0, 2]), np.array([0, 1]))
        np.testing.assert_allclose(r["logprob"], lp_e, atol=g["tolerance"])
        assert r["choice"][0] == ch_e


def _readout_case(seed=0, n_sets=5, H=24, V=50, dtype=synth.F32):
    rng = np.random.default_rng(seed)
    nopt = rng.integers(1, 6, n_sets)
    so = np.concatenate([[0], np.cumsum(nopt)]).astype(np.int32)
    toks = np.concatenate([rng.choice(V, n, replace=False) for n in nopt]).astype(np.int32)
    h = rng.standard_normal((n_sets, H)).astype(np.float32)
    W = (0.3 * rng.standard_normal((V, H))).astype(np.float32)
    if dtype == synth.BF16:
        h, W = synth.f32_to_bf16_bits(h), synth.f32_to_bf16_bits(W)
    return h, W, so, toks


@pytest.mark.parametrize("dtype", [synth.F32, synth.BF16])
def test_readout_against_matmul_and_full_vocab(dtype):
    h, W, so, toks = _readout_case(dtype=dtype)
    r = oracle.candidate_readout(h, W, so, toks)
    hf, Wf = _f64(h), _f64(W)
    Z = hf @ Wf.T  # numpy matmul: every logit
    for s in range(so.size - 1):
        zc = Z[s, toks[so[s]:so[s + 1]]]
        np.testing.assert_allclose(r["score"][so[s]:so[s + 1]], zc, atol=1e-12)
        full_lse = np.log(np.exp(Z[s] - Z[s].max()).sum()) + Z[s].max()
        assert abs(r["row_lse"][s] - full_lse) < 1e-12
        # restricted log-softmax == full-vocab log-softmax renormalised over the set
        full_lp = zc - full_lse
        renorm = full_lp - np.log(np.exp(full_lp).sum())
        np.testing.assert_allclose(r["logprob"][so[s]:so[s + 1]], renorm, atol=1e-12)
        assert abs(np.exp(r["logprob"][so[s]:so[s + 1]]).sum() - 1.0) < 1e-12
        assert r["choice"][s] == int(np.argmax(zc))
    r2 = oracle.candidate_readout(h, W, so, toks, full_vocab=False)
    np.testing.assert_allclose(r2["score"], r["score"], atol=1e-12)
    assert np.array_equal(r2["choice"], r["choice"])


def test_readout_multi_token_candidates_sum_pairs():
    rng = np.random.default_rng(2)
    R, H, V = 6, 16, 30
    h = rng.standard_normal((R, H)).astype(np.float32)
    W = rng.standard_normal((V, H)).astype(np.float32)
    so = np.array([0, 2, 3])
    co = np.array([0, 3, 4, 6])
    prow = np.array([0, 1, 2, 3, 4, 5])
    ptok = np.array([4, 7, 1, 9, 0, 29])
    r = oracle.candidate_readout(h, W, so, ptok, cand_offsets=co, pair_row=prow)
    z = np.array([h[prow[k]].astype(np.float64) @ W[ptok[k]].astype(np.float64) for k in range(6)])
    np.testing.assert_allclose(r["score"], [z[0:3].sum(), z[3], z[4:6].sum()], atol=1e-12)
    lp0 = r["score"][0:2] - np.log(np.exp(r["score"][0:2]).sum())
    np.testing.assert_allclose(r["logprob"][0:2], lp0, atol=1e-12)
    assert r["logprob"][2] == 0.0 and r["choice"][1] == 0 and r["gap"][1] == np.inf


def test_readout_invalid_and_empty_sets():
    h, W, so, toks = _readout_case(n_sets=3)
    toks = toks.copy()
    toks[so[1]] = W.shape[0]  # out of range in set 1
    so2 = np.concatenate([so, [so[-1]]])  # a fourth, empty set
    r = oracle.candidate_readout(h[[0, 1, 2, 2]], W, so2, toks)
    assert r["n_invalid"] == 1
    assert np.isnan(r["score"][so[1]]) and r["choice"][1] == -1 and np.all(np.isnan(r["logprob"][so[1]:so[2]]))
    assert r["choice"][3] == -1 and r["choice"][0] >= 0


# --------------------------------------------------------------------------- trie


def _trie_csr(cands):
    so = np.concatenate([[0], np.cumsum([len(c) for c in cands])]).astype(np.int32)
    toks = np.array([t for c in cands for t in c], np.int32)
    return so, toks


def test_trie_hand_examples():
    for case in _gold("trie_hand.json")["cases"]:
        so, toks = _trie_csr(case["cands"])
        t = oracle.trie_build(so, toks, case["root_len"])
        assert t["parent"].tolist() == case["parent"]
        assert t["tok_off"].tolist() == case["tok_off"]
        assert t["pos0"].tolist() == case["pos0"]
        assert t["node_toks"].tolist() == case["node_toks"]
        assert t["leaf_of"].tolist() == case["leaf_of"]
        pr = t["path_row"].tolist()
        assert [pr[so[c]:so[c + 1]] for c in range(len(case["cands"]))] == case["path_row"]


def _brute_trie(cands, root_len):
    """Canonical trie from sets of prefixes (a second, independent construction)."""
    prefixes = {}
    for ci, c in enumerate(cands):
        for i in range(1, len(c) + 1):
            prefixes.setdefault(tuple(c[:i]), ci)
    ends = {tuple(c) for c in cands if len(c)}
    children = {}
    for p in prefixes:
        children.setdefault(p[:-1], []).append(p)
    for k in children:
        children[k].sort(key=lambda p: prefixes[p])

    def starts_segment(p):
        par = p[:-1]
        return len(par) == 0 or len(children.get(par, [])) >= 2 or par in ends

    parent, tok_off, pos0, node_toks, node_of = [-1], [0, 0], [0], [], {}
    order = []

    def visit(p, par_id):
        nid = len(parent)
        parent.append(par_id)
        pos0.append(root_len + len(p) - 1)
        cur = p
        while True:
            node_of[cur] = (nid, len(node_toks))
            node_toks.append(cur[-1])
            kids = children.get(cur, [])
            if len(kids) == 1 and cur not in ends:
                cur = kids[0]
            else:
                break
        tok_off.append(len(node_toks))
        for k in kids:
            visit(k, nid)

    for k in children.get((), []):
        visit(k, 0)
    leaf_of = [node_of[tuple(c)][0] if len(c) else 0 for c in cands]
    path_row = [[node_of[tuple(c[:i + 1])][1] for i in range(len(c))] for c in cands]
    return dict(parent=parent, tok_off=tok_off, pos0=pos0, node_toks=node_toks, leaf_of=leaf_of, path_row=path_row)


def test_trie_bruteforce_random():
    rng = np.random.default_rng(123)
    for trial in range(400):
        n = int(rng.integers(1, 7))
        cands = [list(rng.integers(0, 4, int(rng.integers(0, 6)))) for _ in range(n)]
        root_len = int(rng.integers(0, 20))
        so, toks = _trie_csr(cands)
        t = oracle.trie_build(so, toks, root_len)
        ref = _brute_trie(cands, root_len)
        assert t["parent"].tolist() == ref["parent"], cands
        assert t["tok_off"].tolist() == ref["tok_off"], cands
        assert t["pos0"].tolist() == ref["pos0"], cands
        assert t["node_toks"].tolist() == ref["node_toks"], cands
        assert t["leaf_of"].tolist() == ref["leaf_of"], cands
        pr = t["path_row"].tolist()
        assert [pr[so[c]:so[c + 1]] for c in range(n)] == ref["path_row"], cands
        # invariants: unique (parent, first token) among siblings; each path spells its candidate
        firsts = {}
        for nd in range(1, t["n_nodes"]):
            key = (int(t["parent"][nd]), int(t["node_toks"][t["tok_off"][nd]]))
            assert key not in firsts
            firsts[key] = nd
        nt = t["node_toks"]
        for c in range(n):
            assert [int(nt[r]) for r in pr[so[c]:so[c + 1]]] == [int(x) for x in cands[c]]
        assert t["tok_off"][-1] == len({tuple(c[:i]) for c in cands for i in range(1, len(c) + 1)})


# --------------------------------------------------------------------------- tree


def _small_tree(seed=0, nq=3, qlen=4, Lp=6, Hq=4, Hkv=2, d=16, V=40, dtype=synth.F32):
    cfg = synth.TreeConfig("t", dtype, Lp, nq, qlen, 2, 3, 1, 3, Hq, Hkv, d, 8, V, seed=seed)
    return synth.tree_case(cfg, with_lm_head=False)


@pytest.mark.parametrize("Lp", [6, 0])
def test_tree_matches_sdpa_on_every_path(Lp):
    # Lp = 0: an empty root, so every first-level node is its own prefix (one question over
    # several images, each an independent row: Ochevid, "One question, multiple images")
    tc = _small_tree(Lp=Lp)
    t = oracle.trie_build(tc.seq_off, tc.toks, tc.cfg.Lp)
    assert t["tok_off"][-1] == tc.n_unique
    out, lse = oracle.tree_attn(t, tc.q, tc.k, tc.v, tc.k_root, tc.v_root)
    Lp, Hq, Hkv, d = tc.cfg.Lp, tc.cfg.Hq, tc.cfg.Hkv, tc.cfg.d
    hm = torch.arange(Hq) // (Hq // Hkv)
    for c in range(tc.seq_off.size - 1):
        rows = t["path_row"][tc.seq_off[c]:tc.seq_off[c + 1]]
        pos = Lp + np.arange(rows.size)
        qp = _rope_complex(tc.q[rows].astype(np.float64).transpose(1, 0, 2), pos, 1e4).transpose(1, 0, 2)
        kp = _rope_complex(tc.k[rows].astype(np.float64).transpose(1, 0, 2), pos, 1e4).transpose(1, 0, 2)
        qf = np.concatenate([np.zeros((Lp, Hq, d)), qp])
        kf = np.concatenate([tc.k_root.astype(np.float64), kp])
        vf = np.concatenate([tc.v_root.astype(np.float64), tc.v[rows].astype(np.float64)])
        o_ref, l_ref = _sdpa_branch(qf, kf, vf, None, Hkv, hm, 1e4, 1 / math.sqrt(d))
        np.testing.assert_allclose(out[rows], o_ref[Lp:], atol=1e-12)
        np.testing.assert_allclose(lse[rows], l_ref[Lp:], atol=1e-12)


def test_tree_of_disjoint_paths_equals_flat():
    """Candidates with distinct first tokens share nothing but the root: the
    trie is one node per candidate and tree attention is the flat problem."""
    rng = np.random.default_rng(5)
    lens = [3, 1, 4, 2]
    cands = [[100 + i] + list(rng.integers(0, 50, n - 1)) for i, n in enumerate(lens)]
    so, toks = _trie_csr(cands)
    t = oracle.trie_build(so, toks, 5)
    assert t["n_nodes"] == 5 and np.all(t["parent"][1:] == 0)
    c = _small_case(B=4, Lp=5, lens=lens, Hq=4, Hkv=2, d=16)
    out_t, lse_t = oracle.tree_attn(t, c.q, c.k_suf, c.v_suf, c.k_pre, c.v_pre)
    out_f, lse_f = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens)
    assert np.array_equal(out_t, out_f) and np.array_equal(lse_t, lse_f)


def test_tree_readout_pairs_teacher_forcing():
    tc = _small_tree(seed=3)
    t = oracle.trie_build(tc.seq_off, tc.toks, tc.cfg.Lp)
    co, prow, tix = oracle.tree_readout_pairs(tc.seq_off, tc.score_from, t["path_row"], tc.set_offsets)
    for c in range(tc.seq_off.size - 1):
        a, e = tc.seq_off[c], tc.seq_off[c + 1]
        k = co[c]
        assert co[c + 1] - co[c] == e - a - tc.score_from[c]
        # first scored token is predicted from the last question token's row
        assert prow[k] == t["path_row"][a + tc.score_from[c] - 1]
        assert tix[k] == a + tc.score_from[c]


def test_tree_readout_hand_golden():
    """Multi-token options against a hand-derived case: every (row, token) pair
    of a 1-, 2- and 3-token option, the summed scores, the set log-softmax and
    the choice.  Scoring a token from the question's last row, or from its own
    row, changes the expected scores."""
    g = _gold("tree_readout.json")
    so, toks = _trie_csr(g["cands"])
    t = oracle.trie_build(so, toks, g["root_len"])
    pr = t["path_row"]
    assert [pr[so[c]:so[c + 1]].tolist() for c in range(len(g["cands"]))] == g["path_row"]
    co, prow, tix = oracle.tree_readout_pairs(so, np.asarray(g["score_from"], np.int32), pr,
                                              np.asarray(g["set_offsets"], np.int32))
    assert co.tolist() == g["cand_offsets"]
    assert prow.tolist() == g["pair_row"]
    assert toks[tix].tolist() == g["pair_tok"]
    h = np.asarray(g["hidden"], np.float32)
    W = np.asarray(g["lm_head"], np.float32)
    r = oracle.candidate_readout(h, W, np.asarray(g["set_offsets"], np.int32), toks[tix], cand_offsets=co,
                                 pair_row=prow)
    tol = g["tolerance"]
    np.testing.assert_allclose(r["score"], g["expected_score"], rtol=0, atol=tol)
    np.testing.assert_allclose(r["logprob"], g["expected_logprob"], rtol=0, atol=tol)
    assert r["choice"].tolist() == [g["expected_choice"]]
    # the rows of each option's last token are never read
    h2 = h.copy()
    h2[[2, 4, 7]] = 100.0
    r2 = oracle.candidate_readout(h2, W, np.asarray(g["set_offsets"], np.int32), toks[tix], cand_offsets=co,
                                  pair_row=prow)
    assert np.array_equal(r2["score"], r["score"])


def test_tree_readout_of_one_token_leaves_is_the_flat_readout():
    """A tree whose options are all one token reads out exactly as the flat
    problem whose branch hidden state is each question's last-token row."""
    cfg = synth.TreeConfig("t1", synth.F32, 5, 4, 3, 2, 5, 1, 1, 4, 2, 16, 24, 60, seed=9)
    tc = synth.tree_case(cfg, with_lm_head=True)
    t = oracle.trie_build(tc.seq_off, tc.toks, cfg.Lp)
    co, prow, tix = oracle.tree_readout_pairs(tc.seq_off, tc.score_from, t["path_row"], tc.set_offsets)
    assert np.array_equal(co, np.arange(co.size, dtype=np.int32))  # one pair per candidate
    tree = oracle.candidate_readout(tc.hidden, tc.W, tc.set_offsets, tc.toks[tix], cand_offsets=co, pair_row=prow)
    # flat: branch b's hidden state is the row of its question's last token
    n_sets = tc.set_offsets.size - 1
    last_q = [int(t["path_row"][tc.seq_off[tc.set_offsets[b]] + cfg.q_len - 1]) for b in range(n_sets)]
    opt_tok = np.array([tc.toks[tc.seq_off[c] + cfg.q_len] for c in range(tc.seq_off.size - 1)], np.int32)
    flat = oracle.candidate_readout(tc.hidden[last_q], tc.W, tc.set_offsets, opt_tok)
    for k in ("score", "logprob", "choice", "gap"):
        assert np.array_equal(tree[k], flat[k]), k


# ---------------------------------------------------------------- full-vocabulary LSE (normalised scoring)

def test_vocab_lse_closed_forms():
    rng = np.random.default_rng(11)
    R, H, V = 4, 16, 37
    h = rng.standard_normal((R, H)).astype(np.float32)
    # all logits zero: log V
    np.testing.assert_allclose(oracle.vocab_lse(h, np.zeros((V, H), np.float32)), math.log(V), rtol=0, atol=1e-12)
    # every vocabulary row the same vector w: log V + h . w
    w = rng.standard_normal(H).astype(np.float32)
    got = oracle.vocab_lse(h, np.tile(w, (V, 1)))
    np.testing.assert_allclose(got, math.log(V) + _f64(h) @ _f64(w), rtol=0, atol=1e-10)
    # one-hot rows: hidden e_j against W = c * I gives one logit c and V - 1 zeros
    c = 3.5
    W = (c * np.eye(H)).astype(np.float32)
    e = np.eye(H, dtype=np.float32)[[0, 5, 15]]
    np.testing.assert_allclose(oracle.vocab_lse(e, W), math.log(math.exp(c) + H - 1), rtol=0, atol=1e-12)


def test_vocab_lse_shift_and_bf16():
    rng = np.random.default_rng(12)
    R, H, V = 3, 24, 41
    h = rng.standard_normal((R, H)).astype(np.float32)
    W = (0.5 * rng.standard_normal((V, H))).astype(np.float32)
    a = rng.standard_normal(H).astype(np.float32)
    # adding one vector to every vocabulary row shifts every logit of row r by h_r . a
    base = oracle.vocab_lse(h, W)
    shifted = oracle.vocab_lse(h, (W.astype(np.float64) + a).astype(np.float32))
    ref_shift = _f64(h) @ _f64(a)
    # (the float32 rounding of W + a is the only difference)
    np.testing.assert_allclose(shifted - base, ref_shift, rtol=0, atol=1e-4)
    # bf16 inputs are widened exactly: same answer as the float32 copy of the bf16 values
    hb, Wb = synth.f32_to_bf16_bits(h), synth.f32_to_bf16_bits(W)
    np.testing.assert_allclose(oracle.vocab_lse(hb, Wb), oracle.vocab_lse(_f64(hb).astype(np.float32),
                                                                           _f64(Wb).astype(np.float32)),
                               rtol=0, atol=1e-12)


def test_sequence_logprob_is_a_distribution_and_adds():
    rng = np.random.default_rng(13)
    R, H, V = 2, 8, 19
    h = rng.standard_normal((R, H)).astype(np.float32)
    W = rng.standard_normal((V, H)).astype(np.float32)
    # every one-token continuation of row 0: the probabilities over the vocabulary sum to 1
    co = np.arange(V + 1, dtype=np.int32)
    lp = oracle.sequence_logprob(h, W, co, np.zeros(V, np.int32), np.arange(V, dtype=np.int32))
    assert abs(np.exp(lp).sum() - 1.0) < 1e-12
    assert np.all(lp < 0)
    # a two-token candidate scores the sum of its two one-token terms
    lp2 = oracle.sequence_logprob(h, W, np.array([0, 2, 3, 4], np.int32), np.array([0, 1, 0, 1], np.int32),
                                  np.array([4, 7, 4, 7], np.int32))
    assert abs(lp2[0] - (lp2[1] + lp2[2])) < 1e-12
    # and the all-pairs table of row 1 also normalises
    lp1 = oracle.sequence_logprob(h, W, co, np.ones(V, np.int32), np.arange(V, dtype=np.int32))
    assert abs(np.exp(lp1).sum() - 1.0) < 1e-12
    assert abs(lp2[2] - lp1[7]) < 1e-12 and abs(lp2[1] - lp[4]) < 1e-12


# ---------------------------------------------------------------- generation over per-branch suffix caches


def _cache_case(rng, Lp=7, Hq=4, Hkv=2, d=16, cached=(0, 3, 5, 2), new=(2, 1, 0, 3), spare=(1, 0, 2, 1),
                dtype=np.float32, theta=1e4, pos_offset=-1):
    """Random new tokens and caches whose keys are the independent complex
    rotation of raw keys at the positions the cached tokens held."""
    B = len(cached)
    po = Lp if pos_offset < 0 else pos_offset
    cap = [c + n + s for c, n, s in zip(cached, new, spare)]
    co = np.concatenate([[0], np.cumsum(cap)]).astype(np.int32)
    cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    C, T = int(co[-1]), int(cu[-1])
    k_pre = rng.standard_normal((Lp, Hkv, d)).astype(np.float32)
    v_pre = rng.standard_normal((Lp, Hkv, d)).astype(np.float32)
    k_cache = np.zeros((C, Hkv, d), np.float32)
    v_cache = rng.standard_normal((C, Hkv, d)).astype(np.float32)
    k_cached_raw = []
    for b in range(B):
        raw = rng.standard_normal((cached[b], Hkv, d))
        k_cached_raw.append(raw)
        rot = _rope_complex(raw.transpose(1, 0, 2), po + np.arange(cached[b]), theta).transpose(1, 0, 2)
        k_cache[co[b]:co[b] + cached[b]] = rot
    q = rng.standard_normal((T, Hq, d)).astype(np.float32)
    k_new = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    v_new = rng.standard_normal((T, Hkv, d)).astype(np.float32)
    return dict(q=q, k_new=k_new, v_new=v_new, k_pre=k_pre, v_pre=v_pre, k_cache=k_cache, v_cache=v_cache,
                cache_off=co, cache_len=np.array(cached, np.int32), cu_new=cu, k_cached_raw=k_cached_raw, po=po)


def test_cache_attn_matches_sdpa_over_prefix_cache_and_new_tokens():
    """Each new token's row equals causal fp64 SDPA over [prefix; the branch's
    cached keys; its rotated new keys] at the row of that token, and the
    appended keys are the complex rotation of the new keys."""
    rng = np.random.default_rng(21)
    theta, Hq, Hkv, d = 1e4, 4, 2, 16
    for pos_offset, head_map in ((-1, None), (40, np.array([1, 0, 1, 0], np.int32))):
        c = _cache_case(rng, theta=theta, pos_offset=pos_offset)
        out, lse, krot = oracle.cache_attn(c["q"], c["k_new"], c["v_new"], c["k_pre"], c["v_pre"], c["k_cache"],
                                           c["v_cache"], c["cache_off"], c["cache_len"], c["cu_new"], theta=theta,
                                           pos_offset=pos_offset, head_map=head_map)
        hm = torch.from_numpy(head_map).long() if head_map is not None else torch.arange(Hq) // (Hq // Hkv)
        cu, co, cl, po = c["cu_new"], c["cache_off"], c["cache_len"], c["po"]
        Lp = c["k_pre"].shape[0]
        for b in range(cu.size - 1):
            n = int(cu[b + 1] - cu[b])
            if n == 0:
                continue
            pos_new = po + cl[b] + np.arange(n)
            kn = _rope_complex(c["k_new"][cu[b]:cu[b + 1]].astype(np.float64).transpose(1, 0, 2), pos_new,
                               theta).transpose(1, 0, 2)
            np.testing.assert_allclose(krot[cu[b]:cu[b + 1]], kn, atol=1e-12)
            qn = _rope_complex(c["q"][cu[b]:cu[b + 1]].astype(np.float64).transpose(1, 0, 2), pos_new,
                               theta).transpose(1, 0, 2)
            L0 = Lp + int(cl[b])
            kf = np.concatenate([c["k_pre"].astype(np.float64), c["k_cache"][co[b]:co[b] + cl[b]].astype(np.float64), kn])
            vf = np.concatenate([c["v_pre"], c["v_cache"][co[b]:co[b] + cl[b]], c["v_new"][cu[b]:cu[b + 1]]]).astype(np.float64)
            qf = np.concatenate([np.zeros((L0, Hq, d)), qn])
            o_ref, l_ref = _sdpa_branch(qf, kf, vf, None, Hkv, hm, theta, 1 / math.sqrt(d))
            np.testing.assert_allclose(out[cu[b]:cu[b + 1]], o_ref[L0:], atol=1e-12)
            np.testing.assert_allclose(lse[cu[b]:cu[b + 1]], l_ref[L0:], atol=1e-12)


def test_cache_attn_with_empty_caches_is_the_prefill():
    """With nothing cached, the step is jev's flat problem on the new tokens."""
    c = _small_case(B=4, lens=(3, 1, 5, 2))
    cu = c.cu_seqlens
    co = cu.copy()  # caches exactly as large as the new tokens
    out, lse, krot = oracle.cache_attn(c.q, c.k_suf, c.v_suf, c.k_pre, c.v_pre, np.zeros_like(c.k_suf),
                                       np.zeros_like(c.v_suf), co, np.zeros(4, np.int32), cu)
    o_ref, l_ref = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, cu)
    np.testing.assert_allclose(out, o_ref, atol=1e-13)
    np.testing.assert_allclose(lse, l_ref, atol=1e-13)


def test_cache_attn_step_is_the_next_row_of_the_whole_suffix():
    """Decoding the last m tokens over a cache of the first ones (rotated
    keys stored in float32) gives the rows of the whole suffix's attention."""
    rng = np.random.default_rng(22)
    lens, m = np.array([4, 1, 6], np.int32), np.array([1, 2, 1], np.int32)
    c = _small_case(B=3, lens=tuple(lens + m), Hq=6, Hkv=2, d=16)
    cu_full = c.cu_seqlens
    full_o, full_l = oracle.prefix_suffix_attn(c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, cu_full)
    Lp = c.k_pre.shape[0]
    co = np.concatenate([[0], np.cumsum(lens + m + 2)]).astype(np.int32)
    k_cache = np.zeros((co[-1], 2, 16), np.float32)
    v_cache = rng.standard_normal((co[-1], 2, 16)).astype(np.float32)
    new_rows = []
    for b in range(3):
        a = cu_full[b]
        raw = c.k_suf[a:a + lens[b]].astype(np.float64)
        k_cache[co[b]:co[b] + lens[b]] = _rope_complex(raw.transpose(1, 0, 2), Lp + np.arange(lens[b]),
                                                        1e4).transpose(1, 0, 2)
        v_cache[co[b]:co[b] + lens[b]] = c.v_suf[a:a + lens[b]]
        new_rows.append(np.arange(a + lens[b], a + lens[b] + m[b]))
    idx = np.concatenate(new_rows)
    cu_new = np.concatenate([[0], np.cumsum(m)]).astype(np.int32)
    out, lse, _ = oracle.cache_attn(c.q[idx], c.k_suf[idx], c.v_suf[idx], c.k_pre, c.v_pre, k_cache, v_cache, co,
                                    lens, cu_new)
    np.testing.assert_allclose(out, full_o[idx], atol=1e-5)
    np.testing.assert_allclose(lse, full_l[idx], atol=1e-5)


def test_cache_attn_rejects_a_branch_beyond_its_cache_rows():
    rng = np.random.default_rng(23)
    c = _cache_case(rng, cached=(2, 1), new=(1, 2), spare=(0, 0))
    cl = c["cache_len"].copy()
    cl[1] += 1  # one more cached token than the branch's rows leave room for
    with pytest.raises(ValueError):
        oracle.cache_attn(c["q"], c["k_new"], c["v_new"], c["k_pre"], c["v_pre"], c["k_cache"], c["v_cache"],
                          c["cache_off"], cl, c["cu_new"])
