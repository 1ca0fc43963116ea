"""The seeded generator: determinism, shapes of the five workloads, row-wise
regeneration of the LM head, and bf16 rounding (checked against torch)."""
import numpy as np
import torch

import synth


def test_flat_case_is_deterministic_and_shaped():
    cfg = synth.scaled(synth.CONFIGS["qwen2vl_2b"], V=4096, H=64)
    a = synth.flat_case(cfg)
    b = synth.flat_case(cfg)
    for x, y in ((a.q, b.q), (a.k_pre, b.k_pre), (a.W, b.W), (a.pair_tok, b.pair_tok), (a.cu_seqlens, b.cu_seqlens)):
        assert np.array_equal(x, y)
    Ls = np.diff(a.cu_seqlens)
    assert Ls.min() >= 8 and Ls.max() <= 24 and Ls.size == 8
    assert a.q.shape == (a.T, 12, 128) and a.k_pre.shape == (1024, 2, 128) and a.q.dtype == np.uint16
    nopt = np.diff(a.set_offsets)
    assert nopt.min() >= 3 and nopt.max() <= 9
    for s in range(8):
        opts = a.pair_tok[a.set_offsets[s]:a.set_offsets[s + 1]]
        assert np.unique(opts).size == opts.size and opts.min() >= 0 and opts.max() < cfg.V


def test_full_config_lengths():
    for name, lo, hi, B in (("qwen25vl_7b", 12, 32, 32), ("wide_7b", 8, 40, 128)):
        Ls = synth.suffix_lengths(synth.CONFIGS[name])
        assert Ls.size == B and Ls.min() >= lo and Ls.max() <= hi


def test_lm_head_rows_match_full_matrix():
    W = synth.lm_head(7, 9000, 16, synth.BF16)
    rows = np.array([0, 4095, 4096, 8999, 17])
    assert np.array_equal(synth.lm_head_rows(7, 9000, 16, rows, synth.BF16), W[rows])


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 3
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(synth.bf16_bits_to_f32(ours), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_tree_case_structure():
    tc = synth.tree_case(synth.CONFIGS["tree_7b"], with_lm_head=False)
    assert tc.set_offsets.size == 17
    nleaf = np.diff(tc.set_offsets)
    assert nleaf.min() >= 3 and nleaf.max() <= 9
    lens = np.diff(tc.seq_off) - 24
    assert lens.min() >= 1 and lens.max() <= 4
    assert tc.q.shape == (tc.n_unique, 28, 128)
