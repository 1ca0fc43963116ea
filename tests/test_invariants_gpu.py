"""GPU invariants the pages state ("Ochevid Jev-VL 2B" model card, Evidence:
question order, added questions and unequal tail lengths preserve answers;
Runtime 0.2: repeated runs reproduce probabilities exactly; the answers match
serial execution), plus split-count invariance, empty inputs and the device
status word on malformed inputs (which must flag, never fault)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, dev, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def jev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import attention_cascade_b200 as m
    return m


def _case(lens, seed=0, dtype=synth.BF16, Lp=640, Hq=14, Hkv=2, d=128):
    cfg = synth.FlatConfig("inv", dtype, Lp, len(lens), 1, 1, Hq, Hkv, d, 16, 32, 2, 3, seed=seed)
    return synth.flat_case(cfg, with_lm_head=False, lengths=np.array(lens, np.int32))


def _run(jev, c, **kw):
    out, lse = jev.jev_prefix_suffix_attn(*(dev(x) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf)),
                                          dev(c.cu_seqlens), **kw)
    torch.cuda.synchronize()
    return out, lse


def test_repeat_runs_are_bit_identical(jev):
    c = _case([13, 29, 7, 40, 1])
    a = _run(jev, c)
    b = _run(jev, c)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_branch_order_and_insertion(jev):
    lens = [13, 29, 7, 40, 1, 22]
    c = _case(lens, seed=1)
    out, lse = _run(jev, c, num_splits=2)
    perm = [3, 0, 5, 2, 1, 4]
    cu = c.cu_seqlens
    idx = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in perm])
    c2 = synth.FlatCase(c.cfg, c.q[idx], c.k_pre, c.v_pre, c.k_suf[idx], c.v_suf[idx],
                        np.concatenate([[0], np.cumsum(np.array(lens)[perm])]).astype(np.int32),
                        c.hidden, c.set_offsets, c.pair_tok)
    o2, l2 = _run(jev, c2, num_splits=2)
    tol = TOL[synth.BF16]
    assert (o2.float() - out[torch.from_numpy(idx).cuda()].float()).abs().max().item() <= tol["max_abs"] / 2
    assert (l2 - lse[torch.from_numpy(idx).cuda()]).abs().max().item() <= 1e-3
    # serial: each branch alone matches its rows in the batch
    for b in range(len(lens)):
        sl = slice(cu[b], cu[b + 1])
        cb = synth.FlatCase(c.cfg, c.q[sl], c.k_pre, c.v_pre, c.k_suf[sl], c.v_suf[sl],
                            np.array([0, lens[b]], np.int32), c.hidden, c.set_offsets, c.pair_tok)
        ob, lb = _run(jev, cb, num_splits=2)
        assert (ob.float() - out[cu[b]:cu[b + 1]].float()).abs().max().item() <= tol["max_abs"] / 2
        assert (lb - lse[cu[b]:cu[b + 1]]).abs().max().item() <= 1e-3


@pytest.mark.parametrize("dtype", [synth.BF16, synth.F32])
def test_split_count_invariance(jev, dtype):
    c = _case([31, 9, 18], seed=2, dtype=dtype, Lp=1500)
    outs = [_run(jev, c, num_splits=s) for s in (1, 2, 5, 0)]
    tol = 2e-2 if dtype == synth.BF16 else 1e-5
    for o, l in outs[1:]:
        assert (o.float() - outs[0][0].float()).abs().max().item() <= tol
        assert (l - outs[0][1]).abs().max().item() <= (1e-3 if dtype == synth.BF16 else 1e-5)


def test_empty_inputs(jev):
    z = torch.zeros((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    kp = torch.zeros((16, 2, 64), dtype=torch.bfloat16, device="cuda")
    n0 = jev.jev_launch_count()
    out, lse = jev.jev_prefix_suffix_attn(z, kp, kp, z[:, :2], z[:, :2], torch.zeros(1, dtype=torch.int32, device="cuda"))
    assert out.numel() == 0 and jev.jev_launch_count() == n0
    # branches that all have an empty suffix: nothing to compute
    out, lse = jev.jev_prefix_suffix_attn(z, kp, kp, z[:, :2], z[:, :2],
                                          torch.zeros(4, dtype=torch.int32, device="cuda"))
    assert jev.jev_launch_count() == n0


def test_status_word_flags_bad_inputs_without_faulting(jev):
    c = _case([5, 6, 7], seed=3, Lp=128)
    q, kp, vp, ks, vs = (dev(x) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf))
    desc = jev.make_attn_desc(3, 128, 14, 2, 128, 18, jev.JEV_BF16)
    ws = jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(desc), "cuda")
    bad_cu = torch.tensor([0, 9, 4, 18], dtype=torch.int32, device="cuda")  # decreasing
    jev.jev_prefix_suffix_attn(q, kp, vp, ks, vs, bad_cu, workspace=ws)
    assert jev.jev_check_device_status(ws) & jev.JEV_DEV_BAD_SEQLENS
    bad_hm = torch.tensor([0] * 14, dtype=torch.int32, device="cuda")  # every head on kv 0
    jev.jev_prefix_suffix_attn(q, kp, vp, ks, vs, dev(c.cu_seqlens), head_map=bad_hm, workspace=ws)
    assert jev.jev_check_device_status(ws) & jev.JEV_DEV_BAD_HEAD_MAP
    # the status word was cleared by the read; a good call leaves it clean
    jev.jev_prefix_suffix_attn(q, kp, vp, ks, vs, dev(c.cu_seqlens), workspace=ws)
    assert jev.jev_check_device_status(ws) == 0
    # the context is still healthy
    torch.cuda.synchronize()
    assert torch.isfinite(torch.ones(4, device="cuda").sum())


def _tree_case(jev, cands, root=64, Hq=4, Hkv=2, d=64, seed=0):
    so = np.concatenate([[0], np.cumsum([len(x) for x in cands])]).astype(np.int32)
    toks = np.array([t for x in cands for t in x], np.int32)
    t = jev.jev_tree_build(so, toks, root)
    N = int(t["tok_off"][-1])
    rng = np.random.default_rng(seed)
    mk = lambda *s: synth.f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32))
    return so, toks, t, (mk(N, Hq, d), mk(N, Hkv, d), mk(N, Hkv, d), mk(root, Hkv, d), mk(root, Hkv, d))


def test_tree_status_flags_malformed_trees_without_faulting(jev):
    """A node whose parent is not earlier than itself, and a tree numbered
    breadth-first instead of in depth-first preorder, set JEV_DEV_BAD_TREE;
    rows of the well-formed nodes of the first tree are still exact."""
    cands = [[1, 2], [1, 3], [4, 5, 6], [4, 7]]
    so, toks, t, (q, k, v, kr, vr) = _tree_case(jev, cands)
    parent = t["parent"].copy()
    last = t["n_nodes"] - 1
    parent[last] = last  # a node that is its own parent
    desc = jev.make_attn_desc(t["n_nodes"] - 1, 64, 4, 2, 64, int(t["tok_off"][-1]), jev.JEV_BF16)
    ws = jev.new_workspace(jev.jev_tree_attn_workspace(desc, t["n_nodes"]), "cuda")
    out, lse = jev.jev_tree_attn(dev(parent), dev(t["tok_off"]), dev(t["pos0"]), dev(q), dev(kr), dev(vr), dev(k),
                                 dev(v), workspace=ws)
    assert jev.jev_check_device_status(ws) & jev.JEV_DEV_BAD_TREE
    ref_o, _ = oracle.tree_attn(oracle.trie_build(so, toks, 64), q, k, v, kr, vr)
    good = np.arange(int(t["tok_off"][last]))  # every token before the corrupted node
    assert np.abs(host_f64(out)[good] - ref_o[good]).max() <= TOL[synth.BF16]["max_abs"]
    # breadth-first numbering: root children A = 1, B = 2, then A's child C = 3
    bfs_parent = np.array([-1, 0, 0, 1], np.int32)
    tok_off = np.array([0, 0, 2, 4, 6], np.int32)
    pos0 = np.array([0, 64, 64, 66], np.int32)
    rng = np.random.default_rng(1)
    mk = lambda *s: dev(synth.f32_to_bf16_bits(rng.standard_normal(s).astype(np.float32)))
    desc = jev.make_attn_desc(3, 64, 4, 2, 64, 6, jev.JEV_BF16)
    ws = jev.new_workspace(jev.jev_tree_attn_workspace(desc, 4), "cuda")
    jev.jev_tree_attn(dev(bfs_parent), dev(tok_off), dev(pos0), mk(6, 4, 64), mk(64, 2, 64), mk(64, 2, 64),
                      mk(6, 2, 64), mk(6, 2, 64), workspace=ws)
    assert jev.jev_check_device_status(ws) & jev.JEV_DEV_BAD_TREE
    torch.cuda.synchronize()
    assert torch.isfinite(torch.ones(4, device="cuda").sum())


def test_fma_pipe_exp2_against_cuda_exp2(jev):
    """The software 2^x used for a share of the softmax exponentials (the
    packed-pair form the attention kernel runs; an odd last element through
    the scalar form) stays within its stated bound of CUDA's exp2 over the
    range softmax feeds it."""
    x = torch.linspace(-125.0, 8.5, 1_000_003, device="cuda", dtype=torch.float32)
    y = jev.jev_selftest_exp2(x)
    ref = torch.exp2(x.double())
    rel = (y.double() / ref - 1.0).abs().max().item()
    assert rel < 2e-4, rel
    z = jev.jev_selftest_exp2(torch.tensor([-float("inf"), -1000.0, -200.0], device="cuda"))
    assert (z >= 0).all() and (z < 1e-37).all()


@pytest.mark.parametrize("rows", [0, 256])
def test_short_wait_limit_flags_a_timeout_and_leaves_the_context_usable(jev, rows, force_tile_rows):
    """Failure detection without a GPU fault: with the tensor-core kernels'
    wait bound cut to 256 cycles and the probe on (each CTA's MMA warp, with
    its first MMAs issued, also waits on a barrier that nothing completes, as
    a stalled pipeline would leave it), that wait runs out on an ordinary
    problem.  Each call must set JEV_DEV_WAIT_TIMEOUT and return (its CTAs
    drain the loads and MMAs they issued before exiting), and the next call
    with the probe off and the default bound must reproduce the earlier result
    exactly."""
    force_tile_rows(rows)  # 0: 128-row tiles (the one-Q-tile kernel) at this size
    c = _case([17, 3, 40, 9, 25], seed=8, Lp=1024, Hq=28, Hkv=4)
    args = [dev(x) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf)] + [dev(c.cu_seqlens)]
    desc = jev.make_attn_desc(5, 1024, 28, 4, 128, int(c.cu_seqlens[-1]), jev.JEV_BF16)
    ws = jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(desc), "cuda")
    o, l = jev.jev_prefix_suffix_attn(*args, workspace=ws)
    assert jev.jev_check_device_status(ws) == 0
    ref_o, ref_l = o.clone(), l.clone()
    rng = np.random.default_rng(4)
    h = dev(synth.f32_to_bf16_bits(rng.standard_normal((300, 512)).astype(np.float32)))
    W = dev(synth.f32_to_bf16_bits((0.05 * rng.standard_normal((20000, 512))).astype(np.float32)))
    lws = jev.new_workspace(jev.jev_vocab_lse_workspace(300, 20000), "cuda")
    ref_lse = jev.jev_vocab_lse(h, W, workspace=lws).clone()
    assert jev.jev_check_device_status(lws) == 0
    jev.jev_debug_set_wait_limit(256)
    jev.jev_debug_set_wait_probe(True)
    try:
        for _ in range(2):
            jev.jev_prefix_suffix_attn(*args, workspace=ws)
            assert jev.jev_check_device_status(ws) & jev.JEV_DEV_WAIT_TIMEOUT
            jev.jev_vocab_lse(h, W, workspace=lws)
            assert jev.jev_check_device_status(lws) & jev.JEV_DEV_WAIT_TIMEOUT
    finally:
        jev.jev_debug_set_wait_probe(False)
        jev.jev_debug_set_wait_limit(0)
    o, l = jev.jev_prefix_suffix_attn(*args, workspace=ws)
    assert jev.jev_check_device_status(ws) == 0
    assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
    assert torch.equal(jev.jev_vocab_lse(h, W, workspace=lws), ref_lse)
    assert jev.jev_check_device_status(lws) == 0
