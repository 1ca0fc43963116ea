"""The allocation-free attention entry point.

Some callers cannot give the library a workspace: their device memory belongs
to a host runtime that budgets it and hands them no allocator, or they run at a
point where cudaMalloc/cudaFree (which synchronise the device) are not allowed.
jev_prefix_suffix_attn_noalloc serves them from a static device array.  These
tests call it through the C ABI twice in a row, on different problems, and
compare each result with jev_prefix_suffix_attn on the same inputs within the
attention tolerance of the other GPU tests.  This file is collected last so
that a run stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

import synth
from gpu_helpers import TOL, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def jev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import attention_cascade_b200 as m
    return m


def _inputs(lens, seed, Lp, Hq, Hkv, d, dtype=synth.BF16):
    cfg = synth.FlatConfig("na", dtype, Lp, len(lens), 1, 1, Hq, Hkv, d, 16, 32, 2, 3, seed=seed)
    c = synth.flat_case(cfg, with_lm_head=False, lengths=np.array(lens, np.int32))
    return [dev(x) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens)]


def test_noalloc_matches_workspace_entry_point_twice(jev):
    cases = [
        _inputs([17, 3, 40, 9], seed=21, Lp=1024, Hq=28, Hkv=4, d=128),
        _inputs([5, 31, 1], seed=22, Lp=300, Hq=12, Hkv=2, d=64),
    ]
    tol = TOL[synth.BF16]
    flags = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for q, kp, vp, ks, vs, cu in cases:
        ref_o, ref_l = jev.jev_prefix_suffix_attn(q, kp, vp, ks, vs, cu)
        out = torch.full_like(q, float("nan"))
        lse = torch.full(ref_l.shape, float("nan"), dtype=torch.float32, device="cuda")
        jev.jev_prefix_suffix_attn_noalloc(q, kp, vp, ks, vs, cu, out, lse, status_flags=flags)
        torch.cuda.synchronize()
        assert flags.item() == 0
        assert torch.isfinite(out.float()).all()
        err = (out.float() - ref_o.float()).abs()
        assert err.max().item() <= tol["max_abs"] and err.mean().item() <= tol["mean_abs"]
        assert (lse - ref_l).abs().max().item() <= tol["lse"]


def test_noalloc_falls_back_to_an_unsplit_plan_at_the_wide_shape(jev):
    """At the wide shape (128 branches over a 4096-token prefix) the automatic
    plan's split partials do not fit in the static scratch, but the unsplit
    plan does: the call must take it and still match the workspace entry
    point, twice in a row."""
    cfg = synth.CONFIGS["wide_7b"]
    c = synth.flat_case(cfg, with_lm_head=False)
    q, kp, vp, ks, vs, cu = [dev(x) for x in (c.q, c.k_pre, c.v_pre, c.k_suf, c.v_suf, c.cu_seqlens)]
    T, Hq, d = q.shape
    desc = jev.make_attn_desc(cfg.B, cfg.Lp, Hq, cfg.Hkv, d, T, jev.JEV_BF16)
    one = jev.make_attn_desc(cfg.B, cfg.Lp, Hq, cfg.Hkv, d, T, jev.JEV_BF16, num_splits=1)
    assert jev.jev_prefix_suffix_attn_workspace(desc) > jev.JEV_NOALLOC_SCRATCH_BYTES
    assert jev.jev_prefix_suffix_attn_workspace(one) <= jev.JEV_NOALLOC_SCRATCH_BYTES
    ref_o, ref_l = jev.jev_prefix_suffix_attn(q, kp, vp, ks, vs, cu)
    tol = TOL[synth.BF16]
    flags = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full(ref_l.shape, float("nan"), dtype=torch.float32, device="cuda")
        jev.jev_prefix_suffix_attn_noalloc(q, kp, vp, ks, vs, cu, out, lse, status_flags=flags)
        torch.cuda.synchronize()
        assert flags.item() == 0
        assert torch.isfinite(out.float()).all()
        err = (out.float() - ref_o.float()).abs()
        assert err.max().item() <= tol["max_abs"] and err.mean().item() <= tol["mean_abs"]
        assert (lse - ref_l).abs().max().item() <= tol["lse"]


def test_noalloc_rejects_problems_beyond_the_static_scratch(jev):
    # 20000 tokens x 28 heads x 128 of bf16 rotated queries alone exceed 32 MiB
    T, Hq, Hkv, d = 20000, 28, 4, 128
    q = torch.zeros((T, Hq, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((T, Hkv, d), dtype=torch.bfloat16, device="cuda")
    kp = torch.zeros((128, Hkv, d), dtype=torch.bfloat16, device="cuda")
    cu = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    n0 = jev.jev_launch_count()
    with pytest.raises(jev.JevError) as e:
        jev.jev_prefix_suffix_attn_noalloc(q, kp, kp, kv, kv, cu, out)
    assert e.value.status == 2 and "static scratch" in str(e.value)
    assert jev.jev_launch_count() == n0
