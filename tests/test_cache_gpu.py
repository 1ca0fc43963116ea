"""GPU parity of a generation step over per-branch suffix caches
(jev_suffix_cache_attn) against oracle.cache_attn, element by element.

A prefill call (nothing cached) fills each branch's cache; decode steps then
append one or more tokens per branch.  The oracle keeps its own caches (its
rotated keys rounded to bf16, the values copied), so no oracle input comes
from the GPU; the GPU's cache rows are compared with the oracle's rotated
keys within one bf16 rounding and its values bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import TOL, check_attn, dev, host_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def jev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import attention_cascade_b200 as m
    return m


def _bf16(a):
    return synth.f32_to_bf16_bits(np.asarray(a, np.float32))


def _check_cache_rows(k_cache_gpu, v_cache_gpu, krot, v_new, rows, what):
    kg = host_f64(k_cache_gpu)[rows]
    # the GPU rotates in fp32 and rounds once to bf16: within one bf16 step of the fp64 value
    assert np.all(np.abs(kg - krot) <= 2.0 ** -7 * np.abs(krot) + 1e-30), what
    vg = v_cache_gpu.view(torch.int16).cpu().numpy().view(np.uint16)[rows]
    assert np.array_equal(vg, v_new), what


class _Caches:
    """Both sides' caches for B branches with the given row capacities."""

    def __init__(self, cap, Hkv, d):
        self.co = np.concatenate([[0], np.cumsum(cap)]).astype(np.int32)
        C = int(self.co[-1])
        self.len = np.zeros(len(cap), np.int32)
        self.k_o = np.zeros((C, Hkv, d), np.uint16)  # oracle side, bf16 bits
        self.v_o = np.zeros((C, Hkv, d), np.uint16)
        self.k_g = torch.zeros((C, Hkv, d), dtype=torch.bfloat16, device="cuda")
        self.v_g = torch.zeros((C, Hkv, d), dtype=torch.bfloat16, device="cuda")


def _step(jev, cc, rng, new, Lp, Hq, Hkv, d, k_pre, v_pre, what, **kw):
    cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    T = int(cu[-1])
    q = _bf16(rng.standard_normal((T, Hq, d)))
    kn = _bf16(rng.standard_normal((T, Hkv, d)))
    vn = _bf16(rng.standard_normal((T, Hkv, d)))
    out, lse = jev.jev_suffix_cache_attn(dev(q), dev(kn), dev(vn), dev(k_pre), dev(v_pre), cc.k_g, cc.v_g,
                                         dev(cc.co), dev(cc.len), dev(cu), **kw)
    torch.cuda.synchronize()
    ref_o, ref_l, krot = oracle.cache_attn(q, kn, vn, k_pre, v_pre, cc.k_o, cc.v_o, cc.co, cc.len, cu, **kw)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, synth.BF16, what)
    rows = np.concatenate([cc.co[b] + cc.len[b] + np.arange(new[b]) for b in range(len(new))]).astype(np.int64)
    _check_cache_rows(cc.k_g, cc.v_g, krot, vn, rows, what + " cache")
    cc.k_o[rows] = _bf16(krot)
    cc.v_o[rows] = vn
    cc.len += np.asarray(new, np.int32)


@pytest.mark.parametrize("Lp,Hq,Hkv,d", [(300, 28, 4, 128), (129, 8, 2, 64), (0, 4, 4, 64)])
def test_prefill_then_decode_steps(jev, Lp, Hq, Hkv, d):
    rng = np.random.default_rng(Lp + d)
    Ls = np.array([5, 17, 1, 30, 9, 12, 0, 40], np.int32)
    cc = _Caches(Ls + 6, Hkv, d)
    k_pre = _bf16(rng.standard_normal((Lp, Hkv, d)))
    v_pre = _bf16(rng.standard_normal((Lp, Hkv, d)))
    _step(jev, cc, rng, Ls, Lp, Hq, Hkv, d, k_pre, v_pre, "prefill")
    for s, new in enumerate(([1] * 8, [1, 0, 1, 2, 1, 1, 3, 1], [1] * 8)):
        _step(jev, cc, rng, np.array(new, np.int32), Lp, Hq, Hkv, d, k_pre, v_pre, f"decode step {s}")


def test_decode_step_at_the_wide_shape(jev):
    """One decode step of 128 branches (one token each) over a 4096-token
    prefix and caches of U[8, 40] tokens, at 7B heads, compared on every row."""
    cfg = synth.CONFIGS["wide_7b"]
    c = synth.flat_case(cfg, with_lm_head=False)
    rng = np.random.default_rng(77)
    Ls = np.diff(c.cu_seqlens).astype(np.int32)
    cc = _Caches(Ls + 1, cfg.Hkv, cfg.d)
    # the caches hold the branches' suffixes, filled by a prefill on both sides
    ref_o, ref_l, krot = oracle.cache_attn(c.q, c.k_suf, c.v_suf, c.k_pre, c.v_pre, cc.k_o, cc.v_o, cc.co, cc.len,
                                           c.cu_seqlens)
    out, lse = jev.jev_suffix_cache_attn(dev(c.q), dev(c.k_suf), dev(c.v_suf), dev(c.k_pre), dev(c.v_pre), cc.k_g,
                                         cc.v_g, dev(cc.co), dev(cc.len), dev(c.cu_seqlens))
    torch.cuda.synchronize()
    rows = np.concatenate([cc.co[b] + np.arange(Ls[b]) for b in range(cfg.B)]).astype(np.int64)
    check_attn(host_f64(out), host_f64(lse), ref_o, ref_l, synth.BF16, "wide prefill")
    cc.k_o[rows] = _bf16(krot)
    cc.v_o[rows] = c.v_suf
    cc.len += Ls
    _step(jev, cc, rng, np.ones(cfg.B, np.int32), cfg.Lp, cfg.Hq, cfg.Hkv, cfg.d, c.k_pre, c.v_pre, "wide decode")


def test_a_branch_beyond_its_cache_rows_is_flagged_and_left_alone(jev):
    rng = np.random.default_rng(5)
    Lp, Hq, Hkv, d = 200, 8, 2, 128
    cap = np.array([4, 3, 5], np.int32)
    co = np.concatenate([[0], np.cumsum(cap)]).astype(np.int32)
    cl = np.array([2, 2, 0], np.int32)
    new = np.array([2, 2, 3], np.int32)  # branch 1 needs 4 rows but owns 3
    cu = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
    T = int(cu[-1])
    mk = lambda *s: _bf16(rng.standard_normal(s))
    q, kn, vn, kp, vp = mk(T, Hq, d), mk(T, Hkv, d), mk(T, Hkv, d), mk(Lp, Hkv, d), mk(Lp, Hkv, d)
    kc, vc = mk(int(co[-1]), Hkv, d), mk(int(co[-1]), Hkv, d)
    kc_g, vc_g = dev(kc), dev(vc)
    desc = jev.make_attn_desc(3, Lp, Hq, Hkv, d, T, jev.JEV_BF16)
    ws = jev.new_workspace(jev.jev_suffix_cache_attn_workspace(desc), "cuda")
    out = torch.full((T, Hq, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    jev.jev_suffix_cache_attn(dev(q), dev(kn), dev(vn), dev(kp), dev(vp), kc_g, vc_g, dev(co), dev(cl), dev(cu),
                              out=out, workspace=ws)
    assert jev.jev_check_device_status(ws) & jev.JEV_DEV_BAD_CACHE
    o = host_f64(out)
    assert np.isnan(o[cu[1]:cu[2]]).all()  # the overflowing branch's rows are untouched
    kg = kc_g.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(kg[co[1]:co[2]], kc[co[1]:co[2]])  # and so are its cache rows
    # the other branches are computed
    ok = [0, 2]
    sel = np.concatenate([np.arange(cu[b], cu[b + 1]) for b in ok])
    cl2, new2 = cl[ok], new[ok]
    co2 = np.concatenate([[0], np.cumsum(cap[ok])]).astype(np.int32)
    cu2 = np.concatenate([[0], np.cumsum(new2)]).astype(np.int32)
    kc2 = np.concatenate([kc[co[b]:co[b + 1]] for b in ok])
    vc2 = np.concatenate([vc[co[b]:co[b + 1]] for b in ok])
    ref_o, ref_l, _ = oracle.cache_attn(q[sel], kn[sel], vn[sel], kp, vp, kc2, vc2, co2, cl2, cu2)
    np.testing.assert_array_less(np.abs(o[sel] - ref_o), TOL[synth.BF16]["max_abs"])
