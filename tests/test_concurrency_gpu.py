"""The library is reentrant (include/jev.h: all work on the caller's stream,
scratch in the caller's workspace): four host threads, each with its own
stream and workspace, run attention and readout calls on different problems
at the same time, and every result equals, bit for bit, the same call run
alone."""
import threading

import pytest
import torch

import synth
from gpu_helpers import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def jev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import attention_cascade_b200 as m
    return m


def _problem(i):
    cfg = synth.FlatConfig(f"conc{i}", synth.BF16, 512 * (i + 1), 6 + 3 * i, 4, 30, 28, 4, 128, 256, 4096, 2, 5,
                           seed=40 + i)
    c = synth.flat_case(cfg)
    return {k: dev(v) for k, v in dict(q=c.q, kp=c.k_pre, vp=c.v_pre, ks=c.k_suf, vs=c.v_suf, cu=c.cu_seqlens,
                                        h=c.hidden, W=c.W, so=c.set_offsets, pt=c.pair_tok).items()}, cfg, c.T


def test_threads_with_own_streams_and_workspaces_match_serial_calls(jev):
    probs = [_problem(i) for i in range(4)]
    ctx = []
    for p, cfg, T in probs:
        desc = jev.make_attn_desc(cfg.B, cfg.Lp, cfg.Hq, cfg.Hkv, cfg.d, T, jev.JEV_BF16)
        ctx.append(dict(ws=jev.new_workspace(jev.jev_prefix_suffix_attn_workspace(desc), "cuda"),
                        stream=torch.cuda.Stream()))

    def call(i):
        p, s = probs[i][0], ctx[i]["stream"]
        with torch.cuda.stream(s):
            o, l = jev.jev_prefix_suffix_attn(p["q"], p["kp"], p["vp"], p["ks"], p["vs"], p["cu"],
                                              workspace=ctx[i]["ws"], stream=s)
            lp, ch = jev.jev_candidate_readout(p["h"], p["W"], p["so"], p["pt"], stream=s)
        s.synchronize()
        return o.clone(), l.clone(), lp.clone(), ch.clone()

    ref = [call(i) for i in range(4)]
    torch.cuda.synchronize()
    errors, results = [], {}

    def worker(i):
        try:
            results[i] = [call(i) for _ in range(10)]
        except Exception as e:  # noqa: BLE001 (reported below)
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(4)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for i in range(4):
        for o, l, lp, ch in results[i]:
            assert torch.equal(o, ref[i][0]) and torch.equal(l, ref[i][1])
            assert torch.equal(lp, ref[i][2]) and torch.equal(ch, ref[i][3])
        assert jev.jev_check_device_status(ctx[i]["ws"]) == 0
