"""Race check of the one-Q-tile tensor-core attention kernel's mbarrier protocol (attn_tc1.cu), on the CPU.

A model of the roles in attn_tc1.cu, each a sequence of barrier operations per
segment of n key tiles (global key-tile index JJ):
  * producer: the first segment's leading K and V tiles first (into stages not
    used before), then per segment: wait q_empty of the previous segment, two
    arrivals on q_full (expect-tx and the published descriptor), then the
    segment's key tiles with K one tile ahead of V: K(JJ) into K stage
    JJ % NK after a wait on that stage's k_empty, V(JJ - 1) into V stage
    (JJ - 1) % NV after a wait on v_empty;
  * MMA warp: wait q_full, K(J), issue S(J) into score buffer J % 2; per key
    tile j: first S(JJ + 1) into the other buffer (commit s_full of that
    buffer and k_empty), then wait V(JJ) and p_full of buffer JJ % 2, issue
    PV(JJ) and commit pv_done and v_empty; q_empty after the p_full wait of
    tile max(0, n - 2) (the rule under test: by then the segment's last S is
    issued and every softmax thread has passed its q_full wait);
  * softmax threads (four here, two per row group, standing for the 512
    threads: four per row, one per quarter of its score columns): wait q_full
    and agree on it at the group barrier; per key tile wait s_full of buffer
    JJ % 2, meet the row's other quarters at the exchange barrier, wait
    pv_done of tile JJ - 1 only when the row maximum moved (O is rescaled;
    modelled as a coin flip), arrive on p_full of the buffer; wait o_full
    (committed after the segment's last PV) and meet at the group barrier
    before the epilogue.  pv_done cannot serve there: s_full of the last tile
    only shows PV of the tile before the previous one complete, so a parity
    wait for the last PV could pass a phase early (the checker shows it).
MMA commits and TMA completions are modelled as immediate (one possible
timing).  A wait follows the hardware rule for parity waits (it passes when
the barrier's completed-phase count has the other parity), and the checker
flags any waiter whose barrier has completed two phases past the one it
waits for (its parity then names a pending phase and it stalls), and any
wait that would pass on parity while the phase before the awaited one is
still pending (it would return early).
Random interleavings, biased so that one thread lags, explore the timings.
The asynchronous model with timeouts and the wait machinery are shared with
the two-Q-tile kernel's model (test_pipeline_protocol.py).
"""
import random

import sys

import pytest

from test_pipeline_protocol import Bar, _async_run, _wait_problem

NK, NV = 3, 2  # K and V ring stages at d = 128
SOFT = 4  # softmax threads in the model: row groups 0 and 1, two quarters each


def _prefetch(segs, prefetch):
    """K and V tiles loaded before anything else: the first segment's leading
    tiles, one per stage of each ring."""
    return (min(segs[0], NK), min(segs[0], NV)) if prefetch else (0, 0)


def _loads(segs, prefetch):
    """The producer's load order: per segment the Q tile (after q_empty of the
    previous one), then K one key tile ahead of V.  Yields ("q", k) and
    ("k" | "v", JJ)."""
    pk, pv = _prefetch(segs, prefetch)
    for j in range(pk):
        yield ("k", j)
    for j in range(pv):
        yield ("v", j)
    kn, vn, J = pk, pv, 0
    for k, n in enumerate(segs):
        yield ("q", k)
        for j in range(n):
            while kn <= J + j:
                yield ("k", kn)
                kn += 1
            while j >= 1 and vn <= J + j - 1:
                yield ("v", vn)
                vn += 1
        while vn <= J + n - 1:
            yield ("v", vn)
            vn += 1
        J += n


def producer(segs, prefetch=False):
    for kind, x in _loads(segs, prefetch):
        if kind == "q":
            if x > 0:
                yield ("wait", "q_empty", x - 1)
            yield ("arrive", "q_full")
            yield ("arrive", "q_full")
        elif kind == "k":
            if x >= NK:
                yield ("wait", f"k_empty{x % NK}", x // NK - 1)
            yield ("arrive", f"k_full{x % NK}")
        else:
            if x >= NV:
                yield ("wait", f"v_empty{x % NV}", x // NV - 1)
            yield ("arrive", f"v_full{x % NV}")


def mma(segs, early_release):
    J = 0
    for k, n in enumerate(segs):
        yield ("wait", "q_full", k)
        yield ("wait", f"k_full{J % NK}", J // NK)
        yield ("arrive", f"s_full{J % 2}")
        yield ("arrive", f"k_empty{J % NK}")
        if early_release and n == 1:
            yield ("arrive", "q_empty")  # released right after the segment's last S, before any softmax acknowledgement
        for j in range(n):
            JJ = J + j
            if j + 1 < n:
                yield ("wait", f"k_full{(JJ + 1) % NK}", (JJ + 1) // NK)
                yield ("arrive", f"s_full{(JJ + 1) % 2}")
                yield ("arrive", f"k_empty{(JJ + 1) % NK}")
                if early_release and j + 2 == n:
                    yield ("arrive", "q_empty")
            yield ("wait", f"v_full{JJ % NV}", JJ // NV)
            yield ("wait", f"p_full{JJ % 2}", JJ // 2)
            yield ("arrive", "pv_done")
            yield ("arrive", f"v_empty{JJ % NV}")
            if j == n - 1:
                yield ("arrive", "o_full")
            if not early_release and j == max(0, n - 2):
                yield ("arrive", "q_empty")
        J += n


def softmax(segs, t, rng, epilogue_bar="o_full"):
    J = 0
    for k, n in enumerate(segs):
        yield ("wait", "q_full", k)
        yield ("sync", "qa")  # the group agrees on the wait before reading the description
        for j in range(n):
            JJ = J + j
            yield ("wait", f"s_full{JJ % 2}", JJ // 2)
            yield ("sync", f"x{t // 2}")  # the quarters of a row exchange their maxima
            if j > 0 and rng.random() < 0.5:
                yield ("wait", "pv_done", JJ - 1)  # O is rescaled: PV(JJ - 1) has completed
            yield ("arrive", f"p_full{JJ % 2}")
        yield ("wait", epilogue_bar, J + n - 1 if epilogue_bar == "pv_done" else k)
        yield ("sync", "ep")
        J += n


def _bars():
    bars = {"q_full": Bar(2), "q_empty": Bar(1), "pv_done": Bar(1), "o_full": Bar(1), "drain": Bar(1)}
    for b in range(2):
        bars[f"s_full{b}"], bars[f"p_full{b}"] = Bar(1), Bar(SOFT)
    for s in range(NK):
        bars[f"k_full{s}"], bars[f"k_empty{s}"] = Bar(1), Bar(1)
    for s in range(NV):
        bars[f"v_full{s}"], bars[f"v_empty{s}"] = Bar(1), Bar(1)
    return bars


def _members(threads, grp):
    """The threads that meet at a named barrier: all softmax threads for the
    group barriers, the two of a row group for an exchange barrier."""
    soft = [m for m in threads if m.startswith("soft")]
    if grp.startswith("x"):
        return [m for m in soft if int(m[4:]) // 2 == int(grp[1:])]
    return soft


def run(segs, early_release, seed, prefetch=False, epilogue_bar="o_full"):
    """Returns None when every role finishes cleanly, else a description."""
    bars = _bars()
    rng = random.Random(seed)
    threads = {"producer": producer(segs, prefetch), "mma": mma(segs, early_release)}
    for t in range(SOFT):
        threads[f"soft{t}"] = softmax(segs, t, random.Random(seed * 31 + t), epilogue_bar)
    cur = {name: next(g, None) for name, g in threads.items()}
    lagger = rng.choice(sorted(threads))

    for name, op in cur.items():
        if _wait_problem(bars, name, op):
            return _wait_problem(bars, name, op)
    for _ in range(200000):
        live = [n for n, op in cur.items() if op is not None]
        if not live:
            return None
        runnable = []
        for n in live:
            op = cur[n]
            if op[0] == "arrive":
                runnable.append(n)
            elif op[0] == "wait":
                if (bars[op[1]].phase & 1) != (op[2] & 1):
                    runnable.append(n)
            else:  # named barrier: every member parked on it
                members = _members(threads, op[1])
                if all(cur[m] is not None and cur[m][0] == "sync" and cur[m][1] == op[1] for m in members):
                    runnable.append(n)
        if not runnable:
            return "deadlock: " + ", ".join(f"{n}@{cur[n]}" for n in live)
        weights = [0.05 if n == lagger else 1.0 for n in runnable]
        n = rng.choices(runnable, weights)[0]
        op = cur[n]
        if op[0] == "arrive":
            b = bars[op[1]]
            b.pending += 1
            if b.pending == b.count:
                b.pending = 0
                b.phase += 1
                for m, mop in cur.items():
                    msg = _wait_problem(bars, m, mop)
                    if msg:
                        return msg
            cur[n] = next(threads[n], None)
            moved = [n]
        elif op[0] == "wait":
            cur[n] = next(threads[n], None)
            moved = [n]
        else:
            moved = _members(threads, op[1])
            for m in moved:
                cur[m] = next(threads[m], None)
        for m in moved:
            msg = _wait_problem(bars, m, cur[m])
            if msg:
                return msg
    return "step limit"


# per-CTA segment patterns (key tiles per segment): single-tile segments between longer ones,
# as the one-unit tail segments and the short windows of long tree nodes produce
PATTERNS = [[17, 9], [17, 8, 1], [3, 1, 2], [1, 1, 1, 1], [2, 1, 1, 3], [4, 1, 4, 1], [1, 2], [5], [2, 2, 2]]


@pytest.mark.parametrize("prefetch", [False, True])
@pytest.mark.parametrize("segs", PATTERNS, ids=["-".join(map(str, p)) for p in PATTERNS])
def test_protocol_has_no_stall_or_aliased_wait(segs, prefetch):
    for seed in range(150):
        msg = run(segs, early_release=False, seed=seed, prefetch=prefetch)
        assert msg is None, f"seed {seed}: {msg}"


@pytest.mark.parametrize("segs", PATTERNS, ids=["-".join(map(str, p)) for p in PATTERNS])
def test_protocol_with_the_d64_rings(segs, monkeypatch):
    # at d = 64 the kernel keeps 6 K and 5 V stages: deeper rings, the same protocol,
    # on the normal path and on the timeout path
    monkeypatch.setattr(sys.modules[__name__], "NK", 6)
    monkeypatch.setattr(sys.modules[__name__], "NV", 5)
    for prefetch in (False, True):
        for seed in range(60):
            msg = run(segs, early_release=False, seed=seed, prefetch=prefetch)
            assert msg is None, f"seed {seed}: {msg}"
        order = list(_loads(segs, prefetch))
        assert [x for kind, x in order if kind == "k"] == list(range(sum(segs)))
        assert [x for kind, x in order if kind == "v"] == list(range(sum(segs)))
    for seed in range(60):
        msg = run_abort(segs, drain=True, seed=seed)
        assert msg is None, f"seed {seed}: {msg}"


def test_checker_finds_the_early_release_race():
    # releasing Q as soon as the segment's last S is issued lets q_full run two
    # phases ahead of a softmax thread that has not yet waited for it
    found = [run([3, 1, 3], early_release=True, seed=s) for s in range(300)]
    bad = [m for m in found if m is not None]
    assert bad, "the checker should catch the aliased q_full wait"
    assert any("q_full" in m for m in bad)


def test_checker_finds_the_early_pass_of_a_last_pv_wait():
    # waiting at the epilogue on pv_done for the segment's last PV can pass
    # while that PV (and the one before) is still running
    bad = [run([5, 4], early_release=False, seed=s, epilogue_bar="pv_done") for s in range(200)]
    bad = [m for m in bad if m is not None]
    assert bad and any("would pass" in m and "pv_done" in m for m in bad)


def test_producer_load_order():
    # K runs one key tile ahead of V inside a segment; every tile is loaded once, in order per ring
    for segs in PATTERNS:
        for prefetch in (False, True):
            order = list(_loads(segs, prefetch))
            ks = [x for kind, x in order if kind == "k"]
            vs = [x for kind, x in order if kind == "v"]
            assert ks == list(range(sum(segs))) and vs == list(range(sum(segs)))
            pos = {o: i for i, o in enumerate(order)}
            J = 0
            for k, n in enumerate(segs):
                for j in range(1, n):
                    assert pos[("k", J + j)] < pos[("v", J + j)]  # K(JJ) before V(JJ)
                J += n


# ---------------------------------------------------------------- the timeout path: nothing in flight at exit


def a_producer(segs, drain, prefetch=True):
    k_armed = v_armed = q_armed = 0  # tiles whose loads this warp has issued
    ok = True
    for kind, x in _loads(segs, prefetch):
        if kind == "q":
            if x > 0:
                ok = yield ("wait", "q_empty", x - 1, True)
                if not ok:
                    break
            yield ("tma", "q_full")
            q_armed += 1
            yield ("arrive", "q_full")  # the published segment description
        elif kind == "k":
            if x >= NK:
                ok = yield ("wait", f"k_empty{x % NK}", x // NK - 1, True)
                if not ok:
                    break
            yield ("tma", f"k_full{x % NK}")
            k_armed = x + 1
        else:
            if x >= NV:
                ok = yield ("wait", f"v_empty{x % NV}", x // NV - 1, True)
                if not ok:
                    break
            yield ("tma", f"v_full{x % NV}")
            v_armed = x + 1
    if drain:
        # the last phase of every stage it armed, and of the Q buffer, ignoring the flag
        for ring, ns, armed in (("k_full", NK, k_armed), ("v_full", NV, v_armed)):
            for s in range(ns):
                uses = (armed - s + ns - 1) // ns if armed > s else 0
                if uses:
                    yield ("wait", f"{ring}{s}", uses - 1, False)
        if q_armed:
            yield ("wait", "q_full", q_armed - 1, False)
    yield ("final",)


def a_mma(segs, drain, probe=False):
    J, ok = 0, True
    for k, n in enumerate(segs):
        if not ok:
            break
        ok = yield ("wait", "q_full", k, True)
        if ok:
            ok = yield ("wait", f"k_full{J % NK}", J // NK, True)
            if ok:
                yield ("mma",)
                yield ("commit", f"s_full{J % 2}")
                yield ("commit", f"k_empty{J % NK}")
            if ok and k == 0 and probe:
                # the failure-detection probe: a barrier that nothing completes
                ok = yield ("wait", "probe", 0, True)
        for j in range(n):
            if not ok:
                break
            JJ = J + j
            if j + 1 < n:
                ok = yield ("wait", f"k_full{(JJ + 1) % NK}", (JJ + 1) // NK, True)
                if not ok:
                    break
                yield ("mma",)
                yield ("commit", f"s_full{(JJ + 1) % 2}")
                yield ("commit", f"k_empty{(JJ + 1) % NK}")
            ok = yield ("wait", f"v_full{JJ % NV}", JJ // NV, True)
            if ok:
                ok = yield ("wait", f"p_full{JJ % 2}", JJ // 2, True)
            if not ok:
                break
            yield ("mma",)
            yield ("commit", "pv_done")
            yield ("commit", f"v_empty{JJ % NV}")
            if j == n - 1:
                yield ("commit", "o_full")
            if j == max(0, n - 2):
                yield ("commit", "q_empty")
        J += n
    yield ("commit", "drain")
    yield ("wait", "drain", 0, not drain)  # the drain rule ignores the flag
    yield ("final",)
    yield ("dealloc",)


def a_softmax(segs, t, rng):
    # the group agrees on the q_full wait before reading the segment; a failed
    # wait inside a segment does not leave it (the row group must meet the same
    # exchange barriers), the group leaves after its epilogue barrier
    J, ok = 0, True
    for k, n in enumerate(segs):
        w = yield ("wait", "q_full", k, True)
        ok = yield ("syncand", "qa", w)
        if not ok:
            break
        for j in range(n):
            JJ = J + j
            w = yield ("wait", f"s_full{JJ % 2}", JJ // 2, True)
            ok = ok and w
            yield ("sync", f"x{t // 2}")
            if j > 0 and rng.random() < 0.5:
                w = yield ("wait", "pv_done", JJ - 1, True)
                ok = ok and w
            yield ("arrive", f"p_full{JJ % 2}")
        if ok:
            ok = yield ("wait", "o_full", k, True)
        ok = yield ("syncand", "ep", ok)
        if not ok:
            break
        J += n
    yield ("final",)


def run_abort(segs, drain, seed, p_timeout=0.02, probe=False):
    bars = _bars()
    bars["probe"] = Bar(1)
    threads = {"producer": a_producer(segs, drain), "mma": a_mma(segs, drain, probe)}
    for t in range(SOFT):
        threads[f"soft{t}"] = a_softmax(segs, t, random.Random(seed * 17 + t))

    def group_of(op):
        if op[0] == "final":
            return list(threads)
        return _members(threads, op[1])
    return _async_run(threads, bars, group_of, seed, p_timeout)


ABORT_PATTERNS = [[5], [3, 2], [17, 9], [1, 1, 1], [4, 1, 4, 1], [2, 3]]


@pytest.mark.parametrize("segs", ABORT_PATTERNS, ids=["-".join(map(str, p)) for p in ABORT_PATTERNS])
def test_timeout_path_drains_before_exit(segs):
    for seed in range(300):
        msg = run_abort(segs, drain=True, seed=seed)
        assert msg is None, f"seed {seed}: {msg}"


@pytest.mark.parametrize("segs", ABORT_PATTERNS, ids=["-".join(map(str, p)) for p in ABORT_PATTERNS])
def test_probe_timeout_drains_before_exit(segs):
    for seed in range(200):
        msg = run_abort(segs, drain=True, seed=seed, p_timeout=0.05, probe=True)
        assert msg is None, f"seed {seed}: {msg}"


def test_timeout_path_without_drain_can_exit_with_work_in_flight():
    bad = [run_abort(s, drain=False, seed=seed) for s in ABORT_PATTERNS for seed in range(200)]
    bad = [m for m in bad if m is not None]
    assert bad and all("pending" in m for m in bad), bad[:3]


def test_normal_path_of_the_async_model_is_clean():
    # no timeout at all: both rules exit cleanly
    for segs in ABORT_PATTERNS:
        for seed in range(50):
            assert run_abort(segs, drain=True, seed=seed, p_timeout=0.0) is None
            assert run_abort(segs, drain=False, seed=seed, p_timeout=0.0) is None
