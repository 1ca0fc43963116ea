"""Race check of the tensor-core attention kernel's mbarrier protocol, on the CPU.

A model of the roles in attn_tc.cu, each a sequence of barrier operations per
segment of n key tiles:
  * producer: the first segment's leading key tiles first (into stages not
    used before), then per segment: wait q_empty of the previous segment, two
    arrivals on q_full (expect-tx and the published descriptor), and per key
    tile its K and V into ring stage JJ % NS after a wait on that stage's
    kv_empty;
  * MMA warp: wait q_full, k_full, commit s_full of both tiles; per key tile
    wait v_full and p_full of each tile, commit o_full after the last PV,
    kv_empty after the tile's last PV, and q_empty after the segment's last S
    MMA (the rule under test);
  * softmax threads (two per tile here, standing for the 256 threads of a
    tile group: two per row, one per half of its score columns): wait q_full
    and agree on it at the group barrier, per key tile wait s_full, meet the
    other half of the row at the pair barrier and arrive on p_full; wait
    o_full and meet at the group barrier before the epilogue.
MMA commits and TMA completions are modelled as immediate (one possible
timing).  A wait follows the hardware rule for parity waits (it passes when
the barrier's completed-phase count has the other parity), and the checker
flags any waiter whose barrier has completed two phases past the one it
waits for: that waiter's parity then names a pending phase and it stalls.
Random interleavings, biased so that one thread lags, explore the timings.
The full-vocabulary LSE kernel (vocab_lse.cu: TMA ring, MMA warp, statistics
threads releasing the TMEM tile) is modelled the same way at the end.
"""
import random
import sys

import pytest

NS = 2  # K/V ring stages at d = 128


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, 0, 0


def _preload(segs, prefetch):
    """Key tiles loaded before anything else: the first segment's leading
    tiles, one per stage."""
    return min(segs[0], NS) if prefetch else 0


def producer(segs, prefetch=False):
    pre = _preload(segs, prefetch)
    for j in range(pre):
        yield ("arrive", f"k_full{j}")
        yield ("arrive", f"v_full{j}")
    J = 0
    for k, n in enumerate(segs):
        if k > 0:
            yield ("wait", "q_empty", k - 1)
        yield ("arrive", "q_full")
        yield ("arrive", "q_full")
        for j in range(pre if k == 0 else 0, n):
            JJ = J + j
            if JJ >= NS:
                yield ("wait", f"kv_empty{JJ % NS}", JJ // NS - 1)
            yield ("arrive", f"k_full{JJ % NS}")
            yield ("arrive", f"v_full{JJ % NS}")
        J += n


def mma(segs, early_release):
    J = 0
    for k, n in enumerate(segs):
        yield ("wait", "q_full", k)
        yield ("wait", f"k_full{J % NS}", J // NS)
        yield ("arrive", "s_full0")
        yield ("arrive", "s_full1")
        if early_release and n == 1:
            yield ("arrive", "q_empty")  # the earlier rule: released before any softmax acknowledgement
        for j in range(n):
            JJ = J + j
            yield ("wait", f"v_full{JJ % NS}", JJ // NS)
            yield ("wait", "p_full0", JJ)
            if j == n - 1:
                yield ("arrive", "o_full0")
            if j + 1 < n:
                yield ("wait", f"k_full{(JJ + 1) % NS}", (JJ + 1) // NS)
                yield ("arrive", "s_full0")
            yield ("wait", "p_full1", JJ)
            yield ("arrive", f"kv_empty{JJ % NS}")
            if j == n - 1:
                yield ("arrive", "o_full1")
            if j + 1 < n:
                yield ("arrive", "s_full1")
                if j + 2 == n:
                    yield ("arrive", "q_empty")
            elif n == 1 and not early_release:
                yield ("arrive", "q_empty")
        J += n


def softmax(segs, i):
    J = 0
    for k, n in enumerate(segs):
        yield ("wait", "q_full", k)
        yield ("sync", f"qa{i}")  # the group agrees on the wait before reading the description
        for j in range(n):
            JJ = J + j
            yield ("wait", f"s_full{i}", JJ)
            yield ("sync", f"pair{i}")  # the two halves of a row exchange their maxima
            yield ("arrive", f"p_full{i}")
        yield ("wait", f"o_full{i}", k)
        yield ("sync", f"ep{i}")
        yield ("sync", f"eq{i}")
        J += n


SOFT = 2  # softmax threads per tile group in the model


def run(segs, early_release, seed, prefetch=False):
    """Returns None when every role finishes cleanly, else a description."""
    bars = {"q_full": Bar(2), "q_empty": Bar(1), "s_full0": Bar(1), "s_full1": Bar(1),
            "p_full0": Bar(SOFT), "p_full1": Bar(SOFT), "o_full0": Bar(1), "o_full1": Bar(1)}
    for s in range(NS):
        bars[f"k_full{s}"], bars[f"v_full{s}"], bars[f"kv_empty{s}"] = Bar(1), Bar(1), Bar(1)
    threads = {"producer": producer(segs, prefetch), "mma": mma(segs, early_release)}
    for i in range(2):
        for t in range(SOFT):
            threads[f"soft{i}.{t}"] = softmax(segs, i)
    cur = {name: next(g, None) for name, g in threads.items()}
    rng = random.Random(seed)
    lagger = rng.choice(sorted(threads))

    def check_alias(name, op):
        if op and op[0] == "wait" and bars[op[1]].phase > op[2] + 1:
            return f"{name} waits for phase {op[2]} of {op[1]}, which has completed {bars[op[1]].phase}"
        return None

    for name, op in cur.items():
        if check_alias(name, op):
            return check_alias(name, op)
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
            else:  # group barrier: every member parked on it
                grp = op[1]
                members = [m for m in threads if m.startswith("soft" + grp[-1] + ".")]
                if all(cur[m] is not None and cur[m][0] == "sync" and cur[m][1] == grp for m in members):
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
                    msg = check_alias(m, mop)
                    if msg:
                        return msg
            cur[n] = next(threads[n], None)
        elif op[0] == "wait":
            cur[n] = next(threads[n], None)
        else:
            grp = op[1]
            members = [m for m in threads if m.startswith("soft" + grp[-1] + ".")]
            for m in members:
                cur[m] = next(threads[m], None)
        for m in ([n] if op[0] != "sync" else members):
            msg = check_alias(m, cur[m])
            if msg:
                return msg
    return "step limit"


# per-CTA segment patterns (key tiles per segment): single-tile segments between longer ones,
# as the one-unit tail segments and the short windows of long tree nodes produce
PATTERNS = [[17, 9], [17, 8, 1], [3, 1, 2], [1, 1, 1, 1], [2, 1, 1, 3], [4, 1, 4, 1], [1, 2], [5]]


@pytest.mark.parametrize("prefetch", [False, True])
@pytest.mark.parametrize("segs", PATTERNS, ids=["-".join(map(str, p)) for p in PATTERNS])
def test_protocol_has_no_stall_or_aliased_wait(segs, prefetch):
    for seed in range(150):
        msg = run(segs, early_release=False, seed=seed, prefetch=prefetch)
        assert msg is None, f"seed {seed}: {msg}"


@pytest.mark.parametrize("segs", PATTERNS, ids=["-".join(map(str, p)) for p in PATTERNS])
def test_protocol_with_the_d64_ring(segs, monkeypatch):
    # at d = 64 the kernel keeps 4 K/V stages: a deeper ring, the same protocol,
    # on the normal path and on the timeout path
    monkeypatch.setattr(sys.modules[__name__], "NS", 4)
    for prefetch in (False, True):
        for seed in range(60):
            msg = run(segs, early_release=False, seed=seed, prefetch=prefetch)
            assert msg is None, f"seed {seed}: {msg}"
    for seed in range(60):
        msg = run_abort(segs, drain=True, seed=seed)
        assert msg is None, f"seed {seed}: {msg}"


def test_checker_finds_the_early_release_race():
    # the earlier rule (q_empty committed right after a one-tile segment's S MMAs)
    # lets q_full run two phases ahead of a lagging softmax thread
    found = [run([3, 1, 3], early_release=True, seed=s) for s in range(300)]
    bad = [m for m in found if m is not None]
    assert bad, "the checker should catch the aliased q_full wait"
    assert any("q_full" in m for m in bad)


# ---------------------------------------------------------------- full-vocabulary LSE kernel (vocab_lse.cu)

LS = 3  # TMA ring stages


def lse_producer(tiles, nk):
    it = 0
    for _ in range(tiles):
        for _ in range(nk):
            st = it % LS
            if it >= LS:
                yield ("wait", f"empty{st}", it // LS - 1)
            yield ("arrive", f"full{st}")
            it += 1


def lse_mma(tiles, nk):
    it = 0
    for tile in range(tiles):
        if tile > 0:
            yield ("wait", "sempty", tile - 1)  # the statistics threads have read the previous tile
        for _ in range(nk):
            st = it % LS
            yield ("wait", f"full{st}", it // LS)
            yield ("arrive", f"empty{st}")
            it += 1
        yield ("arrive", "sfull")


def lse_stats(tiles):
    for tile in range(tiles):
        yield ("wait", "sfull", tile)
        yield ("arrive", "sempty")


def run_lse(tiles, nk, n_stats, seed):
    bars = {"sfull": Bar(1), "sempty": Bar(n_stats)}
    for s in range(LS):
        bars[f"full{s}"], bars[f"empty{s}"] = Bar(1), Bar(1)
    threads = {"producer": lse_producer(tiles, nk), "mma": lse_mma(tiles, nk)}
    for t in range(n_stats):
        threads[f"stats{t}"] = lse_stats(tiles)
    cur = {n: next(g, None) for n, g in threads.items()}
    rng = random.Random(seed)
    lagger = rng.choice(sorted(threads))
    for _ in range(100000):
        live = [n for n, op in cur.items() if op is not None]
        if not live:
            return None
        runnable = [n for n in live if cur[n][0] == "arrive" or (bars[cur[n][1]].phase & 1) != (cur[n][2] & 1)]
        if not runnable:
            return "deadlock: " + ", ".join(f"{n}@{cur[n]}" for n in live)
        n = rng.choices(runnable, [0.05 if m == lagger else 1.0 for m in runnable])[0]
        op = cur[n]
        if op[0] == "arrive":
            b = bars[op[1]]
            b.pending += 1
            if b.pending == b.count:
                b.pending, b.phase = 0, b.phase + 1
        cur[n] = next(threads[n], None)
        for m, mop in cur.items():
            if mop and mop[0] == "wait" and bars[mop[1]].phase > mop[2] + 1:
                return f"{m} waits for phase {mop[2]} of {mop[1]}, which has completed {bars[mop[1]].phase}"
    return "step limit"


@pytest.mark.parametrize("tiles,nk", [(1, 1), (5, 2), (4, 56), (9, 3)])
def test_lse_protocol_has_no_stall_or_aliased_wait(tiles, nk):
    for seed in range(100):
        assert run_lse(tiles, nk, 3, seed) is None


# ---------------------------------------------------------------- the timeout path: nothing in flight at exit
#
# A second model with the asynchronous parts made explicit.  TMA loads are
# in-flight items that arrive on their barrier when they land (in any order);
# tcgen05 MMAs and commits are a queue that the tensor core executes in order,
# a commit arriving on its barrier once every MMA before it has completed.  At
# some random moment a thread blocked on a wait times out: the CTA's abort
# flag is set, and from then on every wait that checks the flag and is not
# already satisfied returns false at once.  Each role then winds down the way
# the kernel does, meets the others at the final CTA barrier, and the MMA warp
# frees TMEM.  The check: when TMEM is freed and the CTA exits, no TMA load
# and no MMA or commit may still be pending (a load landing in the shared
# memory of an exited CTA, or an MMA writing freed TMEM, is what the drain
# exists to prevent).  Under the earlier rule (the producer leaves without
# waiting for its loads, the MMA warp's final drain wait gives up as soon as
# the flag is set) the check fails; under the drain rule it holds.


def a_producer(segs, drain, prefetch=True):
    pre = _preload(segs, prefetch)
    for j in range(pre):
        yield ("tma", f"k_full{j}")
        yield ("tma", f"v_full{j}")
    armed = pre  # key tiles whose K and V loads were issued
    J, q_armed, ok = 0, 0, True
    for k, n in enumerate(segs):
        if not ok:
            break
        if k > 0:
            ok = yield ("wait", "q_empty", k - 1, True)
            if not ok:
                break
        yield ("tma", "q_full")
        q_armed += 1
        yield ("arrive", "q_full")  # the published segment description
        for j in range(pre if k == 0 else 0, n):
            JJ = J + j
            if JJ >= NS:
                ok = yield ("wait", f"kv_empty{JJ % NS}", JJ // NS - 1, True)
                if not ok:
                    break
            yield ("tma", f"k_full{JJ % NS}")
            yield ("tma", f"v_full{JJ % NS}")
            armed = JJ + 1
        J += n
    if drain:
        # the last phase of every stage it armed, and of the Q buffer, ignoring the flag
        for s in range(NS):
            uses = (armed - s + NS - 1) // NS if armed > s else 0
            if uses:
                yield ("wait", f"k_full{s}", uses - 1, False)
                yield ("wait", f"v_full{s}", uses - 1, False)
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
            ok = yield ("wait", f"k_full{J % NS}", J // NS, True)
            if ok:
                for i in range(2):
                    yield ("mma",)
                    yield ("commit", f"s_full{i}")
        if ok and k == 0 and probe:
            # the failure-detection probe: a barrier that nothing completes,
            # waited on with the first MMAs in flight (only a timeout ends it)
            ok = yield ("wait", "probe", 0, True)
        for j in range(n):
            if not ok:
                break
            JJ = J + j
            ok = yield ("wait", f"v_full{JJ % NS}", JJ // NS, True)
            if ok:
                ok = yield ("wait", "p_full0", JJ, True)
            if not ok:
                break
            yield ("mma",)
            if j == n - 1:
                yield ("commit", "o_full0")
            if j + 1 < n:
                ok = yield ("wait", f"k_full{(JJ + 1) % NS}", (JJ + 1) // NS, True)
                if not ok:
                    break
                yield ("mma",)
                yield ("commit", "s_full0")
            ok = yield ("wait", "p_full1", JJ, True)
            if not ok:
                break
            yield ("mma",)
            yield ("commit", f"kv_empty{JJ % NS}")
            if j == n - 1:
                yield ("commit", "o_full1")
            if j + 1 < n:
                yield ("mma",)
                yield ("commit", "s_full1")
                if j + 2 == n:
                    yield ("commit", "q_empty")
            elif n == 1:
                yield ("commit", "q_empty")
        J += n
    yield ("commit", "drain")
    yield ("wait", "drain", 0, not drain)  # the drain rule ignores the flag
    yield ("final",)
    yield ("dealloc",)


def a_softmax(segs, i):
    # the tile group agrees on the q_full wait before reading the segment; a
    # failed wait inside a segment does not leave it (the group must meet the
    # same pair and group barriers), the group leaves after its epilogue barrier
    J, ok = 0, True
    for k, n in enumerate(segs):
        w = yield ("wait", "q_full", k, True)
        ok = yield ("syncand", f"qa{i}", w)
        if not ok:
            break
        for j in range(n):
            w = yield ("wait", f"s_full{i}", J + j, True)
            ok = ok and w
            yield ("sync", f"pair{i}")
            yield ("arrive", f"p_full{i}")
        if ok:
            ok = yield ("wait", f"o_full{i}", k, True)
        ok = yield ("syncand", f"ep{i}", ok)
        yield ("sync", f"eq{i}")
        if not ok:
            break
        J += n
    yield ("final",)


def _wait_problem(bars, name, op):
    """A parity wait that would stall (its barrier has completed two phases past
    the awaited one) or pass early (the phase before the awaited one is still
    pending), else None."""
    if not op or op[0] != "wait":
        return None
    done = bars[op[1]].phase
    if done > op[2] + 1:
        return f"{name} waits for phase {op[2]} of {op[1]}, which has completed {done}"
    if done < op[2] and (done & 1) != (op[2] & 1):
        return f"{name} would pass its wait for phase {op[2]} of {op[1]} with only {done} completed"
    return None


def _async_run(threads, bars, group_of, seed, p_timeout):
    """Random interleaving of roles, in-flight TMA loads and the tensor-core
    queue, with at most one timeout; None when the CTA exits with nothing in
    flight, else a description."""
    cur = {name: next(g) for name, g in threads.items()}
    tma, tc_queue = [], []  # loads in flight (barrier names); MMA / commit queue
    rng = random.Random(seed)
    state = {"abort": False}

    def arrive(name):
        b = bars[name]
        b.pending += 1
        if b.pending == b.count:
            b.pending, b.phase = 0, b.phase + 1

    def ready(op):
        return (bars[op[1]].phase & 1) != (op[2] & 1)

    def advance(n, value=None):
        try:
            cur[n] = threads[n].send(value)
        except StopIteration:
            cur[n] = None

    for _ in range(400000):
        live = [n for n, op in cur.items() if op is not None]
        if not live:
            return None
        moves = []
        for n in live:
            op = cur[n]
            if op[0] in ("arrive", "tma", "mma", "commit", "dealloc"):
                moves.append(("run", n))
            elif op[0] == "wait":
                if ready(op) or (op[3] and state["abort"]):
                    moves.append(("run", n))
                elif op[3] and not state["abort"] and rng.random() < p_timeout:
                    moves.append(("timeout", n))
            elif all(cur[m] is not None and cur[m][:2] == op[:2] for m in group_of(op)):
                moves.append(("run", n))
        if tma:
            moves.append(("tma_done", None))
        if tc_queue:
            moves.append(("tc_step", None))
        if not moves and p_timeout > 0:
            # nothing can move until time passes: a bounded wait runs out
            # (with timeouts off, a stall here is reported as a deadlock)
            moves = [("timeout", n) for n in live
                     if cur[n][0] == "wait" and cur[n][3] and not state["abort"]]
        if not moves:
            return "deadlock: " + ", ".join(f"{n}@{cur[n]}" for n in live)
        kind, n = rng.choice(moves)
        if kind == "tma_done":
            arrive(tma.pop(rng.randrange(len(tma))))
            continue
        if kind == "tc_step":
            item = tc_queue.pop(0)
            if item[0] == "commit":
                arrive(item[1])
            continue
        op = cur[n]
        if kind == "timeout":
            state["abort"] = True
            advance(n, False)
            continue
        if op[0] == "arrive":
            arrive(op[1])
            advance(n)
        elif op[0] == "tma":
            tma.append(op[1])
            advance(n)
        elif op[0] in ("mma", "commit"):
            tc_queue.append(op)
            advance(n)
        elif op[0] == "dealloc":
            if tma or tc_queue:
                return f"TMEM freed and CTA exiting with {len(tma)} loads and {len(tc_queue)} tensor-core ops pending"
            advance(n)
        elif op[0] == "wait":
            # once the CTA is winding down, an abortable wait that passes early
            # is harmless (the segment's results are dropped); a drain wait is not
            if ready(op) and not (op[3] and state["abort"]):
                msg = _wait_problem(bars, n, op)
                if msg:
                    return msg
            advance(n, ready(op))
        else:  # sync / syncand / final: release the whole group together
            members = group_of(op)
            val = all(cur[m][2] for m in members) if op[0] == "syncand" else None
            for m in members:
                advance(m, val)
    return "step limit"


def run_abort(segs, drain, seed, p_timeout=0.02, probe=False):
    bars = {"q_full": Bar(2), "q_empty": Bar(1), "s_full0": Bar(1), "s_full1": Bar(1), "drain": Bar(1),
            "p_full0": Bar(SOFT), "p_full1": Bar(SOFT), "o_full0": Bar(1), "o_full1": Bar(1), "probe": Bar(1)}
    for s in range(NS):
        bars[f"k_full{s}"], bars[f"v_full{s}"], bars[f"kv_empty{s}"] = Bar(1), Bar(1), Bar(1)
    threads = {"producer": a_producer(segs, drain), "mma": a_mma(segs, drain, probe)}
    for i in range(2):
        for t in range(SOFT):
            threads[f"soft{i}.{t}"] = a_softmax(segs, i)

    def group_of(op):
        if op[0] == "final":
            return list(threads)
        return [m for m in threads if m.startswith("soft" + op[1][-1] + ".")]
    return _async_run(threads, bars, group_of, seed, p_timeout)


ABORT_PATTERNS = [[5], [3, 2], [17, 9], [1, 1, 1], [4, 1, 4, 1], [2, 3]]


@pytest.mark.parametrize("segs", ABORT_PATTERNS, ids=["-".join(map(str, p)) for p in ABORT_PATTERNS])
def test_timeout_path_drains_before_exit(segs):
    for seed in range(300):
        msg = run_abort(segs, drain=True, seed=seed)
        assert msg is None, f"seed {seed}: {msg}"


@pytest.mark.parametrize("segs", ABORT_PATTERNS, ids=["-".join(map(str, p)) for p in ABORT_PATTERNS])
def test_probe_timeout_drains_before_exit(segs):
    # with the probe on, the run always ends in a timeout (nothing completes
    # the probe's barrier); the CTA must still exit with nothing in flight
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


# the full-vocabulary LSE kernel's roles with the same asynchronous parts and timeout


def a_lse_producer(tiles, nk, drain):
    it, ok = 0, True
    for _ in range(tiles):
        for _ in range(nk):
            st = it % LS
            if it >= LS:
                ok = yield ("wait", f"empty{st}", it // LS - 1, True)
                if not ok:
                    break
            yield ("tma", f"full{st}")
            it += 1
        if not ok:
            break
    if drain:
        for s in range(LS):
            uses = (it - s + LS - 1) // LS if it > s else 0
            if uses:
                yield ("wait", f"full{s}", uses - 1, False)
    yield ("final",)


def a_lse_mma(tiles, nk, drain):
    it, ok = 0, True
    for tile in range(tiles):
        if tile > 0:
            ok = yield ("wait", "sempty", tile - 1, True)
            if not ok:
                break
        for _ in range(nk):
            st = it % LS
            ok = yield ("wait", f"full{st}", it // LS, True)
            if not ok:
                break
            yield ("mma",)
            yield ("commit", f"empty{st}")
            it += 1
        if not ok:
            break
        yield ("commit", "sfull")
    yield ("commit", "drain")
    yield ("wait", "drain", 0, not drain)
    yield ("final",)
    yield ("dealloc",)


def a_lse_stats(tiles):
    for tile in range(tiles):
        yield ("wait", "sfull", tile, True)
        yield ("arrive", "sempty")
    yield ("final",)


def run_lse_abort(tiles, nk, n_stats, drain, seed, p_timeout=0.02):
    bars = {"sfull": Bar(1), "sempty": Bar(n_stats), "drain": Bar(1)}
    for s in range(LS):
        bars[f"full{s}"], bars[f"empty{s}"] = Bar(1), Bar(1)
    threads = {"producer": a_lse_producer(tiles, nk, drain), "mma": a_lse_mma(tiles, nk, drain)}
    for t in range(n_stats):
        threads[f"stats{t}"] = a_lse_stats(tiles)
    return _async_run(threads, bars, lambda op: list(threads), seed, p_timeout)


@pytest.mark.parametrize("tiles,nk", [(1, 1), (5, 2), (4, 7), (9, 3)])
def test_lse_timeout_path_drains_before_exit(tiles, nk):
    for seed in range(300):
        msg = run_lse_abort(tiles, nk, 3, drain=True, seed=seed)
        assert msg is None, f"seed {seed}: {msg}"


def test_lse_timeout_path_without_drain_can_exit_with_work_in_flight():
    bad = [run_lse_abort(t, k, 3, drain=False, seed=seed) for t, k in [(5, 2), (4, 7)] for seed in range(300)]
    bad = [m for m in bad if m is not None]
    assert bad and all("pending" in m for m in bad), bad[:3]
    for seed in range(50):  # no timeout: both rules exit cleanly
        assert run_lse_abort(4, 7, 3, drain=False, seed=seed, p_timeout=0.0) is None
