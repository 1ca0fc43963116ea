"""Race check of the tensor-core attention kernel's mbarrier protocol, on the CPU.

A model of the roles in attn_tc.cu, each a sequence of barrier operations per
segment of n key tiles:
  * producer: wait q_empty of the previous segment, two arrivals on q_full
    (expect-tx and the published descriptor), then per key tile wait kv_empty
    of the stage's previous use and arrive on k_full / v_full;
  * MMA warp: wait q_full, k_full, commit s_full of both tiles; per key tile
    wait v_full and p_full of each tile, commit o_full after the last PV,
    commit kv_empty, and commit q_empty after the segment's last S MMA (the
    rule under test);
  * softmax threads (two per tile group here, standing for the 256 that
    p_full counts): wait q_full, per key tile wait s_full and arrive on
    p_full, with a pair barrier per tile; wait o_full and two group barriers
    in the epilogue.
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

import pytest

NS = 2  # K/V stages at d = 128


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, 0, 0


def producer(segs, pre0=0):
    # pre0: the first segment's leading prefix tiles, loaded into stages 0 .. pre0-1 before
    # anything else (before the kernel's wait on the previous launch and before the first Q)
    for j in range(pre0):
        yield ("arrive", f"k_full{j}")
        yield ("arrive", f"v_full{j}")
    J = 0
    for k, n in enumerate(segs):
        if k > 0:
            yield ("wait", "q_empty", k - 1)
        yield ("arrive", "q_full")
        yield ("arrive", "q_full")
        for j in range(pre0 if k == 0 else 0, n):
            JJ = J + j
            st = JJ % NS
            if JJ >= NS:
                yield ("wait", f"kv_empty{st}", JJ // NS - 1)
            yield ("arrive", f"k_full{st}")
            yield ("arrive", f"v_full{st}")
        J += n


def mma(segs, early_release):
    J = 0
    for k, n in enumerate(segs):
        yield ("wait", "q_full", k)
        st0 = J % NS
        yield ("wait", f"k_full{st0}", J // NS)
        yield ("arrive", "s_full0")
        yield ("arrive", "s_full1")
        if early_release and n == 1:
            yield ("arrive", "q_empty")  # the earlier rule: released before any softmax acknowledgement
        for j in range(n):
            JJ = J + j
            st, st1 = JJ % NS, (JJ + 1) % NS
            yield ("wait", f"v_full{st}", JJ // NS)
            yield ("wait", "p_full0", JJ)
            if j == n - 1:
                yield ("arrive", "o_full0")
            if j + 1 < n:
                yield ("wait", f"k_full{st1}", (JJ + 1) // NS)
                yield ("arrive", "s_full0")
            yield ("wait", "p_full1", JJ)
            yield ("arrive", f"kv_empty{st}")
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
        for j in range(n):
            JJ = J + j
            yield ("wait", f"s_full{i}", JJ)
            yield ("sync", f"pair{i}")
            yield ("arrive", f"p_full{i}")
        yield ("wait", f"o_full{i}", k)
        yield ("sync", f"grp{i}")
        yield ("sync", f"grp{i}")
        J += n


SOFT = 2  # softmax threads per tile group in the model


def run(segs, early_release, seed, pre0=0):
    """Returns None when every role finishes cleanly, else a description."""
    bars = {"q_full": Bar(2), "q_empty": Bar(1), "s_full0": Bar(1), "s_full1": Bar(1),
            "p_full0": Bar(SOFT), "p_full1": Bar(SOFT), "o_full0": Bar(1), "o_full1": Bar(1)}
    for s in range(NS):
        for b in ("k_full", "v_full", "kv_empty"):
            bars[f"{b}{s}"] = Bar(1)
    threads = {"producer": producer(segs, pre0), "mma": mma(segs, early_release)}
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
    pre0 = min(segs[0], NS) if prefetch else 0  # a first segment of prefix tiles
    for seed in range(150):
        msg = run(segs, early_release=False, seed=seed, pre0=pre0)
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
