"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/jev.h declares, rejects bad arguments on the host before anything is
enqueued, and its host-side trie / readout planning matches the oracle bit
for bit."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def jev():
    import attention_cascade_b200 as m  # built by conftest
    return m


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(jev_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(jev):
    names = _declared()
    assert {"jev_prefix_suffix_attn", "jev_candidate_readout", "jev_tree_attn", "jev_tree_build"} <= names
    lib = C.CDLL(jev.LIB_PATH)
    missing = [n for n in sorted(names) if not hasattr(lib, n)]
    assert not missing, missing


def test_host_rejects_bad_arguments(jev):
    lib = jev._lib
    d = jev.make_attn_desc(2, 16, 4, 2, 96, 8, jev.JEV_BF16)
    assert lib.jev_prefix_suffix_attn(C.byref(d), *([None] * 10), 0, None) == 2  # d = 96 unsupported
    d = jev.make_attn_desc(2, 16, 6, 4, 64, 8, jev.JEV_BF16)
    assert lib.jev_prefix_suffix_attn(C.byref(d), *([None] * 10), 0, None) == 1  # Hq % Hkv
    d = jev.make_attn_desc(2, 16, 4, 2, 64, 8, jev.JEV_BF16)
    assert lib.jev_prefix_suffix_attn(C.byref(d), *([None] * 10), 0, None) == 1  # NULL q
    assert "NULL" in jev.jev_last_error()
    fake = 1 << 20  # never dereferenced: the workspace check fails first
    st = lib.jev_prefix_suffix_attn(C.byref(d), fake, fake, fake, fake, fake, fake, None, fake, None, fake, 64, None)
    assert st == 3 and "workspace" in jev.jev_last_error()
    st = lib.jev_prefix_suffix_attn(C.byref(d), fake + 2, fake, fake, fake, fake, fake, None, fake, None, fake, 1 << 30, None)
    assert st == 1 and "aligned" in jev.jev_last_error()
    d0 = jev.make_attn_desc(0, 16, 4, 2, 64, 0, jev.JEV_BF16)
    assert lib.jev_prefix_suffix_attn(C.byref(d0), *([None] * 10), 0, None) == 0  # empty: no work
    r = jev.jev_readout_desc(3, 5, 5, 3, 100, 1000, jev.JEV_BF16)  # H not a multiple of 8
    assert lib.jev_candidate_readout(C.byref(r), *([None] * 10)) == 2


def test_workspace_size_is_monotone(jev):
    small = jev.jev_prefix_suffix_attn_workspace(jev.make_attn_desc(4, 256, 2, 1, 64, 64, jev.JEV_F32))
    big = jev.jev_prefix_suffix_attn_workspace(jev.make_attn_desc(128, 4096, 28, 4, 128, 3072, jev.JEV_BF16))
    assert 256 < small < big
    # q_rot (bf16) for 3072 tokens x 28 heads x 128 fits in the wide workspace
    assert big >= 3072 * 28 * 128 * 2


def _csr(cands):
    so = np.concatenate([[0], np.cumsum([len(c) for c in cands])]).astype(np.int32)
    return so, np.array([t for c in cands for t in c], np.int32)


def test_tree_build_matches_oracle_bitwise(jev):
    rng = np.random.default_rng(7)
    for trial in range(300):
        n = int(rng.integers(1, 12))
        vocab = int(rng.integers(2, 6))
        cands = [list(rng.integers(0, vocab, int(rng.integers(0, 8)))) for _ in range(n)]
        so, toks = _csr(cands)
        root = int(rng.integers(0, 3000))
        a = jev.jev_tree_build(so, toks, root)
        b = oracle.trie_build(so, toks, root)
        for k in ("parent", "tok_off", "pos0", "leaf_of", "node_toks", "path_row"):
            assert np.array_equal(a[k], b[k]), (k, cands)
        assert a["n_nodes"] == b["n_nodes"]


def test_tree_build_on_tree_workload(jev):
    import synth
    tc = synth.tree_case(synth.CONFIGS["tree_7b"], with_lm_head=False)
    a = jev.jev_tree_build(tc.seq_off, tc.toks, tc.cfg.Lp)
    b = oracle.trie_build(tc.seq_off, tc.toks, tc.cfg.Lp)
    for k in ("parent", "tok_off", "pos0", "leaf_of", "node_toks", "path_row"):
        assert np.array_equal(a[k], b[k])
    assert a["tok_off"][-1] == tc.n_unique
    assert a["n_nodes"] == 1 + 16 + tc.seq_off.size - 1  # root + questions + one node per option
    plan = jev.jev_tree_readout_plan(tc.seq_off, tc.toks, tc.score_from, a["path_row"])
    co, prow, tix = oracle.tree_readout_pairs(tc.seq_off, tc.score_from, b["path_row"], tc.set_offsets)
    assert np.array_equal(plan["cand_offsets"], co)
    assert np.array_equal(plan["pair_row"], prow)
    assert np.array_equal(plan["pair_tok"], tc.toks[tix])



def test_tree_readout_plan_matches_hand_golden(jev):
    """The library's trie and readout plan reproduce the hand-derived pairs of
    a question with 1-, 2- and 3-token options (tests/golden/tree_readout.json)."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "tree_readout.json")) as f:
        g = json.load(f)
    so, toks = _csr(g["cands"])
    a = jev.jev_tree_build(so, toks, g["root_len"])
    pr = a["path_row"]
    assert [pr[so[c]:so[c + 1]].tolist() for c in range(len(g["cands"]))] == g["path_row"]
    plan = jev.jev_tree_readout_plan(so, toks, np.asarray(g["score_from"], np.int32), pr)
    assert plan["cand_offsets"].tolist() == g["cand_offsets"]
    assert plan["pair_row"].tolist() == g["pair_row"]
    assert plan["pair_tok"].tolist() == g["pair_tok"]

def test_tree_build_capacity_and_errors(jev):
    so, toks = _csr([[1, 2, 3], [1, 4]])
    lib = jev._lib
    parent = np.zeros(2, np.int32); tok_off = np.zeros(3, np.int32); pos0 = np.zeros(2, np.int32)
    leaf = np.zeros(2, np.int32); nt = np.zeros(8, np.int32); nn = C.c_int32()
    st = lib.jev_tree_build(2, so.ctypes.data, toks.ctypes.data, 0, 2, 8, parent.ctypes.data, tok_off.ctypes.data,
                            pos0.ctypes.data, leaf.ctypes.data, nt.ctypes.data, None, C.byref(nn))
    assert st == 6  # JEV_ERR_CAPACITY
    with pytest.raises(jev.JevError):
        jev.jev_tree_readout_plan(so, toks, np.array([0, 1], np.int32), np.zeros(5, np.int32))



def test_position_mode_is_checked_on_the_host(jev):
    """pos_mode is 0 (per-branch positions) or 1 (sequential, sink-block
    encoding); anything else, and sequential positions on the tree entry point,
    are rejected before anything is enqueued."""
    bad = jev.make_attn_desc(2, 128, 8, 2, 128, 10, jev.JEV_BF16, pos_mode=2)
    assert jev.jev_prefix_suffix_attn_workspace(bad) == 0
    with pytest.raises(jev.JevError):
        jev.jev_prefix_suffix_attn_plan(bad)
    n0 = jev.jev_launch_count()
    seq = jev.make_attn_desc(2, 128, 8, 2, 128, 10, jev.JEV_BF16, pos_mode=1)
    assert jev.jev_prefix_suffix_attn_workspace(seq) > 0
    st = jev._lib.jev_tree_attn(C.byref(seq), 3, *([C.c_void_p(16)] * 12), C.c_size_t(1 << 20), None)
    assert st == 1 and jev.jev_launch_count() == n0


def test_vocab_lse_host_checks(jev):
    lib = jev._lib
    # bf16 only, H a multiple of 64, sizes positive: rejected before any device query or launch
    assert lib.jev_vocab_lse(None, None, 4, 128, 100, jev.JEV_F32, None, None, 0, None) == 2
    assert lib.jev_vocab_lse(None, None, 4, 96, 100, jev.JEV_BF16, None, None, 0, None) == 2
    assert lib.jev_vocab_lse(None, None, -1, 128, 100, jev.JEV_BF16, None, None, 0, None) == 1
    assert lib.jev_vocab_lse(None, None, 4, 128, 0, jev.JEV_BF16, None, None, 0, None) == 1
    # workspace grows with the row count; the status word comes first
    w1, w2 = jev.jev_vocab_lse_workspace(1, 152064), jev.jev_vocab_lse_workspace(600, 152064)
    assert 256 < w1 < w2
    assert jev.jev_vocab_lse_workspace(-1, 10) == 0
    # the normalised readout runs the readout's own checks
    r = jev.jev_readout_desc(3, 5, 5, 3, 100, 1000, jev.JEV_BF16)
    assert lib.jev_candidate_readout_normalized(C.byref(r), *([None] * 11)) == 2


def test_header_is_plain_c_and_links(jev, tmp_path):
    """include/jev.h compiles as C99 with every warning on, and a C program links against the
    library and calls a host-only entry point through it."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    names = sorted(_declared())
    src = tmp_path / "abi.c"
    src.write_text("#include <stdio.h>\n#include \"jev.h\"\nint main(void) {\n"
                   "  void (*fns[])(void) = {" + ", ".join(f"(void (*)(void)){n}" for n in names) + "};\n"
                   "  printf(\"%d %zu\\n\", (int)(sizeof fns / sizeof fns[0]), jev_vocab_lse_workspace(256, 152064));\n"
                   "  return 0;\n}\n")
    exe = tmp_path / "abi"
    lib = jev.LIB_PATH
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
                        str(src), lib, "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    assert int(out[0]) == len(names) and int(out[1]) == jev.jev_vocab_lse_workspace(256, 152064)


def test_host_calls_are_reentrant_across_threads(jev):
    """The host-only entry points (trie build, readout plan, work plan) give the
    same answers when eight threads call them at once (ctypes releases the
    interpreter lock, so the calls overlap inside the library)."""
    from concurrent.futures import ThreadPoolExecutor
    rng = np.random.default_rng(12)
    problems = []
    for i in range(8):
        n = int(rng.integers(5, 40))
        lens = rng.integers(1, 9, n)
        seq_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        toks = rng.integers(0, 6, int(seq_off[-1])).astype(np.int32)
        problems.append((seq_off, toks))
    descs = [jev.make_attn_desc(8 + i, 256 * (i + 1), 28, 4, 128, 100 * (i + 1), jev.JEV_BF16) for i in range(8)]

    def work(i):
        seq_off, toks = problems[i]
        out = []
        for _ in range(30):
            t = jev.jev_tree_build(seq_off, toks, 16)
            score_from = np.ones(seq_off.size - 1, np.int32)
            p = jev.jev_tree_readout_plan(seq_off, toks, score_from, t["path_row"])
            plan = jev.jev_prefix_suffix_attn_plan(descs[i], 1, 148)
            out.append((t["parent"].tobytes(), t["tok_off"].tobytes(), p["pair_row"].tobytes(),
                        p["pair_tok"].tobytes(), tuple(sorted(plan.items()))))
        return out

    serial = [work(i)[0] for i in range(8)]
    with ThreadPoolExecutor(8) as ex:
        results = list(ex.map(work, range(8)))
    for i in range(8):
        assert all(r == serial[i] for r in results[i])
