"""fp64 CPU oracle for shared-prefix attention, candidate readout and the trie.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA path in ``attention_cascade_b200`` never imports it, and
the two share no code; their only common dependency is the seeded input
generator in ``synth``.

Each function wraps one C routine of ``oracle.c`` (plain C, fp64, OpenMP over
independent rows) and follows the passage cited in ``oracle.h``.

Parity status: every routine here is pinned by ``tests/test_oracle_pins.py``
against hand-derived closed forms, textbook special cases checked through an
independent library routine (PyTorch's fp64 scaled-dot-product attention, a
numpy matrix product), invariants, and brute force on tiny tries.  The one
unpinned aspect is whether the RoPE variant, theta and the multi-token leaf
rule are the ones the models on the pages use; no page prints weights or
logits that could decide it.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "oracle.h"))):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off", "-Wall", "-Wno-unused-variable",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _AttnProblem(C.Structure):
    _fields_ = [("B", C.c_int), ("Lp", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int), ("d", C.c_int),
                ("dtype", C.c_int), ("theta", C.c_double), ("scale", C.c_double), ("pos_offset", C.c_int),
                ("q", C.c_void_p), ("k_pre", C.c_void_p), ("v_pre", C.c_void_p), ("k_suf", C.c_void_p),
                ("v_suf", C.c_void_p), ("cu_seqlens", C.c_void_p), ("head_map", C.c_void_p),
                ("n_rows", C.c_int), ("rows", C.c_void_p), ("n_threads", C.c_int)]


class _CacheProblem(C.Structure):
    _fields_ = [("B", C.c_int), ("Lp", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int), ("d", C.c_int),
                ("dtype", C.c_int), ("theta", C.c_double), ("scale", C.c_double), ("pos_offset", C.c_int),
                ("q", C.c_void_p), ("k_new", C.c_void_p), ("v_new", C.c_void_p), ("k_pre", C.c_void_p),
                ("v_pre", C.c_void_p), ("k_cache", C.c_void_p), ("v_cache", C.c_void_p),
                ("cache_off", C.c_void_p), ("cache_len", C.c_void_p), ("cu_new", C.c_void_p),
                ("head_map", C.c_void_p), ("n_threads", C.c_int)]


class _ReadoutProblem(C.Structure):
    _fields_ = [("n_sets", C.c_int), ("n_cands", C.c_int), ("n_pairs", C.c_int), ("R", C.c_int),
                ("H", C.c_int), ("V", C.c_int), ("dtype", C.c_int), ("hidden", C.c_void_p),
                ("lm_head", C.c_void_p), ("set_offsets", C.c_void_p), ("cand_offsets", C.c_void_p),
                ("pair_row", C.c_void_p), ("pair_tok", C.c_void_p), ("full_vocab", C.c_int),
                ("n_threads", C.c_int)]


class _TreeProblem(C.Structure):
    _fields_ = [("n_nodes", C.c_int), ("N", C.c_int), ("Lp", C.c_int), ("Hq", C.c_int), ("Hkv", C.c_int),
                ("d", C.c_int), ("dtype", C.c_int), ("theta", C.c_double), ("scale", C.c_double),
                ("parent", C.c_void_p), ("tok_off", C.c_void_p), ("q", C.c_void_p), ("k", C.c_void_p),
                ("v", C.c_void_p), ("k_root", C.c_void_p), ("v_root", C.c_void_p), ("head_map", C.c_void_p),
                ("n_threads", C.c_int)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.oracle_rope.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_double, C.c_double]
        _lib.oracle_attend.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                                       C.c_double, C.c_void_p, C.c_void_p]
        _lib.oracle_prefix_suffix_attn.argtypes = [C.POINTER(_AttnProblem), C.c_void_p, C.c_void_p]
        _lib.oracle_prefix_suffix_attn.restype = C.c_int
        _lib.oracle_cache_attn.argtypes = [C.POINTER(_CacheProblem), C.c_void_p, C.c_void_p, C.c_void_p]
        _lib.oracle_cache_attn.restype = C.c_int
        _lib.oracle_candidate_readout.argtypes = [C.POINTER(_ReadoutProblem)] + [C.c_void_p] * 5
        _lib.oracle_candidate_readout.restype = C.c_int
        _lib.oracle_trie_build.argtypes = [C.c_int, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int] + [C.c_void_p] * 6
        _lib.oracle_trie_build.restype = C.c_int
        _lib.oracle_tree_attn.argtypes = [C.POINTER(_TreeProblem), C.c_void_p, C.c_void_p]
        _lib.oracle_tree_attn.restype = C.c_int
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _dtype_of(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle inputs are bf16 bit patterns (uint16) or float32, got {a.dtype}")


def _c(a, dt=None):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dt) if dt is not None else np.ascontiguousarray(a)


def rope(x: np.ndarray, pos: float, theta: float) -> np.ndarray:
    """Rotate-half RoPE of one float64 vector at position ``pos``."""
    x = _c(x, np.float64)
    y = np.empty_like(x)
    lib().oracle_rope(_ptr(x), _ptr(y), x.size, float(pos), float(theta))
    return y


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """softmax(scale q K^T) V over explicit float64 keys; returns (o, lse)."""
    q = _c(q, np.float64); K = _c(K, np.float64); V = _c(V, np.float64)
    n, d = K.shape
    o = np.empty(d, np.float64)
    l = C.c_double()
    lib().oracle_attend(_ptr(q), _ptr(K), _ptr(V), n, d, d, float(scale), _ptr(o), C.addressof(l))
    return o, l.value


def prefix_suffix_attn(q, k_pre, v_pre, k_suf, v_suf, cu_seqlens, *, theta=1e4, scale=0.0,
                       pos_offset=-1, head_map=None, rows: Optional[np.ndarray] = None, n_threads=0):
    """Unshared per-branch attention; returns (out, lse) as float64.

    With ``rows`` (an [n, 2] array of (token, q-head)), only those rows are
    formed and ``out`` is [n, d], ``lse`` [n]; otherwise [T, Hq, d] and [T, Hq].
    """
    q, k_pre, v_pre, k_suf, v_suf = (_c(a) for a in (q, k_pre, v_pre, k_suf, v_suf))
    dt = _dtype_of(q)
    for a in (k_pre, v_pre, k_suf, v_suf):
        assert _dtype_of(a) == dt
    cu = _c(cu_seqlens, np.int32)
    hm = _c(head_map, np.int32)
    T, Hq, d = q.shape
    Lp, Hkv, _ = k_pre.shape
    B = cu.size - 1
    rr = _c(rows, np.int32) if rows is not None else None
    if rr is not None:
        out = np.zeros((rr.shape[0], d), np.float64)
        lse = np.zeros(rr.shape[0], np.float64)
    else:
        out = np.zeros((T, Hq, d), np.float64)
        lse = np.zeros((T, Hq), np.float64)
    pr = _AttnProblem(B, Lp, Hq, Hkv, d, dt, float(theta), float(scale), int(pos_offset),
                      _ptr(q), _ptr(k_pre), _ptr(v_pre), _ptr(k_suf), _ptr(v_suf), _ptr(cu), _ptr(hm),
                      0 if rr is None else rr.shape[0], _ptr(rr), int(n_threads))
    rc = lib().oracle_prefix_suffix_attn(C.byref(pr), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_prefix_suffix_attn: bad arguments")
    return out, lse


def cache_attn(q, k_new, v_new, k_pre, v_pre, k_cache, v_cache, cache_off, cache_len, cu_new, *, theta=1e4,
               scale=0.0, pos_offset=-1, head_map=None, n_threads=0):
    """A generation step over per-branch suffix caches, unshared; returns
    (out [T, Hq, d], lse [T, Hq], k_new_rot [T, Hkv, d]) as float64, the last
    being the rotated new keys the step appends to the cache."""
    q, k_new, v_new, k_pre, v_pre, k_cache, v_cache = (_c(a) for a in (q, k_new, v_new, k_pre, v_pre, k_cache,
                                                                       v_cache))
    dt = _dtype_of(q)
    for a in (k_new, v_new, k_pre, v_pre, k_cache, v_cache):
        assert _dtype_of(a) == dt
    co, cl, cu, hm = (_c(a, np.int32) for a in (cache_off, cache_len, cu_new, head_map))
    T, Hq, d = q.shape
    Lp, Hkv, _ = k_pre.shape
    out = np.zeros((T, Hq, d), np.float64)
    lse = np.full((T, Hq), -np.inf, np.float64)
    krot = np.zeros((T, Hkv, d), np.float64)
    pr = _CacheProblem(cu.size - 1, Lp, Hq, Hkv, d, dt, float(theta), float(scale), int(pos_offset),
                       _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pre), _ptr(v_pre), _ptr(k_cache), _ptr(v_cache),
                       _ptr(co), _ptr(cl), _ptr(cu), _ptr(hm), int(n_threads))
    if lib().oracle_cache_attn(C.byref(pr), _ptr(out), _ptr(lse), _ptr(krot)) != 0:
        raise ValueError("oracle_cache_attn: bad arguments")
    return out, lse, krot


def candidate_readout(hidden, lm_head, set_offsets, pair_tok, *, cand_offsets=None, pair_row=None,
                      full_vocab=True, n_threads=0):
    """Readout over option sets; returns a dict of float64/int32 arrays and the
    count of invalid (row, token) pairs."""
    hidden = _c(hidden); W = _c(lm_head)
    dt = _dtype_of(hidden)
    assert _dtype_of(W) == dt
    so = _c(set_offsets, np.int32); pt = _c(pair_tok, np.int32)
    co = _c(cand_offsets, np.int32); prw = _c(pair_row, np.int32)
    R, H = hidden.shape
    V = W.shape[0]
    n_sets = so.size - 1
    n_cands = int(so[-1])
    n_pairs = pt.size
    score = np.zeros(n_cands, np.float64); lp = np.zeros(n_cands, np.float64)
    choice = np.zeros(n_sets, np.int32); gap = np.zeros(n_sets, np.float64)
    row_lse = np.zeros(R, np.float64)
    pr = _ReadoutProblem(n_sets, n_cands, n_pairs, R, H, V, dt, _ptr(hidden), _ptr(W), _ptr(so), _ptr(co),
                         _ptr(prw), _ptr(pt), int(bool(full_vocab)), int(n_threads))
    bad = lib().oracle_candidate_readout(C.byref(pr), _ptr(score), _ptr(lp), _ptr(choice), _ptr(gap), _ptr(row_lse))
    if bad < 0:
        raise ValueError("oracle_candidate_readout: bad arguments")
    return dict(score=score, logprob=lp, choice=choice, gap=gap, row_lse=row_lse, n_invalid=bad)


def vocab_lse(hidden, lm_head, n_threads=0):
    """Full-vocabulary log-sum-exp of every hidden row, lse[r] = log sum_v
    exp(hidden[r] . lm_head[v]), in fp64: the normaliser of a log-probability
    over the whole vocabulary ("How to Deploy Visual Jev ...", Step 3 takes
    its logits from the full LM-head projection).  Every row is made a used
    row of a one-candidate readout so the full-vocab pass computes its LSE."""
    hidden = _c(hidden)
    R = hidden.shape[0]
    so = np.arange(R + 1, dtype=np.int32)
    toks = np.zeros(R, np.int32)
    return candidate_readout(hidden, lm_head, so, toks, n_threads=n_threads)["row_lse"]


def sequence_logprob(hidden, lm_head, cand_offsets, pair_row, pair_tok, n_threads=0):
    """Normalised score of multi-token candidates: the sum over a candidate's
    teacher-forced (row, token) pairs of the full-vocabulary log-probability
    hidden[row] . lm_head[tok] - lse[row].  Returns float64 [n_cands]."""
    co = _c(cand_offsets, np.int32); prw = _c(pair_row, np.int32); pt = _c(pair_tok, np.int32)
    n_cands = co.size - 1
    so = np.array([0, n_cands], np.int32)  # one set: the scores do not depend on the grouping
    r = candidate_readout(hidden, lm_head, so, pt, cand_offsets=co, pair_row=prw, n_threads=n_threads)
    lse = r["row_lse"]
    out = r["score"].copy()
    for c in range(n_cands):
        for k in range(int(co[c]), int(co[c + 1])):
            out[c] -= lse[prw[k]]
    return out


def trie_build(seq_off, toks, root_len: int):
    """Canonical compressed trie; returns a dict of int32 arrays."""
    so = _c(seq_off, np.int32); tk = _c(toks, np.int32)
    n_cands = so.size - 1
    total = int(so[-1])
    cap_nodes = total + 1
    parent = np.zeros(cap_nodes, np.int32); tok_off = np.zeros(cap_nodes + 1, np.int32)
    pos0 = np.zeros(cap_nodes, np.int32); leaf_of = np.zeros(max(n_cands, 1), np.int32)
    node_toks = np.zeros(max(total, 1), np.int32); path_row = np.zeros(max(total, 1), np.int32)
    n = lib().oracle_trie_build(n_cands, _ptr(so), _ptr(tk), int(root_len), cap_nodes, max(total, 1),
                                _ptr(parent), _ptr(tok_off), _ptr(pos0), _ptr(leaf_of), _ptr(node_toks),
                                _ptr(path_row))
    if n < 0:
        raise ValueError("oracle_trie_build: bad input")
    N = int(tok_off[n])
    return dict(n_nodes=n, parent=parent[:n].copy(), tok_off=tok_off[:n + 1].copy(), pos0=pos0[:n].copy(),
                leaf_of=leaf_of[:n_cands].copy(), node_toks=node_toks[:N].copy(), path_row=path_row[:total].copy())


def tree_readout_pairs(seq_off, score_from, path_row, set_offsets):
    """Teacher-forced (row, token) pairs of each candidate: the option token i
    is scored from the hidden state of the token before it on the candidate's
    own path.  Returns (cand_offsets, pair_row, pair_tok_index) where the last
    indexes into the candidates' token array."""
    so = np.asarray(seq_off, np.int64); sf = np.asarray(score_from, np.int64)
    pr = np.asarray(path_row, np.int64)
    co = [0]; rows = []; tix = []
    for c in range(so.size - 1):
        a, e = int(so[c]), int(so[c + 1])
        s = a + int(sf[c])
        if s <= a:
            raise ValueError("score_from must be >= 1 (the first scored token needs a predecessor)")
        for i in range(s, e):
            rows.append(int(pr[i - 1]))
            tix.append(i)
        co.append(len(rows))
    return np.asarray(co, np.int32), np.asarray(rows, np.int32), np.asarray(tix, np.int64)


def sink_block_attn(q, k, v, k_sink, v_sink, cu_seqlens, *, theta=1e4, scale=0.0, head_map=None):
    """Sink-block parallel encoding ("PEVLM: Parallel Encoding for Vision-
    Language Models", abstract: context blocks share a sink block, position
    embeddings stay sequential), read plainly: block b is one branch over the
    sink cache whose first token sits at position len(sink) + cu_seqlens[b],
    the position it has in the unsplit sequence.  Each block is evaluated as
    its own single-branch problem; returns (out, lse) as float64."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    S = k_sink.shape[0]
    T, Hq, d = q.shape
    out = np.zeros((T, Hq, d), np.float64)
    lse = np.zeros((T, Hq), np.float64)
    for b in range(cu.size - 1):
        a, e = int(cu[b]), int(cu[b + 1])
        if e == a:
            continue
        ob, lb = prefix_suffix_attn(q[a:e], k_sink, v_sink, k[a:e], v[a:e], np.array([0, e - a], np.int32),
                                    theta=theta, scale=scale, pos_offset=S + a, head_map=head_map)
        out[a:e], lse[a:e] = ob, lb
    return out, lse


def tree_attn(trie, q, k, v, k_root, v_root, *, theta=1e4, scale=0.0, head_map=None, n_threads=0):
    """Tree attention by flattening every root->node path; (out, lse) float64."""
    q, k, v, k_root, v_root = (_c(a) for a in (q, k, v, k_root, v_root))
    dt = _dtype_of(q)
    N, Hq, d = q.shape
    Lp, Hkv, _ = k_root.shape
    parent = _c(trie["parent"], np.int32); tok_off = _c(trie["tok_off"], np.int32)
    hm = _c(head_map, np.int32)
    out = np.zeros((N, Hq, d), np.float64); lse = np.zeros((N, Hq), np.float64)
    pr = _TreeProblem(int(trie["n_nodes"]), N, Lp, Hq, Hkv, d, dt, float(theta), float(scale),
                      _ptr(parent), _ptr(tok_off), _ptr(q), _ptr(k), _ptr(v), _ptr(k_root), _ptr(v_root),
                      _ptr(hm), int(n_threads))
    rc = lib().oracle_tree_attn(C.byref(pr), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_tree_attn: bad arguments")
    return out, lse
