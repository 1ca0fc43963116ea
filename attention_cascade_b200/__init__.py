"""Python binding of libjev.so (include/jev.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  Tensors are
torch CUDA tensors (PyTorch supplies device memory and the current stream);
all computation happens in the library's CUDA kernels.  If the library has not
been built this module raises at import time: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjev.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python attention_cascade_b200/_build.py` "
                      "(nvcc, sm_100a) — there is no non-CUDA fallback")

_lib = C.CDLL(LIB_PATH)

JEV_F32, JEV_BF16 = 0, 1
JEV_DEV_BAD_SEQLENS, JEV_DEV_BAD_HEAD_MAP, JEV_DEV_BAD_TREE, JEV_DEV_WAIT_TIMEOUT, JEV_DEV_BAD_WINDOW = 1, 2, 4, 8, 16
JEV_DEV_BAD_CACHE = 32
STATUS_NAMES = {0: "JEV_OK", 1: "JEV_ERR_INVALID_ARG", 2: "JEV_ERR_UNSUPPORTED", 3: "JEV_ERR_WORKSPACE",
                4: "JEV_ERR_CUDA", 5: "JEV_ERR_DEVICE", 6: "JEV_ERR_CAPACITY"}


class JevError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.jev_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")


class jev_attn_desc(C.Structure):
    _fields_ = [("B", C.c_int32), ("Lp", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("d", C.c_int32),
                ("T_total", C.c_int32), ("dtype", C.c_int32), ("rope_theta", C.c_float),
                ("softmax_scale", C.c_float), ("pos_offset", C.c_int32), ("num_splits", C.c_int32),
                ("pos_mode", C.c_int32)]


class jev_attn_plan(C.Structure):
    _fields_ = [("kernel", C.c_int32), ("n_tiles", C.c_int32), ("units_per_tile", C.c_int32), ("n_ctas", C.c_int32),
                ("full_waves", C.c_int32), ("tail0", C.c_int32), ("tail_ctas", C.c_int32), ("split", C.c_int32),
                ("tail_units", C.c_int64), ("simt_splits", C.c_int32), ("split_len", C.c_int32),
                ("tile_rows", C.c_int32)]


class jev_readout_desc(C.Structure):
    _fields_ = [("n_sets", C.c_int32), ("n_cands", C.c_int32), ("n_pairs", C.c_int32), ("R", C.c_int32),
                ("H", C.c_int32), ("V", C.c_int32), ("dtype", C.c_int32)]


_vp, _i32, _sz = C.c_void_p, C.c_int32, C.c_size_t
_lib.jev_last_error.restype = C.c_char_p
_lib.jev_prefix_suffix_attn_workspace.argtypes = [C.POINTER(jev_attn_desc)]
_lib.jev_prefix_suffix_attn_workspace.restype = _sz
_lib.jev_prefix_suffix_attn_plan.argtypes = [C.POINTER(jev_attn_desc), _i32, _i32, C.POINTER(jev_attn_plan)]
_lib.jev_prefix_suffix_attn.argtypes = [C.POINTER(jev_attn_desc)] + [_vp] * 10 + [_sz, _vp]
_lib.jev_candidate_readout.argtypes = [C.POINTER(jev_readout_desc)] + [_vp] * 10
_lib.jev_candidate_readout_normalized.argtypes = [C.POINTER(jev_readout_desc)] + [_vp] * 11
_lib.jev_tree_build.argtypes = [_i32, _vp, _vp, _i32, _i32, _i32] + [_vp] * 7
_lib.jev_tree_readout_plan.argtypes = [_i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp]
_lib.jev_tree_attn_workspace.argtypes = [C.POINTER(jev_attn_desc), _i32]
_lib.jev_tree_attn_workspace.restype = _sz
_lib.jev_tree_attn.argtypes = [C.POINTER(jev_attn_desc), _i32] + [_vp] * 12 + [_sz, _vp]
_lib.jev_rope_inplace.argtypes = [_vp, _i32, _i32, _i32, _i32, C.c_float, _i32, _vp]
_lib.jev_workspace_init.argtypes = [_vp, _sz, _vp]
_lib.jev_check_device_status.argtypes = [_vp, _sz, _vp, C.POINTER(_i32)]
_lib.jev_profile_enable.argtypes = [_i32]
_lib.jev_profile_read.argtypes = [_i32, C.c_char_p, _vp, _vp, _i32]
_lib.jev_profile_read.restype = _i32
_lib.jev_launch_count.restype = C.c_int64
_lib.jev_vocab_lse_workspace.argtypes = [_i32, _i32]
_lib.jev_vocab_lse_workspace.restype = _sz
_lib.jev_vocab_lse.argtypes = [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _sz, _vp]
for _f in ("jev_prefix_suffix_attn", "jev_prefix_suffix_attn_plan", "jev_candidate_readout", "jev_tree_build",
           "jev_tree_readout_plan", "jev_tree_attn", "jev_rope_inplace", "jev_workspace_init", "jev_check_device_status",
           "jev_profile_enable", "jev_vocab_lse", "jev_candidate_readout_normalized"):
    getattr(_lib, _f).restype = C.c_int


def _check(st: int, where: str):
    if st != 0:
        raise JevError(st, where)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return JEV_BF16
    if t.dtype == torch.float32:
        return JEV_F32
    raise TypeError(f"jev: tensors must be bfloat16 or float32, got {t.dtype}")


def _dev(t: Optional[torch.Tensor], name: str, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"jev: {name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"jev: {name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"jev: {name} must be {dtype}, got {t.dtype}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def make_attn_desc(B, Lp, Hq, Hkv, d, T_total, dtype_code, rope_theta=1e4, softmax_scale=0.0, pos_offset=-1,
                   num_splits=0, pos_mode=0) -> jev_attn_desc:
    return jev_attn_desc(int(B), int(Lp), int(Hq), int(Hkv), int(d), int(T_total), int(dtype_code),
                         float(rope_theta), float(softmax_scale), int(pos_offset), int(num_splits), int(pos_mode))


# descriptors of recent calls, reused as they are (the library only reads them)
_desc_cache: dict = {}


def _cached_desc(maker, key):
    d = _desc_cache.get(key)
    if d is None:
        if len(_desc_cache) > 1024:
            _desc_cache.clear()
        d = _desc_cache[key] = maker(*key)
    return d


def jev_prefix_suffix_attn_workspace(desc: jev_attn_desc) -> int:
    return int(_lib.jev_prefix_suffix_attn_workspace(C.byref(desc)))


def jev_prefix_suffix_attn_plan(desc: jev_attn_desc, kernel: int = -1, num_sms: int = 0) -> dict:
    """The work plan for `desc` as a dict (host only; see include/jev.h)."""
    p = jev_attn_plan()
    _check(_lib.jev_prefix_suffix_attn_plan(C.byref(desc), int(kernel), int(num_sms), C.byref(p)),
           "jev_prefix_suffix_attn_plan")
    return {f: int(getattr(p, f)) for f, _ in jev_attn_plan._fields_}


def new_workspace(nbytes: int, device, stream=None) -> torch.Tensor:
    """A zeroed byte buffer usable as a jev workspace (256-byte aligned by torch)."""
    ws = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def jev_prefix_suffix_attn(q, k_pre, v_pre, k_suf, v_suf, cu_seqlens, *, head_map=None, out=None, lse=None,
                           workspace=None, rope_theta=1e4, softmax_scale=0.0, pos_offset=-1, num_splits=0,
                           T_total: Optional[int] = None, want_lse=True, stream=None, pos_mode=0):
    """Shared-prefix attention for B ragged suffix branches; returns (out, lse)."""
    dt = _dtype_code(q)
    T, Hq, d = q.shape
    Lp, Hkv = k_pre.shape[0], k_pre.shape[1]
    for t, n in ((q, "q"), (k_pre, "k_pre"), (v_pre, "v_pre"), (k_suf, "k_suf"), (v_suf, "v_suf")):
        _dev(t, n, q.dtype)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    _dev(head_map, "head_map", torch.int32)
    B = cu_seqlens.numel() - 1
    desc = _cached_desc(make_attn_desc, (B, Lp, Hq, Hkv, d, T if T_total is None else T_total, dt, rope_theta,
                                         softmax_scale, pos_offset, num_splits, pos_mode))
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    _dev(out, "out", q.dtype)
    _dev(lse, "lse", torch.float32)
    if workspace is None:  # (a caller's workspace is size-checked by the library itself)
        workspace = new_workspace(jev_prefix_suffix_attn_workspace(desc), q.device)
    _check(_lib.jev_prefix_suffix_attn(C.byref(desc), _p(q), _p(k_pre), _p(v_pre), _p(k_suf), _p(v_suf),
                                       _p(cu_seqlens), _p(head_map), _p(out), _p(lse), _p(workspace),
                                       workspace.numel(), _stream(stream)), "jev_prefix_suffix_attn")
    return out, lse


_lib.jev_suffix_cache_attn_workspace.argtypes = [C.POINTER(jev_attn_desc)]
_lib.jev_suffix_cache_attn_workspace.restype = _sz
_lib.jev_suffix_cache_attn.argtypes = [C.POINTER(jev_attn_desc)] + [_vp] * 7 + [_i32] + [_vp] * 7 + [_sz, _vp]
_lib.jev_suffix_cache_attn.restype = C.c_int


def jev_suffix_cache_attn_workspace(desc: jev_attn_desc) -> int:
    return int(_lib.jev_suffix_cache_attn_workspace(C.byref(desc)))


def jev_suffix_cache_attn(q, k_new, v_new, k_pre, v_pre, k_cache, v_cache, cache_off, cache_len, cu_new, *,
                          head_map=None, out=None, lse=None, workspace=None, rope_theta=1e4, softmax_scale=0.0,
                          pos_offset=-1, num_splits=0, want_lse=True, stream=None):
    """New tokens of B branches over the shared prefix and each branch's cached
    suffix; appends their rotated keys and values to the caches (cache_len is
    not changed).  Returns (out, lse)."""
    dt = _dtype_code(q)
    T, Hq, d = q.shape
    Lp, Hkv = k_pre.shape[0], k_pre.shape[1]
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_pre, "k_pre"), (v_pre, "v_pre"),
                 (k_cache, "k_cache"), (v_cache, "v_cache")):
        _dev(t, n, q.dtype)
    for t, n in ((cache_off, "cache_off"), (cache_len, "cache_len"), (cu_new, "cu_new"), (head_map, "head_map")):
        _dev(t, n, torch.int32)
    B = cu_new.numel() - 1
    desc = _cached_desc(make_attn_desc, (B, Lp, Hq, Hkv, d, T, dt, rope_theta, softmax_scale, pos_offset,
                                         num_splits, 0))
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((T, Hq), dtype=torch.float32, device=q.device)
    _dev(out, "out", q.dtype)
    _dev(lse, "lse", torch.float32)
    if workspace is None:
        workspace = new_workspace(jev_suffix_cache_attn_workspace(desc), q.device)
    _check(_lib.jev_suffix_cache_attn(C.byref(desc), _p(q), _p(k_new), _p(v_new), _p(k_pre), _p(v_pre),
                                      _p(k_cache), _p(v_cache), int(k_cache.shape[0]), _p(cache_off),
                                      _p(cache_len), _p(cu_new), _p(head_map), _p(out), _p(lse), _p(workspace),
                                      workspace.numel(), _stream(stream)), "jev_suffix_cache_attn")
    return out, lse


JEV_NOALLOC_SCRATCH_BYTES = 32 << 20
_lib.jev_prefix_suffix_attn_noalloc.argtypes = [C.POINTER(jev_attn_desc)] + [_vp] * 11
_lib.jev_prefix_suffix_attn_noalloc.restype = C.c_int


def jev_prefix_suffix_attn_noalloc(q, k_pre, v_pre, k_suf, v_suf, cu_seqlens, out, lse=None, *, head_map=None,
                                   status_flags=None, rope_theta=1e4, softmax_scale=0.0, pos_offset=-1,
                                   num_splits=0, stream=None):
    """The attention of jev_prefix_suffix_attn for callers that cannot allocate
    device memory: the library's static scratch replaces the workspace, and the
    caller passes preallocated outputs.  Calls that overlap on the GPU race on
    that one scratch array."""
    dt = _dtype_code(q)
    T, Hq, d = q.shape
    Lp, Hkv = k_pre.shape[0], k_pre.shape[1]
    for t, n in ((q, "q"), (k_pre, "k_pre"), (v_pre, "v_pre"), (k_suf, "k_suf"), (v_suf, "v_suf"), (out, "out")):
        _dev(t, n, q.dtype)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    _dev(head_map, "head_map", torch.int32)
    _dev(lse, "lse", torch.float32)
    _dev(status_flags, "status_flags", torch.int32)
    desc = make_attn_desc(cu_seqlens.numel() - 1, Lp, Hq, Hkv, d, T, dt, rope_theta, softmax_scale, pos_offset,
                          num_splits)
    _check(_lib.jev_prefix_suffix_attn_noalloc(C.byref(desc), _p(q), _p(k_pre), _p(v_pre), _p(k_suf), _p(v_suf),
                                               _p(cu_seqlens), _p(head_map), _p(out), _p(lse), _p(status_flags),
                                               _stream(stream)), "jev_prefix_suffix_attn_noalloc")
    return out, lse


def jev_candidate_readout(hidden, lm_head, set_offsets, pair_tok, *, cand_offsets=None, pair_row=None,
                          logprob=None, choice=None, score=None, row_lse=None, stream=None):
    """Per-option log-probs and argmax over each option set; returns (logprob, choice).
    With row_lse (fp32 [R], from jev_vocab_lse) every pair's logit is
    normalised over the vocabulary first (jev_candidate_readout_normalized)."""
    dt = _dtype_code(hidden)
    _dev(hidden, "hidden", hidden.dtype)
    _dev(lm_head, "lm_head", hidden.dtype)
    for t, n in ((set_offsets, "set_offsets"), (pair_tok, "pair_tok"), (cand_offsets, "cand_offsets"),
                 (pair_row, "pair_row")):
        _dev(t, n, torch.int32)
    n_sets = set_offsets.numel() - 1
    n_cands = (cand_offsets.numel() - 1) if cand_offsets is not None else pair_tok.numel()
    desc = _cached_desc(jev_readout_desc, (n_sets, n_cands, pair_tok.numel(), hidden.shape[0], hidden.shape[1],
                                           lm_head.shape[0], dt))
    if logprob is None:
        logprob = torch.empty(n_cands, dtype=torch.float32, device=hidden.device)
    if choice is None:
        choice = torch.empty(n_sets, dtype=torch.int32, device=hidden.device)
    _dev(logprob, "logprob", torch.float32)
    _dev(choice, "choice", torch.int32)
    _dev(score, "score", torch.float32)
    if row_lse is None:
        _check(_lib.jev_candidate_readout(C.byref(desc), _p(hidden), _p(lm_head), _p(set_offsets), _p(cand_offsets),
                                          _p(pair_row), _p(pair_tok), _p(logprob), _p(choice), _p(score),
                                          _stream(stream)), "jev_candidate_readout")
    else:
        _dev(row_lse, "row_lse", torch.float32)
        _check(_lib.jev_candidate_readout_normalized(C.byref(desc), _p(hidden), _p(lm_head), _p(set_offsets),
                                                     _p(cand_offsets), _p(pair_row), _p(pair_tok), _p(row_lse),
                                                     _p(logprob), _p(choice), _p(score), _stream(stream)),
               "jev_candidate_readout_normalized")
    return logprob, choice


def jev_sequence_logprob(hidden, lm_head, cand_offsets, pair_row, pair_tok, *, lse=None, workspace=None,
                         stream=None):
    """Sequence log-probability of every multi-token candidate over the whole
    vocabulary: jev_vocab_lse of the hidden rows, then the normalised readout
    with all candidates in one set.  Returns fp32 [n_cands]."""
    lse = jev_vocab_lse(hidden, lm_head, lse=lse, workspace=workspace, stream=stream)
    n_cands = cand_offsets.numel() - 1
    so = torch.tensor([0, n_cands], dtype=torch.int32, device=hidden.device)
    score = torch.empty(n_cands, dtype=torch.float32, device=hidden.device)
    jev_candidate_readout(hidden, lm_head, so, pair_tok, cand_offsets=cand_offsets, pair_row=pair_row, score=score,
                          row_lse=lse, stream=stream)
    return score


def jev_vocab_lse_workspace(R: int, V: int) -> int:
    return int(_lib.jev_vocab_lse_workspace(R, V))


def jev_vocab_lse(hidden, lm_head, *, lse=None, workspace=None, stream=None):
    """Full-vocabulary log-sum-exp of every hidden row, lse [R] fp32."""
    dt = _dtype_code(hidden)
    _dev(hidden, "hidden", hidden.dtype)
    _dev(lm_head, "lm_head", hidden.dtype)
    R, H = hidden.shape
    V = lm_head.shape[0]
    if lse is None:
        lse = torch.empty(R, dtype=torch.float32, device=hidden.device)
    _dev(lse, "lse", torch.float32)
    if workspace is None:
        workspace = new_workspace(jev_vocab_lse_workspace(R, V), hidden.device)
    _check(_lib.jev_vocab_lse(_p(hidden), _p(lm_head), R, H, V, dt, _p(lse), _p(workspace), workspace.numel(),
                              _stream(stream)), "jev_vocab_lse")
    return lse


def jev_tree_build(seq_off: np.ndarray, toks: np.ndarray, root_len: int) -> dict:
    """Host trie build; returns numpy int32 arrays (parent, tok_off, pos0, leaf_of, node_toks, path_row)."""
    so = np.ascontiguousarray(seq_off, dtype=np.int32)
    tk = np.ascontiguousarray(toks, dtype=np.int32)
    n_cands = so.size - 1
    total = int(so[-1]) if so.size else 0
    cap = total + 1
    parent = np.zeros(cap, np.int32); tok_off = np.zeros(cap + 1, np.int32); pos0 = np.zeros(cap, np.int32)
    leaf_of = np.zeros(max(n_cands, 1), np.int32); node_toks = np.zeros(max(total, 1), np.int32)
    path_row = np.zeros(max(total, 1), np.int32)
    nn = C.c_int32()
    _check(_lib.jev_tree_build(n_cands, so.ctypes.data, tk.ctypes.data if tk.size else None, int(root_len), cap,
                               max(total, 1), parent.ctypes.data, tok_off.ctypes.data, pos0.ctypes.data,
                               leaf_of.ctypes.data, node_toks.ctypes.data, path_row.ctypes.data, C.byref(nn)),
           "jev_tree_build")
    n = nn.value
    N = int(tok_off[n])
    return dict(n_nodes=n, parent=parent[:n].copy(), tok_off=tok_off[:n + 1].copy(), pos0=pos0[:n].copy(),
                leaf_of=leaf_of[:n_cands].copy(), node_toks=node_toks[:N].copy(), path_row=path_row[:total].copy())


def jev_tree_readout_plan(seq_off, toks, score_from, path_row) -> dict:
    """Host teacher-forced readout pairs; returns numpy (cand_offsets, pair_row, pair_tok)."""
    so = np.ascontiguousarray(seq_off, dtype=np.int32); tk = np.ascontiguousarray(toks, dtype=np.int32)
    sf = np.ascontiguousarray(score_from, dtype=np.int32); pr = np.ascontiguousarray(path_row, dtype=np.int32)
    n_cands = so.size - 1
    cap = max(int(so[-1]), 1)
    co = np.zeros(n_cands + 1, np.int32); prow = np.zeros(cap, np.int32); ptok = np.zeros(cap, np.int32)
    n = C.c_int32()
    _check(_lib.jev_tree_readout_plan(n_cands, so.ctypes.data, tk.ctypes.data, sf.ctypes.data, pr.ctypes.data, cap,
                                      co.ctypes.data, prow.ctypes.data, ptok.ctypes.data, C.byref(n)),
           "jev_tree_readout_plan")
    return dict(cand_offsets=co, pair_row=prow[:n.value].copy(), pair_tok=ptok[:n.value].copy())


def jev_tree_attn_workspace(desc: jev_attn_desc, n_nodes: int) -> int:
    return int(_lib.jev_tree_attn_workspace(C.byref(desc), int(n_nodes)))


def jev_tree_attn(parent, tok_off, pos0, q, k_root, v_root, k, v, *, head_map=None, out=None, lse=None,
                  workspace=None, rope_theta=1e4, softmax_scale=0.0, num_splits=0, want_lse=True, stream=None):
    """Tree attention over packed trie tokens (device parent/tok_off/pos0); returns (out, lse)."""
    dt = _dtype_code(q)
    N, Hq, d = q.shape
    Lp, Hkv = k_root.shape[0], k_root.shape[1]
    for t, n in ((q, "q"), (k_root, "k_root"), (v_root, "v_root"), (k, "k"), (v, "v")):
        _dev(t, n, q.dtype)
    for t, n in ((parent, "parent"), (tok_off, "tok_off"), (pos0, "pos0"), (head_map, "head_map")):
        _dev(t, n, torch.int32)
    n_nodes = parent.numel()
    desc = _cached_desc(make_attn_desc, (n_nodes - 1, Lp, Hq, Hkv, d, N, dt, rope_theta, softmax_scale, -1,
                                         num_splits))
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((N, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:  # (a caller's workspace is size-checked by the library itself)
        workspace = new_workspace(jev_tree_attn_workspace(desc, n_nodes), q.device)
    _check(_lib.jev_tree_attn(C.byref(desc), n_nodes, _p(parent), _p(tok_off), _p(pos0), _p(q), _p(k_root),
                              _p(v_root), _p(k), _p(v), _p(head_map), _p(out), _p(lse), _p(workspace),
                              workspace.numel(), _stream(stream)), "jev_tree_attn")
    return out, lse


def jev_sink_block_attn(q, k_sink, v_sink, k, v, cu_seqlens, **kw):
    """Sink-block parallel encoding: each block of the packed input attends to
    the whole sink cache and to its own block up to itself; packed token t
    sits at position len(sink) + t, its position in the unsplit sequence
    (jev_prefix_suffix_attn with pos_mode 1); returns (out, lse)."""
    return jev_prefix_suffix_attn(q, k_sink, v_sink, k, v, cu_seqlens, pos_mode=1, **kw)


def jev_rope_inplace(x: torch.Tensor, pos0: int, theta: float = 1e4, stream=None) -> torch.Tensor:
    _dev(x, "x")
    L, H, d = x.shape
    _check(_lib.jev_rope_inplace(_p(x), L, H, d, int(pos0), float(theta), _dtype_code(x), _stream(stream)),
           "jev_rope_inplace")
    return x


_lib.jev_selftest_exp2.argtypes = [_vp, _vp, _i32, _vp]
_lib.jev_selftest_exp2.restype = C.c_int


def jev_selftest_exp2(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x through the attention kernel's FMA-pipe exponential (float32 CUDA tensor)."""
    _dev(x, "x", torch.float32)
    y = torch.empty_like(x)
    _check(_lib.jev_selftest_exp2(_p(x), _p(y), x.numel(), _stream(stream)), "jev_selftest_exp2")
    return y


def jev_workspace_init(workspace: torch.Tensor, stream=None):
    _check(_lib.jev_workspace_init(_p(workspace), workspace.numel(), _stream(stream)), "jev_workspace_init")


def jev_check_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise, read and clear the status word; returns its flag bits (0 = clean)."""
    f = C.c_int32()
    _lib.jev_check_device_status(_p(workspace), workspace.numel(), _stream(stream), C.byref(f))
    return f.value


def jev_last_error() -> str:
    return _lib.jev_last_error().decode(errors="replace")


def jev_profile_enable(on: bool = True):
    _lib.jev_profile_enable(int(bool(on)))


def jev_profile_read(keep: bool = False) -> dict:
    """{kernel name: (launches, total ms)} of the recorded launches.  With
    keep=True the records (and their events) stay registered, so launches
    captured in a CUDA graph can be read again after every replay."""
    cap = 64
    names = C.create_string_buffer(cap * 64)
    launches = np.zeros(cap, np.int32)
    ms = np.zeros(cap, np.float64)
    n = _lib.jev_profile_read(cap, names, launches.ctypes.data, ms.ctypes.data, int(bool(keep)))
    raw = names.raw
    return {raw[64 * i:64 * i + 64].split(b"\0", 1)[0].decode(): (int(launches[i]), float(ms[i])) for i in range(min(n, cap))}


def jev_launch_count() -> int:
    return int(_lib.jev_launch_count())


_lib.jev_debug_set_wait_limit.argtypes = [C.c_int64]
_lib.jev_debug_set_wait_limit.restype = C.c_int


def jev_debug_set_wait_limit(cycles: int):
    """Bound of the tensor-core kernels' mbarrier waits for later launches (0: the default)."""
    _check(_lib.jev_debug_set_wait_limit(int(cycles)), "jev_debug_set_wait_limit")


_lib.jev_debug_set_tc_tile_rows.argtypes = [C.c_int32]
_lib.jev_debug_set_tc_tile_rows.restype = C.c_int


def jev_debug_set_tc_tile_rows(rows: int):
    """Rows per tensor-core work tile for later plans: 128 or 256 forces a kernel, 0 lets the plan choose."""
    _check(_lib.jev_debug_set_tc_tile_rows(int(rows)), "jev_debug_set_tc_tile_rows")


_lib.jev_debug_set_wait_probe.argtypes = [C.c_int32]
_lib.jev_debug_set_wait_probe.restype = C.c_int


def jev_debug_set_wait_probe(on: bool):
    """Failure-detection probe for later launches: each CTA's MMA warp also waits on a barrier nothing completes."""
    _check(_lib.jev_debug_set_wait_probe(1 if on else 0), "jev_debug_set_wait_probe")
