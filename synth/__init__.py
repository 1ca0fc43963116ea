"""Seeded synthetic inputs for shared-prefix attention and candidate readout.

This module is the only code shared by the fp64 oracle (``oracle/``) and the
CUDA path (``attention_cascade_b200``).  It draws random numbers and lays them
out; it holds none of the method's arithmetic (no RoPE, no softmax, no dot
products).  Every tensor comes from its own PCG64 stream keyed by
``(seed, stream id[, chunk])`` so that any tensor, or any row block of the
LM-head weight, can be regenerated on its own.

Workload shapes follow the five synthetic configurations of the hot path:

* tiny_f32     tiny fp32   Lp=256,  B=4,   Ls=16,        Hq=2,  Hkv=1, d=64,  H=256,  V=1024,   3 options
* qwen2vl_2b   2B-shaped   Lp=1024, B=8,   Ls~U[8,24],   Hq=12, Hkv=2, d=128, H=1536, V=151936, U[3,9] options
* qwen25vl_7b  7B-shaped   Lp=2048, B=32,  Ls~U[12,32],  Hq=28, Hkv=4, d=128, H=3584, V=152064, U[2,3] options
* wide_7b      wide        Lp=4096, B=128, Ls~U[8,40],   Hq=28, Hkv=4, d=128, H=3584, V=152064, 3 options
* tree_7b      tree        root Lp=2048; 16 question nodes of 24 tokens, each with U[3,9]
                  option leaves of U[1,4] tokens (distinct first tokens among
                  siblings); Hq=28, Hkv=4, d=128; readout H=3584, V=152064.

Q, K, V and hidden states are N(0,1); the LM head is N(0, 0.02); option ids
are uniform without replacement in [0, V) per option set.  bf16 tensors are
rounded to nearest-even from an fp32 draw and returned as ``uint16`` bit
patterns; fp32 tensors are returned as ``float32``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

BF16 = "bf16"
F32 = "f32"

# stream ids: one independent PCG64 stream per tensor of a case
_S_Q, _S_KP, _S_VP, _S_KS, _S_VS, _S_LEN, _S_HID, _S_W, _S_OPT, _S_NOPT, _S_TREE = range(11)

W_CHUNK_ROWS = 4096  # LM-head rows per independently seeded block


def _rng(seed: int, stream: int, chunk: Optional[int] = None) -> np.random.Generator:
    key = [int(seed), int(stream)] if chunk is None else [int(seed), int(stream), int(chunk)]
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(key)))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); return uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(seed: int, stream: int, shape, std: float, dtype: str, chunk: Optional[int] = None) -> np.ndarray:
    x = _rng(seed, stream, chunk).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x) if dtype == BF16 else x


@dataclass
class FlatConfig:
    name: str
    dtype: str
    Lp: int
    B: int
    Ls_lo: int
    Ls_hi: int
    Hq: int
    Hkv: int
    d: int
    H: int
    V: int
    opt_lo: int
    opt_hi: int
    theta: float = 1e4
    seed: int = 0
    w_std: float = 0.02


@dataclass
class TreeConfig:
    name: str
    dtype: str
    Lp: int
    n_questions: int
    q_len: int
    leaves_lo: int
    leaves_hi: int
    leaf_len_lo: int
    leaf_len_hi: int
    Hq: int
    Hkv: int
    d: int
    H: int
    V: int
    theta: float = 1e4
    seed: int = 4
    w_std: float = 0.02


CONFIGS = {
    "tiny_f32": FlatConfig("tiny_f32", F32, 256, 4, 16, 16, 2, 1, 64, 256, 1024, 3, 3, seed=0),
    "qwen2vl_2b": FlatConfig("qwen2vl_2b", BF16, 1024, 8, 8, 24, 12, 2, 128, 1536, 151936, 3, 9, seed=1),
    "qwen25vl_7b": FlatConfig("qwen25vl_7b", BF16, 2048, 32, 12, 32, 28, 4, 128, 3584, 152064, 2, 3, seed=2),
    "wide_7b": FlatConfig("wide_7b", BF16, 4096, 128, 8, 40, 28, 4, 128, 3584, 152064, 3, 3, seed=3),
    "tree_7b": TreeConfig("tree_7b", BF16, 2048, 16, 24, 3, 9, 1, 4, 28, 4, 128, 3584, 152064, seed=4),
}

WORKLOAD_TEXT = {
    "tiny_f32": "tiny fp32: Lp=256, B=4, Ls=16, Hq=2, Hkv=1, d=64; readout H=256, V=1024, 3 options/branch",
    "qwen2vl_2b": "2B-shaped bf16: Lp=1024, B=8, Ls~U[8,24], Hq=12, Hkv=2, d=128; readout H=1536, V=151936, 3-9 options/branch",
    "qwen25vl_7b": "7B-shaped bf16: Lp=2048, B=32, Ls~U[12,32], Hq=28, Hkv=4, d=128; readout H=3584, V=152064, 2-3 options/branch",
    "wide_7b": "wide bf16: Lp=4096, B=128, Ls~U[8,40], Hq=28, Hkv=4, d=128; readout H=3584, V=152064, 3 options/branch",
    "tree_7b": "tree bf16: root Lp=2048; 16 question nodes x 24 tokens, 3-9 option leaves of 1-4 tokens each; Hq=28, Hkv=4, d=128; readout H=3584, V=152064 per leaf over its siblings",
}


def lm_head_rows(seed: int, V: int, H: int, rows: np.ndarray, dtype: str, std: float = 0.02) -> np.ndarray:
    """Regenerate selected rows of the LM head without drawing the whole matrix."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((rows.size, H), dtype=np.uint16 if dtype == BF16 else np.float32)
    for c in np.unique(rows // W_CHUNK_ROWS):
        blk = lm_head_block(seed, V, H, int(c), dtype, std)
        sel = np.nonzero(rows // W_CHUNK_ROWS == c)[0]
        out[sel] = blk[rows[sel] - c * W_CHUNK_ROWS]
    return out


def lm_head_block(seed: int, V: int, H: int, chunk: int, dtype: str, std: float = 0.02) -> np.ndarray:
    r0 = chunk * W_CHUNK_ROWS
    n = min(W_CHUNK_ROWS, V - r0)
    return _normal(seed, _S_W, (n, H), std, dtype, chunk=chunk)


def lm_head(seed: int, V: int, H: int, dtype: str, std: float = 0.02) -> np.ndarray:
    nchunk = (V + W_CHUNK_ROWS - 1) // W_CHUNK_ROWS
    return np.concatenate([lm_head_block(seed, V, H, c, dtype, std) for c in range(nchunk)], axis=0)


@dataclass
class FlatCase:
    cfg: FlatConfig
    q: np.ndarray          # [T, Hq, d] suffix queries (pre-RoPE)
    k_pre: np.ndarray      # [Lp, Hkv, d] prefix keys (the post-RoPE cache)
    v_pre: np.ndarray      # [Lp, Hkv, d]
    k_suf: np.ndarray      # [T, Hkv, d] suffix keys (pre-RoPE)
    v_suf: np.ndarray      # [T, Hkv, d]
    cu_seqlens: np.ndarray  # [B+1] int32
    hidden: np.ndarray     # [B, H] readout hidden state per branch
    set_offsets: np.ndarray  # [B+1] int32 candidates per branch
    pair_tok: np.ndarray   # [n_cands] int32 option token ids
    W: Optional[np.ndarray] = None  # [V, H] LM head (None when not materialised)

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])


def suffix_lengths(cfg: FlatConfig) -> np.ndarray:
    return _rng(cfg.seed, _S_LEN).integers(cfg.Ls_lo, cfg.Ls_hi + 1, size=cfg.B).astype(np.int32)


def flat_case(cfg: FlatConfig, with_lm_head: bool = True, lengths: Optional[np.ndarray] = None) -> FlatCase:
    """Draw every input of one flat (prefix + B ragged suffix branches) problem."""
    Ls = suffix_lengths(cfg) if lengths is None else np.asarray(lengths, dtype=np.int32)
    B = Ls.size
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(Ls)
    T = int(cu[-1])
    s = cfg.seed
    q = _normal(s, _S_Q, (T, cfg.Hq, cfg.d), 1.0, cfg.dtype)
    k_pre = _normal(s, _S_KP, (cfg.Lp, cfg.Hkv, cfg.d), 1.0, cfg.dtype)
    v_pre = _normal(s, _S_VP, (cfg.Lp, cfg.Hkv, cfg.d), 1.0, cfg.dtype)
    k_suf = _normal(s, _S_KS, (T, cfg.Hkv, cfg.d), 1.0, cfg.dtype)
    v_suf = _normal(s, _S_VS, (T, cfg.Hkv, cfg.d), 1.0, cfg.dtype)
    hidden = _normal(s, _S_HID, (B, cfg.H), 1.0, cfg.dtype)
    nopt = _rng(s, _S_NOPT).integers(cfg.opt_lo, cfg.opt_hi + 1, size=B)
    so = np.zeros(B + 1, dtype=np.int32)
    so[1:] = np.cumsum(nopt)
    orng = _rng(s, _S_OPT)
    toks = [orng.choice(cfg.V, size=int(n), replace=False) for n in nopt]
    pair_tok = (np.concatenate(toks) if toks else np.zeros(0)).astype(np.int32)
    W = lm_head(s, cfg.V, cfg.H, cfg.dtype, cfg.w_std) if with_lm_head else None
    return FlatCase(cfg, q, k_pre, v_pre, k_suf, v_suf, cu, hidden, so, pair_tok, W)


@dataclass
class TreeCase:
    cfg: TreeConfig
    seq_off: np.ndarray    # [n_cands+1] int32 CSR over candidate token sequences
    toks: np.ndarray       # [sum len] int32 candidate tokens (question ++ option)
    score_from: np.ndarray  # [n_cands] int32 index where each candidate's scored tokens start
    set_offsets: np.ndarray  # [n_questions+1] candidates grouped per question
    n_unique: int          # number of distinct non-root token positions in the trie
    q: np.ndarray          # [N, Hq, d] tree-token queries in packed trie order (pre-RoPE)
    k: np.ndarray          # [N, Hkv, d]
    v: np.ndarray          # [N, Hkv, d]
    k_root: np.ndarray     # [Lp, Hkv, d] root (prefix) cache, post-RoPE
    v_root: np.ndarray     # [Lp, Hkv, d]
    hidden: np.ndarray     # [N, H] final hidden state per tree token
    W: Optional[np.ndarray] = None


def tree_case(cfg: TreeConfig, with_lm_head: bool = True) -> TreeCase:
    """Draw a two-level candidate tree: question segments with option leaves.

    Question first tokens are distinct across questions and option first tokens
    are distinct among siblings, so the trie has exactly one node per question
    and one per option and ``n_unique`` packed token rows.
    """
    s = cfg.seed
    rng = _rng(s, _S_TREE)
    qfirst = rng.choice(cfg.V, size=cfg.n_questions, replace=False)
    seqs: List[np.ndarray] = []
    score_from: List[int] = []
    set_off = [0]
    n_unique = 0
    for qi in range(cfg.n_questions):
        qt = rng.integers(0, cfg.V, size=cfg.q_len)
        qt[0] = qfirst[qi]
        n_unique += cfg.q_len
        nleaf = int(rng.integers(cfg.leaves_lo, cfg.leaves_hi + 1))
        first = rng.choice(cfg.V, size=nleaf, replace=False)
        for li in range(nleaf):
            ln = int(rng.integers(cfg.leaf_len_lo, cfg.leaf_len_hi + 1))
            ot = rng.integers(0, cfg.V, size=ln)
            ot[0] = first[li]
            n_unique += ln
            seqs.append(np.concatenate([qt, ot]).astype(np.int32))
            score_from.append(cfg.q_len)
        set_off.append(len(seqs))
    seq_off = np.zeros(len(seqs) + 1, dtype=np.int32)
    seq_off[1:] = np.cumsum([x.size for x in seqs])
    toks = np.concatenate(seqs).astype(np.int32)
    N = n_unique
    q = _normal(s, _S_Q, (N, cfg.Hq, cfg.d), 1.0, cfg.dtype)
    k = _normal(s, _S_KS, (N, cfg.Hkv, cfg.d), 1.0, cfg.dtype)
    v = _normal(s, _S_VS, (N, cfg.Hkv, cfg.d), 1.0, cfg.dtype)
    k_root = _normal(s, _S_KP, (cfg.Lp, cfg.Hkv, cfg.d), 1.0, cfg.dtype)
    v_root = _normal(s, _S_VP, (cfg.Lp, cfg.Hkv, cfg.d), 1.0, cfg.dtype)
    hidden = _normal(s, _S_HID, (N, cfg.H), 1.0, cfg.dtype)
    W = lm_head(s, cfg.V, cfg.H, cfg.dtype, cfg.w_std) if with_lm_head else None
    return TreeCase(cfg, seq_off, toks, np.asarray(score_from, np.int32),
                    np.asarray(set_off, np.int32), n_unique, q, k, v, k_root, v_root, hidden, W)


def scaled(cfg, **kw):
    """Copy of a config with some fields replaced (smaller parity cases)."""
    import dataclasses
    return dataclasses.replace(cfg, **kw)
