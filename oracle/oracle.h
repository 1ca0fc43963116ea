/*
 * oracle.h — plain fp64 CPU reference for shared-prefix attention, candidate
 * readout and the candidate-prefix trie.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * product path (attention_cascade_b200) never calls it and shares no code with
 * it; the two only share the seeded input generator in synth/.
 *
 * Semantics follow the pages:
 *  - "FastJEV: Understanding Redundancy for Compact JEV Inference" (paperlayer.ai
 *    summary of arXiv 2610.11379v1), TL;DR and §3.2/§3.3: sharing a history is
 *    valid only when tokens, positions and masks are identical, so each branch's
 *    result is full causal attention over [prefix; its own suffix].  The oracle
 *    therefore never shares anything: it materialises [prefix; suffix] for every
 *    branch separately.
 *  - "How to Deploy Visual Jev for Sub-20ms Shared Prefix Image Decisions and
 *    Diffusion Filtering" (aiintoai.vercel.app), Step 3: the decision reads the
 *    unmasked last-position logits of the option tokens and applies a softmax
 *    over the candidate set only; ties go to the first option.
 *  - FastJEV §3.3: a prefix tree evaluates matching token histories once and
 *    maps merged nodes back to every candidate's readout entry; merging
 *    respects positions and preceding history.
 *
 * Readings where the pages are silent (each listed in the design notes):
 * rotate-half RoPE with theta_i = theta^(-2i/d) and 1-D positions; suffix token
 * j of a branch sits at position pos_offset + j (pos_offset defaults to Lp);
 * prefix keys arrive already rotated; softmax scale 1/sqrt(d) by default;
 * q-head h uses kv-head h / (Hq/Hkv) unless a head map is given; multi-token
 * candidates score the sum of teacher-forced logits; canonical trie numbering
 * is DFS preorder with children in first-appearance order.
 *
 * All inputs are read as bf16 (uint16 bit patterns) or fp32 and widened
 * exactly to double; all arithmetic is double.
 */
#ifndef JEV_ORACLE_H
#define JEV_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* Rotate-half RoPE of one d-vector at position pos (d even). */
void oracle_rope(const double* x, double* y, int d, double pos, double theta);

/* Attention of one query row over an explicit key list (no mask):
 * s_t = scale * <q, K[t]>, o = sum softmax(s)_t V[t], lse = log sum exp(s).
 * K, V are [n, d] with row stride `stride` doubles. */
void oracle_attend(const double* q, const double* K, const double* V, int n, int d,
                   int stride, double scale, double* o, double* lse);

typedef struct {
  int B, Lp, Hq, Hkv, d, dtype;
  double theta;        /* RoPE base */
  double scale;        /* 0 -> 1/sqrt(d) */
  int pos_offset;      /* < 0 -> Lp */
  const void* q;       /* [T, Hq, d] pre-RoPE */
  const void* k_pre;   /* [Lp, Hkv, d] post-RoPE cache */
  const void* v_pre;   /* [Lp, Hkv, d] */
  const void* k_suf;   /* [T, Hkv, d] pre-RoPE */
  const void* v_suf;   /* [T, Hkv, d] */
  const int32_t* cu_seqlens; /* [B+1] */
  const int32_t* head_map;   /* [Hq] or NULL */
  int n_rows;                /* 0 -> every (t, h) row */
  const int32_t* rows;       /* [n_rows][2] = (t, h) when n_rows > 0 */
  int n_threads;             /* 0 -> OpenMP default */
} oracle_attn_problem;

/* Unshared per-branch attention.  out is [T, Hq, d] (or [n_rows, d]), lse is
 * [T, Hq] (or [n_rows]); both double.  Returns 0, or -1 on bad arguments. */
int oracle_prefix_suffix_attn(const oracle_attn_problem* p, double* out, double* lse);

typedef struct {
  int B, Lp, Hq, Hkv, d, dtype;
  double theta;        /* RoPE base */
  double scale;        /* 0 -> 1/sqrt(d) */
  int pos_offset;      /* < 0 -> Lp */
  const void* q;       /* [T, Hq, d] new tokens, pre-RoPE */
  const void* k_new;   /* [T, Hkv, d] new tokens' keys, pre-RoPE */
  const void* v_new;   /* [T, Hkv, d] */
  const void* k_pre;   /* [Lp, Hkv, d] post-RoPE prefix cache */
  const void* v_pre;   /* [Lp, Hkv, d] */
  const void* k_cache; /* [C, Hkv, d] cached suffix keys, post-RoPE */
  const void* v_cache; /* [C, Hkv, d] */
  const int32_t* cache_off; /* [B+1] branch b's cache rows start at cache_off[b] */
  const int32_t* cache_len; /* [B] tokens cached per branch */
  const int32_t* cu_new;    /* [B+1] new-token offsets */
  const int32_t* head_map;  /* [Hq] or NULL */
  int n_threads;
} oracle_cache_problem;

/* A generation step over per-branch suffix caches, computed unshared: for
 * branch b the key list is [K_pre ; its cache_len[b] cached keys ; RoPE(its
 * new keys)], new token j sits at position pos_offset + cache_len[b] + j and
 * sees keys 0 .. Lp + cache_len[b] + j.  out [T, Hq, d], lse [T, Hq];
 * k_new_rot [T, Hkv, d] receives the rotated new keys (what the step appends
 * to the cache).  Returns 0, or -1 on bad arguments (including a branch whose
 * cache rows cannot hold its tokens). */
int oracle_cache_attn(const oracle_cache_problem* p, double* out, double* lse, double* k_new_rot);

typedef struct {
  int n_sets, n_cands, n_pairs, R, H, V, dtype;
  const void* hidden;          /* [R, H] */
  const void* lm_head;         /* [V, H] */
  const int32_t* set_offsets;  /* [n_sets+1] */
  const int32_t* cand_offsets; /* [n_cands+1] or NULL (one pair per candidate) */
  const int32_t* pair_row;     /* [n_pairs] or NULL (row = set index) */
  const int32_t* pair_tok;     /* [n_pairs] */
  int full_vocab;              /* 1: form every logit of each used row (the
                                  plain definition); 0: only the option logits */
  int n_threads;
} oracle_readout_problem;

/* Candidate readout.  score/logprob: [n_cands]; choice/gap: [n_sets];
 * row_lse: [R] full-vocab log-sum-exp of each used row (NaN if unused or if
 * full_vocab == 0), may be NULL.  Invalid token ids give NaN scores and
 * choice -1 for their set.  Returns the number of invalid pairs, or -1. */
int oracle_candidate_readout(const oracle_readout_problem* p, double* score, double* logprob,
                             int32_t* choice, double* gap, double* row_lse);

/* Canonical compressed trie over candidate token sequences.
 * Outputs (capacity cap_nodes nodes, cap_toks packed tokens):
 *   parent[n] (parent[0] = -1), tok_off[n+1], pos0[n] (absolute position of
 *   the node's first token, root_len for children of the root), leaf_of[c],
 *   node_toks[tok_off[n_nodes]] (packed token ids), and, if path_row is not
 *   NULL, path_row[seq_off[c] + i] = packed row of candidate c's i-th token.
 * Returns n_nodes, or -1 on bad input / overflow. */
int oracle_trie_build(int n_cands, const int32_t* seq_off, const int32_t* toks, int root_len,
                      int cap_nodes, int cap_toks, int32_t* parent, int32_t* tok_off,
                      int32_t* pos0, int32_t* leaf_of, int32_t* node_toks, int32_t* path_row);

typedef struct {
  int n_nodes, N, Lp, Hq, Hkv, d, dtype;
  double theta, scale;
  const int32_t* parent;   /* [n_nodes] */
  const int32_t* tok_off;  /* [n_nodes+1] */
  const void* q;           /* [N, Hq, d] pre-RoPE, packed node order */
  const void* k;           /* [N, Hkv, d] pre-RoPE */
  const void* v;           /* [N, Hkv, d] */
  const void* k_root;      /* [Lp, Hkv, d] post-RoPE */
  const void* v_root;      /* [Lp, Hkv, d] */
  const int32_t* head_map; /* [Hq] or NULL */
  int n_threads;
} oracle_tree_problem;

/* Tree attention by flattening: every node's rows are computed as one flat
 * branch whose suffix is the root->node token path, the path's i-th token at
 * position Lp + i.  out [N, Hq, d], lse [N, Hq]. */
int oracle_tree_attn(const oracle_tree_problem* p, double* out, double* lse);

#ifdef __cplusplus
}
#endif
#endif
