/*
 * jev.h — C ABI of the shared-prefix (cascade) attention and candidate
 * readout library for NVIDIA B200 (sm_100a).
 *
 * The method (pages: "How to Deploy Visual Jev for Sub-20ms Shared Prefix
 * Image Decisions and Diffusion Filtering", Steps 2-3; "FastJEV: Understanding
 * Redundancy for Compact JEV Inference", TL;DR, §3.2, §3.3; "Ochevid Jev-VL
 * 2B" model card, "Run"): an image-plus-context prefix is encoded once and its
 * key/value cache stays in GPU memory; many question/candidate suffix
 * branches attend to it, each one as if it were the only continuation of the
 * prefix; each branch's decision is a softmax over the unmasked logits of its
 * option tokens.
 *
 * Conventions shared by every entry point
 *  - Memory.  Every tensor argument is caller-owned DEVICE memory unless the
 *    comment says "host".  Tensors are dense, row-major, 16-byte aligned.  The
 *    library allocates nothing; scratch space is the caller's `workspace`,
 *    sized by the matching *_workspace() query.
 *  - Streams.  All work is enqueued on `stream` in order; no call blocks the
 *    host except jev_check_device_status() and the host-only tree helpers.
 *  - Errors.  Argument problems the host can see return a non-OK status
 *    before anything is enqueued; jev_last_error() then describes it.
 *    Problems only the device can see (a non-monotone cu_seqlens, a bad head
 *    map, an out-of-range token id, a malformed tree, a bounded wait that ran
 *    out) never trap: the kernels skip the affected rows, write NaN/-1
 *    sentinels where an output exists, and OR a bit into the status word at
 *    the start of the workspace, read by jev_check_device_status().  The
 *    status word is sticky: it is cleared by jev_workspace_init() and by
 *    jev_check_device_status() only.
 *  - Threads.  Entry points are reentrant; jev_last_error() is per thread.
 *  - Precision.  bf16 inputs use fp32 accumulation and return bf16 outputs
 *    (round to nearest even); f32 inputs compute in fp32.
 */
#ifndef JEV_H
#define JEV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* jev_stream_t; /* same object as cudaStream_t */

typedef enum {
  JEV_OK = 0,
  JEV_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent sizes   */
  JEV_ERR_UNSUPPORTED = 2,  /* shape or dtype outside what the kernels cover */
  JEV_ERR_WORKSPACE = 3,    /* workspace missing or too small                */
  JEV_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed          */
  JEV_ERR_DEVICE = 5,       /* jev_check_device_status found flags set       */
  JEV_ERR_CAPACITY = 6      /* a host output buffer is too small             */
} jev_status;

typedef enum { JEV_F32 = 0, JEV_BF16 = 1 } jev_dtype;

/* Bits of the device status word (jev_check_device_status). */
enum {
  JEV_DEV_BAD_SEQLENS = 1,   /* cu_seqlens / tok_off not monotone or != T   */
  JEV_DEV_BAD_HEAD_MAP = 2,  /* head map entry out of range or groups uneven */
  JEV_DEV_BAD_TREE = 4,      /* nodes not in depth-first preorder, or bad offsets */
  JEV_DEV_WAIT_TIMEOUT = 8,  /* a bounded pipeline wait gave up             */
  JEV_DEV_BAD_WINDOW = 16,   /* a row's key window exceeded the kernel limit */
  JEV_DEV_BAD_CACHE = 32     /* a branch's cache rows cannot hold its tokens */
};

/* ------------------------------------------------------------------------ */
/* Shared-prefix attention                                                   */
/* ------------------------------------------------------------------------ */

typedef struct {
  int32_t B;             /* number of suffix branches (>= 0)                        */
  int32_t Lp;            /* prefix length: keys in the shared cache (>= 0)          */
  int32_t Hq;            /* query heads                                             */
  int32_t Hkv;           /* key/value heads; Hq % Hkv == 0                          */
  int32_t d;             /* head dimension: 64 or 128                               */
  int32_t T_total;       /* packed suffix tokens, must equal cu_seqlens[B]          */
  jev_dtype dtype;       /* JEV_BF16 or JEV_F32, same for every tensor              */
  float rope_theta;      /* RoPE base (> 0)                                         */
  float softmax_scale;   /* 0 -> 1/sqrt(d)                                          */
  int32_t pos_offset;    /* position of every branch's first suffix token; <0 -> Lp */
  int32_t num_splits;    /* prefix key splits; 0 -> chosen from Lp and the SM count */
  int32_t pos_mode;      /* 0: token j of every branch at pos_offset + j;
                            1: sequential positions (sink-block parallel encoding,
                            "PEVLM: Parallel Encoding for Vision-Language Models",
                            abstract: blocks share a sink and keep the positions of
                            the unsplit sequence): packed token t at pos_offset + t.
                            jev_prefix_suffix_attn only.                              */
} jev_attn_desc;

/* Bytes of workspace jev_prefix_suffix_attn needs for `desc`. */
size_t jev_prefix_suffix_attn_workspace(const jev_attn_desc* desc);

/*
 * The work plan jev_prefix_suffix_attn follows for `desc` (host only, no
 * device work).  kernel: -1 -> the kernel the current device runs, 0 -> the
 * CUDA-core plan, 1 -> the tensor-core plan (a what-if on any host; only
 * bf16 with d 64 or 128 on sm_100a runs it).  num_sms <= 0 -> the current
 * device's SM count (148 when no device is present); num_sms > 0 plans for
 * that many SMs, as a what-if.  Tensor-core kernel (kernel == 1): stacked query rows of one
 * kv head form work tiles of tile_rows rows, n_tiles in all, each of
 * units_per_tile units (one per 128-key prefix tile plus one for the suffix
 * window).  n_ctas persistent CTAs first take full_waves rounds of whole
 * tiles (tile c + k*n_ctas to CTA c); the tail_units units of tiles
 * tail0 .. n_tiles-1 are spread evenly over CTAs 0 .. tail_ctas-1, CTA c
 * owning [c*tail_units/tail_ctas, (c+1)*tail_units/tail_ctas); split != 0
 * when some tile is shared by several CTAs and a merge kernel combines it.
 * tile_rows is 128 (a kernel with one Q tile a CTA, for twice as many
 * tiles) when 256-row tiles would be fewer than num_sms and their units fewer
 * than 20 x num_sms, else 256 (a kernel with two 128-row Q tiles a CTA); 0
 * for the CUDA-core plan.
 * CUDA-core kernel (kernel == 0): simt_splits prefix splits of split_len
 * keys (a multiple of 32).  Returns the descriptor's error (as jev_prefix_suffix_attn would) or
 * JEV_ERR_INVALID_ARG for a NULL `plan` or a kernel outside -1 .. 1.
 */
typedef struct {
  int32_t kernel;          /* 1 tensor-core (bf16, d 64/128, sm_100a), 0 CUDA-core */
  int32_t n_tiles, units_per_tile, n_ctas, full_waves, tail0, tail_ctas, split;
  int64_t tail_units;
  int32_t simt_splits, split_len;
  int32_t tile_rows;       /* tensor-core plan: stacked rows per work tile (128 or 256) */
} jev_attn_plan;
jev_status jev_prefix_suffix_attn_plan(const jev_attn_desc* desc, int32_t kernel, int32_t num_sms,
                                      jev_attn_plan* plan);

/*
 * jev_prefix_suffix_attn — one attention layer for B branches over a shared
 * prefix.  For branch b with suffix tokens t = cu_seqlens[b] .. cu_seqlens[b+1]-1
 * (local index j = t - cu_seqlens[b]) and query head h (kv head g = head_map[h]):
 *
 *     keys    = [ k_pre[0..Lp) ; RoPE(k_suf[cu_seqlens[b] .. t], pos_offset + j') ]
 *     out[t,h] = softmax(scale * RoPE(q[t,h], pos_offset + j) . keys^T) . values
 *     lse[t,h] = natural-log normaliser of that softmax
 *
 * which is exactly full causal attention over [prefix; this branch's suffix]
 * (FastJEV TL;DR / §3.3: sharing is valid because histories, positions and
 * masks are identical).  No branch sees another branch's tokens.
 *
 *   q          [T, Hq, d]   suffix queries before RoPE
 *   k_pre      [Lp, Hkv, d] prefix keys, already rotated at positions 0..Lp-1
 *   v_pre      [Lp, Hkv, d]
 *   k_suf      [T, Hkv, d]  suffix keys before RoPE
 *   v_suf      [T, Hkv, d]
 *   cu_seqlens [B+1] int32  branch offsets into the packed suffix, cu[0] = 0
 *   head_map   [Hq] int32 or NULL (NULL -> h / (Hq/Hkv)); every kv head must
 *              receive exactly Hq/Hkv query heads
 *   out        [T, Hq, d]   same dtype as q
 *   lse        [T, Hq] fp32 or NULL
 *   workspace  >= jev_prefix_suffix_attn_workspace(desc) bytes, 256-byte
 *              aligned; its first 256 bytes hold the device status word and
 *              must be zeroed once (jev_workspace_init) before first use.
 *
 * B == 0 or T == 0 returns JEV_OK with nothing enqueued.
 */
jev_status jev_prefix_suffix_attn(const jev_attn_desc* desc, const void* q, const void* k_pre,
                                  const void* v_pre, const void* k_suf, const void* v_suf,
                                  const int32_t* cu_seqlens, const int32_t* head_map, void* out,
                                  float* lse, void* workspace, size_t ws_bytes, jev_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Generation over per-branch suffix caches                                  */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace jev_suffix_cache_attn needs for `desc`. */
size_t jev_suffix_cache_attn_workspace(const jev_attn_desc* desc);

/*
 * jev_suffix_cache_attn — one attention layer for the new tokens of B
 * branches that continue over the shared prefix and their own cached suffix
 * tokens: a generation step after the decision, each branch decoding its own
 * continuation ("How to Deploy Visual Jev ...", Step 3 batches the branches
 * over the one cached prefix; "FastJEV ...", Abstract and §5: what is shared
 * and how the work is scheduled are designed together).  Branch b has
 * cache_len[b] suffix tokens already cached: rotated keys and values in rows
 * cache_off[b] .. cache_off[b] + cache_len[b] - 1 of k_cache / v_cache.  Its
 * new tokens are rows cu_new[b] .. cu_new[b+1]-1 of q / k_new / v_new; new
 * token j sits at position pos_offset + cache_len[b] + j and
 *
 *     keys     = [ k_pre[0..Lp) ; cached keys of b ; RoPE(new keys of b, 0..j) ]
 *     out[t,h] = softmax(scale * RoPE(q[t,h]) . keys^T) . values,  lse as in
 *                jev_prefix_suffix_attn
 *
 * which is the row jev_prefix_suffix_attn gives token cache_len[b] + j of the
 * branch's whole suffix.  The call also appends: new token j's rotated key and
 * its value are written to cache row cache_off[b] + cache_len[b] + j.  It does
 * not change cache_len; the caller advances it by the new token counts.  A
 * first call with cache_len = 0 is the prefill and fills the caches.
 *
 *   desc       B, Lp, Hq, Hkv, d, dtype, rope_theta, softmax_scale, pos_offset
 *              (<0 -> Lp), num_splits as for jev_prefix_suffix_attn; T_total
 *              = new tokens (cu_new[B]); pos_mode must be 0
 *   q          [T_total, Hq, d]  new tokens' queries before RoPE
 *   k_new      [T_total, Hkv, d] new tokens' keys before RoPE
 *   v_new      [T_total, Hkv, d]
 *   k_pre/v_pre [Lp, Hkv, d]     the shared prefix cache (k rotated)
 *   k_cache/v_cache [cache_rows, Hkv, d] in/out, same dtype; branch b owns
 *              rows cache_off[b] .. cache_off[b+1]-1
 *   cache_off  device [B+1] int32, non-decreasing, cache_off[B] <= cache_rows
 *   cache_len  device [B] int32, cached tokens per branch
 *   cu_new     device [B+1] int32, new-token offsets, cu_new[0] = 0
 *   head_map, out [T_total, Hq, d], lse [T_total, Hq] fp32 or NULL, workspace
 *              (>= jev_suffix_cache_attn_workspace(desc) bytes) as for
 *              jev_prefix_suffix_attn
 *
 * A branch whose rows cannot hold its new tokens (cache_len[b] + new tokens >
 * cache_off[b+1] - cache_off[b]) sets JEV_DEV_BAD_CACHE; its rows and its cache
 * are left untouched and the other branches are computed.  Rows of the window
 * a work tile reads lie between its branches' first cache rows and last new
 * slots, so caches packed tightly (little unused capacity between branches)
 * cost the fewest masked key tiles.
 */
jev_status jev_suffix_cache_attn(const jev_attn_desc* desc, const void* q, const void* k_new, const void* v_new,
                                 const void* k_pre, const void* v_pre, void* k_cache, void* v_cache,
                                 int32_t cache_rows, const int32_t* cache_off, const int32_t* cache_len,
                                 const int32_t* cu_new, const int32_t* head_map, void* out, float* lse,
                                 void* workspace, size_t ws_bytes, jev_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Fixed-scratch variant (no allocation)                                     */
/* ------------------------------------------------------------------------ */

/* Size of the library's static device scratch used by the variant below. */
#define JEV_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * jev_prefix_suffix_attn_noalloc — the same attention as
 * jev_prefix_suffix_attn (same arguments and results) for callers that cannot
 * hand the library a workspace: code whose device memory is owned and
 * budgeted by a host runtime that exposes no allocator to it (a plugin inside
 * an inference engine, a pre-planned static memory arena), or code that must
 * not call cudaMalloc/cudaFree because those synchronise the device or are
 * not allowed at that point.  The paper has no counterpart; this entry point
 * exists only for such callers.
 *
 * Scratch comes from one file-scope device array of JEV_NOALLOC_SCRATCH_BYTES
 * bytes that every GPU loading the library holds until the process exits.
 * The call allocates nothing (no cudaMalloc, no cudaFree, no allocating
 * library routine).  If the automatic plan, with its split partials, does
 * not fit in the array the call falls back to the plan that splits no work
 * (num_splits = 1, no partials); if that does not fit either
 * it returns JEV_ERR_UNSUPPORTED, naming the bytes needed, before enqueuing
 * anything.
 *
 * The first call on a device looks up the array's device address on that
 * device (cudaGetSymbolAddress, with the device current) and caches it; make
 * that first call before any stream capture.  Every call shares the one array
 * and leaves its contents behind; the call clears the status word at its
 * start.  Calls whose work overlaps on the GPU (different streams, or
 * different host threads on one device) race on the array: serialise them.
 *
 *   status_flags  optional DEVICE int32: receives the call's status-word bits
 *                 (JEV_DEV_*) at the end of the call, in stream order; NULL
 *                 discards them.
 */
jev_status jev_prefix_suffix_attn_noalloc(const jev_attn_desc* desc, const void* q, const void* k_pre,
                                          const void* v_pre, const void* k_suf, const void* v_suf,
                                          const int32_t* cu_seqlens, const int32_t* head_map, void* out,
                                          float* lse, int32_t* status_flags, jev_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Candidate readout                                                         */
/* ------------------------------------------------------------------------ */

typedef struct {
  int32_t n_sets;   /* option sets (one per branch, or per tree question)           */
  int32_t n_cands;  /* candidates over all sets                                     */
  int32_t n_pairs;  /* (hidden row, token) pairs over all candidates                */
  int32_t R;        /* hidden rows                                                  */
  int32_t H;        /* hidden size; multiple of 8                                   */
  int32_t V;        /* vocabulary rows of the LM head                               */
  jev_dtype dtype;  /* dtype of hidden and lm_head                                  */
} jev_readout_desc;

/*
 * jev_candidate_readout — decision from unmasked option logits ("How to Deploy
 * Visual Jev ...", Step 3: last-position logits, the option token is the first
 * sub-token of the option string, softmax over the candidate pair, ties go to
 * the first option; FastJEV §3.3: tree candidates map back to their own
 * readout entries).  No full-vocabulary product is formed: only the option
 * rows of the LM head are read.
 *
 *   z_c        = sum over candidate c's pairs (r, tok) of  hidden[r] . lm_head[tok]
 *   logprob[c] = z_c - log sum_{c' in set(c)} exp(z_c')
 *   choice[s]  = local index of the largest logprob in set s (lowest index on ties),
 *                -1 for an empty set or a set holding an invalid pair
 *
 *   hidden       [R, H]   final hidden states (after the final norm)
 *   lm_head      [V, H]   row-major LM head
 *   set_offsets  [n_sets+1] int32 candidate ranges of each set
 *   cand_offsets [n_cands+1] int32 pair ranges of each candidate, or NULL
 *                (one pair per candidate; n_pairs == n_cands)
 *   pair_row     [n_pairs] int32 hidden row of each pair, or NULL (row = set index)
 *   pair_tok     [n_pairs] int32 token id of each pair, in [0, V)
 *   logprob      [n_cands] fp32;  choice [n_sets] int32;  score [n_cands] fp32 or NULL
 *
 * An out-of-range row or token makes that candidate's score and its set's
 * log-probs NaN and the set's choice -1.
 */
jev_status jev_candidate_readout(const jev_readout_desc* desc, const void* hidden, const void* lm_head,
                                 const int32_t* set_offsets, const int32_t* cand_offsets,
                                 const int32_t* pair_row, const int32_t* pair_tok, float* logprob,
                                 int32_t* choice, float* score, jev_stream_t stream);

/*
 * Full-vocabulary log-sum-exp (normalised multi-token candidate scoring):
 *
 *   lse[r] = log sum_{v < V} exp(hidden[r] . lm_head[v]),   r < R
 *
 * the normaliser that turns an unmasked option logit into a log-probability
 * over the whole vocabulary, log p(tok | r) = hidden[r] . lm_head[tok] -
 * lse[r] ("How to Deploy Visual Jev ...", Step 3 reads its logits from the
 * full LM-head projection; FastJEV, Appendix A (Additional Experimental
 * Results), counts vocabulary-projection scheduling among the tree path's
 * costs).  A candidate of several tokens scored as a
 * sequence log-probability sums those terms over its teacher-forced pairs.
 * The product is formed tile by tile on the tensor cores and reduced on
 * chip: no logit is written to memory.
 *
 *   hidden   [R, H] bf16, row-major, 16-byte aligned
 *   lm_head  [V, H] bf16, row-major, 16-byte aligned
 *   H        multiple of 64;  R >= 0;  V >= 1
 *   lse      [R] fp32 DEVICE output
 *   workspace >= jev_vocab_lse_workspace(R, V) bytes, 256-byte aligned; its
 *            first 256 bytes hold the device status word (jev_workspace_init
 *            once, jev_check_device_status to read it).  A pipeline wait
 *            that gives up sets JEV_DEV_WAIT_TIMEOUT and makes lse NaN.
 *
 * bf16 on sm_100a only (JEV_ERR_UNSUPPORTED otherwise); R == 0 enqueues nothing.
 */
size_t jev_vocab_lse_workspace(int32_t R, int32_t V);
jev_status jev_vocab_lse(const void* hidden, const void* lm_head, int32_t R, int32_t H, int32_t V,
                         jev_dtype dtype, float* lse, void* workspace, size_t ws_bytes, jev_stream_t stream);

/*
 * jev_candidate_readout_normalized — jev_candidate_readout with every pair's
 * term normalised over the whole vocabulary: a candidate's score becomes its
 * sequence log-probability
 *
 *   score[c]   = sum over c's pairs (r, tok) of  hidden[r] . lm_head[tok] - row_lse[r]
 *
 * and logprob / choice are the log-softmax and argmax of those scores over
 * each set.  row_lse [R] fp32 DEVICE, normally jev_vocab_lse of the same
 * hidden rows and head; NULL gives jev_candidate_readout exactly.  Other
 * arguments and errors as jev_candidate_readout.
 */
jev_status jev_candidate_readout_normalized(const jev_readout_desc* desc, const void* hidden, const void* lm_head,
                                            const int32_t* set_offsets, const int32_t* cand_offsets,
                                            const int32_t* pair_row, const int32_t* pair_tok, const float* row_lse,
                                            float* logprob, int32_t* choice, float* score, jev_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Candidate-prefix tree                                                     */
/* ------------------------------------------------------------------------ */

/*
 * jev_tree_build (HOST) — the candidate-prefix trie of FastJEV §3.3: matching
 * token histories are merged into one node, a token after a different history
 * stays separate.  Node 0 is the root (the shared prefix, no packed tokens).
 * A node is a maximal chain of tokens with a single continuation that does not
 * pass the end of a candidate; nodes are numbered in depth-first preorder with
 * children in order of first appearance among the candidates.
 *
 *   seq_off   [n_cands+1] host int32, toks [seq_off[n_cands]] host int32
 *   outputs (host, capacity cap_nodes / cap_toks):
 *     parent[n] (parent[0] = -1, parent[n] < n), tok_off[n+1] (CSR of packed
 *     tokens, tok_off[0] = tok_off[1] = 0), pos0[n] (absolute position of
 *     node n's first token, root_len for children of the root), leaf_of[c]
 *     (node holding candidate c's last token; 0 for an empty candidate),
 *     node_toks[N] (packed token ids), path_row[seq_off[n_cands]] (packed row
 *     of every token of every candidate) — path_row may be NULL.
 *   *n_nodes receives the node count.  JEV_ERR_CAPACITY if a buffer is short.
 */
jev_status jev_tree_build(int32_t n_cands, const int32_t* seq_off, const int32_t* toks, int32_t root_len,
                          int32_t cap_nodes, int32_t cap_toks, int32_t* parent, int32_t* tok_off,
                          int32_t* pos0, int32_t* leaf_of, int32_t* node_toks, int32_t* path_row,
                          int32_t* n_nodes);

/*
 * jev_tree_readout_plan (HOST) — readout pairs for multi-token candidates by
 * teacher forcing: candidate c's tokens i >= score_from[c] are each scored
 * from the hidden state of the token before them on c's own path, so
 * z_c = sum_i hidden[path_row[i-1]] . lm_head[tok_i] (reduces to the pages'
 * single last-position logit for one-token options).  score_from[c] >= 1.
 *   outputs (host): cand_offsets [n_cands+1], pair_row / pair_tok [cap_pairs];
 *   *n_pairs receives the pair count.
 */
jev_status jev_tree_readout_plan(int32_t n_cands, const int32_t* seq_off, const int32_t* toks,
                                 const int32_t* score_from, const int32_t* path_row, int32_t cap_pairs,
                                 int32_t* cand_offsets, int32_t* pair_row, int32_t* pair_tok,
                                 int32_t* n_pairs);

/* Bytes of workspace jev_tree_attn needs. */
size_t jev_tree_attn_workspace(const jev_attn_desc* desc, int32_t n_nodes);

/*
 * jev_tree_attn — attention for every packed tree token (FastJEV §3.3: each
 * shared history is evaluated once and its keys/values serve every
 * descendant).  Token i of node n (local index j, position pos0[n] + j)
 * attends to the root cache (all Lp keys), to every token of every non-root
 * ancestor of n, and to tokens 0..j of n itself — exactly causal attention
 * over its root->leaf path.
 *
 *   desc: Lp = root length, T_total = N packed tokens, B = n_nodes - 1,
 *         pos_offset ignored (positions come from pos0)
 *   parent, tok_off, pos0: DEVICE copies of jev_tree_build's outputs
 *   q [N, Hq, d], k/v [N, Hkv, d] before RoPE, in packed node order;
 *   k_root/v_root [Lp, Hkv, d] the root cache (k already rotated);
 *   out [N, Hq, d]; lse [N, Hq] fp32 or NULL.
 *   Nodes must be numbered in depth-first preorder with their tokens packed
 *   in node order (as jev_tree_build returns them); any depth is allowed.  A
 *   node whose parent is not earlier than itself, or not on the path of the
 *   node before it, or whose token offsets are out of order, sets
 *   JEV_DEV_BAD_TREE and its rows are left unwritten.  The RoPE pack plans
 *   each token's node with warp-wide scans whose length grows with the node's
 *   distance to its parent, to the end of its subtree and to its top-level
 *   ancestor, in node order.
 */
jev_status jev_tree_attn(const jev_attn_desc* desc, int32_t n_nodes, const int32_t* parent,
                         const int32_t* tok_off, const int32_t* pos0, const void* q, const void* k_root,
                         const void* v_root, const void* k, const void* v, const int32_t* head_map,
                         void* out, float* lse, void* workspace, size_t ws_bytes, jev_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Helpers                                                                   */
/* ------------------------------------------------------------------------ */

/* Rotate x [L, H, d] in place at positions pos0 .. pos0+L-1 (rotate-half RoPE,
 * angle p * theta^(-2i/d)); builds a post-RoPE prefix cache from raw keys. */
jev_status jev_rope_inplace(void* x, int32_t L, int32_t H, int32_t d, int32_t pos0, float theta,
                            jev_dtype dtype, jev_stream_t stream);

/* Self-test of the FMA-pipe 2^x the attention kernel uses for a share of its
 * softmax exponentials (cubic on the reduced argument; relative error below
 * 2e-4 for -125 <= x <= 2^22, about 2^-125 below -125): y[i] = 2^x[i] for
 * n device floats. */
jev_status jev_selftest_exp2(const float* x, float* y, int32_t n, jev_stream_t stream);

/* Zero the status word at the start of a workspace (enqueued on stream). */
jev_status jev_workspace_init(void* workspace, size_t ws_bytes, jev_stream_t stream);

/* Synchronise `stream`, read and clear the status word; *flags gets its bits.
 * Returns JEV_ERR_DEVICE if any bit was set. */
jev_status jev_check_device_status(void* workspace, size_t ws_bytes, jev_stream_t stream, int32_t* flags);

/* Message for this thread's last non-OK status ("" if none). */
const char* jev_last_error(void);

/* Kernel timing.  While enabled, every kernel launch is bracketed by CUDA
 * events on its stream (inside a stream capture the events become graph
 * nodes and are re-recorded by every replay).  jev_profile_read synchronises
 * the recorded events and returns, per kernel name, the launch count and
 * summed milliseconds; with keep == 0 it then drops the records, with
 * keep != 0 it leaves them registered so a replayed graph can be read again.
 * Returns the number of kernel names (names: cap x 64 bytes, may be NULL). */
jev_status jev_profile_enable(int32_t on);
int32_t jev_profile_read(int32_t cap, char* names, int32_t* launches, double* ms, int32_t keep);

/* Kernels launched by this process since load (all entry points). */
int64_t jev_launch_count(void);

/*
 * jev_debug_set_wait_limit — bound, in SM clock cycles, of every mbarrier
 * wait in the tensor-core kernels (attention and full-vocabulary LSE) launched
 * after the call; 0 restores the default of 2^31 cycles (about a second).  A
 * wait that runs out sets JEV_DEV_WAIT_TIMEOUT in the status word and the CTA
 * winds down: the remaining waits give up, the TMA producer waits for every
 * load it issued and the MMA warp for every MMA it issued, and the kernel
 * returns with its outputs undefined.  Failure handling is tested with a
 * short limit on an ordinary problem, so that waits run out without any GPU
 * fault; the setting is process-wide.  JEV_ERR_INVALID_ARG for cycles < 0.
 * No page has a counterpart: this is the library's failure detection.
 */
jev_status jev_debug_set_wait_limit(int64_t cycles);

/*
 * jev_debug_set_tc_tile_rows — rows per tensor-core work tile for plans made
 * after the call: 128 or 256 forces the one- or the two-Q-tile attention
 * kernel, 0 (the default) lets the plan choose (see jev_attn_plan).  For
 * tests and timing; process-wide.  JEV_ERR_INVALID_ARG for other values.
 */
jev_status jev_debug_set_tc_tile_rows(int32_t rows);

/*
 * jev_debug_set_wait_probe — failure-detection probe.  When on (nonzero),
 * every CTA of the tensor-core kernels launched after the call (attention and
 * full-vocabulary LSE), once its MMA warp has issued its first MMAs, also
 * waits on an mbarrier that nothing completes, as a stalled pipeline would
 * leave it.  That wait is bounded like every other: with the bound of
 * jev_debug_set_wait_limit cut short it runs out, raises
 * JEV_DEV_WAIT_TIMEOUT, and the CTA winds down with loads and MMAs in flight,
 * draining them before it exits; outputs are undefined.  Under the default
 * bound each CTA waits about a second.  Off (0) by default; process-wide.
 * Always JEV_OK.  No page has a counterpart.
 */
jev_status jev_debug_set_wait_probe(int32_t on);

#ifdef __cplusplus
}
#endif
#endif /* JEV_H */
