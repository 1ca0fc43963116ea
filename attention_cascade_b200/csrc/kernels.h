// kernels.h — launchers of the jev kernels (internal to the library).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace jev {

// Rotate the packed suffix (or tree) tokens and lay queries out group-major:
// q_rot[g][t*G + slot(h)][:] = RoPE(q[t][h][:]), k_rot[t][g][:] = RoPE(k[t][g][:]).
struct RopePackArgs {
  const void* q;           // [T, Hq, d]
  const void* k;           // [T, Hkv, d]
  void* q_rot;             // [Hkv, T*G, d]
  void* k_rot;             // [T, Hkv, d]; cache mode: the key cache [key_rows, Hkv, d]
  TokInfo* info;           // [T]
  int32_t* hinv;           // [Hq]: q-head of group-major slot g*G + s
  int32_t* status;
  const int32_t* offs;     // flat: cu_seqlens [n_segs+1]; tree: tok_off [n_segs+1]
  const int32_t* pos0;     // tree: [n_segs] first-token positions; flat: nullptr
  const int32_t* head_map; // [Hq] or nullptr
  // tree: the parent of every node, and per token (written) the end of the
  // packed tokens of its node's subtree, for the key side of the mask
  const int32_t* parent;
  int32_t* key_end;
  // cache mode (a generation step over per-branch suffix caches): branch b
  // owns cache rows [cache_off[b], cache_off[b+1]) of which cache_len[b] are
  // filled; its new tokens go to the rows after them
  const int32_t* cache_off;  // [n_segs+1] or nullptr
  const int32_t* cache_len;  // [n_segs]
  const void* v;             // cache mode: new values [T, Hkv, d]
  void* v_cache;             // cache mode: value cache [key_rows, Hkv, d]
  int key_rows;              // rows of the key tensor the attention reads
  int n_segs, T, Hq, Hkv, d, pos_offset;
  int pos_seq;             // 1: token t at pos_offset + t (sequential across segments)
  double theta;
  double inv_freq[128];    // theta^(-2i/d), i < d/2, formed on the host in double
};
cudaError_t launch_rope_pack(const RopePackArgs& a, jev_dtype dt, cudaStream_t s);



// Attention over [prefix split s ; own suffix window] for the stacked rows of a kv group.
struct AttnArgs {
  const void* q_rot;        // [Hkv, M, d]
  const void* k_pre;        // [Lp, Hkv, d]
  const void* v_pre;        // [Lp, Hkv, d]
  const void* k_rot;        // [key_rows, Hkv, d] rotated suffix keys (or the key cache)
  const void* v_suf;        // [key_rows, Hkv, d]
  const TokInfo* info;      // [T]
  const int32_t* key_end;   // tree: [T] subtree token end of each key's node; flat: nullptr
  const int32_t* hinv;      // [Hq]
  void* out;                // [T, Hq, d] (num_splits == 1)
  float* lse;               // [T, Hq] or nullptr
  float* o_part;            // [S, Hkv, M, d] (num_splits > 1)
  float* l_part;            // [S, Hkv, M] log2-domain
  int32_t* status;
  int T, M, Lp, Hq, Hkv, G, d, S, split_len;  // split_len: prefix keys per split (CUDA-core kernel: a multiple of 32)
  int key_rows;             // rows of k_rot / v_suf
  float scale_log2;         // softmax scale * log2(e)
  // Tensor-core schedule.  Work tile w = (kv group w / n_mt, tile_rows-row
  // tile w % n_mt of its stacked rows; 256 rows run on the two-Q-tile kernel,
  // 128 on the one-Q-tile kernel) has P = n_pre + 1 units (one per 128-key prefix tile, one for
  // the suffix window).  The first full_waves * n_ctas tiles go whole, tile
  // c + k * n_ctas to CTA c; the U units of the remaining (tail) tiles,
  // counted from tile tail0 = full_waves * n_ctas, are spread evenly over the
  // first tail_ctas CTAs: CTA c < tail_ctas owns tail units
  // [c*U/tail_ctas, (c+1)*U/tail_ctas) after its whole tiles.
  int tile_rows, n_mt, n_tiles, n_pre, P, n_ctas, full_waves, tail0, tail_ctas;
  long long U;
  long long wait_cycles;  // bound of every mbarrier wait (clock cycles)
  int wait_probe;         // failure-detection probe: the MMA warp also waits on a barrier nothing completes
};
// tail units owned by CTAs before c (c <= tail_ctas)
__host__ __device__ inline long long tc_unit_begin(const AttnArgs& a, int c) { return (long long)c * a.U / a.tail_ctas; }
// CTA owning tail unit u: the largest c with tc_unit_begin(c) <= u
__host__ __device__ inline int tc_cta_of(const AttnArgs& a, long long u) { return (int)(((u + 1) * a.tail_ctas - 1) / a.U); }
cudaError_t launch_attn_simt(const AttnArgs& a, jev_dtype dt, cudaStream_t s);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s);   // bf16, d in {64,128}; by a.tile_rows:
cudaError_t launch_attn_tc1(const AttnArgs& a, cudaStream_t s);  // the one-Q-tile kernel (tile_rows 128)
// merge the partial segments of work tiles that the schedule split across CTAs
cudaError_t launch_tc_fixup(const AttnArgs& a, cudaStream_t s);
bool attn_tc_supported(int d);
cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t s);

struct MergeArgs {
  const float* o_part;  // [S, Hkv, M, d]
  const float* l_part;  // [S, Hkv, M]
  const TokInfo* info;  // [T]: rows of skipped tokens (node < 0) are not written
  const int32_t* hinv;
  void* out;            // [T, Hq, d]
  float* lse;
  int M, Hq, Hkv, G, d, S;
};
cudaError_t launch_merge(const MergeArgs& a, jev_dtype dt, cudaStream_t s);

struct ReadoutArgs {
  const void* hidden; const void* lm_head;
  const int32_t* set_offsets; const int32_t* cand_offsets; const int32_t* pair_row; const int32_t* pair_tok;
  float* logprob; int32_t* choice; float* score;
  int n_sets, n_cands, n_pairs, R, H, V;
  const float* row_lse;  // [R] or null: each pair's term becomes logit - row_lse[row]
};
// *n_kernels: how many kernels the call launched (1 or 2)
cudaError_t launch_readout(const ReadoutArgs& a, jev_dtype dt, cudaStream_t s, int* n_kernels);

// Full-vocabulary log-sum-exp of bf16 hidden rows (vocab_lse.cu).
struct VocabLseArgs {
  const void* hidden; const void* lm_head;
  int R, H, V, n_vtiles;
  float2* part;  // [ceil(R/256)][n_ctas][2][256] (max, sum) partials, log2 domain
  float* lse;    // [R] natural log
  int32_t* status;
  long long wait_cycles;  // bound of every mbarrier wait (clock cycles)
  int wait_probe;         // failure-detection probe: the MMA warp also waits on a barrier nothing completes
};
int vocab_lse_ctas(int V, int sms);
size_t vocab_lse_partial_bytes(int R, int n_ctas);
cudaError_t launch_vocab_lse(const VocabLseArgs& a, int n_ctas, cudaStream_t s);

cudaError_t launch_rope_inplace(void* x, int L, int H, int d, int pos0, double theta, jev_dtype dt,
                                cudaStream_t s);

}  // namespace jev
