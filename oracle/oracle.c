/*
 * oracle.c — plain fp64 CPU reference (TEST INFRASTRUCTURE ONLY; see oracle.h).
 *
 * Nothing here is blocked, fused or reordered beyond the definitions it
 * writes out: every branch gets its own materialised [prefix; suffix] key and
 * value list, every readout row gets its full vocabulary of logits, and the
 * trie is built token by token before segments are formed.  OpenMP only runs
 * independent (branch, head) rows or vocabulary rows side by side.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double widen(const void* p, int dtype, size_t i) {
  if (dtype == ORACLE_BF16) {
    uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return (double)((const float*)p)[i];
}

static void set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Rotary position embedding, rotate-half form (pairs i and i + d/2), with the
 * angle of pair i at position p equal to p * theta^(-2i/d).  This is the
 * reading taken for the Qwen-family models the pages name; the pages do not
 * spell RoPE out. */
void oracle_rope(const double* x, double* y, int d, double pos, double theta) {
  int h = d / 2;
  for (int i = 0; i < h; ++i) {
    double inv_freq = pow(theta, -2.0 * (double)i / (double)d);
    double a = pos * inv_freq;
    double c = cos(a), s = sin(a);
    double x0 = x[i], x1 = x[i + h];
    y[i] = x0 * c - x1 * s;
    y[i + h] = x1 * c + x0 * s;
  }
}

/* softmax(scale * q K^T) V over n keys, plus the natural-log normaliser. */
void oracle_attend(const double* q, const double* K, const double* V, int n, int d,
                   int stride, double scale, double* o, double* lse) {
  for (int i = 0; i < d; ++i) o[i] = 0.0;
  if (n <= 0) {
    *lse = -INFINITY;
    return;
  }
  double* s = (double*)malloc(sizeof(double) * (size_t)n);
  double m = -INFINITY;
  for (int t = 0; t < n; ++t) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += q[i] * K[(size_t)t * stride + i];
    s[t] = scale * acc;
    if (s[t] > m) m = s[t];
  }
  double Z = 0.0;
  for (int t = 0; t < n; ++t) {
    s[t] = exp(s[t] - m);
    Z += s[t];
  }
  for (int t = 0; t < n; ++t)
    for (int i = 0; i < d; ++i) o[i] += s[t] * V[(size_t)t * stride + i];
  for (int i = 0; i < d; ++i) o[i] /= Z;
  *lse = m + log(Z);
  free(s);
}

/* ------------------------------------------------------------------------ */
/* Flat shared-prefix attention, computed unshared: for each branch b the key
 * list is [K_pre ; RoPE(K_suf of b)] and suffix query j sees keys 0..Lp+j.   */

int oracle_prefix_suffix_attn(const oracle_attn_problem* p, double* out, double* lse) {
  if (!p || p->B < 0 || p->Lp < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->d <= 0 || (p->d & 1))
    return -1;
  if (!p->head_map && (p->Hq % p->Hkv)) return -1;
  const int32_t* cu = p->cu_seqlens;
  if (p->B > 0 && !cu) return -1;
  if (p->B > 0 && cu[0] != 0) return -1;
  for (int b = 0; b < p->B; ++b)
    if (cu[b + 1] < cu[b]) return -1;
  const int B = p->B, Lp = p->Lp, Hq = p->Hq, Hkv = p->Hkv, d = p->d, G = Hq / Hkv;
  const int T = B > 0 ? cu[B] : 0;
  const double scale = p->scale > 0 ? p->scale : 1.0 / sqrt((double)d);
  const int pos_off = p->pos_offset >= 0 ? p->pos_offset : Lp;
  if (p->head_map)
    for (int h = 0; h < Hq; ++h)
      if (p->head_map[h] < 0 || p->head_map[h] >= Hkv) return -1;

  /* request list per (b, h) task: (j, output slot) */
  const int ntask = B * Hq;
  int* cnt = (int*)calloc((size_t)ntask + 1, sizeof(int));
  int nreq = p->n_rows > 0 ? p->n_rows : T * Hq;
  int* req_j = (int*)malloc(sizeof(int) * (size_t)(nreq > 0 ? nreq : 1));
  int* req_slot = (int*)malloc(sizeof(int) * (size_t)(nreq > 0 ? nreq : 1));
  int* req_task = (int*)malloc(sizeof(int) * (size_t)(nreq > 0 ? nreq : 1));
  for (int r = 0; r < nreq; ++r) {
    int t, h;
    if (p->n_rows > 0) {
      t = p->rows[2 * r];
      h = p->rows[2 * r + 1];
      if (t < 0 || t >= T || h < 0 || h >= Hq) {
        free(cnt); free(req_j); free(req_slot); free(req_task);
        return -1;
      }
    } else {
      t = r / Hq;
      h = r % Hq;
    }
    int b = 0;
    while (cu[b + 1] <= t) ++b; /* branch holding token t */
    req_task[r] = b * Hq + h;
    req_j[r] = t - cu[b];
    cnt[req_task[r] + 1]++;
  }
  for (int i = 0; i < ntask; ++i) cnt[i + 1] += cnt[i];
  int* order = (int*)malloc(sizeof(int) * (size_t)(nreq > 0 ? nreq : 1));
  int* fill = (int*)calloc((size_t)ntask + 1, sizeof(int));
  for (int r = 0; r < nreq; ++r) order[cnt[req_task[r]] + fill[req_task[r]]++] = r;
  (void)req_slot;

  set_threads(p->n_threads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int task = 0; task < ntask; ++task) {
    if (cnt[task + 1] == cnt[task]) continue;
    const int b = task / Hq, h = task % Hq;
    const int g = p->head_map ? p->head_map[h] : h / G;
    const int Ls = cu[b + 1] - cu[b];
    const int n = Lp + Ls;
    double* Kb = (double*)malloc(sizeof(double) * (size_t)n * d);
    double* Vb = (double*)malloc(sizeof(double) * (size_t)n * d);
    double* x = (double*)malloc(sizeof(double) * (size_t)d);
    double* qr = (double*)malloc(sizeof(double) * (size_t)d);
    for (int t = 0; t < Lp; ++t)
      for (int i = 0; i < d; ++i) {
        size_t src = ((size_t)t * Hkv + g) * d + i;
        Kb[(size_t)t * d + i] = widen(p->k_pre, p->dtype, src);
        Vb[(size_t)t * d + i] = widen(p->v_pre, p->dtype, src);
      }
    for (int j = 0; j < Ls; ++j) {
      size_t row = (size_t)(cu[b] + j);
      for (int i = 0; i < d; ++i) {
        x[i] = widen(p->k_suf, p->dtype, (row * Hkv + g) * d + i);
        Vb[(size_t)(Lp + j) * d + i] = widen(p->v_suf, p->dtype, (row * Hkv + g) * d + i);
      }
      oracle_rope(x, Kb + (size_t)(Lp + j) * d, d, (double)(pos_off + j), p->theta);
    }
    for (int k = cnt[task]; k < cnt[task + 1]; ++k) {
      const int r = order[k];
      const int j = req_j[r];
      const size_t row = (size_t)(cu[b] + j);
      for (int i = 0; i < d; ++i) x[i] = widen(p->q, p->dtype, (row * Hq + h) * d + i);
      oracle_rope(x, qr, d, (double)(pos_off + j), p->theta);
      double l;
      size_t slot = p->n_rows > 0 ? (size_t)r : row * Hq + h;
      oracle_attend(qr, Kb, Vb, Lp + j + 1, d, d, scale, out + slot * d, &l);
      if (lse) lse[slot] = l;
    }
    free(Kb); free(Vb); free(x); free(qr);
  }
  free(cnt); free(req_j); free(req_slot); free(req_task); free(order); free(fill);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Generation over per-branch suffix caches: branch b's key list is the prefix,
 * then its cached (already rotated) suffix keys, then its new keys rotated at
 * the positions that follow the cached ones; new token j sees the prefix, the
 * whole cache and new tokens 0..j.                                           */

int oracle_cache_attn(const oracle_cache_problem* p, double* out, double* lse, double* k_new_rot) {
  if (!p || p->B < 0 || p->Lp < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->d <= 0 || (p->d & 1)) return -1;
  if (!p->head_map && (p->Hq % p->Hkv)) return -1;
  const int B = p->B, Lp = p->Lp, Hq = p->Hq, Hkv = p->Hkv, d = p->d, G = Hq / Hkv;
  const int32_t *cu = p->cu_new, *co = p->cache_off, *cl = p->cache_len;
  if (B > 0 && (!cu || !co || !cl || cu[0] != 0)) return -1;
  for (int b = 0; b < B; ++b) {
    if (cu[b + 1] < cu[b] || co[b + 1] < co[b] || co[b] < 0 || cl[b] < 0) return -1;
    if ((long)cl[b] + (cu[b + 1] - cu[b]) > (long)(co[b + 1] - co[b])) return -1;
  }
  if (p->head_map)
    for (int h = 0; h < Hq; ++h)
      if (p->head_map[h] < 0 || p->head_map[h] >= Hkv) return -1;
  const int T = B > 0 ? cu[B] : 0;
  const double scale = p->scale > 0 ? p->scale : 1.0 / sqrt((double)d);
  const int pos_off = p->pos_offset >= 0 ? p->pos_offset : Lp;

  /* the appended keys: new token j of branch b rotated at pos_off + cache_len[b] + j */
  double* x = (double*)malloc(sizeof(double) * (size_t)d);
  for (int b = 0; b < B; ++b)
    for (int t = cu[b]; t < cu[b + 1]; ++t)
      for (int g = 0; g < Hkv; ++g) {
        for (int i = 0; i < d; ++i) x[i] = widen(p->k_new, p->dtype, ((size_t)t * Hkv + g) * d + i);
        oracle_rope(x, k_new_rot + ((size_t)t * Hkv + g) * d, d, (double)(pos_off + cl[b] + (t - cu[b])), p->theta);
      }
  free(x);

  set_threads(p->n_threads);
#pragma omp parallel for schedule(dynamic, 1)
  for (int task = 0; task < B * Hq; ++task) {
    const int b = task / Hq, h = task % Hq;
    const int g = p->head_map ? p->head_map[h] : h / G;
    const int Lc = cl[b], Ln = cu[b + 1] - cu[b];
    if (Ln == 0) continue;
    const int n = Lp + Lc + Ln;
    double* Kb = (double*)malloc(sizeof(double) * (size_t)n * d);
    double* Vb = (double*)malloc(sizeof(double) * (size_t)n * d);
    double* xq = (double*)malloc(sizeof(double) * (size_t)d);
    double* qr = (double*)malloc(sizeof(double) * (size_t)d);
    for (int t = 0; t < Lp; ++t)
      for (int i = 0; i < d; ++i) {
        size_t src = ((size_t)t * Hkv + g) * d + i;
        Kb[(size_t)t * d + i] = widen(p->k_pre, p->dtype, src);
        Vb[(size_t)t * d + i] = widen(p->v_pre, p->dtype, src);
      }
    for (int c = 0; c < Lc; ++c)
      for (int i = 0; i < d; ++i) {
        size_t src = ((size_t)(co[b] + c) * Hkv + g) * d + i;
        Kb[(size_t)(Lp + c) * d + i] = widen(p->k_cache, p->dtype, src);
        Vb[(size_t)(Lp + c) * d + i] = widen(p->v_cache, p->dtype, src);
      }
    for (int j = 0; j < Ln; ++j)
      for (int i = 0; i < d; ++i) {
        size_t src = ((size_t)(cu[b] + j) * Hkv + g) * d + i;
        Kb[(size_t)(Lp + Lc + j) * d + i] = k_new_rot[src];
        Vb[(size_t)(Lp + Lc + j) * d + i] = widen(p->v_new, p->dtype, src);
      }
    for (int j = 0; j < Ln; ++j) {
      const size_t row = (size_t)(cu[b] + j);
      for (int i = 0; i < d; ++i) xq[i] = widen(p->q, p->dtype, (row * Hq + h) * d + i);
      oracle_rope(xq, qr, d, (double)(pos_off + Lc + j), p->theta);
      double l;
      oracle_attend(qr, Kb, Vb, Lp + Lc + j + 1, d, d, scale, out + (row * Hq + h) * d, &l);
      if (lse) lse[row * Hq + h] = l;
    }
    free(Kb); free(Vb); free(xq); free(qr);
  }
  (void)T;
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Candidate readout: logits of the used hidden rows against the LM head, the
 * candidate score as the sum of its (row, token) logits, and a log-softmax
 * over each option set.  Ties pick the lowest candidate index.              */

int oracle_candidate_readout(const oracle_readout_problem* p, double* score, double* logprob,
                             int32_t* choice, double* gap, double* row_lse) {
  if (!p || p->n_sets < 0 || p->n_cands < 0 || p->R < 0 || p->H <= 0 || p->V <= 0) return -1;
  const int n_sets = p->n_sets, n_cands = p->n_cands, R = p->R, H = p->H, V = p->V;
  const int32_t* so = p->set_offsets;
  if (so[0] != 0 || so[n_sets] != n_cands) return -1;
  for (int s = 0; s < n_sets; ++s)
    if (so[s + 1] < so[s]) return -1;
  int n_pairs = p->cand_offsets ? p->cand_offsets[n_cands] : n_cands;
  if (p->cand_offsets && p->cand_offsets[0] != 0) return -1;
  if (p->cand_offsets)
    for (int c = 0; c < n_cands; ++c)
      if (p->cand_offsets[c + 1] < p->cand_offsets[c]) return -1;
  if (n_pairs != p->n_pairs) return -1;

  int* cand_set = (int*)malloc(sizeof(int) * (size_t)(n_cands + 1));
  for (int s = 0; s < n_sets; ++s)
    for (int c = so[s]; c < so[s + 1]; ++c) cand_set[c] = s;
  int* pair_cand = (int*)malloc(sizeof(int) * (size_t)(n_pairs + 1));
  int* prow = (int*)malloc(sizeof(int) * (size_t)(n_pairs + 1));
  for (int c = 0; c < n_cands; ++c) {
    int a = p->cand_offsets ? p->cand_offsets[c] : c;
    int e = p->cand_offsets ? p->cand_offsets[c + 1] : c + 1;
    for (int k = a; k < e; ++k) pair_cand[k] = c;
  }
  int bad = 0;
  int* used = (int*)calloc((size_t)R + 1, sizeof(int));
  unsigned char* pair_ok = (unsigned char*)malloc((size_t)n_pairs + 1);
  for (int k = 0; k < n_pairs; ++k) {
    int r = p->pair_row ? p->pair_row[k] : cand_set[pair_cand[k]];
    int tok = p->pair_tok[k];
    prow[k] = r;
    pair_ok[k] = (r >= 0 && r < R && tok >= 0 && tok < V);
    if (!pair_ok[k]) ++bad;
    else used[r] = 1;
  }
  /* compact list of used rows, widened */
  int nu = 0;
  int* uidx = (int*)malloc(sizeof(int) * (size_t)(R + 1));
  for (int r = 0; r < R; ++r) uidx[r] = used[r] ? nu++ : -1;
  double* hrows = (double*)malloc(sizeof(double) * (size_t)(nu > 0 ? nu : 1) * H);
  for (int r = 0; r < R; ++r)
    if (uidx[r] >= 0)
      for (int i = 0; i < H; ++i) hrows[(size_t)uidx[r] * H + i] = widen(p->hidden, p->dtype, (size_t)r * H + i);
  double* pz = (double*)malloc(sizeof(double) * (size_t)(n_pairs + 1));
  if (row_lse)
    for (int r = 0; r < R; ++r) row_lse[r] = NAN;
  set_threads(p->n_threads);

  if (p->full_vocab && nu > 0) {
    /* every logit of every used row: z[u][v] = <h_u, W[v]> */
    double* z = (double*)malloc(sizeof(double) * (size_t)nu * V);
#pragma omp parallel
    {
      double* w = (double*)malloc(sizeof(double) * (size_t)H);
#pragma omp for schedule(static)
      for (int v = 0; v < V; ++v) {
        for (int i = 0; i < H; ++i) w[i] = widen(p->lm_head, p->dtype, (size_t)v * H + i);
        for (int u = 0; u < nu; ++u) {
          const double* hu = hrows + (size_t)u * H;
          double acc = 0.0;
          for (int i = 0; i < H; ++i) acc += hu[i] * w[i];
          z[(size_t)u * V + v] = acc;
        }
      }
      free(w);
    }
    if (row_lse) {
#pragma omp parallel for schedule(static)
      for (int r = 0; r < R; ++r) {
        if (uidx[r] < 0) continue;
        const double* zu = z + (size_t)uidx[r] * V;
        double m = -INFINITY;
        for (int v = 0; v < V; ++v) if (zu[v] > m) m = zu[v];
        double acc = 0.0;
        for (int v = 0; v < V; ++v) acc += exp(zu[v] - m);
        row_lse[r] = m + log(acc);
      }
    }
    for (int k = 0; k < n_pairs; ++k)
      pz[k] = pair_ok[k] ? z[(size_t)uidx[prow[k]] * V + p->pair_tok[k]] : NAN;
    free(z);
  } else {
#pragma omp parallel for schedule(static)
    for (int k = 0; k < n_pairs; ++k) {
      if (!pair_ok[k]) { pz[k] = NAN; continue; }
      const double* hu = hrows + (size_t)uidx[prow[k]] * H;
      double acc = 0.0;
      for (int i = 0; i < H; ++i) acc += hu[i] * widen(p->lm_head, p->dtype, (size_t)p->pair_tok[k] * H + i);
      pz[k] = acc;
    }
  }

  for (int c = 0; c < n_cands; ++c) {
    int a = p->cand_offsets ? p->cand_offsets[c] : c;
    int e = p->cand_offsets ? p->cand_offsets[c + 1] : c + 1;
    double acc = 0.0;
    for (int k = a; k < e; ++k) acc += pz[k];
    score[c] = acc;
  }
  for (int s = 0; s < n_sets; ++s) {
    int a = so[s], e = so[s + 1];
    if (e == a) { choice[s] = -1; gap[s] = NAN; continue; }
    int any_nan = 0;
    double m = -INFINITY;
    for (int c = a; c < e; ++c) {
      if (isnan(score[c])) any_nan = 1;
      else if (score[c] > m) m = score[c];
    }
    if (any_nan) {
      for (int c = a; c < e; ++c) logprob[c] = NAN;
      choice[s] = -1;
      gap[s] = NAN;
      continue;
    }
    double Z = 0.0;
    for (int c = a; c < e; ++c) Z += exp(score[c] - m);
    double logZ = m + log(Z);
    int best = a;
    for (int c = a; c < e; ++c) {
      logprob[c] = score[c] - logZ;
      if (logprob[c] > logprob[best]) best = c;
    }
    double second = -INFINITY;
    for (int c = a; c < e; ++c)
      if (c != best && logprob[c] > second) second = logprob[c];
    choice[s] = best - a;
    gap[s] = (e - a > 1) ? logprob[best] - second : INFINITY;
  }
  free(cand_set); free(pair_cand); free(prow); free(used); free(pair_ok);
  free(uidx); free(hrows); free(pz);
  return bad;
}

/* ------------------------------------------------------------------------ */
/* Candidate-prefix trie.  Token-level trie first (children kept in the order
 * they were first created), then maximal single-child chains become segment
 * nodes, numbered in DFS preorder.  A chain breaks where a candidate ends, so
 * each candidate's last token is the last token of its leaf segment.        */

typedef struct {
  int32_t* parent; int32_t* tok; int32_t* first; int32_t* last; int32_t* next;
  int32_t* nchild; unsigned char* is_end; int32_t* depth; int32_t* seg; int32_t* packed;
  int n, cap;
} tok_trie;

static int tt_init(tok_trie* t, int cap) {
  memset(t, 0, sizeof *t);
  t->cap = cap;
  t->parent = (int32_t*)malloc(sizeof(int32_t) * cap);
  t->tok = (int32_t*)malloc(sizeof(int32_t) * cap);
  t->first = (int32_t*)malloc(sizeof(int32_t) * cap);
  t->last = (int32_t*)malloc(sizeof(int32_t) * cap);
  t->next = (int32_t*)malloc(sizeof(int32_t) * cap);
  t->nchild = (int32_t*)calloc(cap, sizeof(int32_t));
  t->is_end = (unsigned char*)calloc(cap, 1);
  t->depth = (int32_t*)malloc(sizeof(int32_t) * cap);
  t->seg = (int32_t*)malloc(sizeof(int32_t) * cap);
  t->packed = (int32_t*)malloc(sizeof(int32_t) * cap);
  t->n = 1;
  t->parent[0] = -1; t->tok[0] = -1; t->first[0] = t->last[0] = t->next[0] = -1;
  t->depth[0] = 0; t->seg[0] = 0; t->packed[0] = -1;
  return 0;
}

static void tt_free(tok_trie* t) {
  free(t->parent); free(t->tok); free(t->first); free(t->last); free(t->next);
  free(t->nchild); free(t->is_end); free(t->depth); free(t->seg); free(t->packed);
}

static int tt_child(tok_trie* t, int u, int tok) {
  for (int c = t->first[u]; c >= 0; c = t->next[c])
    if (t->tok[c] == tok) return c;
  int c = t->n++;
  t->parent[c] = u; t->tok[c] = tok; t->first[c] = t->last[c] = t->next[c] = -1;
  t->depth[c] = t->depth[u] + 1; t->seg[c] = -1; t->packed[c] = -1;
  if (t->first[u] < 0) t->first[u] = c;
  else t->next[t->last[u]] = c;
  t->last[u] = c;
  t->nchild[u]++;
  return c;
}

int oracle_trie_build(int n_cands, const int32_t* seq_off, const int32_t* toks, int root_len,
                      int cap_nodes, int cap_toks, int32_t* parent, int32_t* tok_off,
                      int32_t* pos0, int32_t* leaf_of, int32_t* node_toks, int32_t* path_row) {
  if (n_cands < 0 || !seq_off || seq_off[0] != 0 || cap_nodes < 1 || root_len < 0) return -1;
  for (int c = 0; c < n_cands; ++c)
    if (seq_off[c + 1] < seq_off[c]) return -1;
  const int total = seq_off[n_cands];
  tok_trie t;
  tt_init(&t, total + 1);
  int32_t* end_of = (int32_t*)malloc(sizeof(int32_t) * (size_t)(n_cands + 1));
  int32_t* path_tn = (int32_t*)malloc(sizeof(int32_t) * (size_t)(total + 1));
  for (int c = 0; c < n_cands; ++c) {
    int u = 0;
    for (int i = seq_off[c]; i < seq_off[c + 1]; ++i) {
      u = tt_child(&t, u, toks[i]);
      path_tn[i] = u;
    }
    end_of[c] = u;
    if (u != 0) t.is_end[u] = 1;
  }
  /* DFS preorder over segment starts */
  int32_t* stack_u = (int32_t*)malloc(sizeof(int32_t) * (size_t)(t.n + 1));
  int32_t* stack_p = (int32_t*)malloc(sizeof(int32_t) * (size_t)(t.n + 1));
  int32_t* kids = (int32_t*)malloc(sizeof(int32_t) * (size_t)(t.n + 1));
  int sp = 0, n_nodes = 1, cursor = 0, ok = 1;
  parent[0] = -1; pos0[0] = 0; tok_off[0] = 0;
  {
    int nk = 0;
    for (int c = t.first[0]; c >= 0; c = t.next[c]) kids[nk++] = c;
    for (int k = nk - 1; k >= 0; --k) { stack_u[sp] = kids[k]; stack_p[sp] = 0; ++sp; }
  }
  tok_off[1] = 0;
  while (sp > 0 && ok) {
    --sp;
    int u = stack_u[sp], ps = stack_p[sp];
    if (n_nodes >= cap_nodes) { ok = 0; break; }
    int id = n_nodes++;
    parent[id] = ps;
    pos0[id] = root_len + t.depth[u] - 1;
    tok_off[id] = cursor;
    int cur = u;
    for (;;) {
      if (cursor >= cap_toks) { ok = 0; break; }
      node_toks[cursor] = t.tok[cur];
      t.seg[cur] = id;
      t.packed[cur] = cursor;
      ++cursor;
      if (t.nchild[cur] == 1 && !t.is_end[cur]) cur = t.first[cur];
      else break;
    }
    if (!ok) break;
    tok_off[id + 1] = cursor;
    int nk = 0;
    for (int c = t.first[cur]; c >= 0; c = t.next[c]) kids[nk++] = c;
    for (int k = nk - 1; k >= 0; --k) { stack_u[sp] = kids[k]; stack_p[sp] = id; ++sp; }
  }
  if (ok) {
    for (int c = 0; c < n_cands; ++c) leaf_of[c] = end_of[c] ? t.seg[end_of[c]] : 0;
    if (path_row)
      for (int i = 0; i < total; ++i) path_row[i] = t.packed[path_tn[i]];
  }
  free(stack_u); free(stack_p); free(kids); free(end_of); free(path_tn);
  tt_free(&t);
  return ok ? n_nodes : -1;
}

/* ------------------------------------------------------------------------ */
/* Tree attention: node n's rows are the last len(n) rows of one flat branch
 * whose suffix is the token path from the root's child down to node n.      */

int oracle_tree_attn(const oracle_tree_problem* p, double* out, double* lse) {
  if (!p || p->n_nodes < 1 || p->Hq <= 0 || p->Hkv <= 0 || p->d <= 0 || (p->d & 1)) return -1;
  if (!p->head_map && p->Hq % p->Hkv) return -1;
  const int nn = p->n_nodes, Lp = p->Lp, Hq = p->Hq, Hkv = p->Hkv, d = p->d, G = Hq / Hkv;
  const double scale = p->scale > 0 ? p->scale : 1.0 / sqrt((double)d);
  if (p->parent[0] != -1 || p->tok_off[0] != 0 || p->tok_off[1] != 0 || p->tok_off[nn] != p->N) return -1;
  for (int n = 1; n < nn; ++n)
    if (p->parent[n] < 0 || p->parent[n] >= n || p->tok_off[n + 1] < p->tok_off[n]) return -1;
  const int ntask = nn * Hq;
  set_threads(p->n_threads);
  int status = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int task = Hq; task < ntask; ++task) {
    const int n = task / Hq, h = task % Hq;
    const int g = p->head_map ? p->head_map[h] : h / G;
    /* collect the chain root -> n */
    int depth = 0;
    for (int a = n; a > 0; a = p->parent[a]) ++depth;
    int* chain = (int*)malloc(sizeof(int) * (size_t)depth);
    { int k = depth; for (int a = n; a > 0; a = p->parent[a]) chain[--k] = a; }
    int plen = 0;
    for (int k = 0; k < depth; ++k) plen += p->tok_off[chain[k] + 1] - p->tok_off[chain[k]];
    int* path = (int*)malloc(sizeof(int) * (size_t)(plen > 0 ? plen : 1));
    { int w = 0; for (int k = 0; k < depth; ++k) for (int r = p->tok_off[chain[k]]; r < p->tok_off[chain[k] + 1]; ++r) path[w++] = r; }
    const int nkeys = Lp + plen;
    double* Kb = (double*)malloc(sizeof(double) * (size_t)nkeys * d);
    double* Vb = (double*)malloc(sizeof(double) * (size_t)nkeys * d);
    double* x = (double*)malloc(sizeof(double) * (size_t)d);
    double* qr = (double*)malloc(sizeof(double) * (size_t)d);
    for (int t = 0; t < Lp; ++t)
      for (int i = 0; i < d; ++i) {
        size_t src = ((size_t)t * Hkv + g) * d + i;
        Kb[(size_t)t * d + i] = widen(p->k_root, p->dtype, src);
        Vb[(size_t)t * d + i] = widen(p->v_root, p->dtype, src);
      }
    for (int j = 0; j < plen; ++j) {
      size_t row = (size_t)path[j];
      for (int i = 0; i < d; ++i) {
        x[i] = widen(p->k, p->dtype, (row * Hkv + g) * d + i);
        Vb[(size_t)(Lp + j) * d + i] = widen(p->v, p->dtype, (row * Hkv + g) * d + i);
      }
      oracle_rope(x, Kb + (size_t)(Lp + j) * d, d, (double)(Lp + j), p->theta);
    }
    const int len_n = p->tok_off[n + 1] - p->tok_off[n];
    for (int j = plen - len_n; j < plen; ++j) {
      size_t row = (size_t)path[j];
      for (int i = 0; i < d; ++i) x[i] = widen(p->q, p->dtype, (row * Hq + h) * d + i);
      oracle_rope(x, qr, d, (double)(Lp + j), p->theta);
      double l;
      oracle_attend(qr, Kb, Vb, Lp + j + 1, d, d, scale, out + (row * Hq + h) * d, &l);
      if (lse) lse[row * Hq + h] = l;
    }
    free(chain); free(path); free(Kb); free(Vb); free(x); free(qr);
  }
  return status;
}
