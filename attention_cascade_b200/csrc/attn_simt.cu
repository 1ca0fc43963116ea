// attn_simt.cu — CUDA-core attention over [prefix split ; own suffix window]
// for the stacked rows of one kv group.  Used for fp32 inputs, where the
// tensor-core kernel does not apply.
//
// Each block holds 16 stacked rows (row m of group g is token m / G, query
// slot m % G) and streams 32-key tiles of the prefix split through shared
// memory, the next tile's K and V loaded into registers while the current one
// is computed; one warp owns four rows, a lane owns one key of the tile for
// the scores and d/32 output columns for P.V.  The online softmax runs in the
// log2 domain.  The block that holds the last prefix split also walks the
// suffix keys its rows may see: for a flat branch, the keys of the same branch
// up to the row's own token (or its slot in the branch's cache); for a tree
// token, every non-root ancestor's keys plus its own node's keys up to itself.
#include <math_constants.h>

#include "kernels.h"

namespace jev {
namespace {

constexpr int kRows = 16;   // stacked rows per block
constexpr int kKeys = 32;   // keys per tile
constexpr int kThreads = 128;

template <typename T, int D>
__global__ void __launch_bounds__(kThreads) attn_simt_kernel(AttnArgs a) {
  constexpr int C = D / 32;  // output columns per lane
  __shared__ float Qs[kRows][D];
  __shared__ float Ks[kKeys][D + 1];
  __shared__ float Vs[kKeys][D];
  __shared__ int r_t[kRows], r_start[kRows], r_last[kRows];
  __shared__ int s_lo, s_hi;
  const bool tree = a.key_end != nullptr;

  const int g = blockIdx.y, split = blockIdx.z;
  const int m0 = blockIdx.x * kRows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const T* qg = reinterpret_cast<const T*>(a.q_rot) + (size_t)g * a.M * D;

  for (int e = tid; e < kRows * D; e += kThreads) {
    int r = e / D, i = e - r * D;
    int m = m0 + r;
    Qs[r][i] = m < a.M ? to_f32(qg[(size_t)m * D + i]) : 0.f;
  }
  if (tid < kRows) {
    int m = m0 + tid;
    r_t[tid] = -1;
    r_start[tid] = 0;
    r_last[tid] = -1;
    if (m < a.M) {
      const int t = m / a.G;
      const TokInfo inf = a.info[t];
      if (inf.node >= 0) {  // a skipped row sees no suffix keys and is not written
        r_t[tid] = t;
        r_start[tid] = inf.seg_start;
        r_last[tid] = tree ? t : inf.last;
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    int lo = INT_MAX, hi = -1;
    for (int r = 0; r < kRows; ++r) {
      if (r_t[r] < 0) continue;
      lo = min(lo, r_start[r]);
      hi = max(hi, r_last[r]);
    }
    s_lo = lo;
    s_hi = hi;
  }

  float m_r[4], l_r[4], acc[4][C];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m_r[r] = -CUDART_INF_F;
    l_r[r] = 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) acc[r][c] = 0.f;
  }

  // The key tiles of this block, in order: the prefix split, then (for the
  // last split) the suffix window.  Each thread stages kPer elements of a
  // tile's K and of its V; the next tile's are loaded into registers before
  // the current tile is computed.
  constexpr int kPer = kKeys * D / kThreads;
  const T* kp = reinterpret_cast<const T*>(a.k_pre) + (size_t)g * D;
  const T* vp = reinterpret_cast<const T*>(a.v_pre) + (size_t)g * D;
  const T* ks = reinterpret_cast<const T*>(a.k_rot) + (size_t)g * D;
  const T* vs = reinterpret_cast<const T*>(a.v_suf) + (size_t)g * D;
  const int p_lo = split * a.split_len;
  const int p_hi = min(a.Lp, p_lo + a.split_len);
  const int n_pre = p_hi > p_lo ? (p_hi - p_lo + kKeys - 1) / kKeys : 0;
  __syncthreads();  // the window (s_lo, s_hi) is published
  const int lo = s_lo, hi = s_hi;
  const int n_suf = split == a.S - 1 && lo <= hi ? (hi - lo + kKeys) / kKeys : 0;
  // tile i: keys [kb, kb + n) of (Kg, Vg); suffix tiles after the prefix ones
  auto tile_src = [&](int i, const T*& Kg, const T*& Vg, int& kb, int& n) {
    if (i < n_pre) {
      Kg = kp; Vg = vp; kb = p_lo + i * kKeys; n = min(kKeys, p_hi - kb);
    } else {
      Kg = ks; Vg = vs; kb = lo + (i - n_pre) * kKeys; n = min(kKeys, hi + 1 - kb);
    }
  };
  float kr[kPer], vr[kPer];
  auto fetch = [&](int i) {
    const T* Kg; const T* Vg; int kb, n;
    tile_src(i, Kg, Vg, kb, n);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + u * kThreads;
      const int j = e / D, c = e - j * D;
      const bool ok = j < n;
      const size_t off = ((size_t)(kb + j) * a.Hkv) * D + c;
      kr[u] = ok ? to_f32(Kg[off]) : 0.f;
      vr[u] = ok ? to_f32(Vg[off]) : 0.f;
    }
  };
  const int n_tiles = n_pre + n_suf;
  if (n_tiles > 0) fetch(0);
  for (int i = 0; i < n_tiles; ++i) {
    const T* Kg_; const T* Vg_; int kb, n;
    tile_src(i, Kg_, Vg_, kb, n);
    const bool suffix = i >= n_pre;
    __syncthreads();  // every warp is done with the previous tile
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + u * kThreads;
      const int j = e / D, c = e - j * D;
      Ks[j][c] = kr[u];
      Vs[j][c] = vr[u];
    }
    __syncthreads();
    if (i + 1 < n_tiles) fetch(i + 1);  // in flight while this tile is computed
    float p[4];
    const int key = kb + lane;
    // tree key: the end of the packed tokens of its node's subtree
    const int kend = suffix && tree && lane < n ? a.key_end[key] : -1;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int rr = warp * 4 + r;
      float sc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) sc += Qs[rr][c] * Ks[lane][c];
      sc *= a.scale_log2;
      bool ok = lane < n && r_t[rr] >= 0;
      if (ok && suffix)
        ok = tree ? (key <= r_t[rr] && r_t[rr] < kend) : (key >= r_start[rr] && key <= r_last[rr]);
      sc = ok ? sc : -CUDART_INF_F;
      const float mx = warp_max(sc);
      const float m_new = fmaxf(m_r[r], mx);
      float alpha, pv;
      if (m_new == -CUDART_INF_F) {
        alpha = 1.f;
        pv = 0.f;
      } else {
        alpha = exp2f(m_r[r] - m_new);
        pv = exp2f(sc - m_new);
      }
      l_r[r] = l_r[r] * alpha + warp_sum(pv);
      m_r[r] = m_new;
#pragma unroll
      for (int c = 0; c < C; ++c) acc[r][c] *= alpha;
      p[r] = pv;
    }
    for (int j = 0; j < kKeys; ++j) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float pj = __shfl_sync(0xffffffffu, p[r], j);
#pragma unroll
        for (int c = 0; c < C; ++c) acc[r][c] += pj * Vs[j][lane + 32 * c];
      }
    }
  }

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int rr = warp * 4 + r;
    const int m = m0 + rr;
    if (m >= a.M || r_t[rr] < 0) continue;
    const float inv = l_r[r] > 0.f ? 1.f / l_r[r] : 0.f;
    const float lse2 = l_r[r] > 0.f ? m_r[r] + log2f(l_r[r]) : -CUDART_INF_F;
    if (a.S == 1) {
      const int t = m / a.G;
      const int h = min(max(a.hinv[g * a.G + (m - t * a.G)], 0), a.Hq - 1);
      T* o = reinterpret_cast<T*>(a.out) + ((size_t)t * a.Hq + h) * D;
#pragma unroll
      for (int c = 0; c < C; ++c) o[lane + 32 * c] = from_f32<T>(acc[r][c] * inv);
      if (a.lse && lane == 0) a.lse[(size_t)t * a.Hq + h] = lse2 * 0.69314718055994531f;
    } else {
      float* o = a.o_part + (((size_t)split * a.Hkv + g) * a.M + m) * D;
#pragma unroll
      for (int c = 0; c < C; ++c) o[lane + 32 * c] = acc[r][c] * inv;
      if (lane == 0) a.l_part[((size_t)split * a.Hkv + g) * a.M + m] = lse2;
    }
  }
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, jev_dtype dt, cudaStream_t s) {
  dim3 grid((a.M + kRows - 1) / kRows, a.Hkv, a.S);
  if (a.M == 0) return cudaSuccess;
  if (dt == JEV_BF16) {
    if (a.d == 64) attn_simt_kernel<__nv_bfloat16, 64><<<grid, kThreads, 0, s>>>(a);
    else attn_simt_kernel<__nv_bfloat16, 128><<<grid, kThreads, 0, s>>>(a);
  } else {
    if (a.d == 64) attn_simt_kernel<float, 64><<<grid, kThreads, 0, s>>>(a);
    else attn_simt_kernel<float, 128><<<grid, kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace jev
