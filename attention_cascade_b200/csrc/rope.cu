// rope.cu — RoPE of the suffix (or tree) tokens, group-major query packing,
// per-token window info, and the tree ancestor plan.
//
// Positions continue from the prefix: branch token j sits at pos_offset + j
// ("FastJEV: Understanding Redundancy for Compact JEV Inference", TL;DR and
// §3.3 — sharing is valid only at identical positions).  RoPE itself is the
// rotate-half form with angle p * theta^(-2i/d); the angle and its cosine and
// sine are formed in double and rounded once to float.
#include "kernels.h"

namespace jev {
namespace {

template <typename T>
__global__ void __launch_bounds__(256) rope_pack_kernel(RopePackArgs a) {
  const int t = blockIdx.x;
  const int half = a.d >> 1;
  const int G = a.Hq / a.Hkv;
  __shared__ float cs[128], sn[128];
  __shared__ int s_slot[256], s_grp[256];
  __shared__ int s_start, s_pos, s_seg;

  if (threadIdx.x == 0) {
    int seg = upper_segment(a.offs, a.n_segs, t);
    int start = a.offs[seg];
    if (start > t) start = t;
    if (start < 0) start = 0;
    int base = a.pos0 ? a.pos0[seg] : a.pos_offset;
    s_seg = seg;
    s_start = start;
    s_pos = base + (t - start);
  }
  // group and slot of every query head
  for (int h = threadIdx.x; h < a.Hq; h += blockDim.x) {
    int g = a.head_map ? a.head_map[h] : h / G;
    if (g < 0 || g >= a.Hkv) {
      if (t == 0) raise_flag(a.status, JEV_DEV_BAD_HEAD_MAP);
      g = 0;
    }
    s_grp[h] = g;
  }
  // block 0 owns the inverse table: identity first, so every entry stays a
  // valid head index even when a malformed map leaves a slot unclaimed
  if (t == 0)
    for (int h = threadIdx.x; h < a.Hq; h += blockDim.x) a.hinv[h] = h;
  __syncthreads();
  for (int h = threadIdx.x; h < a.Hq; h += blockDim.x) {
    int g = s_grp[h], slot = 0;
    for (int h2 = 0; h2 < h; ++h2) slot += (s_grp[h2] == g);
    if (slot >= G) {
      if (t == 0) raise_flag(a.status, JEV_DEV_BAD_HEAD_MAP);
      slot = G - 1;
    }
    s_slot[h] = slot;
    if (t == 0) a.hinv[g * G + slot] = h;
  }
  if (t == 0) {
    // offsets must start at 0, never decrease and end at T
    for (int i = threadIdx.x; i < a.n_segs; i += blockDim.x)
      if (a.offs[i + 1] < a.offs[i]) raise_flag(a.status, JEV_DEV_BAD_SEQLENS);
    if (threadIdx.x == 0 && (a.offs[0] != 0 || a.offs[a.n_segs] != a.T)) raise_flag(a.status, JEV_DEV_BAD_SEQLENS);
  }
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    double inv_freq = pow(a.theta, -2.0 * (double)i / (double)a.d);
    double ang = (double)s_pos * inv_freq;
    double sv, cv;
    sincos(ang, &sv, &cv);
    cs[i] = (float)cv;
    sn[i] = (float)sv;
  }
  __syncthreads();
  const T* q = reinterpret_cast<const T*>(a.q) + (size_t)t * a.Hq * a.d;
  T* qr = reinterpret_cast<T*>(a.q_rot);
  const size_t M = (size_t)a.T * G;
  for (int e = threadIdx.x; e < a.Hq * half; e += blockDim.x) {
    int h = e / half, i = e - h * half;
    float x0 = to_f32(q[h * a.d + i]), x1 = to_f32(q[h * a.d + i + half]);
    float c = cs[i], s = sn[i];
    T* dst = qr + ((size_t)s_grp[h] * M + (size_t)t * G + s_slot[h]) * a.d;
    dst[i] = from_f32<T>(x0 * c - x1 * s);
    dst[i + half] = from_f32<T>(x1 * c + x0 * s);
  }
  const T* k = reinterpret_cast<const T*>(a.k) + (size_t)t * a.Hkv * a.d;
  T* kr = reinterpret_cast<T*>(a.k_rot) + (size_t)t * a.Hkv * a.d;
  for (int e = threadIdx.x; e < a.Hkv * half; e += blockDim.x) {
    int g = e / half, i = e - g * half;
    float x0 = to_f32(k[g * a.d + i]), x1 = to_f32(k[g * a.d + i + half]);
    float c = cs[i], s = sn[i];
    kr[g * a.d + i] = from_f32<T>(x0 * c - x1 * s);
    kr[g * a.d + i + half] = from_f32<T>(x1 * c + x0 * s);
  }
  if (threadIdx.x == 0) a.info[t] = TokInfo{s_start, s_pos, s_seg, 0};
}

// One thread per node: walk up to the root (parents must precede children, at
// most kMaxDepth non-root levels) and record the ancestors' packed key ranges.
__global__ void tree_plan_kernel(TreePlanArgs a) {
  int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= a.n_nodes) return;
  if (n == 0) {
    if (a.parent[0] != -1 || a.tok_off[0] != 0 || a.tok_off[1] != 0 || a.tok_off[a.n_nodes] != a.N)
      raise_flag(a.status, JEV_DEV_BAD_TREE);
    a.node_nanc[0] = 0;
    return;
  }
  int chain[kMaxDepth];
  int depth = 0, cur = n, ok = 1;
  while (cur > 0) {
    if (depth >= kMaxDepth) { ok = 0; break; }
    chain[depth++] = cur;
    int p = a.parent[cur];
    if (p < 0 || p >= cur) { ok = 0; break; }
    if (a.tok_off[cur + 1] < a.tok_off[cur] || a.tok_off[cur] < 0 || a.tok_off[cur + 1] > a.N) { ok = 0; break; }
    cur = p;
  }
  int2* anc = a.node_anc + (size_t)n * kMaxDepth;
  if (!ok) {
    raise_flag(a.status, JEV_DEV_BAD_TREE);
    a.node_nanc[n] = -1;  // rows of this node are skipped
    return;
  }
  // chain[0] = n itself; ancestors are chain[depth-1] (root side) .. chain[1]
  int w = 0;
  for (int k = depth - 1; k >= 1; --k) anc[w++] = make_int2(a.tok_off[chain[k]], a.tok_off[chain[k] + 1]);
  a.node_nanc[n] = w;
}

template <typename T>
__global__ void rope_inplace_kernel(T* x, int L, int H, int d, int pos0, double theta) {
  int t = blockIdx.x;
  int half = d >> 1;
  __shared__ float cs[128], sn[128];
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    double ang = (double)(pos0 + t) * pow(theta, -2.0 * (double)i / (double)d);
    double sv, cv;
    sincos(ang, &sv, &cv);
    cs[i] = (float)cv;
    sn[i] = (float)sv;
  }
  __syncthreads();
  T* row = x + (size_t)t * H * d;
  for (int e = threadIdx.x; e < H * half; e += blockDim.x) {
    int h = e / half, i = e - h * half;
    float x0 = to_f32(row[h * d + i]), x1 = to_f32(row[h * d + i + half]);
    row[h * d + i] = from_f32<T>(x0 * cs[i] - x1 * sn[i]);
    row[h * d + i + half] = from_f32<T>(x1 * cs[i] + x0 * sn[i]);
  }
}

}  // namespace

cudaError_t launch_rope_pack(const RopePackArgs& a, jev_dtype dt, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  if (dt == JEV_BF16) rope_pack_kernel<__nv_bfloat16><<<a.T, 256, 0, s>>>(a);
  else rope_pack_kernel<float><<<a.T, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_tree_plan(const TreePlanArgs& a, cudaStream_t s) {
  tree_plan_kernel<<<(a.n_nodes + 127) / 128, 128, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_rope_inplace(void* x, int L, int H, int d, int pos0, double theta, jev_dtype dt,
                                cudaStream_t s) {
  if (L == 0) return cudaSuccess;
  if (dt == JEV_BF16) rope_inplace_kernel<<<L, 256, 0, s>>>((__nv_bfloat16*)x, L, H, d, pos0, theta);
  else rope_inplace_kernel<<<L, 256, 0, s>>>((float*)x, L, H, d, pos0, theta);
  return cudaGetLastError();
}

}  // namespace jev
