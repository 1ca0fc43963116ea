// rope.cu — RoPE of the suffix (or tree) tokens, group-major query packing,
// per-token window info, (tree) the plan of each token's node, and (cache mode) the
// append of the new tokens' rotated keys and values to per-branch caches.
//
// Positions continue from the prefix: branch token j sits at pos_offset + j
// ("FastJEV: Understanding Redundancy for Compact JEV Inference", TL;DR and
// §3.3 — sharing is valid only at identical positions).  RoPE itself is the
// rotate-half form with angle p * theta^(-2i/d); the angle and its cosine and
// sine are formed in double and rounded once to float.
#include "kernels.h"

namespace jev {
namespace {

// 8 fp32 values stored as 8 consecutive elements of T (one 16-byte store for bf16, two for fp32).
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 v;
  uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
    w[k] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = v;
}
__device__ __forceinline__ void store8(float* p, const float (&f)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// 8 consecutive elements as one raw vector (16 bytes for bf16, 32 for fp32)
struct F8 { float4 a, b; };
template <typename T> struct RawVec;
template <> struct RawVec<__nv_bfloat16> { using type = uint4; };
template <> struct RawVec<float> { using type = F8; };
__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 x = __bfloat1622float2(h[k]);
    f[2 * k] = x.x;
    f[2 * k + 1] = x.y;
  }
}
__device__ __forceinline__ void unpack8(const F8& v, float (&f)[8]) {
  f[0] = v.a.x; f[1] = v.a.y; f[2] = v.a.z; f[3] = v.a.w; f[4] = v.b.x; f[5] = v.b.y; f[6] = v.b.z; f[7] = v.b.w;
}

constexpr int kPackWarps = 4;  // warps per block

// Tree plan of node m, computed by the warp of each of m's tokens (nodes in
// depth-first preorder, packed tokens in node order).  The keys a token of m
// may see beyond the root are the tokens of m's ancestors and its own, all of
// which lie in [first token of m's top-level ancestor, the token itself]; a
// key of node a is visible to a token t exactly when a's subtree, whose tokens
// are the contiguous range [tok_off[a], tok_off[e(a)]), contains t and the key
// is not after t.  Checks: the parent precedes the node and every node
// between the two descends from the parent (preorder), token offsets are in
// order; a node that fails is flagged and its rows are skipped.  The scans
// read 32 nodes per step; their length is the node's distance to its parent,
// to the end of its subtree and to its top-level ancestor, in node order.
struct NodePlan {
  int start;  // first key of the node's rows' windows; -1: malformed
  int end;    // end of the packed tokens of the node's subtree
};
__device__ NodePlan plan_node(const RopePackArgs& a, int m, int lane) {
  const int32_t* parent = a.parent;
  const int32_t* tok_off = a.offs;
  const int n = a.n_segs;
  NodePlan r{-1, -1};
  if (m <= 0 || m >= n) return r;
  const int p = parent[m];
  bool ok = p >= 0 && p < m && tok_off[m] >= 0 && tok_off[m] <= tok_off[m + 1] && tok_off[m + 1] <= a.T;
  if (ok) {
    bool bad = false;
    for (int j0 = p + 1; j0 < m; j0 += 32) {
      const int j = j0 + lane;
      bad |= j < m && parent[j] < p;
    }
    ok = !__any_sync(0xffffffffu, bad);
  }
  // the subtree is nodes m .. e-1: e is the first later node whose parent precedes m
  int e = n;
  for (int j0 = m + 1; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    const unsigned hit = __ballot_sync(0xffffffffu, j < n && parent[j] < m);
    if (hit) {
      e = j0 + __ffs(hit) - 1;
      break;
    }
  }
  // the top-level ancestor: the last node at or before m whose parent is the root
  int top = 0;
  for (int j0 = m; j0 > 0; j0 -= 32) {
    const int j = j0 - lane;
    const unsigned hit = __ballot_sync(0xffffffffu, j > 0 && parent[j] == 0);
    if (hit) {
      top = j0 - (__ffs(hit) - 1);
      break;
    }
  }
  ok = ok && top > 0;
  if (ok) {
    r.start = min(max(tok_off[top], 0), a.T);
    r.end = min(max(tok_off[e], 0), a.T);
  }
  return r;
}

// Segment of token t: the largest s < n with offs[s] <= t, by a 32-ary
// search of the warp over offs in global memory (one load per lane and round;
// two rounds up to 1024 segments).  Malformed offsets give some s < n.
__device__ __forceinline__ int warp_upper_segment(const int32_t* offs, int n, int t, int lane) {
  int lo = 0;
  while (n > 32) {
    const int step = (n + 31) / 32;
    const int idx = lo + lane * step;
    const unsigned b = __ballot_sync(0xffffffffu, lane * step < n && offs[idx] <= t);
    const int k = b ? 31 - __clz((int)b) : 0;
    lo += k * step;
    n = min(step, n - k * step);
  }
  const unsigned b = __ballot_sync(0xffffffffu, lane < n && offs[lo + lane] <= t);
  return lo + (b ? 31 - __clz((int)b) : 0);
}

// kv group and slot (the query head's place among its group's heads, in head
// order) of query head h
__device__ __forceinline__ void head_slot(const RopePackArgs& a, int G, int h, int& g, int& slot) {
  if (!a.head_map) {
    g = h / G;
    slot = h - g * G;
    return;
  }
  g = a.head_map[h];
  if (g < 0 || g >= a.Hkv) g = 0;  // flagged by block 0
  slot = 0;
  for (int h2 = 0; h2 < h; ++h2) {
    int g2 = a.head_map[h2];
    if (g2 < 0 || g2 >= a.Hkv) g2 = 0;
    slot += g2 == g;
  }
  slot = min(slot, G - 1);  // an uneven map is flagged by block 0
}

// Work item = (token t, chunk c of its Hq + Hkv heads): a warp loads its
// chunk's heads first, then locates the token (segment, position; for a tree
// its node plan, for a generation step its cache row), forms the cosines and
// sines of the token's angles (double angle, rounded once to float) and
// rotates its heads, 8 pair indices per lane and head with 16-byte accesses.
// The chunks of a token are consecutive warps; the token's info (and its
// node plan or cache bookkeeping) is written by the warp of chunk 0.  No
// block-wide barrier outside block 0, which also checks the inputs and
// writes the inverse head table.
// kChunkIt: head iterations per warp (4 or 8 heads per iteration at d = 128
// or 64).  Two iterations give the most parallel, shortest chains for a
// few thousand tokens; four keep more bytes in flight per warp when the grid
// is several waves deep.
template <typename T, int kChunkIt>
__global__ void __launch_bounds__(kPackWarps * 32) rope_pack_kernel(RopePackArgs a) {
  const int half = a.d >> 1;
  const int G = a.Hq / a.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ float cs[kPackWarps][64], sn[kPackWarps][64];
  __shared__ int s_grp[256];
  // The previous kernels of the stream (which may write q, k or the prefix
  // cache, or read this workspace) must be done before anything is read or
  // written.  Only then may the attention kernel begin launching: it starts
  // its prefix K/V loads before its own wait, so everything before this
  // kernel has to be complete when it launches.
  pdl_wait();
  if (threadIdx.x == 0) pdl_trigger();
  const int lanes_per_head = half / 8;           // 8 (d = 128) or 4 (d = 64)
  const int heads_per_it = 32 / lanes_per_head;  // 4 or 8
  const int per_warp = kChunkIt * heads_per_it;
  const int H = a.Hq + a.Hkv;
  const int n_chunks = (H + per_warp - 1) / per_warp;
  const long long wid = (long long)blockIdx.x * kPackWarps + warp;
  const int t = (int)min(wid / n_chunks, (long long)a.T);
  const int chunk = (int)(wid - (long long)t * n_chunks);
  const int h_base = chunk * per_warp;
  const int i0 = (lane % lanes_per_head) * 8, hsub = lane / lanes_per_head;
  using Raw = typename RawVec<T>::type;
  Raw r0[kChunkIt], r1[kChunkIt];
  if (t < a.T) {
#pragma unroll
    for (int it = 0; it < kChunkIt; ++it) {
      const int hh = h_base + it * heads_per_it + hsub;
      if (hh < H) {
        const T* src = hh < a.Hq ? reinterpret_cast<const T*>(a.q) + ((size_t)t * a.Hq + hh) * a.d
                                 : reinterpret_cast<const T*>(a.k) + ((size_t)t * a.Hkv + (hh - a.Hq)) * a.d;
        r0[it] = *reinterpret_cast<const Raw*>(src + i0);
        r1[it] = *reinterpret_cast<const Raw*>(src + i0 + half);
      }
    }
  }
  if (blockIdx.x == 0) {
    // input checks and the inverse head table: identity first, so that every
    // entry stays a valid head index even when a malformed map leaves a slot
    // unclaimed
    for (int h = threadIdx.x; h < a.Hq; h += blockDim.x) {
      int g = a.head_map ? a.head_map[h] : h / G;
      if (g < 0 || g >= a.Hkv) {
        raise_flag(a.status, JEV_DEV_BAD_HEAD_MAP);
        g = 0;
      }
      s_grp[h] = g;
      a.hinv[h] = h;
    }
    __syncthreads();
    for (int h = threadIdx.x; h < a.Hq; h += blockDim.x) {
      const int g = s_grp[h];
      int slot = 0;
      for (int h2 = 0; h2 < h; ++h2) slot += (s_grp[h2] == g);
      if (slot >= G) {
        raise_flag(a.status, JEV_DEV_BAD_HEAD_MAP);
        slot = G - 1;
      }
      a.hinv[g * G + slot] = h;
    }
    if (a.parent && threadIdx.x == 0 && (a.parent[0] != -1 || a.offs[0] != 0 || (a.n_segs > 0 && a.offs[1] != 0)))
      raise_flag(a.status, JEV_DEV_BAD_TREE);  // node 0 is the root: no parent, no packed tokens
    // offsets must start at 0, never decrease and end at T
    for (int i = threadIdx.x; i < a.n_segs; i += blockDim.x)
      if (a.offs[i + 1] < a.offs[i]) raise_flag(a.status, JEV_DEV_BAD_SEQLENS);
    if (threadIdx.x == 0 && (a.offs[0] != 0 || a.offs[a.n_segs] != a.T)) raise_flag(a.status, JEV_DEV_BAD_SEQLENS);
  }
  if (t >= a.T) return;
  const int seg = warp_upper_segment(a.offs, a.n_segs, t, lane);
  int start = a.offs[seg];
  if (start > t) start = t;
  if (start < 0) start = 0;
  int pos = 0, krow = t, kvalid = 1;
  if (a.parent) {
    // tree token: window from its top-level ancestor; as a key, its node's subtree end
    pos = a.pos0[seg] + (t - start);
    if (chunk == 0) {
      const NodePlan np = plan_node(a, seg, lane);
      if (lane == 0) {
        if (np.start < 0) raise_flag(a.status, JEV_DEV_BAD_TREE);
        a.info[t] = TokInfo{max(np.start, 0), pos, np.start < 0 ? -1 : seg, np.end};
        a.key_end[t] = np.start < 0 ? -1 : np.end;
      }
    }
  } else if (a.cache_off) {
    // new token j of branch seg: after the branch's cached tokens, in its cache rows
    const int j = t - start, n_new = a.offs[seg + 1] - start;
    const int len = a.cache_len[seg], c0 = a.cache_off[seg], c1 = a.cache_off[seg + 1];
    kvalid = len >= 0 && c0 >= 0 && c1 <= a.key_rows && (long long)c0 + len + n_new <= (long long)c1;
    krow = kvalid ? c0 + len + j : 0;
    pos = a.pos_offset + (kvalid ? len : 0) + j;
    if (chunk == 0 && lane == 0) {
      if (!kvalid) raise_flag(a.status, JEV_DEV_BAD_CACHE);
      a.info[t] = TokInfo{max(c0, 0), pos, kvalid ? seg : -1, krow};
    }
  } else {
    pos = a.pos_seq ? a.pos_offset + t : (a.pos0 ? a.pos0[seg] : a.pos_offset) + (t - start);
    if (chunk == 0 && lane == 0) a.info[t] = TokInfo{start, pos, seg, t};
  }
  for (int i = lane; i < half; i += 32) {
    // angle formed in double and reduced to [-pi, pi] in double (the error of
    // the reduction is ~1e-12 rad for positions up to 1e6), then one float sincos
    const double ang = (double)pos * a.inv_freq[i];
    const double r = ang - rint(ang * 0.15915494309189535) * 6.283185307179586;
    float sf, cf;
    sincosf((float)r, &sf, &cf);
    cs[warp][i] = cf;
    sn[warp][i] = sf;
  }
  __syncwarp();
  float c8[8], s8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    c8[k] = cs[warp][i0 + k];
    s8[k] = sn[warp][i0 + k];
  }
  const size_t M = (size_t)a.T * G;
#pragma unroll
  for (int it = 0; it < kChunkIt; ++it) {
    const int hh = h_base + it * heads_per_it + hsub;
    if (hh < H) {
      if (hh >= a.Hq && !kvalid) continue;  // a cache row outside the branch's rows is not written
      T* dst;
      if (hh < a.Hq) {
        int g, slot;
        head_slot(a, G, hh, g, slot);
        dst = reinterpret_cast<T*>(a.q_rot) + ((size_t)g * M + (size_t)t * G + slot) * a.d;
      } else {
        dst = reinterpret_cast<T*>(a.k_rot) + ((size_t)krow * a.Hkv + (hh - a.Hq)) * a.d;
      }
      float x0[8], x1[8], y0[8], y1[8];
      unpack8(r0[it], x0);
      unpack8(r1[it], x1);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        y0[k] = x0[k] * c8[k] - x1[k] * s8[k];
        y1[k] = x1[k] * c8[k] + x0[k] * s8[k];
      }
      store8(dst + i0, y0);
      store8(dst + i0 + half, y1);
    }
  }
  // cache mode: the new token's values go to the same cache row as its key
  if (a.v_cache && kvalid && chunk == 0) {
    constexpr int kVec = 16 / sizeof(T);
    const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(a.v) + (size_t)t * a.Hkv * a.d);
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<T*>(a.v_cache) + (size_t)krow * a.Hkv * a.d);
    for (int e = lane; e < a.Hkv * a.d / kVec; e += 32) dst[e] = src[e];
  }
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
  // warps: the token's heads in chunks of `it` iterations of 32 / (d / 16)
  // heads each; four iterations once two would need more than 8192 warps
  // (about two waves of resident warps on 148 SMs)
  auto n_warps = [&](int it) {
    const int per_warp = it * (32 / (a.d / 16));
    return (long long)a.T * ((a.Hq + a.Hkv + per_warp - 1) / per_warp);
  };
  const int it = n_warps(2) > 8192 ? 4 : 2;
  const int blocks = (int)((n_warps(it) + kPackWarps - 1) / kPackWarps);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(kPackWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (dt == JEV_BF16)
    return it == 4 ? cudaLaunchKernelEx(&cfg, rope_pack_kernel<__nv_bfloat16, 4>, a)
                   : cudaLaunchKernelEx(&cfg, rope_pack_kernel<__nv_bfloat16, 2>, a);
  return it == 4 ? cudaLaunchKernelEx(&cfg, rope_pack_kernel<float, 4>, a) : cudaLaunchKernelEx(&cfg, rope_pack_kernel<float, 2>, a);
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
