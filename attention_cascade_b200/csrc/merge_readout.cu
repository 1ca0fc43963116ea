// merge_readout.cu — log-sum-exp merge of split partials, and candidate readout.
#include <math_constants.h>

#include <algorithm>

#include "kernels.h"

namespace jev {
namespace {

// Merge of S partial softmaxes over disjoint key sets: with per-split
// normalised outputs O_s and log2 normalisers L_s,
//   L = log2 sum_s 2^L_s,   O = sum_s 2^(L_s - L) O_s.
// This is exact (no approximation): attention over a union of key sets is the
// normaliser-weighted average of the attentions over the parts.  One warp per
// stacked row.
template <typename T, int D>
__global__ void __launch_bounds__(256) merge_kernel(MergeArgs a) {
  constexpr int C = D / 32;
  constexpr int kMaxS = 16;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int rows = a.Hkv * a.M;
  if (warp >= rows) return;
  const int g = warp / a.M, m = warp - g * a.M;
  const size_t split_stride = (size_t)a.Hkv * a.M;
  const size_t r0 = (size_t)g * a.M + m;
  // pass 1: every split's normaliser (independent loads, all in flight)
  float lp[kMaxS];
  float mx = -CUDART_INF_F;
#pragma unroll
  for (int s = 0; s < kMaxS; ++s) {
    lp[s] = s < a.S ? a.l_part[s * split_stride + r0] : -CUDART_INF_F;
    mx = fmaxf(mx, lp[s]);
  }
  float acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) acc[c] = 0.f;
  float wsum = 0.f;
  if (mx != -CUDART_INF_F) {
    // pass 2: weighted sum of the partial outputs
#pragma unroll
    for (int s = 0; s < kMaxS; ++s) {
      if (s < a.S) {
        const float w = exp2f(lp[s] - mx);
        wsum += w;
        const float* o = a.o_part + (s * split_stride + r0) * D;
#pragma unroll
        for (int c = 0; c < C; ++c) acc[c] += w * o[lane + 32 * c];
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  const int t = m / a.G;
  if (a.info[t].node < 0) return;  // a skipped row is left as it was
  const int h = min(max(a.hinv[g * a.G + (m - t * a.G)], 0), a.Hq - 1);
  T* out = reinterpret_cast<T*>(a.out) + ((size_t)t * a.Hq + h) * D;
#pragma unroll
  for (int c = 0; c < C; ++c) out[lane + 32 * c] = from_f32<T>(acc[c] * inv);
  if (a.lse && lane == 0)
    a.lse[(size_t)t * a.Hq + h] = wsum > 0.f ? (mx + log2f(wsum)) * 0.69314718055994531f : -CUDART_INF_F;
}

// Dot of two length-H rows with 16-byte loads and fp32 accumulation, warp
// wide.  Each lane issues up to kU independent loads of both rows before
// using any of them, so a row costs ceil(H / (kU*32*per16B)) memory latencies.
constexpr int kU = 16;
__device__ __forceinline__ float dot8(uint4 a, uint4 b) {
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 fa = __bfloat1622float2(a2[k]), fb = __bfloat1622float2(b2[k]);
    acc = fmaf(fa.x, fb.x, acc);
    acc = fmaf(fa.y, fb.y, acc);
  }
  return acc;
}
__device__ __forceinline__ float row_dot(const __nv_bfloat16* x, const __nv_bfloat16* w, int H, int lane) {
  const uint4* x4 = reinterpret_cast<const uint4*>(x);
  const uint4* w4 = reinterpret_cast<const uint4*>(w);
  const int n = H >> 3;
  float acc = 0.f;
  for (int base = 0; base < n; base += 32 * kU) {
    uint4 xa[kU], wa[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = base + u * 32 + lane;
      xa[u] = i < n ? __ldg(x4 + i) : make_uint4(0, 0, 0, 0);
      wa[u] = i < n ? __ldg(w4 + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) acc += dot8(xa[u], wa[u]);
  }
  return acc;
}
__device__ __forceinline__ float row_dot(const float* x, const float* w, int H, int lane) {
  const float4* x4 = reinterpret_cast<const float4*>(x);
  const float4* w4 = reinterpret_cast<const float4*>(w);
  const int n = H >> 2;
  float acc = 0.f;
  for (int base = 0; base < n; base += 32 * kU) {
    float4 xa[kU], wa[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = base + u * 32 + lane;
      xa[u] = i < n ? __ldg(x4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      wa[u] = i < n ? __ldg(w4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      acc += xa[u].x * wa[u].x + xa[u].y * wa[u].y + xa[u].z * wa[u].z + xa[u].w * wa[u].w;
  }
  return acc;
}

// Candidate scores: the sum over the candidate's (row, token) pairs of
// hidden[row] . lm_head[token], gathered with 16-byte loads (only option rows
// of the LM head are ever read).  The score is parked in logprob[c] (NaN for
// an invalid pair) for the set kernel below.
//   one pair per candidate (no candidate offsets): a warp per candidate;
//   several pairs: a block per candidate, warp w taking pairs w, w + 4, ...,
//   so the candidate's rows are in flight together; the warps' partial sums
//   are added in warp order.
// One-pair bf16 candidates with H <= 4096 take the fused kernel further down
// instead.
constexpr int kCandWarps = 4;

template <typename T>
__global__ void __launch_bounds__(kCandWarps * 32) readout_cand_kernel(ReadoutArgs a) {
  const int c = blockIdx.x * kCandWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (c >= a.n_cands) return;
  const T* hid = reinterpret_cast<const T*>(a.hidden);
  const T* W = reinterpret_cast<const T*>(a.lm_head);
  int pa = c, pe = c + 1;
  if (a.cand_offsets) {
    pa = a.cand_offsets[c];
    pe = a.cand_offsets[c + 1];
  }
  int set_of_c = 0;
  if (!a.pair_row) set_of_c = upper_segment(a.set_offsets, a.n_sets, c);  // row = set index
  float z = 0.f;
  bool bad = pa < 0 || pe < pa || pe > a.n_pairs;
  if (!bad) {
    for (int k = pa; k < pe; ++k) {
      const int row = a.pair_row ? a.pair_row[k] : set_of_c;
      const int tok = a.pair_tok[k];
      if (row < 0 || row >= a.R || tok < 0 || tok >= a.V) {
        bad = true;
        continue;
      }
      z += row_dot(hid + (size_t)row * a.H, W + (size_t)tok * a.H, a.H, lane);
      if (a.row_lse && lane == 0) z -= a.row_lse[row];
    }
  }
  z = warp_sum(z);
  if (lane == 0) {
    const float zz = bad ? CUDART_NAN_F : z;
    a.logprob[c] = zz;
    if (a.score) a.score[c] = zz;
  }
}

// One 16-byte load of an LM-head or hidden row, through the read-only path.
__device__ __forceinline__ uint4 ld_row16(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// One-pair candidates of bf16 rows with H <= 32 * 8 * NU: a warp per option
// set.  The set's hidden row is loaded once into registers; the candidates'
// LM-head rows stream through two register buffers, the next row's 16-byte
// loads all issued before the current row's dot product, so two rows per warp
// are always in flight.  The scores go to logprob and the same warp then takes
// the set's log-softmax and argmax: no second kernel.  NU (16-byte vectors
// per lane and row) is the smallest of a few sizes that covers H.
template <int NU>
__device__ __forceinline__ void ld_row_chunk(const uint4* p, int n, int lane, uint4 (&v)[NU]) {
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    const int i = u * 32 + lane;
    v[u] = i < n ? ld_row16(p + i) : make_uint4(0, 0, 0, 0);
  }
}
template <int NU>
__device__ __forceinline__ float dot_chunk(const uint4 (&x)[NU], const uint4 (&w)[NU]) {
  float z = 0.f;
#pragma unroll
  for (int u = 0; u < NU; ++u) z += dot8(x[u], w[u]);
  return z;
}
// log-softmax over a set's scores (in logprob[ca .. ce)) and the argmax, lowest
// index on ties; a NaN score (an invalid pair) makes the set's log-probs NaN
// and its choice -1
__device__ __forceinline__ void set_softmax(const ReadoutArgs& a, int s, int ca, int ce, int lane) {
  float mx = -CUDART_INF_F;
  int best = -1;
  bool any_nan = false;
  for (int c = ca + lane; c < ce; c += 32) {
    const float z = a.logprob[c];
    if (isnan(z)) any_nan = true;
    else if (best < 0 || z > mx) { mx = z; best = c; }
  }
  any_nan = __any_sync(0xffffffffu, any_nan);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, mx, o);
    const int ob = __shfl_xor_sync(0xffffffffu, best, o);
    if (ob >= 0 && (best < 0 || om > mx || (om == mx && ob < best))) { mx = om; best = ob; }
  }
  float sum = 0.f;
  for (int c = ca + lane; c < ce; c += 32) sum += exp2f((a.logprob[c] - mx) * 1.4426950408889634f);
  sum = warp_sum(sum);
  const float lse = mx + log2f(sum) * 0.69314718055994531f;
  __syncwarp();
  for (int c = ca + lane; c < ce; c += 32) a.logprob[c] = any_nan ? CUDART_NAN_F : a.logprob[c] - lse;
  if (lane == 0) a.choice[s] = any_nan ? -1 : best - ca;
}

template <int NU>
__global__ void __launch_bounds__(kCandWarps * 32) readout_set_fused_kernel(ReadoutArgs a) {
  const int s = blockIdx.x * kCandWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (s >= a.n_sets) return;
  const int ca = a.set_offsets[s], ce = a.set_offsets[s + 1];
  if (!(ca >= 0 && ce >= ca && ce <= a.n_cands) || ce == ca) {
    if (lane == 0) a.choice[s] = -1;
    return;
  }
  const int n = a.H >> 3;  // 16-byte vectors per row
  const bool row_ok = s < a.R;
  const __nv_bfloat16* W = reinterpret_cast<const __nv_bfloat16*>(a.lm_head);
  uint4 x[NU], w0[NU], w1[NU];
  ld_row_chunk(reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(a.hidden) + (size_t)(row_ok ? s : 0) * a.H),
               n, lane, x);
  auto tok_of = [&](int c) { const int tk = a.pair_tok[c]; return (tk >= 0 && tk < a.V) ? tk : -1; };
  int tk = tok_of(ca);
  if (tk >= 0) ld_row_chunk(reinterpret_cast<const uint4*>(W + (size_t)tk * a.H), n, lane, w0);
  for (int c = ca; c < ce; c += 2) {
    // candidate c is in w0; load c + 1 into w1 before using w0, then c + 2 into w0
    const int tk1 = c + 1 < ce ? tok_of(c + 1) : -1;
    if (tk1 >= 0) ld_row_chunk(reinterpret_cast<const uint4*>(W + (size_t)tk1 * a.H), n, lane, w1);
    float z = warp_sum(dot_chunk(x, w0));
    if (lane == 0) {
      const float zz = (tk < 0 || !row_ok) ? CUDART_NAN_F : (a.row_lse ? z - a.row_lse[s] : z);
      a.logprob[c] = zz;
      if (a.score) a.score[c] = zz;
    }
    if (c + 1 >= ce) break;
    const int tk2 = c + 2 < ce ? tok_of(c + 2) : -1;
    if (tk2 >= 0) ld_row_chunk(reinterpret_cast<const uint4*>(W + (size_t)tk2 * a.H), n, lane, w0);
    z = warp_sum(dot_chunk(x, w1));
    if (lane == 0) {
      const float zz = (tk1 < 0 || !row_ok) ? CUDART_NAN_F : (a.row_lse ? z - a.row_lse[s] : z);
      a.logprob[c + 1] = zz;
      if (a.score) a.score[c + 1] = zz;
    }
    tk = tk2;
  }
  __syncwarp();
  set_softmax(a, s, ca, ce, lane);
}

template <typename T>
__global__ void __launch_bounds__(kCandWarps * 32) readout_cand_block_kernel(ReadoutArgs a) {
  __shared__ float part[kCandWarps];
  __shared__ int part_bad[kCandWarps];
  const int c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* hid = reinterpret_cast<const T*>(a.hidden);
  const T* W = reinterpret_cast<const T*>(a.lm_head);
  const int pa = a.cand_offsets[c], pe = a.cand_offsets[c + 1];
  int set_of_c = 0;
  if (!a.pair_row) set_of_c = upper_segment(a.set_offsets, a.n_sets, c);  // row = set index
  float z = 0.f;
  bool bad = pa < 0 || pe < pa || pe > a.n_pairs;
  if (!bad) {
    for (int k = pa + warp; k < pe; k += kCandWarps) {
      const int row = a.pair_row ? a.pair_row[k] : set_of_c;
      const int tok = a.pair_tok[k];
      if (row < 0 || row >= a.R || tok < 0 || tok >= a.V) {
        bad = true;
        continue;
      }
      z += row_dot(hid + (size_t)row * a.H, W + (size_t)tok * a.H, a.H, lane);
      if (a.row_lse && lane == 0) z -= a.row_lse[row];
    }
  }
  z = warp_sum(z);
  if (lane == 0) {
    part[warp] = z;
    part_bad[warp] = bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float zz = 0.f;
    bool b = false;
#pragma unroll
    for (int q = 0; q < kCandWarps; ++q) {
      zz += part[q];
      b |= part_bad[q] != 0;
    }
    zz = b ? CUDART_NAN_F : zz;
    a.logprob[c] = zz;
    if (a.score) a.score[c] = zz;
  }
}

// One warp per option set: log-sum-exp and argmax (lowest index on ties) of
// the set's scores, written back as log-probabilities.
constexpr int kSetWarps = 4;

__global__ void __launch_bounds__(kSetWarps * 32) readout_set_kernel(ReadoutArgs a) {
  pdl_wait();  // the candidate scores come from the previous kernel
  const int s = blockIdx.x * kSetWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (s >= a.n_sets) return;
  const int ca = a.set_offsets[s], ce = a.set_offsets[s + 1];
  if (!(ca >= 0 && ce >= ca && ce <= a.n_cands) || ce == ca) {
    if (lane == 0) a.choice[s] = -1;
    return;
  }
  set_softmax(a, s, ca, ce, lane);
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, jev_dtype dt, cudaStream_t s) {
  const int rows = a.Hkv * a.M;
  if (rows == 0) return cudaSuccess;
  const int blocks = (rows * 32 + 255) / 256;
  if (dt == JEV_BF16) {
    if (a.d == 64) merge_kernel<__nv_bfloat16, 64><<<blocks, 256, 0, s>>>(a);
    else merge_kernel<__nv_bfloat16, 128><<<blocks, 256, 0, s>>>(a);
  } else {
    if (a.d == 64) merge_kernel<float, 64><<<blocks, 256, 0, s>>>(a);
    else merge_kernel<float, 128><<<blocks, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_readout(const ReadoutArgs& a, jev_dtype dt, cudaStream_t s, int* n_kernels) {
  *n_kernels = 0;
  if (a.n_sets == 0) return cudaSuccess;
  if (a.n_cands > 0) {
    if (a.cand_offsets) {
      if (dt == JEV_BF16) readout_cand_block_kernel<__nv_bfloat16><<<a.n_cands, kCandWarps * 32, 0, s>>>(a);
      else readout_cand_block_kernel<float><<<a.n_cands, kCandWarps * 32, 0, s>>>(a);
    } else {
      const int blocks = (a.n_cands + kCandWarps - 1) / kCandWarps;
      const int nu = (a.H / 8 + 31) / 32;  // 16-byte vectors per lane and row
      if (dt == JEV_BF16 && !a.pair_row && nu <= 16) {
        // a warp per set: scores and the set's softmax in one kernel
        const dim3 g((a.n_sets + kCandWarps - 1) / kCandWarps), b(kCandWarps * 32);
        if (nu <= 4) readout_set_fused_kernel<4><<<g, b, 0, s>>>(a);
        else if (nu <= 6) readout_set_fused_kernel<6><<<g, b, 0, s>>>(a);
        else if (nu <= 8) readout_set_fused_kernel<8><<<g, b, 0, s>>>(a);
        else if (nu <= 12) readout_set_fused_kernel<12><<<g, b, 0, s>>>(a);
        else if (nu <= 14) readout_set_fused_kernel<14><<<g, b, 0, s>>>(a);
        else readout_set_fused_kernel<16><<<g, b, 0, s>>>(a);
        *n_kernels = 1;
        return cudaGetLastError();
      }
      if (dt == JEV_BF16) readout_cand_kernel<__nv_bfloat16><<<blocks, kCandWarps * 32, 0, s>>>(a);
      else readout_cand_kernel<float><<<blocks, kCandWarps * 32, 0, s>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    *n_kernels = 1;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((a.n_sets + kSetWarps - 1) / kSetWarps);
  cfg.blockDim = dim3(kSetWarps * 32);
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  ++*n_kernels;
  return cudaLaunchKernelEx(&cfg, readout_set_kernel, a);
}

}  // namespace jev
