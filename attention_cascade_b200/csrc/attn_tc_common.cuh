// attn_tc_common.cuh — pieces shared by the two tensor-core attention kernels
// (attn_tc.cu: two 128-row Q tiles a CTA, 256-row work tiles; attn_tc1.cu:
// one Q tile, 128-row work tiles): bounded mbarrier waits, named barriers,
// the walk over a CTA's segments, and the host's TMA descriptors.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace jev {
namespace tca {

using namespace tc;

constexpr int kKeyTile = 128;  // keys per K/V tile (one unit)

__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// named barrier that also ANDs a flag over its threads, so that they all
// leave with the same answer
__device__ __forceinline__ bool named_sync_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// Bounded wait (limit: AttnArgs::wait_cycles); once any wait of the CTA has
// run out, the others give up at their first unsatisfied check.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort, int32_t* status,
                                         long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      *abort = 1;
      raise_flag(status, JEV_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait taken by a whole warp: every lane polls, and all take lane 0's
// answer, so that the warp stays converged for the elected issue that follows.
__device__ __forceinline__ bool wait_bar_w(uint32_t bar, uint32_t parity, volatile int* abort, int32_t* status,
                                           long long limit) {
  return __shfl_sync(0xffffffffu, wait_bar(bar, parity, abort, status, limit), 0);
}

// The failure-detection probe: a bounded wait on a barrier that nothing
// completes.  It runs out after the wait bound (checking the clock at least
// every microsecond) and winds the CTA down like any other timeout.
__device__ __forceinline__ bool probe_wait(uint32_t bar, volatile int* abort, int32_t* status, long long limit) {
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait_hint(bar, 0, 1000)) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      *abort = 1;
      raise_flag(status, JEV_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
}

// Wait on the exit path: bounded, but blind to the abort flag, so that a CTA
// that is winding down still sees every load it armed land and every MMA it
// issued complete before it frees TMEM and exits.  Such work completes within
// microseconds; running out of the bound only raises the flag.
constexpr long long kDrainCycles = 1LL << 28;
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity, int32_t* status) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kDrainCycles) {
      raise_flag(status, JEV_DEV_WAIT_TIMEOUT);
      return;
    }
  }
}

__device__ __forceinline__ int warp_min_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int warp_max_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// The suffix keys any row of a work tile of kRows rows from m0 may see: from
// the lowest window start to the highest last key (a tree row's last key is
// its own token).
template <int kRows>
__device__ __forceinline__ void tile_window(const AttnArgs& a, int m0, int lane, int& lo, int& hi) {
  const int m_end = min(m0 + kRows, a.M);
  const int t0 = m0 / a.G, t1 = (m_end - 1) / a.G;
  const bool tree = a.key_end != nullptr;
  int mn = INT_MAX, mx = -1;
  for (int t = t0 + lane; t <= t1; t += 32) {
    const TokInfo inf = a.info[t];
    if (inf.node < 0) continue;
    mn = min(mn, inf.seg_start);
    mx = max(mx, tree ? t : inf.last);
  }
  lo = warp_min_i(mn);
  hi = warp_max_i(mx);
}

// One segment of a CTA's unit range: units [ua, ub) of work tile w.
struct Segment {
  int w, ua, ub;
  int g, m0;
  int n_pre, n;   // prefix key tiles of the segment, key tiles in total
  int lo;         // first suffix key of the window (when the segment holds the suffix unit)
  bool complete;  // the segment is the whole tile: write the final output
  int slot;       // partial slot when not complete
};
static_assert(2 * sizeof(Segment) <= 128, "segment ring");

// A CTA's segments: first its whole tiles (k < full_waves: tile c + k*n_ctas),
// then its tail units.  Every role visits them in the same order and derives
// the same description (the window takes one warp-wide reduction).
struct SegIter {
  int k;                 // segment index
  long long u, u_end;    // tail units still to visit
};

__device__ __forceinline__ bool seg_next(const AttnArgs& a, int c, SegIter& it, int& w, int& ua, int& ub, bool& tail) {
  if (it.k < a.full_waves) {
    w = c + it.k * a.n_ctas;
    ua = 0;
    ub = a.P;
    tail = false;
    return true;
  }
  if (it.u >= it.u_end) return false;
  const int wt = (int)(it.u / a.P);
  const long long t0 = (long long)wt * a.P;
  w = a.tail0 + wt;
  ua = (int)(it.u - t0);
  ub = (int)(min(it.u_end, t0 + a.P) - t0);
  tail = true;
  it.u = t0 + ub;
  return true;
}

template <int kRows>
__device__ __forceinline__ Segment make_segment(const AttnArgs& a, int c, int w, int ua, int ub, bool tail, int lane) {
  Segment sg;
  sg.w = w;
  sg.ua = ua;
  sg.ub = ub;
  const long long t0 = (long long)(w - a.tail0) * a.P;  // tail unit of the tile's first unit
  sg.g = sg.w / a.n_mt;
  sg.m0 = (sg.w - sg.g * a.n_mt) * kRows;
  sg.n_pre = max(0, min(sg.ub, a.n_pre) - sg.ua);
  int n_suf = 0;
  sg.lo = 0;
  if (sg.ub == a.P) {
    int lo, hi;
    tile_window<kRows>(a, sg.m0, lane, lo, hi);
    sg.lo = lo;
    n_suf = lo <= hi ? (hi - lo + kKeyTile) / kKeyTile : 0;
  }
  sg.n = sg.n_pre + n_suf;
  // A segment always has a key tile: the q_empty / p_full handshake that
  // keeps the roles within one q_full phase of each other runs per key tile.
  // n would be 0 only for a suffix-only unit whose rows are all skipped
  // (malformed input); its one tile is then fully masked and nothing is written.
  if (sg.n == 0) {
    sg.lo = 0;
    sg.n = 1;
  }
  sg.complete = sg.ua == 0 && sg.ub == a.P;
  sg.slot = (tail && tc_unit_begin(a, c) >= t0) ? 2 * c : 2 * c + 1;
  return sg;
}

// ---------------------------------------------------------------- host: TMA descriptors
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// bf16 rows of `inner` elements, `rows` rows `stride` bytes apart; 64 x 128 boxes, 128-byte swizzle
inline bool map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the stacked rotated queries [Hkv][M][D]; 64 x 128-row boxes, 128-byte swizzle
inline bool map_q(CUtensorMap* m, const void* base, int D, int M, int Hkv) {
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)M, (cuuint64_t)Hkv};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)M * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The four TMA descriptors of one call: stacked queries, prefix K and V
// (absent when Lp = 0), suffix (rotated) K and V.
inline bool attn_maps(const AttnArgs& a, int D, CUtensorMap* mq, CUtensorMap* mkp, CUtensorMap* mvp, CUtensorMap* mks,
                      CUtensorMap* mvs) {
  memset(mkp, 0, sizeof *mkp);
  memset(mvp, 0, sizeof *mvp);
  const uint64_t row = (uint64_t)a.Hkv * D * 2;
  if (!map_q(mq, a.q_rot, D, a.M, a.Hkv)) return false;
  if (a.Lp > 0 && (!map_2d(mkp, a.k_pre, (uint64_t)a.Hkv * D, a.Lp, row) ||
                   !map_2d(mvp, a.v_pre, (uint64_t)a.Hkv * D, a.Lp, row)))
    return false;
  return map_2d(mks, a.k_rot, (uint64_t)a.Hkv * D, a.key_rows, row) &&
         map_2d(mvs, a.v_suf, (uint64_t)a.Hkv * D, a.key_rows, row);
}

}  // namespace tca
}  // namespace jev
