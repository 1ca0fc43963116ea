// common.cuh — small device helpers shared by the jev kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/jev.h"

namespace jev {

constexpr int kStatusBytes = 256;  // status word lives in the first 256 bytes of a workspace
constexpr int kMaxSplits = 16;    // prefix splits the merge kernel combines

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream finishes;
// pdl_wait() blocks until that kernel has completed and its writes are
// visible (a no-op for an ordinary launch), pdl_trigger() lets the next
// kernel start launching once every CTA of this grid has issued it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void raise_flag(int32_t* status, int32_t bit) {
  if (status) atomicOr(status, bit);
}

// Largest b in [0, n) with offs[b] <= t (offs non-decreasing); 0 if none.
__device__ __forceinline__ int upper_segment(const int32_t* offs, int n, int t) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (offs[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Per query token, written by the RoPE pack.  Suffix keys are rows of the
// suffix key tensor (the packed suffix, the tree tokens, or a per-branch
// cache); a row sees the keys [seg_start, last] that pass its mask.
//   flat row:  keys seg_start .. last of its own branch (its own token, or its
//              slot in the branch's cache), all visible;
//   tree token: as a row, the keys from seg_start (the first token of its
//              top-level ancestor) up to itself that lie on its root path;
//              as a key, `last` is the end of the packed-token range of its
//              node's subtree, so key k is visible to tree row t exactly when
//              k <= t < last(k) (nodes and tokens in depth-first preorder).
// node < 0 marks a row that is not computed (malformed input, already flagged).
struct TokInfo {
  int32_t seg_start;  // first suffix key of the row's window
  int32_t pos;        // RoPE position of the token
  int32_t node;       // tree node / branch index; -1: row skipped
  int32_t last;       // flat: last visible key; tree: subtree token end (key side)
};

}  // namespace jev
