// vocab_lse.cu — log-sum-exp of hidden rows over the whole vocabulary, with
// no logits written to HBM: the normaliser of multi-token candidate scoring
// (log p(tok | row) = hidden[row] . lm_head[tok] - LSE[row]).
//
// The work is a GEMM, hidden [R, H] x lm_head[V, H]^T, of which only each
// row's running maximum and exponential sum survive.  A CTA owns a range of
// 256-row vocabulary tiles; for each 256-row block of hidden rows and each of
// its vocabulary tiles it streams the H dimension in 64-column chunks through
// a TMA ring (both operands K-major with 128-byte swizzle) and accumulates
// S_i = X_i W^T for the two 128-row halves i into TMEM (M = 128, N = 256 per
// tcgen05.mma, 512 columns in all).  The 512 statistics threads (two per row,
// 128 columns each) then fold the tile into a running (max, sum) in the log2
// domain and release TMEM for the next tile.  Each CTA writes one partial
// (max, sum) per row and half; vocab_lse_merge_kernel combines them.
//
// CTA = 18 warps: 16 statistics warps, 1 TMA producer, 1 MMA issuer (which
// also owns TMEM).  Every mbarrier wait is bounded; a wait that runs out
// raises JEV_DEV_WAIT_TIMEOUT in the status word and the CTA winds down, the
// producer and the MMA warp first waiting for the loads and MMAs they issued.
#include <cuda.h>
#include <math_constants.h>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace jev {
namespace {

using namespace tc;

constexpr int kLM = 128;                 // hidden rows per half (TMEM lanes)
constexpr int kLN = 256;                 // vocabulary rows per tile
constexpr int kLK = 64;                  // hidden columns per chunk (one 128-byte swizzled block)
constexpr int kLStages = 3;
constexpr int kLStatWarps = 16;
constexpr int kLThreads = (kLStatWarps + 2) * 32;
constexpr int kLProducer = kLStatWarps, kLMma = kLStatWarps + 1;
constexpr int kXBytes = kLM * kLK * 2;               // 16 KB: one half's chunk
constexpr int kWBytes = kLN * kLK * 2;               // 32 KB: the tile's chunk
constexpr int kStageBytes = 2 * kXBytes + kWBytes;   // 64 KB
constexpr int kOffBar = kLStages * kStageBytes;      // 192 KB
constexpr int kLSmem = kOffBar + 256 + 1024;         // + 1024-byte alignment slack

struct LShared {
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool lwait(uint32_t bar, uint32_t parity, volatile int* abort, int32_t* status,
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

// The failure-detection probe: a bounded wait on a barrier that nothing
// completes; it runs out after the wait bound (checking the clock at least
// every microsecond) and winds the CTA down like any other timeout.
__device__ __forceinline__ bool lprobe(uint32_t bar, volatile int* abort, int32_t* status, long long limit) {
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

// Exit-path wait: bounded but blind to the abort flag (in-flight loads and
// MMAs complete within microseconds; running out of the bound only raises the flag).
constexpr long long kLDrainCycles = 1LL << 28;
__device__ __forceinline__ void ldrain(uint32_t bar, uint32_t parity, int32_t* status) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kLDrainCycles) {
      raise_flag(status, JEV_DEV_WAIT_TIMEOUT);
      return;
    }
  }
}

__global__ void __launch_bounds__(kLThreads, 1)
    vocab_lse_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_w16, const VocabLseArgs a) {
  extern __shared__ uint8_t lsm_raw[];
  uint8_t* smem = lsm_raw + ((1024 - (smem_u32(lsm_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  LShared* sh = reinterpret_cast<LShared*>(smem + kOffBar + 200);
  const uint32_t bar0 = sbase + kOffBar;
  const uint32_t b_full = bar0, b_empty = bar0 + 8 * kLStages, b_sfull = bar0 + 16 * kLStages,
                 b_sempty = b_sfull + 8, b_drain = b_sfull + 16, b_probe = b_sfull + 24;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  // this CTA's vocabulary rows [v_lo, v_hi): an even share of 16-row slabs, walked in 256-row tiles
  // whose last one may be narrower (an MMA of N = its rows rounded up to 16)
  const int n16 = (a.V + 15) / 16;
  const int v_lo = (int)((long long)cta * n16 / gridDim.x) * 16;
  const int v_hi = min(a.V, (int)((long long)(cta + 1) * n16 / gridDim.x) * 16);
  const int n_mb = (a.R + 2 * kLM - 1) / (2 * kLM);  // 256-row blocks of hidden rows
  const int nk = a.H / kLK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLStages; ++s) {
      mbar_init(b_full + 8 * s, 1);
      mbar_init(b_empty + 8 * s, 1);
    }
    mbar_init(b_sfull, 1);
    mbar_init(b_sempty, kLStatWarps * 32);
    mbar_init(b_drain, 1);
    mbar_init(b_probe, 1);  // nothing arrives on it
    sh->abort = 0;
    mbar_fence_init();
  }
  if (warp == kLMma) {
    tmem_alloc(smem_u32(&sh->tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == kLProducer && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_w16);
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;
  pdl_wait();  // hidden rows and the head may come from the previous kernel

  if (warp == kLProducer) {
    // ---------------------------------------------------------------- TMA producer
    // The whole warp runs the loop (its values stay warp-uniform, and lane
    // 0's view of each wait is taken by all); one elected lane issues each
    // load.
    auto wait_w = [&](uint32_t bar, uint32_t parity) {
      return __shfl_sync(0xffffffffu, lwait(bar, parity, abort, a.status, a.wait_cycles), 0);
    };
    long long it = 0;
    bool ok = true;
    for (int mb = 0; ok && mb < n_mb; ++mb)
      for (int v0 = v_lo; ok && v0 < v_hi; v0 += kLN) {
        const int n_t = (min(kLN, v_hi - v0) + 15) & ~15;  // rows of this tile's W chunk
        for (int kc = 0; ok && kc < nk; ++kc, ++it) {
          const int st = (int)(it % kLStages);
          const long long use = it / kLStages;
          if (it >= kLStages && !wait_w(b_empty + 8 * st, (uint32_t)((use - 1) & 1))) {
            ok = false;
            break;
          }
          const uint32_t base = sbase + st * kStageBytes;
          const bool two = mb * 2 * kLM + kLM < a.R;  // the block's second half holds rows
          mbar_expect_tx_w(b_full + 8 * st, (two ? 2 * kXBytes : kXBytes) + n_t * kLK * 2);
          tma_load_2d_w(base, &tm_x, kc * kLK, mb * 2 * kLM, b_full + 8 * st);
          if (two) tma_load_2d_w(base + kXBytes, &tm_x, kc * kLK, mb * 2 * kLM + kLM, b_full + 8 * st);
          // 128-row boxes, then 16-row boxes for a narrow tail (row `o` lands at o * 128 bytes)
          int o = 0;
          for (; o + kLM <= n_t; o += kLM)
            tma_load_2d_w(base + 2 * kXBytes + o * 128, &tm_w, kc * kLK, v0 + o, b_full + 8 * st);
          for (; o < n_t; o += 16)
            tma_load_2d_w(base + 2 * kXBytes + o * 128, &tm_w16, kc * kLK, v0 + o, b_full + 8 * st);
        }
      }
    // drain: the last phase of every stage armed (it loads so far) has
    // completed, so no load lands after the CTA exits
    if (lane == 0)
      for (int st = 0; st < kLStages; ++st) {
        const long long uses = it > st ? (it - st + kLStages - 1) / kLStages : 0;
        if (uses > 0) ldrain(b_full + 8 * st, (uint32_t)((uses - 1) & 1), a.status);
      }
  } else if (warp == kLMma) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop; one elected lane issues each MMA and
    // commit (the same lane every time, so the commits track its MMAs).
    auto wait_w = [&](uint32_t bar, uint32_t parity) {
      return __shfl_sync(0xffffffffu, lwait(bar, parity, abort, a.status, a.wait_cycles), 0);
    };
    long long it = 0, tile = 0;
    bool ok = true;
    for (int mb = 0; ok && mb < n_mb; ++mb) {
      const int halves = mb * 2 * kLM + kLM < a.R ? 2 : 1;
      for (int v0 = v_lo; ok && v0 < v_hi; v0 += kLN, ++tile) {
        const uint32_t idesc = idesc_bf16(kLM, (min(kLN, v_hi - v0) + 15) & ~15, false);
        // the statistics threads have read the previous tile out of TMEM
        if (tile > 0 && !wait_w(b_sempty, (uint32_t)((tile - 1) & 1))) {
          ok = false;
          break;
        }
        fence_after_sync();
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int st = (int)(it % kLStages);
          if (!wait_w(b_full + 8 * st, (uint32_t)((it / kLStages) & 1))) {
            ok = false;
            break;
          }
          fence_after_sync();
          const uint32_t base = sbase + st * kStageBytes;
          for (int i = 0; i < halves; ++i)
#pragma unroll
            for (int kk = 0; kk < kLK / 16; ++kk)
              mma_ss_w(tmem + i * kLN, smem_desc_sw128(base + i * kXBytes + kk * 32, 16, 1024),
                       smem_desc_sw128(base + 2 * kXBytes + kk * 32, 16, 1024), idesc, (kc > 0 || kk > 0) ? 1u : 0u);
          mma_commit_w(b_empty + 8 * st);
          // failure-detection probe (off unless a test sets it): a wait that
          // nothing completes, with this CTA's first MMAs in flight
          if (it == 0 && a.wait_probe &&
              !__shfl_sync(0xffffffffu, lprobe(b_probe, abort, a.status, a.wait_cycles), 0)) {
            ok = false;
            break;
          }
        }
        if (ok) mma_commit_w(b_sfull);
      }
    }
    // every MMA of this CTA has completed before TMEM is released, on the
    // timeout path too (the wait ignores the abort flag)
    mma_commit_w(b_drain);
    ldrain(b_drain, 0, a.status);
  } else {
    // ---------------------------------------------------------------- statistics
    const int i = warp >> 3, hf = (warp >> 2) & 1, q = warp & 3, r = q * 32 + lane;
    const uint32_t s_addr = tmem + i * kLN + hf * (kLN / 2) + ((uint32_t)(q * 32) << 16);
    constexpr float kLog2e = 1.4426950408889634f;
    long long tile = 0;
    bool ok = true;
    for (int mb = 0; mb < n_mb; ++mb) {
      const bool live = mb * 2 * kLM + i * kLM < a.R;  // warp-uniform: this half holds rows
      float m_run = -CUDART_INF_F, l_run = 0.f;  // log2 domain
      for (int t0 = v_lo; t0 < v_hi; t0 += kLN, ++tile) {
        // warp-uniform (the TMEM loads below are warp-wide instructions); a
        // failed wait runs the remaining tiles on stale TMEM so the loop shape stays uniform
        ok = __all_sync(0xffffffffu, ok && lwait(b_sfull, (uint32_t)(tile & 1), abort, a.status, a.wait_cycles));
        fence_after_sync();
        const int v0 = t0 + hf * (kLN / 2);  // vocabulary row of this thread's first column
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int lim = v_hi - (v0 + c * 64);  // columns past this CTA's rows are padding
          if (!live || lim <= 0) break;
          uint32_t xs[64];
          tmem_ld64(s_addr + c * 64, xs);
          // four independent max / sum chains
          float mx[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const float x = j < lim ? __uint_as_float(xs[j]) * kLog2e : -CUDART_INF_F;
            xs[j] = __float_as_uint(x);
            mx[j & 3] = fmaxf(mx[j & 3], x);
          }
          const float m_new = fmaxf(m_run, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])));
          if (m_new != -CUDART_INF_F) {
            float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 64; ++j) sum[j & 3] += ex2(__uint_as_float(xs[j]) - m_new);
            l_run = l_run * ex2(m_run - m_new) + ((sum[0] + sum[1]) + (sum[2] + sum[3]));
            m_run = m_new;
          }
        }
        fence_before_sync();
        mbar_arrive(b_sempty);
      }
      // this CTA's partial for the block's rows: (max, sum) per row and half
      const int row = mb * 2 * kLM + i * kLM + r;
      if (row < a.R) {
        const size_t pidx = (((size_t)mb * gridDim.x + cta) * 2 + hf) * (2 * kLM) + i * kLM + r;
        a.part[pidx] = make_float2(ok ? m_run : CUDART_NAN_F, l_run);
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kLMma) {
    fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// LSE of every row from the (max, sum) partials of all CTAs and both halves
// (the exact log-sum-exp merge), natural log.
__global__ void __launch_bounds__(256) vocab_lse_merge_kernel(const VocabLseArgs a, int n_ctas) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  pdl_wait();
  if (row >= a.R) return;
  const int mb = row / (2 * kLM), rr = row - mb * 2 * kLM;
  float m = -CUDART_INF_F;
  bool nan = false;
  for (int p = 0; p < 2 * n_ctas; ++p) {
    const float2 v = a.part[((size_t)mb * 2 * n_ctas + p) * (2 * kLM) + rr];
    if (isnan(v.x)) nan = true;
    m = fmaxf(m, v.x);
  }
  float l = 0.f;
  for (int p = 0; p < 2 * n_ctas; ++p) {
    const float2 v = a.part[((size_t)mb * 2 * n_ctas + p) * (2 * kLM) + rr];
    if (v.y > 0.f) l += v.y * exp2f(v.x - m);
  }
  a.lse[row] = nan ? CUDART_NAN_F : (m + log2f(l)) * 0.69314718055994531f;
}

// cuTensorMapEncodeTiled from the CUDA driver API, looked up once through the runtime (the
// attention kernels' translation unit keeps its own copy of this lookup).
typedef CUresult (*EncodeTiledFnL)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFnL encode_fn_l() {
  static EncodeTiledFnL fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFnL>(p);
    else
      cudaGetLastError();
  }
  return fn;
}

// bf16 rows of H elements (H*2 bytes apart), `rows` rows; 64 x 128 boxes, 128-byte swizzle
bool map_rows(CUtensorMap* m, const void* base, uint64_t H, uint64_t rows, uint32_t box_rows = 128) {
  if (!encode_fn_l()) return false;
  cuuint64_t dims[2] = {H, rows};
  cuuint64_t strides[1] = {H * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return encode_fn_l()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                       CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int vocab_lse_ctas(int V, int sms) {
  const int n16 = (V + 15) / 16;
  return std::max(1, std::min(n16, sms));
}

size_t vocab_lse_partial_bytes(int R, int n_ctas) {
  const size_t n_mb = (size_t)(R + 2 * kLM - 1) / (2 * kLM);
  return n_mb * n_ctas * 2 * (2 * kLM) * sizeof(float2);
}

cudaError_t launch_vocab_lse(const VocabLseArgs& a, int n_ctas, cudaStream_t s) {
  if (a.R == 0) return cudaSuccess;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(vocab_lse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap mx, mw, mw16;
  if (!map_rows(&mx, a.hidden, (uint64_t)a.H, (uint64_t)a.R) || !map_rows(&mw, a.lm_head, (uint64_t)a.H, (uint64_t)a.V) ||
      !map_rows(&mw16, a.lm_head, (uint64_t)a.H, (uint64_t)a.V, 16))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(n_ctas);
  cfg.blockDim = dim3(kLThreads);
  cfg.dynamicSmemBytes = kLSmem;
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, vocab_lse_kernel, mx, mw, mw16, a);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3((a.R + 255) / 256);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&cfg, vocab_lse_merge_kernel, a, n_ctas);
}

}  // namespace jev
