// attn_tc.cu — tensor-core shared-prefix attention for sm_100a (tcgen05 + TMEM + TMA).
//
// The prefix is shared by every branch ("How to Deploy Visual Jev ...", Step 3;
// "FastJEV ...", §3.2-§3.3), so all branches' queries of one kv group are
// stacked into one M dimension (row m = token m / G, query slot m % G) and the
// prefix K/V of that group streams through shared memory once per 256 stacked
// rows instead of once per branch.  After its prefix split, the CTA holding the
// last split also runs the suffix window: the packed suffix keys its rows may
// see (same branch up to the row's own token; for tree tokens every ancestor
// node's keys too), masked per row.  With one split the CTA normalises and
// writes the final output; with several it writes a normalised partial and
// its log2 normaliser for the merge kernel.
//
// CTA = 10 warps:
//   warps 0-3  softmax + epilogue of Q tile 0 (TMEM lanes 0-127)
//   warps 4-7  softmax + epilogue of Q tile 1
//   warp 8     TMA producer (Q once, then K/V tiles through a ring of stages)
//   warp 9     TMEM allocator and tcgen05.mma issuer (one thread)
// TMEM (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 at 256, O1 at 256+D.
// Per key tile j the MMA thread issues S_i = Q_i K_j^T (SS form), and after
// softmax i has written P_i (bf16, aliasing S_i) it issues O_i += P_i V_j with
// P_i read straight from TMEM (TS form); tile 0's softmax overlaps tile 1's
// MMAs and the other way round.  The online softmax runs in the log2 domain
// with a lazy running max: the max is only raised when a row's new maximum
// exceeds it by more than 8, so O is rescaled rarely and P stays <= 2^8.
// Every mbarrier wait is bounded; a wait that runs out raises
// JEV_DEV_WAIT_TIMEOUT in the status word and the CTA winds down.
#include <cuda.h>
#include <math_constants.h>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace jev {
namespace {

using namespace tc;

constexpr int kBM = 128;  // rows per Q tile (TMEM lanes)
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr long long kWaitCycles = 1LL << 31;
constexpr float kLazy = 8.0f;  // log2 headroom before the running max moves

template <int D>
struct Cfg {
  static constexpr int kNS = D == 128 ? 2 : 4;  // K/V stages
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kBlk = 128 * 128;  // one 64-column, 128-row swizzled block
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + kNS * kKVBytes;
  static constexpr int kOffBar = kOffV + kNS * kKVBytes;
  static constexpr int kSmem = kOffBar + 256 + 1024;  // barriers + 1024-byte alignment slack
  static constexpr int kOCol = 256;                   // first TMEM column of O0
};

struct Bars {
  uint32_t q_full, k_full, v_full, kv_empty, s_full, p_full, o_full, drain;  // smem addresses (arrays: +8*i)
};

struct Shared {
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort, int32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort = 1;
      raise_flag(status, JEV_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ int warp_min_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Lowest suffix key any row of the work tile may see, and the last token.
__device__ __forceinline__ void tile_window(const AttnArgs& a, int m0, int lane, int& lo, int& hi) {
  const int m_end = min(m0 + 2 * kBM, a.M);
  const int t0 = m0 / a.G, t1 = (m_end - 1) / a.G;
  int mn = INT_MAX;
  for (int t = t0 + lane; t <= t1; t += 32) {
    const TokInfo inf = a.info[t];
    int st = inf.seg_start;
    if (a.node_nanc) {
      const int na = a.node_nanc[inf.node];
      if (na < 0) continue;
      if (na > 0) st = min(st, a.node_anc[(size_t)inf.node * kMaxDepth].x);
    }
    mn = min(mn, st);
  }
  lo = warp_min_i(mn);
  hi = t1;
}

template <int D, bool TREE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp,
                   const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_ks,
                   const __grid_constant__ CUtensorMap tm_vs, const AttnArgs a) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  Shared* sh = reinterpret_cast<Shared*>(smem + C::kOffBar + 192);
  const uint32_t bar0 = sbase + C::kOffBar;
  Bars B;
  B.q_full = bar0;
  B.k_full = bar0 + 8;
  B.v_full = B.k_full + 8 * C::kNS;
  B.kv_empty = B.v_full + 8 * C::kNS;
  B.s_full = B.kv_empty + 8 * C::kNS;
  B.p_full = B.s_full + 16;
  B.o_full = B.p_full + 16;
  B.drain = B.o_full + 16;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 2 * kBM, g = blockIdx.y, split = blockIdx.z;
  const int p_lo = split * a.split_len;
  const int p_hi = min(a.Lp, p_lo + a.split_len);
  const int n_pre = p_hi > p_lo ? (p_hi - p_lo + kBN - 1) / kBN : 0;
  const bool last = split == a.S - 1;

  if (threadIdx.x == 0) {
    mbar_init(B.q_full, 1);
    for (int s = 0; s < C::kNS; ++s) {
      mbar_init(B.k_full + 8 * s, 1);
      mbar_init(B.v_full + 8 * s, 1);
      mbar_init(B.kv_empty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B.s_full + 8 * i, 1);
      mbar_init(B.p_full + 8 * i, 128);
      mbar_init(B.o_full + 8 * i, 1);
    }
    mbar_init(B.drain, 1);
    sh->abort = 0;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&sh->tmem_base), 512);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;

  int lo, hi;
  tile_window(a, m0, lane, lo, hi);
  const int n_suf = (last && lo <= hi) ? (hi - lo + kBN) / kBN : 0;
  const int n = n_pre + n_suf;
  auto key_base = [&](int j) { return j < n_pre ? p_lo + j * kBN : lo + (j - n_pre) * kBN; };

  if (warp == kProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      mbar_expect_tx(B.q_full, 2 * C::kQBytes);
      for (int i = 0; i < 2; ++i)
        for (int b = 0; b < D / 64; ++b)
          tma_load_3d(sbase + i * C::kQBytes + b * C::kBlk, &tm_q, b * 64, m0 + i * kBM, g, B.q_full);
      for (int j = 0; j < n; ++j) {
        const int st = j % C::kNS, use = j / C::kNS;
        if (j >= C::kNS && !wait_bar(B.kv_empty + 8 * st, (use - 1) & 1, abort, a.status)) break;
        const int kb = key_base(j);
        const CUtensorMap* mk = j < n_pre ? &tm_kp : &tm_ks;
        const CUtensorMap* mv = j < n_pre ? &tm_vp : &tm_vs;
        const uint32_t ks = sbase + C::kOffK + st * C::kKVBytes, vs = sbase + C::kOffV + st * C::kKVBytes;
        mbar_expect_tx(B.k_full + 8 * st, C::kKVBytes);
        for (int b = 0; b < D / 64; ++b) tma_load_2d(ks + b * C::kBlk, mk, g * D + b * 64, kb, B.k_full + 8 * st);
        mbar_expect_tx(B.v_full + 8 * st, C::kKVBytes);
        for (int b = 0; b < D / 64; ++b) tma_load_2d(vs + b * C::kBlk, mv, g * D + b * 64, kb, B.v_full + 8 * st);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(kBM, kBN, false);
      constexpr uint32_t id_pv = idesc_bf16(kBM, D, true);
      auto issue_s = [&](int i, int st) {
        const uint32_t qa = sbase + i * C::kQBytes, ka = sbase + C::kOffK + st * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlk + (kk & 3) * 32;
          mma_ss(tmem + i * kBN, smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), id_qk,
                 kk > 0);
        }
        mma_commit(B.s_full + 8 * i);
      };
      auto issue_pv = [&](int i, int st, bool acc) {
        const uint32_t va = sbase + C::kOffV + st * C::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          mma_ts(tmem + C::kOCol + i * D, tmem + i * kBN + kk * 8, smem_desc_sw128(va + kk * 16 * 128, C::kBlk, 1024),
                 id_pv, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait_bar(B.q_full, 0, abort, a.status);
      if (ok && n > 0) {
        ok = wait_bar(B.k_full, 0, abort, a.status);
        fence_after_sync();
        if (ok) {
          issue_s(0, 0);
          issue_s(1, 0);
        }
      }
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % C::kNS, ph = (j / C::kNS) & 1;
        const int st1 = (j + 1) % C::kNS, ph1 = ((j + 1) / C::kNS) & 1;
        if (!wait_bar(B.v_full + 8 * st, ph, abort, a.status)) break;
        if (!wait_bar(B.p_full, j & 1, abort, a.status)) break;
        fence_after_sync();
        issue_pv(0, st, j > 0);
        if (j == n - 1) mma_commit(B.o_full);
        if (j + 1 < n) {
          if (!wait_bar(B.k_full + 8 * st1, ph1, abort, a.status)) break;
          fence_after_sync();
          issue_s(0, st1);
        }
        if (!wait_bar(B.p_full + 8, j & 1, abort, a.status)) break;
        fence_after_sync();
        issue_pv(1, st, j > 0);
        mma_commit(B.kv_empty + 8 * st);
        if (j == n - 1) mma_commit(B.o_full + 8);
        if (j + 1 < n) issue_s(1, st1);
      }
      if (n == 0) {
        mma_commit(B.o_full);
        mma_commit(B.o_full + 8);
      }
      // every MMA of this CTA has completed before TMEM is released
      mma_commit(B.drain);
      wait_bar(B.drain, 0, abort, a.status);
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int i = warp >> 2, q = warp & 3, r = q * 32 + lane;
    const int m = m0 + i * kBM + r;
    const bool valid = m < a.M;
    int t = -1, start = 0, nanc = 0;
    int2 anc[TREE ? kMaxDepth : 1];
    if (valid) {
      t = m / a.G;
      const TokInfo inf = a.info[t];
      start = inf.seg_start;
      if (TREE) {
        nanc = a.node_nanc[inf.node];
        if (nanc < 0) t = -1;
#pragma unroll
        for (int k = 0; k < (TREE ? kMaxDepth : 1); ++k)
          anc[k] = k < nanc ? a.node_anc[(size_t)inf.node * kMaxDepth + k] : make_int2(0, 0);
      }
    }
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t s_addr = tmem + i * kBN + lane_off;
    const uint32_t o_addr = tmem + C::kOCol + i * D + lane_off;
    const float sl2 = a.scale_log2;
    float m_run = -CUDART_INF_F, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!wait_bar(B.s_full + 8 * i, j & 1, abort, a.status)) {
        ok = false;
        break;
      }
      fence_after_sync();
      float x[kBN];
      {
        uint32_t u[32];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          tmem_ld32(s_addr + c * 32, u);
#pragma unroll
          for (int k = 0; k < 32; ++k) x[c * 32 + k] = __uint_as_float(u[k]) * sl2;
        }
      }
      const int kb = key_base(j);
      if (j < n_pre) {
        const int lim = p_hi - kb;
        if (lim < kBN) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c >= lim) x[c] = -CUDART_INF_F;
        }
      } else {
        // suffix window: same branch up to the row's own token (+ ancestor nodes)
        const int c_lo = start - kb, c_hi = t - kb;
#pragma unroll
        for (int c = 0; c < kBN; ++c) {
          bool vis = c >= c_lo && c <= c_hi;
          if (TREE) {
#pragma unroll
            for (int k = 0; k < (TREE ? kMaxDepth : 1); ++k)
              if (k < nanc) vis |= (c >= anc[k].x - kb && c < anc[k].y - kb);
          }
          if (!vis) x[c] = -CUDART_INF_F;
        }
      }
      float mx = x[0];
#pragma unroll
      for (int c = 1; c < kBN; ++c) mx = fmaxf(mx, x[c]);
      float m_new = m_run;
      if (mx > m_run + kLazy || (m_run == -CUDART_INF_F && mx > -CUDART_INF_F)) m_new = mx;
      const float base = m_new == -CUDART_INF_F ? 0.f : m_new;
      const float alpha = ex2(m_run - base);
      float rs = 0.f;
#pragma unroll
      for (int h = 0; h < kBN / 64; ++h) {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = ex2(x[h * 64 + 2 * k] - base), p1 = ex2(x[h * 64 + 2 * k + 1] - base);
          rs += p0 + p1;
          pk[k] = pack_bf16(p0, p1);
        }
        tmem_st32(s_addr + h * 32, pk);
      }
      l_run = l_run * alpha + rs;
      if (j > 0 && __any_sync(0xffffffffu, m_new != m_run)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t u[32];
          tmem_ld32(o_addr + c * 32, u);
#pragma unroll
          for (int k = 0; k < 32; ++k) u[k] = __float_as_uint(__uint_as_float(u[k]) * alpha);
          tmem_st32(o_addr + c * 32, u);
        }
      }
      m_run = m_new;
      tmem_wait_st();
      fence_before_sync();
      mbar_arrive(B.p_full + 8 * i);
    }
    if (ok) ok = wait_bar(B.o_full + 8 * i, 0, abort, a.status);
    fence_after_sync();
    const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
    const bool write = ok && valid && t >= 0;
    const int tt = valid ? m / a.G : 0;
    const int h = valid ? min(max(a.hinv[g * a.G + (m - tt * a.G)], 0), a.Hq - 1) : 0;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t u[32];
      tmem_ld32(o_addr + c * 32, u);
      if (write) {
        if (a.S == 1) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + ((size_t)tt * a.Hq + h) * D + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(u[8 * v + 0]) * inv, __uint_as_float(u[8 * v + 1]) * inv);
            w.y = pack_bf16(__uint_as_float(u[8 * v + 2]) * inv, __uint_as_float(u[8 * v + 3]) * inv);
            w.z = pack_bf16(__uint_as_float(u[8 * v + 4]) * inv, __uint_as_float(u[8 * v + 5]) * inv);
            w.w = pack_bf16(__uint_as_float(u[8 * v + 6]) * inv, __uint_as_float(u[8 * v + 7]) * inv);
            dst[v] = w;
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(a.o_part + (((size_t)split * a.Hkv + g) * a.M + m) * D + c * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(u[4 * v]) * inv, __uint_as_float(u[4 * v + 1]) * inv,
                                 __uint_as_float(u[4 * v + 2]) * inv, __uint_as_float(u[4 * v + 3]) * inv);
        }
      }
    }
    if (write) {
      const float lse2 = l_run > 0.f ? m_run + __log2f(l_run) : -CUDART_INF_F;
      if (a.S == 1) {
        if (a.lse) a.lse[(size_t)tt * a.Hq + h] = lse2 * 0.69314718055994531f;
      } else {
        a.l_part[((size_t)split * a.Hkv + g) * a.M + m] = lse2;
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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
bool map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t stride) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t es[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_q(CUtensorMap* m, const void* base, int D, int M, int Hkv) {
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)M, (cuuint64_t)Hkv};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)M * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool TREE>
cudaError_t launch_dt(const AttnArgs& a, cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, TREE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg<D>::kSmem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  CUtensorMap mq, mkp, mvp, mks, mvs;
  memset(&mkp, 0, sizeof mkp);
  memset(&mvp, 0, sizeof mvp);
  const uint64_t row = (uint64_t)a.Hkv * D * 2;
  if (!map_q(&mq, a.q_rot, D, a.M, a.Hkv)) return cudaErrorInvalidValue;
  if (a.Lp > 0 && (!map_2d(&mkp, a.k_pre, (uint64_t)a.Hkv * D, a.Lp, row) ||
                   !map_2d(&mvp, a.v_pre, (uint64_t)a.Hkv * D, a.Lp, row)))
    return cudaErrorInvalidValue;
  if (!map_2d(&mks, a.k_rot, (uint64_t)a.Hkv * D, a.T, row) || !map_2d(&mvs, a.v_suf, (uint64_t)a.Hkv * D, a.T, row))
    return cudaErrorInvalidValue;
  dim3 grid((a.M + 2 * kBM - 1) / (2 * kBM), a.Hkv, a.S);
  attn_tc_kernel<D, TREE><<<grid, kThreads, Cfg<D>::kSmem, s>>>(mq, mkp, mvp, mks, mvs, a);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(int d) {
  if (d != 64 && d != 128) return false;
  static int cc = -1;
  if (cc < 0) {
    int dev = 0, major = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      major = 0;
    }
    cc = major;
  }
  return cc == 10 && encode_fn() != nullptr;
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s) {
  if (a.M == 0) return cudaSuccess;
  const bool tree = a.node_nanc != nullptr;
  if (a.d == 128) return tree ? launch_dt<128, true>(a, s) : launch_dt<128, false>(a, s);
  return tree ? launch_dt<64, true>(a, s) : launch_dt<64, false>(a, s);
}

}  // namespace jev
