// attn_tc.cu — tensor-core shared-prefix attention for sm_100a (tcgen05 + TMEM + TMA).
//
// The prefix is shared by every branch ("How to Deploy Visual Jev ...", Step 3;
// "FastJEV ...", §3.2-§3.3), so all branches' queries of one kv group are
// stacked into one M dimension (row m = token m / G, query slot m % G) and the
// prefix K/V of that group streams through shared memory once per 256 stacked
// rows instead of once per branch.  After the prefix, a work tile also runs
// its suffix window: the suffix keys its rows may see (same branch up to the
// row's own token or, in a generation step, the branch's cache up to the
// row's slot; for tree tokens every ancestor node's keys too), masked per row.
//
// Schedule.  A work tile (256 stacked rows of one kv group) has P = n_pre + 1
// units: its 128-key prefix tiles and the suffix window.  n_ctas persistent
// CTAs first take whole tiles for full_waves rounds; the units of the
// remaining tail tiles are spread evenly over tail_ctas of them.  A CTA visits
// its work as segments (runs inside one tile).  A segment that covers its
// whole tile writes the final output; other segments write a normalised fp32
// partial and its log2 normaliser, and tc_fixup_kernel merges the segments of
// each split tail tile.
//
// CTA = 12 warps (384 threads, 168 registers each):
//   warps 0-3   Q tile 0: one thread per row (TMEM lane), all 128 score
//               columns of the row, then the row's output (the epilogue)
//   warps 4-7   Q tile 1, the same
//   warp 8      TMA producer (Q once per segment, then K/V through a ring of stages)
//   warp 9      TMEM allocator and tcgen05.mma issuer (one thread)
//   warps 10-11 no role (they complete the third warpgroup)
// TMEM (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 at 256, O1 at 256+D.
// Per key tile j the MMA thread issues S_i = Q_i K_j^T (SS form), and after
// the 128 threads of tile i have written P_i (bf16, aliasing S_i) it issues
// O_i += P_i V_j with P_i read from TMEM (TS form); tile 0's softmax overlaps
// tile 1's MMAs and the other way round.  A thread owns a whole row, so the
// row maximum needs no exchange; the softmax runs in the log2 domain with a
// lazy running max (raised only when a row's maximum exceeds it by more than
// 8, so O is rescaled rarely and P stays <= 2^8), its scale-and-subtract and
// row sums as packed f32x2 operations, and a share of its exponentials on the
// FMA pipe (a cubic with shifter range reduction): one exponential per score
// on the MUFU unit alone would take as long as the tile's MMAs.
// Every mbarrier wait is bounded; a wait that runs out raises
// JEV_DEV_WAIT_TIMEOUT in the status word and the CTA winds down: the other
// waits give up, but before the CTA exits the producer waits for every load
// it armed and the MMA warp for every MMA it issued.
#include <cuda.h>
#include <math_constants.h>

#include "kernels.h"
#include "tc_ptx.cuh"

namespace jev {
namespace {

using namespace tc;

constexpr int kBM = 128;  // rows per Q tile (TMEM lanes)
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kSoftWarps = 8;  // two warpgroups: one thread per row of each 128-row Q tile
// + the TMA producer and the MMA issuer, and two warps that only complete the
// last warpgroup: 384 threads leave 168 registers to a thread, room for a
// row's 128 scores
constexpr int kThreads = (kSoftWarps + 4) * 32;
constexpr int kProducerWarp = kSoftWarps;
constexpr int kMmaWarp = kSoftWarps + 1;
constexpr float kLazy = 8.0f;  // log2 headroom before the running max moves
// Share of softmax exponentials computed on the FMA pipe (every kPolyEvery-th
// score pair; 0 = none).  Measured on B200 at the wide workload: 0 is fastest
// (the softmax is issue-bound, not MUFU-bound), so it is off by default.
#ifndef JEV_POLY_EVERY
#define JEV_POLY_EVERY 0
#endif
constexpr int kPolyEvery = JEV_POLY_EVERY;

// K and V tiles stream through separate rings: a K tile is released as soon
// as its last S MMA has run, a V tile after its last PV MMA.
#ifndef JEV_K_STAGES
#define JEV_K_STAGES 3
#endif
#ifndef JEV_V_STAGES
#define JEV_V_STAGES 2
#endif
// Each segment sweeps its prefix key tiles starting at a tile that depends on
// its work tile, so the CTAs of one kv group are not all reading the same
// tile at the same moment.
#ifndef JEV_STAGGER
#define JEV_STAGGER 1
#endif

template <int D>
struct Cfg {
  static constexpr int kNK = D == 128 ? JEV_K_STAGES : 4;  // K stages
  static constexpr int kNV = D == 128 ? JEV_V_STAGES : 4;  // V stages
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kBlk = 128 * 128;  // one 64-column, 128-row swizzled block
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + kNK * kKVBytes;
  static constexpr int kOffBar = kOffV + kNV * kKVBytes;
  static constexpr int kOffSeg = kOffBar + 256;                  // two published segment descriptions
  static constexpr int kSmem = kOffSeg + 128 + 1024;                   // + 1024-byte alignment slack
  static constexpr int kOCol = 256;                               // first TMEM column of O0
};

struct Bars {
  uint32_t q_full, q_empty, k_full, k_empty, v_full, v_empty, s_full, p_full, o_full, drain;  // arrays: +8*i
};

struct Shared {
  uint32_t tmem_base;
  int abort;
};

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

// The suffix keys any row of the work tile may see: from the lowest window
// start to the highest last key (a tree row's last key is its own token).
__device__ __forceinline__ void tile_window(const AttnArgs& a, int m0, int lane, int& lo, int& hi) {
  const int m_end = min(m0 + 2 * kBM, a.M);
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
  int rot;        // the segment's prefix tiles are visited from tile ua + rot on, cyclically
};

// The prefix tiles of work tile w's segment of n_pre of them start at this offset.
__device__ __forceinline__ int seg_rot(int w, int n_pre) {
  return (JEV_STAGGER && n_pre > 1) ? (int)(((long long)w * 7) % n_pre) : 0;
}
// Unit (128-key prefix tile) of the segment's j-th prefix tile, j < n_pre.
__device__ __forceinline__ int pre_unit(int ua, int rot, int n_pre, int j) {
  const int x = j + rot;
  return ua + (x >= n_pre ? x - n_pre : x);
}
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

__device__ __forceinline__ Segment make_segment(const AttnArgs& a, int c, int w, int ua, int ub, bool tail, int lane) {
  Segment sg;
  sg.w = w;
  sg.ua = ua;
  sg.ub = ub;
  const long long t0 = (long long)(w - a.tail0) * a.P;  // tail unit of the tile's first unit
  sg.g = sg.w / a.n_pairs;
  sg.m0 = (sg.w - sg.g * a.n_pairs) * 2 * kBM;
  sg.n_pre = max(0, min(sg.ub, a.n_pre) - sg.ua);
  int n_suf = 0;
  sg.lo = 0;
  if (sg.ub == a.P) {
    int lo, hi;
    tile_window(a, sg.m0, lane, lo, hi);
    sg.lo = lo;
    n_suf = lo <= hi ? (hi - lo + kBN) / kBN : 0;
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
  sg.rot = seg_rot(w, sg.n_pre);
  return sg;
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
  Shared* sh = reinterpret_cast<Shared*>(smem + C::kOffBar + 224);
  // The producer derives each segment's description (its key window takes a
  // warp-wide read of token info) and publishes it here before its arrive on
  // q_full; the other roles read it after their wait on q_full.  Two slots:
  // slot k & 1 is rewritten for segment k + 2 only after q_empty of segment
  // k + 1, by which time every role has read it.
  Segment* seg_sm = reinterpret_cast<Segment*>(smem + C::kOffSeg);
  const uint32_t bar0 = sbase + C::kOffBar;
  Bars B;
  B.q_full = bar0;
  B.q_empty = bar0 + 8;
  B.k_full = bar0 + 16;
  B.k_empty = B.k_full + 8 * C::kNK;
  B.v_full = B.k_empty + 8 * C::kNK;
  B.v_empty = B.v_full + 8 * C::kNV;
  B.s_full = B.v_empty + 8 * C::kNV;
  B.p_full = B.s_full + 16;
  B.o_full = B.p_full + 16;
  B.drain = B.o_full + 16;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const bool has_tail = a.U > 0 && cta < a.tail_ctas;
  const long long u_begin = has_tail ? tc_unit_begin(a, cta) : 0, u_end = has_tail ? tc_unit_begin(a, cta + 1) : 0;

  if (threadIdx.x == 0) {
    mbar_init(B.q_full, 2);  // the producer's expect-tx arrival, then its arrival after publishing the segment
    mbar_init(B.q_empty, 1);
    for (int s = 0; s < C::kNK; ++s) {
      mbar_init(B.k_full + 8 * s, 1);
      mbar_init(B.k_empty + 8 * s, 1);
    }
    for (int s = 0; s < C::kNV; ++s) {
      mbar_init(B.v_full + 8 * s, 1);
      mbar_init(B.v_empty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B.s_full + 8 * i, 1);
      mbar_init(B.p_full + 8 * i, kBM);  // one arrival per row of the tile
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
  // Everything above is independent of the previous kernel (the RoPE pack);
  // each role waits for it (pdl_wait) before it reads the pack's outputs:
  // rotated queries and suffix keys, token info and the head map.

  if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- TMA producer
    // Per segment: Q, then key tile 0's K, then for each tile j the K of tile
    // j + 1 ahead of the V of tile j (a K tile is needed one MMA earlier than
    // the V tile of the same index).  Key tile JJ (counted over the CTA's
    // segments) goes to K stage JJ % kNK and V stage JJ % kNV.
    long long J = 0;
    long long k_armed = 0, v_armed = 0;  // K / V tiles whose loads this warp has issued
    int q_armed = 0;                     // Q tiles loaded
    int k = 0;
    bool ok = true;
    // lane 0: load the K (or V) tile of the segment's j-th key tile (global index JJ)
    auto load_kv = [&](bool is_k, const Segment& sg, int j, long long JJ) -> bool {
      const int ns = is_k ? C::kNK : C::kNV;
      const int st = (int)(JJ % ns);
      const long long use = JJ / ns;
      if (JJ >= ns && !wait_bar((is_k ? B.k_empty : B.v_empty) + 8 * st, (uint32_t)((use - 1) & 1), abort, a.status,
                                a.wait_cycles))
        return false;
      const bool pre = j < sg.n_pre;
      const int kb = pre ? pre_unit(sg.ua, sg.rot, sg.n_pre, j) * kBN : sg.lo + (j - sg.n_pre) * kBN;
      const CUtensorMap* m = is_k ? (pre ? &tm_kp : &tm_ks) : (pre ? &tm_vp : &tm_vs);
      const uint32_t dst = sbase + (is_k ? C::kOffK : C::kOffV) + st * C::kKVBytes;
      const uint32_t full = (is_k ? B.k_full : B.v_full) + 8 * st;
      mbar_expect_tx(full, C::kKVBytes);
      for (int b = 0; b < D / 64; ++b) tma_load_2d(dst + b * C::kBlk, m, sg.g * D + b * 64, kb, full);
      if (is_k) k_armed = JJ + 1;
      else v_armed = JJ + 1;
      return true;
    };
    tma_prefetch_desc(&tm_q);
    // the first segment's leading prefix key tiles need nothing from the pack:
    // their loads start before the wait (the pack lets this kernel launch only
    // once every kernel before it in the stream has completed), in the same
    // order as below and only into stages not used before
    int pre_k = 0, pre_v = 0;
    {
      SegIter it0{0, u_begin, u_end};
      int w0, ua0, ub0;
      bool tl0;
      if (seg_next(a, cta, it0, w0, ua0, ub0, tl0)) {
        Segment s0{};
        s0.ua = ua0;
        s0.g = w0 / a.n_pairs;
        s0.n_pre = max(0, min(ub0, a.n_pre) - ua0);
        s0.rot = seg_rot(w0, s0.n_pre);
        pre_k = min(s0.n_pre, C::kNK);
        pre_v = min(s0.n_pre, C::kNV);
        if (lane == 0) {
          if (pre_k > 0) load_kv(true, s0, 0, 0);
          for (int j = 0; j < max(pre_k, pre_v); ++j) {
            if (j + 1 < pre_k) load_kv(true, s0, j + 1, j + 1);
            if (j < pre_v) load_kv(false, s0, j, j);
          }
        }
      }
    }
    pdl_wait();
    SegIter it{0, u_begin, u_end};
    int sw, sua, sub;
    bool stail;
    for (; ok && seg_next(a, cta, it, sw, sua, sub, stail); ++k, ++it.k) {
      // The Q tile goes first: it needs only the tile's group and rows.
      const int qg = sw / a.n_pairs, qm0 = (sw - qg * a.n_pairs) * 2 * kBM;
      if (lane == 0) {
        if (k > 0 && !wait_bar(B.q_empty, (k - 1) & 1, abort, a.status, a.wait_cycles)) ok = false;
        if (ok) {
          mbar_expect_tx(B.q_full, 2 * C::kQBytes);
          for (int i = 0; i < 2; ++i)
            for (int b = 0; b < D / 64; ++b)
              tma_load_3d(sbase + i * C::kQBytes + b * C::kBlk, &tm_q, b * 64, qm0 + i * kBM, qg, B.q_full);
          ++q_armed;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // The description (for the suffix unit, its key window: a warp-wide read
      // of token info) is published with q_full's second arrival.
      const Segment sg = make_segment(a, cta, sw, sua, sub, stail, lane);
      if (lane == 0) {
        if (ok) {
          seg_sm[k & 1] = sg;
          mbar_arrive(B.q_full);
        }
        const int dk = k == 0 ? pre_k : 0, dv = k == 0 ? pre_v : 0;  // tiles already loaded
        if (ok && dk == 0) ok = load_kv(true, sg, 0, J);
        for (int j = 0; ok && j < sg.n; ++j) {
          if (j + 1 < sg.n && j + 1 >= dk) ok = load_kv(true, sg, j + 1, J + j + 1);
          if (ok && j >= dv) ok = load_kv(false, sg, j, J + j);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      J += sg.n;
    }
    if (lane == 0) {
      // Drain: the last phase of every stage this warp armed, and of the Q
      // buffer, has completed (its loads have landed) before the CTA may
      // exit.  On the normal path these phases completed long ago.
      for (int st = 0; st < C::kNK; ++st) {
        const long long uses = k_armed > st ? (k_armed - st + C::kNK - 1) / C::kNK : 0;
        if (uses > 0) drain_bar(B.k_full + 8 * st, (uint32_t)((uses - 1) & 1), a.status);
      }
      for (int st = 0; st < C::kNV; ++st) {
        const long long uses = v_armed > st ? (v_armed - st + C::kNV - 1) / C::kNV : 0;
        if (uses > 0) drain_bar(B.v_full + 8 * st, (uint32_t)((uses - 1) & 1), a.status);
      }
      if (q_armed > 0) drain_bar(B.q_full, (uint32_t)((q_armed - 1) & 1), a.status);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t id_qk = idesc_bf16(kBM, kBN, false);
    constexpr uint32_t id_pv = idesc_bf16(kBM, D, true);
    // Shared-memory descriptors are formed once; an operand's descriptor is a
    // base plus its byte offset >> 4 in the address field (every operand lies
    // below 256 KB of shared memory, so the 14-bit field never carries), so
    // the one issuing thread spends a couple of instructions per MMA.
    const uint64_t dq0 = smem_desc_sw128(sbase, 16, 1024);
    const uint64_t dk0 = smem_desc_sw128(sbase + C::kOffK, 16, 1024);
    const uint64_t dv0 = smem_desc_sw128(sbase + C::kOffV, C::kBlk, 1024);
    auto issue_s = [&](int i, int st) {
      const uint64_t qa = dq0 + (uint32_t)((i * C::kQBytes) >> 4), ka = dk0 + (uint32_t)((st * C::kKVBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        constexpr int kBlk4 = C::kBlk >> 4;
        const uint32_t off = (uint32_t)((kk >> 2) * kBlk4 + (kk & 3) * 2);
        mma_ss(tmem + i * kBN, qa + off, ka + off, id_qk, kk > 0);
      }
      mma_commit(B.s_full + 8 * i);
    };
    auto issue_pv = [&](int i, int st, bool acc) {
      const uint64_t va = dv0 + (uint32_t)((st * C::kKVBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        mma_ts(tmem + C::kOCol + i * D, tmem + i * kBN + kk * 8, va + (uint32_t)(kk * 16 * 128 / 16), id_pv,
               (acc || kk > 0) ? 1u : 0u);
    };
    long long J = 0;
    int k = 0;
    bool ok = true;
    pdl_wait();
    SegIter it{0, u_begin, u_end};
    int sw, sua, sub;
    bool stail;
    for (; ok && seg_next(a, cta, it, sw, sua, sub, stail); ++k, ++it.k) {
      ok = wait_bar(B.q_full, k & 1, abort, a.status, a.wait_cycles);
      const Segment sg = seg_sm[k & 1];
      if (lane == 0) {
        const int n = sg.n;  // >= 1
        if (ok) {
          const int sk0 = (int)(J % C::kNK);
          ok = wait_bar(B.k_full + 8 * sk0, (uint32_t)((J / C::kNK) & 1), abort, a.status, a.wait_cycles);
          fence_after_sync();
          if (ok) {
            issue_s(0, sk0);
            issue_s(1, sk0);
            mma_commit(B.k_empty + 8 * sk0);  // the K tile's last MMA
          }
        }
        for (int j = 0; ok && j < n; ++j) {
          const long long JJ = J + j, JJ1 = JJ + 1;
          const int sv = (int)(JJ % C::kNV), sk1 = (int)(JJ1 % C::kNK);
          const uint32_t phv = (uint32_t)((JJ / C::kNV) & 1), phk1 = (uint32_t)((JJ1 / C::kNK) & 1);
          const uint32_t pp = (uint32_t)(JJ & 1);
          if (!wait_bar(B.v_full + 8 * sv, phv, abort, a.status, a.wait_cycles)) { ok = false; break; }
          if (!wait_bar(B.p_full, pp, abort, a.status, a.wait_cycles)) { ok = false; break; }
          fence_after_sync();
          issue_pv(0, sv, j > 0);
          if (j == n - 1) mma_commit(B.o_full);
          if (j + 1 < n) {
            if (!wait_bar(B.k_full + 8 * sk1, phk1, abort, a.status, a.wait_cycles)) { ok = false; break; }
            fence_after_sync();
            issue_s(0, sk1);
          }
          if (!wait_bar(B.p_full + 8, pp, abort, a.status, a.wait_cycles)) { ok = false; break; }
          fence_after_sync();
          issue_pv(1, sv, j > 0);
          mma_commit(B.v_empty + 8 * sv);  // the V tile's last MMA
          if (j == n - 1) mma_commit(B.o_full + 8);
          // q_empty releases the Q buffer and lets the producer publish the next
          // segment.  It is committed only after both p_full waits of a tile of
          // this segment, i.e. after all 512 softmax threads have passed their
          // q_full wait for it: were q_full to complete two phases ahead of a
          // softmax thread still in the previous epilogue, that thread's parity
          // wait would alias the later phase and never return.
          if (j + 1 < n) {
            issue_s(1, sk1);
            mma_commit(B.k_empty + 8 * sk1);
            if (j + 2 == n) mma_commit(B.q_empty);
          } else if (n == 1) {
            mma_commit(B.q_empty);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      J += sg.n;
    }
    if (lane == 0) {
      // every MMA of this CTA has completed before TMEM is released, on the
      // timeout path too (the wait ignores the abort flag)
      mma_commit(B.drain);
      drain_bar(B.drain, 0, a.status);
    }
  } else if (warp < kSoftWarps) {
    // ---------------------------------------------------------------- softmax + epilogue
    // warp w: tile i = w / 4, TMEM lanes 32 (w % 4) .. +31; thread = one row of
    // the tile's 128, holding all 128 of its scores (no exchange with another thread)
    const int i = warp >> 2, q = warp & 3, r = q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t s_addr = tmem + i * kBN + lane_off;  // the row's 128 score columns; P packed over the first 64
    const uint32_t o_addr = tmem + C::kOCol + i * D + lane_off;
    const float sl2 = a.scale_log2;
    long long J = 0;
    int k = 0;
    bool ok = true;
    pdl_wait();
    // every CTA has passed its wait: the merge kernel may launch now
    if (threadIdx.x == 0) pdl_trigger();
    SegIter it{0, u_begin, u_end};
    int sw, sua, sub;
    bool stail;
    for (; ok && seg_next(a, cta, it, sw, sua, sub, stail); ++k, ++it.k) {
      // waits are warp-uniform: the TMEM loads and stores below are warp-wide
      ok = __all_sync(0xffffffffu, wait_bar(B.q_full, k & 1, abort, a.status, a.wait_cycles));
      if (!ok) break;
      const Segment sg = seg_sm[k & 1];
      const int m = sg.m0 + i * kBM + r;
      const bool valid = m < a.M;
      // t: the row's token (-1: not computed); suffix keys start .. last may be visible
      int t = -1, start = 0, last = -1;
      if (valid) {
        const TokInfo inf = a.info[m / a.G];
        if (inf.node >= 0) {
          t = m / a.G;
          start = inf.seg_start;
          last = TREE ? t : inf.last;
        }
      }
      float m_run = -CUDART_INF_F, l_run = 0.f;
      for (int j = 0; j < sg.n; ++j) {
        const long long JJ = J + j;
        ok = __all_sync(0xffffffffu, wait_bar(B.s_full + 8 * i, (uint32_t)(JJ & 1), abort, a.status, a.wait_cycles));
        if (!ok) break;
        fence_after_sync();
        // the row's 128 raw scores; P is later packed in place into xs[0..63]
        uint32_t xs[kBN];
        constexpr uint32_t kNegInf = 0xff800000u;
        auto load_masked = [&]() {
          tmem_ld128(s_addr, xs);
          if (j < sg.n_pre) {
            const int lim = a.Lp - pre_unit(sg.ua, sg.rot, sg.n_pre, j) * kBN;  // keys past the prefix are padding
            if (lim < kBN) {
#pragma unroll
              for (int c = 0; c < kBN; ++c)
                if (c >= lim) xs[c] = kNegInf;
            }
          } else {
            // suffix window
            const int kb = sg.lo + (j - sg.n_pre) * kBN;
            if (!TREE) {
              // flat row: the keys start .. last of its own branch
              const int c_lo = start - kb, c_hi = last - kb;
              // the mask is skipped when every row of the warp sees every key of this tile
              const bool whole = __all_sync(0xffffffffu, c_lo <= 0 && c_hi >= kBN - 1);
              if (!whole) {
#pragma unroll
                for (int c = 0; c < kBN; ++c)
                  if (!(c >= c_lo && c <= c_hi)) xs[c] = kNegInf;
              }
            } else {
              // tree row t: key k is on its root path when k <= t and t lies in the
              // packed tokens of k's node's subtree (read here, where needed)
#pragma unroll
              for (int c = 0; c < kBN; ++c) {
                const int kk = kb + c;
                const int e = kk < a.key_rows ? __ldg(a.key_end + kk) : -1;
                if (!(kk <= t && t < e)) xs[c] = kNegInf;
              }
            }
          }
        };
        // p = 2^(s * scale * log2e - base) for the row's 128 scores, packed in
        // place as bf16 pairs into xs[0..63]; returns the row sum.  The
        // scale-and-subtract and the sum run as packed f32x2 operations, every
        // kPolyEvery-th pair of exponentials on the FMA pipe, the rest on
        // MUFU.  With `mxp`, the maximum of the raw scores is taken alongside.
        auto exp_pack = [&](float base, float* mxp) -> float {
          const uint64_t sc2 = f2_pack(sl2, sl2), nb2 = f2_pack(-base, -base);
          uint64_t ps2[4];
          float pm[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            ps2[q4] = 0;
            pm[q4] = -CUDART_INF_F;
          }
#pragma unroll
          for (int kk = 0; kk < kBN / 2; ++kk) {
            if (mxp) pm[kk & 3] = fmax3(pm[kk & 3], __uint_as_float(xs[2 * kk]), __uint_as_float(xs[2 * kk + 1]));
            const uint64_t x2 = f2_fma(((uint64_t)xs[2 * kk + 1] << 32) | xs[2 * kk], sc2, nb2);
            const bool fma_pipe = kPolyEvery > 0 && (kk % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1;
            const uint64_t p2 = fma_pipe ? exp2_fma2(x2) : f2_pack(ex2(f2_lo(x2)), ex2(f2_hi(x2)));
            ps2[kk & 3] = f2_add(ps2[kk & 3], p2);
            xs[kk] = pack_bf16(f2_lo(p2), f2_hi(p2));
          }
          if (mxp) *mxp = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
          const uint64_t s03 = f2_add(f2_add(ps2[0], ps2[1]), f2_add(ps2[2], ps2[3]));
          return f2_lo(s03) + f2_hi(s03);
        };
        load_masked();
        float m_new, rs;
        if (__all_sync(0xffffffffu, m_run != -CUDART_INF_F)) {
          // every row of the warp has a running maximum: the exponentials start
          // from it at once and the tile's maximum is found alongside; only a
          // row whose maximum rises by more than kLazy (rare) makes the warp
          // reload S and start again from the new maxima
          float mxs;
          rs = exp_pack(m_run, &mxs);
          const float mx = mxs * sl2;
          const bool raise = mx > m_run + kLazy;
          m_new = raise ? mx : m_run;
          if (__any_sync(0xffffffffu, raise)) {
            load_masked();
            rs = exp_pack(m_new, nullptr);
          }
        } else {
          // the row's maximum first (the first tile, or rows still without one)
          float pm[8];
#pragma unroll
          for (int q8 = 0; q8 < 8; ++q8) pm[q8] = __uint_as_float(xs[q8]);
#pragma unroll
          for (int c = 8; c < kBN; c += 2)
            pm[(c >> 1) & 7] = fmax3(pm[(c >> 1) & 7], __uint_as_float(xs[c]), __uint_as_float(xs[c + 1]));
          const float mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7])) * sl2;
          m_new = m_run;
          if (mx > m_run + kLazy || (m_run == -CUDART_INF_F && mx > -CUDART_INF_F)) m_new = mx;
          rs = exp_pack(m_new == -CUDART_INF_F ? 0.f : m_new, nullptr);
        }
        const float alpha = ex2(m_run - (m_new == -CUDART_INF_F ? 0.f : m_new));
        tmem_st32(s_addr, *reinterpret_cast<const uint32_t(*)[32]>(&xs[0]));
        tmem_st32(s_addr + 32, *reinterpret_cast<const uint32_t(*)[32]>(&xs[32]));
        l_run = l_run * alpha + rs;
        // O holds the tiles before j (their PV completed before this tile's S
        // did); rescale it when some row of the warp raised its maximum
        if (j > 0 && __any_sync(0xffffffffu, m_new != m_run)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t uu[32];
            tmem_ld32(o_addr + c * 32, uu);
#pragma unroll
            for (int e = 0; e < 32; ++e) uu[e] = __float_as_uint(__uint_as_float(uu[e]) * alpha);
            tmem_st32(o_addr + c * 32, uu);
          }
        }
        m_run = m_new;
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(B.p_full + 8 * i);
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, wait_bar(B.o_full + 8 * i, (uint32_t)(k & 1), abort, a.status, a.wait_cycles));
      if (!ok) break;
      fence_after_sync();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      const bool write = valid && t >= 0;
      const int tt = valid ? m / a.G : 0;
      const int h = valid ? min(max(a.hinv[sg.g * a.G + (m - tt * a.G)], 0), a.Hq - 1) : 0;
      if (sg.complete) {
        // bf16 output row (t, h): D * 2 contiguous bytes, 64 per 32 columns
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) + ((size_t)tt * a.Hq + h) * D);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t uu[32];
          tmem_ld32(o_addr + c * 32, uu);
          if (write) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              dst[c * 4 + e] = make_uint4(pack_bf16(__uint_as_float(uu[8 * e]) * inv, __uint_as_float(uu[8 * e + 1]) * inv),
                                          pack_bf16(__uint_as_float(uu[8 * e + 2]) * inv, __uint_as_float(uu[8 * e + 3]) * inv),
                                          pack_bf16(__uint_as_float(uu[8 * e + 4]) * inv, __uint_as_float(uu[8 * e + 5]) * inv),
                                          pack_bf16(__uint_as_float(uu[8 * e + 6]) * inv, __uint_as_float(uu[8 * e + 7]) * inv));
          }
        }
      } else {
        // fp32 partial rows, stored [slot][row / 32][column / 4][row % 32] as
        // float4 so that a warp's 32 rows fill 512 contiguous bytes per store
        float4* dst = reinterpret_cast<float4*>(a.o_part) +
                      ((size_t)(sg.slot * (2 * kBM / 32) + i * (kBM / 32) + q) * (D / 4)) * 32 + lane;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t uu[32];
          tmem_ld32(o_addr + c * 32, uu);
          if (write) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[(size_t)(c * 8 + v) * 32] =
                  make_float4(__uint_as_float(uu[4 * v]) * inv, __uint_as_float(uu[4 * v + 1]) * inv,
                              __uint_as_float(uu[4 * v + 2]) * inv, __uint_as_float(uu[4 * v + 3]) * inv);
          }
        }
      }
      const float lse2 = l_run > 0.f ? m_run + __log2f(l_run) : -CUDART_INF_F;
      if (sg.complete) {
        if (write && a.lse) a.lse[(size_t)tt * a.Hq + h] = lse2 * 0.69314718055994531f;
      } else {
        // rows outside the problem merge to nothing
        a.l_part[(size_t)sg.slot * 2 * kBM + i * kBM + r] = write ? lse2 : -CUDART_INF_F;
      }
      J += sg.n;
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the partial segments of every work tile the schedule split.  Block
// (w, y, z) covers rows [32y, 32y + 32) of tail tile w, one row per lane, and
// the z-th group of 8 * kCols float4 columns; warp c of the block takes
// columns c, c + 8, ... of the group, so every load of a partial (stored
// row-minor in float4 columns) or of a normaliser is one contiguous 512- or
// 128-byte access.  The partials were just written and sit in L2, so the
// merge is latency-bound: the normalisers and partial rows of kBatch segments
// are in flight together, and an online log-sum-exp rescaling folds each
// batch into the running result (the split merge rule applied
// incrementally).  Tiles split into few segments take (kCols, kBatch) =
// (all columns / 8, 4), tiles split into many take half the columns and 8.
// A tile that one CTA finished is skipped.
constexpr int kFixRows = 32;

template <int D, int kCols, int kFixBatch>
__global__ void __launch_bounds__(256) tc_fixup_kernel(const AttnArgs a) {
  const int w = a.tail0 + blockIdx.x;  // only tail tiles can be split
  const long long t0 = (long long)blockIdx.x * a.P;
  const int c_lo = tc_cta_of(a, t0), c_hi = tc_cta_of(a, t0 + a.P - 1);
  if (c_lo == c_hi) return;  // one CTA finished this tile and wrote it
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * kFixRows + lane;  // row within the 256-row tile
  const int g = w / a.n_pairs, m = (w - g * a.n_pairs) * 2 * kBM + r;
  if (m >= a.M) return;
  const int nseg = c_hi - c_lo + 1;
  // CTA c_lo holds this tile as its first segment only if its range starts here
  const int slot_lo = tc_unit_begin(a, c_lo) >= t0 ? 2 * c_lo : 2 * c_lo + 1;
  auto slot_of = [&](int s) { return s == 0 ? slot_lo : 2 * (c_lo + s); };
  const int t = m / a.G;
  if (a.info[t].node < 0) return;  // a skipped row is left as it was
  const int h = min(max(a.hinv[g * a.G + (m - t * a.G)], 0), a.Hq - 1);  // written before the attention kernel
  const int c4 = blockIdx.z * 8 * kCols + warp;  // this thread's first float4 column
  const float4* op = reinterpret_cast<const float4*>(a.o_part) + (size_t)(r >> 5) * (D / 4) * 32 + c4 * 32 + (r & 31);
  pdl_wait();  // the partials are written by the attention kernel
  float mx = -CUDART_INF_F, wsum = 0.f;
  float4 acc[kCols];
#pragma unroll
  for (int c = 0; c < kCols; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < nseg; s0 += kFixBatch) {
    float lv[kFixBatch];
    float4 ov[kFixBatch][kCols];
#pragma unroll
    for (int e = 0; e < kFixBatch; ++e) {
      lv[e] = -CUDART_INF_F;
      if (s0 + e < nseg) {
        const int slot = slot_of(s0 + e);
        lv[e] = a.l_part[(size_t)slot * 2 * kBM + r];
        const float4* src = op + (size_t)slot * (2 * kBM / 32) * (D / 4) * 32;
#pragma unroll
        for (int c = 0; c < kCols; ++c) ov[e][c] = src[c * 8 * 32];
      } else {
#pragma unroll
        for (int c = 0; c < kCols; ++c) ov[e][c] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float bm = lv[0];
#pragma unroll
    for (int e = 1; e < kFixBatch; ++e) bm = fmaxf(bm, lv[e]);
    const float m_new = fmaxf(mx, bm);
    if (m_new == -CUDART_INF_F) continue;
    const float sc = exp2f(mx - m_new);  // 0 while nothing has been folded in
    wsum *= sc;
#pragma unroll
    for (int c = 0; c < kCols; ++c) {
      acc[c].x *= sc; acc[c].y *= sc; acc[c].z *= sc; acc[c].w *= sc;
    }
#pragma unroll
    for (int e = 0; e < kFixBatch; ++e) {
      const float we = exp2f(lv[e] - m_new);  // 0 for absent segments; their rows are never read
      if (we > 0.f) {
        wsum += we;
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
          acc[c].x = fmaf(we, ov[e][c].x, acc[c].x);
          acc[c].y = fmaf(we, ov[e][c].y, acc[c].y);
          acc[c].z = fmaf(we, ov[e][c].z, acc[c].z);
          acc[c].w = fmaf(we, ov[e][c].w, acc[c].w);
        }
      }
    }
    mx = m_new;
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + ((size_t)t * a.Hq + h) * D + c4 * 4;
#pragma unroll
  for (int c = 0; c < kCols; ++c)
    *reinterpret_cast<uint2*>(o + c * 32) =
        make_uint2(pack_bf16(acc[c].x * inv, acc[c].y * inv), pack_bf16(acc[c].z * inv, acc[c].w * inv));
  if (a.lse && c4 == 0)
    a.lse[(size_t)t * a.Hq + h] = wsum > 0.f ? (mx + log2f(wsum)) * 0.69314718055994531f : -CUDART_INF_F;
}

__global__ void exp2_selftest_kernel(const float* x, float* y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) y[i] = exp2_fma(x[i]);
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
  if (!map_2d(&mks, a.k_rot, (uint64_t)a.Hkv * D, a.key_rows, row) ||
      !map_2d(&mvs, a.v_suf, (uint64_t)a.Hkv * D, a.key_rows, row))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(a.n_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = Cfg<D>::kSmem;
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel<D, TREE>, mq, mkp, mvp, mks, mvs, a);
}

}  // namespace

cudaError_t launch_exp2_selftest(const float* x, float* y, int n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

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

cudaError_t launch_tc_fixup(const AttnArgs& a, cudaStream_t s) {
  if (a.tail_ctas < 2 || a.n_tiles <= a.tail0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  // the most segments any tail tile is split into
  const long long max_segs = ((long long)a.P * a.tail_ctas + a.U - 1) / a.U + 1;
  const bool many = max_segs > 4;
  const int z = many ? 2 : 1;
  cfg.gridDim = dim3(a.n_tiles - a.tail0, 2 * kBM / kFixRows, z);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.d == 128)
    return many ? cudaLaunchKernelEx(&cfg, tc_fixup_kernel<128, 2, 8>, a) : cudaLaunchKernelEx(&cfg, tc_fixup_kernel<128, 4, 4>, a);
  return many ? cudaLaunchKernelEx(&cfg, tc_fixup_kernel<64, 1, 8>, a) : cudaLaunchKernelEx(&cfg, tc_fixup_kernel<64, 2, 4>, a);
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s) {
  if (a.M == 0 || a.n_ctas == 0) return cudaSuccess;
  const bool tree = a.key_end != nullptr;
  if (a.d == 128) return tree ? launch_dt<128, true>(a, s) : launch_dt<128, false>(a, s);
  return tree ? launch_dt<64, true>(a, s) : launch_dt<64, false>(a, s);
}

}  // namespace jev
