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
// CTA = 18 warps:
//   warps 0-7   Q tile 0: warps 0-3 columns 0-63, warps 4-7 columns 64-127 of
//               the S/P rows (TMEM lanes 0-127), and the matching halves of O
//   warps 8-15  Q tile 1, same split
//   warp 16     TMA producer (Q once per segment, then K/V through a ring of stages)
//   warp 17     TMEM allocator and tcgen05.mma issuer (the loop runs warp-wide;
//               an elected lane issues each MMA and commit)
// TMEM (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 at 256, O1 at 256+D.
// Per key tile j the MMA warp issues S_i = Q_i K_j^T (SS form), and after
// both halves of tile i have written P_i (bf16, aliasing S_i) it issues
// O_i += P_i V_j with P_i read from TMEM (TS form); tile 0's softmax overlaps
// tile 1's MMAs and the other way round.  The two halves of a row exchange
// their maxima through shared memory each key tile (a 64-thread barrier per
// pair of warps); the softmax runs in the log2 domain with a lazy running max
// (raised only when a row's maximum exceeds it by more than 8, so O is
// rescaled rarely and P stays <= 2^8), its scale-and-subtract and row sums as
// packed f32x2 operations.
// Every mbarrier wait is bounded; a wait that runs out raises
// JEV_DEV_WAIT_TIMEOUT in the status word and the CTA winds down: the other
// waits give up, but before the CTA exits the producer waits for every load
// it armed and the MMA warp for every MMA it issued.
#include <cuda.h>
#include <math_constants.h>

#include "attn_tc_common.cuh"

namespace jev {
namespace {

using namespace tc;
using namespace tca;

constexpr int kBM = 128;  // rows per Q tile (TMEM lanes)
constexpr int kBN = 128;  // keys per K/V tile
constexpr int kSoftWarps = 16;
constexpr int kThreads = (kSoftWarps + 2) * 32;
constexpr int kProducerWarp = kSoftWarps;
constexpr int kMmaWarp = kSoftWarps + 1;
constexpr float kLazy = 8.0f;  // log2 headroom before the running max moves
// Share of softmax exponentials computed on the FMA pipe (every kPolyEvery-th
// score pair, as one packed f32x2 polynomial; 0 = none).  Measured on B200,
// attention call alone: every 8th pair (12.5%) is fastest, about 1.8% below
// none at the wide workload; every 2nd, 4th, 6th or 12th pair is slower than
// none (the softmax is mostly bound by issue and latency, and MUFU is about
// half busy).
#ifndef JEV_POLY_EVERY
#define JEV_POLY_EVERY 8
#endif
constexpr int kPolyEvery = JEV_POLY_EVERY;

template <int D>
struct Cfg {
  static constexpr int kNS = D == 128 ? 2 : 4;  // K/V stages
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kBlk = 128 * 128;  // one 64-column, 128-row swizzled block
  static constexpr int kOffK = 2 * kQBytes;
  static constexpr int kOffV = kOffK + kNS * kKVBytes;
  static constexpr int kOffBar = kOffV + kNS * kKVBytes;
  static constexpr int kOffX = kOffBar + 256;                     // row-max exchange [tile][parity][half][row]
  static constexpr int kOffL = kOffX + 2 * 2 * 2 * kBM * 4;       // row-sum exchange [tile][half][row]
  static constexpr int kOffStg = kOffL + 2 * 2 * kBM * 4;        // per-warp output staging
  static constexpr int kStgBytes = 8 * 64;                         // 8 rows x 32 bf16 columns
  static constexpr int kOffSeg = kOffStg + kSoftWarps * kStgBytes;  // two published segment descriptions
  static constexpr int kSmem = kOffSeg + 128 + 1024;                   // + 1024-byte alignment slack
  static constexpr int kOCol = 256;                               // first TMEM column of O0
};

struct Bars {
  uint32_t q_full, q_empty, k_full, v_full, kv_empty, s_full, p_full, o_full, drain, probe;  // arrays: +8*i
};

struct Shared {
  uint32_t tmem_base;
  int abort;
};

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
  float* xmax = reinterpret_cast<float*>(smem + C::kOffX);
  float* xsum = reinterpret_cast<float*>(smem + C::kOffL);
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
  B.v_full = B.k_full + 8 * C::kNS;
  B.kv_empty = B.v_full + 8 * C::kNS;
  B.s_full = B.kv_empty + 8 * C::kNS;
  B.p_full = B.s_full + 16;
  B.o_full = B.p_full + 16;
  B.drain = B.o_full + 16;
  B.probe = B.drain + 8;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const bool has_tail = a.U > 0 && cta < a.tail_ctas;
  const long long u_begin = has_tail ? tc_unit_begin(a, cta) : 0, u_end = has_tail ? tc_unit_begin(a, cta + 1) : 0;

  if (threadIdx.x == 0) {
    mbar_init(B.q_full, 2);  // the producer's expect-tx arrival, then its arrival after publishing the segment
    mbar_init(B.q_empty, 1);
    for (int s = 0; s < C::kNS; ++s) {
      mbar_init(B.k_full + 8 * s, 1);
      mbar_init(B.v_full + 8 * s, 1);
      mbar_init(B.kv_empty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B.s_full + 8 * i, 1);
      mbar_init(B.p_full + 8 * i, 256);
      mbar_init(B.o_full + 8 * i, 1);
    }
    mbar_init(B.drain, 1);
    mbar_init(B.probe, 1);  // nothing arrives on it
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
    // The whole warp runs the loop (its values stay warp-uniform); one
    // elected lane issues each load.
    long long J = 0;
    long long kv_armed = 0;  // key tiles whose K and V loads this warp has issued
    int q_armed = 0;         // Q tiles loaded
    int k = 0;
    bool ok = true;
    if (lane == 0) tma_prefetch_desc(&tm_q);
    // the first segment's leading prefix key tiles need nothing from the pack:
    // their loads start before the wait (the pack lets this kernel launch only
    // once every kernel before it in the stream has completed)
    int pre0 = 0;
    {
      SegIter it0{0, u_begin, u_end};
      int w0, ua0, ub0;
      bool tl0;
      if (seg_next(a, cta, it0, w0, ua0, ub0, tl0)) {
        pre0 = min(max(0, min(ub0, a.n_pre) - ua0), C::kNS);
        const int g0 = w0 / a.n_mt;
        for (int j = 0; j < pre0; ++j) {
          const uint32_t ks = sbase + C::kOffK + j * C::kKVBytes, vs = sbase + C::kOffV + j * C::kKVBytes;
          mbar_expect_tx_w(B.k_full + 8 * j, C::kKVBytes);
          for (int b = 0; b < D / 64; ++b)
            tma_load_2d_w(ks + b * C::kBlk, &tm_kp, g0 * D + b * 64, (ua0 + j) * kBN, B.k_full + 8 * j);
          mbar_expect_tx_w(B.v_full + 8 * j, C::kKVBytes);
          for (int b = 0; b < D / 64; ++b)
            tma_load_2d_w(vs + b * C::kBlk, &tm_vp, g0 * D + b * 64, (ua0 + j) * kBN, B.v_full + 8 * j);
        }
        kv_armed = pre0;
      }
    }
    pdl_wait();
    SegIter it{0, u_begin, u_end};
    int sw, sua, sub;
    bool stail;
    for (; ok && seg_next(a, cta, it, sw, sua, sub, stail); ++k, ++it.k) {
      // The Q tile goes first: it needs only the tile's group and rows.
      const int qg = sw / a.n_mt, qm0 = (sw - qg * a.n_mt) * 2 * kBM;
      if (k > 0 && !wait_bar_w(B.q_empty, (k - 1) & 1, abort, a.status, a.wait_cycles)) ok = false;
      if (ok) {
        mbar_expect_tx_w(B.q_full, 2 * C::kQBytes);
        for (int i = 0; i < 2; ++i)
          for (int b = 0; b < D / 64; ++b)
            tma_load_3d_w(sbase + i * C::kQBytes + b * C::kBlk, &tm_q, b * 64, qm0 + i * kBM, qg, B.q_full);
        ++q_armed;
      }
      // The description (for the suffix unit, its key window: a warp-wide read
      // of token info) is published with q_full's second arrival.
      const Segment sg = make_segment<2 * kBM>(a, cta, sw, sua, sub, stail, lane);
      if (ok) {
        if (lane == 0) {
          seg_sm[k & 1] = sg;
          mbar_arrive(B.q_full);
        }
        __syncwarp();
        for (int j = k == 0 ? pre0 : 0; ok && j < sg.n; ++j) {
          const long long JJ = J + j;
          const int st = (int)(JJ % C::kNS);
          const long long use = JJ / C::kNS;
          if (JJ >= C::kNS &&
              !wait_bar_w(B.kv_empty + 8 * st, (uint32_t)((use - 1) & 1), abort, a.status, a.wait_cycles)) {
            ok = false;
            break;
          }
          const bool pre = j < sg.n_pre;
          const int kb = pre ? (sg.ua + j) * kBN : sg.lo + (j - sg.n_pre) * kBN;
          const CUtensorMap* mk = pre ? &tm_kp : &tm_ks;
          const CUtensorMap* mv = pre ? &tm_vp : &tm_vs;
          const uint32_t ks = sbase + C::kOffK + st * C::kKVBytes, vs = sbase + C::kOffV + st * C::kKVBytes;
          mbar_expect_tx_w(B.k_full + 8 * st, C::kKVBytes);
          for (int b = 0; b < D / 64; ++b)
            tma_load_2d_w(ks + b * C::kBlk, mk, sg.g * D + b * 64, kb, B.k_full + 8 * st);
          mbar_expect_tx_w(B.v_full + 8 * st, C::kKVBytes);
          for (int b = 0; b < D / 64; ++b)
            tma_load_2d_w(vs + b * C::kBlk, mv, sg.g * D + b * 64, kb, B.v_full + 8 * st);
          kv_armed = JJ + 1;
        }
      }
      J += sg.n;
    }
    if (lane == 0) {
      // Drain: the last phase of every stage this warp armed, and of the Q
      // buffer, has completed (its loads have landed) before the CTA may
      // exit.  On the normal path these phases completed long ago.
      for (int st = 0; st < C::kNS; ++st) {
        const long long uses = kv_armed > st ? (kv_armed - st + C::kNS - 1) / C::kNS : 0;
        if (uses > 0) {
          drain_bar(B.k_full + 8 * st, (uint32_t)((uses - 1) & 1), a.status);
          drain_bar(B.v_full + 8 * st, (uint32_t)((uses - 1) & 1), a.status);
        }
      }
      if (q_armed > 0) drain_bar(B.q_full, (uint32_t)((q_armed - 1) & 1), a.status);
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop, so descriptors and addresses stay
    // warp-uniform; one elected lane issues each MMA and commit.
    constexpr uint32_t id_qk = idesc_bf16(kBM, kBN, false);
    constexpr uint32_t id_pv = idesc_bf16(kBM, D, true);
    // Shared-memory descriptors are formed once; an operand's descriptor is a
    // base plus its byte offset >> 4 in the address field (every operand lies
    // below 256 KB of shared memory, so the 14-bit field never carries), so
    // each MMA costs the warp's loop a couple of instructions.
    const uint64_t dq0 = smem_desc_sw128(sbase, 16, 1024);
    const uint64_t dk0 = smem_desc_sw128(sbase + C::kOffK, 16, 1024);
    const uint64_t dv0 = smem_desc_sw128(sbase + C::kOffV, C::kBlk, 1024);
    auto issue_s = [&](int i, int st) {
      const uint64_t qa = dq0 + (uint32_t)((i * C::kQBytes) >> 4), ka = dk0 + (uint32_t)((st * C::kKVBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        constexpr int kBlk4 = C::kBlk >> 4;
        const uint32_t off = (uint32_t)((kk >> 2) * kBlk4 + (kk & 3) * 2);
        mma_ss_w(tmem + i * kBN, qa + off, ka + off, id_qk, kk > 0);
      }
      mma_commit_w(B.s_full + 8 * i);
    };
    auto issue_pv = [&](int i, int st, bool acc) {
      const uint64_t va = dv0 + (uint32_t)((st * C::kKVBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        mma_ts_w(tmem + C::kOCol + i * D, tmem + i * kBN + kk * 8, va + (uint32_t)(kk * 16 * 128 / 16), id_pv,
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
      ok = wait_bar_w(B.q_full, k & 1, abort, a.status, a.wait_cycles);
      const Segment sg = seg_sm[k & 1];
      {
        const int n = sg.n;  // >= 1
        if (ok) {
          const int st0 = (int)(J % C::kNS);
          ok = wait_bar_w(B.k_full + 8 * st0, (uint32_t)((J / C::kNS) & 1), abort, a.status, a.wait_cycles);
          fence_after_sync();
          if (ok) {
            issue_s(0, st0);
            issue_s(1, st0);
          }
          // failure-detection probe (off unless a test sets it): a wait that
          // nothing completes, with this segment's first MMAs in flight
          if (ok && k == 0 && a.wait_probe)
            ok = __shfl_sync(0xffffffffu, probe_wait(B.probe, abort, a.status, a.wait_cycles), 0);
        }
        for (int j = 0; ok && j < n; ++j) {
          const long long JJ = J + j, JJ1 = JJ + 1;
          const int st = (int)(JJ % C::kNS), st1 = (int)(JJ1 % C::kNS);
          const uint32_t ph = (uint32_t)((JJ / C::kNS) & 1), ph1 = (uint32_t)((JJ1 / C::kNS) & 1);
          const uint32_t pp = (uint32_t)(JJ & 1);
          if (!wait_bar_w(B.v_full + 8 * st, ph, abort, a.status, a.wait_cycles)) { ok = false; break; }
          if (!wait_bar_w(B.p_full, pp, abort, a.status, a.wait_cycles)) { ok = false; break; }
          fence_after_sync();
          issue_pv(0, st, j > 0);
          if (j == n - 1) mma_commit_w(B.o_full);
          if (j + 1 < n) {
            if (!wait_bar_w(B.k_full + 8 * st1, ph1, abort, a.status, a.wait_cycles)) { ok = false; break; }
            fence_after_sync();
            issue_s(0, st1);
          }
          if (!wait_bar_w(B.p_full + 8, pp, abort, a.status, a.wait_cycles)) { ok = false; break; }
          fence_after_sync();
          issue_pv(1, st, j > 0);
          mma_commit_w(B.kv_empty + 8 * st);
          if (j == n - 1) mma_commit_w(B.o_full + 8);
          // q_empty releases the Q buffer and lets the producer publish the next
          // segment.  It is committed only after both p_full waits of a tile of
          // this segment, i.e. after all 512 softmax threads have passed their
          // q_full wait for it: were q_full to complete two phases ahead of a
          // softmax thread still in the previous epilogue, that thread's parity
          // wait would alias the later phase and never return.
          if (j + 1 < n) {
            issue_s(1, st1);
            if (j + 2 == n) mma_commit_w(B.q_empty);
          } else if (n == 1) {
            mma_commit_w(B.q_empty);
          }
        }
      }
      J += sg.n;
    }
    // every MMA of this CTA has completed before TMEM is released, on the
    // timeout path too (the wait ignores the abort flag); the commit comes
    // from the lane that issued the MMAs
    mma_commit_w(B.drain);
    drain_bar(B.drain, 0, a.status);
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    constexpr int kHalfCols = kBN / 2;  // score columns per thread
    constexpr int kHalfD = D / 2;       // output columns per thread
    const int i = warp >> 3, hf = (warp >> 2) & 1, q = warp & 3, r = q * 32 + lane;
    const int bar_id = 1 + i;  // named barrier of the 256 threads of tile i
    // named barrier of the two warps that hold the two halves of the same 32 rows
    const int pair_bar = 3 + i * 4 + q;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t s_addr = tmem + i * kBN + hf * kHalfCols + lane_off;       // this half's score columns
    const uint32_t p_addr = tmem + i * kBN + hf * (kHalfCols / 2) + lane_off;  // its packed P columns
    const uint32_t o_addr = tmem + C::kOCol + i * D + hf * kHalfD + lane_off;
    const int c_base = hf * kHalfCols;  // key column of this thread's first score
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
      // The 256 threads of the tile group agree on the q_full wait before any
      // reads the segment description: a thread whose wait gave up must not
      // read a description the producer may not have published, and the
      // group must run the same number of key tiles (the same named barriers).
      ok = named_sync_and(bar_id, 256, wait_bar(B.q_full, k & 1, abort, a.status, a.wait_cycles));
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
      // tree: the warp's first and last computed rows (tokens), for the
      // whole-tile test of the suffix window
      int w_lo = 0, w_hi = -1;
      if (TREE) {
        w_lo = warp_min_i(t >= 0 ? t : INT_MAX);
        w_hi = warp_max_i(t);
      }
      float m_run = -CUDART_INF_F, l_run = 0.f;
      // A wait that fails (a timeout somewhere in the CTA) does not leave the
      // loop: the thread runs the remaining tiles on whatever TMEM holds, so
      // that every thread of the tile group meets the same named barriers, and
      // the group agrees on the outcome at the epilogue's reducing barrier.
      for (int j = 0; j < sg.n; ++j) {
        const long long JJ = J + j;
        if (!wait_bar(B.s_full + 8 * i, (uint32_t)(JJ & 1), abort, a.status, a.wait_cycles)) ok = false;
        fence_after_sync();
        // this half's 64 raw scores; P is later packed in place into xs[0..31]
        uint32_t xs[kHalfCols];
        tmem_ld64(s_addr, xs);
        constexpr uint32_t kNegInf = 0xff800000u;
        if (j < sg.n_pre) {
          const int lim = a.Lp - (sg.ua + j) * kBN - c_base;  // keys past the prefix are padding
          if (lim < kHalfCols) {
#pragma unroll
            for (int c = 0; c < kHalfCols; ++c)
              if (c >= lim) xs[c] = kNegInf;
          }
        } else {
          // suffix window
          const int kb = sg.lo + (j - sg.n_pre) * kBN + c_base;
          if (!TREE) {
            // flat row: the keys start .. last of its own branch
            const int c_lo = start - kb, c_hi = last - kb;
            // the mask is skipped when every row of the warp sees all 64 of its keys in this tile
            const bool whole = __all_sync(0xffffffffu, c_lo <= 0 && c_hi >= kHalfCols - 1);
            if (!whole) {
#pragma unroll
              for (int c = 0; c < kHalfCols; ++c)
                if (!(c >= c_lo && c <= c_hi)) xs[c] = kNegInf;
            }
          } else {
            // tree row t: key k is on its root path when k <= t and t lies in the
            // packed tokens of k's node's subtree.  The warp's rows share the
            // tile's 64 keys: lane l reads the subtree ends of keys l and l + 32
            // once, and the mask is skipped when every key is at or before the
            // warp's first row and every subtree holds its last row.
            const int e_a = kb + lane < a.key_rows ? __ldg(a.key_end + kb + lane) : -1;
            const int e_b = kb + 32 + lane < a.key_rows ? __ldg(a.key_end + kb + 32 + lane) : -1;
            const bool whole = kb + kHalfCols - 1 <= w_lo && warp_min_i(min(e_a, e_b)) > w_hi;
            if (!whole) {
#pragma unroll
              for (int c = 0; c < kHalfCols; ++c) {
                const int e = __shfl_sync(0xffffffffu, c < 32 ? e_a : e_b, c & 31);
                if (!(kb + c <= t && t < e)) xs[c] = kNegInf;
              }
            }
          }
        }
        // this half's maximum with three-input max instructions (8 independent chains)
        float pm[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) pm[q8] = __uint_as_float(xs[q8]);
#pragma unroll
        for (int c = 8; c < kHalfCols; c += 2)
          pm[(c >> 1) & 7] = fmax3(pm[(c >> 1) & 7], __uint_as_float(xs[c]), __uint_as_float(xs[c + 1]));
        const float half_max = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
        // both halves of the row agree on the maximum (double-buffered by tile parity)
        float* xm = xmax + ((i * 2 + (int)(JJ & 1)) * 2) * kBM;
        xm[hf * kBM + r] = half_max;
        named_sync(pair_bar, 64);
        const float mx = fmaxf(half_max, xm[(1 - hf) * kBM + r]) * sl2;
        float m_new = m_run;
        if (mx > m_run + kLazy || (m_run == -CUDART_INF_F && mx > -CUDART_INF_F)) m_new = mx;
        const float base = m_new == -CUDART_INF_F ? 0.f : m_new;
        const float alpha = ex2(m_run - base);
        // p = 2^(s * scale * log2e - max): one exponential per score; the
        // scale-and-subtract and the row sum run as packed f32x2 operations
        // (one instruction per pair of scores)
        const uint64_t sc2 = f2_pack(sl2, sl2), nb2 = f2_pack(-base, -base);
        uint64_t ps2[4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) ps2[q4] = 0;
#pragma unroll
        for (int kk = 0; kk < kHalfCols / 2; ++kk) {
          const uint64_t x2 = f2_fma(((uint64_t)xs[2 * kk + 1] << 32) | xs[2 * kk], sc2, nb2);
          const bool fma_pipe = kPolyEvery > 0 && (kk % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1;
          const uint64_t p2 = fma_pipe ? exp2_fma2(x2) : f2_pack(ex2(f2_lo(x2)), ex2(f2_hi(x2)));
          ps2[kk & 3] = f2_add(ps2[kk & 3], p2);
          xs[kk] = pack_bf16(f2_lo(p2), f2_hi(p2));
        }
        tmem_st32(p_addr, *reinterpret_cast<const uint32_t(*)[32]>(&xs[0]));
        const uint64_t s01 = f2_add(ps2[0], ps2[1]), s23 = f2_add(ps2[2], ps2[3]);
        const uint64_t s03 = f2_add(s01, s23);
        const float rs = f2_lo(s03) + f2_hi(s03);
        l_run = l_run * alpha + rs;
        if (j > 0 && __any_sync(0xffffffffu, m_new != m_run)) {
#pragma unroll
          for (int c = 0; c < kHalfD / 32; ++c) {
            uint32_t uu[32];
            tmem_ld32(o_addr + c * 32, uu);
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) uu[kk] = __float_as_uint(__uint_as_float(uu[kk]) * alpha);
            tmem_st32(o_addr + c * 32, uu);
          }
        }
        m_run = m_new;
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(B.p_full + 8 * i);
      }
      if (ok) ok = wait_bar(B.o_full + 8 * i, (uint32_t)(k & 1), abort, a.status, a.wait_cycles);
      fence_after_sync();
      // the row's normaliser is the sum of both halves' partial sums
      xsum[(i * 2 + hf) * kBM + r] = l_run;
      ok = named_sync_and(bar_id, 256, ok);
      const float l_row = l_run + xsum[(i * 2 + 1 - hf) * kBM + r];
      named_sync(bar_id, 256);  // the exchange slots are free again
      const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
      const bool write = ok && valid && t >= 0;
      const int tt = valid ? m / a.G : 0;
      const int h = valid ? min(max(a.hinv[sg.g * a.G + (m - tt * a.G)], 0), a.Hq - 1) : 0;
      if (sg.complete) {
        // bf16 output rows (t, h) lie D*2 bytes apart or more; per 32 columns
        // a warp stages eight of its half-rows at a time in shared memory so
        // that each global store writes 64 contiguous bytes of each of 8 rows
        const unsigned long long dst_row =
            write ? reinterpret_cast<unsigned long long>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                                         ((size_t)tt * a.Hq + h) * D + hf * kHalfD)
                  : 0ull;
        uint8_t* stg = smem + C::kOffStg + warp * C::kStgBytes;
        const int rd_row = lane >> 2, rd_c = lane & 3;  // the 16-byte chunk this lane stores
#pragma unroll
        for (int c = 0; c < kHalfD / 32; ++c) {
          uint32_t uu[32];
          tmem_ld32(o_addr + c * 32, uu);
          uint32_t* pk = uu;  // packed in place: entry kk reads entries 2kk, 2kk+1 >= kk
#pragma unroll
          for (int kk = 0; kk < 16; ++kk)
            pk[kk] = pack_bf16(__uint_as_float(uu[2 * kk]) * inv, __uint_as_float(uu[2 * kk + 1]) * inv);
#pragma unroll
          for (int rq = 0; rq < 4; ++rq) {
            if ((lane >> 3) == rq) {
              const int rr = lane & 7;
#pragma unroll
              for (int e = 0; e < 4; ++e)
                *reinterpret_cast<uint4*>(stg + rr * 64 + ((e ^ (rr & 3)) * 16)) =
                    make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
            __syncwarp();
            const uint4 v = *reinterpret_cast<const uint4*>(stg + rd_row * 64 + ((rd_c ^ (rd_row & 3)) * 16));
            const unsigned long long d = __shfl_sync(0xffffffffu, dst_row, rq * 8 + rd_row);
            if (d) reinterpret_cast<uint4*>(d)[c * 4 + rd_c] = v;
            __syncwarp();
          }
        }
      } else {
        // fp32 partial rows, stored [slot][row / 32][column / 4][row % 32] as
        // float4 so that a warp's 32 rows fill 512 contiguous bytes per store
        float4* dst = reinterpret_cast<float4*>(a.o_part) +
                      ((size_t)(sg.slot * (2 * kBM / 32) + i * (kBM / 32) + q) * (D / 4)) * 32 + lane;
#pragma unroll
        for (int c = 0; c < kHalfD / 32; ++c) {
          uint32_t uu[32];
          tmem_ld32(o_addr + c * 32, uu);
          if (write) {
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[(size_t)((hf * kHalfD + c * 32) / 4 + v) * 32] =
                  make_float4(__uint_as_float(uu[4 * v]) * inv, __uint_as_float(uu[4 * v + 1]) * inv,
                              __uint_as_float(uu[4 * v + 2]) * inv, __uint_as_float(uu[4 * v + 3]) * inv);
          }
        }
      }
      const size_t prow = (size_t)sg.slot * 2 * kBM + i * kBM + r;  // partial row of this thread
      if (hf == 0) {
        const float lse2 = l_row > 0.f ? m_run + __log2f(l_row) : -CUDART_INF_F;
        if (write) {
          if (sg.complete) {
            if (a.lse) a.lse[(size_t)tt * a.Hq + h] = lse2 * 0.69314718055994531f;
          } else {
            a.l_part[prow] = lse2;
          }
        } else if (!sg.complete && ok) {
          a.l_part[prow] = -CUDART_INF_F;  // rows outside the problem merge to nothing
        }
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
// (2, 4), tiles split into many (1, 8); grid.z covers the rest of the
// columns, and 64 registers a thread keep four blocks on an SM, so the grid
// runs in about one wave.  A tile that one CTA finished is skipped.
constexpr int kFixRows = 32;

template <int D, int kCols, int kFixBatch>
__global__ void __launch_bounds__(256, 4) tc_fixup_kernel(const AttnArgs a) {
  const int w = a.tail0 + blockIdx.x;  // only tail tiles can be split
  const long long t0 = (long long)blockIdx.x * a.P;
  const int c_lo = tc_cta_of(a, t0), c_hi = tc_cta_of(a, t0 + a.P - 1);
  if (c_lo == c_hi) return;  // one CTA finished this tile and wrote it
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * kFixRows + lane;  // row within the work tile
  const int g = w / a.n_mt, m = (w - g * a.n_mt) * a.tile_rows + r;
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
        lv[e] = a.l_part[(size_t)slot * a.tile_rows + r];
        const float4* src = op + (size_t)slot * (a.tile_rows / 32) * (D / 4) * 32;
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

// The softmax's FMA-pipe 2^x as the kernel runs it: packed pairs (the last
// element of an odd count through the scalar form, the same arithmetic).
__global__ void exp2_selftest_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const uint64_t p2 = exp2_fma2(f2_pack(x[i], x[i + 1]));
    y[i] = f2_lo(p2);
    y[i + 1] = f2_hi(p2);
  } else if (i < n) {
    y[i] = exp2_fma(x[i]);
  }
}

// ---------------------------------------------------------------- host side
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
  if (!attn_maps(a, D, &mq, &mkp, &mvp, &mks, &mvs)) return cudaErrorInvalidValue;
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
  exp2_selftest_kernel<<<((n + 1) / 2 + 255) / 256, 256, 0, s>>>(x, y, n);
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

// One launch of the merge kernel: grid.z covers the D / 4 float4 columns in
// groups of 8 warps x kCols.
template <int D, int kCols, int kFixBatch>
cudaError_t launch_fix(cudaLaunchConfig_t cfg, const AttnArgs& a) {
  static_assert((D / 4) % (8 * kCols) == 0, "column groups");
  cfg.gridDim.z = (D / 4) / (8 * kCols);
  return cudaLaunchKernelEx(&cfg, tc_fixup_kernel<D, kCols, kFixBatch>, a);
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
  cfg.gridDim = dim3(a.n_tiles - a.tail0, a.tile_rows / kFixRows, 1);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (a.d == 128) return many ? launch_fix<128, 1, 8>(cfg, a) : launch_fix<128, 2, 4>(cfg, a);
  return many ? launch_fix<64, 1, 8>(cfg, a) : launch_fix<64, 2, 4>(cfg, a);
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s) {
  if (a.M == 0 || a.n_ctas == 0) return cudaSuccess;
  if (a.tile_rows == 128) return launch_attn_tc1(a, s);
  const bool tree = a.key_end != nullptr;
  if (a.d == 128) return tree ? launch_dt<128, true>(a, s) : launch_dt<128, false>(a, s);
  return tree ? launch_dt<64, true>(a, s) : launch_dt<64, false>(a, s);
}

}  // namespace jev
