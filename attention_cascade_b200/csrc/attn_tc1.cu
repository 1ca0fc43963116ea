// attn_tc1.cu — tensor-core shared-prefix attention for sm_100a (tcgen05 + TMEM + TMA),
// one 128-row Q tile per CTA: the kernel the plan picks when 256-row work
// tiles (attn_tc.cu) would not fill one wave of CTAs.
//
// The prefix is shared by every branch ("How to Deploy Visual Jev ...", Step 3;
// "FastJEV ...", §3.2-§3.3), so all branches' queries of one kv group are
// stacked into one M dimension (row m = token m / G, query slot m % G) and the
// prefix K/V of that group streams through shared memory once per 128 stacked
// rows instead of once per branch.  After the prefix, a work tile also runs
// its suffix window: the suffix keys its rows may see (same branch up to the
// row's own token or, in a generation step, the branch's cache up to the
// row's slot; for tree tokens every ancestor node's keys too), masked per row.
//
// Schedule.  A work tile (128 stacked rows of one kv group) has P = n_pre + 1
// units: its 128-key prefix tiles and the suffix window.  n_ctas persistent
// CTAs first take whole tiles for full_waves rounds; the units of the
// remaining tail tiles are spread evenly over tail_ctas of them.  A CTA visits
// its work as segments (runs inside one tile).  A segment that covers its
// whole tile writes the final output; other segments write a normalised fp32
// partial and its log2 normaliser, and tc_fixup_kernel merges the segments of
// each split tail tile.
//
// CTA = 18 warps:
//   warps 0-15  softmax and epilogue: warp w holds rows 32(w % 4) .. +31 (TMEM
//               lanes) and score columns 32(w / 4) .. +31 of each key tile, and
//               output columns (D / 4)(w / 4) .. of O: four threads per row
//   warp 16     TMA producer (Q once per segment; K and V through two rings)
//   warp 17     TMEM allocator and tcgen05.mma issuer (the loop runs warp-wide;
//               an elected lane issues each MMA and commit)
// TMEM (512 columns): score buffers S0 [0,128) and S1 [128,256), O at 256.
// Key tile j's scores go to buffer j % 2.  The MMA warp issues S(j+1) =
// Q K(j+1)^T (SS form) before it waits for the softmax of tile j, then
// O += P(j) V(j) (TS form, P(j) bf16 in TMEM, aliasing S(j)), so the softmax
// of tile j+1 starts as soon as tile j's is done while the tensor core runs
// PV(j) and S(j+2) behind it.  Each thread packs its 32 probabilities into
// the first 16 columns of its own 32 score columns; the PV MMA over keys
// 16k .. 16k+15 reads 8 columns at 32(k / 2) + 8(k % 2).  The four quarters
// of a row exchange their maxima through shared memory each key tile (a
// 128-thread barrier per 32 rows); the softmax runs in the log2 domain with a
// lazy running max (raised only when a row's maximum exceeds it by more than
// 8, so O is rescaled rarely, after PV(j-1) has completed, and P stays
// <= 2^8), its scale-and-subtract and row sums as packed f32x2 operations.
// Once a row has a running max, the exponentials start from it before the
// quarters have exchanged the tile's maxima, and a warp whose rows moved it
// recomputes them (the scores are still in TMEM).
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

constexpr int kBM = 128;          // rows per work tile (TMEM lanes)
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kSoftWarps = 16;
constexpr int kThreads = (kSoftWarps + 2) * 32;
constexpr int kProducerWarp = kSoftWarps;
constexpr int kMmaWarp = kSoftWarps + 1;
constexpr int kQCols = kBN / 4;  // score columns per softmax thread
constexpr float kLazy = 8.0f;    // log2 headroom before the running max moves
// Share of softmax exponentials computed on the FMA pipe (every kPolyEvery-th
// score pair, as one packed f32x2 polynomial; 0 = none).  Measured on B200,
// attention call alone: every 16th pair (one of a thread's 16 per key tile)
// is about 1 us faster than every 8th at the 7B and tree workloads, every
// 4th about 0.5-1 us slower.
#ifndef JEV_POLY_EVERY1
#define JEV_POLY_EVERY1 16
#endif
constexpr int kPolyEvery = JEV_POLY_EVERY1;
static_assert(kBM == 128, "one TMEM lane per row");

template <int D>
struct Cfg {
  static constexpr int kNK = D == 128 ? 3 : 6;  // K stages
  static constexpr int kNV = D == 128 ? 2 : 5;  // V stages
  static constexpr int kQD = D / 4;             // output columns per softmax thread
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kKVBytes = kBN * D * 2;
  static constexpr int kBlk = 128 * 128;  // one 64-column, 128-row swizzled block
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffV = kOffK + kNK * kKVBytes;
  static constexpr int kOffBar = kOffV + kNV * kKVBytes;
  static constexpr int kOffX = kOffBar + 512;              // row-max exchange [tile parity][quarter][row]
  static constexpr int kOffL = kOffX + 2 * 4 * kBM * 4;     // row-sum exchange [quarter][row]
  static constexpr int kOffStg = kOffL + 4 * kBM * 4;       // per-warp output staging
  static constexpr int kStgBytes = 512;                     // 32 rows x kQD bf16 columns, in rounds
  static constexpr int kOffSeg = kOffStg + kSoftWarps * kStgBytes;  // two published segment descriptions
  static constexpr int kSmem = kOffSeg + 128 + 1024;                 // + 1024-byte alignment slack
  static constexpr int kOCol = 256;                                  // first TMEM column of O
  static_assert(2 + 2 * kNK + 2 * kNV + 2 + 2 + 4 <= 60, "barriers below the shared words");
};

struct Bars {
  uint32_t q_full, q_empty, k_full, k_empty, v_full, v_empty, s_full, p_full, pv_done, o_full, drain, probe;  // arrays: +8*i
};

struct Shared {
  uint32_t tmem_base;
  int abort;
};

template <int D, bool TREE>
__global__ void __launch_bounds__(kThreads, 1)
    attn_tc1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kp,
                   const __grid_constant__ CUtensorMap tm_vp, const __grid_constant__ CUtensorMap tm_ks,
                   const __grid_constant__ CUtensorMap tm_vs, const AttnArgs a) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  Shared* sh = reinterpret_cast<Shared*>(smem + C::kOffBar + 480);
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
  B.k_empty = B.k_full + 8 * C::kNK;
  B.v_full = B.k_empty + 8 * C::kNK;
  B.v_empty = B.v_full + 8 * C::kNV;
  B.s_full = B.v_empty + 8 * C::kNV;
  B.p_full = B.s_full + 16;
  B.pv_done = B.p_full + 16;
  B.o_full = B.pv_done + 8;
  B.drain = B.o_full + 8;
  B.probe = B.drain + 8;

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
    for (int b = 0; b < 2; ++b) {
      mbar_init(B.s_full + 8 * b, 1);
      mbar_init(B.p_full + 8 * b, kSoftWarps * 32);
    }
    mbar_init(B.pv_done, 1);
    mbar_init(B.o_full, 1);
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
    // Key tiles are numbered over the CTA's whole run (x); tile x goes to K
    // stage x % kNK and V stage x % kNV.  Inside a segment K runs one tile
    // ahead of V: the MMA warp needs K(x + 1) before it consumes V(x).
    // The whole warp runs this loop (its values stay warp-uniform); one
    // elected lane issues each load.
    // Key-tile counters are 32-bit: a CTA's tiles stay far below 2^32, and the
    // stage and phase arithmetic (division by the 3 K stages) then costs a few
    // instructions in warps that share their sub-partition with four busy
    // softmax warps.
    uint32_t kn = 0, vn = 0;  // K and V tiles whose loads this warp has issued
    int q_armed = 0;           // Q tiles loaded
    int k = 0;
    bool ok = true;
    if (lane == 0) tma_prefetch_desc(&tm_q);
    auto load_tile = [&](bool is_k, uint32_t x, const Segment& sg, uint32_t J, bool pre_only) -> bool {
      const int ns = is_k ? C::kNK : C::kNV;
      const int st = (int)(x % ns);
      const uint32_t full = (is_k ? B.k_full : B.v_full) + 8 * st;
      if (x >= ns && !wait_bar_w((is_k ? B.k_empty : B.v_empty) + 8 * st, (uint32_t)((x / ns - 1) & 1), abort,
                                 a.status, a.wait_cycles))
        return false;
      const int j = (int)(x - J);
      const bool pre = pre_only || j < sg.n_pre;
      const int kb = pre ? (sg.ua + j) * kBN : sg.lo + (j - sg.n_pre) * kBN;
      const CUtensorMap* m = is_k ? (pre ? &tm_kp : &tm_ks) : (pre ? &tm_vp : &tm_vs);
      const uint32_t dst = sbase + (is_k ? C::kOffK : C::kOffV) + st * C::kKVBytes;
      mbar_expect_tx_w(full, C::kKVBytes);
      for (int b = 0; b < D / 64; ++b) tma_load_2d_w(dst + b * C::kBlk, m, sg.g * D + b * 64, kb, full);
      return true;
    };
    // the first segment's leading prefix key tiles need nothing from the pack:
    // their loads start before the wait (the pack lets this kernel launch only
    // once every kernel before it in the stream has completed)
    {
      SegIter it0{0, u_begin, u_end};
      int w0, ua0, ub0;
      bool tl0;
      if (seg_next(a, cta, it0, w0, ua0, ub0, tl0)) {
        const int npre = max(0, min(ub0, a.n_pre) - ua0);
        Segment s0{};
        s0.ua = ua0;
        s0.g = w0 / a.n_mt;
        s0.n_pre = npre;
        const int pk = min(npre, C::kNK), pv = min(npre, C::kNV);
        for (int j = 0; j < pk; ++j) load_tile(true, j, s0, 0, true);
        for (int j = 0; j < pv; ++j) load_tile(false, j, s0, 0, true);
        kn = pk;
        vn = pv;
      }
    }
    pdl_wait();
    uint32_t J = 0;
    SegIter it{0, u_begin, u_end};
    int sw, sua, sub;
    bool stail;
    for (; ok && seg_next(a, cta, it, sw, sua, sub, stail); ++k, ++it.k) {
      // The Q tile goes first: it needs only the tile's group and rows.
      const int qg = sw / a.n_mt, qm0 = (sw - qg * a.n_mt) * kBM;
      if (k > 0 && !wait_bar_w(B.q_empty, (k - 1) & 1, abort, a.status, a.wait_cycles)) ok = false;
      if (ok) {
        mbar_expect_tx_w(B.q_full, C::kQBytes);
        for (int b = 0; b < D / 64; ++b) tma_load_3d_w(sbase + b * C::kBlk, &tm_q, b * 64, qm0, qg, B.q_full);
        ++q_armed;
      }
      // The description (for the suffix unit, its key window: a warp-wide read
      // of token info) is published with q_full's second arrival.
      const Segment sg = make_segment<kBM>(a, cta, sw, sua, sub, stail, lane);
      if (ok) {
        if (lane == 0) {
          seg_sm[k & 1] = sg;
          mbar_arrive(B.q_full);
        }
        __syncwarp();
        for (int j = 0; ok && j < sg.n; ++j) {
          while (ok && kn <= J + j) {
            ok = load_tile(true, kn, sg, J, false);
            if (ok) ++kn;
          }
          while (ok && j >= 1 && vn <= J + j - 1) {
            ok = load_tile(false, vn, sg, J, false);
            if (ok) ++vn;
          }
        }
        while (ok && vn <= J + sg.n - 1) {
          ok = load_tile(false, vn, sg, J, false);
          if (ok) ++vn;
        }
      }
      J += sg.n;
    }
    if (lane == 0) {
      // Drain: the last phase of every stage this warp armed, and of the Q
      // buffer, has completed (its loads have landed) before the CTA may
      // exit.  On the normal path these phases completed long ago.  (A load
      // whose empty-wait gave up was not issued and is not counted: the loop
      // above advances kn / vn only past issued loads.)
      for (int st = 0; st < C::kNK; ++st) {
        const uint32_t uses = kn > (uint32_t)st ? (kn - st + C::kNK - 1) / C::kNK : 0;
        if (uses > 0) drain_bar(B.k_full + 8 * st, (uint32_t)((uses - 1) & 1), a.status);
      }
      for (int st = 0; st < C::kNV; ++st) {
        const uint32_t uses = vn > (uint32_t)st ? (vn - st + C::kNV - 1) / C::kNV : 0;
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
    // S(x) = Q K(x)^T into score buffer x % 2; its commits release the buffer
    // to the softmax and the K stage to the producer
    auto issue_s = [&](uint32_t x) {
      const int st = (int)(x % C::kNK), buf = (int)(x & 1);
      const uint64_t ka = dk0 + (uint32_t)((st * C::kKVBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        constexpr int kBlk4 = C::kBlk >> 4;
        const uint32_t off = (uint32_t)((kk >> 2) * kBlk4 + (kk & 3) * 2);
        mma_ss_w(tmem + buf * kBN, dq0 + off, ka + off, id_qk, kk > 0);
      }
      mma_commit_w(B.s_full + 8 * buf);
      mma_commit_w(B.k_empty + 8 * st);
    };
    // O (+)= P(x) V(x), P read from TMEM where the softmax threads packed it
    auto issue_pv = [&](uint32_t x, bool acc) {
      const int st = (int)(x % C::kNV), buf = (int)(x & 1);
      const uint64_t va = dv0 + (uint32_t)((st * C::kKVBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        mma_ts_w(tmem + C::kOCol, tmem + buf * kBN + (kk >> 1) * kQCols + (kk & 1) * 8,
                 va + (uint32_t)(kk * 16 * 128 / 16), id_pv, (acc || kk > 0) ? 1u : 0u);
      mma_commit_w(B.pv_done);
      mma_commit_w(B.v_empty + 8 * st);
    };
    uint32_t J = 0;
    int k = 0;
    bool ok = true;
    pdl_wait();
    SegIter it{0, u_begin, u_end};
    int sw, sua, sub;
    bool stail;
    for (; ok && seg_next(a, cta, it, sw, sua, sub, stail); ++k, ++it.k) {
      ok = wait_bar_w(B.q_full, k & 1, abort, a.status, a.wait_cycles);
      const Segment sg = seg_sm[k & 1];
      const int n = sg.n;  // >= 1
      if (ok) {
        ok = wait_bar_w(B.k_full + 8 * (int)(J % C::kNK), (uint32_t)((J / C::kNK) & 1), abort, a.status,
                        a.wait_cycles);
        fence_after_sync();
        if (ok) issue_s(J);
        // failure-detection probe (off unless a test sets it): a wait that
        // nothing completes, with this segment's first MMAs in flight
        if (ok && k == 0 && a.wait_probe)
          ok = __shfl_sync(0xffffffffu, probe_wait(B.probe, abort, a.status, a.wait_cycles), 0);
      }
      for (int j = 0; ok && j < n; ++j) {
        const uint32_t JJ = J + j, JJ1 = JJ + 1;
        // the next tile's scores first: the tensor core computes them while
        // the softmax threads work on this tile
        if (j + 1 < n) {
          if (!wait_bar_w(B.k_full + 8 * (int)(JJ1 % C::kNK), (uint32_t)((JJ1 / C::kNK) & 1), abort, a.status,
                          a.wait_cycles)) {
            ok = false;
            break;
          }
          fence_after_sync();
          issue_s(JJ1);
        }
        if (!wait_bar_w(B.v_full + 8 * (int)(JJ % C::kNV), (uint32_t)((JJ / C::kNV) & 1), abort, a.status,
                        a.wait_cycles)) {
          ok = false;
          break;
        }
        if (!wait_bar_w(B.p_full + 8 * (int)(JJ & 1), (uint32_t)((JJ >> 1) & 1), abort, a.status, a.wait_cycles)) {
          ok = false;
          break;
        }
        fence_after_sync();
        issue_pv(JJ, j > 0);
        if (j == n - 1) mma_commit_w(B.o_full);
        // q_empty releases the Q buffer and lets the producer publish the next
        // segment.  It is committed once the segment's last S MMA is issued
        // and after a p_full wait of the segment, i.e. after all 512 softmax
        // threads have passed their q_full wait for it: were q_full to
        // complete two phases ahead of a softmax thread still in the previous
        // epilogue, that thread's parity wait would alias the later phase and
        // never return.
        if (j == max(0, n - 2)) mma_commit_w(B.q_empty);
      }
      J += n;
    }
    // every MMA of this CTA has completed before TMEM is released, on the
    // timeout path too (the wait ignores the abort flag); the commit comes
    // from the lane that issued the MMAs
    mma_commit_w(B.drain);
    drain_bar(B.drain, 0, a.status);
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    constexpr int kQD = C::kQD;  // output columns per thread
    const int q = warp & 3, cq = warp >> 2, r = q * 32 + lane;
    constexpr int kGroupBar = 1;      // named barrier of the 512 softmax threads
    const int row_bar = 2 + q;        // named barrier of the four warps that share rows 32q .. 32q+31
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int c_base = cq * kQCols;  // key column of this thread's first score
    const uint32_t s_addr0 = tmem + c_base + lane_off;  // + buffer * kBN: this quarter's scores, then its packed P
    const uint32_t o_addr = tmem + C::kOCol + cq * kQD + lane_off;
    const float sl2 = a.scale_log2;
    uint32_t J = 0;
    int k = 0;
    bool ok = true;
    pdl_wait();
    // every CTA has passed its wait: the merge kernel may launch now
    if (threadIdx.x == 0) pdl_trigger();
    SegIter it{0, u_begin, u_end};
    int sw, sua, sub;
    bool stail;
    for (; ok && seg_next(a, cta, it, sw, sua, sub, stail); ++k, ++it.k) {
      // The 512 threads agree on the q_full wait before any reads the segment
      // description: a thread whose wait gave up must not read a description
      // the producer may not have published, and the row groups must run the
      // same number of key tiles (the same named barriers).  This barrier also
      // orders the previous epilogue's reads of the row-sum exchange before
      // the next epilogue's writes.
      ok = named_sync_and(kGroupBar, kSoftWarps * 32, wait_bar(B.q_full, k & 1, abort, a.status, a.wait_cycles));
      if (!ok) break;
      const Segment sg = seg_sm[k & 1];
      const int m = sg.m0 + r;
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
      // that every thread of the row group meets the same named barriers, and
      // the threads agree on the outcome at the epilogue's reducing barrier.
      for (int j = 0; j < sg.n; ++j) {
        const uint32_t JJ = J + j;
        const int buf = (int)(JJ & 1);
        if (!wait_bar(B.s_full + 8 * buf, (uint32_t)((JJ >> 1) & 1), abort, a.status, a.wait_cycles)) ok = false;
        fence_after_sync();
        // this quarter's 32 raw scores with the masks applied; P is later
        // packed in place into xs[0..15]
        uint32_t xs[kQCols];
        auto load_scores = [&]() {
          tmem_ld32(s_addr0 + buf * kBN, xs);
          constexpr uint32_t kNegInf = 0xff800000u;
          if (j < sg.n_pre) {
            const int lim = a.Lp - (sg.ua + j) * kBN - c_base;  // keys past the prefix are padding
            if (lim < kQCols) {
#pragma unroll
              for (int c = 0; c < kQCols; ++c)
                if (c >= lim) xs[c] = kNegInf;
            }
          } else {
            // suffix window
            const int kb = sg.lo + (j - sg.n_pre) * kBN + c_base;
            if (!TREE) {
              // flat row: the keys start .. last of its own branch
              const int c_lo = start - kb, c_hi = last - kb;
              // the mask is skipped when every row of the warp sees all 32 of its keys in this tile
              const bool whole = __all_sync(0xffffffffu, c_lo <= 0 && c_hi >= kQCols - 1);
              if (!whole) {
#pragma unroll
                for (int c = 0; c < kQCols; ++c)
                  if (!(c >= c_lo && c <= c_hi)) xs[c] = kNegInf;
              }
            } else {
              // tree row t: key k is on its root path when k <= t and t lies in the
              // packed tokens of k's node's subtree.  The warp's rows share the
              // quarter's 32 keys: lane l reads the subtree end of key l once, and
              // the mask is skipped when every key is at or before the warp's
              // first row and every subtree holds its last row.
              const int e_l = kb + lane < a.key_rows ? __ldg(a.key_end + kb + lane) : -1;
              const bool whole = kb + kQCols - 1 <= w_lo && warp_min_i(e_l) > w_hi;
              if (!whole) {
#pragma unroll
                for (int c = 0; c < kQCols; ++c) {
                  const int e = __shfl_sync(0xffffffffu, e_l, c);
                  if (!(kb + c <= t && t < e)) xs[c] = kNegInf;
                }
              }
            }
          }
        };
        // p = 2^(s * scale * log2e - base): one exponential per score; the
        // scale-and-subtract and the row sum run as packed f32x2 operations
        // (one instruction per pair of scores).  Packs P into xs[0..15] and
        // returns this quarter's share of the row sum.
        auto exps = [&](float base) -> float {
          const uint64_t sc2 = f2_pack(sl2, sl2), nb2 = f2_pack(-base, -base);
          uint64_t ps2[4];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) ps2[q4] = 0;
#pragma unroll
          for (int kk = 0; kk < kQCols / 2; ++kk) {
            const uint64_t x2 = f2_fma(((uint64_t)xs[2 * kk + 1] << 32) | xs[2 * kk], sc2, nb2);
            const bool fma_pipe = kPolyEvery > 0 && (kk % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1;
            const uint64_t p2 = fma_pipe ? exp2_fma2(x2) : f2_pack(ex2(f2_lo(x2)), ex2(f2_hi(x2)));
            ps2[kk & 3] = f2_add(ps2[kk & 3], p2);
            xs[kk] = pack_bf16(f2_lo(p2), f2_hi(p2));
          }
          const uint64_t s01 = f2_add(ps2[0], ps2[1]), s23 = f2_add(ps2[2], ps2[3]);
          const uint64_t s03 = f2_add(s01, s23);
          return f2_lo(s03) + f2_hi(s03);
        };
        load_scores();
        // this quarter's maximum with three-input max instructions (8 independent chains)
        float pm[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) pm[q8] = __uint_as_float(xs[q8]);
#pragma unroll
        for (int c = 8; c < kQCols; c += 2)
          pm[(c >> 1) & 7] = fmax3(pm[(c >> 1) & 7], __uint_as_float(xs[c]), __uint_as_float(xs[c + 1]));
        const float q_max = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
        // the four quarters of the row agree on the maximum (double-buffered by
        // tile parity); the warps of a row group all hold the same rows, so
        // they take the same branch below and meet the barrier once each
        float* xm = xmax + buf * 4 * kBM;
        xm[cq * kBM + r] = q_max;
        auto row_max = [&]() { return fmaxf(fmax3(xm[r], xm[kBM + r], xm[2 * kBM + r]), xm[3 * kBM + r]) * sl2; };
        float m_new, rs;
        if (__all_sync(0xffffffffu, m_run != -CUDART_INF_F)) {
          // Most tiles leave the lazy running max where it is: the
          // exponentials start from it before the quarters have agreed on the
          // tile's maximum, and a warp whose rows moved it recomputes them
          // (its scores are still in TMEM: P is stored below).
          rs = exps(m_run);
          named_sync(row_bar, 128);
          const float mx = row_max();
          m_new = mx > m_run + kLazy ? mx : m_run;
          if (__any_sync(0xffffffffu, m_new != m_run)) {
            load_scores();
            rs = exps(m_new);
          }
        } else {
          named_sync(row_bar, 128);
          const float mx = row_max();
          m_new = m_run;
          if (mx > m_run + kLazy || (m_run == -CUDART_INF_F && mx > -CUDART_INF_F)) m_new = mx;
          rs = exps(m_new == -CUDART_INF_F ? 0.f : m_new);
        }
        const float alpha = ex2(m_run - (m_new == -CUDART_INF_F ? 0.f : m_new));
        tmem_st16(s_addr0 + buf * kBN, *reinterpret_cast<const uint32_t(*)[16]>(&xs[0]));
        l_run = l_run * alpha + rs;
        if (j > 0 && __any_sync(0xffffffffu, m_new != m_run)) {
          // O holds the sum through tile JJ - 1 once that PV has completed
          // (S(JJ) completing shows only PV(JJ - 2) done)
          if (!wait_bar(B.pv_done, (uint32_t)((JJ - 1) & 1), abort, a.status, a.wait_cycles)) ok = false;
          fence_after_sync();
          if constexpr (kQD == 32) {
            uint32_t uu[32];
            tmem_ld32(o_addr, uu);
#pragma unroll
            for (int kk = 0; kk < 32; ++kk) uu[kk] = __float_as_uint(__uint_as_float(uu[kk]) * alpha);
            tmem_st32(o_addr, uu);
          } else {
            uint32_t uu[16];
            tmem_ld16(o_addr, uu);
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) uu[kk] = __float_as_uint(__uint_as_float(uu[kk]) * alpha);
            tmem_st16(o_addr, uu);
          }
        }
        m_run = m_new;
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(B.p_full + 8 * buf);
      }
      if (ok) ok = wait_bar(B.o_full, (uint32_t)(k & 1), abort, a.status, a.wait_cycles);
      fence_after_sync();
      // the row's normaliser is the sum of the four quarters' partial sums
      xsum[cq * kBM + r] = l_run;
      ok = named_sync_and(kGroupBar, kSoftWarps * 32, ok);
      const float l_row = (xsum[r] + xsum[kBM + r]) + (xsum[2 * kBM + r] + xsum[3 * kBM + r]);
      const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
      const bool write = ok && valid && t >= 0;
      const int tt = valid ? m / a.G : 0;
      const int h = valid ? min(max(a.hinv[sg.g * a.G + (m - tt * a.G)], 0), a.Hq - 1) : 0;
      // this thread's kQD output columns of its row
      uint32_t uu[kQD];
      if constexpr (kQD == 32)
        tmem_ld32(o_addr, uu);
      else
        tmem_ld16(o_addr, uu);
      if (sg.complete) {
        // bf16 output rows (t, h) lie D*2 bytes apart or more; the warp stages
        // kRows of its rows' kRowB-byte pieces at a time in shared memory so
        // that each global store writes whole 16-byte chunks of kRows rows
        constexpr int kRowB = kQD * 2, kChunks = kRowB / 16, kRows = C::kStgBytes / kRowB;
        const unsigned long long dst_row =
            write ? reinterpret_cast<unsigned long long>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                                         ((size_t)tt * a.Hq + h) * D + cq * kQD)
                  : 0ull;
        uint8_t* stg = smem + C::kOffStg + warp * C::kStgBytes;
        uint32_t* pk = uu;  // packed in place: entry kk reads entries 2kk, 2kk+1 >= kk
#pragma unroll
        for (int kk = 0; kk < kQD / 2; ++kk)
          pk[kk] = pack_bf16(__uint_as_float(uu[2 * kk]) * inv, __uint_as_float(uu[2 * kk + 1]) * inv);
        const int rd_row = lane / kChunks, rd_c = lane % kChunks;  // the 16-byte chunk this lane stores
#pragma unroll
        for (int rq = 0; rq < 32 / kRows; ++rq) {
          if (lane / kRows == rq) {
            const int rr = lane % kRows;
#pragma unroll
            for (int e = 0; e < kChunks; ++e)
              *reinterpret_cast<uint4*>(stg + rr * kRowB + ((e ^ (rr & (kChunks - 1))) * 16)) =
                  make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
          }
          __syncwarp();
          const uint4 v = *reinterpret_cast<const uint4*>(stg + rd_row * kRowB + ((rd_c ^ (rd_row & (kChunks - 1))) * 16));
          const unsigned long long d = __shfl_sync(0xffffffffu, dst_row, rq * kRows + rd_row);
          if (d) reinterpret_cast<uint4*>(d)[rd_c] = v;
          __syncwarp();
        }
      } else if (write) {
        // fp32 partial rows, stored [slot][row / 32][column / 4][row % 32] as
        // float4 so that a warp's 32 rows fill 512 contiguous bytes per store
        float4* dst = reinterpret_cast<float4*>(a.o_part) + ((size_t)(sg.slot * (kBM / 32) + q) * (D / 4)) * 32 + lane;
#pragma unroll
        for (int v = 0; v < kQD / 4; ++v)
          dst[(size_t)(cq * kQD / 4 + v) * 32] =
              make_float4(__uint_as_float(uu[4 * v]) * inv, __uint_as_float(uu[4 * v + 1]) * inv,
                          __uint_as_float(uu[4 * v + 2]) * inv, __uint_as_float(uu[4 * v + 3]) * inv);
      }
      const size_t prow = (size_t)sg.slot * kBM + r;  // partial row of this thread
      if (cq == 0) {
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

template <int D, bool TREE>
cudaError_t launch_dt1(const AttnArgs& a, cudaStream_t s) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc1_kernel<D, TREE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  return cudaLaunchKernelEx(&cfg, attn_tc1_kernel<D, TREE>, mq, mkp, mvp, mks, mvs, a);
}

}  // namespace

cudaError_t launch_attn_tc1(const AttnArgs& a, cudaStream_t s) {
  if (a.M == 0 || a.n_ctas == 0) return cudaSuccess;
  const bool tree = a.key_end != nullptr;
  if (a.d == 128) return tree ? launch_dt1<128, true>(a, s) : launch_dt1<128, false>(a, s);
  return tree ? launch_dt1<64, true>(a, s) : launch_dt1<64, false>(a, s);
}

}  // namespace jev
