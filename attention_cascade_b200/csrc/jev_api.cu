// jev_api.cu — the C ABI declared in include/jev.h: argument checks,
// workspace layout, split planning, kernel launches, kernel timing and the
// host-side candidate-prefix trie.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "kernels.h"

namespace jev {
namespace {

thread_local char g_err[512] = "";

jev_status fail(jev_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

// ---------------------------------------------------------------- timing
struct Rec {
  int name;
  cudaEvent_t a, b;
};
std::mutex g_mu;
std::atomic<bool> g_prof{false};
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;
std::vector<std::string> g_names;
std::atomic<long long> g_launches{0};
// bound of the tensor-core kernels' mbarrier waits, in clock cycles (about a
// second at the B200's clock); jev_debug_set_wait_limit changes it
constexpr long long kDefaultWaitCycles = 1LL << 31;
std::atomic<long long> g_wait_cycles{kDefaultWaitCycles};
std::atomic<int> g_wait_probe{0};
std::atomic<int> g_tile_rows{0};  // 0: rows per tensor-core work tile as the plan chooses, else 128 or 256

int name_id(const char* n) {
  for (size_t i = 0; i < g_names.size(); ++i)
    if (g_names[i] == n) return (int)i;
  g_names.emplace_back(n);
  return (int)g_names.size() - 1;
}
cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e;
  cudaEventCreate(&e);
  return e;
}

// Record a timing event on s; inside a stream capture the record becomes an
// external event node that every replay of the graph re-records.
bool record(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const unsigned flags = cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
  if (cudaEventRecordWithFlags(ev, s, flags) != cudaSuccess) {
    cudaGetLastError();  // timing is best effort; never let it fail a launch
    return false;
  }
  return true;
}

// Launch one kernel through `fn`, bracketed by timing events when enabled.
template <class F>
jev_status run(const char* name, cudaStream_t s, F&& fn) {
  Rec r{-1, nullptr, nullptr};
  bool on = g_prof.load();
  if (on) {
    std::lock_guard<std::mutex> lk(g_mu);
    r.name = name_id(name);
    r.a = take_event();
    r.b = take_event();
  }
  if (on) on = record(r.a, s);
  cudaError_t e = fn();
  if (on && e == cudaSuccess) on = record(r.b, s);
  if (r.a) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (on) {
      g_recs.push_back(r);
    } else {
      g_pool.push_back(r.a);
      g_pool.push_back(r.b);
    }
  }
  g_launches++;
  if (e != cudaSuccess) return fail(JEV_ERR_CUDA, "%s launch failed: %s", name, cudaGetErrorString(e));
  return JEV_OK;
}

// ---------------------------------------------------------------- checks
bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }
size_t esize(jev_dtype dt) { return dt == JEV_BF16 ? 2 : 4; }

int num_sms() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
  }
  return sms;
}

// The tcgen05 / TMA kernels run on an sm_100a device with the tensor-map encoder available.
bool tcgen05_device() { return attn_tc_supported(128); }

bool use_tc(const jev_attn_desc* d) {
  static int forced = -1;
  if (forced < 0) {
    const char* e = getenv("JEV_ATTN_KERNEL");
    forced = (e && !strcmp(e, "simt")) ? 1 : 0;
  }
  return !forced && d->dtype == JEV_BF16 && attn_tc_supported(d->d);
}

// Work plan.  Tensor-core kernel: work tiles of tile_rows stacked rows of one
// kv group, each with P = ceil(Lp/128) + 1 units (prefix key tiles + the
// suffix window).  256-row tiles run on the two-Q-tile kernel, which is the
// faster per unit; 128-row tiles on the one-Q-tile kernel, chosen when
// 256-row tiles would leave little work per CTA (twice the tiles, so fewer of
// them are split and merged; the rule is at the choice below).  n_ctas persistent CTAs first take full_waves rounds of whole
// tiles; the remaining tail tiles' units are spread evenly over tail_ctas of
// them, so a tail tile may be split across CTAs and merged afterwards.
// num_splits: 1 -> no tile split (one CTA per tile up to one per SM),
// s > 1 -> every tile spread over about s CTAs, 0 -> the cheapest schedule
// under a cost model.  CUDA-core kernel: S prefix splits of split_len keys
// (a multiple of 128) and a merge.
struct Plan {
  int S, split_len, M, G;
  bool tc, split;
  int tile_rows, n_mt, n_tiles, n_pre, P, n_ctas, full_waves, tail0, tail_ctas;
  long long U;
};

// Estimated time (microseconds) of the tensor-core schedule: the busiest
// CTA's units and segments plus the merge of split tiles.  Calibrated on
// B200 at d = 128: a unit of 256 rows x 128 keys costs about 2.5 us (one of
// 128 rows, on the one-Q-tile kernel, about 0.6 of that), the
// first segment of a CTA about 8 us of pipeline fill and drain, each later
// one about 3 us, a segment left partial about 2 us more (fp32 output), and
// the merge about 5 us plus 0.7 us per eight segments of one tile.
double tc_schedule_us(int P, int d, int full_waves, long long U, int tail_ctas, int tile_rows) {
  const double unit_us = (tile_rows == 256 ? 1.0 : 0.6) * 4.0 * 256 * 128 * d / 6.8e12 * 1e6;
  const double first_us = 8.0, seg_us = 3.0, part_us = 2.0;
  double worst = 0.0;
  bool split = false;
  long long max_tile_segs = 1;
  for (int c = 0; c < std::max(1, tail_ctas); ++c) {
    long long units = (long long)full_waves * P, segs = full_waves;
    bool part = false;
    if (U > 0 && c < tail_ctas) {
      const long long u0 = c * U / tail_ctas, u1 = (c + 1) * U / tail_ctas;
      if (u1 > u0) {
        units += u1 - u0;
        segs += (u1 - 1) / P - u0 / P + 1;
        if (u0 % P || u1 % P) part = split = true;
      }
    }
    if (segs == 0) continue;
    worst = std::max(worst, first_us + (segs - 1) * seg_us + units * unit_us + (part ? part_us : 0.0));
  }
  if (split) {
    max_tile_segs = (P * (long long)tail_ctas + U - 1) / U + 1;
    worst += 5.0 + 0.7 * (double)((max_tile_segs + 7) / 8);
  }
  return worst;
}

// The tensor-core schedule for work tiles of `rows` stacked rows: fills p's
// tile fields and returns the cost model's estimate (microseconds).
double tc_plan(Plan& p, const jev_attn_desc* d, int rows, int sms) {
  const int ktiles = (d->Lp + 127) / 128;
  p.tile_rows = rows;
  p.n_mt = (p.M + rows - 1) / rows;
  p.n_tiles = p.n_mt * d->Hkv;
  p.n_pre = ktiles;
  p.P = ktiles + 1;
  const int s = d->num_splits;
  // whole tiles only: full_waves rounds over min(n_tiles, sms) CTAs, the
  // rest one tile to each of the first tail_ctas CTAs
  auto no_split = [&] {
    p.n_ctas = std::max(1, std::min(p.n_tiles, sms));
    p.full_waves = p.n_tiles / p.n_ctas;
    p.tail0 = p.full_waves * p.n_ctas;
    p.tail_ctas = std::max(1, p.n_tiles - p.tail0);
    p.U = (long long)(p.n_tiles - p.tail0) * p.P;
  };
  double best = 0.0;
  if (s == 1 || p.n_tiles == 0) {
    no_split();
    best = tc_schedule_us(p.P, d->d, p.full_waves, p.U, p.tail_ctas, rows);
  } else if (s > 1) {
    const long long U = (long long)p.n_tiles * p.P;
    p.full_waves = 0;
    p.tail0 = 0;
    p.U = U;
    p.n_ctas = p.tail_ctas = (int)std::max(1LL, std::min((long long)p.n_tiles * s, U));
    best = tc_schedule_us(p.P, d->d, 0, U, p.tail_ctas, rows);
  } else {
    no_split();
    best = tc_schedule_us(p.P, d->d, p.full_waves, p.U, p.tail_ctas, rows);
    // Spread the tail (every tile when there are fewer tiles than SMs)
    // over more CTAs, up to one per SM; keep the cheapest estimate.
    const int fw = p.n_tiles >= sms ? p.n_tiles / sms : 0;
    const int r = p.n_tiles - fw * sms;
    const long long U = (long long)r * p.P;
    // a tile spread over many CTAs costs a long merge; keep it within 64 segments
    const long long t_max = std::min<long long>({(long long)sms, U, (long long)std::max(1, r) * 64});
    for (long long t = std::max(1, r); r > 0 && t <= t_max; ++t) {
      const double e = tc_schedule_us(p.P, d->d, fw, U, (int)t, rows);
      if (e < best * 0.98) {
        best = e;
        p.full_waves = fw;
        p.tail0 = fw * sms;
        p.U = U;
        p.tail_ctas = (int)t;
        p.n_ctas = fw > 0 ? sms : (int)t;
      }
    }
  }
  p.split = false;
  for (int c = 1; c < p.tail_ctas && p.U > 0 && !p.split; ++c)
    if (((long long)c * p.U / p.tail_ctas) % p.P != 0) p.split = true;
  return best;
}

// kernel: -1 as the device chooses, 0 CUDA-core, 1 tensor-core; sms <= 0: the device's count
Plan compute_plan(const jev_attn_desc* d, int T, int kernel, int sms_hint) {
  Plan p{};
  p.G = d->Hq / d->Hkv;
  p.M = T * p.G;
  const int ktiles = (d->Lp + 127) / 128;
  p.tc = kernel < 0 ? use_tc(d) : kernel == 1;
  if (p.tc) {
    const int sms = std::max(1, sms_hint > 0 ? sms_hint : num_sms());
    // 128-row tiles (the one-Q-tile kernel) when 256-row tiles would not fill
    // a wave of CTAs and their units, spread over the CTAs, come to fewer than
    // 20 a CTA: there the per-segment costs and the merge weigh most, and the
    // finer tiles save them; with more work per CTA the two-Q-tile kernel's
    // lower cost per row wins.  Timed on B200 with both forced (attention
    // call, 28 / 4 heads, d = 128; 256-row tiles x units per tile / SMs):
    // 128-row tiles win at 8.3-11.5 units a CTA (by 2-22%), tie at 21.4, and
    // lose at 59.7 (Lp 8192, 136 tiles) and whenever there is a whole wave.
    const int forced_rows = g_tile_rows.load();
    const long long tiles256 = (long long)((p.M + 255) / 256) * d->Hkv;
    const long long units256 = tiles256 * (ktiles + 1);
    tc_plan(p, d, forced_rows ? forced_rows : (tiles256 < sms && units256 < 20LL * sms ? 128 : 256), sms);
    p.S = 1;
    p.split_len = std::max(1, ktiles) * 128;
    return p;
  }
  // CUDA-core kernel: splits of whole 32-key tiles (the kernel's tile)
  const int kt32 = (d->Lp + 31) / 32;
  int S = d->num_splits;
  if (S <= 0) {
    const long ctas = (long)((p.M + 15) / 16) * d->Hkv;
    const long target = 4L * num_sms();
    S = ctas > 0 ? (int)((target + ctas - 1) / ctas) : 1;
    // keep at least 2 key tiles per split so partial traffic stays small
    S = std::min(S, std::max(1, kt32 / 2));
  }
  S = std::max(1, std::min(std::min(S, kMaxSplits), std::max(1, kt32)));
  p.split_len = kt32 > 0 ? ((kt32 + S - 1) / S) * 32 : 32;
  p.S = d->Lp > 0 ? (d->Lp + p.split_len - 1) / p.split_len : 1;
  return p;
}

// Plans are cached by the fields they depend on: the tensor-core schedule's
// cost-model search takes tens to hundreds of microseconds of host time, and
// every call (and every workspace query) needs the plan.
Plan plan_of(const jev_attn_desc* d, int T, int kernel = -1, int sms_hint = 0) {
  struct Key {
    int T, Lp, Hq, Hkv, d, dtype, num_splits, kernel, sms, rows;
    bool operator==(const Key& o) const {
      return T == o.T && Lp == o.Lp && Hq == o.Hq && Hkv == o.Hkv && d == o.d && dtype == o.dtype &&
             num_splits == o.num_splits && kernel == o.kernel && sms == o.sms && rows == o.rows;
    }
  };
  struct Hash {
    size_t operator()(const Key& k) const {
      size_t h = 1469598103934665603ull;
      for (int v : {k.T, k.Lp, k.Hq, k.Hkv, k.d, k.dtype, k.num_splits, k.kernel, k.sms, k.rows})
        h = (h ^ (size_t)(uint32_t)v) * 1099511628211ull;
      return h;
    }
  };
  static std::mutex mu;
  static std::unordered_map<Key, Plan, Hash> cache;
  const int kern = kernel < 0 ? (use_tc(d) ? 1 : 0) : kernel;
  const int sms = sms_hint > 0 ? sms_hint : num_sms();
  const Key key{T, d->Lp, d->Hq, d->Hkv, d->d, (int)d->dtype, d->num_splits, kern, sms, g_tile_rows.load()};
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const Plan p = compute_plan(d, T, kern, sms);
  std::lock_guard<std::mutex> lk(mu);
  if (cache.size() > 4096) cache.clear();
  cache.emplace(key, p);
  return p;
}

struct Layout {
  size_t hinv, info, qrot, krot, opart, lpart, kend, total;
};
// cache: a generation step writes its rotated keys into the caller's cache,
// so the workspace holds no rotated-key buffer
Layout layout_of(const jev_attn_desc* d, int T, const Plan& p, int n_nodes, bool cache = false) {
  Layout L;
  const size_t s = esize(d->dtype);
  size_t off = kStatusBytes;
  L.hinv = off; off += up256((size_t)d->Hq * 4);
  L.info = off; off += up256((size_t)T * sizeof(TokInfo));
  L.qrot = off; off += up256((size_t)p.M * d->Hkv * d->d * s);
  L.krot = off;
  if (!cache) off += up256((size_t)T * d->Hkv * d->d * s);
  L.opart = off;
  L.lpart = off;
  if (p.tc && p.split) {
    const size_t rows = (size_t)2 * p.n_ctas * p.tile_rows;  // two partial segments per CTA at most
    L.opart = off; off += up256(rows * d->d * 4);
    L.lpart = off; off += up256(rows * 4);
  } else if (!p.tc && p.S > 1) {
    L.opart = off; off += up256((size_t)p.S * d->Hkv * p.M * d->d * 4);
    L.lpart = off; off += up256((size_t)p.S * d->Hkv * p.M * 4);
  }
  L.kend = off;
  if (n_nodes > 0) {
    L.kend = off; off += up256((size_t)T * 4);
  }
  L.total = off;
  return L;
}

jev_status check_desc(const jev_attn_desc* d) {
  if (!d) return fail(JEV_ERR_INVALID_ARG, "desc is NULL");
  if (d->B < 0 || d->Lp < 0 || d->T_total < 0) return fail(JEV_ERR_INVALID_ARG, "negative B, Lp or T_total");
  if (d->Hq <= 0 || d->Hkv <= 0 || d->Hq % d->Hkv) return fail(JEV_ERR_INVALID_ARG, "Hq must be a positive multiple of Hkv");
  if (d->Hq > 256) return fail(JEV_ERR_UNSUPPORTED, "Hq > 256");
  if (d->d != 64 && d->d != 128) return fail(JEV_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d->d);
  if (d->dtype != JEV_BF16 && d->dtype != JEV_F32) return fail(JEV_ERR_UNSUPPORTED, "dtype");
  if (!(d->rope_theta > 0.f)) return fail(JEV_ERR_INVALID_ARG, "rope_theta must be > 0");
  if (d->softmax_scale < 0.f) return fail(JEV_ERR_INVALID_ARG, "softmax_scale must be >= 0");
  if (d->pos_mode != 0 && d->pos_mode != 1) return fail(JEV_ERR_INVALID_ARG, "pos_mode must be 0 or 1");
  if ((long long)d->T_total * (d->Hq / d->Hkv) > (1LL << 30)) return fail(JEV_ERR_UNSUPPORTED, "too many rows");
  return JEV_OK;
}

float scale_log2_of(const jev_attn_desc* d) {
  const double sc = d->softmax_scale > 0.f ? (double)d->softmax_scale : 1.0 / std::sqrt((double)d->d);
  return (float)(sc * 1.4426950408889634);
}

// Per-branch suffix caches of a generation step (jev_suffix_cache_attn).
struct CacheArgs {
  void* k_cache;
  void* v_cache;
  int rows;
  const int32_t* off;
  const int32_t* len;
};

// Shared tail of the flat, tree and cache entry points.
jev_status attention_core(const jev_attn_desc* d, int T, const Plan& p, const Layout& L, char* ws,
                          const void* q, const void* k_pre, const void* v_pre, const void* k_suf,
                          const void* v_suf, const int32_t* offs, int n_segs, const int32_t* pos0,
                          const int32_t* head_map, bool tree, const int32_t* tree_parent, void* out, float* lse,
                          cudaStream_t s, const CacheArgs* cache = nullptr) {
  int32_t* status = reinterpret_cast<int32_t*>(ws);
  jev_status st = JEV_OK;
  RopePackArgs r{};
  r.q = q; r.k = k_suf;
  r.q_rot = ws + L.qrot;
  r.k_rot = cache ? cache->k_cache : ws + L.krot;
  r.info = reinterpret_cast<TokInfo*>(ws + L.info);
  r.hinv = reinterpret_cast<int32_t*>(ws + L.hinv);
  r.status = status;
  r.offs = offs; r.pos0 = pos0; r.head_map = head_map;
  r.parent = tree ? tree_parent : nullptr;
  r.key_end = tree ? reinterpret_cast<int32_t*>(ws + L.kend) : nullptr;
  if (cache) {
    r.cache_off = cache->off;
    r.cache_len = cache->len;
    r.v = v_suf;
    r.v_cache = cache->v_cache;
  }
  r.key_rows = cache ? cache->rows : T;
  r.n_segs = n_segs; r.T = T; r.Hq = d->Hq; r.Hkv = d->Hkv; r.d = d->d;
  r.pos_offset = d->pos_offset >= 0 ? d->pos_offset : d->Lp;
  r.pos_seq = d->pos_mode == 1 ? 1 : 0;
  r.theta = (double)d->rope_theta;
  for (int i = 0; i < d->d / 2; ++i) r.inv_freq[i] = std::pow(r.theta, -2.0 * i / d->d);
  st = run("rope_pack", s, [&] { return launch_rope_pack(r, d->dtype, s); });
  if (st) return st;

  AttnArgs a{};
  a.q_rot = r.q_rot; a.k_pre = k_pre; a.v_pre = v_pre; a.k_rot = r.k_rot;
  a.v_suf = cache ? cache->v_cache : v_suf;
  a.info = r.info;
  a.key_end = r.key_end;
  a.key_rows = r.key_rows;
  a.hinv = r.hinv;
  a.out = out; a.lse = lse;
  a.o_part = reinterpret_cast<float*>(ws + L.opart);
  a.l_part = reinterpret_cast<float*>(ws + L.lpart);
  a.status = status;
  a.T = T; a.M = p.M; a.Lp = d->Lp; a.Hq = d->Hq; a.Hkv = d->Hkv; a.G = p.G; a.d = d->d;
  a.S = p.S; a.split_len = p.split_len;
  a.scale_log2 = scale_log2_of(d);
  a.tile_rows = p.tile_rows; a.n_mt = p.n_mt; a.n_tiles = p.n_tiles; a.n_pre = p.n_pre; a.P = p.P; a.n_ctas = p.n_ctas; a.U = p.U;
  a.full_waves = p.full_waves; a.tail0 = p.tail0; a.tail_ctas = p.tail_ctas;
  a.wait_cycles = g_wait_cycles.load();
  a.wait_probe = g_wait_probe.load();
  if (p.tc) {
    st = run("attn_tc", s, [&] { return launch_attn_tc(a, s); });
    if (st == JEV_OK && p.split) st = run("tc_fixup", s, [&] { return launch_tc_fixup(a, s); });
    return st;
  }
  st = run("attn_simt", s, [&] { return launch_attn_simt(a, d->dtype, s); });
  if (st) return st;
  if (p.S > 1) {
    MergeArgs m{};
    m.o_part = a.o_part; m.l_part = a.l_part; m.info = a.info; m.hinv = a.hinv; m.out = out; m.lse = lse;
    m.M = p.M; m.Hq = d->Hq; m.Hkv = d->Hkv; m.G = p.G; m.d = d->d; m.S = p.S;
    st = run("merge_splits", s, [&] { return launch_merge(m, d->dtype, s); });
  }
  return st;
}

// ---------------------------------------------------------------- trie (host)
// Token-level trie in hash maps, then segments in DFS preorder.
struct HostTrie {
  std::vector<int32_t> tok, depth, nchild, first_child, packed, seg;
  std::vector<std::vector<int32_t>> kids;  // children in order of creation
  std::vector<uint8_t> ends;
  std::unordered_map<uint64_t, int32_t> edge;  // (parent << 32 | token) -> child
  HostTrie() { add(-1, 0); }
  int32_t add(int32_t tk, int32_t dep) {
    tok.push_back(tk); depth.push_back(dep); kids.emplace_back(); ends.push_back(0);
    packed.push_back(-1); seg.push_back(-1);
    return (int32_t)tok.size() - 1;
  }
  int32_t step(int32_t u, int32_t tk) {
    const uint64_t key = ((uint64_t)(uint32_t)u << 32) | (uint32_t)tk;
    auto it = edge.find(key);
    if (it != edge.end()) return it->second;
    int32_t c = add(tk, depth[u] + 1);
    kids[u].push_back(c);
    edge.emplace(key, c);
    return c;
  }
};

}  // namespace
}  // namespace jev

using namespace jev;

extern "C" {

const char* jev_last_error(void) { return g_err; }

int64_t jev_launch_count(void) { return (int64_t)g_launches.load(); }

jev_status jev_debug_set_wait_limit(int64_t cycles) {
  if (cycles < 0) return fail(JEV_ERR_INVALID_ARG, "wait limit must be >= 0");
  g_wait_cycles.store(cycles == 0 ? kDefaultWaitCycles : (long long)cycles);
  return JEV_OK;
}

jev_status jev_debug_set_tc_tile_rows(int32_t rows) {
  if (rows != 0 && rows != 128 && rows != 256) return fail(JEV_ERR_INVALID_ARG, "tile rows must be 0, 128 or 256");
  g_tile_rows.store(rows);
  return JEV_OK;
}

jev_status jev_debug_set_wait_probe(int32_t on) {
  g_wait_probe.store(on != 0 ? 1 : 0);
  return JEV_OK;
}

jev_status jev_profile_enable(int32_t on) {
  g_prof.store(on != 0);
  return JEV_OK;
}

int32_t jev_profile_read(int32_t cap, char* names, int32_t* launches, double* ms, int32_t keep) {
  std::lock_guard<std::mutex> lk(g_mu);
  std::vector<double> tot(g_names.size(), 0.0);
  std::vector<int> cnt(g_names.size(), 0);
  for (const Rec& r : g_recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      cudaGetLastError();  // an event of a graph that was never replayed
      continue;
    }
    tot[r.name] += t;
    cnt[r.name] += 1;
    if (!keep) {
      g_pool.push_back(r.a);
      g_pool.push_back(r.b);
    }
  }
  if (!keep) g_recs.clear();
  int n = 0;
  for (size_t i = 0; i < g_names.size(); ++i) {
    if (!cnt[i]) continue;
    if (n < cap) {
      if (names) {
        strncpy(names + 64 * n, g_names[i].c_str(), 63);
        names[64 * n + 63] = 0;
      }
      if (launches) launches[n] = cnt[i];
      if (ms) ms[n] = tot[i];
    }
    ++n;
  }
  return n;
}

size_t jev_prefix_suffix_attn_workspace(const jev_attn_desc* d) {
  if (check_desc(d) != JEV_OK) return 0;
  Plan p = plan_of(d, d->T_total);
  return layout_of(d, d->T_total, p, 0).total;
}

jev_status jev_prefix_suffix_attn_plan(const jev_attn_desc* d, int32_t kernel, int32_t sms, jev_attn_plan* out) {
  if (!out) return fail(JEV_ERR_INVALID_ARG, "plan is NULL");
  if (kernel < -1 || kernel > 1) return fail(JEV_ERR_INVALID_ARG, "kernel must be -1, 0 or 1");
  jev_status st = check_desc(d);
  if (st) return st;
  const Plan p = plan_of(d, d->T_total, kernel, sms);
  jev_attn_plan r{};
  r.kernel = p.tc ? 1 : 0;
  r.n_tiles = p.n_tiles; r.units_per_tile = p.P; r.n_ctas = p.n_ctas; r.full_waves = p.full_waves;
  r.tail0 = p.tail0; r.tail_ctas = p.tail_ctas; r.split = p.split ? 1 : 0; r.tail_units = p.U;
  r.simt_splits = p.S; r.split_len = p.split_len;
  r.tile_rows = p.tc ? p.tile_rows : 0;
  *out = r;
  return JEV_OK;
}

jev_status jev_selftest_exp2(const float* x, float* y, int32_t n, jev_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return fail(JEV_ERR_INVALID_ARG, "bad arguments");
  return run("selftest_exp2", (cudaStream_t)stream, [&] { return launch_exp2_selftest(x, y, n, (cudaStream_t)stream); });
}

jev_status jev_workspace_init(void* ws, size_t ws_bytes, jev_stream_t stream) {
  if (!ws || ws_bytes < (size_t)kStatusBytes) return fail(JEV_ERR_WORKSPACE, "workspace smaller than the status word");
  cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(JEV_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
  return JEV_OK;
}

jev_status jev_check_device_status(void* ws, size_t ws_bytes, jev_stream_t stream, int32_t* flags) {
  if (!ws || ws_bytes < (size_t)kStatusBytes) return fail(JEV_ERR_WORKSPACE, "workspace smaller than the status word");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(JEV_ERR_CUDA, "stream sync: %s", cudaGetErrorString(e));
  int32_t f = 0;
  e = cudaMemcpyAsync(&f, ws, sizeof f, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, kStatusBytes, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(JEV_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  if (flags) *flags = f;
  if (f) return fail(JEV_ERR_DEVICE, "device status flags 0x%x", f);
  return JEV_OK;
}

jev_status jev_prefix_suffix_attn(const jev_attn_desc* d, const void* q, const void* k_pre, const void* v_pre,
                                  const void* k_suf, const void* v_suf, const int32_t* cu_seqlens,
                                  const int32_t* head_map, void* out, float* lse, void* workspace,
                                  size_t ws_bytes, jev_stream_t stream) {
  jev_status st = check_desc(d);
  if (st) return st;
  if (d->B == 0 || d->T_total == 0) return JEV_OK;
  if (!q || !k_suf || !v_suf || !cu_seqlens || !out) return fail(JEV_ERR_INVALID_ARG, "required pointer is NULL");
  if (d->Lp > 0 && (!k_pre || !v_pre)) return fail(JEV_ERR_INVALID_ARG, "prefix pointers are NULL with Lp > 0");
  const void* ptrs[] = {q, k_pre, v_pre, k_suf, v_suf, out, lse};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(JEV_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  if (!aligned16(cu_seqlens) && ((uintptr_t)cu_seqlens & 3)) return fail(JEV_ERR_INVALID_ARG, "cu_seqlens misaligned");
  const int T = d->T_total;
  Plan p = plan_of(d, T);
  Layout L = layout_of(d, T, p, 0);
  if (!workspace || ((uintptr_t)workspace & 255)) return fail(JEV_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < L.total) return fail(JEV_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  return attention_core(d, T, p, L, (char*)workspace, q, k_pre, v_pre, k_suf, v_suf, cu_seqlens, d->B, nullptr,
                        head_map, false, nullptr, out, lse, (cudaStream_t)stream);
}

size_t jev_suffix_cache_attn_workspace(const jev_attn_desc* d) {
  if (check_desc(d) != JEV_OK) return 0;
  Plan p = plan_of(d, d->T_total);
  return layout_of(d, d->T_total, p, 0, true).total;
}

jev_status jev_suffix_cache_attn(const jev_attn_desc* d, const void* q, const void* k_new, const void* v_new,
                                 const void* k_pre, const void* v_pre, void* k_cache, void* v_cache,
                                 int32_t cache_rows, const int32_t* cache_off, const int32_t* cache_len,
                                 const int32_t* cu_new, const int32_t* head_map, void* out, float* lse,
                                 void* workspace, size_t ws_bytes, jev_stream_t stream) {
  jev_status st = check_desc(d);
  if (st) return st;
  if (d->pos_mode != 0) return fail(JEV_ERR_INVALID_ARG, "positions follow each branch's cache (pos_mode must be 0)");
  if (d->B == 0 || d->T_total == 0) return JEV_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !cache_off || !cache_len || !cu_new || !out)
    return fail(JEV_ERR_INVALID_ARG, "required pointer is NULL");
  if (d->Lp > 0 && (!k_pre || !v_pre)) return fail(JEV_ERR_INVALID_ARG, "prefix pointers are NULL with Lp > 0");
  if (cache_rows < 1) return fail(JEV_ERR_INVALID_ARG, "cache_rows must be >= 1");
  const void* ptrs[] = {q, k_new, v_new, k_pre, v_pre, k_cache, v_cache, out, lse};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(JEV_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  if (((uintptr_t)cache_off | (uintptr_t)cache_len | (uintptr_t)cu_new) & 3)
    return fail(JEV_ERR_INVALID_ARG, "index array misaligned");
  const int T = d->T_total;
  Plan p = plan_of(d, T);
  Layout L = layout_of(d, T, p, 0, true);
  if (!workspace || ((uintptr_t)workspace & 255)) return fail(JEV_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < L.total) return fail(JEV_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  const CacheArgs ca{k_cache, v_cache, cache_rows, cache_off, cache_len};
  return attention_core(d, T, p, L, (char*)workspace, q, k_pre, v_pre, k_new, v_new, cu_new, d->B, nullptr,
                        head_map, false, nullptr, out, lse, (cudaStream_t)stream, &ca);
}

}  // extern "C"

// ---------------------------------------------------------------- fixed scratch
// Scratch of jev_prefix_suffix_attn_noalloc for callers that cannot allocate.
// Host code must not use this symbol as an address: the device address of
// each GPU's copy is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[JEV_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

jev_status noalloc_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(JEV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(JEV_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(JEV_ERR_CUDA, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
    g_noalloc_addr[dev] = p;
  }
  *ptr = g_noalloc_addr[dev];
  return JEV_OK;
}
}  // namespace

extern "C" {

jev_status jev_prefix_suffix_attn_noalloc(const jev_attn_desc* d, const void* q, const void* k_pre,
                                          const void* v_pre, const void* k_suf, const void* v_suf,
                                          const int32_t* cu_seqlens, const int32_t* head_map, void* out,
                                          float* lse, int32_t* status_flags, jev_stream_t stream) {
  jev_status st = check_desc(d);
  if (st) return st;
  if (d->B == 0 || d->T_total == 0) return JEV_OK;
  if (!q || !k_suf || !v_suf || !cu_seqlens || !out) return fail(JEV_ERR_INVALID_ARG, "required pointer is NULL");
  if (d->Lp > 0 && (!k_pre || !v_pre)) return fail(JEV_ERR_INVALID_ARG, "prefix pointers are NULL with Lp > 0");
  const void* ptrs[] = {q, k_pre, v_pre, k_suf, v_suf, out, lse};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(JEV_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  if ((uintptr_t)cu_seqlens & 3) return fail(JEV_ERR_INVALID_ARG, "cu_seqlens misaligned");
  const int T = d->T_total;
  jev_attn_desc dd = *d;
  Plan p = plan_of(&dd, T);
  Layout L = layout_of(&dd, T, p, 0);
  // the tensor-core plan holds split partials when it splits a tile, the
  // CUDA-core plan when it has more than one prefix split
  if (L.total > JEV_NOALLOC_SCRATCH_BYTES && (p.tc ? p.split : p.S > 1)) {
    dd.num_splits = 1;  // no split: no partials
    p = plan_of(&dd, T);
    L = layout_of(&dd, T, p, 0);
  }
  if (L.total > JEV_NOALLOC_SCRATCH_BYTES)
    return fail(JEV_ERR_UNSUPPORTED, "problem needs %zu bytes of scratch; the static scratch holds %u bytes",
                L.total, (unsigned)JEV_NOALLOC_SCRATCH_BYTES);
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(scratch, 0, kStatusBytes, s);
  if (e != cudaSuccess) return fail(JEV_ERR_CUDA, "clearing the status word: %s", cudaGetErrorString(e));
  st = attention_core(&dd, T, p, L, (char*)scratch, q, k_pre, v_pre, k_suf, v_suf, cu_seqlens, dd.B, nullptr,
                      head_map, false, nullptr, out, lse, s);
  if (st) return st;
  if (status_flags) {
    e = cudaMemcpyAsync(status_flags, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return fail(JEV_ERR_CUDA, "copying the status word: %s", cudaGetErrorString(e));
  }
  return JEV_OK;
}

jev_status jev_candidate_readout(const jev_readout_desc* d, const void* hidden, const void* lm_head,
                                 const int32_t* set_offsets, const int32_t* cand_offsets, const int32_t* pair_row,
                                 const int32_t* pair_tok, float* logprob, int32_t* choice, float* score,
                                 jev_stream_t stream) {
  return jev_candidate_readout_normalized(d, hidden, lm_head, set_offsets, cand_offsets, pair_row, pair_tok, nullptr,
                                          logprob, choice, score, stream);
}

jev_status jev_candidate_readout_normalized(const jev_readout_desc* d, const void* hidden, const void* lm_head,
                                            const int32_t* set_offsets, const int32_t* cand_offsets,
                                            const int32_t* pair_row, const int32_t* pair_tok, const float* row_lse,
                                            float* logprob, int32_t* choice, float* score, jev_stream_t stream) {
  if (!d) return fail(JEV_ERR_INVALID_ARG, "desc is NULL");
  if (d->n_sets < 0 || d->n_cands < 0 || d->n_pairs < 0 || d->R < 0 || d->V <= 0 || d->H <= 0)
    return fail(JEV_ERR_INVALID_ARG, "negative or zero sizes");
  if (d->dtype != JEV_BF16 && d->dtype != JEV_F32) return fail(JEV_ERR_UNSUPPORTED, "dtype");
  if (d->H % 8) return fail(JEV_ERR_UNSUPPORTED, "hidden size must be a multiple of 8");
  if (!cand_offsets && d->n_pairs != d->n_cands) return fail(JEV_ERR_INVALID_ARG, "n_pairs != n_cands without cand_offsets");
  if (d->n_sets == 0) return JEV_OK;
  if (!set_offsets || !choice) return fail(JEV_ERR_INVALID_ARG, "set_offsets / choice NULL");
  if (d->n_cands > 0 && (!hidden || !lm_head || !pair_tok || !logprob))
    return fail(JEV_ERR_INVALID_ARG, "required pointer is NULL");
  if ((hidden && !aligned16(hidden)) || (lm_head && !aligned16(lm_head)))
    return fail(JEV_ERR_INVALID_ARG, "hidden / lm_head not 16-byte aligned");
  if (!pair_row && d->R < d->n_sets) return fail(JEV_ERR_INVALID_ARG, "R < n_sets with pair_row NULL");
  if (row_lse && ((uintptr_t)row_lse & 3)) return fail(JEV_ERR_INVALID_ARG, "row_lse misaligned");
  ReadoutArgs a{hidden, lm_head, set_offsets, cand_offsets, pair_row, pair_tok, logprob, choice, score,
                d->n_sets, d->n_cands, d->n_pairs, d->R, d->H, d->V, row_lse};
  int n_kernels = 0;
  const jev_status st =
      run("readout", (cudaStream_t)stream, [&] { return launch_readout(a, d->dtype, (cudaStream_t)stream, &n_kernels); });
  if (st == JEV_OK && n_kernels > 1) g_launches += n_kernels - 1;  // run() counted one
  return st;
}

size_t jev_vocab_lse_workspace(int32_t R, int32_t V) {
  if (R < 0 || V <= 0) return 0;
  return kStatusBytes + up256(vocab_lse_partial_bytes(R, vocab_lse_ctas(V, num_sms())));
}

jev_status jev_vocab_lse(const void* hidden, const void* lm_head, int32_t R, int32_t H, int32_t V, jev_dtype dt,
                         float* lse, void* workspace, size_t ws_bytes, jev_stream_t stream) {
  if (R < 0 || V <= 0 || H <= 0) return fail(JEV_ERR_INVALID_ARG, "negative or zero sizes");
  if (dt != JEV_BF16) return fail(JEV_ERR_UNSUPPORTED, "vocab_lse takes bf16 only");
  if (H % 64) return fail(JEV_ERR_UNSUPPORTED, "hidden size must be a multiple of 64");
  if (!tcgen05_device()) return fail(JEV_ERR_UNSUPPORTED, "vocab_lse needs an sm_100a device");
  if (R == 0) return JEV_OK;
  if (!hidden || !lm_head || !lse) return fail(JEV_ERR_INVALID_ARG, "required pointer is NULL");
  if (!aligned16(hidden) || !aligned16(lm_head)) return fail(JEV_ERR_INVALID_ARG, "hidden / lm_head not 16-byte aligned");
  if (((uintptr_t)lse & 3)) return fail(JEV_ERR_INVALID_ARG, "lse misaligned");
  const size_t need = jev_vocab_lse_workspace(R, V);
  if (!workspace || ((uintptr_t)workspace & 255)) return fail(JEV_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < need) return fail(JEV_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
  const int n_ctas = vocab_lse_ctas(V, num_sms());
  char* ws = (char*)workspace;
  VocabLseArgs a{hidden, lm_head, R, H, V, (V + 255) / 256, (float2*)(ws + kStatusBytes), lse, (int32_t*)ws,
                 g_wait_cycles.load(), g_wait_probe.load()};
  const jev_status st =
      run("vocab_lse", (cudaStream_t)stream, [&] { return launch_vocab_lse(a, n_ctas, (cudaStream_t)stream); });
  if (st == JEV_OK) g_launches++;  // GEMM + online LSE, then the partial merge: two kernels
  return st;
}

jev_status jev_rope_inplace(void* x, int32_t L, int32_t H, int32_t d, int32_t pos0, float theta, jev_dtype dt,
                            jev_stream_t stream) {
  if (L < 0 || H <= 0 || d <= 0 || (d & 1) || d > 256) return fail(JEV_ERR_INVALID_ARG, "bad shape");
  if (!(theta > 0.f)) return fail(JEV_ERR_INVALID_ARG, "theta must be > 0");
  if (L == 0) return JEV_OK;
  if (!x) return fail(JEV_ERR_INVALID_ARG, "x is NULL");
  return run("rope_inplace", (cudaStream_t)stream,
             [&] { return launch_rope_inplace(x, L, H, d, pos0, (double)theta, dt, (cudaStream_t)stream); });
}

jev_status jev_tree_build(int32_t n_cands, const int32_t* seq_off, const int32_t* toks, int32_t root_len,
                          int32_t cap_nodes, int32_t cap_toks, int32_t* parent, int32_t* tok_off, int32_t* pos0,
                          int32_t* leaf_of, int32_t* node_toks, int32_t* path_row, int32_t* n_nodes_out) {
  if (n_cands < 0 || !seq_off || root_len < 0 || !parent || !tok_off || !pos0 || !n_nodes_out)
    return fail(JEV_ERR_INVALID_ARG, "bad arguments");
  if (n_cands > 0 && (!leaf_of)) return fail(JEV_ERR_INVALID_ARG, "leaf_of is NULL");
  if (seq_off[0] != 0) return fail(JEV_ERR_INVALID_ARG, "seq_off[0] != 0");
  for (int c = 0; c < n_cands; ++c)
    if (seq_off[c + 1] < seq_off[c]) return fail(JEV_ERR_INVALID_ARG, "seq_off decreases at %d", c);
  const int total = seq_off[n_cands];
  if (total > 0 && !toks) return fail(JEV_ERR_INVALID_ARG, "toks is NULL");
  HostTrie tr;
  std::vector<int32_t> end_of(n_cands), path_tn(total);
  for (int c = 0; c < n_cands; ++c) {
    int32_t u = 0;
    for (int i = seq_off[c]; i < seq_off[c + 1]; ++i) path_tn[i] = u = tr.step(u, toks[i]);
    end_of[c] = u;
    tr.ends[u] = (u != 0);
  }
  if (cap_nodes < 1) return fail(JEV_ERR_CAPACITY, "cap_nodes < 1");
  // depth-first preorder over chain heads
  struct Item { int32_t u, par; };
  std::vector<Item> stack;
  for (auto it = tr.kids[0].rbegin(); it != tr.kids[0].rend(); ++it) stack.push_back({*it, 0});
  int32_t nn = 1, cursor = 0;
  parent[0] = -1; pos0[0] = 0; tok_off[0] = 0;
  if (cap_nodes >= 1) tok_off[1] = 0;
  while (!stack.empty()) {
    Item it = stack.back();
    stack.pop_back();
    if (nn >= cap_nodes) return fail(JEV_ERR_CAPACITY, "more than %d nodes", cap_nodes);
    const int32_t id = nn++;
    parent[id] = it.par;
    pos0[id] = root_len + tr.depth[it.u] - 1;
    tok_off[id] = cursor;
    int32_t u = it.u;
    for (;;) {
      if (cursor >= cap_toks) return fail(JEV_ERR_CAPACITY, "more than %d packed tokens", cap_toks);
      if (node_toks) node_toks[cursor] = tr.tok[u];
      tr.packed[u] = cursor++;
      tr.seg[u] = id;
      if (tr.kids[u].size() == 1 && !tr.ends[u]) u = tr.kids[u][0];
      else break;
    }
    tok_off[id + 1] = cursor;
    for (auto k = tr.kids[u].rbegin(); k != tr.kids[u].rend(); ++k) stack.push_back({*k, id});
  }
  for (int c = 0; c < n_cands; ++c) leaf_of[c] = end_of[c] ? tr.seg[end_of[c]] : 0;
  if (path_row)
    for (int i = 0; i < total; ++i) path_row[i] = tr.packed[path_tn[i]];
  *n_nodes_out = nn;
  return JEV_OK;
}

jev_status jev_tree_readout_plan(int32_t n_cands, const int32_t* seq_off, const int32_t* toks,
                                 const int32_t* score_from, const int32_t* path_row, int32_t cap_pairs,
                                 int32_t* cand_offsets, int32_t* pair_row, int32_t* pair_tok, int32_t* n_pairs) {
  if (n_cands < 0 || !seq_off || !score_from || !path_row || !cand_offsets || !n_pairs)
    return fail(JEV_ERR_INVALID_ARG, "bad arguments");
  int32_t k = 0;
  cand_offsets[0] = 0;
  for (int c = 0; c < n_cands; ++c) {
    const int a = seq_off[c], e = seq_off[c + 1];
    if (score_from[c] < 1 || a + score_from[c] > e)
      return fail(JEV_ERR_INVALID_ARG, "score_from[%d] = %d outside [1, len]", c, score_from[c]);
    for (int i = a + score_from[c]; i < e; ++i) {
      if (k >= cap_pairs) return fail(JEV_ERR_CAPACITY, "more than %d pairs", cap_pairs);
      pair_row[k] = path_row[i - 1];
      pair_tok[k] = toks[i];
      ++k;
    }
    cand_offsets[c + 1] = k;
  }
  *n_pairs = k;
  return JEV_OK;
}

size_t jev_tree_attn_workspace(const jev_attn_desc* d, int32_t n_nodes) {
  if (check_desc(d) != JEV_OK || n_nodes < 1) return 0;
  Plan p = plan_of(d, d->T_total);
  return layout_of(d, d->T_total, p, n_nodes).total;
}

jev_status jev_tree_attn(const jev_attn_desc* d, int32_t n_nodes, const int32_t* parent, const int32_t* tok_off,
                         const int32_t* pos0, const void* q, const void* k_root, const void* v_root, const void* k,
                         const void* v, const int32_t* head_map, void* out, float* lse, void* workspace,
                         size_t ws_bytes, jev_stream_t stream) {
  jev_status st = check_desc(d);
  if (st) return st;
  if (n_nodes < 1) return fail(JEV_ERR_INVALID_ARG, "n_nodes < 1");
  if (d->pos_mode != 0) return fail(JEV_ERR_INVALID_ARG, "tree positions come from pos0 (pos_mode must be 0)");
  if (d->T_total == 0) return JEV_OK;
  if (!parent || !tok_off || !pos0 || !q || !k || !v || !out) return fail(JEV_ERR_INVALID_ARG, "required pointer is NULL");
  if (d->Lp > 0 && (!k_root || !v_root)) return fail(JEV_ERR_INVALID_ARG, "root pointers are NULL with Lp > 0");
  const void* ptrs[] = {q, k_root, v_root, k, v, out, lse};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return fail(JEV_ERR_INVALID_ARG, "tensor pointer not 16-byte aligned");
  const int T = d->T_total;
  Plan p = plan_of(d, T);
  Layout L = layout_of(d, T, p, n_nodes);
  if (!workspace || ((uintptr_t)workspace & 255)) return fail(JEV_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned");
  if (ws_bytes < L.total) return fail(JEV_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
  char* ws = (char*)workspace;
  return attention_core(d, T, p, L, ws, q, k_root, v_root, k, v, tok_off, n_nodes, pos0, head_map, true, parent, out,
                        lse, (cudaStream_t)stream);
}

}  // extern "C"
