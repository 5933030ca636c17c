// Host side of libfb: argument checks, launch planning and the FlashBlock step
// policy (FlashBlock summary, "Mécanisme Central" and "Stratégies de
// Réutilisation Adaptatives").  Every entry point validates on the host before
// touching CUDA, so a rejected call launches nothing.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <new>
#include <vector>

#include "fb_internal.cuh"

namespace fb {

// Per-device status word written by kernels whose bounded waits expire.
__device__ int g_fb_status = 0;

static uint64_t g_wait_limit_ns = 2000000000ull;
uint64_t wait_limit_ns() { return g_wait_limit_ns; }
static bool g_pdl = true;
bool pdl_enabled() { return g_pdl; }
static bool g_stall = false;
bool debug_stall() { return g_stall; }
static bool g_inblock_bulk = false;
bool inblock_bulk_loads() { return g_inblock_bulk; }
static int g_inblock_rows = 0;
int inblock_rows_setting() { return g_inblock_rows; }
static int g_inblock_kernel = 0;   // 0 automatic, 1 the paired tcgen05 kernel wherever it applies

// Device address of this device's status word, looked up once per device (the
// first launch on a device should come before any stream capture on it; a
// cudaDeviceReset in the process invalidates the cached address).
int* device_status_ptr() {
  static int* cache[kMaxDevices] = {};
  static std::mutex mu;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    int* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_fb_status) != cudaSuccess) return nullptr;
    cache[dev] = p;
  }
  return cache[dev];
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

RowMap make_rowmap(int B, int Hq, int Hkv, int Nb, int per_head, int tile_rows) {
  RowMap rm;
  rm.B = B; rm.Hq = Hq; rm.Hkv = Hkv; rm.G = Hq / Hkv; rm.Nb = Nb;
  rm.per_head = per_head;
  rm.rows_per_unit = per_head ? Nb : rm.G * Nb;
  rm.row_tiles = (rm.rows_per_unit + tile_rows - 1) / tile_rows;
  rm.units = per_head ? B * Hq : B * Hkv;
  return rm;
}

// Split [0, nkeys) into nsplit ranges of keys_per_split (a multiple of
// key_tile) so that tiles * nsplit fills the SMs ctas_per_sm deep.
void plan_split(int64_t tiles, int64_t nkeys, int ctas_per_sm, int key_tile, int32_t* nsplit,
                int64_t* keys_per_split) {
  const int64_t target = (int64_t)num_sms() * ctas_per_sm;
  const int64_t max_split = std::max<int64_t>(1, (nkeys + key_tile - 1) / key_tile);
  int64_t ns = std::max<int64_t>(1, (target + tiles - 1) / tiles);
  ns = std::min(ns, max_split);
  int64_t kps = (nkeys + ns - 1) / ns;
  kps = std::max<int64_t>(key_tile, (kps + key_tile - 1) / key_tile * key_tile);
  ns = std::max<int64_t>(1, (nkeys + kps - 1) / kps);
  *nsplit = (int32_t)ns;
  *keys_per_split = kps;
}

// ------------------------------------------------------------- profiling --
// Event pairs around launches, kept until fb_profile_read folds them in.
struct ProfRecord {
  int kind;
  cudaEvent_t start, stop;
  double bytes;
};
static struct {
  bool on = false;
  std::vector<ProfRecord> pending;
  std::vector<cudaEvent_t> pool;
  int64_t launches[FB_PROFILE_KINDS] = {0, 0, 0};
  double ms[FB_PROFILE_KINDS] = {0, 0, 0};
  double bytes[FB_PROFILE_KINDS] = {0, 0, 0};
} g_prof;

static cudaEvent_t prof_event() {
  if (!g_prof.pool.empty()) {
    cudaEvent_t e = g_prof.pool.back();
    g_prof.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Begin/end a profiled launch on stream s (events: no-ops while profiling is off).
static const char* const kProfNames[FB_PROFILE_KINDS] = {"fb block-external pass", "fb block-internal pass",
                                                         "fb merge/gate/append"};
ProfScope::ProfScope(int kind, double bytes, cudaStream_t s) : kind_(kind), bytes_(bytes), s_(s) {
  nvtxRangePushA(kProfNames[kind]);
  if (!g_prof.on) return;
  start_ = prof_event();
  cudaEventRecord(start_, s_);
}
ProfScope::~ProfScope() {
  nvtxRangePop();
  if (!g_prof.on || !start_) return;
  cudaEvent_t stop = prof_event();
  cudaEventRecord(stop, s_);
  g_prof.pending.push_back({kind_, start_, stop, bytes_});
}

}  // namespace fb

using namespace fb;

// ------------------------------------------------------------------ checks --
static inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static inline int esize(int dt) { return dt == FB_BF16 ? 2 : 4; }

static fb_status check_strides(const int64_t* st, int es) {
  for (int i = 0; i < 3; ++i) {
    if (st[i] < 0) return FB_EINVAL;
    if ((st[i] * es) % 16 != 0) return FB_EALIGN;
  }
  return FB_OK;
}

static fb_status check_desc(const fb_attn_desc* d) {
  if (!d) return FB_EINVAL;
  if (d->B < 1 || d->Hq < 1 || d->Hkv < 1 || d->Nb < 1 || d->D < 1) return FB_EINVAL;
  if (d->Hq % d->Hkv != 0) return FB_EINVAL;
  if ((d->in_dtype != FB_F32 && d->in_dtype != FB_BF16) || (d->out_dtype != FB_F32 && d->out_dtype != FB_BF16))
    return FB_EDTYPE;
  if (d->D != 64 && d->D != 128) return FB_EUNSUPPORTED;
  if (!(d->scale >= 0.f) || isinf(d->scale)) return FB_EINVAL;
  if (d->kp_capacity < 0) return FB_EINVAL;
  fb_status s;
  const int es = esize(d->in_dtype);
  if ((s = check_strides(d->q_strides, es)) != FB_OK) return s;
  if ((s = check_strides(d->kin_strides, es)) != FB_OK) return s;
  if ((s = check_strides(d->kp_strides, es)) != FB_OK) return s;
  if ((s = check_strides(d->o_strides, esize(d->out_dtype))) != FB_OK) return s;
  return FB_OK;
}

static float scale_log2(const fb_attn_desc& d) {
  const float sc = d.scale > 0.f ? d.scale : 1.0f / sqrtf((float)d.D);
  return sc * kLog2e;
}

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
static inline int64_t rows_of(const fb_attn_desc& d) { return (int64_t)d.B * d.Hq * d.Nb; }
static inline size_t part_bytes(const fb_attn_desc& d, int32_t n) {
  return align256((size_t)n * rows_of(d) * d.D * 4) + align256((size_t)n * rows_of(d) * 4);
}

// Upper bound of the split count of one pass over up to max_keys keys (both
// the generic kernel's plan and, for dense prefix passes, the tcgen05 plan).
static int32_t split_bound(const fb_attn_desc& d, int per_head, int64_t max_keys) {
  const RowMap rm = make_rowmap(d.B, d.Hq, d.Hkv, d.Nb, per_head, generic_tile_rows(d.in_dtype == FB_BF16));
  int32_t ns;
  int64_t kps;
  plan_split((int64_t)rm.units * rm.row_tiles, std::max<int64_t>(max_keys, 1),
             generic_ctas_per_sm(d.D, d.in_dtype == FB_BF16), generic_key_tile(), &ns, &kps);
  int mode, hg, tpu, units;
  if (!per_head && tc_tiling(d, &mode, &hg, &tpu, &units)) {
    ns = std::max(ns, tc_split_cap((int64_t)units * tpu, max_keys));
    ns = std::max(ns, pair_slot_cap(d, max_keys));
  }
  return ns;
}

// One attention pass of the block's queries over a key source.
struct PassPlan {
  AttnArgs a;
  int32_t nsplit;
};

static PassPlan plan_pass(const fb_attn_desc& d, const void* q, const void* k, const void* v,
                          const int64_t* kstr, int64_t nkeys, const int32_t* sel, int32_t sel_k,
                          int32_t max_split) {
  PassPlan p;
  memset(&p.a, 0, sizeof(p.a));
  AttnArgs& a = p.a;
  const int bf16 = d.in_dtype == FB_BF16;
  a.rm = make_rowmap(d.B, d.Hq, d.Hkv, d.Nb, sel != nullptr, generic_tile_rows(bf16));
  a.q = q; a.q_sb = d.q_strides[0]; a.q_sh = d.q_strides[1]; a.q_st = d.q_strides[2];
  a.k = k; a.v = v; a.k_sb = kstr[0]; a.k_sh = kstr[1]; a.k_st = kstr[2];
  a.nkeys = sel ? sel_k : nkeys;
  a.sel = sel; a.sel_k = sel_k;
  a.key_rows = nkeys;
  a.scale_log2 = scale_log2(d);
  plan_split((int64_t)a.rm.units * a.rm.row_tiles, a.nkeys, generic_ctas_per_sm(d.D, bf16), generic_key_tile(),
             &a.nsplit, &a.keys_per_split);
  if (sel && a.keys_per_split > generic_max_gather_keys()) {   // a CTA stages at most this many list entries
    a.keys_per_split = generic_max_gather_keys();
    a.nsplit = (int32_t)std::max<int64_t>(1, (a.nkeys + a.keys_per_split - 1) / a.keys_per_split);
  }
  if (max_split > 0 && a.nsplit > max_split) {  // workspace sized smaller: fewer, longer splits
    const int kt = generic_key_tile();
    int64_t kps = (a.nkeys + max_split - 1) / max_split;
    a.keys_per_split = std::max<int64_t>(kt, (kps + kt - 1) / kt * kt);
    a.nsplit = (int32_t)std::max<int64_t>(1, (a.nkeys + a.keys_per_split - 1) / a.keys_per_split);
  }
  p.nsplit = a.nsplit;
  return p;
}

// Algorithmic bytes of one attention pass: each key/value row of the source
// read once per unit that needs it, Q read once, the final (A, L) written once.
static double pass_bytes(const fb_attn_desc& d, const AttnArgs& a) {
  const int es = esize(d.in_dtype);
  const double kv = 2.0 * a.rm.units * (double)a.nkeys * d.D * es;
  return kv + (double)rows_of(d) * d.D * es + (double)rows_of(d) * (d.D + 1) * 4;
}

static fb_status launch_pass(const fb_attn_desc& d, AttnArgs& a, float* pa, float* pl, cudaStream_t s) {
  a.part_a = pa; a.part_l = pl;
  a.part_stride_a = rows_of(d) * d.D;
  a.part_stride_l = rows_of(d);
  ProfScope prof(kProfPrefix, pass_bytes(d, a), s);
  return launch_attn_generic(a, d.D, d.in_dtype == FB_BF16, s) == cudaSuccess ? FB_OK : FB_ECUDA;
}

// Dense block-external pass over prefix rows [0, nkeys): the tcgen05 kernel
// when the shape and strides allow it, else the generic kernel.
static int g_prefix_kernel = 0;  // 0 auto, 1 generic only, 2 tcgen05 whenever it applies, 3 the split
                                 // tcgen05 kernel without clusters, 4 the split kernel with the cluster
                                 // reduction taken at no cost in the plan (3 and 4 never take the paired kernel)

struct PrefixPlan {
  bool tc;
  bool pair;         // the paired stream-K kernel applies (dense passes only)
  PairPlan pp;
  int32_t nsplit;    // CTAs along the keys
  int32_t cluster;   // > 1: the splits reduce inside one cluster
  int32_t nparts;    // parts written: 1 when reduced in-kernel, else nsplit
  int64_t kps;
  PassPlan gen;
  TcMaps maps;
  const uint32_t* excl;   // non-null: per (b, query head) key bitmap
  int64_t excl_words;
  bool excl_invert;       // false: the pass leaves out the set keys; true: it covers only them
};

static PrefixPlan plan_prefix(const fb_attn_desc& d, const void* q, const void* kp, const void* vp, int64_t nkeys,
                              int32_t cap) {
  PrefixPlan p;
  p.gen = plan_pass(d, q, kp, vp, d.kp_strides, nkeys, nullptr, 0, cap);
  p.tc = false;
  p.nsplit = p.nparts = p.gen.nsplit;
  p.cluster = 1;
  p.kps = p.gen.a.keys_per_split;
  p.excl = nullptr;
  p.excl_words = 0;
  p.excl_invert = false;
  p.pair = false;
  const int64_t min_keys = g_prefix_kernel >= 2 ? 1 : 256;
  if (g_prefix_kernel != 1 && nkeys >= min_keys && tc_make_maps(d, q, kp, vp, nkeys, d.kp_strides, &p.maps)) {
    tc_plan_split((int64_t)p.maps.units * p.maps.tiles_per_unit, nkeys, cap, g_prefix_kernel != 3, &p.nsplit,
                  &p.kps, &p.cluster, &p.nparts, g_prefix_kernel == 4 ? 0.0 : 4.0);
    p.tc = true;
    p.pair = (g_prefix_kernel == 0 || g_prefix_kernel == 2) && pair_plan(d, nkeys, &p.pp) && p.pp.smax <= cap;
  }
  return p;
}

static double prefix_bytes(const fb_attn_desc& d, int64_t nkeys) {
  const int es = esize(d.in_dtype);
  return 2.0 * d.B * d.Hkv * (double)nkeys * d.D * es + (double)rows_of(d) * d.D * es +
         (double)rows_of(d) * (d.D + 1) * 4;
}

// The paired pass (plan p.pair, no key bitmap): the final (A, L) at dst, with
// the parts at pa / pl and the slot counts at ns as scratch.
static fb_status launch_prefix_pair(const fb_attn_desc& d, PrefixPlan& p, int64_t nkeys, const int8_t* mask,
                                    int mask_active, float* pa, float* pl, int32_t* ns, float* dst_a, float* dst_l,
                                    cudaStream_t s) {
  {
    ProfScope prof(kProfPrefix, prefix_bytes(d, nkeys), s);
    if (launch_attn_pair(d, p.maps, p.pp, nkeys, mask, mask_active, scale_log2(d), pa, pl, dst_a, dst_l, ns, s,
                         false) != cudaSuccess)
      return FB_ECUDA;
  }
  ProfScope prof(kProfAux, (p.pp.smax + 1.0) * rows_of(d) * (d.D + 1) * 4.0, s);
  return launch_attn_pair(d, p.maps, p.pp, nkeys, mask, mask_active, scale_log2(d), pa, pl, dst_a, dst_l, ns, s,
                          true) == cudaSuccess
             ? FB_OK
             : FB_ECUDA;
}

static fb_status launch_prefix(const fb_attn_desc& d, PrefixPlan& p, int64_t nkeys, const int8_t* mask,
                               int mask_active, float* pa, float* pl, cudaStream_t s) {
  if (!p.tc) {
    p.gen.a.mask = mask;
    p.gen.a.mask_active = mask_active;
    p.gen.a.excl = p.excl;
    p.gen.a.excl_words = p.excl_words;
    return launch_pass(d, p.gen.a, pa, pl, s);
  }
  ProfScope prof(kProfPrefix, prefix_bytes(d, nkeys), s);
  return launch_attn_tc(d, p.maps, nkeys, p.nsplit, p.kps, p.cluster, mask, mask_active, scale_log2(d), pa, pl, s,
                        p.excl, p.excl_words, p.excl_invert) ==
                 cudaSuccess
             ? FB_OK
             : FB_ECUDA;
}

// ---- sparse selected keys over the union of each KV head's selections ----
// Scratch of the union pass for up to umax union keys per KV head: the compact
// K and V rows, the union's positions and sizes, and per query head a
// membership bitmap over the union.
struct UnionWs {
  void* ck;
  void* cv;
  int32_t* upos;
  int32_t* ucount;
  uint32_t* memb;
};
static int64_t union_keys(const fb_attn_desc& d, int64_t prefix_len, int32_t sel_k) {
  return std::min<int64_t>(prefix_len, (int64_t)(d.Hq / d.Hkv) * sel_k);
}
static size_t union_bytes(const fb_attn_desc& d, int64_t umax) {
  const int64_t wu = (umax + 31) / 32;
  return 2 * align256((size_t)d.B * d.Hkv * umax * d.D * esize(d.in_dtype)) +
         align256((size_t)d.B * d.Hkv * umax * 4) + align256((size_t)d.B * d.Hkv * 4) +
         align256((size_t)d.B * d.Hq * wu * 4);
}
static UnionWs union_carve(const fb_attn_desc& d, int64_t umax, uint8_t* base) {
  UnionWs u;
  const int64_t wu = (umax + 31) / 32;
  const size_t kvb = align256((size_t)d.B * d.Hkv * umax * d.D * esize(d.in_dtype));
  u.ck = base;
  u.cv = base + kvb;
  u.upos = reinterpret_cast<int32_t*>(base + 2 * kvb);
  u.ucount = reinterpret_cast<int32_t*>(base + 2 * kvb + align256((size_t)d.B * d.Hkv * umax * 4));
  u.memb = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(u.ucount) + align256((size_t)d.B * d.Hkv * 4));
  (void)wu;
  return u;
}
// The union pass pays off when the union's rows, read, written compact and read
// again, are fewer bytes than one pass over the prefix.
static bool union_applies(const fb_attn_desc& d, int64_t prefix_len, int32_t sel_k) {
  const int64_t u = union_keys(d, prefix_len, sel_k);
  int mode, hg, tpu, units;
  return g_prefix_kernel != 1 && u > 0 && 3 * u < prefix_len && tc_tiling(d, &mode, &hg, &tpu, &units);
}
// Selected keys: the selections' key bitmaps (at `bitmap`) and the union of
// each KV head's selections with every query head's membership over it —
// from the selections in one shared-memory kernel where that fits, else the
// bitmaps first and the union from them; then the union's rows gathered
// compact, and the tcgen05 pass over them that leaves out, per query head,
// the union keys it did not select.
static fb_status launch_selected_union(const fb_attn_desc& d, const void* q, const void* kp, const void* vp,
                                       int64_t prefix_len, const int32_t* sel, uint32_t* bitmap, int32_t sel_k,
                                       const UnionWs& u, int32_t cap, float* pa, float* pl, int32_t* nparts,
                                       cudaStream_t s) {
  const int64_t umax = union_keys(d, prefix_len, sel_k);
  const int64_t wp = (prefix_len + 31) / 32, wu = (umax + 31) / 32;
  const int es = esize(d.in_dtype);
  {
    ProfScope prof(kProfAux, (double)d.B * d.Hq * (sel_k * 4.0 + wp * 4.0 + wu * 4.0), s);
    if (union_build_fits(d, wp, umax)) {
      if (launch_union_build(d, sel, sel_k, bitmap, wp, u.upos, u.ucount, umax, u.memb, wu, s) != cudaSuccess)
        return FB_ECUDA;
    } else if (launch_build_bitmap(sel, sel_k, d.B * d.Hq, bitmap, wp, s) != cudaSuccess ||
               launch_union_select(d, bitmap, wp, u.upos, u.ucount, umax, u.memb, wu, s) != cudaSuccess) {
      return FB_ECUDA;
    }
  }
  {
    ProfScope prof(kProfAux, 4.0 * d.B * d.Hkv * umax * d.D * es, s);
    if (launch_gather_union(d, kp, vp, u.upos, u.ucount, umax, u.ck, u.cv, s) != cudaSuccess) return FB_ECUDA;
  }
  fb_attn_desc dc = d;
  dc.kp_capacity = umax;
  dc.kp_strides[0] = (int64_t)d.Hkv * umax * d.D;
  dc.kp_strides[1] = umax * d.D;
  dc.kp_strides[2] = d.D;
  PrefixPlan p = plan_prefix(dc, q, u.ck, u.cv, umax, cap);
  if (!p.tc) return FB_EUNSUPPORTED;
  p.pair = false;
  p.excl = u.memb;
  p.excl_words = wu;
  p.excl_invert = true;
  *nparts = p.nparts;
  return launch_prefix(dc, p, umax, nullptr, 0, pa, pl, s);
}

static PartGroup group_of(const float* a, const float* l, int32_t n, const fb_attn_desc& d) {
  PartGroup g;
  g.a = a; g.l = l; g.count = n;
  g.stride_a = rows_of(d) * d.D;
  g.stride_l = rows_of(d);
  return g;
}

// Merge `pl` into packed fp32 (A, L) at dst_a / dst_l.
static fb_status merge_to_part(const fb_attn_desc& d, const PartList& pl, float* dst_a, float* dst_l,
                               const int8_t* mask, int mask_active, cudaStream_t s) {
  MergeArgs m;
  memset(&m, 0, sizeof(m));
  m.B = d.B; m.Hq = d.Hq; m.Nb = d.Nb; m.D = d.D;
  m.parts = pl;
  m.o = dst_a; m.o_sb = (int64_t)d.Hq * d.Nb * d.D; m.o_sh = (int64_t)d.Nb * d.D; m.o_st = d.D;
  m.o_bf16 = 0;
  m.lse = dst_l;
  m.mask = mask; m.mask_active = mask_active;
  double nparts = 0;
  for (int i = 0; i < pl.ngroups; ++i) nparts += pl.g[i].count;
  ProfScope prof(kProfAux, (nparts + 1) * rows_of(d) * (d.D + 1) * 4.0, s);
  return launch_merge(m, s) == cudaSuccess ? FB_OK : FB_ECUDA;
}

// Merge `pl` into the output O (the descriptor's output dtype and strides) and LSE.
static fb_status merge_to_out(const fb_attn_desc& d, const PartList& pl, void* o, float* lse, cudaStream_t s) {
  MergeArgs m;
  memset(&m, 0, sizeof(m));
  m.B = d.B; m.Hq = d.Hq; m.Nb = d.Nb; m.D = d.D;
  m.parts = pl;
  m.o = o; m.o_sb = d.o_strides[0]; m.o_sh = d.o_strides[1]; m.o_st = d.o_strides[2];
  m.o_bf16 = d.out_dtype == FB_BF16;
  m.lse = lse;
  double nparts = 0;
  for (int i = 0; i < pl.ngroups; ++i) nparts += pl.g[i].count;
  ProfScope prof(kProfAux, nparts * rows_of(d) * (d.D + 1) * 4.0 + rows_of(d) * (d.D * esize(d.out_dtype) + 4.0),
                 s);
  return launch_merge(m, s) == cudaSuccess ? FB_OK : FB_ECUDA;
}

// Block-internal attention merged with the external parts `ext` into O and
// LSE.  Small blocks: one fused kernel (which can also write the merge of the
// external parts into cache_a / cache_l).  Larger bf16 blocks with a parts
// workspace (ws_a / ws_l, ws_cap parts): the tcgen05 attention kernel over
// the block's own keys writes split parts there, and the merge kernel
// combines them with ext.  Otherwise the generic kernel, fused with the merge.
static fb_status run_inblock(const fb_attn_desc& d, const void* q, const void* kin, const void* vin,
                             const PartList& ext, void* o, float* lse, cudaStream_t s, float* cache_a = nullptr,
                             float* cache_l = nullptr, float* ws_a = nullptr, float* ws_l = nullptr,
                             int32_t ws_cap = 0, int32_t* ws_ns = nullptr) {
  PassPlan p = plan_pass(d, q, kin, vin, d.kin_strides, d.Nb, nullptr, 0, 1);
  AttnArgs& a = p.a;
  a.nsplit = 1;
  a.keys_per_split = d.Nb;
  a.merge_out = 1;
  // the external parts, flattened (the small kernel takes up to 4)
  const float* fa[FB_MAX_PARTS];
  const float* fl[FB_MAX_PARTS];
  int nflat = 0;
  for (int gi = 0; gi < ext.ngroups; ++gi)
    for (int p = 0; p < ext.g[gi].count; ++p) {
      if (nflat < FB_MAX_PARTS) {
        fa[nflat] = ext.g[gi].a + p * ext.g[gi].stride_a;
        fl[nflat] = ext.g[gi].l + p * ext.g[gi].stride_l;
      }
      ++nflat;
    }
  a.next = std::min(nflat, (int)FB_MAX_PARTS);
  for (int i = 0; i < a.next; ++i) { a.ext_a[i] = fa[i]; a.ext_l[i] = fl[i]; }
  a.o = o; a.o_sb = d.o_strides[0]; a.o_sh = d.o_strides[1]; a.o_st = d.o_strides[2];
  a.o_bf16 = d.out_dtype == FB_BF16;
  a.lse = lse;
  double ext_parts = 0;
  for (int i = 0; i < ext.ngroups; ++i) ext_parts += ext.g[i].count;
  const int es = esize(d.in_dtype);
  const double bytes = (double)rows_of(d) * d.D * es + 2.0 * d.B * d.Hkv * d.Nb * d.D * es +
                       ext_parts * rows_of(d) * (d.D + 1) * 4.0 +
                       (double)rows_of(d) * (d.D * esize(d.out_dtype) + (lse ? 4 : 0));
  TcMaps maps;
  PairPlan pw;
  const bool pair_ok = (g_prefix_kernel == 0 || g_prefix_kernel == 2) && nflat <= FB_MAX_PARTS - 1 && !cache_a &&
                       tc_make_maps(d, q, kin, vin, d.Nb, d.kin_strides, &maps) && pair_plan_whole(d, d.Nb, &pw);
  if (inblock_small_applies(d, nflat) && !(g_inblock_kernel == 1 && pair_ok)) {
    ProfScope prof(kProfInblock, bytes, s);
    return launch_inblock_small(d, q, kin, vin, nflat, fa, fl, o, lse, cache_a, cache_l, a.scale_log2, s) ==
                   cudaSuccess
               ? FB_OK
               : FB_ECUDA;
  }
  if (nflat > FB_MAX_PARTS) return FB_EINVAL;
  if (cache_a) return FB_EUNSUPPORTED;   // callers only ask for the cache write where the small kernel runs
  if (pair_ok) {
    // large blocks: the paired kernel over the block's own keys, merged with
    // the external parts in its epilogue.  When the pairs outnumber the CTAs
    // and leave a partial last round (video frame blocks: 168 pairs on 148
    // SMs), the remainder's key tiles are split over the grid instead and
    // their slots merged with the external parts by the merge kernel.
    PairPlan pp;
    ProfScope prof(kProfInblock, bytes, s);
    if (ws_a && ws_ns && pw.npairs > pw.grid && pw.npairs % pw.grid != 0 && pair_plan(d, d.Nb, &pp) &&
        pp.smax <= ws_cap)
      return launch_attn_pair_split_fused(d, maps, pp, d.Nb, a.scale_log2, nflat, fa, fl, o, lse, ws_a, ws_l,
                                          ws_ns, s) == cudaSuccess
                 ? FB_OK
                 : FB_ECUDA;
    return launch_attn_pair_fused(d, maps, pw, d.Nb, a.scale_log2, nflat, fa, fl, o, lse, s) == cudaSuccess
               ? FB_OK
               : FB_ECUDA;
  }
  if (ws_a && ws_cap >= 1 && g_prefix_kernel != 1 && d.Nb >= 128 && ext.ngroups < 8 &&
      tc_make_maps(d, q, kin, vin, d.Nb, d.kin_strides, &maps)) {
    int32_t ns, cl, np;
    int64_t kps;
    tc_plan_split((int64_t)maps.units * maps.tiles_per_unit, d.Nb, ws_cap, false, &ns, &kps, &cl, &np);
    {
      const double tc_bytes = (double)rows_of(d) * d.D * es + 2.0 * d.B * d.Hkv * d.Nb * d.D * es +
                              (double)np * rows_of(d) * (d.D + 1) * 4.0;
      ProfScope prof(kProfInblock, tc_bytes, s);
      if (launch_attn_tc(d, maps, d.Nb, ns, kps, 1, nullptr, 0, a.scale_log2, ws_a, ws_l, s) != cudaSuccess)
        return FB_ECUDA;
    }
    PartList all = ext;
    all.g[all.ngroups++] = group_of(ws_a, ws_l, np, d);
    return merge_to_out(d, all, o, lse, s);
  }
  ProfScope prof(kProfInblock, bytes, s);
  return launch_attn_generic(a, d.D, d.in_dtype == FB_BF16, s) == cudaSuccess ? FB_OK : FB_ECUDA;
}

// ------------------------------------------------------------- public API --
extern "C" {

const char* fb_status_string(fb_status s) {
  switch (s) {
    case FB_OK: return "FB_OK";
    case FB_EINVAL: return "FB_EINVAL: invalid argument";
    case FB_EALIGN: return "FB_EALIGN: pointer or stride not 16-byte aligned";
    case FB_EDTYPE: return "FB_EDTYPE: unsupported dtype";
    case FB_EUNSUPPORTED: return "FB_EUNSUPPORTED: unsupported configuration";
    case FB_ESTATE: return "FB_ESTATE: handle state forbids the call";
    case FB_ECUDA: return "FB_ECUDA: CUDA runtime error";
    case FB_ETIMEOUT: return "FB_ETIMEOUT: a kernel wait expired";
    case FB_ENOSPACE: return "FB_ENOSPACE: workspace too small";
  }
  return "unknown fb_status";
}

int32_t fb_version(void) { return (1 << 16) | 0; }

fb_status fb_outblock_workspace_bytes(const fb_attn_desc* d, int64_t prefix_len, int32_t sel_k, size_t* bytes) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!bytes || prefix_len < 0 || sel_k < 0) return FB_EINVAL;
  size_t n = part_bytes(*d, std::max(split_bound(*d, 0, prefix_len), sel_k ? split_bound(*d, 1, sel_k) : 1));
  n += align256((size_t)pair_count(*d) * 4);
  if (sel_k) n += align256((size_t)d->B * d->Hq * ((prefix_len + 31) / 32) * 4);
  if (sel_k && union_applies(*d, prefix_len, sel_k)) n += union_bytes(*d, union_keys(*d, prefix_len, sel_k));
  *bytes = n;
  return FB_OK;
}

fb_status fb_attn_outblock(const fb_attn_desc* d, const void* q, const void* kp, const void* vp,
                           int64_t prefix_len, const int32_t* sel, int32_t sel_k, float* a_out, float* l_out,
                           float* a_res, float* l_res, void* ws, size_t ws_bytes, cudaStream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!q || !kp || !vp || !a_out || !l_out) return FB_EINVAL;
  if (prefix_len < 0 || prefix_len > d->kp_capacity) return FB_EINVAL;
  if (sel && (sel_k < 0 || sel_k > prefix_len)) return FB_EINVAL;
  if (!sel && (a_res || l_res)) return FB_EINVAL;
  if ((a_res == nullptr) != (l_res == nullptr)) return FB_EINVAL;
  if (!al16(q) || !al16(kp) || !al16(vp) || !al16(a_out) || !al16(l_out) || !al16(sel) || !al16(a_res) ||
      !al16(l_res) || !al16(ws))
    return FB_EALIGN;
  size_t need = 0;
  if ((st = fb_outblock_workspace_bytes(d, prefix_len, sel ? sel_k : 0, &need)) != FB_OK) return st;
  if (!ws || ws_bytes < need) return FB_ENOSPACE;

  uint8_t* w = static_cast<uint8_t*>(ws);
  uint32_t* bitmap = nullptr;
  const int64_t words = (prefix_len + 31) / 32;
  if (sel) {
    bitmap = reinterpret_cast<uint32_t*>(w);
    w += align256((size_t)d->B * d->Hq * words * 4);
  }
  const int32_t cap = std::max(split_bound(*d, 0, prefix_len), sel ? split_bound(*d, 1, sel_k) : 1);
  float* pa = reinterpret_cast<float*>(w);
  float* pl = reinterpret_cast<float*>(w + align256((size_t)cap * rows_of(*d) * d->D * 4));
  int32_t* ns = reinterpret_cast<int32_t*>(w + part_bytes(*d, cap));

  // pass 1: dense prefix, or the selected keys
  if (!sel) {
    PrefixPlan p = plan_prefix(*d, q, kp, vp, prefix_len, cap);
    if (p.pair) return launch_prefix_pair(*d, p, prefix_len, nullptr, 0, pa, pl, ns, a_out, l_out, stream);
    if (p.nparts == 1) return launch_prefix(*d, p, prefix_len, nullptr, 0, a_out, l_out, stream);
    if ((st = launch_prefix(*d, p, prefix_len, nullptr, 0, pa, pl, stream)) != FB_OK) return st;
    PartList lst;
    memset(&lst, 0, sizeof(lst));
    lst.ngroups = 1;
    lst.g[0] = group_of(pa, pl, p.nparts, *d);
    return merge_to_part(*d, lst, a_out, l_out, nullptr, 0, stream);
  }
  const bool via_union = union_applies(*d, prefix_len, sel_k);
  if (via_union) {
    // the union's rows once per KV head, then the pass over them
    const UnionWs u = union_carve(*d, union_keys(*d, prefix_len, sel_k),
                                  reinterpret_cast<uint8_t*>(ns) + align256((size_t)pair_count(*d) * 4));
    int32_t np = 0;
    if ((st = launch_selected_union(*d, q, kp, vp, prefix_len, sel, bitmap, sel_k, u, cap, pa, pl, &np, stream)) !=
        FB_OK)
      return st;
    PartList lst;
    memset(&lst, 0, sizeof(lst));
    lst.ngroups = 1;
    lst.g[0] = group_of(pa, pl, np, *d);
    if ((st = merge_to_part(*d, lst, a_out, l_out, nullptr, 0, stream)) != FB_OK) return st;
  }
  PassPlan p = plan_pass(*d, q, kp, vp, d->kp_strides, prefix_len, sel, sel_k, cap);
  if (via_union) {
  } else if (p.nsplit == 1) {
    if ((st = launch_pass(*d, p.a, a_out, l_out, stream)) != FB_OK) return st;
  } else {
    if ((st = launch_pass(*d, p.a, pa, pl, stream)) != FB_OK) return st;
    PartList lst;
    memset(&lst, 0, sizeof(lst));
    lst.ngroups = 1;
    lst.g[0] = group_of(pa, pl, p.nsplit, *d);
    if ((st = merge_to_part(*d, lst, a_out, l_out, nullptr, 0, stream)) != FB_OK) return st;
  }
  if (!sel || !a_res) return FB_OK;
  // pass 2: the residual (prefix minus the selection)
  if (!via_union && launch_build_bitmap(sel, sel_k, d->B * d->Hq, bitmap, words, stream) != cudaSuccess)
    return FB_ECUDA;
  PrefixPlan r = plan_prefix(*d, q, kp, vp, prefix_len, cap);
  r.excl = bitmap;
  r.excl_words = words;
  if (r.nparts == 1) return launch_prefix(*d, r, prefix_len, nullptr, 0, a_res, l_res, stream);
  if ((st = launch_prefix(*d, r, prefix_len, nullptr, 0, pa, pl, stream)) != FB_OK) return st;
  PartList lst;
  memset(&lst, 0, sizeof(lst));
  lst.ngroups = 1;
  lst.g[0] = group_of(pa, pl, r.nparts, *d);
  return merge_to_part(*d, lst, a_res, l_res, nullptr, 0, stream);
}

fb_status fb_select_workspace_bytes(const fb_attn_desc* d, int64_t prefix_len, size_t* bytes) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!bytes || prefix_len < 0) return FB_EINVAL;
  size_t ob = 0;
  if ((st = fb_outblock_workspace_bytes(d, prefix_len, 0, &ob)) != FB_OK) return st;
  *bytes = align256(ob) + align256((size_t)rows_of(*d) * d->D * 4) + align256((size_t)rows_of(*d) * 4) +
           align256((size_t)d->B * d->Hq * prefix_len * 4);
  return FB_OK;
}

fb_status fb_select_mass(const fb_attn_desc* d, const void* q, const void* kp, const void* vp, int64_t prefix_len,
                         int32_t k, int32_t* sel_out, float* mass_out, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!q || !kp || !vp || (!sel_out && k > 0)) return FB_EINVAL;
  if (prefix_len < 1 || prefix_len > d->kp_capacity || k < 0 || k > prefix_len) return FB_EINVAL;
  if (!mass_applies(*d)) return FB_EUNSUPPORTED;
  if (!al16(q) || !al16(kp) || !al16(vp) || !al16(sel_out) || !al16(mass_out) || !al16(ws)) return FB_EALIGN;
  size_t need = 0, ob = 0;
  if ((st = fb_select_workspace_bytes(d, prefix_len, &need)) != FB_OK) return st;
  if ((st = fb_outblock_workspace_bytes(d, prefix_len, 0, &ob)) != FB_OK) return st;
  if (!ws || ws_bytes < need) return FB_ENOSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* A = reinterpret_cast<float*>(w + align256(ob));
  float* L = reinterpret_cast<float*>(w + align256(ob) + align256((size_t)rows_of(*d) * d->D * 4));
  float* mass = mass_out ? mass_out
                         : reinterpret_cast<float*>(w + align256(ob) + align256((size_t)rows_of(*d) * d->D * 4) +
                                                    align256((size_t)rows_of(*d) * 4));
  // L_out of every block query over the prefix, then each key's mass, then the top k
  if ((st = fb_attn_outblock(d, q, kp, vp, prefix_len, nullptr, 0, A, L, nullptr, nullptr, ws, ob, stream)) !=
      FB_OK)
    return st;
  {
    ProfScope prof(kProfAux, (double)d->B * d->Hkv * prefix_len * d->D * 2 + (double)rows_of(*d) * d->D * 2 +
                                 (double)d->B * d->Hq * prefix_len * 4,
                   stream);
    if (launch_mass(*d, q, kp, prefix_len, L, mass, scale_log2(*d), stream) != cudaSuccess) return FB_ECUDA;
  }
  ProfScope prof(kProfAux, (double)d->B * d->Hq * prefix_len * 4 * 5, stream);
  return launch_topk(mass, d->B * d->Hq, prefix_len, k, sel_out, stream) == cudaSuccess ? FB_OK : FB_ECUDA;
}

static fb_status check_parts(int32_t nparts, const float* const* a, const float* const* l, int32_t maxn) {
  if (nparts < 0 || nparts > maxn) return FB_EINVAL;
  if (nparts > 0 && (!a || !l)) return FB_EINVAL;
  for (int i = 0; i < nparts; ++i) {
    if (!a[i] || !l[i]) return FB_EINVAL;
    if (!al16(a[i]) || !al16(l[i])) return FB_EALIGN;
  }
  return FB_OK;
}

fb_status fb_attn_inblock(const fb_attn_desc* d, const void* q, const void* kin, const void* vin, int32_t nparts,
                          const float* const* a_parts, const float* const* l_parts, void* o, float* lse,
                          cudaStream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!q || !kin || !vin || !o) return FB_EINVAL;
  if ((st = check_parts(nparts, a_parts, l_parts, FB_MAX_PARTS - 1)) != FB_OK) return st;
  if (!al16(q) || !al16(kin) || !al16(vin) || !al16(o) || !al16(lse)) return FB_EALIGN;
  PartList ext;
  memset(&ext, 0, sizeof(ext));
  ext.ngroups = nparts;
  for (int i = 0; i < nparts; ++i) ext.g[i] = group_of(a_parts[i], l_parts[i], 1, *d);
  return run_inblock(*d, q, kin, vin, ext, o, lse, stream);
}

fb_status fb_merge(const fb_attn_desc* d, int32_t nparts, const float* const* a_parts,
                   const float* const* l_parts, void* o, float* lse, cudaStream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!o || nparts < 1) return FB_EINVAL;
  if ((st = check_parts(nparts, a_parts, l_parts, FB_MAX_PARTS)) != FB_OK) return st;
  if (!al16(o) || !al16(lse)) return FB_EALIGN;
  MergeArgs m;
  memset(&m, 0, sizeof(m));
  m.B = d->B; m.Hq = d->Hq; m.Nb = d->Nb; m.D = d->D;
  m.parts.ngroups = nparts;
  for (int i = 0; i < nparts; ++i) m.parts.g[i] = group_of(a_parts[i], l_parts[i], 1, *d);
  m.o = o; m.o_sb = d->o_strides[0]; m.o_sh = d->o_strides[1]; m.o_st = d->o_strides[2];
  m.o_bf16 = d->out_dtype == FB_BF16;
  m.lse = lse;
  ProfScope prof(kProfAux, (double)nparts * rows_of(*d) * (d->D + 1) * 4.0 + rows_of(*d) * d->D * esize(d->out_dtype),
                 stream);
  return launch_merge(m, stream) == cudaSuccess ? FB_OK : FB_ECUDA;
}

fb_status fb_kv_append(const fb_attn_desc* d, void* kp, void* vp, int64_t prefix_len, const void* kin,
                       const void* vin, cudaStream_t stream) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!kp || !vp || !kin || !vin) return FB_EINVAL;
  if (prefix_len < 0 || prefix_len + d->Nb > d->kp_capacity) return FB_EINVAL;
  if (!al16(kp) || !al16(vp) || !al16(kin) || !al16(vin)) return FB_EALIGN;
  ProfScope prof(kProfAux, 4.0 * d->B * d->Hkv * d->Nb * d->D * esize(d->in_dtype), stream);
  return launch_kv_append(*d, kp, vp, prefix_len, kin, vin, stream) == cudaSuccess ? FB_OK : FB_ECUDA;
}

fb_status fb_get_device_status(cudaStream_t stream, fb_status* device_status) {
  if (!device_status) return FB_EINVAL;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FB_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fb_status, sizeof(int)) != cudaSuccess) return FB_ECUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fb_status, &zero, sizeof(int)) != cudaSuccess) return FB_ECUDA;
  }
  *device_status = v == 0 ? FB_OK : static_cast<fb_status>(v);
  return FB_OK;
}

fb_status fb_profile_enable(int32_t on) {
  g_prof.on = on != 0;
  return FB_OK;
}

fb_status fb_profile_read(int32_t reset, int64_t* launches, double* total_ms, double* alg_bytes) {
  for (const ProfRecord& r : g_prof.pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess)
      return FB_ECUDA;
    g_prof.launches[r.kind] += 1;
    g_prof.ms[r.kind] += ms;
    g_prof.bytes[r.kind] += r.bytes;
    g_prof.pool.push_back(r.start);
    g_prof.pool.push_back(r.stop);
  }
  g_prof.pending.clear();
  for (int k = 0; k < FB_PROFILE_KINDS; ++k) {
    if (launches) launches[k] = g_prof.launches[k];
    if (total_ms) total_ms[k] = g_prof.ms[k];
    if (alg_bytes) alg_bytes[k] = g_prof.bytes[k];
    if (reset) { g_prof.launches[k] = 0; g_prof.ms[k] = 0; g_prof.bytes[k] = 0; }
  }
  return FB_OK;
}

fb_status fb_debug_set_prefix_kernel(int32_t which) {
  if (which < 0 || which > 4) return FB_EINVAL;
  g_prefix_kernel = which;
  return FB_OK;
}

fb_status fb_debug_set_stall(int32_t on) {
  g_stall = on != 0;
  return FB_OK;
}

fb_status fb_debug_set_inblock_kernel(int32_t which) {
  if (which < 0 || which > 1) return FB_EINVAL;
  g_inblock_kernel = which;
  return FB_OK;
}

fb_status fb_debug_set_inblock_loads(int32_t bulk) {
  g_inblock_bulk = bulk != 0;
  return FB_OK;
}

fb_status fb_debug_set_inblock_rows(int32_t rows) {
  if (rows != 0 && rows != 1 && rows != 16 && rows != 32 && rows != 64) return FB_EINVAL;
  g_inblock_rows = rows;
  return FB_OK;
}

fb_status fb_debug_set_pdl(int32_t on) {
  g_pdl = on != 0;
  return FB_OK;
}

fb_status fb_debug_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns = ns;
  return FB_OK;
}

}  // extern "C"

// -------------------------------------------------------------- the cache --
struct fb_cache {
  fb_attn_desc d;
  int32_t flags;
  int64_t max_prefix;
  int32_t max_sel_k;
  bool valid;
  int32_t last_recomputed;
  int64_t cached_prefix;   // prefix length and selection size the cached part was computed over
  int32_t cached_sel_k;    // -1: dense
  float* cache_a;     // block-external (or residual) part, packed fp32
  float* cache_l;
  float* part_a;      // split partials of the prefix / residual pass
  float* part_l;
  int32_t part_cap;
  float* sel_a;       // split partials of the selected-keys pass (sparse)
  float* sel_l;
  int32_t sel_cap;
  uint32_t* bitmap;   // sparse membership
  int64_t bitmap_words;
  int8_t* mask;       // gamma: reuse flags for the next step
  float* sim;         // gamma: last similarity per (b, h)
  float* gpart;       // gamma: per-chunk partial sums
  int32_t* counters;  // gamma: per-head arrival counters (kept at zero)
  int32_t chunks;
  int32_t* pair_ns;   // slot counts of the paired prefix pass
  uint8_t* union_base;  // sparse: scratch of the union pass (UnionWs)
  int64_t union_cap;    // union keys per KV head it holds
  void* act_q;        // active subsets: compact queries [B, Hq, Nb, D]
  float* act_a;       // active subsets: compact block-external part
  float* act_l;
};

namespace {
struct Carve {
  size_t off = 0;
  template <class T>
  T* take(uint8_t* base, size_t bytes) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += align256(bytes);
    return p;
  }
};

fb_status layout_cache(const fb_attn_desc& d, int32_t flags, int64_t max_prefix, int32_t max_sel_k,
                       uint8_t* base, fb_cache* c, size_t* total) {
  Carve cv;
  const int64_t rows = rows_of(d);
  const int32_t part_cap = split_bound(d, 0, max_prefix);
  // the selected-keys pass is a per-head gather or, for dense selections, a
  // masked pass over the whole prefix: room for the larger of the two plans
  const int32_t sel_cap =
      (flags & FB_CACHE_SPARSE) ? std::max(split_bound(d, 1, std::max(max_sel_k, 1)), part_cap) : 0;
  const int64_t words = (max_prefix + 31) / 32;
  const int32_t chunks = (d.Nb + gamma_chunk_rows() - 1) / gamma_chunk_rows();
  float* ca = cv.take<float>(base, rows * d.D * 4);
  float* cl = cv.take<float>(base, rows * 4);
  float* pa = cv.take<float>(base, (size_t)part_cap * rows * d.D * 4);
  float* pl = cv.take<float>(base, (size_t)part_cap * rows * 4);
  int32_t* pn = cv.take<int32_t>(base, (size_t)pair_count(d) * 4);
  float* sa = nullptr; float* sl = nullptr; uint32_t* bm = nullptr;
  uint8_t* ub = nullptr;
  int64_t ucap = 0;
  if (flags & FB_CACHE_SPARSE) {
    sa = cv.take<float>(base, (size_t)sel_cap * rows * d.D * 4);
    sl = cv.take<float>(base, (size_t)sel_cap * rows * 4);
    bm = cv.take<uint32_t>(base, (size_t)d.B * d.Hq * words * 4);
    ucap = union_keys(d, max_prefix, max_sel_k);
    ub = cv.take<uint8_t>(base, union_bytes(d, ucap));
  }
  void* aq = nullptr; float* aa = nullptr; float* al = nullptr;
  if (flags & FB_CACHE_ACTIVE) {
    aq = cv.take<uint8_t>(base, (size_t)rows * d.D * esize(d.in_dtype));
    aa = cv.take<float>(base, (size_t)rows * d.D * 4);
    al = cv.take<float>(base, (size_t)rows * 4);
  }
  int8_t* mk = nullptr; float* sm = nullptr; float* gp = nullptr; int32_t* ct = nullptr;
  if (flags & FB_CACHE_GAMMA) {
    mk = cv.take<int8_t>(base, (size_t)d.B * d.Hq);
    sm = cv.take<float>(base, (size_t)d.B * d.Hq * 4);
    gp = cv.take<float>(base, (size_t)d.B * d.Hq * chunks * 3 * 4);
    ct = cv.take<int32_t>(base, (size_t)d.B * d.Hq * 4);
  }
  *total = cv.off;
  if (c) {
    c->cache_a = ca; c->cache_l = cl; c->part_a = pa; c->part_l = pl; c->part_cap = part_cap;
    c->sel_a = sa; c->sel_l = sl; c->sel_cap = sel_cap; c->bitmap = bm; c->bitmap_words = words;
    c->mask = mk; c->sim = sm; c->gpart = gp; c->counters = ct; c->chunks = chunks;
    c->pair_ns = pn;
    c->act_q = aq; c->act_a = aa; c->act_l = al;
    c->union_base = ub; c->union_cap = ucap;
  }
  return FB_OK;
}
}  // namespace

extern "C" {

fb_status fb_cache_workspace_bytes(const fb_attn_desc* d, int32_t flags, int64_t max_prefix, int32_t max_sel_k,
                                   size_t* bytes) {
  fb_status st = check_desc(d);
  if (st != FB_OK) return st;
  if (!bytes || max_prefix < 0 || max_sel_k < 0 || (flags & ~(FB_CACHE_SPARSE | FB_CACHE_GAMMA | FB_CACHE_ACTIVE)))
    return FB_EINVAL;
  return layout_cache(*d, flags, max_prefix, max_sel_k, nullptr, nullptr, bytes);
}

fb_status fb_cache_create(const fb_attn_desc* d, int32_t flags, int64_t max_prefix, int32_t max_sel_k,
                          void* dev_mem, size_t bytes, cudaStream_t stream, fb_cache_t* out) {
  size_t need = 0;
  fb_status st = fb_cache_workspace_bytes(d, flags, max_prefix, max_sel_k, &need);
  if (st != FB_OK) return st;
  if (!out || !dev_mem) return FB_EINVAL;
  if ((reinterpret_cast<uintptr_t>(dev_mem) & 255u) != 0) return FB_EALIGN;
  if (bytes < need) return FB_ENOSPACE;
  fb_cache* c = new (std::nothrow) fb_cache;
  if (!c) return FB_EINVAL;
  memset(c, 0, sizeof(*c));
  c->d = *d; c->flags = flags; c->max_prefix = max_prefix; c->max_sel_k = max_sel_k;
  c->valid = false;
  layout_cache(*d, flags, max_prefix, max_sel_k, static_cast<uint8_t*>(dev_mem), c, &need);
  if (flags & FB_CACHE_GAMMA) {
    if (cudaMemsetAsync(c->mask, 0, (size_t)d->B * d->Hq, stream) != cudaSuccess ||
        cudaMemsetAsync(c->sim, 0xFF, (size_t)d->B * d->Hq * 4, stream) != cudaSuccess ||
        cudaMemsetAsync(c->counters, 0, (size_t)d->B * d->Hq * 4, stream) != cudaSuccess) {
      delete c;
      return FB_ECUDA;
    }
  }
  *out = c;
  return FB_OK;
}

fb_status fb_cache_destroy(fb_cache_t c) {
  if (!c) return FB_EINVAL;
  delete c;
  return FB_OK;
}

fb_status fb_cache_begin_block(fb_cache_t c, cudaStream_t stream) {
  (void)stream;
  if (!c) return FB_EINVAL;
  c->valid = false;
  return FB_OK;
}

fb_status fb_cache_last_step(fb_cache_t c, int32_t* recomputed) {
  if (!c || !recomputed) return FB_EINVAL;
  *recomputed = c->last_recomputed;
  return FB_OK;
}

fb_status fb_step(fb_cache_t c, const fb_step_args* a, cudaStream_t s) {
  NvtxRange range("fb_step");
  if (!c || !a) return FB_EINVAL;
  const fb_attn_desc& d = c->d;
  if (!a->q || !a->kin || !a->vin || !a->kp || !a->vp || !a->o) return FB_EINVAL;
  if (a->prefix_len < 0 || a->prefix_len > c->max_prefix || a->prefix_len > d.kp_capacity) return FB_EINVAL;
  if (a->M < 0) return FB_EINVAL;
  const bool sparse = a->sel != nullptr;
  const bool gamma = a->gamma != nullptr;
  if (sparse && !(c->flags & FB_CACHE_SPARSE)) return FB_ESTATE;
  if (gamma && !(c->flags & FB_CACHE_GAMMA)) return FB_ESTATE;
  if (sparse && gamma) return FB_EUNSUPPORTED;
  if (sparse && (a->sel_k < 0 || a->sel_k > a->prefix_len || a->sel_k > c->max_sel_k)) return FB_EINVAL;
  const bool subset = a->active != nullptr;
  if (subset) {
    if (!(c->flags & FB_CACHE_ACTIVE)) return FB_ESTATE;
    if (a->n_active < 1 || a->n_active > d.Nb) return FB_EINVAL;
    if (sparse || gamma || !inblock_small_applies(d, 1)) return FB_EUNSUPPORTED;
    if (!al16(a->active)) return FB_EALIGN;
  }
  if (!al16(a->q) || !al16(a->kin) || !al16(a->vin) || !al16(a->kp) || !al16(a->vp) || !al16(a->o) ||
      !al16(a->lse) || !al16(a->sel) || !al16(a->gamma))
    return FB_EALIGN;

  // The cached part is attention over one block-external key set; a step over
  // another set (the prefix grew, or the selection size changed) cannot reuse
  // it, so it starts over as at a new block.
  if (c->valid && (a->prefix_len != c->cached_prefix || (sparse ? a->sel_k : -1) != c->cached_sel_k))
    c->valid = false;
  const bool tau_reuse = c->valid && (a->M < a->tau);
  const int BH = d.B * d.Hq;
  c->cached_prefix = a->prefix_len;
  c->cached_sel_k = sparse ? a->sel_k : -1;
  fb_status st;
  PartList ext;
  memset(&ext, 0, sizeof(ext));

  if (subset) {
    // only the active queries: on a full step their block-external part, from
    // a compact copy of their rows, lands in their cache rows
    if (!tau_reuse) {
      const int32_t n = a->n_active;
      fb_attn_desc dc = d;
      dc.Nb = n;
      dc.q_strides[0] = (int64_t)d.Hq * n * d.D;
      dc.q_strides[1] = (int64_t)n * d.D;
      dc.q_strides[2] = d.D;
      {
        ProfScope prof(kProfAux, 2.0 * rows_of(dc) * d.D * esize(d.in_dtype), s);
        if (launch_gather_active_q(d, a->q, c->act_q, a->active, n, s) != cudaSuccess) return FB_ECUDA;
      }
      PrefixPlan p = plan_prefix(dc, c->act_q, a->kp, a->vp, a->prefix_len, c->part_cap);
      p.pair = false;   // its slot counts are sized for the full block
      if (p.nparts == 1) {
        if ((st = launch_prefix(dc, p, a->prefix_len, nullptr, 0, c->act_a, c->act_l, s)) != FB_OK) return st;
      } else {
        if ((st = launch_prefix(dc, p, a->prefix_len, nullptr, 0, c->part_a, c->part_l, s)) != FB_OK) return st;
        PartList lst;
        memset(&lst, 0, sizeof(lst));
        lst.ngroups = 1;
        lst.g[0] = group_of(c->part_a, c->part_l, p.nparts, dc);
        if ((st = merge_to_part(dc, lst, c->act_a, c->act_l, nullptr, 0, s)) != FB_OK) return st;
      }
      ProfScope prof(kProfAux, 2.0 * rows_of(dc) * (d.D + 1) * 4.0, s);
      if (launch_scatter_active_part(d, c->act_a, c->act_l, c->cache_a, c->cache_l, a->active, n, s) != cudaSuccess)
        return FB_ECUDA;
    }
    if (a->reuse_out && launch_fill_decision(a->reuse_out, BH, tau_reuse ? 1 : 0, s) != cudaSuccess)
      return FB_ECUDA;
    if (a->sim_out && cudaMemsetAsync(a->sim_out, 0xFF, (size_t)BH * 4, s) != cudaSuccess) return FB_ECUDA;
    const float* ca[1] = {c->cache_a};
    const float* cl[1] = {c->cache_l};
    const int es = esize(d.in_dtype);
    const double rows = (double)d.B * d.Hq * a->n_active;
    {
      ProfScope prof(kProfInblock, rows * d.D * es + 2.0 * d.B * d.Hkv * d.Nb * d.D * es + rows * (d.D + 1) * 4.0 +
                                       rows * (d.D * esize(d.out_dtype) + (a->lse ? 4 : 0)),
                     s);
      if (launch_inblock_small(d, a->q, a->kin, a->vin, 1, ca, cl, a->o, a->lse, nullptr, nullptr, scale_log2(d), s,
                               a->active, a->n_active) != cudaSuccess)
        return FB_ECUDA;
    }
    c->valid = true;
    c->last_recomputed = !tau_reuse;
    return FB_OK;
  }
  if (gamma) {
    PrefixPlan p = plan_prefix(d, a->q, a->kp, a->vp, a->prefix_len, c->part_cap);
    int32_t fresh_parts = p.nparts;
    if (p.pair) {
      // the fresh part of every computed head, merged, in part 0
      if ((st = launch_prefix_pair(d, p, a->prefix_len, c->mask, tau_reuse, c->part_a, c->part_l, c->pair_ns,
                                   c->part_a, c->part_l, s)) != FB_OK)
        return st;
      fresh_parts = 1;
    } else if ((st = launch_prefix(d, p, a->prefix_len, c->mask, tau_reuse, c->part_a, c->part_l, s)) != FB_OK) {
      return st;
    }
    GammaArgs g;
    memset(&g, 0, sizeof(g));
    g.B = d.B; g.Hq = d.Hq; g.Nb = d.Nb; g.D = d.D;
    g.fresh.ngroups = 1;
    g.fresh.g[0] = group_of(c->part_a, c->part_l, fresh_parts, d);
    g.cache_a = c->cache_a; g.cache_l = c->cache_l;
    g.mask = c->mask; g.gate_active = tau_reuse; g.cache_valid = c->valid;
    g.gamma = a->gamma; g.sim = c->sim; g.partials = c->gpart; g.counters = c->counters;
    g.chunks = c->chunks; g.reuse_out = a->reuse_out; g.sim_out = a->sim_out;
    {
      ProfScope prof(kProfAux, (fresh_parts + 2.0) * rows_of(d) * (d.D + 1) * 4.0, s);
      if (launch_gamma_update(g, s) != cudaSuccess) return FB_ECUDA;
    }
  } else {
    bool bitmap_built = false;
    if (sparse) {
      // Selected keys: gathered row by row per query head, or — when the
      // selection covers more than 1/(3G) of the prefix, where gathering per
      // query head would read a third of the prefix bytes or more (and reads
      // them at a fraction of the rate of the streaming kernel) — a tcgen05
      // pass over the whole prefix that leaves out every key not selected.
      int32_t nsel = 0;
      PrefixPlan sp;
      sp.tc = false;
      const bool via_union = union_applies(d, a->prefix_len, a->sel_k) &&
                             union_keys(d, a->prefix_len, a->sel_k) <= c->union_cap;
      if (!via_union && (int64_t)a->sel_k * 3 * (d.Hq / d.Hkv) > a->prefix_len) {
        sp = plan_prefix(d, a->q, a->kp, a->vp, a->prefix_len, c->sel_cap);
      }
      if (via_union) {
        bitmap_built = true;
        const UnionWs u = union_carve(d, union_keys(d, a->prefix_len, a->sel_k), c->union_base);
        if ((st = launch_selected_union(d, a->q, a->kp, a->vp, a->prefix_len, a->sel, c->bitmap, a->sel_k, u,
                                        c->sel_cap, c->sel_a, c->sel_l, &nsel, s)) != FB_OK)
          return st;
      } else if (sp.tc) {
        if (launch_build_bitmap(a->sel, a->sel_k, BH, c->bitmap, (a->prefix_len + 31) / 32, s) != cudaSuccess)
          return FB_ECUDA;
        bitmap_built = true;
        sp.excl = c->bitmap;
        sp.excl_words = (a->prefix_len + 31) / 32;
        sp.excl_invert = true;
        if ((st = launch_prefix(d, sp, a->prefix_len, nullptr, 0, c->sel_a, c->sel_l, s)) != FB_OK) return st;
        nsel = sp.nparts;
      } else {
        PassPlan p = plan_pass(d, a->q, a->kp, a->vp, d.kp_strides, a->prefix_len, a->sel, a->sel_k, c->sel_cap);
        if ((st = launch_pass(d, p.a, c->sel_a, c->sel_l, s)) != FB_OK) return st;
        nsel = p.nsplit;
      }
      if (nsel > FB_MAX_PARTS - 1) {
        // fold the splits into split 0's slot (each row is read fully before it is written)
        PartList lst;
        memset(&lst, 0, sizeof(lst));
        lst.ngroups = 1;
        lst.g[0] = group_of(c->sel_a, c->sel_l, nsel, d);
        if ((st = merge_to_part(d, lst, c->sel_a, c->sel_l, nullptr, 0, s)) != FB_OK) return st;
        ext.g[ext.ngroups++] = group_of(c->sel_a, c->sel_l, 1, d);
      } else {
        ext.g[ext.ngroups++] = group_of(c->sel_a, c->sel_l, nsel, d);
      }
    }
    if (!tau_reuse) {
      // dense: the whole prefix; sparse: the prefix minus each head's selection
      PrefixPlan p = plan_prefix(d, a->q, a->kp, a->vp, a->prefix_len, c->part_cap);
      if (sparse) {
        if (!bitmap_built &&
            launch_build_bitmap(a->sel, a->sel_k, BH, c->bitmap, (a->prefix_len + 31) / 32, s) != cudaSuccess)
          return FB_ECUDA;
        p.excl = c->bitmap;
        p.excl_words = (a->prefix_len + 31) / 32;
      }
      if (!sparse && p.pair) {
        if ((st = launch_prefix_pair(d, p, a->prefix_len, nullptr, 0, c->part_a, c->part_l, c->pair_ns, c->cache_a,
                                     c->cache_l, s)) != FB_OK)
          return st;
      } else if (!sparse && p.nparts > 1 && inblock_small_applies(d, p.nparts)) {
        // the in-block kernel can take the split parts itself and write their
        // merge into the cache, saving a merge pass
        if ((st = launch_prefix(d, p, a->prefix_len, nullptr, 0, c->part_a, c->part_l, s)) != FB_OK) return st;
        ext.g[ext.ngroups++] = group_of(c->part_a, c->part_l, p.nparts, d);
        if (a->reuse_out && launch_fill_decision(a->reuse_out, BH, 0, s) != cudaSuccess) return FB_ECUDA;
        if (a->sim_out && cudaMemsetAsync(a->sim_out, 0xFF, (size_t)BH * 4, s) != cudaSuccess) return FB_ECUDA;
        if ((st = run_inblock(d, a->q, a->kin, a->vin, ext, a->o, a->lse, s, c->cache_a, c->cache_l)) != FB_OK)
          return st;
        c->valid = true;
        c->last_recomputed = 1;
        return FB_OK;
      } else if (p.nparts == 1) {
        if ((st = launch_prefix(d, p, a->prefix_len, nullptr, 0, c->cache_a, c->cache_l, s)) != FB_OK) return st;
      } else {
        if ((st = launch_prefix(d, p, a->prefix_len, nullptr, 0, c->part_a, c->part_l, s)) != FB_OK) return st;
        PartList lst;
        memset(&lst, 0, sizeof(lst));
        lst.ngroups = 1;
        lst.g[0] = group_of(c->part_a, c->part_l, p.nparts, d);
        if ((st = merge_to_part(d, lst, c->cache_a, c->cache_l, nullptr, 0, s)) != FB_OK) return st;
      }
    }
    if (a->reuse_out && launch_fill_decision(a->reuse_out, BH, tau_reuse ? 1 : 0, s) != cudaSuccess)
      return FB_ECUDA;
    if (a->sim_out && cudaMemsetAsync(a->sim_out, 0xFF, (size_t)BH * 4, s) != cudaSuccess) return FB_ECUDA;
  }
  ext.g[ext.ngroups++] = group_of(c->cache_a, c->cache_l, 1, d);
  // the split parts of the prefix pass are consumed by now: their slots take
  // the block-internal pass's parts
  if ((st = run_inblock(d, a->q, a->kin, a->vin, ext, a->o, a->lse, s, nullptr, nullptr, c->part_a, c->part_l,
                        c->part_cap, c->pair_ns)) != FB_OK)
    return st;
  c->valid = true;
  c->last_recomputed = !tau_reuse;
  return FB_OK;
}

}  // extern "C"
