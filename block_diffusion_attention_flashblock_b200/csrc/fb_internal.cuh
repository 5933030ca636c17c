// Internal declarations shared by the libfb translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>
#include "fb.h"

namespace fb {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// A group of `count` packed fp32 parts, part p at (a + p*stride_a, l + p*stride_l).
struct PartGroup {
  const float* a;
  const float* l;
  int32_t count;
  int64_t stride_a, stride_l;
};

struct PartList {
  int32_t ngroups;
  PartGroup g[FB_MAX_PARTS];
};

// Where an attention kernel's (b, h, i) rows come from and how they are tiled.
//   packed   (per_head = 0): unit = (b, kv head); its G*Nb rows are the block
//            queries of the G query heads sharing that KV head, row r = g*Nb+i.
//   per_head (per_head = 1): unit = (b, query head); rows are its Nb queries.
struct RowMap {
  int32_t B, Hq, Hkv, G, Nb;
  int32_t per_head;
  int32_t rows_per_unit;
  int32_t row_tiles;       // tiles of the kernel's row count per unit
  int32_t units;
};

// Arguments of the attention kernels (one launch = one key source).
struct AttnArgs {
  RowMap rm;
  const void* q;
  int64_t q_sb, q_sh, q_st;
  const void* k;
  const void* v;
  int64_t k_sb, k_sh, k_st;
  int64_t nkeys;               // keys in the source: [0, nkeys) or list entries
  const int32_t* sel;          // per (b, query head) key list (per_head units only)
  int32_t sel_k;
  int64_t key_rows;            // rows addressable in the key source (list entries outside are skipped)
  const uint32_t* excl;        // per (b, query head) bitmap: 1 = key excluded
  int64_t excl_words;
  int32_t nsplit;
  int64_t keys_per_split;
  const int8_t* mask;          // gamma: [B, Hq]; heads with mask=1 may be skipped
  int32_t mask_active;         // 0: ignore mask
  // epilogue 0: write part (A, L) of split s at part_a + s*part_stride_a ...
  float* part_a;
  float* part_l;
  int64_t part_stride_a, part_stride_l;
  // epilogue 1: merge with up to FB_MAX_PARTS packed parts and write O / LSE
  int32_t merge_out;
  int32_t next;
  const float* ext_a[FB_MAX_PARTS];
  const float* ext_l[FB_MAX_PARTS];
  void* o;
  int64_t o_sb, o_sh, o_st;
  int32_t o_bf16;
  float* lse;
  float scale_log2;            // softmax scale * log2(e)
};

// An NVTX range for the host-side span of one API call or launch (a no-op
// unless a profiler is attached).
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Profiling scope: brackets one launch with events on its stream when the
// profiling hook is on (fb_profile_enable), and with an NVTX range named for
// its kind; kinds as in fb.h.
enum { kProfPrefix = 0, kProfInblock = 1, kProfAux = 2 };
class ProfScope {
 public:
  ProfScope(int kind, double alg_bytes, cudaStream_t s);
  ~ProfScope();
  ProfScope(const ProfScope&) = delete;
  ProfScope& operator=(const ProfScope&) = delete;

 private:
  int kind_;
  double bytes_;
  cudaStream_t s_;
  cudaEvent_t start_ = nullptr;
};

// Kernel launch with programmatic dependent launch allowed (when enabled):
// the next kernel in the stream may start its launch while this one drains;
// every kernel begins with ptx::pdl_prologue(), so it touches no global
// memory before the kernels it depends on have completed.
bool pdl_enabled();
bool debug_stall();   // test hook: kernels first wait on a barrier nothing completes
bool inblock_bulk_loads();   // tuning hook: the small in-block kernel loads by bulk copy per row
int inblock_rows_setting();   // tuning hook: 0 automatic, 1 the split-warp kernel, 16/32/64 rows per CTA
template <class... KArgs, class... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// Index of the current device for per-device host caches (0 when it cannot
// be read; caches hold kMaxDevices entries).
constexpr int kMaxDevices = 64;
inline int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  return dev;
}

// Host-side planning helpers (fb_api.cu).
int num_sms();
RowMap make_rowmap(int B, int Hq, int Hkv, int Nb, int per_head, int tile_rows);
void plan_split(int64_t tiles, int64_t nkeys, int ctas_per_sm, int key_tile,
                int32_t* nsplit, int64_t* keys_per_split);

// Launchers (return cudaGetLastError()).
cudaError_t launch_attn_generic(const AttnArgs& a, int D, int in_bf16, cudaStream_t s);
int generic_tile_rows(int in_bf16);
int generic_key_tile();
int generic_max_gather_keys();   // longest key-list slice per CTA of a gather pass
int generic_ctas_per_sm(int D, int in_bf16);

// tcgen05 prefix pass (fb_attn_tc.cu).
struct TcMaps {
  CUtensorMap q, k, v;
  int mode, hg, tiles_per_unit, units;
};
bool tc_tiling(const fb_attn_desc& d, int* mode, int* hg, int* tiles_per_unit, int* units);
// Tensor maps for a pass over keys [0, nkeys) of K/V with (b, h, t) strides kstr.
bool tc_make_maps(const fb_attn_desc& d, const void* q, const void* k, const void* v, int64_t nkeys,
                  const int64_t* kstr, TcMaps* m);
void tc_plan_split(int64_t tiles, int64_t nkeys, int32_t max_parts, bool allow_cluster, int32_t* nsplit,
                   int64_t* kps, int32_t* cluster, int32_t* nparts, double cluster_cost = 4.0);
int32_t tc_split_cap(int64_t tiles, int64_t max_keys);
cudaError_t launch_attn_tc(const fb_attn_desc& d, const TcMaps& m, int64_t nkeys, int32_t nsplit, int64_t kps,
                           int32_t cluster, const int8_t* mask, int mask_active, float scale_log2, float* pa,
                           float* pl, cudaStream_t s, const uint32_t* excl = nullptr, int64_t excl_words = 0,
                           bool excl_invert = false);

// Paired tcgen05 prefix pass, persistent stream-K grid (fb_attn_pair.cu).
struct PairPlan {
  int32_t mode, hg, tph, tiles_per_kv, pairs_per_kv, npairs, nkt, grid, smax;
};
bool pair_plan(const fb_attn_desc& d, int64_t nkeys, PairPlan* p);
int32_t pair_slot_cap(const fb_attn_desc& d, int64_t max_keys);
int32_t pair_count(const fb_attn_desc& d);   // pairs of the paired pass (0: it never applies)
bool pair_plan_whole(const fb_attn_desc& d, int64_t nkeys, PairPlan* p);
// Whole-pair mode: each CTA takes whole pairs and merges each row with `next`
// external parts into O (out dtype, strides) and LSE; one launch, no scratch.
cudaError_t launch_attn_pair_split_fused(const fb_attn_desc& d, const TcMaps& m, const PairPlan& pp, int64_t nkeys,
                                         float scale_log2, int32_t next, const float* const* ext_a,
                                         const float* const* ext_l, void* o, float* lse, float* pa, float* pl,
                                         int32_t* nslots, cudaStream_t s);
cudaError_t launch_attn_pair_fused(const fb_attn_desc& d, const TcMaps& m, const PairPlan& pp, int64_t nkeys,
                                   float scale_log2, int32_t next, const float* const* ext_a,
                                   const float* const* ext_l, void* o, float* lse, cudaStream_t s);
// The pass (merge_only = false) leaves the final (A, L) of rows whose pair one
// CTA covered at dst_a / dst_l and partial results in pp.smax parts at pa /
// pl (npairs slot counts at nslots); the merge (merge_only = true, launched
// after it with the same arguments) combines the partials into dst.  dst may
// be part 0.
cudaError_t launch_attn_pair(const fb_attn_desc& d, const TcMaps& m, const PairPlan& pp, int64_t nkeys,
                             const int8_t* mask, int mask_active, float scale_log2, float* pa, float* pl,
                             float* dst_a, float* dst_l, int32_t* nslots, cudaStream_t s, bool merge_only);

// Selection by attention mass (fb_select.cu).
bool mass_applies(const fb_attn_desc& d);
cudaError_t launch_mass(const fb_attn_desc& d, const void* q, const void* kp, int64_t nkeys, const float* l_out,
                        float* mass, float scale_log2, cudaStream_t s);
cudaError_t launch_topk(const float* mass, int32_t BH, int64_t n, int32_t k, int32_t* sel, cudaStream_t s);

// Small-block in-block attention + merge (fb_inblock.cu).
bool inblock_small_applies(const fb_attn_desc& d, int next);
// With `active` ([B, n_act] block positions) only those queries are computed
// and only their rows of O, LSE and the cache are written.
cudaError_t launch_inblock_small(const fb_attn_desc& d, const void* q, const void* kin, const void* vin, int next,
                                 const float* const* ext_a, const float* const* ext_l, void* o, float* lse,
                                 float* cache_a, float* cache_l, float scale_log2, cudaStream_t s,
                                 const int32_t* active = nullptr, int32_t n_act = 0);
cudaError_t launch_gather_active_q(const fb_attn_desc& d, const void* q, void* out, const int32_t* active,
                                   int32_t n_act, cudaStream_t s);
cudaError_t launch_scatter_active_part(const fb_attn_desc& d, const float* ca, const float* cl, float* a, float* l,
                                       const int32_t* active, int32_t n_act, cudaStream_t s);

struct MergeArgs {
  int32_t B, Hq, Nb, D;
  PartList parts;
  void* o;
  int64_t o_sb, o_sh, o_st;
  int32_t o_bf16;
  float* lse;
  const int8_t* mask;       // rows of heads with mask=1 are skipped (or NULL)
  int32_t mask_active;
};
cudaError_t launch_merge(const MergeArgs& m, cudaStream_t s);

struct GammaArgs {
  int32_t B, Hq, Nb, D;
  PartList fresh;           // the fresh block-external part (split partials)
  float* cache_a;           // packed [B, Hq, Nb, D]
  float* cache_l;           // packed [B, Hq, Nb]
  int8_t* mask;             // [B, Hq] reuse-next-step flags (read, then updated)
  int32_t gate_active;      // host: cache valid && M < tau
  int32_t cache_valid;      // host: a similarity can be formed
  const float* gamma;       // device [Hq]
  float* sim;               // device [B, Hq] state
  float* partials;          // [B*Hq*chunks*3] scratch
  int32_t* counters;        // [B*Hq], zero between launches
  int32_t chunks;
  int8_t* reuse_out;        // [B, Hq] or NULL
  float* sim_out;           // [B, Hq] or NULL
};
cudaError_t launch_gamma_update(const GammaArgs& g, cudaStream_t s);
int gamma_chunk_rows();

cudaError_t launch_kv_append(const fb_attn_desc& d, void* kp, void* vp, int64_t prefix_len,
                             const void* kin, const void* vin, cudaStream_t s);
cudaError_t launch_build_bitmap(const int32_t* sel, int32_t sel_k, int32_t BH,
                                uint32_t* bitmap, int64_t words, cudaStream_t s);
cudaError_t launch_fill_decision(int8_t* reuse_out, int32_t n, int8_t value, cudaStream_t s);
// The union of each KV head's query heads' selections (positions in key order,
// at most umax) and per query head a membership bitmap over it; then its
// rows of K/V gathered into a compact [B, Hkv, umax, D] block.
cudaError_t launch_union_select(const fb_attn_desc& d, const uint32_t* bitmap, int64_t words_p, int32_t* upos,
                                int32_t* ucount, int64_t umax, uint32_t* memb, int64_t words_u, cudaStream_t s);
// The selections' key bitmaps (written to `bitmap`) and the union select above
// in one launch, in shared memory, where the G bitmaps and umax positions fit.
bool union_build_fits(const fb_attn_desc& d, int64_t words_p, int64_t umax);
cudaError_t launch_union_build(const fb_attn_desc& d, const int32_t* sel, int32_t sel_k, uint32_t* bitmap,
                               int64_t words_p, int32_t* upos, int32_t* ucount, int64_t umax, uint32_t* memb,
                               int64_t words_u, cudaStream_t s);
cudaError_t launch_gather_union(const fb_attn_desc& d, const void* kp, const void* vp, const int32_t* upos,
                                const int32_t* ucount, int64_t umax, void* ck, void* cv, cudaStream_t s);

}  // namespace fb
