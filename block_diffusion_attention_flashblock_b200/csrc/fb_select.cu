// Selection of the sparse keys by attention mass: the keys of the prefix that
// the block's queries attend to most, per query head.  FlashBlock treats the
// keys a sparse method leaves out as its block-external set and caches their
// residual contribution (FlashBlock summary, "Stratégies de Réutilisation
// Adaptatives", sparse bullet; "Résultats Expérimentaux", SparseD at 20-40 %
// density).  The pages do not give the sparse method's rule; the one built
// here is the top-k of
//     mass[b, h, j] = sum_i exp(s_ij - L_out,i),   s_ij = scale * q_i . k_j,
// the softmax probability over the prefix that key j receives from the
// block's queries i, summed over them, ties to the lower index.
//
// Three launches: the prefix pass for L_out (the dense block-external pass),
// the mass kernel, and the top-k kernel.
//   mass_kernel: one CTA per (key tile of 128 keys, b, KV head).  One tcgen05
//     MMA gives D = K Q^T (128 keys x the KV head's G * Nb packed query rows,
//     which must fit one 128-row tile), so TMEM lane = key and each thread
//     sums its own key's probabilities over each head's Nb columns in a fixed
//     order: no atomics, the same bits on every run.
//   topk_kernel: one CTA per (b, h); a four-pass radix select on the fp32
//     bits (masses are non-negative, so their bits order like their values)
//     finds the k-th largest value, then a scan in key order keeps every key
//     above it and the lowest-index keys equal to it, ascending.
#include <cub/block/block_scan.cuh>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <algorithm>

#include "fb_internal.cuh"
#include "fb_ptx.cuh"
#include "fb_tc.cuh"

namespace fb {

namespace {

using namespace tc;

constexpr int kD = 128, kBN = 128;
constexpr uint32_t kHalf = 16384, kTile = 32768;
constexpr uint32_t kSmemBytes = 2 * kTile + 1024 + 512 + 64;   // K, Q, alignment, L, barriers

// NB columns at a column offset that is a multiple of NB
template <int NB>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* v) {
  static_assert(NB == 16 || NB == 32, "columns per head");
  uint32_t r[NB];
  if constexpr (NB == 16) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
  } else {
    float f[32];
    tmem_ld32(taddr, f);
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(f[i]);
  }
#pragma unroll
  for (int i = 0; i < NB; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace

struct MassArgs {
  int32_t B, Hq, Hkv, G, Nb;
  int64_t nkeys;
  float scale_log2;
  const float* l_out;      // [B, Hq, Nb] natural log, packed
  float* mass;             // [B, Hq, nkeys]
  int* status;
  uint64_t wait_limit_ns;
};

// NB: block length (columns per head); the KV head's G * NB rows fit one tile.
template <int NB>
__global__ void __launch_bounds__(128, 1)
    mass_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, const MassArgs a) {
  ptx::pdl_prologue();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (smem - smem_raw > 1024) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0, (int)FB_EUNSUPPORTED);
    return;
  }
  const uint32_t sK = smem_addr(smem), sQ = sK + kTile;
  float* sL = reinterpret_cast<float*>(smem + 2 * kTile);          // log2-domain L of the tile's rows
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kTile + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 3);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  const uint32_t bar_ld = smem_addr(bars), bar_mma = bar_ld + 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x;                       // key tile
  const int u = blockIdx.y, b = u / a.Hkv, kvh = u % a.Hkv;
  const int rows = a.G * NB;
  const int64_t rbase = ((int64_t)b * a.Hq + (int64_t)kvh * a.G) * NB;
  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_ld, 1);
    ptx::mbar_init(bar_mma, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  for (int r = threadIdx.x; r < kBN; r += blockDim.x) sL[r] = r < rows ? a.l_out[rbase + r] * kLog2e : 0.f;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(128));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Ctl ctl{abort_flag, a.status, a.wait_limit_ns};
  bool ok = true;
  if (threadIdx.x == 0) {
    ptx::mbar_expect_tx(bar_ld, kTile + 256u * (uint32_t)rows);   // K tile + the G x NB query rows
    tma_load_4d(sK, &tmK, bar_ld, 0, j * kBN, kvh, b);
    tma_load_4d(sK + kHalf, &tmK, bar_ld, 64, j * kBN, kvh, b);
    tma_load_4d(sQ, &tmQ, bar_ld, 0, 0, kvh * a.G, b);
    tma_load_4d(sQ + kHalf, &tmQ, bar_ld, 64, 0, kvh * a.G, b);
    ok = wait_phase(bar_ld, 0, ctl);
    if (ok) {
      tc_fence_after();
      // D[key][row] = K Q^T: A = the K tile, B = the Q tile (both K-major)
      const uint64_t dK = sw128_desc(sK, 16, 1024), dQ = sw128_desc(sQ, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
        tc_mma(tmem, dK + off, dQ + off, kIdescQK, kk > 0 ? 1u : 0u);
      }
    }
    tc_commit(bar_mma);   // also quiesces the MMA before TMEM is freed
    if (!ok) wait_phase(bar_ld, 0, ctl, true);   // the copies land before the CTA exits
  }
  __syncwarp();
  ok = __all_sync(0xffffffffu, wait_phase(bar_mma, 0, ctl, !ok ? true : false));
  if (ok && !*abort_flag) {
    tc_fence_after();
    const int64_t key = (int64_t)j * kBN + threadIdx.x;   // TMEM lane = key
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
    for (int g = 0; g < a.G; ++g) {
      float s[NB];
      tmem_ld_cols<NB>(tl + g * NB, s);
      tmem_wait_ld();
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < NB; ++i) acc += fast_exp2(fmaf(s[i], a.scale_log2, -sL[g * NB + i]));
      if (key < a.nkeys) a.mass[((int64_t)b * a.Hq + kvh * a.G + g) * a.nkeys + key] = acc;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128));
  }
}

// Top-k per (b, h) of mass [B*Hq, n] -> sel [B*Hq, k] ascending, ties to the
// lower index.
constexpr int kTopkThreads = 1024;
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* mass, int64_t n, int32_t k, int32_t* sel) {
  ptx::pdl_prologue();
  using Scan = cub::BlockScan<int, kTopkThreads>;
  __shared__ typename Scan::TempStorage scan_tmp;
  __shared__ int hist[256];
  __shared__ uint32_t s_prefix;
  __shared__ int s_remaining;
  const int64_t bh = blockIdx.x;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(mass + bh * n);
  int32_t* out = sel + bh * (int64_t)k;
  if (threadIdx.x == 0) {
    s_prefix = 0u;
    s_remaining = k;
  }
  // radix select of the k-th largest value, eight bits per pass, high first
  uint32_t mask = 0u;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    // every lane takes the same trip count, so the warp can aggregate equal
    // bins (masses share their leading bits) into one shared-memory atomic
    const int64_t n_round = (n + blockDim.x - 1) / blockDim.x * blockDim.x;
    for (int64_t x = threadIdx.x; x < n_round; x += blockDim.x) {
      uint32_t bin = 256u;   // no bin
      if (x < n) {
        const uint32_t v = bits[x];
        if ((v & mask) == prefix) bin = (v >> shift) & 255u;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin < 256u && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int rem = s_remaining, d = 255;
      for (; d > 0 && hist[d] < rem; --d) rem -= hist[d];
      s_remaining = rem;
      s_prefix = prefix | ((uint32_t)d << shift);
    }
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t thr = s_prefix;       // bits of the k-th largest value
  const int take_eq = s_remaining;     // keys equal to it that are kept (lowest index first)
  // keep, in key order: every key above thr and the first take_eq keys equal to it
  const int64_t chunk = (n + blockDim.x - 1) / blockDim.x;
  const int64_t x0 = threadIdx.x * chunk, x1 = min(n, x0 + chunk);
  int n_eq = 0;
  for (int64_t x = x0; x < x1; ++x) n_eq += bits[x] == thr;
  int eq_before;
  Scan(scan_tmp).ExclusiveSum(n_eq, eq_before);
  __syncthreads();
  int n_keep = 0, e = eq_before;
  for (int64_t x = x0; x < x1; ++x) {
    const uint32_t v = bits[x];
    if (v > thr || (v == thr && e++ < take_eq)) ++n_keep;
  }
  int pos;
  Scan(scan_tmp).ExclusiveSum(n_keep, pos);
  e = eq_before;
  for (int64_t x = x0; x < x1; ++x) {
    const uint32_t v = bits[x];
    if (v > thr || (v == thr && e++ < take_eq)) {
      if (pos < k) out[pos] = (int32_t)x;
      ++pos;
    }
  }
}

// ------------------------------------------------------------------ host --
int* device_status_ptr();
uint64_t wait_limit_ns();

namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn_sel() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

bool map4(CUtensorMap* m, const void* base, uint64_t d1, uint64_t d2, uint64_t d3, int64_t s1, int64_t s2, int64_t s3,
          uint32_t b1, uint32_t b2) {
  auto fn = encode_fn_sel();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)kD, d1, d2, d3};
  cuuint64_t strides[3] = {(cuuint64_t)s1 * 2, (cuuint64_t)s2 * 2, (cuuint64_t)s3 * 2};
  cuuint32_t box[4] = {64, b1, b2, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

bool mass_applies(const fb_attn_desc& d) {
  const int G = d.Hq / d.Hkv;
  return d.in_dtype == FB_BF16 && d.D == kD && (d.Nb == 16 || d.Nb == 32) && G * d.Nb <= kBN;
}

cudaError_t launch_mass(const fb_attn_desc& d, const void* q, const void* kp, int64_t nkeys, const float* l_out,
                        float* mass, float scale_log2, cudaStream_t s) {
  MassArgs a;
  memset(&a, 0, sizeof(a));
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.G = d.Hq / d.Hkv; a.Nb = d.Nb;
  a.nkeys = nkeys; a.scale_log2 = scale_log2; a.l_out = l_out; a.mass = mass;
  a.status = device_status_ptr();
  a.wait_limit_ns = wait_limit_ns();
  if (!a.status || !mass_applies(d) || nkeys <= 0) return cudaErrorInvalidValue;
  CUtensorMap mq, mk;
  if (!map4(&mq, q, d.Nb, d.Hq, d.B, d.q_strides[2], d.q_strides[1], d.q_strides[0], (uint32_t)d.Nb,
            (uint32_t)a.G) ||
      !map4(&mk, kp, nkeys, d.Hkv, d.B, d.kp_strides[2], d.kp_strides[1], d.kp_strides[0], kBN, 1))
    return cudaErrorInvalidValue;
  const dim3 grid((unsigned)((nkeys + kBN - 1) / kBN), (unsigned)(d.B * d.Hkv));
  auto run = [&](auto kern) -> cudaError_t {
    static bool attr[kMaxDevices][2] = {};
    const int slot = d.Nb == 16 ? 0 : 1;
    bool& done = attr[current_device()][slot];
    if (!done) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e != cudaSuccess) return e;
      done = true;
    }
    return launch_k(kern, grid, dim3(128), kSmemBytes, s, mq, mk, a);
  };
  return d.Nb == 16 ? run(mass_kernel<16>) : run(mass_kernel<32>);
}

cudaError_t launch_topk(const float* mass, int32_t BH, int64_t n, int32_t k, int32_t* sel, cudaStream_t s) {
  if (k <= 0) return cudaSuccess;
  return launch_k(topk_kernel, dim3((unsigned)BH), dim3(kTopkThreads), 0, s, mass, n, k, sel);
}

}  // namespace fb
