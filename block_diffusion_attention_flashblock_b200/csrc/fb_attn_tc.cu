// Block-external attention on the fifth-generation tensor cores (sm_100a):
// the FlashBlock prefix pass, A_out with L_out = log Z_out over the prefix KV
// cache (FlashBlock summary, "Mécanisme Central"), for bf16 inputs, D = 128.
//
// One CTA = one tile of 128 query rows (the block queries of the query heads
// that share a KV head, packed) x one split of the prefix keys.  Warp roles:
//   warp 0      TMA producer, no multicast: Q once, then K tiles of 128 keys
//               into a three-stage ring (128-byte swizzle).
//   warp 11     TMA producer of the V tiles, its own three-stage ring (a warp
//               of its own, so a wait on one ring never stalls the other).
//   warp 1      allocates TMEM; one thread issues S = Q K^T (tcgen05.mma, A
//               and B in shared memory) into one of three TMEM S buffers.
//   warp 10     one thread issues O += P_hi V + P_lo V with P read from TMEM.
//               Two issuing threads on different SM sub-partitions keep the
//               tensor core fed while each waits on its own barriers.
//   warps 2..9  softmax, two threads per query row (TMEM lane = row): warps
//               w and w+4 share a TMEM lane quarter and take columns 0..63 and
//               64..127 of S; they trade their row maxima (and at the end
//               their row sums) through shared memory and a bounded
//               mbarrier.  Each writes its half of P = 2^(s - m), as bf16 hi
//               and lo parts, back over the 64 TMEM columns its half of S
//               came from; the final O / l and L are staged in shared memory
//               and leave as whole rows (512 contiguous bytes per warp store).
//               A sparse pass masks keys by a per-head bitmap before the max.
// P lives in the S buffer it replaces, so S_{j+3} is only issued once PV_j
// has completed (a completion barrier per buffer); three buffers leave two
// softmax tiles for the chain P_j -> PV_j -> S_{j+3}.
// The running max is only moved (and O rescaled in TMEM) when a row's max
// grows by more than 2^8, so P stays <= 256 and most tiles skip the rescale.
// With a cluster launch, each cluster of key splits of one row tile reduces
// its parts through distributed shared memory before anything reaches global
// memory (one part per cluster): every rank sends each other rank the rows
// that rank owns with one bulk shared-to-shared copy, and each owner merges
// its rows.  The last split also takes the ragged remainder of the keys.
// Every mbarrier wait is bounded; on expiry the CTA records FB_ETIMEOUT in
// the device status word, drains its own TMA and MMA work, frees TMEM and
// exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <algorithm>

#include "fb_internal.cuh"
#include "fb_ptx.cuh"
#include "fb_tc.cuh"

namespace fb {

namespace {

constexpr int kBM = 128, kBN = 128, kD = 128;
constexpr int kThreads = 384;
constexpr int kStages = 3;                        // K and V ring depth
constexpr uint32_t kHalf = 16384;                 // [128 rows][64 bf16] 128B-swizzled block
constexpr uint32_t kTile = 2 * kHalf;             // one 128 x 128 bf16 tile
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTile;
constexpr uint32_t kOffV = kOffK + kStages * kTile;
constexpr uint32_t kOffBar = kOffV + kStages * kTile;   // barriers and flags (256 bytes)
constexpr uint32_t kOffX = kOffBar + 256;               // row-statistics exchange, 2 x 2 x 128 fp32
constexpr uint32_t kSmemSlack = 768;                    // the aligned base may sit up to this far in
constexpr uint32_t kSmemBytes = kOffX + 2048 + kSmemSlack;
constexpr int kSBuf = 3;                          // S/P buffers in TMEM
constexpr uint32_t kTmemCols = 512;               // S/P buffers [0,128) [128,256) [256,384), O [384,512)
constexpr uint32_t kTmemO = 384;
constexpr float kRescaleLog2 = 8.0f;

// barrier slots
enum {
  B_QFULL = 0, B_KFULL = 1, B_KEMPTY = 4, B_VFULL = 7, B_VEMPTY = 10, B_SFULL = 13, B_PFULL = 16,
  B_PVDONE = 19, B_DRAIN = 22, B_PAIR = 24, B_RECV = 28, B_STALL = 29, B_COUNT = 30
};

using namespace tc;

// Thread-block cluster helpers (split-KV reduction through distributed shared memory).
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\nbarrier.cluster.wait.acquire;\n" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// Bulk copy of `bytes` (a multiple of 16) from this CTA's shared memory into
// another cluster rank's, completing on that rank's mbarrier (no multicast).
__device__ __forceinline__ void bulk_to_rank(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                             uint32_t bar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(src), "r"(bytes), "r"(bar_cluster)
               : "memory");
}
using ptx::fence_proxy_async_smem;
// Epilogue staging, inside the idle K/V rings: this CTA's normalised rows
// [128][kRedStride] fp32 (columns 0..127 = O, column 128 = L), then, with a
// cluster launch, the rows this rank owns as received from every rank
// [ranks x rows per rank <= 143][kRedStride].
constexpr int kRedStride = 132;
constexpr uint32_t kRowBytes = kRedStride * 4u;   // 528, a multiple of 16
constexpr uint32_t kRecvOff = 128u * kRowBytes;
static_assert(kRecvOff + 144u * kRowBytes <= 2u * 3u * 32768u, "epilogue staging must fit in the K/V rings");

// This thread's 64 output columns (a half row of O in TMEM, zero when the
// split had no keys), scaled by inv, handed to put(float4 index, value).
template <class F>
__device__ __forceinline__ void load_o_scaled(uint32_t tl, int half, int T, float inv, F&& put) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    float o[32];
    if (T > 0) {
      tmem_ld32(tl + kTmemO + half * 64 + c * 32, o);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < 32; e += 4)
      put((c * 32 + e) / 4, make_float4(o[e] * inv, o[e + 1] * inv, o[e + 2] * inv, o[e + 3] * inv));
  }
}

}  // namespace

struct TcArgs {
  int32_t B, Hq, Hkv, G, Nb;
  int32_t mode;            // 0: unit (b, kv head), tile = hg heads x Nb queries; 1: unit (b, q head), 128 queries
  int32_t hg;
  int32_t tiles_per_unit;
  int64_t nkeys;
  int64_t keys_per_split;
  float scale_log2;
  float* part_a;
  float* part_l;
  int64_t part_stride_a, part_stride_l;
  const int8_t* mask;
  int32_t mask_active;
  int* status;
  uint64_t wait_limit_ns;
  uint32_t q_bytes;        // bytes of one Q half-box (64 columns)
  int32_t cluster;         // > 1: clusters of this many consecutive splits reduce in-kernel
  const uint32_t* excl;    // non-null: per (b, query head) key bitmap (sparse passes)
  int64_t excl_words;
  int32_t excl_invert;     // 0: a set bit excludes the key (residual pass); 1: a clear bit does (selected-keys pass)
  int32_t stall;           // test hook: the S issuer first waits on a barrier nothing completes
};

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
  ptx::pdl_prologue();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (smem - smem_raw > (ptrdiff_t)kSmemSlack) {   // the layout would not fit: report, touch nothing
    if (threadIdx.x == 0) atomicCAS(a.status, 0, (int)FB_EUNSUPPORTED);
    return;
  }
  const uint32_t sbase = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + B_COUNT * 8);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + B_COUNT * 8 + 4);
  auto bar = [&](int i) { return smem_addr(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile_id = blockIdx.x, split = blockIdx.y;
  const int unit = tile_id / a.tiles_per_unit, t = tile_id % a.tiles_per_unit;
  int b, kvh, h0, i0;
  if (a.mode == 0) {
    b = unit / a.Hkv; kvh = unit % a.Hkv; h0 = kvh * a.G + t * a.hg; i0 = 0;
  } else {
    b = unit / a.Hq; h0 = unit % a.Hq; kvh = h0 / a.G; i0 = t * kBM;
  }
  // gamma gate: skip the tile when every query head in it reuses its cache
  if (a.mask_active) {
    const int hn = a.mode == 0 ? min(a.hg, a.G - t * a.hg) : 1;
    bool all = true;
    for (int h = h0; h < h0 + hn; ++h) all = all && a.mask[b * a.Hq + h];
    if (all) return;
  }
  // The tile's rows [0, nrows) exist and are the consecutive rows
  // [rbase, rbase + nrows) of the packed (b, h, i) part layout.
  int64_t rbase;
  int nrows;
  if (a.mode == 0) {
    rbase = ((int64_t)b * a.Hq + (int64_t)kvh * a.G + (int64_t)t * a.hg) * a.Nb;
    nrows = min(a.hg, a.G - t * a.hg) * a.Nb;
  } else {
    rbase = ((int64_t)b * a.Hq + h0) * a.Nb + i0;
    nrows = min(kBM, a.Nb - i0);
  }
  if (warp == 1 && lane == 1) {
    // warm the address translation of the part rows this CTA writes at the end
    const int part = a.cluster > 1 ? split / a.cluster : split;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a.part_a + part * a.part_stride_a + rbase * kD));
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a.part_l + part * a.part_stride_l + rbase));
  }
  const int64_t kbeg = (int64_t)split * a.keys_per_split;
  const int64_t kend = split == (int)gridDim.y - 1 ? a.nkeys : min(kbeg + a.keys_per_split, a.nkeys);
  const int T = kend > kbeg ? (int)((kend - kbeg + kBN - 1) / kBN) : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i >= B_PFULL && i < B_PFULL + kSBuf) cnt = 256;
      if (i >= B_PAIR && i < B_PAIR + 4) cnt = 64;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Ctl ctl{abort_flag, a.status, a.wait_limit_ns};

  if (warp == 0 || warp == 11) {
    // ------------------------------------------------------------ producers
    if (lane == 0 && T > 0) {
      // warp 0: Q, then the K ring; warp 11: the V ring
      const bool is_k = warp == 0;
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(is_k ? &tmK : &tmV)) : "memory");
      if (is_k) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      const int full = is_k ? B_KFULL : B_VFULL, empty = is_k ? B_KEMPTY : B_VEMPTY;
      const uint32_t ring = sbase + (is_k ? kOffK : kOffV);
      int armed[kStages] = {-1, -1, -1};
      bool ok = true;
      if (is_k) {
        mbar_expect_tx(bar(B_QFULL), 2 * a.q_bytes);
        tma_load_4d(sbase + kOffQ, &tmQ, bar(B_QFULL), 0, i0, h0, b);
        tma_load_4d(sbase + kOffQ + kHalf, &tmQ, bar(B_QFULL), 64, i0, h0, b);
      }
      for (int j = 0; j < T && ok; ++j) {
        const int st = j % kStages, round = j / kStages;
        if (j >= kStages) ok = wait_phase(bar(empty + st), (round - 1) & 1, ctl);
        if (!ok) break;
        const int key0 = (int)(kbeg + (int64_t)j * kBN);
        mbar_expect_tx(bar(full + st), kTile);
        tma_load_4d(ring + st * kTile, tm, bar(full + st), 0, key0, kvh, b);
        tma_load_4d(ring + st * kTile + kHalf, tm, bar(full + st), 64, key0, kvh, b);
        armed[st] = round;
      }
      // Let every copy this thread started land before the CTA can exit.
      if (is_k) wait_phase(bar(B_QFULL), 0, ctl, true);
      for (int st = 0; st < kStages; ++st)
        if (armed[st] >= 0) wait_phase(bar(full + st), armed[st] & 1, ctl, true);
    }
  } else if (warp == 1 || warp == 10) {
    // ------------------------------------------------------------ MMA issuers
    // Descriptors are built once; a shared-memory offset moves the start
    // address field (bits 0..13, in 16-byte units), so each MMA only adds a
    // constant (the whole CTA's shared memory stays below 2^18 bytes).
    if (lane == 0 && T > 0 && warp == 1) {
      // S_j = Q K_j^T into buffer j % 3, once K_j has landed and PV_{j-3} has
      // finished reading the P that buffer held
      const uint64_t dQ = sw128_desc(sbase + kOffQ, 16, 1024);
      const uint64_t dK = sw128_desc(sbase + kOffK, 16, 1024);
      bool ok = !a.stall || wait_phase(bar(B_STALL), 0, ctl);
      ok = ok && wait_phase(bar(B_QFULL), 0, ctl);
      for (int j = 0; j < T && ok; ++j) {
        const int sb = j % kSBuf, st = j % kStages;
        ok = wait_phase(bar(B_KFULL + st), (j / kStages) & 1, ctl);
        if (ok && j >= kSBuf) ok = wait_phase(bar(B_PVDONE + sb), (j / kSBuf - 1) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dKs = dK + (uint64_t)((st * kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
          tc_mma(tmem + sb * kBN, dQ + off, dKs + off, kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_SFULL + sb));
        tc_commit(bar(B_KEMPTY + st));
      }
      // quiesce this thread's tensor-core work before TMEM is freed
      tc_commit(bar(B_DRAIN));
      wait_phase(bar(B_DRAIN), 0, ctl, true);
    }
    if (lane == 0 && T > 0 && warp == 10) {
      // O += P_j V_j (hi then lo) once softmax has written P_j and V_j landed
      const uint64_t dV = sw128_desc(sbase + kOffV, kHalf, 1024);
      bool ok = true;
      for (int j = 0; j < T && ok; ++j) {
        const int sb = j % kSBuf, st = j % kStages;
        ok = wait_phase(bar(B_PFULL + sb), (j / kSBuf) & 1, ctl);
        if (ok) ok = wait_phase(bar(B_VFULL + st), (j / kStages) & 1, ctl);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dVs = dV + (uint64_t)((st * kTile) >> 4);
        const uint32_t pt = tmem + sb * kBN;
#pragma unroll
        for (int part = 0; part < 2; ++part)   // P_hi, then P_lo (keys 64h.. at 64h + 32 part + 8 (kk & 3))
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            tc_mma_ts(tmem + kTmemO, pt + (kk >> 2) * 64 + part * 32 + (kk & 3) * 8,
                      dVs + (uint64_t)((kk * 2048) >> 4), kIdescPV, (j > 0 || part > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_VEMPTY + st));
        tc_commit(bar(B_PVDONE + sb));
      }
      tc_commit(bar(B_DRAIN + 1));
      wait_phase(bar(B_DRAIN + 1), 0, ctl, true);
    }
  } else if (warp >= 2 && warp <= 9) {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int half = (warp - 2) >> 2;          // 0: columns 0..63, 1: columns 64..127
    const int row = q4 * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t pair = bar(B_PAIR + q4);
    float* xch = reinterpret_cast<float*>(smem + kOffX);   // [slot][half][row]
    float m = -CUDART_INF_F, l = 0.f;
    bool ok = true;
    // tcgen05.ld/st are warp-collective: every branch around them is warp-uniform.
    auto uniform = [](bool v) { return __all_sync(0xffffffffu, v); };
    // Trade one value per row with the partner warp through shared memory
    // slot `slot` (phase `ph` of this lane quarter's pair barrier; the barrier
    // arrive/wait orders the store before the partner's load).
    auto trade = [&](float mine, int slot, int ph, float& theirs) -> bool {
      xch[(slot * 2 + half) * kBM + row] = mine;
      mbar_arrive(pair);
      if (!uniform(wait_phase(pair, ph & 1, ctl))) return false;
      theirs = xch[(slot * 2 + (half ^ 1)) * kBM + row];
      return true;
    };
    // sparse residual pass: this row's bitmap of excluded keys (a padding row
    // reads the tile's last real row, whose result is discarded)
    const uint32_t* exrow = nullptr;
    if (a.excl) {
      const int rr = min(row, nrows - 1);
      const int hh = a.mode == 0 ? kvh * a.G + t * a.hg + rr / a.Nb : h0;
      exrow = a.excl + ((int64_t)b * a.Hq + hh) * a.excl_words;
    }
    for (int j = 0; j < T && ok; ++j) {
      const int sb = j % kSBuf;
      const int64_t key0 = kbeg + (int64_t)j * kBN;
      uint32_t ex0 = 0u, ex1 = 0u;   // exclusion bits of this thread's 64 keys, loaded before the wait
      if (exrow) {
        const int64_t w0 = (key0 + half * 64) >> 5;
        if (w0 < a.excl_words) ex0 = __ldg(exrow + w0);
        if (w0 + 1 < a.excl_words) ex1 = __ldg(exrow + w0 + 1);
        if (a.excl_invert) {
          ex0 = ~ex0;
          ex1 = ~ex1;
        }
      }
      ok = uniform(wait_phase(bar(B_SFULL + sb), (j / kSBuf) & 1, ctl));
      if (!ok) break;
      tc_fence_after();
      // this thread's 64 scores, ragged tail and excluded keys masked to -inf
      float s[64];
      const int nvalid = (int)min((int64_t)kBN, kend - key0) - half * 64;
      auto load_s = [&]() {
        tmem_ld32(tl + sb * kBN + half * 64, s);
        tmem_ld32(tl + sb * kBN + half * 64 + 32, s + 32);
        tmem_wait_ld();
        if (nvalid < 64) {   // only the last tile of the last split is ragged
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= nvalid) s[c] = -CUDART_INF_F;
        }
        if (exrow) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (((c < 32 ? ex0 : ex1) >> (c & 31)) & 1u) s[c] = -CUDART_INF_F;
        }
      };
      // p = 2^(s * scale - ref) in place: one FFMA and one MUFU op per score,
      // 8 sum chains
      auto exp_pass = [&](float ref) -> float {
        const float nref = (ref == -CUDART_INF_F) ? 0.f : -ref;
        float sm8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          s[c] = fast_exp2(fmaf(s[c], a.scale_log2, nref));
          sm8[c & 7] += s[c];
        }
        return ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
      };
      load_s();
      // Half-row max of the raw scores (scale > 0 keeps the order).  Once the
      // row has a reference max m, P is formed against it in the same pass
      // (the common case: the tile's max stays within m + 2^8); the row's
      // first tile takes the max first.  The partner's half is traded either
      // way, so both threads of a row see the same max.
      const bool two_pass = __any_sync(0xffffffffu, m == -CUDART_INF_F);
      float mx8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx8[e] = -CUDART_INF_F;
      float psum = 0.f;
      if (two_pass) {
#pragma unroll
        for (int c = 0; c < 64; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
      } else {
        const float nref = -m;
        float sm8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          mx8[c & 7] = fmaxf(mx8[c & 7], s[c]);
          s[c] = fast_exp2(fmaf(s[c], a.scale_log2, nref));
          sm8[c & 7] += s[c];
        }
        psum = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) + ((sm8[4] + sm8[5]) + (sm8[6] + sm8[7]));
      }
      float tmax =
          fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])), fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) *
          a.scale_log2;
      float other;
      ok = trade(tmax, j & 1, j, other);
      if (!ok) break;
      tmax = fmaxf(tmax, other);
      // Move this row's reference max when it grew by more than 2^8; rows whose
      // O already holds values rescale their half of it (alpha = 1 otherwise).
      const bool move = tmax > m + kRescaleLog2;
      const bool scale_o = move && j > 0 && m != -CUDART_INF_F;
      const float alpha = scale_o ? fast_exp2(m - tmax) : 1.f;
      if (__any_sync(0xffffffffu, scale_o)) {
        ok = uniform(wait_phase(bar(B_PVDONE + (j - 1) % kSBuf), ((j - 1) / kSBuf) & 1, ctl));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float o[32];
          tmem_ld32(tl + kTmemO + half * 64 + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tl + kTmemO + half * 64 + c * 32, o);
        }
        tmem_wait_st();
      }
      if (move) {
        l *= alpha;
        m = tmax;
      }
      // P again from the scores (still in TMEM: each half writes P only over
      // its own columns) when a row of the warp moved its reference, or on
      // the first tile
      if (two_pass || __any_sync(0xffffffffu, move)) {
        if (!two_pass) load_s();
        psum = exp_pass(m);
      }
      l += psum;
      // P (bf16 pairs, lower key in the low half) over this half's own S
      // columns: hi parts at half*64 + [0, 32), lo parts at half*64 + [32, 64).
      uint32_t hi[32], lo[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) split_pair(s[2 * e], s[2 * e + 1], hi[e], lo[e]);
      tmem_st32u(tl + sb * kBN + half * 64, hi);
      tmem_st32u(tl + sb * kBN + half * 64 + 32, lo);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL + sb));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && T > 0) ok = uniform(wait_phase(bar(B_PVDONE + (T - 1) % kSBuf), ((T - 1) / kSBuf) & 1, ctl));
    float lo_other = 0.f;
    if (ok) ok = trade(l, T & 1, T, lo_other);   // the row sum is the two halves' sum
    if (ok) {
      l += lo_other;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float Lrow = l > 0.f ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
      // stage the normalised row and its L in this CTA's shared memory (the
      // K/V rings are idle now)
      tc_fence_after();
      float* st = reinterpret_cast<float*>(smem + kOffK) + row * kRedStride;
      load_o_scaled(tl, half, T, inv,
                    [&](int c, float4 v) { *reinterpret_cast<float4*>(st + half * 64 + c * 4) = v; });
      if (half == 0) st[128] = Lrow;
      fence_proxy_async_smem();   // the rows may leave by bulk copy
    }
  }

  const int CS = a.cluster;
  const int R = (kBM + CS - 1) / CS;   // rows owned by each cluster rank
  const int rank = CS > 1 ? (int)cluster_rank() : 0;
  const int own = CS > 1 ? max(0, min(R, kBM - rank * R)) : 0;
  if (CS > 1 && threadIdx.x == 0) mbar_expect_tx(bar(B_RECV), (uint32_t)(CS * own) * kRowBytes);
  tc_fence_before();
  __syncthreads();
  const int nwarps = kThreads / 32;
  const float* stage = reinterpret_cast<const float*>(smem + kOffK);
  if (CS <= 1) {
    // The tile's rows are one contiguous range of the part: every thread
    // copies up to 11 of its 16-byte pieces, all loads before all stores, a
    // warp covering 512 contiguous bytes per store instruction.
    constexpr int kPieces = (kBM * 32 + kThreads - 1) / kThreads;
    float* dst = a.part_a + split * a.part_stride_a + rbase * kD;
    float4 v[kPieces];
#pragma unroll
    for (int k = 0; k < kPieces; ++k) {
      const int idx = threadIdx.x + k * kThreads, rr = idx >> 5;
      if (rr < nrows) v[k] = *reinterpret_cast<const float4*>(stage + rr * kRedStride + (idx & 31) * 4);
    }
#pragma unroll
    for (int k = 0; k < kPieces; ++k) {
      const int idx = threadIdx.x + k * kThreads, rr = idx >> 5;
      if (rr < nrows) *reinterpret_cast<float4*>(dst + (size_t)idx * 4) = v[k];
    }
    if ((int)threadIdx.x < nrows) a.part_l[split * a.part_stride_l + rbase + threadIdx.x] = stage[threadIdx.x * kRedStride + 128];
  } else {
    // Split-KV reduction over the cluster.  Rank c owns rows [c*R, c*R + R).
    // Once every rank is past its main loop, each rank sends each owner that
    // owner's block of its staged rows with one bulk copy into the owner's
    // receive area (slot p*R + i for rank p's row c*R + i), completing on
    // the owner's receive barrier; the owner merges its rows in log space,
    // ranks in fixed order, and writes the cluster's part.
    cluster_sync_all();
    if (threadIdx.x == 0) {
      for (int o = 0; o < CS; ++o) {
        const int n = max(0, min(R, kBM - o * R));
        if (n == 0) continue;
        bulk_to_rank(map_rank(sbase + kOffK + kRecvOff + (uint32_t)(rank * R) * kRowBytes, (uint32_t)o),
                     sbase + kOffK + (uint32_t)(o * R) * kRowBytes, (uint32_t)n * kRowBytes,
                     map_rank(bar(B_RECV), (uint32_t)o));
      }
    }
    // waited on even after a failure elsewhere in this CTA (draining), so no copy
    // into this CTA is still in flight when it exits
    if (wait_phase(bar(B_RECV), 0, ctl, true)) {
      const float* recv = reinterpret_cast<const float*>(smem + kOffK + kRecvOff);
      const int own_valid = min(own, nrows - rank * R);
#pragma unroll 2
      for (int rl = warp; rl < own_valid; rl += nwarps) {
        const int64_t r = rbase + rank * R + rl;
        float m = -CUDART_INF_F;
#pragma unroll 1
        for (int p = 0; p < CS; ++p) m = fmaxf(m, recv[(p * R + rl) * kRedStride + 128]);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float wsum = 0.f;
#pragma unroll 1
        for (int p = 0; p < CS; ++p) {
          const float* rowp = recv + (p * R + rl) * kRedStride;
          const float Lp = rowp[128];
          if (Lp == -CUDART_INF_F) continue;
          const float w = __expf(Lp - m);
          const float4 v = *reinterpret_cast<const float4*>(rowp + lane * 4);
          wsum += w;
          acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
          acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
        }
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        const int part = split / CS;
        *reinterpret_cast<float4*>(a.part_a + part * a.part_stride_a + r * kD + lane * 4) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        if (lane == 0) a.part_l[part * a.part_stride_l + r] = m == -CUDART_INF_F ? -CUDART_INF_F : m + __logf(wsum);
      }
    }
    cluster_sync_all();   // every copy out of this CTA's staging has landed
  }
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ------------------------------------------------------------------ host --
namespace {
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

bool map_4d(CUtensorMap* m, const void* base, uint64_t d1, uint64_t d2, uint64_t d3, int64_t s1, int64_t s2,
            int64_t s3, uint32_t b1, uint32_t b2) {
  auto fn = encode_fn();
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

int* device_status_ptr();
uint64_t wait_limit_ns();

// Row tiling of the tcgen05 prefix pass, or false when the shape does not fit it.
bool tc_tiling(const fb_attn_desc& d, int* mode, int* hg, int* tiles_per_unit, int* units) {
  if (d.in_dtype != FB_BF16 || d.D != kD) return false;
  const int G = d.Hq / d.Hkv;
  if (d.Nb <= kBM && kBM % d.Nb == 0 && G * d.Nb >= 64) {
    *mode = 0;
    *hg = std::min(G, kBM / d.Nb);
    *tiles_per_unit = (G + *hg - 1) / *hg;
    *units = d.B * d.Hkv;
    return true;
  }
  if (d.Nb >= 64) {
    *mode = 1;
    *hg = 1;
    *tiles_per_unit = (d.Nb + kBM - 1) / kBM;
    *units = d.B * d.Hq;
    return true;
  }
  return false;
}

bool tc_make_maps(const fb_attn_desc& d, const void* q, const void* k, const void* v, int64_t nkeys,
                  const int64_t* kstr, TcMaps* m) {
  if (nkeys <= 0 || !tc_tiling(d, &m->mode, &m->hg, &m->tiles_per_unit, &m->units)) return false;
  const uint32_t qrows = m->mode == 0 ? (uint32_t)d.Nb : (uint32_t)kBM;
  const uint32_t qheads = m->mode == 0 ? (uint32_t)m->hg : 1u;
  return map_4d(&m->q, q, d.Nb, d.Hq, d.B, d.q_strides[2], d.q_strides[1], d.q_strides[0], qrows, qheads) &&
         map_4d(&m->k, k, nkeys, d.Hkv, d.B, kstr[2], kstr[1], kstr[0], kBN, 1) &&
         map_4d(&m->v, v, nkeys, d.Hkv, d.B, kstr[2], kstr[1], kstr[0], kBN, 1);
}

// Upper bound of the split count the planner may choose (sizes workspaces).
int32_t tc_split_cap(int64_t tiles, int64_t max_keys) {
  const int64_t ktiles = std::max<int64_t>(1, (max_keys + kBN - 1) / kBN);
  const int64_t want = std::max<int64_t>(2, (4 * (int64_t)num_sms() + tiles - 1) / std::max<int64_t>(tiles, 1));
  return (int32_t)std::min(ktiles, want);
}

// Largest number of clusters of `cs` CTAs that can run at once (0: not launchable).
static int max_active_clusters(int cs) {
  static int cache[64][17];
  static bool init[64][17];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64 || cs < 2 || cs > 16) return 0;
  if (init[dev][cs]) return cache[dev][cs];
  int n = 0;
  if (cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) == cudaSuccess &&
      (cs <= 8 || cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                      cudaSuccess)) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, cs, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = cs;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, (void*)attn_tc_kernel, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cache[dev][cs] = n;
  init[dev][cs] = true;
  return n;
}

// Split plan for `tiles` row tiles over nkeys keys: nsplit splits of kps keys
// (the last one takes the rest), grouped into clusters of `cluster` splits
// that reduce in-kernel (1: no cluster), leaving nparts parts per row for a
// later merge.  Candidates are scored as waves of concurrently resident CTAs
// (or clusters) x (the longest split in key tiles + a fixed cost of about two
// tiles), plus a small cost per extra part; nparts is at most max_parts.
void tc_plan_split(int64_t tiles, int64_t nkeys, int32_t max_parts, bool allow_cluster, int32_t* nsplit,
                   int64_t* kps, int32_t* cluster, int32_t* nparts, double cluster_cost) {
  const int64_t sms = num_sms();
  const int64_t ktiles = std::max<int64_t>(1, (nkeys + kBN - 1) / kBN);
  double best = 1e300;
  int64_t b_ns = 1, b_cs = 1, b_per = ktiles;
  for (int cs = 1; cs <= (allow_cluster ? 16 : 1); ++cs) {
    const int64_t conc = cs == 1 ? sms : (int64_t)max_active_clusters(cs);
    if (conc <= 0) continue;
    for (int64_t nc = 1; nc * cs <= ktiles; ++nc) {
      const int64_t ns = nc * cs;
      const int64_t parts = cs == 1 ? ns : nc;
      if (parts > std::max(1, max_parts)) break;
      const int64_t per = ktiles / ns, last = ktiles - (ns - 1) * per;
      const int64_t units = cs == 1 ? tiles * ns : tiles * nc;
      const int64_t waves = (units + conc - 1) / conc;
      // a cluster's in-kernel reduction (two cluster barriers and the
      // shared-to-shared copies) costs cluster_cost key tiles per CTA
      const double cost = (double)waves * (last + 2 + (cs > 1 ? cluster_cost : 0.0)) +
                          (parts > 1 ? 1.5 + 0.1 * parts : 0.0) + 0.01 * ns;
      if (cost < best) { best = cost; b_ns = ns; b_cs = cs; b_per = per; }
    }
  }
  *nsplit = (int32_t)b_ns;
  *kps = b_per * kBN;
  *cluster = (int32_t)b_cs;
  *nparts = (int32_t)(b_cs == 1 ? b_ns : b_ns / b_cs);
}

cudaError_t launch_attn_tc(const fb_attn_desc& d, const TcMaps& m, int64_t nkeys, int32_t nsplit, int64_t kps,
                           int32_t cluster, const int8_t* mask, int mask_active, float scale_log2, float* pa,
                           float* pl, cudaStream_t s, const uint32_t* excl, int64_t excl_words,
                           bool excl_invert) {
  TcArgs a;
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.G = d.Hq / d.Hkv; a.Nb = d.Nb;
  a.mode = m.mode; a.hg = m.hg; a.tiles_per_unit = m.tiles_per_unit;
  a.nkeys = nkeys; a.keys_per_split = kps; a.scale_log2 = scale_log2;
  a.part_a = pa; a.part_l = pl;
  a.part_stride_a = (int64_t)d.B * d.Hq * d.Nb * d.D;
  a.part_stride_l = (int64_t)d.B * d.Hq * d.Nb;
  a.mask = mask; a.mask_active = mask_active;
  a.q_bytes = 64u * 2u * (uint32_t)(m.mode == 0 ? d.Nb * m.hg : kBM);
  a.status = device_status_ptr();
  a.wait_limit_ns = wait_limit_ns();
  a.cluster = cluster > 1 ? cluster : 1;
  a.excl = excl;
  a.excl_words = excl_words;
  a.excl_invert = excl_invert ? 1 : 0;
  a.stall = debug_stall() ? 1 : 0;
  if (!a.status) return cudaErrorInvalidValue;
  static bool attr[kMaxDevices] = {};   // the attribute is per device
  bool& done = attr[current_device()];
  if (!done) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    done = true;
  }
  dim3 grid(m.units * m.tiles_per_unit, nsplit);
  if (a.cluster <= 1) return launch_k(attn_tc_kernel, grid, dim3(kThreads), kSmemBytes, s, m.q, m.k, m.v, a);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 1;
  at[0].val.clusterDim.y = (unsigned)cluster;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel, m.q, m.k, m.v, a);
}

}  // namespace fb
