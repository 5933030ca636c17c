// Block-external attention on the fifth-generation tensor cores (sm_100a), two
// query tiles per CTA: the FlashBlock prefix pass, A_out with L_out = log Z_out
// over the prefix KV cache (FlashBlock summary, "Mécanisme Central"), for bf16
// inputs, D = 128, wherever a KV head has two or more 128-row query tiles
// (long-context diffusion-LM blocks, video frame blocks).
//
// Work decomposition.  The query tiles of one KV head are paired; a pair and
// one key tile of 128 keys is one work item.  The grid is persistent (at most
// one CTA per SM) and stream-K: CTA c takes the items [c*T/C, (c+1)*T/C) of
// the T = pairs x key-tiles items, so every CTA gets the same number of key
// tiles whatever the shape.  A CTA's range splits into segments, one per pair
// it touches; each segment leaves a partial (A, L) of its pair's rows in the
// pair's slot (the index of the CTA among those touching the pair), or the
// final result when one CTA covers the whole pair, and a small merge kernel
// combines the slots in log space.  With the gamma gate, pairs whose heads
// all reuse their cache are left out of the item space on the device.
//
// Warp roles (384 threads; the softmax warpgroups run with 192 registers a
// thread, the other warps with 120):
//   warps 0..3  softmax of query tile 0 (slot 0), one thread per query row
//   warps 4..7  softmax of query tile 1 (slot 1)
//   warp 8      TMA producer, no multicast: the pair's Q tiles, then K and V
//               tiles of 128 keys into a two-stage K ring and a three-stage
//               V ring (128-byte swizzle)
//   warp 9      allocates TMEM; one thread issues every tcgen05.mma
//   warps 10,11 convert each landed V tile to fp16 in place where that is
//               exact (see the converter below), so P V runs in one pass
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).  Softmax s
// reads its row of S_s and writes P = 2^(s - m) over the same columns: as
// fp16 (columns 0..63) where V_j is fp16, and the issuer runs O_s += P V in
// one pass; else as bf16 hi (columns 0..63) and lo (64..127) parts, and the
// issuer runs O_s += P_hi V + P_lo V.  The scaling of the scores and the row
// sums take two lanes per instruction (f32x2), the exponentials the MUFU
// unit; V_j's format is read before S_j lands, off the softmax's critical
// path.  The issuer orders the tensor core as
//   S0(j) S1(j) | PV0(j) S0(j+1) PV1(j) S1(j+1) | PV0(j+1) ...
// so while one softmax group works on its tile the tensor core runs the other
// group's P V and next S.  S_s(j+1) overwrites P_s(j) only after PV_s(j) has
// read it: tcgen05.mma operations issued by one thread execute in order.
// The running max moves only when a row's max grows by more than 2^8 (O is
// then rescaled in TMEM by its own thread; the previous P V of that slot has
// completed, since S_s(j) completed after it).  Every mbarrier wait is
// bounded; on expiry the CTA records FB_ETIMEOUT, drains its own copies and
// MMAs, frees TMEM and exits.
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

constexpr int kBM = 128, kBN = 128, kD = 128;
constexpr int kThreads = 384;                    // three warpgroups
// Register split (setmaxnreg): the launch gives every thread kRegsLaunch;
// the producer / MMA warpgroup drops to kRegsIO and the two softmax
// warpgroups, which hold a row's 128 scores, rise to kRegsSoftmax.  The
// shares add up to the launch's allocation exactly; the host checks the
// kernel's launch register count before the first launch.
constexpr int kRegsLaunch = 168, kRegsIO = 120, kRegsSoftmax = 192;
static_assert(4 * 32 * kRegsIO + 8 * 32 * kRegsSoftmax == kThreads * kRegsLaunch, "register split");
constexpr int kKSt = 2, kVSt = 3;                 // K and V ring depths (V is converted after it lands)
constexpr uint32_t kHalf = 16384;                 // [128 rows][64 bf16], 128-byte swizzle
constexpr uint32_t kTile = 2 * kHalf;             // one 128 x 128 bf16 tile
constexpr uint32_t kOffQ = 0;                     // Q0, Q1
constexpr uint32_t kOffK = 2 * kTile;
constexpr uint32_t kOffV = kOffK + kKSt * kTile;
constexpr uint32_t kOffBar = kOffV + kVSt * kTile;
constexpr uint32_t kBarBytes = 384;               // barriers and control words
constexpr uint32_t kOffSeg = kOffBar + kBarBytes;  // segment list
constexpr int kMaxSeg = 32;
constexpr uint32_t kOffAct = kOffSeg + kMaxSeg * 16;   // active-pair bitmap
constexpr int kMaxPairs = 2048;
constexpr uint32_t kSmemSlack = 1024;
constexpr uint32_t kSmemBytes = kOffAct + kMaxPairs / 8 + kSmemSlack;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;
constexpr float kRescaleLog2 = 8.0f;

// barrier slots, laid out from the ring depths
enum {
  B_QFULL = 0,
  B_QEMPTY = 1,
  B_KFULL = 2,
  B_KEMPTY = B_KFULL + kKSt,
  B_VFULL = B_KEMPTY + kKSt,
  B_VEMPTY = B_VFULL + kVSt,
  B_VCONV = B_VEMPTY + kVSt,
  B_SFULL = B_VCONV + kVSt,
  B_PFULL = B_SFULL + 2,
  B_OREADY = B_PFULL + 2,
  B_OFREE = B_OREADY + 2,
  B_DRAIN = B_OFREE + 2,
  B_STALL = B_DRAIN + 1,
  B_VRELOAD = B_STALL + 1,   // the converter fetches a tile's bf16 values again
  B_COUNT = B_VRELOAD + 1
};
// after the barriers: abort flag, TMEM base, segment count, the V stages'
// formats (1: converted to fp16), the converter's reduction words
constexpr uint32_t kOffAbort = B_COUNT * 8, kOffTmem = kOffAbort + 4, kOffNseg = kOffTmem + 4,
                   kOffVmode = kOffNseg + 4, kOffRed = kOffVmode + 4 * kVSt, kOffCtlEnd = kOffRed + 12;
static_assert(kOffCtlEnd <= kBarBytes, "control block");

// P V in fp16: A (P, in TMEM) and B (V, MN-major) fp16, D fp32, M = N = 128
constexpr uint32_t kIdescPV16 = (1u << 4) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// CTA-partial barrier of the two converter warps
__device__ __forceinline__ void conv_sync() { asm volatile("bar.sync 1, 64;" ::: "memory"); }

}  // namespace

struct PairArgs {
  int32_t B, Hq, Hkv, G, Nb;
  int32_t mode;            // 0: tile = hg heads x Nb queries of one KV head; 1: 128 queries of one head
  int32_t hg, tph;         // heads per tile (mode 0); tiles per head (mode 1)
  int32_t tiles_per_kv, pairs_per_kv, npairs;
  int32_t nkt;             // key tiles
  int64_t nkeys;
  int32_t smax;            // slots per pair in the part buffer
  float scale_log2;
  float* part_a;           // slot s of row r at part_a + s * part_stride_a + r * D
  float* part_l;
  int64_t part_stride_a, part_stride_l;
  float* dst_a;            // final (A, L) of pairs covered by one CTA (packed rows)
  float* dst_l;
  int32_t* nslots;         // [npairs]: CTAs that touched the pair (written by its slot-0 CTA)
  const int8_t* mask;      // gamma: [B, Hq], 1 = head reuses (may be skipped)
  int32_t mask_active;
  int* status;
  uint64_t wait_limit_ns;
  uint32_t q_bytes;        // bytes of one Q tile (both 64-column halves)
  int32_t stall;           // test hook: the MMA issuer first waits on a barrier nothing completes
  // whole-pair mode: every CTA takes whole pairs (no slots, no merge kernel)
  // and its epilogue merges each row with `next` external parts and writes
  // O (out dtype and strides) and LSE directly
  int32_t whole;
  int32_t next;
  const float* ext_a[FB_MAX_PARTS];
  const float* ext_l[FB_MAX_PARTS];
  void* o;
  int64_t o_sb, o_sh, o_st;
  int32_t o_bf16;
  float* lse;
};

namespace {

struct Tile {
  int b, kvh, h0, nheads, i0, nrows;
  int64_t rbase;           // first packed (b, h, i) row
};

// Query tile `tl` (0 .. tiles_per_kv-1) of KV unit `u` = b * Hkv + kvh.
__device__ __forceinline__ Tile tile_of(const PairArgs& a, int u, int tl) {
  Tile t;
  t.b = u / a.Hkv;
  t.kvh = u % a.Hkv;
  if (a.mode == 0) {
    t.h0 = t.kvh * a.G + tl * a.hg;
    t.nheads = min(a.hg, a.G - tl * a.hg);
    t.i0 = 0;
    t.nrows = t.nheads * a.Nb;
  } else {
    const int g = tl / a.tph, tt = tl % a.tph;
    t.h0 = t.kvh * a.G + g;
    t.nheads = 1;
    t.i0 = tt * kBM;
    t.nrows = min(kBM, a.Nb - t.i0);
  }
  t.rbase = ((int64_t)t.b * a.Hq + t.h0) * a.Nb + t.i0;
  return t;
}

__device__ __forceinline__ bool pair_has_slot1(const PairArgs& a, int p) {
  return 2 * (p % a.pairs_per_kv) + 1 < a.tiles_per_kv;
}

// A pair needs computing unless the gamma gate lets every head in it reuse.
__device__ bool pair_active(const PairArgs& a, int p) {
  if (!a.mask_active) return true;
  const int u = p / a.pairs_per_kv, tl0 = 2 * (p % a.pairs_per_kv);
  for (int k = 0; k < 2; ++k) {
    if (tl0 + k >= a.tiles_per_kv) break;
    const Tile t = tile_of(a, u, tl0 + k);
    for (int h = t.h0; h < t.h0 + t.nheads; ++h)
      if (!a.mask[t.b * a.Hq + h]) return true;
  }
  return false;
}

// CTA of the stream-K grid (C CTAs over T items) that holds item i.
__device__ __forceinline__ int cta_of(int64_t i, int C, int64_t T) { return (int)(((i + 1) * C - 1) / T); }

struct Seg {
  int32_t pair, j0, j1, slot_ns;   // slot in the low 16 bits, slot count in the high 16
};

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const PairArgs a) {
  ptx::pdl_prologue();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (smem - smem_raw > (ptrdiff_t)kSmemSlack) {   // the layout would not fit: report, touch nothing
    if (threadIdx.x == 0) atomicCAS(a.status, 0, (int)FB_EUNSUPPORTED);
    return;
  }
  const uint32_t sbase = smem_addr(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + kOffAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + kOffTmem);
  int* nseg_sh = reinterpret_cast<int*>(smem + kOffBar + kOffNseg);
  volatile int* vmode = reinterpret_cast<volatile int*>(smem + kOffBar + kOffVmode);
  volatile uint32_t* red = reinterpret_cast<volatile uint32_t*>(smem + kOffBar + kOffRed);
  Seg* segs = reinterpret_cast<Seg*>(smem + kOffSeg);
  uint32_t* act = reinterpret_cast<uint32_t*>(smem + kOffAct);
  auto bar = [&](int i) { return smem_addr(bars + i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- the active pairs (all of them unless the gamma gate is on) ----
  const int words = (a.npairs + 31) / 32;
  if (a.mask_active) {
    for (int w = threadIdx.x; w < words; w += kThreads) act[w] = 0u;
    __syncthreads();
    for (int p = threadIdx.x; p < a.npairs; p += kThreads)
      if (pair_active(a, p)) atomicOr(act + (p >> 5), 1u << (p & 31));
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) {
      uint32_t cnt = 1;
      if (i >= B_PFULL && i < B_PFULL + 2) cnt = 4;   // one arrival per softmax warp
      if (i >= B_OFREE && i < B_OFREE + 2) cnt = 128;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    tc_fence_before();
  }
  __syncthreads();
  // ---- this CTA's segments (thread 0) ----
  if (threadIdx.x == 0) {
    int nact = a.npairs;
    if (a.mask_active) {
      nact = 0;
      for (int w = 0; w < words; ++w) nact += __popc(act[w]);
    }
    const int c = blockIdx.x;
    int n = 0;
    // the ai-th active pair (every pair is active without the gamma gate)
    auto active_pair = [&](int64_t ai) -> int {
      if (!a.mask_active) return (int)ai;
      int64_t left = ai;
      for (int w = 0; w < words; ++w) {
        uint32_t bits = act[w];
        const int cnt = __popc(bits);
        if (left >= cnt) { left -= cnt; continue; }
        while (left > 0) { bits &= bits - 1; --left; }
        return w * 32 + __ffs(bits) - 1;
      }
      return -1;
    };
    auto push_whole = [&](int p) {
      Seg sg;
      sg.pair = p;
      sg.j0 = 0;
      sg.j1 = a.nkt;
      sg.slot_ns = 1 << 16;
      segs[n++] = sg;
    };
    if (a.whole) {
      // whole pairs: active pairs c, c + C, c + 2C, ...
      const int C = min((int)gridDim.x, nact);
      if (!a.mask_active) {
        for (int p = c; p < a.npairs && n < kMaxSeg; p += C) push_whole(p);
      } else {
        int ai = 0;
        for (int p = 0; p < a.npairs && n < kMaxSeg; ++p) {
          if (!((act[p >> 5] >> (p & 31)) & 1u)) continue;
          if (ai++ % C == c) push_whole(p);
        }
      }
    } else {
      // Rounds of whole pairs first: with at least as many pairs as CTAs,
      // CTA c takes active pairs c, c + G, ... in lock step with its
      // neighbours, which hold the other query tiles of the same KV head and
      // stream the same K/V tiles at the same time (L2 serves the second
      // read).  The remaining pairs' key tiles are then split evenly
      // (stream-K) over up to G CTAs, each pair over at most smax - 1 of them.
      const int G = (int)gridDim.x;
      const int R = nact / G;
      for (int r = 0; r < R && n < kMaxSeg; ++r) {
        const int p = active_pair((int64_t)r * G + c);
        if (p >= 0) push_whole(p);
      }
      const int rem = nact - R * G;
      const int64_t T = (int64_t)rem * a.nkt;
      const int C = (int)min((int64_t)min((int64_t)G, T), (int64_t)rem * (a.smax - 1));
      if (c < C) {
        const int64_t i0 = (int64_t)c * T / C, i1 = (int64_t)(c + 1) * T / C;
        int64_t ai = i0 / a.nkt;            // index of the first pair among the remaining ones
        int p = active_pair((int64_t)R * G + ai);
        for (int64_t it = i0; it < i1 && n < kMaxSeg && p >= 0 && p < a.npairs;) {
          const int64_t base = ai * a.nkt;
          const int64_t e = min(i1, base + a.nkt);
          const int first = cta_of(base, C, T), last = cta_of(base + a.nkt - 1, C, T);
          Seg sg;
          sg.pair = p;
          sg.j0 = (int)(it - base);
          sg.j1 = (int)(e - base);
          sg.slot_ns = (c - first) | ((last - first + 1) << 16);
          segs[n++] = sg;
          it = e;
          ++ai;
          // next active pair
          ++p;
          if (a.mask_active)
            while (p < a.npairs && !((act[p >> 5] >> (p & 31)) & 1u)) ++p;
        }
      }
    }
    *nseg_sh = n;
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nseg = *nseg_sh;
  const Ctl ctl{abort_flag, a.status, a.wait_limit_ns};

  if (warp >= 8) {
    // the third warpgroup: all four warps give up registers, then the
    // producer and the MMA issuer run (warps 10 and 11 have nothing to do)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsIO));
  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nseg > 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)) : "memory");
      int kt = 0, vt = 0;   // K and V tiles issued so far (stage = count % depth, round = count / depth)
      int qarm = -1;
      bool ok = true;
      auto load_k = [&](int b, int kvh, int j) -> bool {
        const int st = kt % kKSt, round = kt / kKSt;
        if (kt >= kKSt && !wait_bounded_inl(bar(B_KEMPTY + st), (round - 1) & 1, ctl)) return false;
        mbar_expect_tx(bar(B_KFULL + st), kTile);
        const uint32_t dst = sbase + kOffK + st * kTile;
        tma_load_4d(dst, &tmK, bar(B_KFULL + st), 0, j * kBN, kvh, b);
        tma_load_4d(dst + kHalf, &tmK, bar(B_KFULL + st), 64, j * kBN, kvh, b);
        ++kt;
        return true;
      };
      auto load_v = [&](int b, int kvh, int j) -> bool {
        const int st = vt % kVSt, round = vt / kVSt;
        if (vt >= kVSt && !wait_bounded_inl(bar(B_VEMPTY + st), (round - 1) & 1, ctl)) return false;
        mbar_expect_tx(bar(B_VFULL + st), kTile);
        const uint32_t dst = sbase + kOffV + st * kTile;
        tma_load_4d(dst, &tmV, bar(B_VFULL + st), 0, j * kBN, kvh, b);
        tma_load_4d(dst + kHalf, &tmV, bar(B_VFULL + st), 64, j * kBN, kvh, b);
        ++vt;
        return true;
      };
      for (int si = 0; si < nseg && ok; ++si) {
        const Seg sg = segs[si];
        const int u = sg.pair / a.pairs_per_kv, tl0 = 2 * (sg.pair % a.pairs_per_kv);
        const bool two = pair_has_slot1(a, sg.pair);
        const Tile t0 = tile_of(a, u, tl0);
        if (si > 0 && !(ok = wait_bounded_inl(bar(B_QEMPTY), (si - 1) & 1, ctl))) break;
        mbar_expect_tx(bar(B_QFULL), a.q_bytes * (two ? 2u : 1u));
        tma_load_4d(sbase + kOffQ, &tmQ, bar(B_QFULL), 0, t0.i0, t0.h0, t0.b);
        tma_load_4d(sbase + kOffQ + kHalf, &tmQ, bar(B_QFULL), 64, t0.i0, t0.h0, t0.b);
        if (two) {
          const Tile t1 = tile_of(a, u, tl0 + 1);
          tma_load_4d(sbase + kOffQ + kTile, &tmQ, bar(B_QFULL), 0, t1.i0, t1.h0, t1.b);
          tma_load_4d(sbase + kOffQ + kTile + kHalf, &tmQ, bar(B_QFULL), 64, t1.i0, t1.h0, t1.b);
        }
        qarm = si;
        for (int j = sg.j0; j < sg.j1 && ok; ++j) {
          ok = load_k(t0.b, t0.kvh, j);
          if (ok) ok = load_v(t0.b, t0.kvh, j);
        }
      }
      // let every copy this thread started land before the CTA can exit
      if (qarm >= 0) wait_bounded_inl(bar(B_QFULL), qarm & 1, ctl, true);
      // (stage st was last armed in round (count - 1 - st) / depth)
      for (int st = 0; st < kKSt; ++st)
        if (kt > st) wait_bounded_inl(bar(B_KFULL + st), ((kt - 1 - st) / kKSt) & 1, ctl, true);
      for (int st = 0; st < kVSt; ++st)
        if (vt > st) wait_bounded_inl(bar(B_VFULL + st), ((vt - 1 - st) / kVSt) & 1, ctl, true);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nseg > 0) {
      const uint64_t dQ0 = sw128_desc(sbase + kOffQ, 16, 1024);
      const uint64_t dQ1 = sw128_desc(sbase + kOffQ + kTile, 16, 1024);
      const uint64_t dK = sw128_desc(sbase + kOffK, 16, 1024);
      const uint64_t dV = sw128_desc(sbase + kOffV, kHalf, 1024);
      int kt = 0, vt = 0;
      int pcnt[2] = {0, 0}, segcnt[2] = {0, 0};
      bool ok = !a.stall || wait_bounded_inl(bar(B_STALL), 0, ctl);
      // S_s = Q_s K^T for the K tile in stage kst
      auto issue_s = [&](int s, int kst) {
        const uint64_t dKs = dK + (uint64_t)((kst * kTile) >> 4);
        const uint64_t dQs = s ? dQ1 : dQ0;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
          tc_mma(tmem + s * kBN, dQs + off, dKs + off, kIdescQK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_SFULL + s));
      };
      // O_s += P V for the V tile in stage vst: one pass in fp16 where the
      // converter turned the tile into fp16, else P_hi V + P_lo V in bf16
      auto issue_pv = [&](int s, int vst, bool first, bool f16) {
        const uint64_t dVs = dV + (uint64_t)((vst * kTile) >> 4);
        const uint32_t pt = tmem + s * kBN;
        if (f16) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            tc_mma_ts(tmem + kTmemO + s * kBN, pt + kk * 8, dVs + (uint64_t)((kk * 2048) >> 4), kIdescPV16,
                      (!first || kk > 0) ? 1u : 0u);
          return;
        }
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            tc_mma_ts(tmem + kTmemO + s * kBN, pt + hl * 64 + kk * 8, dVs + (uint64_t)((kk * 2048) >> 4),
                      kIdescPV, (!first || hl > 0 || kk > 0) ? 1u : 0u);
      };
      for (int si = 0; si < nseg && ok; ++si) {
        const Seg sg = segs[si];
        const bool two = pair_has_slot1(a, sg.pair);
        const int ns = two ? 2 : 1;
        if (!(ok = wait_bounded_inl(bar(B_QFULL), si & 1, ctl))) break;
        int kst = kt % kKSt;
        if (!(ok = wait_bounded_inl(bar(B_KFULL + kst), (kt / kKSt) & 1, ctl))) break;
        tc_fence_after();
        issue_s(0, kst);
        if (ns > 1) issue_s(1, kst);
        tc_commit(bar(B_KEMPTY + kst));
        ++kt;
        if (sg.j1 - sg.j0 == 1) tc_commit(bar(B_QEMPTY));
        for (int j = sg.j0; j < sg.j1 && ok; ++j) {
          const int vst = vt % kVSt;
          const bool more = j + 1 < sg.j1;
          kst = kt % kKSt;
          // V_j's format and K_(j+1) depend only on earlier tiles and are
          // normally ready long before P_0(j): waiting for them first keeps
          // these waits off the chain P_s(j) -> P V(j) -> S_s(j+1)
          if (!(ok = wait_bounded_inl(bar(B_VCONV + vst), (vt / kVSt) & 1, ctl))) break;
          const bool vf16 = vmode[vst] != 0;
          if (more && !(ok = wait_bounded_inl(bar(B_KFULL + kst), (kt / kKSt) & 1, ctl))) break;
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            if (s >= ns || !ok) break;
            ok = wait_bounded_inl(bar(B_PFULL + s), pcnt[s] & 1, ctl);
            if (ok && j == sg.j0 && segcnt[s] > 0) ok = wait_bounded_inl(bar(B_OFREE + s), (segcnt[s] - 1) & 1, ctl);
            if (!ok) break;
            ++pcnt[s];
            tc_fence_after();
            issue_pv(s, vst, j == sg.j0, vf16);
            if (more) issue_s(s, kst);
            if (!more) tc_commit(bar(B_OREADY + s));
          }
          if (!ok) break;
          tc_commit(bar(B_VEMPTY + vst));
          ++vt;
          if (more) {
            tc_commit(bar(B_KEMPTY + kst));
            ++kt;
            if (j + 2 == sg.j1) tc_commit(bar(B_QEMPTY));   // the segment's last S has been issued
          }
        }
        ++segcnt[0];
        if (ns > 1) ++segcnt[1];
      }
      // quiesce this thread's tensor-core work before TMEM is freed
      tc_commit(bar(B_DRAIN));
      wait_bounded_inl(bar(B_DRAIN), 0, ctl, true);
    }
  } else if (nseg > 0) {
    // ------------------------------------------------------------ converter
    // Warps 10 and 11 turn each landed V tile into fp16 in place, in one
    // pass that also finds the tile's largest |v|.  The fp16 tile stands when
    // every value converted exactly or negligibly: that largest |v| has a
    // binary exponent in [-4, 15] (below 2^16 nothing overflows; values under
    // fp16's 2^-14 lose at most 2^-25, under 2^-21 of the tile's largest).
    // Any other tile (huge, tiny, NaN or inf values) is fetched again in
    // bf16 and takes the hi/lo P V.  The tile's format goes out with the
    // VCONV barrier.  Thread 0 alone waits on mbarriers and broadcasts the
    // outcome, so the two warps always meet at their barrier.
    const int ct = threadIdx.x - 320;   // 0..63
    int vt = 0, nreload = 0;
    bool ok = true;
    for (int si = 0; si < nseg && ok; ++si) {
      const Seg sg = segs[si];
      for (int j = sg.j0; j < sg.j1; ++j, ++vt) {
        const int st = vt % kVSt;
        if (ct == 0) red[2] = wait_bounded_inl(bar(B_VFULL + st), (vt / kVSt) & 1, ctl) ? 1u : 0u;
        conv_sync();
        ok = red[2] != 0;
        if (!ok) break;
        // one pass: convert every value and track the largest |v|; a tile
        // that did not convert exactly is fetched again in bf16 below
        uint4* tile = reinterpret_cast<uint4*>(smem + kOffV + st * kTile);
        uint32_t mx = 0u;
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
          const uint4 v = tile[ct + 64 * i];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t h[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            mx = max(mx, max(w[e] & 0x7FFFu, (w[e] >> 16) & 0x7FFFu));
            h[e] = f16x2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
          }
          tile[ct + 64 * i] = make_uint4(h[0], h[1], h[2], h[3]);
        }
        ptx::fence_proxy_async_smem();   // the tensor core (or a refetch) reaches the tile through the async proxy
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) red[warp - 10] = mx;
        conv_sync();
        mx = max(red[0], red[1]);
        const int e2 = (int)(mx >> 7) - 127;   // binary exponent of the largest |v|
        const bool f16 = mx == 0u || (mx < 0x7F80u && e2 >= -4 && e2 <= 15);
        conv_sync();
        if (ct == 0) {
          if (!f16) {
            const Tile tv = tile_of(a, sg.pair / a.pairs_per_kv, 2 * (sg.pair % a.pairs_per_kv));
            const uint32_t dst = sbase + kOffV + st * kTile;
            mbar_expect_tx(bar(B_VRELOAD), kTile);
            tma_load_4d(dst, &tmV, bar(B_VRELOAD), 0, j * kBN, tv.kvh, tv.b);
            tma_load_4d(dst + kHalf, &tmV, bar(B_VRELOAD), 64, j * kBN, tv.kvh, tv.b);
            // the refetch lands whatever happens elsewhere (a draining wait)
            wait_bounded_inl(bar(B_VRELOAD), nreload & 1, ctl, true);
            ++nreload;
          }
          vmode[st] = f16 ? 1 : 0;
          mbar_arrive(bar(B_VCONV + st));
        }
      }
    }
  }
  } else {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int s = warp >> 2;                 // slot: query tile 0 or 1 of the pair
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t tS = tl + s * kBN, tO = tl + kTmemO + s * kBN;
    int scnt = 0, ocnt = 0;
    bool ok = true;
    auto uniform = [](bool v) { return __all_sync(0xffffffffu, v); };
    int vtc = 0;   // V tiles of every segment so far (slot 1 counts the lone-tile segments it skips)
    bool skipped = false;
    // the format of this tile's V (fp16, or bf16 for the hi/lo P V)
    auto v_format = [&](bool& f16) -> bool {
      if (!uniform(wait_bounded_inl(bar(B_VCONV + vtc % kVSt), (vtc / kVSt) & 1, ctl))) return false;
      f16 = vmode[vtc % kVSt] != 0;
      ++vtc;
      return true;
    };
    for (int si = 0; si < nseg && ok; ++si) {
      const Seg sg = segs[si];
      if (s == 1 && !pair_has_slot1(a, sg.pair)) {
        vtc += sg.j1 - sg.j0;
        skipped = true;
        continue;
      }
      float m = -CUDART_INF_F, l = 0.f;
      for (int j = sg.j0; j < sg.j1; ++j) {
        // V_j lands with K_j, so the format is normally known long before S_j
        // and its wait comes first, off the chain S_j -> P_j.  A parity wait
        // is only sound within one phase of the converter, which holds once
        // this slot has had the tile before (S_s(j - 1) was issued after a P V
        // that waited for the format of tile j - 2); after slot 1 skipped
        // lone-tile segments, the first tile's format is read after S_j
        // instead (S_j was issued after the skipped tiles' P V).
        const bool late = skipped && j == sg.j0;
        bool vf16 = false;
        if (!late && !(ok = v_format(vf16))) break;
        ok = uniform(wait_bounded_inl(bar(B_SFULL + s), scnt & 1, ctl));
        if (ok && late) ok = v_format(vf16);
        skipped = false;
        if (!ok) break;
        ++scnt;
        tc_fence_after();
        float sv[128];
        tmem_ld32(tS, sv);
        tmem_ld32(tS + 32, sv + 32);
        tmem_ld32(tS + 64, sv + 64);
        tmem_ld32(tS + 96, sv + 96);
        tmem_wait_ld();
        const int64_t nvalid = a.nkeys - (int64_t)j * kBN;
        if (nvalid < kBN) {   // ragged last key tile
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= nvalid) sv[c] = -CUDART_INF_F;
        }
        float mx[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) mx[e] = sv[e];
#pragma unroll
        for (int c = 4; c < 128; c += 8) {
#pragma unroll
          for (int e = 0; e < 4; ++e) mx[e] = fmax3(mx[e], sv[c + e], c + 4 + e < 128 ? sv[c + 4 + e] : mx[e]);
        }
        const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * a.scale_log2;
        const bool move = tmax > m + kRescaleLog2;
        const bool scale_o = move && m != -CUDART_INF_F;
        const float alpha = scale_o ? fast_exp2(m - tmax) : 1.f;
        if (__any_sync(0xffffffffu, scale_o)) {
          // O_s holds this segment's earlier tiles: PV_s(j-1) has completed
          // (S_s(j), issued after it, has), and PV_s(j) waits for this P
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {   // 8 columns at a time: few live registers beside the scores
            uint32_t o[8];
            tmem_ld8u(tO + c * 8, o);
            tmem_wait_ld();
            const uint64_t al2 = pack2(alpha, alpha);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              float lo, hi;
              unpack2(fmul2(pack2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2), lo, hi);
              o[e] = __float_as_uint(lo);
              o[e + 1] = __float_as_uint(hi);
            }
            tmem_st8u(tO + c * 8, o);
          }
          tmem_wait_st();
        }
        if (move) {
          l *= alpha;
          m = tmax;
        }
        const float nref = m == -CUDART_INF_F ? 0.f : -m;
        // x = s * scale - m and the row sum two lanes per instruction
        const uint64_t sc2 = pack2(a.scale_log2, a.scale_log2), nr2 = pack2(nref, nref);
        uint64_t acc[2] = {0ull, 0ull};   // +0.0f pairs
        if (vf16) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {   // 32 keys: 16 fp16 pairs at 16c
            uint32_t hw[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float x0, x1;
              unpack2(ffma2(pack2(sv[32 * c + 2 * e], sv[32 * c + 2 * e + 1]), sc2, nr2), x0, x1);
              const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
              acc[e & 1] = fadd2(acc[e & 1], pack2(p0, p1));
              hw[e] = f16x2(p0, p1);
            }
            tmem_st16u(tS + 16 * c, hw);
          }
        } else
#pragma unroll
        for (int c = 0; c < 4; ++c) {   // 32 keys: 16 hi words at 16c, 16 lo words at 64 + 16c
          // the hi and lo words take the registers of the two scores they replace
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            unpack2(ffma2(pack2(sv[32 * c + 2 * e], sv[32 * c + 2 * e + 1]), sc2, nr2), x0, x1);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            acc[e & 1] = fadd2(acc[e & 1], pack2(p0, p1));
            uint32_t h, lw;
            split_pair(p0, p1, h, lw);
            sv[32 * c + 2 * e] = __uint_as_float(h);
            sv[32 * c + 2 * e + 1] = __uint_as_float(lw);
          }
          uint32_t hi[16], lo[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            hi[e] = __float_as_uint(sv[32 * c + 2 * e]);
            lo[e] = __float_as_uint(sv[32 * c + 2 * e + 1]);
          }
          tmem_st16u(tS + 16 * c, hi);
          tmem_st16u(tS + 64 + 16 * c, lo);
        }
        {
          float s0, s1, s2, s3;
          unpack2(acc[0], s0, s1);
          unpack2(acc[1], s2, s3);
          l += (s0 + s1) + (s2 + s3);
        }
        // P_s is in TMEM: one arrival per warp
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PFULL + s));
      }
      if (!ok) break;
      // ---- epilogue of the segment: O / l and L of this row ----
      ok = uniform(wait_bounded_inl(bar(B_OREADY + s), ocnt & 1, ctl));
      if (!ok) break;
      ++ocnt;
      tc_fence_after();
      const Tile t = tile_of(a, sg.pair / a.pairs_per_kv, 2 * (sg.pair % a.pairs_per_kv) + s);
      if (a.o && (sg.slot_ns >> 16) == 1) {
        // a pair this CTA covers alone, with O requested (whole-pair mode, or
        // a direct pair of the split mode): merge with the external parts
        // (log space, as the standalone merge) and write this row of O and LSE
        const bool mine = row < t.nrows;
        const int64_t r = t.rbase + row;
        const float Lin = l > 0.f ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
        float mm = Lin;
        float Lx[FB_MAX_PARTS];
#pragma unroll
        for (int p = 0; p < FB_MAX_PARTS - 1; ++p) {
          Lx[p] = (p < a.next && mine) ? a.ext_l[p][r] : -CUDART_INF_F;
          mm = fmaxf(mm, Lx[p]);
        }
        const bool empty = mm == -CUDART_INF_F;
        const float win = (empty || Lin == -CUDART_INF_F) ? 0.f : __expf(Lin - mm);
        float wx[FB_MAX_PARTS];
        float wsum = win;
#pragma unroll
        for (int p = 0; p < FB_MAX_PARTS - 1; ++p) {
          wx[p] = (empty || Lx[p] == -CUDART_INF_F) ? 0.f : __expf(Lx[p] - mm);
          wsum += wx[p];
        }
        const float inv = empty ? 0.f : 1.f / wsum;
        const float wi = l > 0.f ? win / l : 0.f;   // O in TMEM is unnormalised
        const int h = a.mode == 0 ? t.h0 + row / a.Nb : t.h0;
        const int i = a.mode == 0 ? row % a.Nb : t.i0 + row;
        const int64_t obase = t.b * a.o_sb + (int64_t)h * a.o_sh + (int64_t)i * a.o_st;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_wait_ld();
          if (mine) {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= wi;
#pragma unroll
            for (int p = 0; p < FB_MAX_PARTS - 1; ++p) {
              if (p >= a.next || wx[p] == 0.f) continue;   // an empty part may hold anything
              const float4* src = reinterpret_cast<const float4*>(a.ext_a[p] + r * kD + c * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float4 v = src[e];
                o[4 * e] = fmaf(wx[p], v.x, o[4 * e]);
                o[4 * e + 1] = fmaf(wx[p], v.y, o[4 * e + 1]);
                o[4 * e + 2] = fmaf(wx[p], v.z, o[4 * e + 2]);
                o[4 * e + 3] = fmaf(wx[p], v.w, o[4 * e + 3]);
              }
            }
            if (a.o_bf16) {
              uint4* d4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.o) + obase + c * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint32_t w[4];
#pragma unroll
                for (int f = 0; f < 4; ++f) {
                  const __nv_bfloat162 pr = __floats2bfloat162_rn(o[8 * e + 2 * f] * inv, o[8 * e + 2 * f + 1] * inv);
                  w[f] = *reinterpret_cast<const uint32_t*>(&pr);
                }
                d4[e] = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else {
              float4* d4 = reinterpret_cast<float4*>(static_cast<float*>(a.o) + obase + c * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                d4[e] = make_float4(o[4 * e] * inv, o[4 * e + 1] * inv, o[4 * e + 2] * inv, o[4 * e + 3] * inv);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bar(B_OFREE + s));
        if (mine && a.lse) a.lse[r] = empty ? -CUDART_INF_F : mm + __logf(wsum);
        if (!a.whole && mine && row == 0 && s == 0) a.nslots[sg.pair] = 1;   // the merge kernel skips the pair
        continue;
      }
      const int slot = sg.slot_ns & 0xFFFF, nsl = sg.slot_ns >> 16;
      const bool direct = nsl == 1;
      const int64_t r = t.rbase + row;
      float* dA = direct ? a.dst_a : a.part_a + slot * a.part_stride_a;
      float* dL = direct ? a.dst_l : a.part_l + slot * a.part_stride_l;
      const bool mine = row < t.nrows;
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
        if (mine) {
          float4* d4 = reinterpret_cast<float4*>(dA + r * kD + c * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            d4[e] = make_float4(o[4 * e] * inv, o[4 * e + 1] * inv, o[4 * e + 2] * inv, o[4 * e + 3] * inv);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(B_OFREE + s));   // O_s may be overwritten by the next segment
      if (mine) dL[r] = l > 0.f ? (m + log2f(l)) * kLn2 : -CUDART_INF_F;
      if (mine && row == 0 && s == 0 && slot == 0) a.nslots[sg.pair] = nsl;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// Log-space merge of the slots of every pair covered by two or more CTAs into
// the final (A, L), or, when O is requested, together with the external parts
// into O and LSE; one warp per packed row.  Rows of heads that reuse their
// cache (gamma) and rows of pairs finished by one CTA are left alone.
__global__ void __launch_bounds__(256) pair_merge_kernel(const PairArgs a) {
  ptx::pdl_prologue();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + warp;
  const int64_t nrows = (int64_t)a.B * a.Hq * a.Nb;
  if (r >= nrows) return;
  const int64_t bh = r / a.Nb;
  if (a.mask_active && a.mask[bh]) return;
  const int b = (int)(bh / a.Hq), h = (int)(bh % a.Hq), i = (int)(r % a.Nb);
  const int kvh = h / a.G, g = h % a.G;
  const int tl = a.mode == 0 ? g / a.hg : g * a.tph + i / kBM;
  const int p = (b * a.Hkv + kvh) * a.pairs_per_kv + tl / 2;
  const int ns = a.nslots[p];
  if (ns <= 1 || ns > a.smax) return;   // one CTA wrote dst itself (a count outside [2, smax]: the pass failed)
  float m = -CUDART_INF_F;
  for (int s = 0; s < ns; ++s) m = fmaxf(m, a.part_l[s * a.part_stride_l + r]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float Ls = a.part_l[s * a.part_stride_l + r];
    if (Ls == -CUDART_INF_F) continue;
    const float w = __expf(Ls - m);
    const float4 v = *reinterpret_cast<const float4*>(a.part_a + s * a.part_stride_a + r * kD + lane * 4);
    wsum += w;
    acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
  }
  if (a.o) {
    // the split mode with O requested: fold in the external parts and write
    // this row of O (out dtype, O strides) and LSE
    float mx = m;
    for (int p = 0; p < a.next; ++p) mx = fmaxf(mx, a.ext_l[p][r]);
    const float scl = (m == -CUDART_INF_F || mx == -CUDART_INF_F) ? 0.f : __expf(m - mx);
    acc.x *= scl; acc.y *= scl; acc.z *= scl; acc.w *= scl;
    wsum *= scl;
    for (int p = 0; p < a.next; ++p) {
      const float Lx = a.ext_l[p][r];
      if (Lx == -CUDART_INF_F) continue;   // an empty part may hold anything
      const float w = __expf(Lx - mx);
      const float4 v = *reinterpret_cast<const float4*>(a.ext_a[p] + r * kD + lane * 4);
      wsum += w;
      acc.x = fmaf(w, v.x, acc.x); acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z); acc.w = fmaf(w, v.w, acc.w);
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    const int64_t obase = b * a.o_sb + (int64_t)h * a.o_sh + (int64_t)i * a.o_st + lane * 4;
    if (a.o_bf16) {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
      uint2 w2;
      w2.x = *reinterpret_cast<const uint32_t*>(&lo);
      w2.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.o) + obase) = w2;
    } else {
      *reinterpret_cast<float4*>(static_cast<float*>(a.o) + obase) =
          make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (lane == 0 && a.lse) a.lse[r] = wsum > 0.f ? mx + __logf(wsum) : -CUDART_INF_F;
    return;
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __syncwarp();   // every lane has read the slots before any writes (dst may be slot 0)
  *reinterpret_cast<float4*>(a.dst_a + r * kD + lane * 4) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lane == 0) a.dst_l[r] = m == -CUDART_INF_F ? -CUDART_INF_F : m + __logf(wsum);
}

// ------------------------------------------------------------------ host --
int* device_status_ptr();
uint64_t wait_limit_ns();

// Plan of the paired pass over nkeys keys, or false where it does not apply
// (fewer than two query tiles per KV head, too few key tiles, or more pairs
// than one CTA can list).
// The register split of the kernel holds only if every thread is launched
// with kRegsLaunch registers (checked once per device).
static bool pair_regs_ok() {
  static int cache[kMaxDevices] = {};   // 0 unknown, 1 ok, 2 not
  int& c = cache[current_device()];
  if (c == 0) {
    cudaFuncAttributes fa;
    c = (cudaFuncGetAttributes(&fa, attn_pair_kernel) == cudaSuccess && fa.numRegs == kRegsLaunch) ? 1 : 2;
    cudaGetLastError();
  }
  return c == 1;
}

bool pair_plan(const fb_attn_desc& d, int64_t nkeys, PairPlan* p) {
  int mode, hg, tpu, units;
  if (nkeys <= 0 || !tc_tiling(d, &mode, &hg, &tpu, &units)) return false;
  const int G = d.Hq / d.Hkv;
  p->mode = mode;
  p->hg = hg;
  p->tph = mode == 0 ? 1 : tpu;
  p->tiles_per_kv = mode == 0 ? tpu : G * tpu;
  if (p->tiles_per_kv < 2) return false;
  p->pairs_per_kv = (p->tiles_per_kv + 1) / 2;
  p->npairs = d.B * d.Hkv * p->pairs_per_kv;
  p->nkt = (int32_t)((nkeys + kBN - 1) / kBN);
  if (p->nkt < 4 || p->npairs > kMaxPairs || !pair_regs_ok()) return false;
  const int64_t T = (int64_t)p->npairs * p->nkt;
  p->grid = (int32_t)std::min<int64_t>(num_sms(), T);
  // R rounds of whole pairs, then the remaining pairs' key tiles split over
  // the grid: segments per CTA at most R + ceil(items per CTA / key tiles) + 1
  const int64_t R = p->npairs / p->grid, rem = p->npairs - R * p->grid;
  const int64_t per = (rem * p->nkt + p->grid - 1) / p->grid;
  if (R + (per + p->nkt - 1) / p->nkt + 1 > kMaxSeg) return false;
  // slots per pair: a remaining pair spans at most ceil(grid / rem) + 1 CTAs;
  // after whole-pair rounds the split is capped (the kernel then uses fewer
  // CTAs for the remaining pairs) to keep the part buffers small
  constexpr int64_t kSlotCapAfterRounds = 8;
  const int64_t span = rem > 0 ? (p->grid + rem - 1) / rem + 1 : 2;
  p->smax = (int32_t)(R == 0 ? span : std::max<int64_t>(2, std::min(span, kSlotCapAfterRounds)));
  return true;
}

// Slots the paired pass may use for a prefix of up to max_keys keys (sizes workspaces).
int32_t pair_slot_cap(const fb_attn_desc& d, int64_t max_keys) {
  PairPlan p;
  if (!pair_plan(d, std::max<int64_t>(max_keys, kBN * 4), &p)) return 0;
  return p.smax;
}

cudaError_t launch_attn_pair(const fb_attn_desc& d, const TcMaps& m, const PairPlan& pp, int64_t nkeys,
                             const int8_t* mask, int mask_active, float scale_log2, float* pa, float* pl,
                             float* dst_a, float* dst_l, int32_t* nslots, cudaStream_t s, bool merge_only) {
  PairArgs a;
  memset(&a, 0, sizeof(a));
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.G = d.Hq / d.Hkv; a.Nb = d.Nb;
  a.mode = pp.mode; a.hg = pp.hg; a.tph = pp.tph;
  a.tiles_per_kv = pp.tiles_per_kv; a.pairs_per_kv = pp.pairs_per_kv; a.npairs = pp.npairs;
  a.nkt = pp.nkt; a.nkeys = nkeys; a.smax = pp.smax;
  a.scale_log2 = scale_log2;
  a.part_a = pa; a.part_l = pl;
  a.part_stride_a = (int64_t)d.B * d.Hq * d.Nb * d.D;
  a.part_stride_l = (int64_t)d.B * d.Hq * d.Nb;
  a.dst_a = dst_a; a.dst_l = dst_l; a.nslots = nslots;
  a.mask = mask; a.mask_active = mask_active;
  a.status = device_status_ptr();
  a.wait_limit_ns = wait_limit_ns();
  a.q_bytes = 2u * 64u * 2u * (uint32_t)(pp.mode == 0 ? d.Nb * pp.hg : kBM);
  a.stall = debug_stall() ? 1 : 0;
  if (!a.status) return cudaErrorInvalidValue;
  static bool attr[kMaxDevices] = {};
  bool& done = attr[current_device()];
  if (!done) {
    cudaError_t e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    done = true;
  }
  if (merge_only) {
    const int64_t nrows = (int64_t)d.B * d.Hq * d.Nb;
    return launch_k(pair_merge_kernel, dim3((unsigned)((nrows + 7) / 8)), dim3(256), 0, s, a);
  }
  return launch_k(attn_pair_kernel, dim3(pp.grid), dim3(kThreads), kSmemBytes, s, m.q, m.k, m.v, a);
}

// Whole-pair fused pass over the keys of (k, v) [0, nkeys): attention of the
// block's queries merged with `next` external parts, written to O and LSE.
cudaError_t launch_attn_pair_fused(const fb_attn_desc& d, const TcMaps& m, const PairPlan& pp, int64_t nkeys,
                                   float scale_log2, int32_t next, const float* const* ext_a,
                                   const float* const* ext_l, void* o, float* lse, cudaStream_t s) {
  PairArgs a;
  memset(&a, 0, sizeof(a));
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.G = d.Hq / d.Hkv; a.Nb = d.Nb;
  a.mode = pp.mode; a.hg = pp.hg; a.tph = pp.tph;
  a.tiles_per_kv = pp.tiles_per_kv; a.pairs_per_kv = pp.pairs_per_kv; a.npairs = pp.npairs;
  a.nkt = pp.nkt; a.nkeys = nkeys; a.smax = 1;
  a.scale_log2 = scale_log2;
  a.status = device_status_ptr();
  a.wait_limit_ns = wait_limit_ns();
  a.q_bytes = 2u * 64u * 2u * (uint32_t)(pp.mode == 0 ? d.Nb * pp.hg : kBM);
  a.stall = debug_stall() ? 1 : 0;
  a.whole = 1;
  a.next = next;
  for (int p = 0; p < next; ++p) { a.ext_a[p] = ext_a[p]; a.ext_l[p] = ext_l[p]; }
  a.o = o; a.o_sb = d.o_strides[0]; a.o_sh = d.o_strides[1]; a.o_st = d.o_strides[2];
  a.o_bf16 = d.out_dtype == FB_BF16;
  a.lse = lse;
  if (!a.status || next < 0 || next > FB_MAX_PARTS - 1) return cudaErrorInvalidValue;
  static bool attr[kMaxDevices] = {};
  bool& done = attr[current_device()];
  if (!done) {
    cudaError_t e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    done = true;
  }
  const int grid = std::min(num_sms(), pp.npairs);
  return launch_k(attn_pair_kernel, dim3(grid), dim3(kThreads), kSmemBytes, s, m.q, m.k, m.v, a);
}

// Split pass over the keys of (k, v) [0, nkeys) with O requested: pairs a CTA
// covers alone are merged with the `next` external parts and written to O
// and LSE in the kernel's epilogue; the slots of pairs split over several
// CTAs (the stream-K remainder after the whole-pair rounds) are merged with
// the external parts by the merge kernel.  pa/pl hold pp.smax slots, nslots
// one count per pair.
cudaError_t launch_attn_pair_split_fused(const fb_attn_desc& d, const TcMaps& m, const PairPlan& pp, int64_t nkeys,
                                         float scale_log2, int32_t next, const float* const* ext_a,
                                         const float* const* ext_l, void* o, float* lse, float* pa, float* pl,
                                         int32_t* nslots, cudaStream_t s) {
  PairArgs a;
  memset(&a, 0, sizeof(a));
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.G = d.Hq / d.Hkv; a.Nb = d.Nb;
  a.mode = pp.mode; a.hg = pp.hg; a.tph = pp.tph;
  a.tiles_per_kv = pp.tiles_per_kv; a.pairs_per_kv = pp.pairs_per_kv; a.npairs = pp.npairs;
  a.nkt = pp.nkt; a.nkeys = nkeys; a.smax = pp.smax;
  a.scale_log2 = scale_log2;
  a.part_a = pa; a.part_l = pl;
  a.part_stride_a = (int64_t)d.B * d.Hq * d.Nb * d.D;
  a.part_stride_l = (int64_t)d.B * d.Hq * d.Nb;
  a.nslots = nslots;
  a.status = device_status_ptr();
  a.wait_limit_ns = wait_limit_ns();
  a.q_bytes = 2u * 64u * 2u * (uint32_t)(pp.mode == 0 ? d.Nb * pp.hg : kBM);
  a.stall = debug_stall() ? 1 : 0;
  a.whole = 0;
  a.next = next;
  for (int p = 0; p < next; ++p) { a.ext_a[p] = ext_a[p]; a.ext_l[p] = ext_l[p]; }
  a.o = o; a.o_sb = d.o_strides[0]; a.o_sh = d.o_strides[1]; a.o_st = d.o_strides[2];
  a.o_bf16 = d.out_dtype == FB_BF16;
  a.lse = lse;
  if (!a.status || !o || next < 0 || next > FB_MAX_PARTS - 1) return cudaErrorInvalidValue;
  static bool attr[kMaxDevices] = {};
  bool& done = attr[current_device()];
  if (!done) {
    cudaError_t e = cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    done = true;
  }
  cudaError_t e = launch_k(attn_pair_kernel, dim3(pp.grid), dim3(kThreads), kSmemBytes, s, m.q, m.k, m.v, a);
  if (e != cudaSuccess) return e;
  const int64_t nrows = (int64_t)d.B * d.Hq * d.Nb;
  return launch_k(pair_merge_kernel, dim3((unsigned)((nrows + 7) / 8)), dim3(256), 0, s, a);
}

// A whole-pair plan: as pair_plan, without the slot bookkeeping (each CTA
// takes whole pairs; up to kMaxSeg pairs per CTA).
bool pair_plan_whole(const fb_attn_desc& d, int64_t nkeys, PairPlan* p) {
  int mode, hg, tpu, units;
  if (!pair_regs_ok()) return false;
  if (nkeys <= 0 || !tc_tiling(d, &mode, &hg, &tpu, &units)) return false;
  const int G = d.Hq / d.Hkv;
  p->mode = mode;
  p->hg = hg;
  p->tph = mode == 0 ? 1 : tpu;
  p->tiles_per_kv = mode == 0 ? tpu : G * tpu;
  if (p->tiles_per_kv < 2) return false;
  p->pairs_per_kv = (p->tiles_per_kv + 1) / 2;
  p->npairs = d.B * d.Hkv * p->pairs_per_kv;
  p->nkt = (int32_t)((nkeys + kBN - 1) / kBN);
  p->grid = std::min(num_sms(), p->npairs);
  p->smax = 1;
  return p->npairs <= kMaxPairs && (p->npairs + p->grid - 1) / p->grid <= kMaxSeg;
}

int32_t pair_count(const fb_attn_desc& d) {
  int mode, hg, tpu, units;
  if (!tc_tiling(d, &mode, &hg, &tpu, &units)) return 0;
  const int tiles_per_kv = mode == 0 ? tpu : (d.Hq / d.Hkv) * tpu;
  if (tiles_per_kv < 2) return 0;
  return d.B * d.Hkv * ((tiles_per_kv + 1) / 2);
}

}  // namespace fb
