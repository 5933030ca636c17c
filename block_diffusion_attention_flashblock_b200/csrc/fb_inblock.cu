// Block-internal attention fused with the log-space merge, for small blocks
// (FlashBlock summary, "Mécanisme Central": A_in over the block's own keys
// J_in, then A = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (...)).  This is the
// whole reuse step of a diffusion LM, so it is built for latency.  Two
// kernels, chosen by how many CTAs the step makes:
//   - split-warp (inblock_small_kernel): one CTA = 16 packed query rows of
//     one KV head (G query heads x Nb queries) and 4 warps; each warp forms
//     S for a quarter of the block's keys, the row maxima and sums meet in
//     shared memory, and each warp owns a quarter (32 columns) of the head
//     dimension in P V, the merge and the stores, which keeps every warp's
//     dependent instruction chain short (small steps: dllm_8k, blocks of 4);
//   - warp-per-rows (inblock_rows_kernel): each warp owns 16 rows outright
//     and a CTA of up to four warps shares one staging of K_in and V_in
//     (steps large enough that 64-row CTAs still fill the GPU);
//   - loads are 16-byte cp.async chunks from every thread, K_in and V_in
//     first (a tuning hook switches the split-warp kernel to one bulk copy
//     per row); the parts' L values are plain loads issued early;
//   - S = Q K_in^T and O = P V on mma.sync m16n8k16 (bf16 in, fp32 out) with
//     the block's keys padded to NB in {16, 32, 64}; P V uses a bf16 hi + lo
//     split of P so the product keeps fp32-level accuracy;
//   - the merge with NX (0..4, a template parameter) external parts reads
//     them from shared memory; O (bf16 or fp32), LSE and, on a full step, the
//     merged external part for the cache leave straight from registers.
#include <math_constants.h>

#include "fb_internal.cuh"
#include "fb_ptx.cuh"

namespace fb {

namespace {

constexpr int kRows = 16;          // query rows per CTA (one m16 tile)
constexpr int kD = 128;
constexpr int kRowE = kD + 8;      // bf16 row stride of staged Q, K, V (272 bytes: conflict-free ldmatrix)
constexpr int kExtStride = 132;    // fp32 row stride of staged parts and output rows (bank spread)
constexpr int kMaxExt = 4;
constexpr int kPE = 64 + 8;        // bf16 row stride of the staged P tile (144 bytes: conflict-free ldmatrix)
// bytes of the staged P (hi and lo), the row maxima / sums of up to four
// warps and the CTA's row table (packed row, query and output offsets)
constexpr int kPBytes = 2 * kRows * kPE * 2 + 2 * 4 * kRows * 4 + 3 * kRows * 8;

__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ void ldsm2(uint32_t a, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(a));
}
__device__ __forceinline__ void ldsm4t(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void split2(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  const float hx = __uint_as_float(hi << 16), hy = __uint_as_float(hi & 0xFFFF0000u);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x - hx, y - hy);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

}  // namespace

struct InblockArgs {
  int32_t B, Hq, Hkv, G, Nb;
  int32_t tiles_per_unit;
  const __nv_bfloat16* q;
  int64_t q_sb, q_sh, q_st;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  int64_t k_sb, k_sh, k_st;
  int32_t next;
  const float* ext_a[kMaxExt];
  const float* ext_l[kMaxExt];
  void* o;
  int64_t o_sb, o_sh, o_st;
  int32_t o_bf16;
  float* lse;
  float* cache_a;     // non-null: also store merge(external parts) here (packed fp32)
  float* cache_l;
  float scale_log2;
  int* status;
  uint64_t wait_limit_ns;
  int32_t stall;      // test hook: thread 0 first waits on a barrier nothing completes
  const int32_t* active;  // non-null: [B, n_act] block positions of the queries to compute (the rest untouched)
  int32_t n_act;
  int32_t bulk;           // 1: one bulk copy per row; 0: 16-byte cp.async chunks from every thread
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bounded wait on phase 0 of a load barrier; the first expiry is recorded.  A
// drain (the last wait before exit after an expiry) is bounded by at least
// one second whatever the configured limit, so the CTA never exits with a
// copy into its shared memory in flight.
__device__ __forceinline__ bool wait_loaded(uint32_t bar, const InblockArgs& a, bool drain = false) {
  if (ptx::mbar_test(bar, 0)) return true;
  const uint64_t limit = drain && a.wait_limit_ns < 1000000000ull ? 1000000000ull : a.wait_limit_ns;
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try(bar, 0)) {
    if (ptx::globaltimer() - t0 > limit) {
      atomicCAS(a.status, 0, (int)FB_ETIMEOUT);
      return false;
    }
  }
  return true;
}

template <int NB, int NX>
__global__ void __launch_bounds__(128) inblock_small_kernel(const InblockArgs a) {
  ptx::pdl_prologue();
  constexpr int NT = NB / 8;     // key n-tiles of S
  constexpr int KK = NB / 16;    // key k-steps of P V
  constexpr int NXS = NX > 0 ? NX : 1;
  extern __shared__ __align__(128) uint8_t sm[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(sm);             // [16][kRowE]
  __nv_bfloat16* sK = sQ + kRows * kRowE;                                // [NB][kRowE]
  __nv_bfloat16* sV = sK + NB * kRowE;                                   // [NB][kRowE]
  float* sE = reinterpret_cast<float*>(sV + NB * kRowE);                 // [NX][16][kExtStride]
  float* sL = sE + NXS * kRows * kExtStride;                             // [NX][16]
  __nv_bfloat16* sPh = reinterpret_cast<__nv_bfloat16*>(sL + NXS * kRows);  // [16][kPE] P, bf16 hi
  __nv_bfloat16* sPl = sPh + kRows * kPE;                                   // [16][kPE] P, bf16 lo
  float* sX = reinterpret_cast<float*>(sPl + kRows * kPE);                  // [2][4][16] row maxima, sums
  int64_t* sRowPr = reinterpret_cast<int64_t*>(sX + 2 * 4 * kRows);         // [16] packed (b, h, i) row or -1
  int64_t* sRowQ = sRowPr + kRows;                                          // [16] the row's element offset in q
  int64_t* sRowO = sRowQ + kRows;                                           // [16] the row's element offset in o
  uint64_t* bars = reinterpret_cast<uint64_t*>(sRowO + kRows);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x / a.tiles_per_unit, tile = blockIdx.x % a.tiles_per_unit;
  const int b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int nqh = a.active ? a.n_act : a.Nb;     // queries per head computed
  const int rows_unit = a.G * nqh;
  const int row0 = tile * kRows;
  const int nq = min(kRows, rows_unit - row0);   // rows of this CTA that exist
  // CTA row r -> (query head kvh*G + g, block position i) with g, k = the
  // row's head and index among the computed queries (i = k, or the k-th
  // active position); returns the packed (b, h, i) row of parts and LSE, or
  // -1 for a row that does not exist or names a position outside the block.
  const int g0 = row0 / nqh, k0 = row0 % nqh;   // head and query index of the CTA's first row
  auto row_at = [&](int r, int& h, int& i) -> int64_t {
    if (r >= nq) return -1;
    int g = g0, k = k0 + r;   // row0 + r = g * nqh + k (r < 16: a short walk, no division)
    while (k >= nqh) {
      k -= nqh;
      ++g;
    }
    i = a.active ? a.active[(int64_t)b * a.n_act + k] : k;
    if (i < 0 || i >= a.Nb) return -1;
    h = kvh * a.G + g;
    return ((int64_t)b * a.Hq + h) * a.Nb + i;
  };
  const uint32_t bar_qk = ptx::smem_addr(bars), bar_v = bar_qk + 8, bar_e = bar_qk + 16;

  // ---- every load issued up front: one bulk copy per row (a.bulk), or
  // 16-byte cp.async chunks from all 128 threads in two commit groups (K_in,
  // V_in and Q; the parts), which keeps the SM's copy engine out of the way
  // when a CTA needs a hundred or more rows.  K_in and V_in do not depend on
  // the CTA's rows and go first ----
  const __nv_bfloat16* kb = a.k + b * a.k_sb + (int64_t)kvh * a.k_sh;
  const __nv_bfloat16* vb = a.v + b * a.k_sb + (int64_t)kvh * a.k_sh;
  if (!a.bulk) {
    for (int c = tid; c < NB * 16; c += 128) {      // K rows
      const int r = c >> 4, ch = c & 15;
      if (r < a.Nb)
        cp_async16(ptx::smem_addr(sK + r * kRowE + ch * 8), kb + (int64_t)r * a.k_st + ch * 8);
      else
        *reinterpret_cast<uint4*>(sK + r * kRowE + ch * 8) = make_uint4(0, 0, 0, 0);
    }
    for (int c = tid; c < NB * 16; c += 128) {      // V rows
      const int r = c >> 4, ch = c & 15;
      if (r < a.Nb)
        cp_async16(ptx::smem_addr(sV + r * kRowE + ch * 8), vb + (int64_t)r * a.k_st + ch * 8);
      else
        *reinterpret_cast<uint4*>(sV + r * kRowE + ch * 8) = make_uint4(0, 0, 0, 0);
    }
  }
  // the CTA's row table, one thread per row
  bool valid = false;
  if (tid < kRows) {
    int h = 0, i = 0;
    const int64_t pr = row_at(tid, h, i);
    valid = pr >= 0;
    sRowPr[tid] = pr;
    sRowQ[tid] = valid ? b * a.q_sb + (int64_t)h * a.q_sh + (int64_t)i * a.q_st : 0;
    sRowO[tid] = valid ? b * a.o_sb + (int64_t)h * a.o_sh + (int64_t)i * a.o_st : 0;
  }
  const int nvalid = __syncthreads_count(valid);
  if (tid == 0) {
    if (nvalid < nq) atomicCAS(a.status, 0, (int)FB_EINVAL);
    ptx::mbar_init(bar_qk, 1);
    ptx::mbar_init(bar_v, 1);
    ptx::mbar_init(bar_e, 1);
    ptx::mbar_init(bar_e + 8, 1);
    ptx::fence_mbar_init();
    if (a.bulk) {
      ptx::mbar_expect_tx(bar_qk, (uint32_t)(nvalid + a.Nb) * (kD * 2));
      ptx::mbar_expect_tx(bar_v, (uint32_t)a.Nb * (kD * 2));
      ptx::mbar_expect_tx(bar_e, (uint32_t)(NX * nvalid) * (kD * 4));
    }
  }
  // L of (part, row) = (idx / 16, idx % 16) for idx = tid, tid + 128: read
  // early, stored to shared memory after P V
  float lx[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int idx = tid + k * 128;
    const int64_t pr = idx < NX * kRows ? sRowPr[idx & 15] : -1;
    if (pr >= 0) lx[k] = a.ext_l[idx >> 4][pr];
  }
  if (a.bulk) __syncthreads();   // the barriers' initialisation, before any bulk copy names them
  if (!a.bulk) {
    for (int c = tid; c < kRows * 16; c += 128) {   // Q rows, 16 chunks each
      const int r = c >> 4, ch = c & 15;
      if (sRowPr[r] >= 0)
        cp_async16(ptx::smem_addr(sQ + r * kRowE + ch * 8), a.q + sRowQ[r] + ch * 8);
      else
        *reinterpret_cast<uint4*>(sQ + r * kRowE + ch * 8) = make_uint4(0, 0, 0, 0);
    }
    cp_async_commit();
    for (int c = tid; c < NX * kRows * 32; c += 128) {   // the parts' rows, 32 chunks each
      const int p = c / (kRows * 32), r = (c >> 5) % kRows, ch = c & 31;
      const int64_t pr = sRowPr[r];
      if (pr >= 0)
        cp_async16(ptx::smem_addr(sE + (p * kRows + r) * kExtStride + ch * 4), a.ext_a[p] + pr * kD + ch * 4);
    }
    cp_async_commit();
  } else if (warp == 0) {
    if (lane < kRows) {
      const int r = lane;
      if (sRowPr[r] >= 0) {
        ptx::bulk_g2s(ptx::smem_addr(sQ + r * kRowE), a.q + sRowQ[r], kD * 2, bar_qk);
      } else {
#pragma unroll 1
        for (int c = 0; c < kD / 8; ++c) reinterpret_cast<uint4*>(sQ + r * kRowE)[c] = make_uint4(0, 0, 0, 0);
      }
    }
  } else if (warp == 1 || warp == 2) {
    const bool isk = warp == 1;
    __nv_bfloat16* dst = isk ? sK : sV;
    const __nv_bfloat16* src = isk ? kb : vb;
#pragma unroll 1
    for (int r = lane; r < NB; r += 32) {
      if (r < a.Nb) {
        ptx::bulk_g2s(ptx::smem_addr(dst + r * kRowE), src + (int64_t)r * a.k_st, kD * 2, isk ? bar_qk : bar_v);
      } else {
#pragma unroll 1
        for (int c = 0; c < kD / 8; ++c) reinterpret_cast<uint4*>(dst + r * kRowE)[c] = make_uint4(0, 0, 0, 0);
      }
    }
  } else if (NX > 0) {
    const int p = lane >> 4, r = lane & 15;
    const int64_t pr = sRowPr[r];
#pragma unroll
    for (int pp = 0; pp < NX; pp += 2)
      if (pp + p < NX && pr >= 0)
        ptx::bulk_g2s(ptx::smem_addr(sE + ((pp + p) * kRows + r) * kExtStride), a.ext_a[pp + p] + pr * kD, kD * 4,
                      bar_e);
  }
  if (!a.bulk) cp_async_wait<1>();   // this thread's K, V and Q chunks
  __syncthreads();   // every thread's chunks, and the zero-filled rows
  bool ok = !(a.stall && tid == 0) || wait_loaded(bar_e + 8, a);
  if (a.bulk) ok = wait_loaded(bar_qk, a) && ok;

  // ---- S = Q K^T: warp w forms the key n-tiles [w NTW, (w + 1) NTW) of the
  // CTA's 16 rows (with 16 keys, warps 0 and 1 one n-tile each) ----
  const int dq = warp;   // this warp's quarter of D in P V: columns dq*32 .. dq*32+31
  constexpr int NTW = NT >= 4 ? NT / 4 : 1;   // key n-tiles per S warp
  constexpr int SW = NT / NTW;                // warps that form S
  const bool swarp = warp < SW;
  // two accumulators per n-tile (even and odd k-steps) halve the chain of
  // dependent MMAs
  float s[NTW][4], s2[NTW][4];
#pragma unroll
  for (int n = 0; n < NTW; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[n][e] = s2[n][e] = 0.f;
  if (swarp) {
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      uint32_t qa[4];
      ldsm4(ptx::smem_addr(sQ + (lane & 15) * kRowE + (2 * kk + (lane >> 4)) * 8), qa[0], qa[1], qa[2], qa[3]);
#pragma unroll
      for (int n = 0; n < NTW; n += 2) {
        const int nt = warp * NTW + n;
        float(*acc)[4] = (kk & 1) ? s2 : s;
        if (NTW >= 2) {
          const int r = (nt + (lane >> 4)) * 8 + (lane & 7), ch = 2 * kk + ((lane >> 3) & 1);
          uint32_t b0, b1, b2, b3;
          ldsm4(ptx::smem_addr(sK + r * kRowE + ch * 8), b0, b1, b2, b3);
          mma16816(acc[n], qa, b0, b1);
          mma16816(acc[n + 1], qa, b2, b3);
        } else {
          const int r = nt * 8 + (lane & 7), ch = 2 * kk + ((lane >> 3) & 1);
          uint32_t b0, b1;
          ldsm2(ptx::smem_addr(sK + r * kRowE + ch * 8), b0, b1);
          mma16816(acc[n], qa, b0, b1);
        }
      }
    }
#pragma unroll
    for (int n = 0; n < NTW; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[n][e] += s2[n][e];
  }
  // ---- softmax over the block's keys (rows lane/4 and lane/4 + 8): the
  // row maxima and sums of the S warps meet in shared memory ----
  float mrow[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
  for (int n = 0; n < NTW; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = (warp * NTW + n) * 8 + 2 * (lane & 3) + (e & 1);
      s[n][e] = key < a.Nb ? s[n][e] * a.scale_log2 : -CUDART_INF_F;
      mrow[e >> 1] = fmaxf(mrow[e >> 1], s[n][e]);
    }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 1));
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 2));
  }
  if (swarp && (lane & 3) == 0) {
    sX[warp * kRows + (lane >> 2)] = mrow[0];
    sX[warp * kRows + (lane >> 2) + 8] = mrow[1];
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float m = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < SW; ++w) m = fmaxf(m, sX[w * kRows + (lane >> 2) + 8 * h]);
    mrow[h] = m;
  }
  float lrow[2] = {0.f, 0.f};
  if (swarp) {
#pragma unroll
    for (int n = 0; n < NTW; ++n) {
      const float p0 = ex2(s[n][0] - mrow[0]), p1 = ex2(s[n][1] - mrow[0]);
      const float p2 = ex2(s[n][2] - mrow[1]), p3 = ex2(s[n][3] - mrow[1]);
      lrow[0] += p0 + p1;
      lrow[1] += p2 + p3;
      // P as bf16 hi + lo pairs, rows lane/4 and lane/4 + 8 of the P tile
      const int col = (warp * NTW + n) * 8 + 2 * (lane & 3);
      uint32_t h0, l0, h1, l1;
      split2(p0, p1, h0, l0);
      split2(p2, p3, h1, l1);
      *reinterpret_cast<uint32_t*>(sPh + (lane >> 2) * kPE + col) = h0;
      *reinterpret_cast<uint32_t*>(sPl + (lane >> 2) * kPE + col) = l0;
      *reinterpret_cast<uint32_t*>(sPh + ((lane >> 2) + 8) * kPE + col) = h1;
      *reinterpret_cast<uint32_t*>(sPl + ((lane >> 2) + 8) * kPE + col) = l1;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
      lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
    }
    if ((lane & 3) == 0) {
      sX[(SW + warp) * kRows + (lane >> 2)] = lrow[0];
      sX[(SW + warp) * kRows + (lane >> 2) + 8] = lrow[1];
    }
  }
  if (a.bulk) ok = wait_loaded(bar_v, a) && ok;
  __syncthreads();   // V_in (the bulk copies), P and the row sums
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < SW; ++w) l += sX[(SW + w) * kRows + (lane >> 2) + 8 * h];
    lrow[h] = l;
  }
  // ---- O[:, dq*32 : dq*32+32] = P V ----
  constexpr int DT = 4;    // 8-column tiles in this warp's quarter
  float o[DT][4];
#pragma unroll
  for (int d = 0; d < DT; ++d) o[d][0] = o[d][1] = o[d][2] = o[d][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < KK; ++kk) {
    uint32_t ah[4], al[4];
    ldsm4(ptx::smem_addr(sPh + (lane & 15) * kPE + (2 * kk + (lane >> 4)) * 8), ah[0], ah[1], ah[2], ah[3]);
    ldsm4(ptx::smem_addr(sPl + (lane & 15) * kPE + (2 * kk + (lane >> 4)) * 8), al[0], al[1], al[2], al[3]);
#pragma unroll
    for (int d = 0; d < DT; d += 2) {
      const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, ch = dq * DT + d + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm4t(ptx::smem_addr(sV + r * kRowE + ch * 8), b0, b1, b2, b3);
      mma16816(o[d], ah, b0, b1);
      mma16816(o[d + 1], ah, b2, b3);
      mma16816(o[d], al, b0, b1);
      mma16816(o[d + 1], al, b2, b3);
    }
  }
#pragma unroll
  for (int k = 0; k < 2; ++k)
    if (tid + k * 128 < NX * kRows) sL[tid + k * 128] = lx[k];
  if (a.bulk)
    ok = wait_loaded(bar_e, a) && ok;
  else
    cp_async_wait<0>();
  __syncthreads();   // sL (and the parts' rows)
  // ---- merge with the external parts; rows staged for whole-row stores ----
  const bool obf = a.o_bf16 != 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = (lane >> 2) + 8 * h;
    const int64_t pr = sRowPr[r];
    if (pr < 0) continue;
    const int64_t obase = sRowO[r];
    const float Lin = lrow[h] > 0.f ? (mrow[h] + __log2f(lrow[h])) * kLn2 : -CUDART_INF_F;
    float m = Lin;
    float Lx[NXS];
#pragma unroll
    for (int p = 0; p < NX; ++p) {
      Lx[p] = sL[p * kRows + r];
      m = fmaxf(m, Lx[p]);
    }
    const bool empty = m == -CUDART_INF_F;
    const float w_in = (empty || Lin == -CUDART_INF_F) ? 0.f : __expf(Lin - m);
    float wx[NXS], wext = 0.f;
#pragma unroll
    for (int p = 0; p < NX; ++p) {
      wx[p] = (empty || Lx[p] == -CUDART_INF_F) ? 0.f : __expf(Lx[p] - m);
      wext += wx[p];
    }
    const float wsum = w_in + wext;
    const float inv = empty ? 0.f : 1.f / wsum;
    const float inv_ext = wext > 0.f ? 1.f / wext : 0.f;
    const float win = lrow[h] > 0.f ? w_in / lrow[h] : 0.f;
#pragma unroll
    for (int d = 0; d < DT; ++d) {
      const int col = dq * 32 + d * 8 + 2 * (lane & 3);
      float ex = 0.f, ey = 0.f;   // sum of w_p A_p over the external parts (a part with w = 0 may hold -inf rows)
#pragma unroll
      for (int p = 0; p < NX; ++p) {
        const float2 e = *reinterpret_cast<const float2*>(sE + (p * kRows + r) * kExtStride + col);
        ex = wx[p] == 0.f ? ex : fmaf(wx[p], e.x, ex);
        ey = wx[p] == 0.f ? ey : fmaf(wx[p], e.y, ey);
      }
      if (a.cache_a) *reinterpret_cast<float2*>(a.cache_a + pr * kD + col) = make_float2(ex * inv_ext, ey * inv_ext);
      const float x = (win * o[d][2 * h] + ex) * inv, y = (win * o[d][2 * h + 1] + ey) * inv;
      if (obf)
        *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.o) + obase + col) = __floats2bfloat162_rn(x, y);
      else
        *reinterpret_cast<float2*>(static_cast<float*>(a.o) + obase + col) = make_float2(x, y);
    }
    if (dq == 0 && (lane & 3) == 0) {
      if (a.cache_l) a.cache_l[pr] = wext > 0.f ? m + logf(wext) : -CUDART_INF_F;
      if (a.lse) a.lse[pr] = empty ? -CUDART_INF_F : m + logf(wsum);
    }
  }
  if (!ok && tid == 0 && a.bulk) {
    // a load wait expired: let every copy into shared memory land before exit
    wait_loaded(bar_qk, a, true);
    wait_loaded(bar_v, a, true);
    wait_loaded(bar_e, a, true);
  }
}

// ------------------------------------------------- warp-per-rows variant --
// The same step with each warp owning 16 query rows outright: S for all the
// block's keys, the softmax in registers (the S accumulators become the A
// fragments of P V), P V over the whole head dimension, the merge and the
// stores, with no exchange between warps.  A CTA of W warps takes 16 W rows
// of one KV head, so K_in and V_in are staged once per 16 W rows (the
// per-16-row kernel above stages them once per 16 rows); O, LSE and the
// cache rows leave straight from registers.
template <int NB, int NX>
__global__ void __launch_bounds__(128) inblock_rows_kernel(const InblockArgs a) {
  ptx::pdl_prologue();
  constexpr int NT = NB / 8;     // key n-tiles of S
  constexpr int KK = NB / 16;    // key k-steps of P V
  constexpr int NXS = NX > 0 ? NX : 1;
  const int W = blockDim.x >> 5;
  extern __shared__ __align__(128) uint8_t sm[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(sm);   // [NB][kRowE]
  __nv_bfloat16* sV = sK + NB * kRowE;                          // [NB][kRowE]
  __nv_bfloat16* sQ = sV + NB * kRowE;                          // [16 W][kRowE]
  float* sE = reinterpret_cast<float*>(sQ + W * kRows * kRowE);  // [NX][16 W][kExtStride]
  uint64_t* sbar = reinterpret_cast<uint64_t*>(sE + NXS * W * kRows * kExtStride);
  int* sok = reinterpret_cast<int*>(sbar + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x / a.tiles_per_unit, tile = blockIdx.x % a.tiles_per_unit;
  const int b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int nqh = a.active ? a.n_act : a.Nb;     // queries per head computed
  const int rows_unit = a.G * nqh;
  const int wrow0 = (tile * W + warp) * kRows;   // the warp's first row among the KV head's rows
  const bool has_rows = wrow0 < rows_unit;

  // ---- K_in and V_in (every thread, 16-byte chunks; rows past the block
  // are zero) ----
  const __nv_bfloat16* kb = a.k + b * a.k_sb + (int64_t)kvh * a.k_sh;
  const __nv_bfloat16* vb = a.v + b * a.k_sb + (int64_t)kvh * a.k_sh;
  for (int c = tid; c < NB * 16; c += blockDim.x) {
    const int r = c >> 4, ch = c & 15;
    if (r < a.Nb) {
      cp_async16(ptx::smem_addr(sK + r * kRowE + ch * 8), kb + (int64_t)r * a.k_st + ch * 8);
      cp_async16(ptx::smem_addr(sV + r * kRowE + ch * 8), vb + (int64_t)r * a.k_st + ch * 8);
    } else {
      *reinterpret_cast<uint4*>(sK + r * kRowE + ch * 8) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sV + r * kRowE + ch * 8) = make_uint4(0, 0, 0, 0);
    }
  }
  // ---- this warp's rows: lane r < 16 maps row wrow0 + r to its packed
  // (b, h, i) row (or -1) and its Q and O offsets ----
  int64_t pr = -1, qoff = 0, ooff = 0;
  if (lane < kRows && wrow0 + lane < rows_unit) {
    const int rr = wrow0 + lane;
    const int g = rr / nqh, k = rr - g * nqh;
    const int i = a.active ? a.active[(int64_t)b * a.n_act + k] : k;
    if (i >= 0 && i < a.Nb) {
      const int h = kvh * a.G + g;
      pr = ((int64_t)b * a.Hq + h) * a.Nb + i;
      qoff = b * a.q_sb + (int64_t)h * a.q_sh + (int64_t)i * a.q_st;
      ooff = b * a.o_sb + (int64_t)h * a.o_sh + (int64_t)i * a.o_st;
    } else {
      atomicCAS(a.status, 0, (int)FB_EINVAL);   // an active position outside the block
    }
  }
  // Q rows of the warp (16 chunks each), then the parts' rows (32 chunks)
  __nv_bfloat16* sQw = sQ + warp * kRows * kRowE;
#pragma unroll
  for (int c = lane; c < kRows * 16; c += 32) {
    const int r = c >> 4, ch = c & 15;
    const int64_t prr = __shfl_sync(0xffffffffu, pr, r), qo = __shfl_sync(0xffffffffu, qoff, r);
    if (prr >= 0)
      cp_async16(ptx::smem_addr(sQw + r * kRowE + ch * 8), a.q + qo + ch * 8);
    else
      *reinterpret_cast<uint4*>(sQw + r * kRowE + ch * 8) = make_uint4(0, 0, 0, 0);
  }
  cp_async_commit();   // K_in, V_in, Q
#pragma unroll
  for (int p = 0; p < NX; ++p)
#pragma unroll 4
    for (int c = lane; c < kRows * 32; c += 32) {
      const int r = c >> 5, ch = c & 31;
      const int64_t prr = __shfl_sync(0xffffffffu, pr, r);
      if (prr >= 0)
        cp_async16(ptx::smem_addr(sE + ((p * W + warp) * kRows + r) * kExtStride + ch * 4),
                   a.ext_a[p] + prr * kD + ch * 4);
    }
  cp_async_commit();   // the parts
  // the rows of this lane's accumulators (lane/4 and lane/4 + 8) and their
  // parts' L, read early
  int64_t prh[2];
  float lx[2][NXS];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    prh[h] = __shfl_sync(0xffffffffu, pr, (lane >> 2) + 8 * h);
#pragma unroll
    for (int p = 0; p < NXS; ++p) lx[h][p] = (p < NX && prh[h] >= 0) ? a.ext_l[p][prh[h]] : -CUDART_INF_F;
  }
  if (tid == 0) {
    *sok = 1;
    if (a.stall) {   // test hook: a wait that nothing completes runs out
      ptx::mbar_init(ptx::smem_addr(sbar), 1);
      ptx::fence_mbar_init();
      if (!wait_loaded(ptx::smem_addr(sbar), a)) *sok = 0;
    }
  }
  cp_async_wait<1>();   // this thread's K, V and Q chunks
  __syncthreads();      // every thread's chunks, the zero-filled rows and the stall outcome
  if (!*sok || !has_rows) {
    cp_async_wait<0>();
    return;
  }

  // ---- S = Q K^T for the warp's 16 rows and all NB keys ----
  float s[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    uint32_t qa[4];
    ldsm4(ptx::smem_addr(sQw + (lane & 15) * kRowE + (2 * kk + (lane >> 4)) * 8), qa[0], qa[1], qa[2], qa[3]);
#pragma unroll
    for (int n = 0; n < NT; n += 2) {
      const int r = (n + (lane >> 4)) * 8 + (lane & 7), ch = 2 * kk + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm4(ptx::smem_addr(sK + r * kRowE + ch * 8), b0, b1, b2, b3);
      mma16816(s[n], qa, b0, b1);
      mma16816(s[n + 1], qa, b2, b3);
    }
  }
  // ---- softmax of rows lane/4 and lane/4 + 8 (a quad holds a row) ----
  float mrow[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = n * 8 + 2 * (lane & 3) + (e & 1);
      s[n][e] = key < a.Nb ? s[n][e] * a.scale_log2 : -CUDART_INF_F;
      mrow[e >> 1] = fmaxf(mrow[e >> 1], s[n][e]);
    }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 1));
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 2));
  }
  const float mref[2] = {mrow[0] == -CUDART_INF_F ? 0.f : mrow[0], mrow[1] == -CUDART_INF_F ? 0.f : mrow[1]};
  float lrow[2] = {0.f, 0.f};
  // P as bf16 hi + lo A fragments: k-step kk covers n-tiles 2kk and 2kk + 1
  uint32_t ph[KK][4], pl[KK][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const float p0 = ex2(s[n][0] - mref[0]), p1 = ex2(s[n][1] - mref[0]);
    const float p2 = ex2(s[n][2] - mref[1]), p3 = ex2(s[n][3] - mref[1]);
    lrow[0] += p0 + p1;
    lrow[1] += p2 + p3;
    const int kk = n >> 1, hf = (n & 1) * 2;
    split2(p0, p1, ph[kk][hf], pl[kk][hf]);
    split2(p2, p3, ph[kk][hf + 1], pl[kk][hf + 1]);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
  }
  // ---- O = P V over the whole head dimension (16 column tiles) ----
  float o[kD / 8][4];
#pragma unroll
  for (int d = 0; d < kD / 8; ++d) o[d][0] = o[d][1] = o[d][2] = o[d][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < KK; ++kk) {
#pragma unroll
    for (int d = 0; d < kD / 8; d += 2) {
      const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, ch = d + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm4t(ptx::smem_addr(sV + r * kRowE + ch * 8), b0, b1, b2, b3);
      mma16816(o[d], ph[kk], b0, b1);
      mma16816(o[d + 1], ph[kk], b2, b3);
      mma16816(o[d], pl[kk], b0, b1);
      mma16816(o[d + 1], pl[kk], b2, b3);
    }
  }
  cp_async_wait<0>();   // this lane's part chunks
  __syncwarp();         // and the rest of the warp's
  // ---- merge with the external parts; stores straight from registers ----
  const bool obf = a.o_bf16 != 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = (lane >> 2) + 8 * h;
    const int64_t obase = __shfl_sync(0xffffffffu, ooff, r);   // every lane takes part in the shuffle
    if (prh[h] < 0) continue;
    const float Lin = lrow[h] > 0.f ? (mrow[h] + __log2f(lrow[h])) * kLn2 : -CUDART_INF_F;
    float m = Lin;
#pragma unroll
    for (int p = 0; p < NX; ++p) m = fmaxf(m, lx[h][p]);
    const bool empty = m == -CUDART_INF_F;
    const float w_in = (empty || Lin == -CUDART_INF_F) ? 0.f : __expf(Lin - m);
    float wx[NXS], wext = 0.f;
#pragma unroll
    for (int p = 0; p < NXS; ++p) {
      wx[p] = (p >= NX || empty || lx[h][p] == -CUDART_INF_F) ? 0.f : __expf(lx[h][p] - m);
      wext += wx[p];
    }
    const float wsum = w_in + wext;
    const float inv = empty ? 0.f : 1.f / wsum;
    const float inv_ext = wext > 0.f ? 1.f / wext : 0.f;
    const float win = lrow[h] > 0.f ? w_in / lrow[h] : 0.f;
#pragma unroll
    for (int d = 0; d < kD / 8; ++d) {
      const int col = d * 8 + 2 * (lane & 3);
      float ex = 0.f, ey = 0.f;   // sum of w_p A_p (a part with w = 0 may hold -inf rows)
#pragma unroll
      for (int p = 0; p < NX; ++p) {
        const float2 e = *reinterpret_cast<const float2*>(sE + ((p * W + warp) * kRows + r) * kExtStride + col);
        ex = wx[p] == 0.f ? ex : fmaf(wx[p], e.x, ex);
        ey = wx[p] == 0.f ? ey : fmaf(wx[p], e.y, ey);
      }
      if (a.cache_a) *reinterpret_cast<float2*>(a.cache_a + prh[h] * kD + col) = make_float2(ex * inv_ext, ey * inv_ext);
      const float x = (win * o[d][2 * h] + ex) * inv, y = (win * o[d][2 * h + 1] + ey) * inv;
      if (obf)
        *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.o) + obase + col) = __floats2bfloat162_rn(x, y);
      else
        *reinterpret_cast<float2*>(static_cast<float*>(a.o) + obase + col) = make_float2(x, y);
    }
    if ((lane & 3) == 0) {
      if (a.cache_l) a.cache_l[prh[h]] = wext > 0.f ? m + logf(wext) : -CUDART_INF_F;
      if (a.lse) a.lse[prh[h]] = empty ? -CUDART_INF_F : m + logf(wsum);
    }
  }
}

// ------------------------------------------------------------------ host --
int* device_status_ptr();
uint64_t wait_limit_ns();

bool inblock_small_applies(const fb_attn_desc& d, int next) {
  return d.in_dtype == FB_BF16 && d.D == kD && d.Nb <= 64 && next <= kMaxExt;
}

cudaError_t launch_inblock_small(const fb_attn_desc& d, const void* q, const void* kin, const void* vin, int next,
                                 const float* const* ext_a, const float* const* ext_l, void* o, float* lse,
                                 float* cache_a, float* cache_l, float scale_log2, cudaStream_t s,
                                 const int32_t* active, int32_t n_act) {
  InblockArgs a;
  memset(&a, 0, sizeof(a));
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.G = d.Hq / d.Hkv; a.Nb = d.Nb;
  a.active = active;
  a.n_act = active ? n_act : d.Nb;
  a.tiles_per_unit = (a.G * a.n_act + kRows - 1) / kRows;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.q_sb = d.q_strides[0]; a.q_sh = d.q_strides[1]; a.q_st = d.q_strides[2];
  a.k = static_cast<const __nv_bfloat16*>(kin);
  a.v = static_cast<const __nv_bfloat16*>(vin);
  a.k_sb = d.kin_strides[0]; a.k_sh = d.kin_strides[1]; a.k_st = d.kin_strides[2];
  a.next = next;
  for (int p = 0; p < next; ++p) { a.ext_a[p] = ext_a[p]; a.ext_l[p] = ext_l[p]; }
  a.o = o; a.o_sb = d.o_strides[0]; a.o_sh = d.o_strides[1]; a.o_st = d.o_strides[2];
  a.o_bf16 = d.out_dtype == FB_BF16;
  a.lse = lse;
  a.cache_a = cache_a;
  a.cache_l = cache_l;
  a.scale_log2 = scale_log2;
  a.status = device_status_ptr();
  a.wait_limit_ns = wait_limit_ns();
  a.stall = debug_stall() ? 1 : 0;
  a.bulk = inblock_bulk_loads() ? 1 : 0;
  if (!a.status) return cudaErrorInvalidValue;
  const int NB = d.Nb <= 16 ? 16 : d.Nb <= 32 ? 32 : 64;
  const int nxs = next > 0 ? next : 1;
  const int rows_unit = a.G * a.n_act;
  const int units = d.B * d.Hkv;
  const int dev = current_device();
  int W = inblock_rows_setting() / kRows;   // 0: automatic; -1 below: the split-warp kernel
  if (inblock_rows_setting() == 1) W = -1;
  if (W == 0) {
    // measured: 64-row CTAs win where they still fill about the whole GPU
    // (dllm_64k_b4: 7.7 vs 8.3 us); with fewer CTAs than that the split-warp
    // kernel's short per-warp chains win (dllm_8k 5.2 vs 6.1 us, blocks of
    // 4: 4.9 vs 5.1 us)
    W = (int64_t)units * ((rows_unit + 4 * kRows - 1) / (4 * kRows)) >= (num_sms() * 3) / 4 ? 4 : -1;
  }
  if (W > 0) {
    a.tiles_per_unit = (rows_unit + kRows * W - 1) / (kRows * W);
    const size_t smem_r = (size_t)(2 * NB + W * kRows) * kRowE * 2 + (size_t)nxs * W * kRows * kExtStride * 4 + 16;
    const dim3 grid_r(units * a.tiles_per_unit);
    static bool opted_r[kMaxDevices][3][kMaxExt + 1] = {};
    auto run_r = [&](void (*kern)(InblockArgs), int nbi) -> cudaError_t {
      if (smem_r > 48 * 1024 && !opted_r[dev][nbi][next]) {
        // sized for the largest CTA this instance can get
        const size_t most = (size_t)(2 * NB + 4 * kRows) * kRowE * 2 + (size_t)nxs * 4 * kRows * kExtStride * 4 + 16;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most);
        if (e != cudaSuccess) return e;
        opted_r[dev][nbi][next] = true;
      }
      return launch_k(kern, grid_r, dim3(32 * W), smem_r, s, a);
    };
#define FB_INR_CASE(nb, nx) \
  if (NB == nb && next == nx) return run_r(inblock_rows_kernel<nb, nx>, nb == 16 ? 0 : nb == 32 ? 1 : 2);
#define FB_INR_NB(nb) FB_INR_CASE(nb, 0) FB_INR_CASE(nb, 1) FB_INR_CASE(nb, 2) FB_INR_CASE(nb, 3) FB_INR_CASE(nb, 4)
    FB_INR_NB(16)
    FB_INR_NB(32)
    FB_INR_NB(64)
#undef FB_INR_NB
#undef FB_INR_CASE
    return cudaErrorInvalidValue;
  }
  const size_t smem = (size_t)(kRows + 2 * NB) * kRowE * 2 + (size_t)nxs * kRows * (kExtStride + 1) * 4 + kPBytes + 4 * 8;
  const dim3 grid(d.B * d.Hkv * a.tiles_per_unit);
  // instances above the default 48 KB of dynamic shared memory opt in once
  static bool opted[kMaxDevices][3][kMaxExt + 1] = {};   // the attribute is per device
  auto run = [&](void (*kern)(InblockArgs), int nbi) -> cudaError_t {
    if (smem > 48 * 1024 && !opted[dev][nbi][next]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      opted[dev][nbi][next] = true;
    }
    return launch_k(kern, grid, dim3(128), smem, s, a);
  };
#define FB_INB_CASE(nb, nx) \
  if (NB == nb && next == nx) return run(inblock_small_kernel<nb, nx>, nb == 16 ? 0 : nb == 32 ? 1 : 2);
#define FB_INB_NB(nb) FB_INB_CASE(nb, 0) FB_INB_CASE(nb, 1) FB_INB_CASE(nb, 2) FB_INB_CASE(nb, 3) FB_INB_CASE(nb, 4)
  FB_INB_NB(16)
  FB_INB_NB(32)
  FB_INB_NB(64)
#undef FB_INB_NB
#undef FB_INB_CASE
  return cudaErrorInvalidValue;
}

}  // namespace fb
