// Block-internal attention fused with the log-space merge, for small blocks
// (FlashBlock summary, "Mécanisme Central": A_in over the block's own keys
// J_in, then A = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (...)).  This is the
// whole reuse step of a diffusion LM, so it is built for latency:
//   - one CTA = 32 packed query rows of one KV head (G query heads x Nb
//     queries); 4 warps: two 16-row slabs, and for each slab two warps that
//     both form S and P but split the P V product and the epilogue by halves
//     of the head dimension (shorter per-warp instruction chains);
//   - every global load (Q, K_in, V_in and the external parts A, L) is issued
//     up front with cp.async in three groups (Q and K_in; V_in; the parts), so
//     S and the softmax start while V_in and the parts are still arriving;
//   - S = Q K_in^T and O = P V on mma.sync m16n8k16 (bf16 in, fp32 out) with
//     the block's keys padded to NB in {16, 32, 64}; P V uses a bf16 hi + lo
//     split of P so the product keeps fp32-level accuracy;
//   - the merge with up to four external parts reads them from shared memory
//     and writes O (bf16 or fp32) and the merged natural-log LSE; on a full
//     step it can also write the merged external part (the block-external
//     attention combined over its key splits) into the cache.
#include <math_constants.h>

#include "fb_internal.cuh"

namespace fb {

namespace {

constexpr int kRows = 32;          // query rows per CTA
constexpr int kD = 128;
constexpr int kExtStride = 132;    // fp32 row stride of staged external parts (bank spread)
constexpr int kMaxExt = 4;

__device__ __forceinline__ uint32_t saddr(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes));
}
__device__ __forceinline__ void cp4(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(bytes));
}
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
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
// swizzled offset (elements) of 16-byte chunk `ch` of row `r` in a [rows][128] bf16 tile
__device__ __forceinline__ int swz(int r, int ch) { return r * kD + ((ch ^ (r & 7)) << 3); }

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
};

template <int NB>
__global__ void __launch_bounds__(128) inblock_small_kernel(const InblockArgs a) {
  constexpr int NT = NB / 8;     // key n-tiles of S
  constexpr int KK = NB / 16;    // key k-steps of P V
  extern __shared__ __align__(128) uint8_t sm[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(sm);             // [64][128]
  __nv_bfloat16* sK = sQ + kRows * kD;                                   // [NB][128]
  __nv_bfloat16* sV = sK + NB * kD;                                      // [NB][128]
  float* sE = reinterpret_cast<float*>(sV + NB * kD);                    // [next][64][132]
  float* sL = sE + kMaxExt * kRows * kExtStride;                         // [next][64]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x / a.tiles_per_unit, tile = blockIdx.x % a.tiles_per_unit;
  const int b = unit / a.Hkv, kvh = unit % a.Hkv;
  const int rows_unit = a.G * a.Nb;
  const int row0 = tile * kRows;
  // packed row r -> (query head kvh*G + r / Nb, query r % Nb); the rows of one
  // KV head are consecutive in the packed (b, h, i) order of parts and LSE.
  const int64_t prow0 = ((int64_t)b * a.Hq + (int64_t)kvh * a.G) * a.Nb + row0;

  if (tid == 0) {
    // warm the address translation of the rows this CTA stores at the end
    const int g = min(row0 / a.Nb, a.G - 1), i = row0 % a.Nb;
    const size_t esz = a.o_bf16 ? 2 : 4;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const char*>(a.o) +
                                                  (b * a.o_sb + (int64_t)(kvh * a.G + g) * a.o_sh +
                                                   (int64_t)i * a.o_st) * esz));
    if (a.cache_a) asm volatile("prefetch.global.L2 [%0];" ::"l"(a.cache_a + prow0 * kD));
    if (a.lse) asm volatile("prefetch.global.L2 [%0];" ::"l"(a.lse + prow0));
  }
  // ---- one batch of asynchronous loads ----
  for (int c = tid; c < kRows * 16; c += 128) {
    const int r = c >> 4, ch = c & 15;
    const int rr = row0 + r;
    const bool ok = rr < rows_unit;
    const int g = ok ? rr / a.Nb : 0, i = ok ? rr % a.Nb : 0;
    const __nv_bfloat16* src = a.q + b * a.q_sb + (int64_t)(kvh * a.G + g) * a.q_sh + (int64_t)i * a.q_st + ch * 8;
    cp16(saddr(sQ + swz(r, ch)), ok ? src : a.q, ok ? 16 : 0);
  }
  for (int c = tid; c < NB * 16; c += 128) {
    const int r = c >> 4, ch = c & 15;
    const bool ok = r < a.Nb;
    const int64_t off = b * a.k_sb + (int64_t)kvh * a.k_sh + (int64_t)(ok ? r : 0) * a.k_st + ch * 8;
    cp16(saddr(sK + swz(r, ch)), a.k + off, ok ? 16 : 0);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");   // group: Q, K_in
  for (int c = tid; c < NB * 16; c += 128) {
    const int r = c >> 4, ch = c & 15;
    const bool ok = r < a.Nb;
    const int64_t off = b * a.k_sb + (int64_t)kvh * a.k_sh + (int64_t)(ok ? r : 0) * a.k_st + ch * 8;
    cp16(saddr(sV + swz(r, ch)), a.v + off, ok ? 16 : 0);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");   // group: V_in
  for (int p = 0; p < a.next; ++p) {
    for (int c = tid; c < kRows * 32; c += 128) {
      const int r = c >> 5, ch = c & 31;
      const bool ok = row0 + r < rows_unit;
      cp16(saddr(sE + (p * kRows + r) * kExtStride + ch * 4), ok ? a.ext_a[p] + (prow0 + r) * kD + ch * 4 : a.ext_a[p],
           ok ? 16 : 0);
    }
    for (int r = tid; r < kRows; r += 128) {
      const bool ok = row0 + r < rows_unit;
      cp4(saddr(sL + p * kRows + r), ok ? a.ext_l[p] + prow0 + r : a.ext_l[p], ok ? 4 : 0);
    }
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 2;\n" ::: "memory");   // group: parts
  __syncthreads();

  // ---- S = Q K^T for this warp's 16-row slab ----
  const int slab = warp & 1, dh = warp >> 1;   // dh: which 64 columns of D this warp outputs
  float s[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk) {
    uint32_t qa[4];
    {
      const int r = slab * 16 + (lane & 15), ch = 2 * kk + (lane >> 4);
      ldsm4(saddr(sQ + swz(r, ch)), qa[0], qa[1], qa[2], qa[3]);
    }
#pragma unroll
    for (int n = 0; n < NT; n += 2) {
      const int r = (n + (lane >> 4)) * 8 + (lane & 7), ch = 2 * kk + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm4(saddr(sK + swz(r, ch)), b0, b1, b2, b3);
      mma16816(s[n], qa, b0, b1);
      if (n + 1 < NT) mma16816(s[n + 1], qa, b2, b3);
    }
  }
  // ---- softmax over the block's keys (rows lane/4 and lane/4 + 8) ----
  float mrow[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = n * 8 + 2 * (lane & 3) + (e & 1);
      s[n][e] = key < a.Nb ? s[n][e] * a.scale_log2 : -CUDART_INF_F;
      mrow[e >> 1] = fmaxf(mrow[e >> 1], s[n][e]);
    }
  float lrow[2] = {0.f, 0.f};
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 1));
    mrow[h] = fmaxf(mrow[h], __shfl_xor_sync(0xffffffffu, mrow[h], 2));
  }
  uint32_t ph[NT][2], pl[NT][2];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const float p0 = ex2(s[n][0] - mrow[0]), p1 = ex2(s[n][1] - mrow[0]);
    const float p2 = ex2(s[n][2] - mrow[1]), p3 = ex2(s[n][3] - mrow[1]);
    lrow[0] += p0 + p1;
    lrow[1] += p2 + p3;
    split2(p0, p1, ph[n][0], pl[n][0]);
    split2(p2, p3, ph[n][1], pl[n][1]);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 1);
    lrow[h] += __shfl_xor_sync(0xffffffffu, lrow[h], 2);
  }
  asm volatile("cp.async.wait_group 1;\n" ::: "memory");
  __syncthreads();
  // ---- O[:, dh*64 : dh*64+64] = P V ----
  constexpr int DT = kD / 16;    // 8-column tiles in this warp's half
  float o[DT][4];
#pragma unroll
  for (int d = 0; d < DT; ++d) o[d][0] = o[d][1] = o[d][2] = o[d][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < KK; ++kk) {
    const uint32_t ah[4] = {ph[2 * kk][0], ph[2 * kk][1], ph[2 * kk + 1][0], ph[2 * kk + 1][1]};
    const uint32_t al[4] = {pl[2 * kk][0], pl[2 * kk][1], pl[2 * kk + 1][0], pl[2 * kk + 1][1]};
#pragma unroll
    for (int d = 0; d < DT; d += 2) {
      const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, ch = dh * DT + d + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm4t(saddr(sV + swz(r, ch)), b0, b1, b2, b3);
      mma16816(o[d], ah, b0, b1);
      mma16816(o[d + 1], ah, b2, b3);
      mma16816(o[d], al, b0, b1);
      mma16816(o[d + 1], al, b2, b3);
    }
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();
  // ---- merge with the external parts and store ----
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = slab * 16 + (lane >> 2) + 8 * h;
    const int rr = row0 + r;
    if (rr >= rows_unit) continue;
    const float Lin = lrow[h] > 0.f ? (mrow[h] + __log2f(lrow[h])) * kLn2 : -CUDART_INF_F;
    float Lx[kMaxExt];
    float m = Lin;
#pragma unroll
    for (int p = 0; p < kMaxExt; ++p) {
      Lx[p] = p < a.next ? sL[p * kRows + r] : -CUDART_INF_F;
      m = fmaxf(m, Lx[p]);
    }
    const bool empty = m == -CUDART_INF_F;
    const float w_in = (empty || Lin == -CUDART_INF_F) ? 0.f : __expf(Lin - m);
    float wx[kMaxExt], wext = 0.f;
#pragma unroll
    for (int p = 0; p < kMaxExt; ++p) {
      wx[p] = (empty || Lx[p] == -CUDART_INF_F) ? 0.f : __expf(Lx[p] - m);
      wext += wx[p];
    }
    const float wsum = w_in + wext;
    const float inv = empty ? 0.f : 1.f / wsum;
    const float inv_ext = wext > 0.f ? 1.f / wext : 0.f;
    const float win = lrow[h] > 0.f ? w_in / lrow[h] : 0.f;
    const int g = rr / a.Nb, i = rr % a.Nb;
    const int64_t obase = b * a.o_sb + (int64_t)(kvh * a.G + g) * a.o_sh + (int64_t)i * a.o_st;
#pragma unroll
    for (int d = 0; d < DT; ++d) {
      const int col = dh * 64 + d * 8 + 2 * (lane & 3);
      float ex = 0.f, ey = 0.f;   // sum of w_p A_p over the external parts
#pragma unroll
      for (int p = 0; p < kMaxExt; ++p) {
        if (wx[p] == 0.f) continue;
        const float2 e = *reinterpret_cast<const float2*>(sE + (p * kRows + r) * kExtStride + col);
        ex = fmaf(wx[p], e.x, ex);
        ey = fmaf(wx[p], e.y, ey);
      }
      if (a.cache_a)
        *reinterpret_cast<float2*>(a.cache_a + (prow0 + r) * kD + col) = make_float2(ex * inv_ext, ey * inv_ext);
      const float x = (win * o[d][2 * h] + ex) * inv, y = (win * o[d][2 * h + 1] + ey) * inv;
      if (a.o_bf16)
        *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.o) + obase + col) = __floats2bfloat162_rn(x, y);
      else
        *reinterpret_cast<float2*>(static_cast<float*>(a.o) + obase + col) = make_float2(x, y);
    }
    if (a.cache_l && dh == 0 && (lane & 3) == 0)
      a.cache_l[prow0 + r] = wext > 0.f ? m + logf(wext) : -CUDART_INF_F;
    if (a.lse && dh == 0 && (lane & 3) == 0) a.lse[prow0 + r] = empty ? -CUDART_INF_F : m + logf(wsum);
  }
}

// ------------------------------------------------------------------ host --
bool inblock_small_applies(const fb_attn_desc& d, int next) {
  return d.in_dtype == FB_BF16 && d.D == kD && d.Nb <= 64 && next <= kMaxExt;
}

cudaError_t launch_inblock_small(const fb_attn_desc& d, const void* q, const void* kin, const void* vin, int next,
                                 const float* const* ext_a, const float* const* ext_l, void* o, float* lse,
                                 float* cache_a, float* cache_l, float scale_log2, cudaStream_t s) {
  InblockArgs a;
  memset(&a, 0, sizeof(a));
  a.B = d.B; a.Hq = d.Hq; a.Hkv = d.Hkv; a.G = d.Hq / d.Hkv; a.Nb = d.Nb;
  a.tiles_per_unit = (a.G * d.Nb + kRows - 1) / kRows;
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
  const int NB = d.Nb <= 16 ? 16 : d.Nb <= 32 ? 32 : 64;
  const size_t smem = (size_t)(kRows + 2 * NB) * kD * 2 + (size_t)kMaxExt * kRows * (kExtStride + 1) * 4;
  const dim3 grid(d.B * d.Hkv * a.tiles_per_unit);
  static bool attr[3] = {false, false, false};
  auto run = [&](auto kern, int idx) -> cudaError_t {
    if (!attr[idx]) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      attr[idx] = true;
    }
    kern<<<grid, 128, smem, s>>>(a);
    return cudaGetLastError();
  };
  if (NB == 16) return run(inblock_small_kernel<16>, 0);
  if (NB == 32) return run(inblock_small_kernel<32>, 1);
  return run(inblock_small_kernel<64>, 2);
}

}  // namespace fb
