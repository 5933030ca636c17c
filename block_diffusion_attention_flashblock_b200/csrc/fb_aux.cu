// Row-wise kernels of libfb: the N-way log-space merge, the gamma-gate
// similarity/cache update, the KV-cache append and the sparse membership
// bitmap (FlashBlock summary, "Mécanisme Central" and "Stratégies de
// Réutilisation Adaptatives").
#include "fb_internal.cuh"
#include "fb_ptx.cuh"
#include <cub/block/block_scan.cuh>
#include <math_constants.h>

namespace fb {

namespace {

template <int D>
struct Vec;  // D/32 fp32 values per lane
template <>
struct Vec<64> {
  float v[2];
  __device__ void load(const float* p) {
    const float2 x = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = x.x; v[1] = x.y;
  }
  __device__ void store(float* p) const { *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]); }
};
template <>
struct Vec<128> {
  float v[4];
  __device__ void load(const float* p) {
    const float4 x = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  }
  __device__ void store(float* p) const { *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]); }
};

template <int D>
__device__ __forceinline__ void store_out(void* o, int64_t off, bool bf16, const float* v) {
  constexpr int E = D / 32;
  if (bf16) {
    __nv_bfloat16* p = static_cast<__nv_bfloat16*>(o) + off;
#pragma unroll
    for (int e = 0; e < E; e += 2)
      *reinterpret_cast<__nv_bfloat162*>(p + e) = __floats2bfloat162_rn(v[e], v[e + 1]);
  } else {
    float* p = static_cast<float*>(o) + off;
#pragma unroll
    for (int e = 0; e < E; e += 2) *reinterpret_cast<float2*>(p + e) = make_float2(v[e], v[e + 1]);
  }
}

// Merge all parts of one row (lane holds columns lane*E .. lane*E+E-1):
// m = max L_p, w_p = e^{L_p - m}; returns sum w_p A_p / sum w_p and the LSE.
// Parts are taken in batches of U whose loads are all issued before any is
// used, with a running max across batches, so a row costs one memory round
// trip per U parts; the summation order is fixed.
template <int D>
__device__ __forceinline__ float merge_row(const PartList& pl, int64_t row, int lane, float* out) {
  constexpr int E = D / 32, U = 16;
  float m = -CUDART_INF_F, wsum = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] = 0.f;
  for (int gi = 0; gi < pl.ngroups; ++gi) {
    const PartGroup& g = pl.g[gi];
    for (int p0 = 0; p0 < g.count; p0 += U) {
      float Ls[U];
      Vec<D> A[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const bool ok = p0 + u < g.count;
        const int p = ok ? p0 + u : p0;
        Ls[u] = __ldg(g.l + p * g.stride_l + row);
        A[u].load(g.a + p * g.stride_a + row * D + lane * E);
        if (!ok) Ls[u] = -CUDART_INF_F;
      }
      float bm = Ls[0];
#pragma unroll
      for (int u = 1; u < U; ++u) bm = fmaxf(bm, Ls[u]);
      if (bm > m) {
        const float sc = (m == -CUDART_INF_F) ? 0.f : expf(m - bm);
        wsum *= sc;
#pragma unroll
        for (int e = 0; e < E; ++e) out[e] *= sc;
        m = bm;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float w = Ls[u] == -CUDART_INF_F ? 0.f : expf(Ls[u] - m);
        wsum += w;
#pragma unroll
        for (int e = 0; e < E; ++e) out[e] = fmaf(w, A[u].v[e], out[e]);
      }
    }
  }
  if (m == -CUDART_INF_F) {
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = 0.f;
    return -CUDART_INF_F;
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int e = 0; e < E; ++e) out[e] *= inv;
  return m + logf(wsum);
}

}  // namespace

// One warp per (b, h, i) row.
template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const MergeArgs m) {
  ptx::pdl_prologue();
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + warp;
  const int64_t nrows = (int64_t)m.B * m.Hq * m.Nb;
  if (row >= nrows) return;
  const int64_t bh = row / m.Nb;
  if (m.mask_active && m.mask[bh]) return;
  const int b = (int)(bh / m.Hq), h = (int)(bh % m.Hq), i = (int)(row % m.Nb);
  float out[E];
  const float lse = merge_row<D>(m.parts, row, lane, out);
  store_out<D>(m.o, b * m.o_sb + h * m.o_sh + i * m.o_st + lane * E, m.o_bf16, out);
  if (m.lse && lane == 0) m.lse[row] = lse;
}

cudaError_t launch_merge(const MergeArgs& m, cudaStream_t s) {
  const int64_t nrows = (int64_t)m.B * m.Hq * m.Nb;
  const unsigned grid = (unsigned)((nrows + 7) / 8);
  if (grid == 0) return cudaSuccess;
  if (m.D == 64) return launch_k(merge_kernel<64>, grid, dim3(256), 0, s, m);
  return launch_k(merge_kernel<128>, grid, dim3(256), 0, s, m);
}

// ---------------------------------------------------------------------------
// Gamma gate (summary, "Stratégies de Réutilisation Adaptatives", video
// bullet): for every head that recomputed this step, merge its fresh split
// partials into A_new, form <A_new, A_cached>, |A_new|^2, |A_cached|^2 over the
// head's Nb x D values, write A_new into the cache, and let the last CTA of the
// head turn the sums into sim = cos(A_new, A_cached) and the next step's
// reuse flag sim > gamma[h].  Sums use a fixed order (lane tree, warp order,
// chunk order), so the result does not depend on scheduling.
// ---------------------------------------------------------------------------
constexpr int kGammaRows = 64;
int gamma_chunk_rows() { return kGammaRows; }

template <int D>
__global__ void __launch_bounds__(256) gamma_update_kernel(const GammaArgs g) {
  ptx::pdl_prologue();
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, chunk = blockIdx.x;
  const int h = bh % g.Hq;
  const bool reuse = g.gate_active && g.mask[bh];
  if (reuse) {
    if (chunk == 0 && threadIdx.x == 0) {
      if (g.reuse_out) g.reuse_out[bh] = 1;
      if (g.sim_out) g.sim_out[bh] = g.sim[bh];
    }
    return;
  }
  float dot = 0.f, na = 0.f, nc = 0.f;
  const int r0 = chunk * kGammaRows;
  const int r1 = min(r0 + kGammaRows, g.Nb);
  for (int i = r0 + warp; i < r1; i += 8) {
    const int64_t row = (int64_t)bh * g.Nb + i;
    float a_new[E];
    const float L = merge_row<D>(g.fresh, row, lane, a_new);
    float* cp = g.cache_a + row * D + lane * E;
    if (g.cache_valid) {
      Vec<D> c;
      c.load(cp);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        dot = fmaf(a_new[e], c.v[e], dot);
        na = fmaf(a_new[e], a_new[e], na);
        nc = fmaf(c.v[e], c.v[e], nc);
      }
    }
    Vec<D> w;
#pragma unroll
    for (int e = 0; e < E; ++e) w.v[e] = a_new[e];
    w.store(cp);
    if (lane == 0) g.cache_l[row] = L;
  }
  __shared__ float red[8][3];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, off);
    na += __shfl_xor_sync(0xffffffffu, na, off);
    nc += __shfl_xor_sync(0xffffffffu, nc, off);
  }
  if (lane == 0) { red[warp][0] = dot; red[warp][1] = na; red[warp][2] = nc; }
  __syncthreads();
  if (threadIdx.x != 0) return;
  float s0 = 0.f, s1 = 0.f, s2 = 0.f;
  for (int w = 0; w < 8; ++w) { s0 += red[w][0]; s1 += red[w][1]; s2 += red[w][2]; }
  float* part = g.partials + ((int64_t)bh * g.chunks + chunk) * 3;
  part[0] = s0; part[1] = s1; part[2] = s2;
  if (chunk == 0 && g.reuse_out) g.reuse_out[bh] = 0;
  __threadfence();
  const int prev = atomicAdd(g.counters + bh, 1);
  if (prev != g.chunks - 1) return;
  __threadfence();
  float t0 = 0.f, t1 = 0.f, t2 = 0.f;
  const volatile float* all = g.partials + (int64_t)bh * g.chunks * 3;
  for (int c = 0; c < g.chunks; ++c) { t0 += all[3 * c]; t1 += all[3 * c + 1]; t2 += all[3 * c + 2]; }
  float sim = CUDART_NAN_F;
  int8_t next = 0;
  if (g.cache_valid) {
    sim = (t1 > 0.f && t2 > 0.f) ? t0 / (sqrtf(t1) * sqrtf(t2)) : 0.f;
    next = sim > g.gamma[h] ? 1 : 0;
  }
  g.sim[bh] = sim;
  g.mask[bh] = next;
  if (g.sim_out) g.sim_out[bh] = sim;
  g.counters[bh] = 0;
}

cudaError_t launch_gamma_update(const GammaArgs& g, cudaStream_t s) {
  dim3 grid(g.chunks, g.B * g.Hq);
  if (g.D == 64) return launch_k(gamma_update_kernel<64>, grid, dim3(256), 0, s, g);
  return launch_k(gamma_update_kernel<128>, grid, dim3(256), 0, s, g);
}

// ---------------------------------------------------------------------------
// KV append: K_p/V_p rows [prefix_len, prefix_len + Nb) <- K_in/V_in, 16-byte
// vectors, one thread per vector of K and of V.
// ---------------------------------------------------------------------------
__global__ void kv_append_kernel(uint8_t* kp, uint8_t* vp, const uint8_t* kin, const uint8_t* vin,
                                 int32_t Hkv, int32_t Nb, int32_t vec_per_row, int64_t rows,
                                 int64_t kp_sb, int64_t kp_sh, int64_t kp_st, int64_t kin_sb,
                                 int64_t kin_sh, int64_t kin_st, int64_t prefix_len) {
  ptx::pdl_prologue();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * vec_per_row) return;
  const int64_t r = idx / vec_per_row;
  const int c = (int)(idx % vec_per_row);
  const int i = (int)(r % Nb);
  const int64_t bh = r / Nb;
  const int h = (int)(bh % Hkv);
  const int64_t b = bh / Hkv;
  const int64_t src = b * kin_sb + h * kin_sh + i * kin_st + c * 16;
  const int64_t dst = b * kp_sb + h * kp_sh + (prefix_len + i) * kp_st + c * 16;
  *reinterpret_cast<uint4*>(kp + dst) = __ldg(reinterpret_cast<const uint4*>(kin + src));
  *reinterpret_cast<uint4*>(vp + dst) = __ldg(reinterpret_cast<const uint4*>(vin + src));
}

cudaError_t launch_kv_append(const fb_attn_desc& d, void* kp, void* vp, int64_t prefix_len,
                             const void* kin, const void* vin, cudaStream_t s) {
  const int es = d.in_dtype == FB_BF16 ? 2 : 4;
  const int vec = d.D * es / 16;
  const int64_t rows = (int64_t)d.B * d.Hkv * d.Nb;
  const int64_t n = rows * vec;
  const int threads = 256;
  const unsigned grid = (unsigned)((n + threads - 1) / threads);
  return launch_k(kv_append_kernel, dim3(grid), dim3(threads), 0, s, static_cast<uint8_t*>(kp),
                  static_cast<uint8_t*>(vp), static_cast<const uint8_t*>(kin), static_cast<const uint8_t*>(vin),
                  (int32_t)d.Hkv, (int32_t)d.Nb, (int32_t)vec, rows, d.kp_strides[0] * es, d.kp_strides[1] * es,
                  d.kp_strides[2] * es, d.kin_strides[0] * es, d.kin_strides[1] * es, d.kin_strides[2] * es,
                  prefix_len);
}

// ---------------------------------------------------------------------------
// Sparse membership bitmap: bit j of (b, h) set iff j is in sel[b, h, :].
// ---------------------------------------------------------------------------
__global__ void build_bitmap_kernel(const int32_t* sel, int32_t sel_k, uint32_t* bitmap, int64_t words) {
  ptx::pdl_prologue();
  const int64_t bh = blockIdx.x;
  uint32_t* w = bitmap + bh * words;
  for (int64_t j = threadIdx.x; j < words; j += blockDim.x) w[j] = 0u;
  __syncthreads();
  const int32_t* s = sel + bh * sel_k;
  for (int j = threadIdx.x; j < sel_k; j += blockDim.x) {
    const int32_t key = s[j];
    if (key >= 0 && (int64_t)(key >> 5) < words) atomicOr(w + (key >> 5), 1u << (key & 31));
  }
}

cudaError_t launch_build_bitmap(const int32_t* sel, int32_t sel_k, int32_t BH, uint32_t* bitmap,
                                int64_t words, cudaStream_t s) {
  return launch_k(build_bitmap_kernel, dim3(BH), dim3(256), 0, s, sel, sel_k, bitmap, words);
}

// ---------------------------------------------------------------------------
// Active-query subsets (SureLock page, "Principes de Fonctionnement"): the
// query rows of the still-active block positions gathered into a compact
// block, and a compact part scattered back to the rows of those positions.
// One warp per row; positions outside [0, Nb) are skipped and reported as
// FB_EINVAL in the device status word.
// ---------------------------------------------------------------------------
__global__ void gather_active_q_kernel(const uint8_t* q, int64_t q_sb, int64_t q_sh, int64_t q_st, uint8_t* out,
                                       const int32_t* active, int32_t n_act, int32_t B, int32_t Hq, int32_t Nb,
                                       int32_t row_bytes, int* status) {
  ptx::pdl_prologue();
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);   // compact (b, h, k)
  const int lane = threadIdx.x & 31;
  const int64_t bh = r / n_act;
  const int k = (int)(r % n_act);
  const int b = (int)(bh / Hq), h = (int)(bh % Hq);
  if (b >= B) return;
  const int i = active[(int64_t)b * n_act + k];
  if (i < 0 || i >= Nb) {
    if (lane == 0) atomicCAS(status, 0, (int)FB_EINVAL);
    return;
  }
  const uint8_t* src = q + b * q_sb + h * q_sh + i * q_st;
  uint8_t* dst = out + r * row_bytes;
  for (int c = lane * 16; c < row_bytes; c += 512)
    *reinterpret_cast<uint4*>(dst + c) = __ldg(reinterpret_cast<const uint4*>(src + c));
}

__global__ void scatter_active_part_kernel(const float* ca, const float* cl, float* a, float* l,
                                           const int32_t* active, int32_t n_act, int32_t B, int32_t Hq, int32_t Nb,
                                           int32_t D, int* status) {
  ptx::pdl_prologue();
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t bh = r / n_act;
  const int k = (int)(r % n_act);
  const int b = (int)(bh / Hq);
  if (b >= B) return;
  const int i = active[(int64_t)b * n_act + k];
  if (i < 0 || i >= Nb) {
    if (lane == 0) atomicCAS(status, 0, (int)FB_EINVAL);
    return;
  }
  const int64_t dst = bh * Nb + i;
  for (int c = lane * 4; c < D; c += 128)
    *reinterpret_cast<float4*>(a + dst * D + c) = *reinterpret_cast<const float4*>(ca + r * D + c);
  if (lane == 0) l[dst] = cl[r];
}

// ---------------------------------------------------------------------------
// Sparse selected keys, gathered once per KV head: the union of its G query
// heads' selections (from their membership bitmaps over the prefix), in key
// order, and per query head a membership bitmap over that union.  The
// tcgen05 pass then runs over the union's rows (gathered into a compact K/V
// block) and leaves out, per query head, the union keys it did not select.
// One CTA per (b, KV head); the union has at most `umax` keys.
// ---------------------------------------------------------------------------
constexpr int kUnionThreads = 1024;
__global__ void __launch_bounds__(kUnionThreads)
    union_select_kernel(const uint32_t* bitmap, int64_t words_p, int32_t G, int32_t Hq, int32_t Hkv, int32_t* upos,
                        int32_t* ucount, int64_t umax, uint32_t* memb, int64_t words_u) {
  ptx::pdl_prologue();
  using Scan = cub::BlockScan<int, kUnionThreads>;   // union sizes fit in 32 bits (prefix < 2^31 keys)
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int s_total;
  const int kv = blockIdx.x, b = kv / Hkv, kvh = kv % Hkv;
  const uint32_t* hb = bitmap + ((int64_t)b * Hq + (int64_t)kvh * G) * words_p;   // G head bitmaps
  int32_t* up = upos + (int64_t)kv * umax;
  auto uword = [&](int64_t w) {
    uint32_t u = 0u;
    for (int g = 0; g < G; ++g) u |= hb[g * words_p + w];
    return u;
  };
  // the union's positions, in key order
  const int64_t chunk = (words_p + kUnionThreads - 1) / kUnionThreads;
  const int64_t w0 = threadIdx.x * chunk, w1 = min(words_p, w0 + chunk);
  int cnt = 0;
  for (int64_t w = w0; w < w1; ++w) cnt += __popc(uword(w));
  int base, total;
  Scan(tmp).ExclusiveSum(cnt, base, total);
  if (threadIdx.x == 0) s_total = total;
  for (int64_t w = w0; w < w1; ++w) {
    uint32_t u = uword(w);
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      if (base < umax) up[base] = (int32_t)(w * 32 + bit);
      ++base;
    }
  }
  __syncthreads();
  const int64_t n = min((int64_t)s_total, umax);
  if (threadIdx.x == 0) ucount[kv] = (int32_t)n;
  // membership of each union key in each query head's selection: one warp
  // per 32-key word, lane j testing union key 32 cw + j (coalesced reads)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t i = warp; i < (int64_t)G * words_u; i += kUnionThreads / 32) {
    const int g = (int)(i / words_u);
    const int64_t cw = i % words_u;
    const int64_t idx = cw * 32 + lane;
    bool in = false;
    if (idx < n) {
      const int32_t pos = up[idx];
      in = (hb[g * words_p + (pos >> 5)] >> (pos & 31)) & 1u;
    }
    const uint32_t bits = __ballot_sync(0xffffffffu, in);
    if (lane == 0) memb[((int64_t)b * Hq + (int64_t)kvh * G + g) * words_u + cw] = bits;
  }
}

// The same result straight from the selections, in shared memory: the G
// query heads' key bitmaps are built there (and copied out to `bitmap` for
// passes that need them later), then the union's positions and each head's
// membership over the union are taken from them without a global-memory
// round trip per bit.  One CTA per (b, KV head); the launcher checks that the
// G bitmaps and the umax positions fit in shared memory.
__global__ void __launch_bounds__(kUnionThreads)
    union_build_kernel(const int32_t* sel, int32_t sel_k, uint32_t* bitmap, int32_t words_p, int32_t G, int32_t Hq,
                       int32_t Hkv, int32_t* upos, int32_t* ucount, int32_t umax, uint32_t* memb, int32_t words_u) {
  ptx::pdl_prologue();
  using Scan = cub::BlockScan<int, kUnionThreads>;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ int s_total;
  extern __shared__ uint32_t sm_words[];
  uint32_t* hbm = sm_words;                                     // [G][words_p] head bitmaps
  int32_t* spos = reinterpret_cast<int32_t*>(sm_words + G * words_p);   // [umax] union positions
  const int tid = threadIdx.x;
  const int kv = blockIdx.x, b = kv / Hkv, kvh = kv % Hkv;
  const int64_t bh0 = (int64_t)b * Hq + (int64_t)kvh * G;      // the first query head's (b, h) row
  for (int i = tid; i < G * words_p; i += kUnionThreads) hbm[i] = 0u;
  __syncthreads();
  {
    // the G heads' selections are contiguous ([B, Hq, sel_k]): eight keys in
    // flight per thread across all of them before their atomics, so the
    // loads cost one memory round trip rather than one per head
    const int32_t* sg = sel + bh0 * sel_k;
    const int total = G * sel_k;
    for (int j0 = tid; j0 < total; j0 += 8 * kUnionThreads) {
      int32_t key[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * kUnionThreads;
        key[u] = j < total ? sg[j] : -1;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * kUnionThreads;
        if (key[u] >= 0 && (key[u] >> 5) < words_p) {
          const int g = j / sel_k;
          atomicOr(hbm + g * words_p + (key[u] >> 5), 1u << (key[u] & 31));
        }
      }
    }
  }
  __syncthreads();
  for (int g = 0; g < G; ++g)
    for (int w = tid; w < words_p; w += kUnionThreads) bitmap[(bh0 + g) * words_p + w] = hbm[g * words_p + w];
  auto uword = [&](int w) {
    uint32_t u = 0u;
    for (int g = 0; g < G; ++g) u |= hbm[g * words_p + w];
    return u;
  };
  // the union's positions, in key order
  const int chunk = (words_p + kUnionThreads - 1) / kUnionThreads;
  const int w0 = tid * chunk, w1 = min(words_p, w0 + chunk);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(uword(w));
  int base, total;
  Scan(tmp).ExclusiveSum(cnt, base, total);
  if (tid == 0) s_total = total;
  int32_t* up = upos + (int64_t)kv * umax;
  for (int w = w0; w < w1; ++w) {
    uint32_t u = uword(w);
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      if (base < umax) {
        up[base] = w * 32 + bit;
        spos[base] = w * 32 + bit;
      }
      ++base;
    }
  }
  __syncthreads();
  const int n = min(s_total, umax);
  if (tid == 0) ucount[kv] = n;
  // membership of each union key in each query head's selection: one warp
  // per 32-key word, lane j testing union key 32 cw + j
  const int warp = tid >> 5, lane = tid & 31;
  for (int cw = warp; cw < words_u; cw += kUnionThreads / 32) {
    const int idx = cw * 32 + lane;
    const int32_t pos = idx < n ? spos[idx] : -1;
    for (int g = 0; g < G; ++g) {
      const bool in = pos >= 0 && ((hbm[g * words_p + (pos >> 5)] >> (pos & 31)) & 1u);
      const uint32_t bits = __ballot_sync(0xffffffffu, in);
      if (lane == 0) memb[(bh0 + g) * words_u + cw] = bits;
    }
  }
}

// Rows [0, ucount) of the compact K/V block of each (b, KV head) <- the
// prefix rows at the union's positions; rows [ucount, umax) <- zeros (their
// keys are excluded for every head, and zeros keep P V finite).  One thread
// per 16-byte vector of a row of K and of V.
__global__ void gather_union_kernel(const uint8_t* kp, const uint8_t* vp, int64_t kp_sb, int64_t kp_sh,
                                    int64_t kp_st, const int32_t* upos, const int32_t* ucount, int64_t umax,
                                    int32_t Hkv, int32_t vec_per_row, int64_t nrows, uint8_t* ck, uint8_t* cv) {
  ptx::pdl_prologue();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= nrows * vec_per_row) return;
  const int64_t r = idx / vec_per_row;   // compact row: (b * Hkv + kvh) * umax + i
  const int c = (int)(idx % vec_per_row);
  const int64_t kv = r / umax, i = r % umax;
  const int64_t dst = r * vec_per_row * 16 + c * 16;
  uint4 kx = make_uint4(0, 0, 0, 0), vx = kx;
  if (i < ucount[kv]) {
    const int64_t b = kv / Hkv, h = kv % Hkv;
    const int64_t src = b * kp_sb + h * kp_sh + (int64_t)upos[r] * kp_st + c * 16;
    kx = __ldg(reinterpret_cast<const uint4*>(kp + src));
    vx = __ldg(reinterpret_cast<const uint4*>(vp + src));
  }
  *reinterpret_cast<uint4*>(ck + dst) = kx;
  *reinterpret_cast<uint4*>(cv + dst) = vx;
}

cudaError_t launch_union_select(const fb_attn_desc& d, const uint32_t* bitmap, int64_t words_p, int32_t* upos,
                                int32_t* ucount, int64_t umax, uint32_t* memb, int64_t words_u, cudaStream_t s) {
  return launch_k(union_select_kernel, dim3((unsigned)(d.B * d.Hkv)), dim3(kUnionThreads), 0, s, bitmap, words_p,
                  (int32_t)(d.Hq / d.Hkv), (int32_t)d.Hq, (int32_t)d.Hkv, upos, ucount, umax, memb, words_u);
}

static size_t union_build_smem(const fb_attn_desc& d, int64_t words_p, int64_t umax) {
  return (size_t)(d.Hq / d.Hkv) * words_p * 4 + (size_t)umax * 4;
}

bool union_build_fits(const fb_attn_desc& d, int64_t words_p, int64_t umax) {
  return union_build_smem(d, words_p, umax) <= 200 * 1024;
}

cudaError_t launch_union_build(const fb_attn_desc& d, const int32_t* sel, int32_t sel_k, uint32_t* bitmap,
                               int64_t words_p, int32_t* upos, int32_t* ucount, int64_t umax, uint32_t* memb,
                               int64_t words_u, cudaStream_t s) {
  const size_t smem = union_build_smem(d, words_p, umax);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  static size_t opted[kMaxDevices] = {};   // the attribute is per device
  size_t& cur = opted[current_device()];
  if (smem > cur) {   // the static scan storage counts too: opt in for any size above the last
    cudaError_t e = cudaFuncSetAttribute(union_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cur = smem;
  }
  return launch_k(union_build_kernel, dim3((unsigned)(d.B * d.Hkv)), dim3(kUnionThreads), smem, s, sel, sel_k,
                  bitmap, (int32_t)words_p, (int32_t)(d.Hq / d.Hkv), (int32_t)d.Hq, (int32_t)d.Hkv, upos, ucount,
                  (int32_t)umax, memb, (int32_t)words_u);
}

cudaError_t launch_gather_union(const fb_attn_desc& d, const void* kp, const void* vp, const int32_t* upos,
                                const int32_t* ucount, int64_t umax, void* ck, void* cv, cudaStream_t s) {
  const int es = d.in_dtype == FB_BF16 ? 2 : 4;
  const int vec = d.D * es / 16;
  const int64_t rows = (int64_t)d.B * d.Hkv * umax;
  const int threads = 256;
  const unsigned grid = (unsigned)((rows * vec + threads - 1) / threads);
  return launch_k(gather_union_kernel, dim3(grid), dim3(threads), 0, s, static_cast<const uint8_t*>(kp),
                  static_cast<const uint8_t*>(vp), d.kp_strides[0] * es, d.kp_strides[1] * es, d.kp_strides[2] * es,
                  upos, ucount, umax, (int32_t)d.Hkv, (int32_t)vec, rows, static_cast<uint8_t*>(ck),
                  static_cast<uint8_t*>(cv));
}

int* device_status_ptr();

cudaError_t launch_gather_active_q(const fb_attn_desc& d, const void* q, void* out, const int32_t* active,
                                   int32_t n_act, cudaStream_t s) {
  const int es = d.in_dtype == FB_BF16 ? 2 : 4;
  int* st = device_status_ptr();
  if (!st) return cudaErrorInvalidValue;
  const int64_t rows = (int64_t)d.B * d.Hq * n_act;
  return launch_k(gather_active_q_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, s,
                  static_cast<const uint8_t*>(q), d.q_strides[0] * es, d.q_strides[1] * es, d.q_strides[2] * es,
                  static_cast<uint8_t*>(out), active, n_act, (int32_t)d.B, (int32_t)d.Hq, (int32_t)d.Nb,
                  (int32_t)(d.D * es), st);
}

cudaError_t launch_scatter_active_part(const fb_attn_desc& d, const float* ca, const float* cl, float* a, float* l,
                                       const int32_t* active, int32_t n_act, cudaStream_t s) {
  int* st = device_status_ptr();
  if (!st) return cudaErrorInvalidValue;
  const int64_t rows = (int64_t)d.B * d.Hq * n_act;
  return launch_k(scatter_active_part_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, s, ca, cl, a, l,
                  active, n_act, (int32_t)d.B, (int32_t)d.Hq, (int32_t)d.Nb, (int32_t)d.D, st);
}

cudaError_t launch_fill_decision(int8_t* reuse_out, int32_t n, int8_t value, cudaStream_t s) {
  return cudaMemsetAsync(reuse_out, value, (size_t)n, s);
}

}  // namespace fb
