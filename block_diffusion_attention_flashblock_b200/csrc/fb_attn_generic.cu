// Generic attention kernels of libfb: one launch computes, for a tile of
// packed query rows, softmax attention over one key source (the prefix KV
// cache, a gathered key list, or the block's own keys) and either writes the
// fp32 part (A, L = log Z) of its key split or merges it on the spot with
// external parts (FlashBlock summary, "Mécanisme Central": A_out/L_out,
// A_in/L_in and their log-space merge).
//
//   attn_mma_kernel<D>: bf16 inputs, tensor cores through mma.sync m16n8k16
//     (fp32 accumulate), 64 rows x 64 keys per iteration, cp.async double
//     buffering.  Used for block-internal attention (few keys, fused merge),
//     gathered sparse keys, and as the prefix pass when the tcgen05 kernel does
//     not apply.
//   attn_f32_kernel<D>: fp32 inputs, plain FFMA (no TF32), one query row per
//     D/64 threads.  Used by fp32 workloads.
//
// Both take the same AttnArgs; numerics: scores in the log2 domain
// (s * scale * log2 e), online max/sum per row, exp2f, fp32 accumulation.
#include "fb_internal.cuh"
#include "fb_ptx.cuh"
#include <math_constants.h>

namespace fb {

// Longest key-list slice one CTA of a gather pass stages in shared memory.
constexpr int kMaxGatherKeys = 4096;

namespace {

struct RowInfo {
  int b, h, i;
  bool valid;
};

__device__ __forceinline__ RowInfo map_row(const RowMap& rm, int unit, int r) {
  RowInfo ri;
  if (rm.per_head) {
    ri.b = unit / rm.Hq;
    ri.h = unit % rm.Hq;
    ri.i = r;
    ri.valid = r < rm.Nb;
  } else {
    const int kvh = unit % rm.Hkv;
    ri.b = unit / rm.Hkv;
    ri.valid = r < rm.rows_per_unit;
    const int rr = ri.valid ? r : 0;
    ri.h = kvh * rm.G + rr / rm.Nb;
    ri.i = rr % rm.Nb;
  }
  if (!ri.valid) ri.i = 0;
  return ri;
}

__device__ __forceinline__ int unit_batch(const RowMap& rm, int unit) {
  return rm.per_head ? unit / rm.Hq : unit / rm.Hkv;
}
__device__ __forceinline__ int unit_kvhead(const RowMap& rm, int unit) {
  return rm.per_head ? (unit % rm.Hq) / rm.G : unit % rm.Hkv;
}

// True when every query head covered by rows [row0, row0 + n) of `unit` has
// mask = 1 (gamma gate: reuse this step), so the tile need not be computed.
__device__ bool tile_all_masked(const AttnArgs& a, int unit, int row0, int n) {
  const RowMap& rm = a.rm;
  const int last = min(row0 + n, rm.rows_per_unit) - 1;
  if (last < row0) return true;
  const RowInfo f = map_row(rm, unit, row0), l = map_row(rm, unit, last);
  for (int h = f.h; h <= l.h; ++h)
    if (!a.mask[f.b * rm.Hq + h]) return false;
  return true;
}

__device__ __forceinline__ bool key_excluded(const AttnArgs& a, int b, int h, int64_t key) {
  if (a.excl == nullptr) return false;
  const uint32_t w = __ldg(a.excl + (int64_t)(b * a.rm.Hq + h) * a.excl_words + (key >> 5));
  return (w >> (key & 31)) & 1u;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Split a pair of fp32 values into bf16 hi + lo parts (x = hi + lo to about
// 2^-16 relative), so that P V with bf16 operands keeps fp32-level accuracy.
__device__ __forceinline__ void split_bf16(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Merge epilogue weights of one row: the in-kernel part has normaliser L_in,
// the external parts L_p (prefetched in Lx); m = max, w = e^{L - m}.
struct RowMerge {
  float m, w_in, inv_sum, lse;
  float w[FB_MAX_PARTS];
  bool empty;
};

__device__ __forceinline__ RowMerge row_merge(int next, const float* Lx, float L_in) {
  RowMerge r;
  float m = L_in;
#pragma unroll
  for (int p = 0; p < FB_MAX_PARTS; ++p)
    if (p < next) m = fmaxf(m, Lx[p]);
  r.m = m;
  r.empty = (m == -CUDART_INF_F);
  float sum = 0.f;
  r.w_in = (r.empty || L_in == -CUDART_INF_F) ? 0.f : expf(L_in - m);
  sum += r.w_in;
#pragma unroll
  for (int p = 0; p < FB_MAX_PARTS; ++p) {
    r.w[p] = (p < next && !r.empty && Lx[p] != -CUDART_INF_F) ? expf(Lx[p] - m) : 0.f;
    sum += r.w[p];
  }
  r.inv_sum = r.empty ? 0.f : 1.f / sum;
  r.lse = r.empty ? -CUDART_INF_F : m + logf(sum);
  return r;
}

}  // namespace

// ---------------------------------------------------------------------------
// bf16 tensor-core (mma.sync) kernel
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(128) attn_mma_kernel(const AttnArgs a) {
  ptx::pdl_prologue();
  constexpr int BM = 64, BN = 64, CH = D / 8, NT = BN / 8, DT = D / 8, KS = D / 16;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sK = sQ + BM * D;
  __nv_bfloat16* sV = sK + 2 * BN * D;

  const RowMap& rm = a.rm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x / rm.row_tiles, tile = blockIdx.x % rm.row_tiles;
  const int split = blockIdx.y;
  const int b = unit_batch(rm, unit), kvh = unit_kvhead(rm, unit);
  const int row0 = tile * BM;

  if (a.mask_active && tile_all_masked(a, unit, row0, BM)) return;

  const int64_t kbeg = (int64_t)split * a.keys_per_split;
  const int64_t kend = min(kbeg + a.keys_per_split, a.nkeys);
  const int ntiles = kend > kbeg ? (int)((kend - kbeg + BN - 1) / BN) : 0;

  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(a.k) + b * a.k_sb + kvh * a.k_sh;
  const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(a.v) + b * a.k_sb + kvh * a.k_sh;
  // per_head units with a key list: this split's slice of the (b, query head)
  // list is staged in shared memory first, so a tile's gather does not wait
  // on its own index loads
  // (slices longer than kMaxGatherKeys, which the host gives no staging
  // space, read their indices directly)
  int32_t* sSel = reinterpret_cast<int32_t*>(sV + 2 * BN * D);
  const bool gather = a.sel != nullptr;
  const bool staged = gather && a.keys_per_split <= kMaxGatherKeys;
  const int32_t* sel = gather ? a.sel + (int64_t)unit * a.sel_k : nullptr;
  if (staged) {
    for (int64_t k = kbeg + tid; k < kend; k += 128) sSel[k - kbeg] = __ldg(sel + k);
    __syncthreads();
  }

  // Q tile -> smem (swizzled 16-byte chunks: chunk c of row r at c ^ (r & 7)).
  for (int c = tid; c < BM * CH; c += 128) {
    const int r = c / CH, ch = c % CH;
    const RowInfo ri = map_row(rm, unit, row0 + r);
    const __nv_bfloat16* src = q + ri.b * a.q_sb + ri.h * a.q_sh + ri.i * a.q_st + ch * 8;
    cp_async16(smem_u32(sQ + r * D + ((ch ^ (r & 7)) * 8)), ri.valid ? src : q, ri.valid ? 16 : 0);
  }
  auto load_kv = [&](int t, int stage) {
    const int64_t key0 = kbeg + (int64_t)t * BN;
    __nv_bfloat16* dk = sK + stage * BN * D;
    __nv_bfloat16* dv = sV + stage * BN * D;
    for (int c = tid; c < BN * CH; c += 128) {
      const int r = c / CH, ch = c % CH;
      const int64_t key = key0 + r;
      int64_t phys = key < kend ? (staged ? (int64_t)sSel[key - kbeg] : gather ? (int64_t)__ldg(sel + key) : key)
                                : -1;
      const bool ok = phys >= 0 && phys < a.key_rows;
      if (!ok) phys = 0;
      const int off = r * D + ((ch ^ (r & 7)) * 8);
      cp_async16(smem_u32(dk + off), kb + phys * a.k_st + ch * 8, ok ? 16 : 0);
      cp_async16(smem_u32(dv + off), vb + phys * a.k_st + ch * 8, ok ? 16 : 0);
    }
  };
  if (ntiles > 0) load_kv(0, 0);
  cp_async_commit();

  // Row ownership inside the warp's 16-row slab: rows rA = lane/4 and rA + 8.
  const int rA = warp * 16 + (lane >> 2);
  RowInfo rowi[2] = {map_row(rm, unit, row0 + rA), map_row(rm, unit, row0 + rA + 8)};

  // Normalisers of the external parts of this thread's two rows, fetched
  // early so the merge epilogue waits on memory only once per part.
  float Lx[2][FB_MAX_PARTS];
  if (a.merge_out) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int64_t row = ((int64_t)rowi[rr].b * rm.Hq + rowi[rr].h) * rm.Nb + rowi[rr].i;
#pragma unroll
      for (int p = 0; p < FB_MAX_PARTS; ++p)
        Lx[rr][p] = (p < a.next && rowi[rr].valid) ? __ldg(a.ext_l[p] + row) : -CUDART_INF_F;
    }
  }

  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_run[2] = {-CUDART_INF_F, -CUDART_INF_F};
  float l_run[2] = {0.f, 0.f};

  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) {
      load_kv(t + 1, (t + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* cK = sK + (t & 1) * BN * D;
    const __nv_bfloat16* cV = sV + (t & 1) * BN * D;

    // S = Q K^T for this warp's 16 rows x 64 keys.
    float s[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t qf[4];   // Q fragment, re-read from shared memory (keeps registers for P hi/lo)
      {
        const int r = warp * 16 + (lane & 15), ch = 2 * kk + (lane >> 4);
        ldsm_x4(smem_u32(sQ + r * D + ((ch ^ (r & 7)) * 8)), qf[0], qf[1], qf[2], qf[3]);
      }
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        const int r = (nt + (lane >> 4)) * 8 + (lane & 7), ch = 2 * kk + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(cK + r * D + ((ch ^ (r & 7)) * 8)), b0, b1, b2, b3);
        mma_bf16(s[nt], qf, b0, b1);
        mma_bf16(s[nt + 1], qf, b2, b3);
      }
    }

    // Scale to log2 units, mask keys past the split end or excluded.
    const int64_t key0 = kbeg + (int64_t)t * BN;
    uint32_t exw[2][2] = {{0u, 0u}, {0u, 0u}};
    if (a.excl) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int64_t kw = key0 + 32 * w;
          exw[rr][w] = (kw < kend) ? __ldg(a.excl + (int64_t)(rowi[rr].b * rm.Hq + rowi[rr].h) * a.excl_words +
                                           (kw >> 5))
                                   : 0u;
        }
    }
    float tmax[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kc = nt * 8 + 2 * (lane & 3) + (e & 1);
        const int rr = e >> 1;
        bool valid = key0 + kc < kend;
        if (sel && valid) {
          const int32_t pk = __ldg(sel + key0 + kc);
          valid = pk >= 0 && pk < a.key_rows;
        }
        if (a.excl) valid = valid && !((exw[rr][kc >> 5] >> (kc & 31)) & 1u);
        const float v = valid ? s[nt][e] * a.scale_log2 : -CUDART_INF_F;
        s[nt][e] = v;
        tmax[rr] = fmaxf(tmax[rr], v);
      }
    float alpha[2], mref[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      tmax[rr] = fmaxf(tmax[rr], __shfl_xor_sync(0xffffffffu, tmax[rr], 1));
      tmax[rr] = fmaxf(tmax[rr], __shfl_xor_sync(0xffffffffu, tmax[rr], 2));
      const float mnew = fmaxf(m_run[rr], tmax[rr]);
      mref[rr] = (mnew == -CUDART_INF_F) ? 0.f : mnew;
      alpha[rr] = exp2f(m_run[rr] - mref[rr]);
      m_run[rr] = mnew;
      l_run[rr] *= alpha[rr];
    }
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      o[i][0] *= alpha[0]; o[i][1] *= alpha[0];
      o[i][2] *= alpha[1]; o[i][3] *= alpha[1];
    }
    // P = 2^(s - m) as bf16 hi + lo (P V below adds both products).
    uint32_t pf[NT][2], pr[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float p0 = exp2f(s[nt][0] - mref[0]), p1 = exp2f(s[nt][1] - mref[0]);
      const float p2 = exp2f(s[nt][2] - mref[1]), p3 = exp2f(s[nt][3] - mref[1]);
      l_run[0] += p0 + p1;
      l_run[1] += p2 + p3;
      split_bf16(p0, p1, pf[nt][0], pr[nt][0]);
      split_bf16(p2, p3, pf[nt][1], pr[nt][1]);
    }
    // O += P_hi V + P_lo V.
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
      const uint32_t af[4] = {pf[2 * kk][0], pf[2 * kk][1], pf[2 * kk + 1][0], pf[2 * kk + 1][1]};
      const uint32_t ar[4] = {pr[2 * kk][0], pr[2 * kk][1], pr[2 * kk + 1][0], pr[2 * kk + 1][1]};
#pragma unroll
      for (int dt = 0; dt < DT; dt += 2) {
        const int r = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, ch = dt + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(cV + r * D + ((ch ^ (r & 7)) * 8)), b0, b1, b2, b3);
        mma_bf16(o[dt], af, b0, b1);
        mma_bf16(o[dt + 1], af, b2, b3);
        mma_bf16(o[dt], ar, b0, b1);
        mma_bf16(o[dt + 1], ar, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // Finish: row sums across the quad, natural-log normaliser.
  float Lrow[2], inv[2];
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    float l = l_run[rr];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    if (l > 0.f) {
      inv[rr] = 1.f / l;
      Lrow[rr] = (m_run[rr] + log2f(l)) * kLn2;
    } else {
      inv[rr] = 0.f;
      Lrow[rr] = -CUDART_INF_F;
    }
  }

  const int Hq = rm.Hq, Nb = rm.Nb;
  if (!a.merge_out) {
    float* pa = a.part_a + split * a.part_stride_a;
    float* pl = a.part_l + split * a.part_stride_l;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const RowInfo& ri = rowi[rr];
      if (!ri.valid) continue;
      const int64_t row = ((int64_t)ri.b * Hq + ri.h) * Nb + ri.i;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        const int col = dt * 8 + 2 * (lane & 3);
        *reinterpret_cast<float2*>(pa + row * D + col) =
            make_float2(o[dt][2 * rr] * inv[rr], o[dt][2 * rr + 1] * inv[rr]);
      }
      if ((lane & 3) == 0) pl[row] = Lrow[rr];
    }
  } else {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const RowInfo& ri = rowi[rr];
      if (!ri.valid) continue;
      const int64_t row = ((int64_t)ri.b * Hq + ri.h) * Nb + ri.i;
      const RowMerge w = row_merge(a.next, Lx[rr], Lrow[rr]);
      const float win = w.w_in * inv[rr];
      float2 acc[DT];
#pragma unroll
      for (int dt = 0; dt < DT; ++dt)
        acc[dt] = make_float2(win * o[dt][2 * rr], win * o[dt][2 * rr + 1]);
#pragma unroll
      for (int p = 0; p < FB_MAX_PARTS; ++p) {
        if (p >= a.next || w.w[p] == 0.f) continue;
        const float* pa = a.ext_a[p] + row * D + 2 * (lane & 3);
        float2 v[DT];
#pragma unroll
        for (int dt = 0; dt < DT; ++dt) v[dt] = __ldg(reinterpret_cast<const float2*>(pa + dt * 8));
#pragma unroll
        for (int dt = 0; dt < DT; ++dt) {
          acc[dt].x = fmaf(w.w[p], v[dt].x, acc[dt].x);
          acc[dt].y = fmaf(w.w[p], v[dt].y, acc[dt].y);
        }
      }
      const int64_t obase = ri.b * a.o_sb + ri.h * a.o_sh + ri.i * a.o_st;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        const int col = dt * 8 + 2 * (lane & 3);
        const float2 r2 = make_float2(acc[dt].x * w.inv_sum, acc[dt].y * w.inv_sum);
        if (a.o_bf16) {
          *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.o) + obase + col) =
              __floats2bfloat162_rn(r2.x, r2.y);
        } else {
          *reinterpret_cast<float2*>(static_cast<float*>(a.o) + obase + col) = r2;
        }
      }
      if (a.lse && (lane & 3) == 0) a.lse[row] = w.lse;
    }
  }
}

// ---------------------------------------------------------------------------
// fp32 FFMA kernel: TPR = D/64 threads per row, 64 rows per CTA.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(64 * (D / 64)) attn_f32_kernel(const AttnArgs a) {
  ptx::pdl_prologue();
  constexpr int TPR = D / 64, BM = 64, BN = 32, DH = 64;
  constexpr int NTH = BM * TPR;
  __shared__ __align__(16) float sK[BN * D];
  __shared__ __align__(16) float sV[BN * D];

  const RowMap& rm = a.rm;
  const int tid = threadIdx.x;
  const int unit = blockIdx.x / rm.row_tiles, tile = blockIdx.x % rm.row_tiles;
  const int split = blockIdx.y;
  const int b = unit_batch(rm, unit), kvh = unit_kvhead(rm, unit);
  const int row0 = tile * BM;
  if (a.mask_active && tile_all_masked(a, unit, row0, BM)) return;

  const int r = tid / TPR, half = tid % TPR;
  const RowInfo ri = map_row(rm, unit, row0 + r);
  const float* q = static_cast<const float*>(a.q) + ri.b * a.q_sb + ri.h * a.q_sh + ri.i * a.q_st + half * DH;
  const float* kb = static_cast<const float*>(a.k) + b * a.k_sb + kvh * a.k_sh;
  const float* vb = static_cast<const float*>(a.v) + b * a.k_sb + kvh * a.k_sh;
  const int32_t* sel = a.sel ? a.sel + (int64_t)unit * a.sel_k : nullptr;

  float qr[DH], o[DH];
#pragma unroll
  for (int d = 0; d < DH; ++d) {
    qr[d] = ri.valid ? q[d] : 0.f;
    o[d] = 0.f;
  }
  float m_run = -CUDART_INF_F, l_run = 0.f;

  const int64_t kbeg = (int64_t)split * a.keys_per_split;
  const int64_t kend = min(kbeg + a.keys_per_split, a.nkeys);
  for (int64_t key0 = kbeg; key0 < kend; key0 += BN) {
    __syncthreads();
    for (int c = tid; c < BN * D / 4; c += NTH) {
      const int kr = c / (D / 4), c4 = c % (D / 4);
      const int64_t key = key0 + kr;
      float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
      const int64_t phys = key < kend ? (sel ? (int64_t)__ldg(sel + key) : key) : -1;
      if (phys >= 0 && phys < a.key_rows) {
        kv = __ldg(reinterpret_cast<const float4*>(kb + phys * a.k_st) + c4);
        vv = __ldg(reinterpret_cast<const float4*>(vb + phys * a.k_st) + c4);
      }
      reinterpret_cast<float4*>(sK)[c] = kv;
      reinterpret_cast<float4*>(sV)[c] = vv;
    }
    __syncthreads();
    const int nk = (int)min((int64_t)BN, kend - key0);
    for (int j = 0; j < nk; ++j) {
      const float* kr = sK + j * D + half * DH;
      float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};   // 8 independent FMA chains
#pragma unroll
      for (int d = 0; d < DH; ++d) s8[d & 7] = fmaf(qr[d], kr[d], s8[d & 7]);
      float s = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
      if (TPR == 2) s += __shfl_xor_sync(0xffffffffu, s, 1);
      s *= a.scale_log2;
      if (key_excluded(a, ri.b, ri.h, key0 + j)) s = -CUDART_INF_F;
      if (sel) {
        const int32_t pk = __ldg(sel + key0 + j);
        if (pk < 0 || pk >= a.key_rows) s = -CUDART_INF_F;
      }
      if (s == -CUDART_INF_F) continue;
      const float mnew = fmaxf(m_run, s);
      const float alpha = exp2f(m_run - mnew);
      const float p = exp2f(s - mnew);
      l_run = l_run * alpha + p;
      const float* vr = sV + j * D + half * DH;
#pragma unroll
      for (int d = 0; d < DH; ++d) o[d] = fmaf(p, vr[d], o[d] * alpha);
      m_run = mnew;
    }
  }

  const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
  const float Lrow = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -CUDART_INF_F;
  if (!ri.valid) return;
  const int64_t row = ((int64_t)ri.b * rm.Hq + ri.h) * rm.Nb + ri.i;
  if (!a.merge_out) {
    float* pa = a.part_a + split * a.part_stride_a + row * D + half * DH;
#pragma unroll
    for (int d = 0; d < DH; d += 4)
      *reinterpret_cast<float4*>(pa + d) = make_float4(o[d] * inv, o[d + 1] * inv, o[d + 2] * inv, o[d + 3] * inv);
    if (half == 0) (a.part_l + split * a.part_stride_l)[row] = Lrow;
  } else {
    float Lx[FB_MAX_PARTS];
#pragma unroll
    for (int p = 0; p < FB_MAX_PARTS; ++p) Lx[p] = p < a.next ? __ldg(a.ext_l[p] + row) : -CUDART_INF_F;
    const RowMerge w = row_merge(a.next, Lx, Lrow);
    const int64_t obase = ri.b * a.o_sb + ri.h * a.o_sh + ri.i * a.o_st + half * DH;
    const float win = w.w_in * inv;
#pragma unroll
    for (int d = 0; d < DH; ++d) o[d] *= win;
#pragma unroll
    for (int p = 0; p < FB_MAX_PARTS; ++p) {
      if (p >= a.next || w.w[p] == 0.f) continue;
      const float* pa = a.ext_a[p] + row * D + half * DH;
#pragma unroll
      for (int d = 0; d < DH; d += 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(pa + d));
        o[d] = fmaf(w.w[p], v.x, o[d]); o[d + 1] = fmaf(w.w[p], v.y, o[d + 1]);
        o[d + 2] = fmaf(w.w[p], v.z, o[d + 2]); o[d + 3] = fmaf(w.w[p], v.w, o[d + 3]);
      }
    }
#pragma unroll
    for (int d = 0; d < DH; d += 2) {
      const float2 r2 = make_float2(o[d] * w.inv_sum, o[d + 1] * w.inv_sum);
      if (a.o_bf16)
        *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.o) + obase + d) =
            __floats2bfloat162_rn(r2.x, r2.y);
      else
        *reinterpret_cast<float2*>(static_cast<float*>(a.o) + obase + d) = r2;
    }
    if (a.lse && half == 0) a.lse[row] = w.lse;
  }
}

// ---------------------------------------------------------------------------
int generic_tile_rows(int) { return 64; }
int generic_max_gather_keys() { return kMaxGatherKeys; }
int generic_key_tile() { return 64; }
int generic_ctas_per_sm(int D, int in_bf16) {
  if (!in_bf16) return 4;
  return D == 64 ? 4 : 2;
}

template <int D>
static cudaError_t launch_mma(const AttnArgs& a, cudaStream_t s) {
  // Q, two K and two V stages, and (gather passes) the split's key list
  constexpr int base = (64 * D + 4 * 64 * D) * 2;
  const int smem =
      base + (a.sel && a.keys_per_split <= kMaxGatherKeys ? (int)((a.keys_per_split * 4 + 15) / 16 * 16) : 0);
  static bool attr_set[kMaxDevices] = {};   // the attribute is per device
  bool& done = attr_set[current_device()];
  if (!done) {
    cudaError_t e = cudaFuncSetAttribute(attn_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         base + kMaxGatherKeys * 4);
    if (e != cudaSuccess) return e;
    done = true;
  }
  dim3 grid(a.rm.units * a.rm.row_tiles, a.nsplit);
  return launch_k(attn_mma_kernel<D>, grid, dim3(128), smem, s, a);
}

cudaError_t launch_attn_generic(const AttnArgs& a, int D, int in_bf16, cudaStream_t s) {
  if (in_bf16) return D == 64 ? launch_mma<64>(a, s) : launch_mma<128>(a, s);
  dim3 grid(a.rm.units * a.rm.row_tiles, a.nsplit);
  if (D == 64) return launch_k(attn_f32_kernel<64>, grid, dim3(64), 0, s, a);
  return launch_k(attn_f32_kernel<128>, grid, dim3(128), 0, s, a);
}

}  // namespace fb
