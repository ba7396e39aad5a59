// Fused epilogue of the tensor-core Newton-Schulz products: one thread
// holds 32 consecutive fp32 accumulator columns of one output row (from
// tcgen05.ld) and applies the product's epilogue (see EPI_* in dm_internal.h).
#pragma once

#include "dm_common.cuh"
#include "dm_sm100.cuh"

namespace dm {
namespace tcepi {

__device__ __forceinline__ void tmem_ld32_at(uint32_t taddr, float v[32]) {
  sm100::tmem_ld32(taddr, v);
}

__device__ __forceinline__ void ld_bf16x8(const void* p, float v[8]) {
  ld8(p, 0, DT_BF16, v);
}
__device__ __forceinline__ void st_bf16x8(void* p, const float v[8]) { st8(p, 0, DT_BF16, v); }

__device__ __forceinline__ bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

// Loads 32 consecutive elements of row r of a bf16 matrix (scalar tail).
__device__ __forceinline__ void load_row32(const __nv_bfloat16* base, int ld, int r, int c0,
                                           int ncols, float v[32]) {
  const __nv_bfloat16* p = base + (int64_t)r * ld + c0;
  if (c0 + 32 <= ncols) {
#pragma unroll
    for (int q = 0; q < 4; ++q) ld_bf16x8(p + 8 * q, v + 8 * q);
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) v[q] = (c0 + q < ncols) ? __bfloat162float(p[q]) : 0.f;
  }
}

__device__ __forceinline__ void store_row32(__nv_bfloat16* base, int ld, int r, int c0, int ncols,
                                            const float v[32]) {
  __nv_bfloat16* p = base + (int64_t)r * ld + c0;
  if (c0 + 32 <= ncols) {
#pragma unroll
    for (int q = 0; q < 4; ++q) st_bf16x8(p + 8 * q, v + 8 * q);
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q)
      if (c0 + q < ncols) p[q] = __float2bfloat16_rn(v[q]);
  }
}

// Symmetric store of 32 values of row r: element (r, c) for c >= r, and its
// mirror (c, r) for c > r.
__device__ __forceinline__ void store_sym32(const GemmMat& g, int r, int c0, const float v[32]) {
  __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(g.out);
  const int n = g.M;  // square output
  if (c0 >= r && c0 + 32 <= n) {
    store_row32(o, g.ldo, r, c0, n, v);
  } else {
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const int c = c0 + q;
      if (c < n && c >= r) o[(int64_t)r * g.ldo + c] = __float2bfloat16_rn(v[q]);
    }
  }
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const int c = c0 + q;
    if (c < n && c > r) o[(int64_t)c * g.ldo + r] = __float2bfloat16_rn(v[q]);
  }
}

__device__ __forceinline__ bool needs_aux(int epi) { return epi != EPI_SYRK; }

// Fused epilogue for 32 accumulator columns of one output row; `ax` holds
// the same 32 columns of the aux matrix (unused for EPI_SYRK).
__device__ __forceinline__ void epilogue32(const GemmMat& g, float lr, float decay, int r, int c0,
                                           float v[32], const float ax[32], float S, float valid,
                                           float& sx, float& sy) {
  switch (g.epi) {
    case EPI_SYRK: {
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] *= S;
      store_sym32(g, r, c0, v);
      break;
    }
    case EPI_POLY: {
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = fmaf(g.coef_acc, v[q], g.coef_aux * ax[q]);
      store_sym32(g, r, c0, v);
      break;
    }
    case EPI_GEMM: {
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = fmaf(g.coef_aux, ax[q], v[q]) * S;
      store_row32(reinterpret_cast<__nv_bfloat16*>(g.out), g.ldo, r, c0, g.N, v);
      break;
    }
    case EPI_FINAL_MUON: {
      const float ks = valid != 0.f ? g.kappa * S : 0.f;
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = (valid != 0.f) ? fmaf(g.coef_aux, ax[q], v[q]) * ks : 0.f;
      const int64_t wi = (int64_t)r * g.ldw + c0;
      const bool full = c0 + 32 <= g.N;
      const int es = g.wdt == DT_BF16 ? 2 : 4;
      const void* wp = reinterpret_cast<const char*>(g.W) + wi * es;
      if (full && aligned16(wp)) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float w8[8];
          ld8(g.W, wi + 8 * q, g.wdt, w8);
#pragma unroll
          for (int e = 0; e < 8; ++e) w8[e] = decay * w8[e] - lr * v[8 * q + e];
          st8(g.W, wi + 8 * q, g.wdt, w8);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (c0 + q < g.N)
            st_elem(g.W, wi + q, g.wdt, decay * ld_elem(g.W, wi + q, g.wdt) - lr * v[q]);
      }
      if (g.upd) {
        if (full && aligned16(g.upd + wi)) {
#pragma unroll
          for (int q = 0; q < 4; ++q) st8(g.upd, wi + 8 * q, DT_FP32, v + 8 * q);
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q)
            if (c0 + q < g.N) g.upd[wi + q] = v[q];
        }
      }
      break;
    }
    case EPI_FINAL_DIMUON: {
      const float rr = g.R[r];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        v[q] = round_to(fmaf(g.coef_aux, ax[q], v[q]) * S, DT_BF16);
        if (c0 + q < g.N) {
          const float y = rr * v[q] * g.C[c0 + q];
          sx += v[q] * v[q];
          sy += y * y;
        }
      }
      store_row32(reinterpret_cast<__nv_bfloat16*>(g.out), g.ldo, r, c0, g.N, v);
      break;
    }
  }
}

// Epilogue of chunks [ch_begin, ch_end) (32 columns each) of one accumulator
// row: tcgen05.ld of each chunk, with the next chunk's aux row in flight while
// the current one is processed.  Must be executed by all 32 lanes of the warp
// (tcgen05.ld is warp-collective); rows outside the matrix only skip stores.
__device__ __forceinline__ void epilogue_row(const GemmMat& g, float lr, float decay, int r,
                                             bool row_ok, int col0, uint32_t taddr, int ch_begin,
                                             int ch_end, int nch, float& sx, float& sy) {
  const float S = g.scal_idx >= 0 ? g.scal[g.scal_idx] : 1.f;
  const float valid = g.scal ? g.scal[SC_VALID] : 1.f;
  const bool aux = needs_aux(g.epi);
  const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(g.aux);
  float axn[32];
  if (aux && row_ok && ch_begin < nch) load_row32(ab, g.ldaux, r, col0 + ch_begin * 32, g.N, axn);
#pragma unroll 1
  for (int ch = ch_begin; ch < ch_end; ++ch) {
    float v[32], ax[32];
    tmem_ld32_at(taddr + (uint32_t)(ch * 32), v);
#pragma unroll
    for (int q = 0; q < 32; ++q) ax[q] = axn[q];
    if (aux && row_ok && ch + 1 < ch_end && ch + 1 < nch)
      load_row32(ab, g.ldaux, r, col0 + (ch + 1) * 32, g.N, axn);
    if (row_ok && ch < nch) epilogue32(g, lr, decay, r, col0 + ch * 32, v, ax, S, valid, sx, sy);
  }
}

}  // namespace tcepi
}  // namespace dm
