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

// ---------------------------------------------------------------------------
// Staged epilogue for whole 32 x 32 blocks.  A thread holds one row of the
// accumulator (tcgen05.ld 32x32b), so its own row accesses would make every
// warp-wide load or store touch 32 rows.  Instead the warp moves whole blocks
// through a 32 x 32 bf16 tile in shared memory: global loads and stores are
// 16 bytes per lane covering 8 rows x 64 bytes per instruction (4 instructions
// per block instead of 4 x 32 row segments), and the symmetric products'
// mirrored block leaves the tile transposed the same way.  Diagonal blocks of
// the symmetric products, partial blocks at the matrix edges and fp32 weights
// keep the row-per-thread path (epilogue32).
// ---------------------------------------------------------------------------
constexpr int SP = 40;                             // tile pitch in bf16 (80 bytes)
constexpr int STAGE_TILE_BYTES = 32 * SP * 2;      // one epilogue warp's tile

// Lane l's slot of a block: row (l >> 2) + 8 i, columns 8 (l & 3) .. + 7.
__device__ __forceinline__ void blk_ld(const __nv_bfloat16* base, int ld, int r0, int c0,
                                       uint4 q[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    q[i] = *reinterpret_cast<const uint4*>(base + (int64_t)(r0 + (lane >> 2) + 8 * i) * ld + c0 +
                                           8 * (lane & 3));
}
__device__ __forceinline__ void blk_st(__nv_bfloat16* base, int ld, int r0, int c0, const uint4 q[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint4*>(base + (int64_t)(r0 + (lane >> 2) + 8 * i) * ld + c0 + 8 * (lane & 3)) =
        q[i];
}
__device__ __forceinline__ void tile_put_blk(__nv_bfloat16* st, const uint4 q[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint4*>(st + ((lane >> 2) + 8 * i) * SP + 8 * (lane & 3)) = q[i];
}
__device__ __forceinline__ void tile_get_blk(const __nv_bfloat16* st, uint4 q[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    q[i] = *reinterpret_cast<const uint4*>(st + ((lane >> 2) + 8 * i) * SP + 8 * (lane & 3));
}
// Row `lane` of the tile from / to 32 fp32 values (bf16 stores round to
// nearest even, as the row-per-thread path does).
__device__ __forceinline__ void tile_put_row(__nv_bfloat16* st, const float v[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < 4; ++k) st_bf16x8(st + lane * SP + 8 * k, v + 8 * k);
}
__device__ __forceinline__ void tile_get_row(const __nv_bfloat16* st, float v[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 0; k < 4; ++k) ld_bf16x8(st + lane * SP + 8 * k, v + 8 * k);
}
// Transposes the bf16 tile in place: its 16 8x8 blocks are read transposed
// into registers (ldmatrix .trans, four blocks per instruction; lane 8q + i
// gives the address of row i of block q), then written back with stmatrix
// to the mirrored block positions.  Rows are 80 bytes apart, so the eight
// 16-byte rows of a block fall on distinct banks.
__device__ __forceinline__ void tile_transpose(__nv_bfloat16* st) {
  const int lane = threadIdx.x & 31;
  const int q = lane >> 3, i = lane & 7;
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(st));
  uint32_t f[4][4];  // f[a][b]: block (a, b) of the tile, transposed
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const uint32_t addr = base + (uint32_t)(((8 * a + i) * SP + 8 * q) * 2);
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(f[a][0]), "=r"(f[a][1]), "=r"(f[a][2]), "=r"(f[a][3])
                 : "r"(addr)
                 : "memory");
  }
  __syncwarp();
#pragma unroll
  for (int d = 0; d < 4; ++d) {  // block (d, b) of the transpose is block (b, d) transposed
    const uint32_t addr = base + (uint32_t)(((8 * d + i) * SP + 8 * q) * 2);
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};"
                 :
                 : "r"(addr), "r"(f[0][d]), "r"(f[1][d]), "r"(f[2][d]), "r"(f[3][d])
                 : "memory");
  }
}

// Whether the block of rows r0 .. r0 + 31, columns c0 .. c0 + 31 takes the
// staged path (warp-uniform).
__device__ __forceinline__ bool staged_ok(const GemmMat& g, int r0, int c0) {
  if (r0 + 32 > g.M || c0 + 32 > g.N) return false;
  switch (g.epi) {
    case EPI_SYRK:
    case EPI_POLY:
      return c0 >= r0 + 32 || c0 + 32 <= r0;  // off the diagonal
    case EPI_GEMM:
    case EPI_FINAL_DIMUON:
      return true;
    case EPI_FINAL_MUON:
      return g.wdt == DT_BF16 && (g.ldw & 7) == 0 && aligned16(g.W);
  }
  return false;
}

// A finished bf16 block (thread = row) to rows r0.., columns c0.. of `out`.
__device__ __forceinline__ void staged_store(__nv_bfloat16* st, __nv_bfloat16* out, int ld, int r0,
                                             int c0, const float v[32]) {
  uint4 q[4];
  tile_put_row(st, v);
  __syncwarp();
  tile_get_blk(st, q);
  blk_st(out, ld, r0, c0, q);
  __syncwarp();
}

// The staged form of epilogue32 for one whole block; `ax` already holds the
// thread's row of the aux block.
__device__ __forceinline__ void staged_epilogue32(const GemmMat& g, float lr, float decay, int r,
                                                  int r0, int c0, float v[32], const float ax[32],
                                                  float S, float valid, float& sx, float& sy,
                                                  __nv_bfloat16* st) {
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(g.out);
  switch (g.epi) {
    case EPI_SYRK:
    case EPI_POLY: {
      if (c0 + 32 <= r0) break;  // below the diagonal: another tile's mirror
#pragma unroll
      for (int q = 0; q < 32; ++q)
        v[q] = g.epi == EPI_SYRK ? v[q] * S : fmaf(g.coef_acc, v[q], g.coef_aux * ax[q]);
      staged_store(st, out, g.ldo, r0, c0, v);  // leaves the bf16 block in the tile
      // the mirrored block: element (c, r) at row c of the output
      uint4 q4[4];
      tile_transpose(st);
      __syncwarp();
      tile_get_blk(st, q4);
      blk_st(out, g.ldo, c0, r0, q4);
      __syncwarp();
      break;
    }
    case EPI_GEMM: {
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = fmaf(g.coef_aux, ax[q], v[q]) * S;
      staged_store(st, out, g.ldo, r0, c0, v);
      break;
    }
    case EPI_FINAL_DIMUON: {
      const float rr = g.R[r];
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        v[q] = round_to(fmaf(g.coef_aux, ax[q], v[q]) * S, DT_BF16);
        const float y = rr * v[q] * g.C[c0 + q];
        sx += v[q] * v[q];
        sy += y * y;
      }
      staged_store(st, out, g.ldo, r0, c0, v);
      break;
    }
    case EPI_FINAL_MUON: {
      const float ks = valid != 0.f ? g.kappa * S : 0.f;
#pragma unroll
      for (int q = 0; q < 32; ++q) v[q] = (valid != 0.f) ? fmaf(g.coef_aux, ax[q], v[q]) * ks : 0.f;
      __nv_bfloat16* W = reinterpret_cast<__nv_bfloat16*>(g.W);
      uint4 q4[4];
      float w[32];
      blk_ld(W, g.ldw, r0, c0, q4);
      tile_put_blk(st, q4);
      __syncwarp();
      tile_get_row(st, w);
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 32; ++q) w[q] = decay * w[q] - lr * v[q];
      staged_store(st, W, g.ldw, r0, c0, w);
      if (g.upd) {
        const int64_t wi = (int64_t)r * g.ldw + c0;
        if (aligned16(g.upd + wi)) {
#pragma unroll
          for (int q = 0; q < 4; ++q) st8(g.upd, wi + 8 * q, DT_FP32, v + 8 * q);
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) g.upd[wi + q] = v[q];
        }
      }
      break;
    }
  }
}

// The aux of one chunk in flight: a whole block for staged chunks, the
// thread's row otherwise.
struct AuxPrefetch {
  float row[32];
  uint4 blk[4];
  float S, valid;  // the product's scalars (written by an earlier launch)
};

// The product's scalars, loaded with the first aux block before the wait on
// the accumulator.
__device__ __forceinline__ void fetch_scalars(const GemmMat& g, AuxPrefetch& pf) {
  pf.S = g.scal_idx >= 0 ? g.scal[g.scal_idx] : 1.f;
  pf.valid = g.scal ? g.scal[SC_VALID] : 1.f;
}

__device__ __forceinline__ void fetch_aux(const GemmMat& g, int r, bool row_ok, int col0, int ch,
                                          int ch_end, int nch, AuxPrefetch& pf) {
  if (!needs_aux(g.epi) || ch >= ch_end || ch >= nch) return;
  const int r0 = r - (int)(threadIdx.x & 31);
  const int c0 = col0 + ch * 32;
  const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(g.aux);
  if (staged_ok(g, r0, c0))
    blk_ld(ab, g.ldaux, r0, c0, pf.blk);
  else if (row_ok)
    load_row32(ab, g.ldaux, r, c0, g.N, pf.row);
}

// Epilogue of chunks [ch_begin, ch_end) (32 columns each) of one accumulator
// row: tcgen05.ld of each chunk, with the next chunk's aux in flight while
// the current one is processed.  `pf` holds chunk ch_begin's aux and the
// scalars, fetched by the caller (fetch_aux, fetch_scalars) before it waited
// for the accumulator, since they do not depend on it.  Must be executed by all 32 lanes of the warp
// (tcgen05.ld is warp-collective); rows outside the matrix only skip stores.
// `st` is this warp's staging tile (STAGE_TILE_BYTES of shared memory).
__device__ __forceinline__ void epilogue_row(const GemmMat& g, float lr, float decay, int r,
                                             bool row_ok, int col0, uint32_t taddr, int ch_begin,
                                             int ch_end, int nch, float& sx, float& sy,
                                             __nv_bfloat16* st, AuxPrefetch& pf) {
  const int r0 = r - (int)(threadIdx.x & 31);
  const float S = pf.S, valid = pf.valid;
  const bool aux = needs_aux(g.epi);
#pragma unroll 1
  for (int ch = ch_begin; ch < ch_end; ++ch) {
    float v[32], ax[32];
    uint4 q[4];
    tmem_ld32_at(taddr + (uint32_t)(ch * 32), v);
    const int c0 = col0 + ch * 32;
    const bool stg = ch < nch && staged_ok(g, r0, c0);
#pragma unroll
    for (int k = 0; k < 4; ++k) q[k] = pf.blk[k];
#pragma unroll
    for (int k = 0; k < 32; ++k) ax[k] = pf.row[k];
    fetch_aux(g, r, row_ok, col0, ch + 1, ch_end, nch, pf);
    if (stg) {
      if (aux) {
        tile_put_blk(st, q);
        __syncwarp();
        tile_get_row(st, ax);
        __syncwarp();
      }
      staged_epilogue32(g, lr, decay, r, r0, c0, v, ax, S, valid, sx, sy, st);
    } else if (row_ok && ch < nch) {
      epilogue32(g, lr, decay, r, c0, v, ax, S, valid, sx, sy);
    }
  }
}

}  // namespace tcepi
}  // namespace dm
