// fp32 SIMT products of the quintic Newton-Schulz iteration (precision mode
// DM_PREC_FP32).  One launch runs one product kind for a group of matrices:
//   A = X X^T (symmetric), B = b A + c A A (symmetric), X' = a X + B X
// (sitech.ge Muon post, "Instead of SVD - Newton-Schulz";
//  "Muon Optimizer 정리", "Why orthogonalise").  The last product of the step
// also applies the update (Muon) or emits X_5 and its norm partials (Dimuon).
// 128 x 128 output tiles, 256 threads, an 8 x 8 register block per thread.
#include "dm_common.cuh"
#include "dm_tiles.cuh"

namespace dm {

constexpr int SB = 128;  // tile edge
constexpr int SK = 16;   // k step

__device__ __forceinline__ float load_op(const float* p, int ld, int mn, int i, int k, int I, int K) {
  if (i >= I || k >= K) return 0.f;
  return mn ? p[(int64_t)k * ld + i] : p[(int64_t)i * ld + k];
}

// Loads a 128 x 16 operand slab into s[k][i].
__device__ __forceinline__ void load_slab(float (*s)[SB], const float* p, int ld, int mn, int i0,
                                          int k0, int I, int K) {
#pragma unroll
  for (int e = 0; e < (SB * SK) / 256; ++e) {
    const int idx = threadIdx.x + 256 * e;
    int ii, kk;
    if (mn) {  // contiguous along i
      kk = idx / SB;
      ii = idx % SB;
    } else {   // contiguous along k
      ii = idx / SK;
      kk = idx % SK;
    }
    s[kk][ii] = load_op(p, ld, mn, i0 + ii, k0 + kk, I, K);
  }
}

__device__ __forceinline__ void sym_store_f32(const GemmMat& g, int r, int c, float v) {
  float* o = reinterpret_cast<float*>(g.out);
  if (c >= r) o[(int64_t)r * g.ldo + c] = v;
  if (c > r) o[(int64_t)c * g.ldo + r] = v;
}

__global__ void __launch_bounds__(256) simt_ns_product(const __grid_constant__ SimtParams p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  __shared__ __align__(16) float As[SK][SB];
  __shared__ __align__(16) float Bs[SK][SB];
  __shared__ float red[2][8];
  const int gi = find_group(p.starts, p.count, blockIdx.x);
  const SimtMat& sm = p.mats[gi];
  const GemmMat& g = sm.g;
  const int lt = blockIdx.x - p.starts[gi];
  int tm, tn;
  gemm_tile_coord(g, lt, SB, SB, tm, tn);
  const int i0 = tm * SB, j0 = tn * SB;
  const int a_mn = g.flags & GF_A_MN ? 1 : 0, b_mn = g.flags & GF_B_MN ? 1 : 0;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < g.K; k0 += SK) {
    load_slab(As, sm.a, sm.lda, a_mn, i0, k0, g.M, g.K);
    load_slab(Bs, sm.b, sm.ldb, b_mn, j0, k0, g.N, g.K);
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float av[8], bv[8];
      const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
      av[0] = a0.x; av[1] = a0.y; av[2] = a0.z; av[3] = a0.w;
      av[4] = a1.x; av[5] = a1.y; av[6] = a1.z; av[7] = a1.w;
      bv[0] = b0.x; bv[1] = b0.y; bv[2] = b0.z; bv[3] = b0.w;
      bv[4] = b1.x; bv[5] = b1.y; bv[6] = b1.z; bv[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

  // Epilogue.
  const float S = g.scal_idx >= 0 ? g.scal[g.scal_idx] : 1.f;
  const float valid = g.scal ? g.scal[SC_VALID] : 1.f;
  float sx = 0.f, sy = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = i0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (r >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = j0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (c >= g.N) continue;
      const float a = acc[i][j];
      switch (g.epi) {
        case EPI_SYRK:
          sym_store_f32(g, r, c, a * S);
          break;
        case EPI_POLY: {
          const float ax = reinterpret_cast<const float*>(g.aux)[(int64_t)r * g.ldaux + c];
          sym_store_f32(g, r, c, fmaf(g.coef_acc, a, g.coef_aux * ax));
          break;
        }
        case EPI_GEMM: {
          const float ax = reinterpret_cast<const float*>(g.aux)[(int64_t)r * g.ldaux + c];
          reinterpret_cast<float*>(g.out)[(int64_t)r * g.ldo + c] = fmaf(g.coef_aux, ax, a) * S;
          break;
        }
        case EPI_FINAL_MUON: {
          const float ax = reinterpret_cast<const float*>(g.aux)[(int64_t)r * g.ldaux + c];
          const float x = fmaf(g.coef_aux, ax, a) * S;
          const float o = valid != 0.f ? g.kappa * x : 0.f;
          const int64_t wi = (int64_t)r * g.ldw + c;
          st_elem(g.W, wi, g.wdt, p.decay * ld_elem(g.W, wi, g.wdt) - p.lr * o);
          if (g.upd) g.upd[wi] = o;
          break;
        }
        case EPI_FINAL_DIMUON: {
          const float ax = reinterpret_cast<const float*>(g.aux)[(int64_t)r * g.ldaux + c];
          const float x = fmaf(g.coef_aux, ax, a) * S;
          reinterpret_cast<float*>(g.out)[(int64_t)r * g.ldo + c] = x;
          const float y = g.R[r] * x * g.C[c];
          sx += x * x;
          sy += y * y;
          break;
        }
      }
    }
  }
  if (g.epi == EPI_FINAL_DIMUON) {
    sx = warp_sum(sx);
    sy = warp_sum(sy);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    if (lane == 0) {
      red[0][w] = sx;
      red[1][w] = sy;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float tx_ = 0.f, ty_ = 0.f;
      for (int q = 0; q < 8; ++q) {
        tx_ += red[0][q];
        ty_ += red[1][q];
      }
      const int tile_id = tm * g.tiles_n + tn;
      g.part[2 * tile_id] = tx_;
      g.part[2 * tile_id + 1] = ty_;
    }
  }
}

cudaError_t launch_simt(const SimtParams& p, int total_tiles, cudaStream_t s) {
  if (total_tiles <= 0) return cudaSuccess;
  simt_ns_product<<<total_tiles, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace dm
