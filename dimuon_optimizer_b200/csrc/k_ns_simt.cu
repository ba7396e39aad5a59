// fp32 SIMT products of the quintic Newton-Schulz iteration (precision mode
// DM_PREC_FP32).  One launch runs one product kind for a group of matrices:
//   A = X X^T (symmetric), B = b A + c A A (symmetric), X' = a X + B X
// (sitech.ge Muon post, "Instead of SVD - Newton-Schulz";
//  "Muon Optimizer 정리", "Why orthogonalise").  The last product of the step
// also applies the update (Muon) or emits X_5 and its norm partials (Dimuon).
// 128 x 128 output tiles (64 x 64 when the launch has too few tiles of 128
// to fill the SMs), 256 threads, an 8 x 8 (4 x 4) register block per thread.
#include "dm_common.cuh"
#include "dm_tiles.cuh"

namespace dm {
namespace {

#ifndef DM_SIMT_MINB
#define DM_SIMT_MINB 2  // resident CTAs per SM asked of the 128 x 128 kernel
#endif
constexpr int SK = 16;    // k per stage
constexpr int PADF = 4;   // row padding of the staged slabs (floats)

__device__ __forceinline__ float load_op(const float* p, int ld, int mn, int i, int k, int I, int K) {
  if (i >= I || k >= K) return 0.f;
  return mn ? p[(int64_t)k * ld + i] : p[(int64_t)i * ld + k];
}

// One TB x SK operand slab (element (i, k) at mn ? p[k ld + i] : p[i ld + k])
// in registers, V floats per thread: 4-float vectors along the operand's
// contiguous direction when the slab is inside the matrix and the rows are
// 16-byte aligned (the workspace buffers always are), else element by
// element with zero fill.
template <int TB>
struct Slab {
  static constexpr int V = TB * SK / 256;  // floats per thread
  float v[V];

  __device__ __forceinline__ void load(const float* p, int ld, int mn, int i0, int k0, int I, int K,
                                       bool vec) {
    const int t = threadIdx.x;
    if (vec) {
#pragma unroll
      for (int q = 0; q < V / 4; ++q) {
        const int idx = t + 256 * q;
        float4 f;
        if (mn) {  // contiguous along i: row kk, columns 4 ii4 .. +3
          const int kk = idx / (TB / 4), ii4 = idx % (TB / 4);
          f = *reinterpret_cast<const float4*>(p + (int64_t)(k0 + kk) * ld + i0 + 4 * ii4);
        } else {   // contiguous along k: row ii, k 4 kk4 .. +3
          const int ii = idx / (SK / 4), kk4 = idx % (SK / 4);
          f = *reinterpret_cast<const float4*>(p + (int64_t)(i0 + ii) * ld + k0 + 4 * kk4);
        }
        v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < V / 4; ++q) {
        const int idx = t + 256 * q;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int ii, kk;
          if (mn) {
            kk = idx / (TB / 4);
            ii = 4 * (idx % (TB / 4)) + e;
          } else {
            ii = idx / (SK / 4);
            kk = 4 * (idx % (SK / 4)) + e;
          }
          v[4 * q + e] = load_op(p, ld, mn, i0 + ii, k0 + kk, I, K);
        }
      }
    }
  }

  // Into s[k][i] (k-major staging for the inner product).
  __device__ __forceinline__ void store(float (*s)[TB + PADF], int mn) const {
    const int t = threadIdx.x;
#pragma unroll
    for (int q = 0; q < V / 4; ++q) {
      const int idx = t + 256 * q;
      if (mn) {
        const int kk = idx / (TB / 4), ii4 = idx % (TB / 4);
        *reinterpret_cast<float4*>(&s[kk][4 * ii4]) =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      } else {
        const int ii = idx / (SK / 4), kk4 = idx % (SK / 4);
#pragma unroll
        for (int e = 0; e < 4; ++e) s[4 * kk4 + e][ii] = v[4 * q + e];
      }
    }
  }
};

__device__ __forceinline__ void sym_store_f32(const GemmMat& g, int r, int c, float v) {
  float* o = reinterpret_cast<float*>(g.out);
  if (c >= r) o[(int64_t)r * g.ldo + c] = v;
  if (c > r) o[(int64_t)c * g.ldo + r] = v;
}

// TB x TB output tiles, 256 threads in a 16 x 16 grid, an RB x RB register
// block per thread (RB = TB / 16: rows ty * RB/2 .. and TB/2 + ty * RB/2 ..,
// likewise for columns).  The next k slab is read into registers while the
// current one is multiplied, and staged in the other shared-memory buffer:
// one barrier per k step.
template <int TB>
__global__ void __launch_bounds__(256, TB == 128 ? DM_SIMT_MINB : 3)
    simt_ns_product(const __grid_constant__ SimtParams p) {
  constexpr int RB = TB / 16, H = RB / 2;
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  __shared__ __align__(16) float As[2][SK][TB + PADF];
  __shared__ __align__(16) float Bs[2][SK][TB + PADF];
  __shared__ float red[2][8];
  const int gi = find_group(p.starts, p.count, blockIdx.x);
  const SimtMat& sm = p.mats[gi];
  const GemmMat& g = sm.g;
  const int lt = blockIdx.x - p.starts[gi];
  int tm, tn;
  gemm_tile_coord(g, lt, TB, TB, tm, tn);
  const int i0 = tm * TB, j0 = tn * TB;
  const int a_mn = g.flags & GF_A_MN ? 1 : 0, b_mn = g.flags & GF_B_MN ? 1 : 0;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const bool al_a = (sm.lda & 3) == 0 && (reinterpret_cast<uintptr_t>(sm.a) & 15u) == 0;
  const bool al_b = (sm.ldb & 3) == 0 && (reinterpret_cast<uintptr_t>(sm.b) & 15u) == 0;
  auto vec_ok = [&](bool al, int i_0, int I, int k_0) {
    return al && i_0 + TB <= I && k_0 + SK <= g.K;
  };

  float acc[RB][RB];
#pragma unroll
  for (int i = 0; i < RB; ++i)
#pragma unroll
    for (int j = 0; j < RB; ++j) acc[i][j] = 0.f;

  Slab<TB> la, lb;
  la.load(sm.a, sm.lda, a_mn, i0, 0, g.M, g.K, vec_ok(al_a, i0, g.M, 0));
  lb.load(sm.b, sm.ldb, b_mn, j0, 0, g.N, g.K, vec_ok(al_b, j0, g.N, 0));
  la.store(As[0], a_mn);
  lb.store(Bs[0], b_mn);
  __syncthreads();
  int buf = 0;
  for (int k0 = 0; k0 < g.K; k0 += SK) {
    const bool more = k0 + SK < g.K;
    if (more) {
      la.load(sm.a, sm.lda, a_mn, i0, k0 + SK, g.M, g.K, vec_ok(al_a, i0, g.M, k0 + SK));
      lb.load(sm.b, sm.ldb, b_mn, j0, k0 + SK, g.N, g.K, vec_ok(al_b, j0, g.N, k0 + SK));
    }
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float av[RB], bv[RB];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float* pa = &As[buf][kk][h * (TB / 2) + ty * H];
        const float* pb = &Bs[buf][kk][h * (TB / 2) + tx * H];
        if constexpr (H == 4) {
          const float4 a4 = *reinterpret_cast<const float4*>(pa);
          const float4 b4 = *reinterpret_cast<const float4*>(pb);
          av[h * H] = a4.x; av[h * H + 1] = a4.y; av[h * H + 2] = a4.z; av[h * H + 3] = a4.w;
          bv[h * H] = b4.x; bv[h * H + 1] = b4.y; bv[h * H + 2] = b4.z; bv[h * H + 3] = b4.w;
        } else {
          static_assert(H == 2, "register block halves of 2 or 4");
          const float2 a2 = *reinterpret_cast<const float2*>(pa);
          const float2 b2 = *reinterpret_cast<const float2*>(pb);
          av[h * H] = a2.x; av[h * H + 1] = a2.y;
          bv[h * H] = b2.x; bv[h * H + 1] = b2.y;
        }
      }
#pragma unroll
      for (int i = 0; i < RB; ++i)
#pragma unroll
        for (int j = 0; j < RB; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (more) {
      la.store(As[buf ^ 1], a_mn);
      lb.store(Bs[buf ^ 1], b_mn);
    }
    __syncthreads();
    buf ^= 1;
  }

  // Epilogue.
  const float S = g.scal_idx >= 0 ? g.scal[g.scal_idx] : 1.f;
  const float valid = g.scal ? g.scal[SC_VALID] : 1.f;
  float sx = 0.f, sy = 0.f;
#pragma unroll
  for (int i = 0; i < RB; ++i) {
    const int r = i0 + (i < H ? ty * H + i : TB / 2 + ty * H + (i - H));
    if (r >= g.M) continue;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      const int c = j0 + (j < H ? tx * H + j : TB / 2 + tx * H + (j - H));
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

}  // namespace

cudaError_t launch_simt(const SimtParams& p, int total_tiles, int tile, cudaStream_t s) {
  if (total_tiles <= 0) return cudaSuccess;
  if (tile == 64)
    simt_ns_product<64><<<total_tiles, 256, 0, s>>>(p);
  else
    simt_ns_product<128><<<total_tiles, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace dm
