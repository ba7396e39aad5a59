// Pieces shared by the thin-factor kernels (k_thin.cu: register path and
// the r x r iteration; k_thin_bulk.cu: shared-memory staged path): the
// padded-rank configuration, the fp64 tensor-core MMA, the conditioning
// weight, vector element access and the factor geometry.
#pragma once

#include <cuda_bf16.h>

#include "dm_common.cuh"

namespace dm {
namespace thin {

constexpr int TT = 128;  // threads per CTA
constexpr int TW = TT / 32;

template <int RP>
struct TCfg {
  static constexpr bool MMA = RP >= 8;
  static constexpr int NB = MMA ? RP / 8 : 1;       // 8-row blocks
  static constexpr int KB = MMA ? RP / 4 : 1;       // 4-wide k steps
  static constexpr int NUB = NB * (NB + 1) / 2;     // upper-triangle 8x8 blocks
  static constexpr int PART = MMA ? NUB * 64 : RP * RP;  // doubles per Gram partial
  // padded r x r row of the iteration's shared matrices: RP + 4 doubles puts
  // the MMA fragment reads of 16 lanes on 16 distinct 8-byte bank pairs
  static constexpr int SLD = RP >= 16 ? RP + 4 : RP + 1;
  // long-side columns per slab (work unit of thin_gram / thin_apply)
  static constexpr int SLAB = RP <= 4 ? 2048 : RP <= 16 ? 512 : 1024;
  // the next step's loads are issued before the current step computes
  static constexpr bool DB = RP <= 16;
};

// D (8x8, two values per lane) += A (8x4) * B (4x8) in fp64.
// Lane l = 4g + t holds A[g][t], B[t][g], D[g][2t], D[g][2t+1].
__device__ __forceinline__ void dmma(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

// Two fp32 values as bf16 pairs hi = RNE(x) and lo = RNE(x - hi): hi + lo
// carries x to about 2^-17 relative (x - hi is exact in fp32), so a product
// of two split operands taken as hi hi + hi lo + lo hi has an error of about
// 2^-16 relative per term (the dropped lo lo term and the two roundings).
// The first value goes to the low half, the k-slot order of the fragments.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// D (16x8, fp32) += A (16x16, bf16) * B (16x8, bf16).  Lane l = 4g + t holds
// A rows g, g + 8 at k slots 2t, 2t + 1 (a[0], a[1]) and 2t + 8, 2t + 9
// (a[2], a[3]); B column g at k slots 2t, 2t + 1 (b0) and 2t + 8, 2t + 9
// (b1); D rows g (d[0], d[1]) and g + 8 (d[2], d[3]) at columns 2t, 2t + 1.
__device__ __forceinline__ void hmma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A B for split operands: the small cross terms first, then hi hi.
__device__ __forceinline__ void hmma_split(float (&d)[4], const uint32_t (&ah)[4],
                                           const uint32_t (&al)[4], const uint32_t (&bh)[2],
                                           const uint32_t (&bl)[2]) {
  hmma16816(d, al, bh[0], bh[1]);
  hmma16816(d, ah, bl[0], bl[1]);
  hmma16816(d, ah, bh[0], bh[1]);
}

// C_j^2 = (e_j / mean(e) + eps)^(-1/2); the same expression in every launch.
__device__ __forceinline__ float col_weight(float e, float inv_mean, float eps) {
  return rsqrtf(__fmaf_rn(e, inv_mean, eps));
}

// 4 consecutive elements at flat index i (aligned to 4 elements).
__device__ __forceinline__ void ld4(const void* p, int64_t i, int dt, float v[4]) {
  if (dt == DT_BF16) {
    const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(p) + i);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  } else {
    const float4 f = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + i);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
}

__device__ __forceinline__ void st4(void* p, int64_t i, int dt, const float v[4]) {
  if (dt == DT_BF16) {
    uint2 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
    h[0] = __floats2bfloat162_rn(v[0], v[1]);
    h[1] = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p) + i) = u;
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + i) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// Two consecutive elements (aligned to 2 elements).
__device__ __forceinline__ void ld2(const void* p, int64_t i, int dt, float& v0, float& v1) {
  if (dt == DT_BF16) {
    const float2 a = __bfloat1622float2(
        *reinterpret_cast<const __nv_bfloat162*>(reinterpret_cast<const __nv_bfloat16*>(p) + i));
    v0 = a.x; v1 = a.y;
  } else {
    const float2 f = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(p) + i);
    v0 = f.x; v1 = f.y;
  }
}

__device__ __forceinline__ void st2(void* p, int64_t i, int dt, float v0, float v1) {
  if (dt == DT_BF16)
    *reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(p) + i) =
        __floats2bfloat162_rn(v0, v1);
  else
    *reinterpret_cast<float2*>(reinterpret_cast<float*>(p) + i) = make_float2(v0, v1);
}

// Factor geometry in the orientation of the iteration: r short-side rows,
// n long-side columns; element (i, j) sits at j * r + i (tall storage) or
// i * n + j (wide storage).
struct Geo {
  bool tall;
  int r;
  int64_t n;
  float* e_r;  // energies along the short side (r entries)
  float* e_c;  // energies along the long side (n entries)
  bool cond;
  bool vec;    // 4-element vector access is aligned
  __device__ __forceinline__ int64_t off(int i, int64_t j) const {
    return tall ? j * r + i : (int64_t)i * n + j;
  }
};

__device__ __forceinline__ Geo geometry(const ThinMat& mt, int conditioned) {
  Geo q;
  q.tall = mt.rows > mt.cols;
  q.r = (int)(q.tall ? mt.cols : mt.rows);
  q.n = q.tall ? mt.rows : mt.cols;
  q.e_r = q.tall ? mt.e_col : mt.e_row;
  q.e_c = q.tall ? mt.e_row : mt.e_col;
  q.cond = conditioned && q.e_r != nullptr && q.e_c != nullptr;
  // wide rows must start on 4-element boundaries; tall runs of four
  // long-side columns are 4r contiguous elements starting at a multiple of 4r
  q.vec = mt.vec && (q.tall || (q.n & 3) == 0);
  return q;
}

// ---------------------------------------------------------------------------
// The r x r Newton-Schulz iteration of one factor by one warp (RP <= 8; no
// block-wide barrier).  The iterate is X_k = P_k X_0 with P_k an r x r
// polynomial in A_0 = X_0 X_0^T ("From PCG to Muon", section 6 "Muon's Gram
// Matrix"): P_k = Q_k P_{k-1}, A_k = Q_k A_{k-1} Q_k with
// Q_k = a_k I + b_k A_{k-1} + c_k A_{k-1}^2 (sitech.ge Muon post, "Instead of
// SVD - Newton-Schulz"), A normalised by ||X_0||_F^2 = tr A_0.
// ---------------------------------------------------------------------------
template <int RP>
struct WarpIterSmem {
  double G[RP][RP + 1], H[RP][RP + 1], P[RP][RP + 1], A[RP][RP + 1], Q[RP][RP + 1], S[RP][RP + 1];
  double R[RP];
};

template <int RP>
__device__ __forceinline__ void mm_warp(double (*C)[RP + 1], double (*A)[RP + 1], double (*B)[RP + 1]) {
  const int lane = threadIdx.x & 31;
  if constexpr (RP == 8) {
    const int g = lane >> 2, t = lane & 3;
    double d0 = 0.0, d1 = 0.0;
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) dmma(d0, d1, A[g][kb * 4 + t], B[kb * 4 + t][g]);
    __syncwarp();  // every lane has read A and B (C may alias neither, but keep order)
    C[g][2 * t] = d0;
    C[g][2 * t + 1] = d1;
  } else {
    static_assert(RP * RP <= 32, "one lane per element");
    if (lane < RP * RP) {
      const int i = lane / RP, j = lane % RP;
      double s = 0.0;
#pragma unroll
      for (int k = 0; k < RP; ++k) s = fma(A[i][k], B[k][j], s);
      C[i][j] = s;
    }
  }
  __syncwarp();
}

// What the iteration needs besides the two Gram sums.
struct IterIn {
  double sc, sr;          // sums of the previous long- / short-side energies
  bool cond;              // Dimuon energies given
  int r;                  // short side (<= RP)
  const float* e_r;       // previous short-side energies (read before they are replaced)
  float eps;              // conditioning damping
  const float (*coef)[3]; // (a_k, b_k, c_k) per iteration
  int ns_steps;
  float kappa;            // update scale
  int* status;            // device status word (non-finite norm)
};

// On entry s.G and s.H hold S_1 = sum_j C_j^2 b_j b_j^T and S_2 = sum_j C_j^4
// b_j b_j^T.  On return s.R holds R, s.P holds P_5, and the result is the
// update factor kappa / ||X_0|| (times ||X_5|| / ||R X_5 C|| when
// conditioning is on; "Dimuon: LoRA 에 맞춰 다시 짠 Muon", Problem 4 (c)), 0
// for a degenerate norm; *on_out tells whether conditioning was on.
template <int RP>
__device__ double iterate_gram_warp(const IterIn& in, WarpIterSmem<RP>& s, bool* on_out) {
  const int lane = threadIdx.x & 31;
  const int r = in.r;
  const bool on = in.cond && in.sr > 0.0 && in.sc > 0.0;
  if (lane < RP) {
    double rv = lane < r ? 1.0 : 0.0;
    if (on && lane < r) rv = 1.0 / sqrt(sqrt((double)in.e_r[lane] * ((double)r / in.sr) + (double)in.eps));
    s.R[lane] = rv;
  }
  __syncwarp();
  double tr = 0.0;
  for (int idx = lane; idx < RP * RP; idx += 32) {
    const int i = idx / RP, j = idx % RP;
    const double rr = s.R[i] * s.R[j];
    s.G[i][j] *= rr;
    s.H[i][j] *= rr;
    if (i == j) tr += s.G[i][j];
  }
  const double s2 = warp_sum_d(tr);
  const bool finite = isfinite(s2);
  const bool valid = finite && s2 >= NORM2_FLOOR;
  const double inv_s2 = valid ? 1.0 / s2 : 0.0;
  for (int idx = lane; idx < RP * RP; idx += 32) {
    const int i = idx / RP, j = idx % RP;
    s.A[i][j] = valid ? s.G[i][j] * inv_s2 : 0.0;
    s.P[i][j] = i == j ? 1.0 : 0.0;
  }
  __syncwarp();
  for (int it = 0; it < in.ns_steps; ++it) {
    const double a = in.coef[it][0], b = in.coef[it][1], c = in.coef[it][2];
    mm_warp<RP>(s.Q, s.A, s.A);
    for (int idx = lane; idx < RP * RP; idx += 32) {
      const int i = idx / RP, j = idx % RP;
      s.Q[i][j] = c * s.Q[i][j] + b * s.A[i][j] + (i == j ? a : 0.0);
    }
    __syncwarp();
    mm_warp<RP>(s.S, s.Q, s.P);
    for (int idx = lane; idx < RP * RP; idx += 32) s.P[idx / RP][idx % RP] = s.S[idx / RP][idx % RP];
    __syncwarp();
    mm_warp<RP>(s.S, s.Q, s.A);
    mm_warp<RP>(s.A, s.S, s.Q);
  }
  // ||X_5||^2 s^2 = tr(P A_0 P^T); ||R X_5 C||^2 s^2 = sum_i R_i^2 (P H P^T)_ii
  mm_warp<RP>(s.S, s.P, s.G);
  double nx = 0.0;
  for (int idx = lane; idx < RP * RP; idx += 32) nx += s.S[idx / RP][idx % RP] * s.P[idx / RP][idx % RP];
  nx = warp_sum_d(nx);
  mm_warp<RP>(s.Q, s.P, s.H);
  double ny = 0.0;
  for (int idx = lane; idx < RP * RP; idx += 32) {
    const int i = idx / RP;
    ny += s.R[i] * s.R[i] * s.Q[i][idx % RP] * s.P[i][idx % RP];
  }
  ny = warp_sum_d(ny);
  double factor = 0.0;
  if (valid) {
    factor = (double)in.kappa / sqrt(s2);
    if (on) factor = ny > 0.0 ? factor * sqrt(nx / ny) : 0.0;
  }
  if (!finite && lane == 0) raise_status(in.status, ST_NONFINITE);
  *on_out = on;
  return factor;
}

}  // namespace thin
}  // namespace dm
