// Whole Muon / Dimuon step for thin factors (short side r <= 32, e.g. LoRA A
// (r x n) and B (n x r)) in one CTA per factor.
//
// The Newton-Schulz iterate is a left-multiple of the start matrix: each step
// X <- (aI + bA + cA^2) X with A = X X^T, so X_k = P_k X_0 with an r x r
// polynomial P_k in the Gram matrix A_0 = X_0 X_0^T; A_{k+1} = Q_k A_k Q_k.
// ("From PCG to Muon", section 6 "Muon's Gram Matrix": the orthogonaliser
// normalises the global Gram matrix G^T G; sitech.ge, "Instead of SVD -
// Newton-Schulz" for the iteration itself.)  So the factor is streamed
// twice and all iteration work happens in r x r space:
//   pass 1  M_t = mu M_{t-1} + G (stored), X_0 = R M_t C in fp64, A_0 += X_0
//           X_0^T (fp64, exact products), H += X_0 C^2 X_0^T, row energies
//   iterate P <- Q P, A <- Q A Q in fp64 shared memory; Frobenius norms of
//           X_5 = P X_0 / s and Y = R X_5 C follow from A_0 and H
//   pass 2  reload M_t (L2-resident), O = (factor) R (P X_0) C, W update,
//           column energies of M_t
// Dimuon conditioning, renormalisation, scale and decay follow "Dimuon: LoRA
// 에 맞춰 다시 짠 Muon" ("-1/4 power from both sides", Problem 4) and
// "Muon Optimizer 정리" (eq. (1)-(3), "Scaling up").
#include "dm_common.cuh"

namespace dm {
namespace {

constexpr int CH = 64;  // columns per chunk

template <int RP>
struct ThinSmem {
  double xs[RP][CH];       // X_0 chunk (fp64)
  float ms[RP][CH];        // stored momentum chunk / update chunk
  double G[RP][RP];        // A_0
  double H[RP][RP];        // X_0 C^2 X_0^T
  union {
    double part[256 * 16];           // per-thread 4x4 Gram partials
    struct {
      double P[RP][RP], A[RP][RP], Q[RP][RP], T[RP][RP];
    } it;
  } u;
  float Rv[RP];
  float Cc[CH];
  double red[32];
  double sc[4];
};

// C = A * B for RP x RP fp64 matrices in shared memory.
template <int RP>
__device__ __forceinline__ void mm(double (*C)[RP], double (*A)[RP], double (*B)[RP]) {
  for (int idx = threadIdx.x; idx < RP * RP; idx += blockDim.x) {
    const int i = idx / RP, j = idx % RP;
    double s = 0.0;
#pragma unroll 8
    for (int k = 0; k < RP; ++k) s = fma(A[i][k], B[k][j], s);
    C[i][j] = s;
  }
  __syncthreads();
}

template <int RP>
__global__ void __launch_bounds__(256) thin_step(const __grid_constant__ ThinParams p) {
  constexpr int NB = RP / 4, NBLK = NB * NB, TPB = 256 / NBLK;
  static_assert(TPB * NBLK == 256, "block split");
  static_assert(TPB <= 64, "partials buffer");
  extern __shared__ __align__(16) uint8_t smem_raw[];
  ThinSmem<RP>& s = *reinterpret_cast<ThinSmem<RP>*>(smem_raw);
  const int tid = threadIdx.x;

  const ThinMat& mt = p.mats[blockIdx.x];
  const bool tall = mt.rows > mt.cols;
  const int r = (int)(tall ? mt.cols : mt.rows);
  const int64_t n = tall ? mt.rows : mt.cols;
  float* e_r = tall ? mt.e_col : mt.e_row;  // energies along the short side
  float* e_c = tall ? mt.e_row : mt.e_col;  // energies along the long side
  const bool cond = p.conditioned && e_r != nullptr && e_c != nullptr;
  auto off = [&](int i, int64_t k) -> int64_t { return tall ? k * r + i : (int64_t)i * n + k; };

  // ---- conditioning from the previous momentum's energies ------------------
  double sr = 0.0, sc = 0.0;
  if (cond) {
    for (int i = tid; i < r; i += 256) sr += (double)e_r[i];
    for (int64_t k = tid; k < n; k += 256) sc += (double)e_c[k];
  }
  sr = block_sum_d(sr, s.red);
  sc = block_sum_d(sc, s.red);
  const bool on = cond && sr > 0.0 && sc > 0.0;
  const float inv_mr = on ? (float)((double)r / sr) : 0.f;
  const float inv_mc = on ? (float)((double)n / sc) : 0.f;
  if (tid < RP)
    s.Rv[tid] = tid < r ? (on ? powf(e_r[tid] * inv_mr + p.eps, -0.25f) : 1.f) : 0.f;

  // ---- pass 1 --------------------------------------------------------------
  const int blk = tid / TPB, sub = tid % TPB;
  const int bi = blk / NB, bj = blk % NB;
  double ga[4][4];
  float ha[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      ga[a][b] = 0.0;
      ha[a][b] = 0.f;
    }
  float rowe = 0.f;

  for (int64_t k0 = 0; k0 < n; k0 += CH) {
    const int cw = (int)min((int64_t)CH, n - k0);
    if (tid < CH)
      s.Cc[tid] = tid < cw ? (on ? powf(e_c[k0 + tid] * inv_mc + p.eps, -0.25f) : 1.f) : 0.f;
    __syncthreads();
    for (int idx = tid; idx < RP * CH; idx += 256) {
      int i, kk;
      if (tall) { kk = idx / RP; i = idx % RP; } else { i = idx / CH; kk = idx % CH; }
      float m = 0.f;
      if (i < r && kk < cw) {
        const int64_t o = off(i, k0 + kk);
        m = momentum_value(p.mu, ld_elem(mt.M, o, mt.mdt), ld_elem(mt.G, o, mt.gdt), mt.mdt);
        st_elem(mt.M, o, mt.mdt, m);
      }
      s.ms[i][kk] = m;
      s.xs[i][kk] = (double)s.Rv[i] * (double)m * (double)s.Cc[kk];
    }
    __syncthreads();
    if (cond && tid >= 64 && tid < 64 + r) {
      const int i = tid - 64;
      for (int kk = 0; kk < cw; ++kk) rowe = fmaf(s.ms[i][kk], s.ms[i][kk], rowe);
    }
    for (int kk = sub; kk < CH; kk += TPB) {
      double xa[4], xb[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        xa[a] = s.xs[bi * 4 + a][kk];
        xb[a] = s.xs[bj * 4 + a][kk];
      }
      const float c2 = s.Cc[kk] * s.Cc[kk];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          ga[a][b] = fma(xa[a], xb[b], ga[a][b]);
          ha[a][b] = fmaf((float)(xa[a] * xb[b]), c2, ha[a][b]);
        }
    }
    __syncthreads();
  }
  if (cond && tid >= 64 && tid < 64 + r) e_r[tid - 64] = rowe;

  // ---- deterministic reduction of the Gram partials ------------------------
  // part[(sub * NBLK + blk) * 16 + a * 4 + b]: one 4 x 4 block per thread.
  for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b)
        s.u.part[(sub * NBLK + blk) * 16 + a * 4 + b] = pass == 0 ? ga[a][b] : (double)ha[a][b];
    __syncthreads();
    for (int idx = tid; idx < RP * RP; idx += 256) {
      const int i = idx / RP, j = idx % RP;
      const int bk = (i / 4) * NB + (j / 4), e = (i % 4) * 4 + (j % 4);
      double t = 0.0;
      for (int q = 0; q < TPB; ++q) t += s.u.part[(q * NBLK + bk) * 16 + e];
      if (pass == 0) s.G[i][j] = t; else s.H[i][j] = t;
    }
    __syncthreads();
  }

  // ---- Newton-Schulz in r x r space (fp64) ---------------------------------
  if (tid == 0) {
    double tr = 0.0;
    for (int i = 0; i < r; ++i) tr += s.G[i][i];
    s.sc[0] = tr;
  }
  __syncthreads();
  const double s2 = s.sc[0];
  const bool finite = isfinite(s2);
  const bool valid = finite && s2 >= NORM2_FLOOR;  // else the update is zero
  const double inv_s2 = valid ? 1.0 / s2 : 0.0;
  for (int idx = tid; idx < RP * RP; idx += 256) {
    const int i = idx / RP, j = idx % RP;
    s.u.it.A[i][j] = valid ? s.G[i][j] * inv_s2 : 0.0;
    s.u.it.P[i][j] = i == j ? 1.0 : 0.0;
  }
  __syncthreads();
  const double a = p.a, b = p.b, c = p.c;
  for (int it = 0; it < p.ns_steps; ++it) {
    mm<RP>(s.u.it.Q, s.u.it.A, s.u.it.A);  // Q = A A
    for (int idx = tid; idx < RP * RP; idx += 256) {
      const int i = idx / RP, j = idx % RP;
      s.u.it.Q[i][j] = c * s.u.it.Q[i][j] + b * s.u.it.A[i][j] + (i == j ? a : 0.0);
    }
    __syncthreads();
    mm<RP>(s.u.it.T, s.u.it.Q, s.u.it.P);  // P <- Q P
    for (int idx = tid; idx < RP * RP; idx += 256) s.u.it.P[idx / RP][idx % RP] = s.u.it.T[idx / RP][idx % RP];
    __syncthreads();
    mm<RP>(s.u.it.T, s.u.it.Q, s.u.it.A);  // A <- Q A Q
    mm<RP>(s.u.it.A, s.u.it.T, s.u.it.Q);
  }
  // ||X_5||^2 s^2 = tr(P A_0 P^T), ||R X_5 C||^2 s^2 = sum_i R_i^2 (P H P^T)_ii
  mm<RP>(s.u.it.T, s.u.it.P, s.G);
  double nx = 0.0;
  for (int idx = tid; idx < RP * RP; idx += 256) nx += s.u.it.T[idx / RP][idx % RP] * s.u.it.P[idx / RP][idx % RP];
  nx = block_sum_d(nx, s.red);
  mm<RP>(s.u.it.Q, s.u.it.P, s.H);
  double ny = 0.0;
  for (int idx = tid; idx < RP * RP; idx += 256) {
    const int i = idx / RP;
    ny += (double)s.Rv[i] * s.Rv[i] * s.u.it.Q[i][idx % RP] * s.u.it.P[i][idx % RP];
  }
  ny = block_sum_d(ny, s.red);
  double factor = 0.0;
  if (valid) {
    factor = (double)mt.kappa / sqrt(s2);
    if (on) factor = ny > 0.0 ? factor * sqrt(nx / ny) : 0.0;
  }
  if (!finite && tid == 0) raise_status(p.status, ST_NONFINITE);
  for (int idx = tid; idx < RP * RP; idx += 256) {
    const int i = idx / RP, j = idx % RP;
    s.u.it.T[i][j] = factor * s.u.it.P[i][j];
  }
  __syncthreads();

  // ---- pass 2 --------------------------------------------------------------
  const int kk_o = tid % CH, ig = tid / CH;  // 4 row groups
  for (int64_t k0 = 0; k0 < n; k0 += CH) {
    const int cw = (int)min((int64_t)CH, n - k0);
    if (tid < CH)
      s.Cc[tid] = tid < cw ? (on ? powf(e_c[k0 + tid] * inv_mc + p.eps, -0.25f) : 1.f) : 0.f;
    __syncthreads();
    for (int idx = tid; idx < RP * CH; idx += 256) {
      int i, kk;
      if (tall) { kk = idx / RP; i = idx % RP; } else { i = idx / CH; kk = idx % CH; }
      float m = 0.f;
      if (i < r && kk < cw) m = ld_elem(mt.M, off(i, k0 + kk), mt.mdt);
      s.ms[i][kk] = m;
      s.xs[i][kk] = (double)s.Rv[i] * (double)m * (double)s.Cc[kk];
    }
    __syncthreads();
    if (cond && tid < cw) {
      float e = 0.f;
      for (int i = 0; i < r; ++i) e = fmaf(s.ms[i][tid], s.ms[i][tid], e);
      e_c[k0 + tid] = e;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < RP / 4; ++q) {
      const int i = ig * (RP / 4) + q;
      double acc = 0.0;
#pragma unroll 8
      for (int j = 0; j < RP; ++j) acc = fma(s.u.it.T[i][j], s.xs[j][kk_o], acc);
      s.ms[i][kk_o] = factor != 0.0 ? (float)((double)s.Rv[i] * acc * (double)s.Cc[kk_o]) : 0.f;
    }
    __syncthreads();
    for (int idx = tid; idx < RP * CH; idx += 256) {
      int i, kk;
      if (tall) { kk = idx / RP; i = idx % RP; } else { i = idx / CH; kk = idx % CH; }
      if (i < r && kk < cw) {
        const int64_t o = off(i, k0 + kk);
        const float u = s.ms[i][kk];
        st_elem(mt.W, o, mt.wdt, p.decay * ld_elem(mt.W, o, mt.wdt) - p.lr * u);
        if (mt.upd) mt.upd[o] = u;
      }
    }
    __syncthreads();
  }
}

template <int RP>
cudaError_t launch_rp(const ThinParams& p, cudaStream_t st) {
  const int bytes = (int)sizeof(ThinSmem<RP>);
  static int configured = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured != dev) {
    cudaError_t e = cudaFuncSetAttribute(thin_step<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    configured = dev;
  }
  thin_step<RP><<<p.count, 256, bytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

// All factors of one launch share the padded short side RP = p.pad (8, 16, 32).
cudaError_t launch_thin(const ThinParams& p, cudaStream_t s) {
  if (p.count <= 0) return cudaSuccess;
  switch (p.pad) {
    case 8: return launch_rp<8>(p, s);
    case 16: return launch_rp<16>(p, s);
    default: return launch_rp<32>(p, s);
  }
}

}  // namespace dm
