// HBM-bound kernels of the Muon / Dimuon step:
//   K0  Dimuon conditioning vectors R, C from the previous momentum's energies
//       ("Dimuon: LoRA 에 맞춰 다시 짠 Muon", "-1/4 power from both sides",
//       Problem 4: (relative energy + eps)^(-1/4); off when M_{t-1} = 0,
//       "Why the *last* momentum").
//   K1  M_t = mu M_{t-1} + G ("Muon Optimizer 정리", "Update rule", eq. (1)),
//       X_0 = R M_t C (R B_t C with B_t = G + mu M_t under Nesterov), per-tile sums of squares of X_0 and partial row /
//       column energies of the stored M_t.
//   K1b deterministic reduction of the K1 partials: energies of M_t (output
//       for the next Dimuon step) and the Frobenius-norm scalars.
//   K3a Dimuon renormalisation factor kappa * ||X_5||_F / ||R X_5 C||_F
//       (Dimuon page, Problem 4 (c): the norm is fixed afterwards).
//   K3  W_t = (1 - lr wd) W_{t-1} - lr O_t with O_t = factor * R X_5 C
//       ("Muon Optimizer 정리", eq. (3) and "Scaling up").
#include "dm_common.cuh"

namespace dm {

// ---------------------------------------------------------------------------
// K0: one CTA per matrix.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k0_conditioning(const __grid_constant__ K0Params p) {
  __shared__ double red[32];
  const K0Mat& mt = p.mats[blockIdx.x];
  double sr = 0.0, sc = 0.0;
  for (int64_t i = threadIdx.x; i < mt.rows; i += blockDim.x) sr += (double)mt.e_row[i];
  for (int64_t j = threadIdx.x; j < mt.cols; j += blockDim.x) sc += (double)mt.e_col[j];
  sr = block_sum_d(sr, red);
  sc = block_sum_d(sc, red);
  // The conditioning is off as a whole when the previous momentum was zero.
  const bool on = (sr > 0.0) && (sc > 0.0);
  const float inv_mr = on ? (float)((double)mt.rows / sr) : 0.f;
  const float inv_mc = on ? (float)((double)mt.cols / sc) : 0.f;
  for (int64_t i = threadIdx.x; i < mt.rows; i += blockDim.x)
    mt.R[i] = on ? powf(mt.e_row[i] * inv_mr + p.eps, -0.25f) : 1.f;
  for (int64_t j = threadIdx.x; j < mt.cols; j += blockDim.x)
    mt.C[j] = on ? powf(mt.e_col[j] * inv_mc + p.eps, -0.25f) : 1.f;
}

// ---------------------------------------------------------------------------
// K1: one CTA per K1_ROWS x K1_COLS tile; 256 threads = 8 warps; lane l
// covers columns [c0 + 8l, c0 + 8l + 8), warp w covers rows w, w+8, ...
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k1_momentum(const __grid_constant__ K1Params p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  __shared__ float col_acc[8][K1_COLS];
  __shared__ float red[32];
  const int tile = blockIdx.x;
  const int g = find_group(p.starts, p.count, tile);
  const K1Mat& mt = p.mats[g];
  const int lt = tile - p.starts[g];
  const int rt = lt / mt.n_ct, ct = lt % mt.n_ct;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t r0 = (int64_t)rt * K1_ROWS;
  const int64_t c0 = (int64_t)ct * K1_COLS + lane * 8;
  const bool energies = mt.part_erow != nullptr;

  float cscale[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int64_t c = c0 + q;
    cscale[q] = (mt.C && c < mt.cols) ? mt.C[c] : 1.f;
  }
  float csum[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) csum[q] = 0.f;
  float xsq = 0.f;

  for (int rr = warp; rr < K1_ROWS; rr += 8) {
    const int64_t r = r0 + rr;
    if (r >= mt.rows) break;
    const float rs = mt.R ? mt.R[r] : 1.f;
    float g8[8], m8[8], x8[8];
    const int64_t base = r * mt.cols + c0;
    float rsum = 0.f;
    if (mt.vec) {
      if (c0 < mt.cols) {
        ld8(mt.G, base, mt.gdt, g8);
        ld8(mt.M, base, mt.mdt, m8);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          m8[q] = momentum_value(p.mu, m8[q], g8[q], mt.mdt);
          const float b = p.nesterov ? fmaf(p.mu, m8[q], g8[q]) : m8[q];
          x8[q] = round_to(rs * b * cscale[q], mt.xdt);
          rsum += m8[q] * m8[q];
          csum[q] += m8[q] * m8[q];
          xsq += x8[q] * x8[q];
        }
        st8(mt.M, base, mt.mdt, m8);
        st8(mt.X0, r * mt.ldx + c0, mt.xdt, x8);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int64_t c = c0 + q;
        if (c < mt.cols) {
          const float gv = ld_elem(mt.G, base + q, mt.gdt);
          const float mv = momentum_value(p.mu, ld_elem(mt.M, base + q, mt.mdt), gv, mt.mdt);
          const float bv = p.nesterov ? fmaf(p.mu, mv, gv) : mv;
          const float xv = round_to(rs * bv * cscale[q], mt.xdt);
          st_elem(mt.M, base + q, mt.mdt, mv);
          st_elem(mt.X0, r * mt.ldx + c, mt.xdt, xv);
          rsum += mv * mv;
          csum[q] += mv * mv;
          xsq += xv * xv;
        }
      }
    }
    if (energies) {
      rsum = warp_sum(rsum);
      if (lane == 0) mt.part_erow[(int64_t)ct * mt.rows + r] = rsum;
    }
  }

  const float tot = block_sum(xsq, red);
  if (threadIdx.x == 0) mt.part_sumsq[lt] = tot;
  if (energies) {
#pragma unroll
    for (int q = 0; q < 8; ++q) col_acc[warp][lane * 8 + q] = csum[q];
    __syncthreads();
    const int c = threadIdx.x;
    const int64_t cg = (int64_t)ct * K1_COLS + c;
    if (cg < mt.cols) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) s += col_acc[w][c];
      mt.part_ecol[(int64_t)rt * mt.cols + cg] = s;
    }
  }
}

// ---------------------------------------------------------------------------
// K1b: block 0 of each matrix reduces the norm partials; the other blocks
// each produce K1B_THREADS energies (rows first, then columns).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(K1B_THREADS) k1b_reduce(const __grid_constant__ K1bParams p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  __shared__ double red[32];
  const int g = find_group(p.starts, p.count, blockIdx.x);
  const K1bMat& mt = p.mats[g];
  const int lb = blockIdx.x - p.starts[g];
  if (lb == 0) {
    const int nt = mt.n_rt * mt.n_ct;
    double s = 0.0;
    for (int i = threadIdx.x; i < nt; i += blockDim.x) s += (double)mt.part_sumsq[i];
    s = block_sum_d(s, red);
    if (threadIdx.x == 0) {
      // A non-finite norm is reported; a norm below the floor is a zero
      // update.  Either way the update of this matrix is forced to zero.
      const bool finite = isfinite(s);
      const bool ok = finite && s >= NORM2_FLOOR;
      const double inv = ok ? 1.0 / sqrt(s) : 0.0;
      mt.scal[SC_SUMSQ] = (float)s;
      mt.scal[SC_INV_S] = (float)inv;
      mt.scal[SC_INV_S2] = (float)(inv * inv);
      mt.scal[SC_VALID] = ok ? 1.f : 0.f;
      if (!finite) raise_status(p.status, ST_NONFINITE);
    }
    return;
  }
  const int64_t idx = (int64_t)(lb - 1) * K1B_THREADS + threadIdx.x;
  if (idx < mt.rows) {
    float s = 0.f;
    for (int c = 0; c < mt.n_ct; ++c) s += mt.part_erow[(int64_t)c * mt.rows + idx];
    mt.e_row[idx] = s;
  } else if (idx < mt.rows + mt.cols) {
    const int64_t j = idx - mt.rows;
    float s = 0.f;
    for (int r = 0; r < mt.n_rt; ++r) s += mt.part_ecol[(int64_t)r * mt.cols + j];
    mt.e_col[j] = s;
  }
}

// ---------------------------------------------------------------------------
// K3a: one CTA per matrix.  Partials are (sum x^2, sum y^2) pairs written by
// the epilogue of the last Newton-Schulz product.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k3a_factor(const __grid_constant__ K3Params p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  __shared__ double red[32];
  const K3Mat& mt = p.mats[blockIdx.x];
  double sx = 0.0, sy = 0.0;
  for (int i = threadIdx.x; i < mt.n_part; i += blockDim.x) {
    sx += (double)mt.part[2 * i];
    sy += (double)mt.part[2 * i + 1];
  }
  sx = block_sum_d(sx, red);
  sy = block_sum_d(sy, red);
  if (threadIdx.x == 0) {
    const bool ok = mt.scal[SC_VALID] != 0.f && sy > 0.0 && isfinite(sy);
    mt.scal[SC_FINAL] = ok ? (float)((double)mt.kappa * sqrt(sx / sy)) : 0.f;
  }
}

// ---------------------------------------------------------------------------
// K3: same tiling as K1.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k3_apply(const __grid_constant__ K3Params p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  const int tile = blockIdx.x;
  const int g = find_group(p.starts, p.count, tile);
  const K3Mat& mt = p.mats[g];
  const int lt = tile - p.starts[g];
  const int rt = lt / mt.n_ct, ct = lt % mt.n_ct;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t r0 = (int64_t)rt * K1_ROWS;
  const int64_t c0 = (int64_t)ct * K1_COLS + lane * 8;
  const float f = mt.scal[SC_FINAL];
  float cs[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) cs[q] = (c0 + q < mt.cols) ? mt.C[c0 + q] * f : 0.f;
  for (int rr = warp; rr < K1_ROWS; rr += 8) {
    const int64_t r = r0 + rr;
    if (r >= mt.rows) break;
    const float rs = mt.R[r];
    const int64_t base = r * mt.cols + c0;
    if (mt.vec) {
      if (c0 < mt.cols) {
        float x8[8], w8[8], o8[8];
        ld8(mt.X5, r * mt.ldx + c0, mt.xdt, x8);
        ld8(mt.W, base, mt.wdt, w8);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          o8[q] = f != 0.f ? rs * x8[q] * cs[q] : 0.f;
          w8[q] = p.decay * w8[q] - p.lr * o8[q];
        }
        st8(mt.W, base, mt.wdt, w8);
        if (mt.upd) st8(mt.upd, base, DT_FP32, o8);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (c0 + q < mt.cols) {
          const float o = f != 0.f ? rs * ld_elem(mt.X5, r * mt.ldx + c0 + q, mt.xdt) * cs[q] : 0.f;
          st_elem(mt.W, base + q, mt.wdt, p.decay * ld_elem(mt.W, base + q, mt.wdt) - p.lr * o);
          if (mt.upd) mt.upd[base + q] = o;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Canary fill / check of the checked-workspace mode: one CTA of 64 threads per
// 256-byte canary.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(64) k_canary(const __grid_constant__ CanaryParams p) {
  uint32_t* base = reinterpret_cast<uint32_t*>(p.status);
  uint32_t* c = base + (size_t)p.blk[blockIdx.x] * 64;
  if (p.mode == 0)
    c[threadIdx.x] = (p.plant && blockIdx.x == 0 && threadIdx.x == 0) ? ~CANARY_FILL : CANARY_FILL;
  else if (c[threadIdx.x] != CANARY_FILL)
    raise_status(p.status, ST_CANARY);
}

cudaError_t launch_canary(const CanaryParams& p, cudaStream_t s) {
  if (p.count <= 0) return cudaSuccess;
  k_canary<<<p.count, 64, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_k0(const K0Params& p, cudaStream_t s) {
  if (p.count <= 0) return cudaSuccess;
  k0_conditioning<<<p.count, 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_k1(const K1Params& p, int total_tiles, cudaStream_t s) {
  if (total_tiles <= 0) return cudaSuccess;
  k1_momentum<<<total_tiles, 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_k1b(const K1bParams& p, int total_blocks, cudaStream_t s) {
  if (total_blocks <= 0) return cudaSuccess;
  k1b_reduce<<<total_blocks, K1B_THREADS, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_k3a(const K3Params& p, cudaStream_t s) {
  if (p.count <= 0) return cudaSuccess;
  k3a_factor<<<p.count, 256, 0, s>>>(p);
  return cudaGetLastError();
}
cudaError_t launch_k3(const K3Params& p, int total_tiles, cudaStream_t s) {
  if (total_tiles <= 0) return cudaSuccess;
  k3_apply<<<total_tiles, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace dm
