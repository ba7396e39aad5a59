// Whole Muon / Dimuon step for thin factors (short side r <= 32, e.g. LoRA A
// (r x n) and B (n x r)), per padded short side RP.
//
// The Newton-Schulz iterate is a left-multiple of the start matrix: each step
// X <- (aI + bA + cA^2) X with A = X X^T, so X_k = P_k X_0 with an r x r
// polynomial P_k in the Gram matrix A_0 = X_0 X_0^T ("From PCG to Muon",
// section 6 "Muon's Gram Matrix": the orthogonaliser normalises the global
// Gram matrix; sitech.ge, "Instead of SVD - Newton-Schulz" for the iteration).
// With X_0 = R B C (B = M_t, or G + mu M_t under Nesterov; R = C = I in Muon
// mode) and b_j the j-th long-side column of B:
//   A_0 = R S_1 R,  S_1 = sum_j C_j^2 b_j b_j^T
//   H   = X_0 C^2 X_0^T = R S_2 R,  S_2 = sum_j C_j^4 b_j b_j^T
//   O(:, j) = C_j^2 T b_j,  T = f R P_5 R,
// f = kappa / ||X_0||_F, times ||X_5||_F / ||R X_5 C||_F when Dimuon
// conditioning is on; both norms follow from A_0 and H.  Launches:
//   thin_setup   one CTA per factor (up to THIN_MAX per launch): descriptor
//                into the workspace, sums of the previous energies
//   thin_gram    persistent CTAs taking slabs of long-side columns from a
//                device counter: M_t = mu M_{t-1} + G (the exact value rounded
//                once, stored), the slab's S_1 / S_2 partials (fp64), short-side
//                energy partials
//   thin_iterate one CTA per factor: partials summed in slab order, R, the
//                r x r iteration, T, the new short-side energies
//   thin_apply   persistent CTAs over slabs: O = C^2 T B, W update, the new
//                long-side energies
// fp64 products use the fp64 tensor-core MMA (mma.sync m8n8k4) for RP >= 8
// (RP = 8, 16, 32); RP <= 4 (RP == r) uses fp64 FMAs, one lane per four
// long-side columns.  The streaming loops keep everything in registers, with
// the next step's loads in flight while the current step computes; each warp
// walks its own columns of the slab with no block-wide barrier.
// Dimuon conditioning, renormalisation, scale and decay follow "Dimuon: LoRA
// 에 맞춰 다시 짠 Muon" ("-1/4 power from both sides", "Why the *last*
// momentum", Problem 4) and "Muon Optimizer 정리" (eq. (1)-(3), "Scaling up").
#include <algorithm>

#include "dm_common.cuh"
#include "dm_thin.cuh"

namespace dm {
namespace {

using namespace thin;

// Next slab for this CTA from the device counter (the same for every thread).
__device__ __forceinline__ int next_unit(int* counter, int* slot) {
  __syncthreads();  // every thread is done with the previous slab's shared state
  if (threadIdx.x == 0) *slot = atomicAdd(counter, 1);
  __syncthreads();
  return *slot;
}

// Runs step() over this warp's long-side positions c0, c0 + stride, ... < c_hi,
// with the loads of the next position issued before the current one computes
// (DB) or one position at a time.
template <bool DB, typename Frag, typename Load, typename Step>
__device__ __forceinline__ void stream_positions(int64_t c0, int64_t stride, int64_t c_hi,
                                                 Load&& load, Step&& step) {
  if (c0 >= c_hi) return;
  Frag fa, fb;
  load(fa, c0);
  if constexpr (DB) {
    for (int64_t c = c0;;) {
      const int64_t c1 = c + stride;
      if (c1 < c_hi) load(fb, c1);
      step(fa, c);
      if (c1 >= c_hi) break;
      const int64_t c2 = c1 + stride;
      if (c2 < c_hi) load(fa, c2);
      step(fb, c1);
      if (c2 >= c_hi) break;
      c = c2;
    }
  } else {
    for (int64_t c = c0; c < c_hi; c += stride) {
      if (c != c0) load(fa, c);
      step(fa, c);
    }
  }
}

// ===========================================================================
// thin_setup: descriptors into the workspace, sums of the previous energies
// ===========================================================================
__global__ void __launch_bounds__(256) thin_setup(const __grid_constant__ ThinSetupParams p) {
  __shared__ double red[32];
  const int b = blockIdx.x, tid = threadIdx.x;
  const ThinMat& mt = p.mats[b];
  const int f = p.first + b;
  if (tid == 0) {
    p.mats_dst[f] = mt;
    p.starts_dst[f] = p.starts[b];
    if (b == p.count - 1) p.starts_dst[f + 1] = p.starts[b + 1];
  }
  for (int u = p.starts[b] + tid; u < p.starts[b + 1]; u += blockDim.x) p.unit_f_dst[u] = f;
  const Geo q = geometry(mt, p.conditioned);
  double sc = 0.0, sr = 0.0;
  if (q.cond) {
    for (int i = tid; i < q.r; i += blockDim.x) sr += (double)q.e_r[i];
    if ((reinterpret_cast<uintptr_t>(q.e_c) & 15u) == 0) {
      const float4* e4 = reinterpret_cast<const float4*>(q.e_c);
      const int64_t n4 = q.n >> 2;
#pragma unroll 4
      for (int64_t k = tid; k < n4; k += blockDim.x) {
        const float4 v = e4[k];
        sc += ((double)v.x + (double)v.y) + ((double)v.z + (double)v.w);
      }
      for (int64_t k = 4 * n4 + tid; k < q.n; k += blockDim.x) sc += (double)q.e_c[k];
    } else {
      for (int64_t k = tid; k < q.n; k += blockDim.x) sc += (double)q.e_c[k];
    }
  }
  sc = block_sum_d(sc, red);
  sr = block_sum_d(sr, red);
  if (tid == 0) {
    p.fsc[4 * f] = sc;
    p.fsc[4 * f + 1] = sr;
  }
}

// ===========================================================================
// thin_gram: momentum, Gram partials, short-side energy partials
// ===========================================================================
template <int RP>
struct GramFrag {
  static constexpr int ROWS = TCfg<RP>::MMA ? TCfg<RP>::NB : RP;
  float m[ROWS][4], g[ROWS][4];
  float ec[4];  // previous long-side energies of the four columns
};

template <int RP>
__global__ void __launch_bounds__(TT) thin_gram(const __grid_constant__ ThinParams p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  using Cf = TCfg<RP>;
  using Frag = GramFrag<RP>;
  __shared__ double red_s[TW][2][Cf::PART];
  __shared__ float red_e[TW][RP];
  __shared__ int s_unit;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float mu = p.mu, eps = p.eps;

  for (int u = next_unit(p.counters, &s_unit); u < p.units; u = next_unit(p.counters, &s_unit)) {
    const int f = p.unit_f[u];
    const ThinMat mt = p.mats[f];  // by value: stores cannot alias it
    const Geo q = geometry(mt, p.conditioned);
    const int r = q.r;
    const int mdt = mt.mdt, gdt = mt.gdt;
    const int64_t c_lo = (int64_t)(u - p.starts[f]) * Cf::SLAB;
    const int64_t c_hi = min(q.n, c_lo + Cf::SLAB);
    const bool on = q.cond && p.fsc[4 * f] > 0.0 && p.fsc[4 * f + 1] > 0.0;
    const float inv_mc = on ? (float)((double)q.n / p.fsc[4 * f]) : 0.f;

    if constexpr (Cf::MMA) {
      constexpr int NB = Cf::NB, NUB = Cf::NUB;
      const int g = lane >> 2, t = lane & 3;
      double s1[NUB][2], s2[NUB][2];
      float er[NB];
#pragma unroll
      for (int b = 0; b < NUB; ++b) s1[b][0] = s1[b][1] = s2[b][0] = s2[b][1] = 0.0;
#pragma unroll
      for (int b = 0; b < NB; ++b) er[b] = 0.f;
      const bool quad = !q.tall && q.vec;
      // lane (g, t) holds rows g + 8 blk at long-side columns col(e), e = 0..3:
      // wide c + 4t + e (one 4-vector per row), tall c + t + 4e
      auto col_of = [&](int64_t c, int e) -> int64_t { return q.tall ? c + t + 4 * e : c + 4 * t + e; };
      auto load = [&](Frag& fr, int64_t c) {
#pragma unroll
        for (int blk = 0; blk < NB; ++blk) {
          const int row = g + 8 * blk;
          if (quad) {
            if (row < r && c + 4 * t < c_hi) {
              ld4(mt.M, q.off(row, c + 4 * t), mdt, fr.m[blk]);
              ld4(mt.G, q.off(row, c + 4 * t), gdt, fr.g[blk]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) fr.m[blk][e] = fr.g[blk][e] = 0.f;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int64_t col = col_of(c, e);
              const bool ok = row < r && col < c_hi;
              const int64_t o = ok ? q.off(row, col) : 0;
              fr.m[blk][e] = ok ? ld_elem(mt.M, o, mdt) : 0.f;
              fr.g[blk][e] = ok ? ld_elem(mt.G, o, gdt) : 0.f;
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t col = col_of(c, e);
          fr.ec[e] = (on && col < c_hi) ? q.e_c[col] : 0.f;
        }
      };
      auto step = [&](Frag& fr, int64_t c) {
        // momentum (invalid positions hold zeros and stay zero)
        double bx[NB][4];
#pragma unroll
        for (int blk = 0; blk < NB; ++blk)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float m = momentum_value(mu, fr.m[blk][e], fr.g[blk][e], mdt);
            fr.m[blk][e] = m;
            bx[blk][e] = p.nesterov ? fma((double)mu, (double)m, (double)fr.g[blk][e]) : (double)m;
            er[blk] = fmaf(m, m, er[blk]);
          }
#pragma unroll
        for (int blk = 0; blk < NB; ++blk) {
          const int row = g + 8 * blk;
          if (quad) {
            if (row < r && c + 4 * t < c_hi) st4(mt.M, q.off(row, c + 4 * t), mdt, fr.m[blk]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int64_t col = col_of(c, e);
              if (row < r && col < c_hi) st_elem(mt.M, q.off(row, col), mdt, fr.m[blk][e]);
            }
          }
        }
        // Gram partials: the DMMA's k slot t is column col(e)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double w =
              on ? (col_of(c, e) < c_hi ? (double)col_weight(fr.ec[e], inv_mc, eps) : 0.0) : 1.0;
          double xw[NB], xw2[NB];
#pragma unroll
          for (int blk = 0; blk < NB; ++blk) {
            xw[blk] = w * bx[blk][e];
            xw2[blk] = w * xw[blk];
          }
          int ub = 0;
#pragma unroll
          for (int bi = 0; bi < NB; ++bi)
#pragma unroll
            for (int bj = bi; bj < NB; ++bj, ++ub) {
              dmma(s1[ub][0], s1[ub][1], bx[bi][e], xw[bj]);
              if (on) dmma(s2[ub][0], s2[ub][1], bx[bi][e], xw2[bj]);
            }
        }
      };
      stream_positions<Cf::DB, Frag>(c_lo + 16 * warp, 16 * TW, c_hi, load, step);
      // block ub's entry (g, 2t + h) -> slot ub * 64 + g * 8 + 2t + h
#pragma unroll
      for (int ub = 0; ub < NUB; ++ub)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          red_s[warp][0][ub * 64 + g * 8 + 2 * t + h] = s1[ub][h];
          red_s[warp][1][ub * 64 + g * 8 + 2 * t + h] = s2[ub][h];
        }
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        float e = er[blk];
        e += __shfl_xor_sync(0xffffffffu, e, 1);
        e += __shfl_xor_sync(0xffffffffu, e, 2);
        if (t == 0) red_e[warp][g + 8 * blk] = e;
      }
    } else {
      // RP == r <= 4: lane owns long-side columns c .. c + 3
      double s1[RP][RP], s2[RP][RP];
      float er[RP];
#pragma unroll
      for (int i = 0; i < RP; ++i) {
        er[i] = 0.f;
#pragma unroll
        for (int k = 0; k < RP; ++k) s1[i][k] = s2[i][k] = 0.0;
      }
      auto load = [&](Frag& fr, int64_t c) {
        const bool full = q.vec && c + 4 <= c_hi;
        if (full && q.tall) {
          float fm[4 * RP], fg[4 * RP];  // four long-side columns, r each
#pragma unroll
          for (int s = 0; s < RP; ++s) {
            ld4(mt.M, c * RP + 4 * s, mdt, &fm[4 * s]);
            ld4(mt.G, c * RP + 4 * s, gdt, &fg[4 * s]);
          }
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              fr.m[i][e] = fm[e * RP + i];
              fr.g[i][e] = fg[e * RP + i];
            }
        } else if (full) {
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            ld4(mt.M, q.off(i, c), mdt, fr.m[i]);
            ld4(mt.G, q.off(i, c), gdt, fr.g[i]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const bool ok = c + e < c_hi;
              const int64_t o = ok ? q.off(i, c + e) : 0;
              fr.m[i][e] = ok ? ld_elem(mt.M, o, mdt) : 0.f;
              fr.g[i][e] = ok ? ld_elem(mt.G, o, gdt) : 0.f;
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) fr.ec[e] = (on && c + e < c_hi) ? q.e_c[c + e] : 0.f;
      };
      auto step = [&](Frag& fr, int64_t c) {
        const bool full = q.vec && c + 4 <= c_hi;
        double bx[RP][4];
#pragma unroll
        for (int i = 0; i < RP; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float m = momentum_value(mu, fr.m[i][e], fr.g[i][e], mdt);
            fr.m[i][e] = m;
            bx[i][e] = p.nesterov ? fma((double)mu, (double)m, (double)fr.g[i][e]) : (double)m;
            er[i] = fmaf(m, m, er[i]);
          }
        if (full && q.tall) {
          float fm[4 * RP];
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) fm[e * RP + i] = fr.m[i][e];
#pragma unroll
          for (int s = 0; s < RP; ++s) st4(mt.M, c * RP + 4 * s, mdt, &fm[4 * s]);
        } else if (full) {
#pragma unroll
          for (int i = 0; i < RP; ++i) st4(mt.M, q.off(i, c), mdt, fr.m[i]);
        } else {
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (c + e < c_hi) st_elem(mt.M, q.off(i, c + e), mdt, fr.m[i][e]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double w = on ? (c + e < c_hi ? (double)col_weight(fr.ec[e], inv_mc, eps) : 0.0) : 1.0;
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int k = i; k < RP; ++k) {
              const double xk = w * bx[k][e];
              s1[i][k] = fma(bx[i][e], xk, s1[i][k]);
              if (on) s2[i][k] = fma(bx[i][e], w * xk, s2[i][k]);
            }
        }
      };
      stream_positions<Cf::DB, Frag>(c_lo + 4 * (lane + 32 * warp), 4 * TT, c_hi, load, step);
#pragma unroll
      for (int i = 0; i < RP; ++i) {
#pragma unroll
        for (int k = i; k < RP; ++k) {
          const double a = warp_sum_d(s1[i][k]), b = warp_sum_d(s2[i][k]);
          if (lane == 0) {
            red_s[warp][0][i * RP + k] = red_s[warp][0][k * RP + i] = a;
            red_s[warp][1][i * RP + k] = red_s[warp][1][k * RP + i] = b;
          }
        }
        const float e = warp_sum(er[i]);
        if (lane == 0) red_e[warp][i] = e;
      }
    }
    __syncthreads();
    double* dst = p.part + (size_t)u * 2 * Cf::PART;
    for (int i = tid; i < 2 * Cf::PART; i += TT) {
      double s = 0.0;
#pragma unroll
      for (int w = 0; w < TW; ++w) s += (&red_s[w][0][0])[i];
      dst[i] = s;
    }
    if (q.cond)
      for (int i = tid; i < RP; i += TT) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < TW; ++w) s += red_e[w][i];
        p.rpart[(size_t)u * RP + i] = s;
      }
  }
}

// ===========================================================================
// thin_iterate: one CTA per factor
// ===========================================================================
// Sums over one factor's nu slab partials, in slab order (the same additions
// as a plain loop), with the loads of up to 8 slabs issued before their
// additions so that their L2 latencies overlap instead of adding up.
// sum_slabs: entries base[v * stride + src] and base[v * stride + off + src].
__device__ __forceinline__ void sum_slabs(const double* base, size_t stride, int off, int nu, int src,
                                          double& g1, double& g2) {
  g1 = 0.0;
  g2 = 0.0;
  for (int v0 = 0; v0 < nu; v0 += 8) {
    double a[8], b[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool in = v0 + k < nu;
      const double* pp = base + (size_t)(v0 + k) * stride;
      a[k] = in ? pp[src] : 0.0;
      b[k] = in ? pp[off + src] : 0.0;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      g1 += a[k];
      g2 += b[k];
    }
  }
}

// sum_slabs for the float entries base[v * stride].
__device__ __forceinline__ float sum_slabs_f(const float* base, size_t stride, int nu) {
  float e = 0.f;
  for (int v0 = 0; v0 < nu; v0 += 8) {
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = v0 + k < nu ? base[(size_t)(v0 + k) * stride] : 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) e += a[k];
  }
  return e;
}

// Shared matrices of the one-CTA-per-factor iteration, in fp64, or in fp32
// (products on tf32 tensor cores with split operands) when the Gram sums
// came from the split bf16 tensor-core path (their ~2^-16 relative error is
// far above fp32's, so fp64 buys nothing there).
template <int RP, typename T>
struct IterLd {
  static constexpr int V = TCfg<RP>::SLD;
};
template <int RP>
struct IterLd<RP, float> {
  static constexpr int V = RP + 4;  // A-fragment reads on distinct banks; even for float2
};
template <int RP, typename T = double>
struct IterSmem {
  static constexpr int LD = IterLd<RP, T>::V;
  T G[RP][LD], H[RP][LD], P[RP][LD], A[RP][LD], Q[RP][LD], S[RP][LD];
  double R[RP];
  double red[32];
};

// Threads of the one-CTA-per-factor iteration (RP = 16, 32).
constexpr int IT = 256;
constexpr int IW = IT / 32;

// x = hi + lo with hi, lo tf32 values (round to nearest, ties away: the PTX
// conversion); hi + lo carries x to about 2^-22 relative.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(hi) : "f"(x));
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(lo) : "f"(x - __uint_as_float(hi)));
}

// D (16x8, fp32) += A (16x8, tf32) * B (8x8, tf32).  Lane l = 4g + t holds
// A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]; B[t][g], B[t+4][g]; D rows g
// and g + 8 at columns 2t, 2t + 1.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// C = A * B for RP x RP fp32 matrices in shared memory on tensor cores: one
// 16 x 8 output tile per warp, each operand split into tf32 hi + lo and each
// product taken as hi hi + hi lo + lo hi (fp32-level accuracy).
template <int RP>
__device__ __forceinline__ void mm(float (*C)[RP + 4], float (*A)[RP + 4], float (*B)[RP + 4]) {
  constexpr int MT = RP / 16, NT = RP / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  for (int tile = warp; tile < MT * NT; tile += IW) {
    const int i0 = 16 * (tile / NT), j0 = 8 * (tile % NT);
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k0 = 0; k0 < RP; k0 += 8) {
      uint32_t ah[4], al[4], bh0, bl0, bh1, bl1;
      split_tf32(A[i0 + g][k0 + t], ah[0], al[0]);
      split_tf32(A[i0 + g + 8][k0 + t], ah[1], al[1]);
      split_tf32(A[i0 + g][k0 + t + 4], ah[2], al[2]);
      split_tf32(A[i0 + g + 8][k0 + t + 4], ah[3], al[3]);
      split_tf32(B[k0 + t][j0 + g], bh0, bl0);
      split_tf32(B[k0 + t + 4][j0 + g], bh1, bl1);
      mma_tf32(d, al, bh0, bh1);
      mma_tf32(d, ah, bl0, bl1);
      mma_tf32(d, ah, bh0, bh1);
    }
    *reinterpret_cast<float2*>(&C[i0 + g][j0 + 2 * t]) = make_float2(d[0], d[1]);
    *reinterpret_cast<float2*>(&C[i0 + g + 8][j0 + 2 * t]) = make_float2(d[2], d[3]);
  }
  __syncthreads();
}

// C = A * B for RP x RP fp64 matrices in shared memory (padded rows); each
// warp interleaves the k chains of its 8x8 output blocks.
template <int RP>
__device__ __forceinline__ void mm(double (*C)[TCfg<RP>::SLD], double (*A)[TCfg<RP>::SLD],
                                   double (*B)[TCfg<RP>::SLD]) {
  if constexpr (TCfg<RP>::MMA) {
    constexpr int NB = TCfg<RP>::NB, NBLK = NB * NB, PER = (NBLK + IW - 1) / IW;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    double d[PER][2];
#pragma unroll
    for (int q = 0; q < PER; ++q) d[q][0] = d[q][1] = 0.0;
#pragma unroll
    for (int kb = 0; kb < RP / 4; ++kb)
#pragma unroll
      for (int q = 0; q < PER; ++q) {
        const int blk = warp + q * IW;
        if (blk < NBLK) {
          const int rb = blk / NB, cb = blk % NB;
          dmma(d[q][0], d[q][1], A[rb * 8 + g][kb * 4 + t], B[kb * 4 + t][cb * 8 + g]);
        }
      }
#pragma unroll
    for (int q = 0; q < PER; ++q) {
      const int blk = warp + q * IW;
      if (blk < NBLK) {
        const int rb = blk / NB, cb = blk % NB;
        C[rb * 8 + g][cb * 8 + 2 * t] = d[q][0];
        C[rb * 8 + g][cb * 8 + 2 * t + 1] = d[q][1];
      }
    }
  } else {
    for (int idx = threadIdx.x; idx < RP * RP; idx += IT) {
      const int i = idx / RP, j = idx % RP;
      double s = 0.0;
#pragma unroll
      for (int k = 0; k < RP; ++k) s = fma(A[i][k], B[k][j], s);
      C[i][j] = s;
    }
  }
  __syncthreads();
}

// The r x r iteration of factor f by one warp (iterate_gram_warp in
// dm_thin.cuh) with this launch's parameters.
template <int RP>
__device__ double iterate_factor_warp(const ThinParams& p, int f, const ThinMat& mt, const Geo& q,
                                      WarpIterSmem<RP>& s, bool* on_out) {
  IterIn in;
  in.sc = p.fsc[4 * f];
  in.sr = p.fsc[4 * f + 1];
  in.cond = q.cond;
  in.r = q.r;
  in.e_r = q.e_r;
  in.eps = p.eps;
  in.coef = p.coef;
  in.ns_steps = p.ns_steps;
  in.kappa = mt.kappa;
  in.status = p.status;
  return iterate_gram_warp<RP>(in, s, on_out);
}

template <int RP>
__global__ void __launch_bounds__(TT) thin_iterate_warp(const __grid_constant__ ThinParams p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  using Cf = TCfg<RP>;
  __shared__ WarpIterSmem<RP> sm[TW];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int f = blockIdx.x * TW + warp;
  if (f >= p.count) return;  // the whole warp leaves; no block-wide barrier follows
  WarpIterSmem<RP>& s = sm[warp];
  const ThinMat mt = p.mats[f];
  const Geo q = geometry(mt, p.conditioned);
  const int r = q.r;
  const int u0 = p.starts[f], nu = p.starts[f + 1] - p.starts[f];

  for (int idx = lane; idx < RP * RP; idx += 32) {
    const int i = idx / RP, j = idx % RP;
    int src;
    if constexpr (Cf::MMA) {
      src = (i & 7) * 8 + (j & 7);  // one 8x8 block
    } else {
      src = idx;
    }
    double g1, g2;
    sum_slabs(p.part + (size_t)u0 * 2 * Cf::PART, 2 * Cf::PART, Cf::PART, nu, src, g1, g2);
    s.G[i][j] = g1;
    s.H[i][j] = g2;
  }
  __syncwarp();
  bool on;
  const double factor = iterate_factor_warp<RP>(p, f, mt, q, s, &on);
  // new short-side energies (R has been taken from the previous ones)
  if (q.cond && lane < r) q.e_r[lane] = sum_slabs_f(p.rpart + (size_t)u0 * RP + lane, RP, nu);
  double* T = p.T + (size_t)f * RP * RP;
  for (int idx = lane; idx < RP * RP; idx += 32) {
    int i, j;
    if constexpr (Cf::MMA) {  // fragment order, KB = 2, one row block
      const int l = idx & 31, kb = idx >> 5;
      i = l >> 2;
      j = 4 * kb + (l & 3);
    } else {
      i = idx / RP;
      j = idx % RP;
    }
    T[idx] = factor * s.R[i] * s.P[i][j] * s.R[j];
  }
  if (lane == 0) {
    p.fsc[4 * f + 2] = on ? 1.0 : 0.0;
    p.fsc[4 * f + 3] = factor == 0.0 ? 1.0 : 0.0;
  }
}

template <int RP, typename T>
__global__ void __launch_bounds__(IT) thin_iterate(const __grid_constant__ ThinParams p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  using Cf = TCfg<RP>;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  IterSmem<RP, T>& s = *reinterpret_cast<IterSmem<RP, T>*>(smem_raw);
  const int tid = threadIdx.x;
  const int f = blockIdx.x;
  const ThinMat mt = p.mats[f];  // by value: stores cannot alias it
  const Geo q = geometry(mt, p.conditioned);
  const int r = q.r;
  const int u0 = p.starts[f], nu = p.starts[f + 1] - p.starts[f];

  // S_1, S_2: slab partials in slab order; lower 8x8 blocks mirror upper ones
  for (int idx = tid; idx < RP * RP; idx += IT) {
    const int i = idx / RP, j = idx % RP;
    int src;
    if constexpr (Cf::MMA) {
      constexpr int NB = Cf::NB;
      const int bi = i >> 3, bj = j >> 3;
      const int lo = bi <= bj ? bi : bj, hi = bi <= bj ? bj : bi;
      const int ub = lo * NB - lo * (lo - 1) / 2 + (hi - lo);
      src = ub * 64 + (bi <= bj ? (i & 7) * 8 + (j & 7) : (j & 7) * 8 + (i & 7));
    } else {
      src = idx;
    }
    double g1, g2;
    sum_slabs(p.part + (size_t)u0 * 2 * Cf::PART, 2 * Cf::PART, Cf::PART, nu, src, g1, g2);
    s.G[i][j] = g1;
    s.H[i][j] = g2;
  }
  // R from the previous short-side energies (read before they are replaced)
  const double sc = p.fsc[4 * f], sr = p.fsc[4 * f + 1];
  const bool on = q.cond && sr > 0.0 && sc > 0.0;
  if (tid < RP) {
    double rv = tid < r ? 1.0 : 0.0;
    if (on && tid < r) rv = 1.0 / sqrt(sqrt((double)q.e_r[tid] * ((double)r / sr) + (double)p.eps));
    s.R[tid] = rv;
  }
  __syncthreads();
  if (q.cond && tid < r) {
    q.e_r[tid] = sum_slabs_f(p.rpart + (size_t)u0 * RP + tid, RP, nu);
  }
  // A_0 = R S_1 R, H = R S_2 R; ||X_0||^2 = tr A_0
  double tr = 0.0;
  for (int idx = tid; idx < RP * RP; idx += IT) {
    const int i = idx / RP, j = idx % RP;
    const double rr = s.R[i] * s.R[j];
    s.G[i][j] *= rr;
    s.H[i][j] *= rr;
    if (i == j) tr += s.G[i][j];
  }
  const double s2 = block_sum_d(tr, s.red);
  const bool finite = isfinite(s2);
  const bool valid = finite && s2 >= NORM2_FLOOR;  // else the update is zero
  const double inv_s2 = valid ? 1.0 / s2 : 0.0;
  for (int idx = tid; idx < RP * RP; idx += IT) {
    const int i = idx / RP, j = idx % RP;
    s.A[i][j] = valid ? s.G[i][j] * inv_s2 : 0.0;
    s.P[i][j] = i == j ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int it = 0; it < p.ns_steps; ++it) {
    const T a = p.coef[it][0], b = p.coef[it][1], c = p.coef[it][2];
    mm<RP>(s.Q, s.A, s.A);  // Q = A A
    for (int idx = tid; idx < RP * RP; idx += IT) {
      const int i = idx / RP, j = idx % RP;
      s.Q[i][j] = c * s.Q[i][j] + b * s.A[i][j] + (i == j ? a : T(0));
    }
    __syncthreads();
    mm<RP>(s.S, s.Q, s.P);  // P <- Q P
    for (int idx = tid; idx < RP * RP; idx += IT) s.P[idx / RP][idx % RP] = s.S[idx / RP][idx % RP];
    __syncthreads();
    mm<RP>(s.S, s.Q, s.A);  // A <- Q A Q
    mm<RP>(s.A, s.S, s.Q);
  }
  // ||X_5||^2 s^2 = tr(P A_0 P^T); ||R X_5 C||^2 s^2 = sum_i R_i^2 (P H P^T)_ii
  mm<RP>(s.S, s.P, s.G);
  double nx = 0.0;
  for (int idx = tid; idx < RP * RP; idx += IT)
    nx += (double)s.S[idx / RP][idx % RP] * (double)s.P[idx / RP][idx % RP];
  nx = block_sum_d(nx, s.red);
  mm<RP>(s.Q, s.P, s.H);
  double ny = 0.0;
  for (int idx = tid; idx < RP * RP; idx += IT) {
    const int i = idx / RP;
    ny += s.R[i] * s.R[i] * (double)s.Q[i][idx % RP] * (double)s.P[i][idx % RP];
  }
  ny = block_sum_d(ny, s.red);
  double factor = 0.0;
  if (valid) {
    factor = (double)mt.kappa / sqrt(s2);
    if (on) factor = ny > 0.0 ? factor * sqrt(nx / ny) : 0.0;
  }
  if (!finite && tid == 0) raise_status(p.status, ST_NONFINITE);
  // T = f R P R; for RP >= 8 in MMA fragment order: T(8 bo + l/4, 4 kb + l%4)
  // at ((bo * KB + kb) * 32 + l)
  double* Tm = p.T + (size_t)f * RP * RP;
  for (int idx = tid; idx < RP * RP; idx += IT) {
    int i, j;
    if constexpr (Cf::MMA) {
      const int l = idx & 31, fr = idx >> 5;
      const int bo = fr / Cf::KB, kb = fr % Cf::KB;
      i = 8 * bo + (l >> 2);
      j = 4 * kb + (l & 3);
    } else {
      i = idx / RP;
      j = idx % RP;
    }
    Tm[idx] = factor * s.R[i] * (double)s.P[i][j] * s.R[j];
  }
  if (tid == 0) {
    p.fsc[4 * f + 2] = on ? 1.0 : 0.0;
    p.fsc[4 * f + 3] = factor == 0.0 ? 1.0 : 0.0;
  }
}

// ===========================================================================
// thin_apply: O = C^2 T B, W update, long-side energies
// ===========================================================================
template <int RP>
struct ApplyFrag {
  static constexpr bool MMA = TCfg<RP>::MMA;
  static constexpr int MR = MMA ? TCfg<RP>::KB : RP;  // B values per column slot
  static constexpr int WR = MMA ? TCfg<RP>::NB : RP;
  float m[MR][4], g[MR][4];
  float w[WR][MMA ? 2 : 1][4];  // current weights at the lane's output positions
  float ec[4];                  // previous long-side energies of the four column slots
};

template <int RP>
__global__ void __launch_bounds__(TT) thin_apply(const __grid_constant__ ThinParams p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  using Cf = TCfg<RP>;
  using Frag = ApplyFrag<RP>;
  __shared__ double Ts[RP * RP];
  __shared__ int s_unit;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float mu = p.mu, lr = p.lr, decay = p.decay, eps = p.eps;
  int f_loaded = -1;

  for (int u = next_unit(p.counters + 1, &s_unit); u < p.units;
       u = next_unit(p.counters + 1, &s_unit)) {
    const int f = p.unit_f[u];
    if (f != f_loaded) {  // uniform: every thread saw the same u
      const double* Tg = p.T + (size_t)f * RP * RP;
      for (int i = tid; i < RP * RP; i += TT) Ts[i] = Tg[i];
      f_loaded = f;
      __syncthreads();
    }
    const ThinMat mt = p.mats[f];  // by value: stores cannot alias it
    const Geo q = geometry(mt, p.conditioned);
    const int r = q.r;
    const int64_t c_lo = (int64_t)(u - p.starts[f]) * Cf::SLAB;
    const int64_t c_hi = min(q.n, c_lo + Cf::SLAB);
    const bool on = p.fsc[4 * f + 2] != 0.0;
    const bool zero = p.fsc[4 * f + 3] != 0.0;
    const float inv_mc = on ? (float)((double)q.n / p.fsc[4 * f]) : 0.f;
    const int mdt = mt.mdt, gdt = mt.gdt, wdt = mt.wdt;
    const bool nest = p.nesterov != 0;

    if constexpr (Cf::MMA) {
      constexpr int NB = Cf::NB, KB = Cf::KB;
      const int g = lane >> 2, t = lane & 3;
      const bool quad = !q.tall && q.vec;
      const bool pair = q.tall && mt.vec && (r & 1) == 0;  // two short-side neighbours aligned
      // lane (g, t) holds B rows 4 kb + t at long-side column slots col(e):
      // wide c + 4g + e (4-vectors), tall c + 8e + g.  Wide computes
      // D = T B (output rows 8 bo + g, columns c + 8t .. c + 8t + 7); tall
      // computes D = B^T T^T (output rows 8 bo + 2t, +1 at column c + 8e + g).
      auto col_of = [&](int64_t c, int e) -> int64_t { return q.tall ? c + 8 * e + g : c + 4 * g + e; };
      auto load = [&](Frag& fr, int64_t c) {
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
          const int row = 4 * kb + t;
          if (quad) {
            if (row < r && c + 4 * g < c_hi) {
              ld4(mt.M, q.off(row, c + 4 * g), mdt, fr.m[kb]);
              if (nest) {
                ld4(mt.G, q.off(row, c + 4 * g), gdt, fr.g[kb]);
              } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) fr.g[kb][e] = 0.f;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) fr.m[kb][e] = fr.g[kb][e] = 0.f;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int64_t col = col_of(c, e);
              const bool ok = row < r && col < c_hi;
              const int64_t o = ok ? q.off(row, col) : 0;
              fr.m[kb][e] = ok ? ld_elem(mt.M, o, mdt) : 0.f;
              fr.g[kb][e] = (ok && nest) ? ld_elem(mt.G, o, gdt) : 0.f;
            }
          }
        }
#pragma unroll
        for (int bo = 0; bo < NB; ++bo) {
          if (!q.tall) {
            const int row = 8 * bo + g;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int64_t col0 = c + 8 * t + 4 * h;
              if (quad) {
                if (row < r && col0 < c_hi) {
                  ld4(mt.W, q.off(row, col0), wdt, fr.w[bo][h]);
                } else {
#pragma unroll
                  for (int e = 0; e < 4; ++e) fr.w[bo][h][e] = 0.f;
                }
              } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  fr.w[bo][h][e] =
                      (row < r && col0 + e < c_hi) ? ld_elem(mt.W, q.off(row, col0 + e), wdt) : 0.f;
              }
            }
          } else {
            const int row0 = 8 * bo + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int64_t col = c + 8 * e + g;
              if (pair && row0 + 1 < r && col < c_hi) {
                ld2(mt.W, q.off(row0, col), wdt, fr.w[bo][0][e], fr.w[bo][1][e]);
              } else {
#pragma unroll
                for (int h = 0; h < 2; ++h)
                  fr.w[bo][h][e] =
                      (row0 + h < r && col < c_hi) ? ld_elem(mt.W, q.off(row0 + h, col), wdt) : 0.f;
              }
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t col = col_of(c, e);
          fr.ec[e] = (on && col < c_hi) ? q.e_c[col] : 0.f;
        }
      };
      auto step = [&](Frag& fr, int64_t c) {
        float ce[4];
        double x[KB][4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double w =
              on ? (col_of(c, e) < c_hi ? (double)col_weight(fr.ec[e], inv_mc, eps) : 0.0) : 1.0;
          float sq = 0.f;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const double m = (double)fr.m[kb][e];
            x[kb][e] = w * (nest ? fma((double)mu, m, (double)fr.g[kb][e]) : m);
            sq = fmaf(fr.m[kb][e], fr.m[kb][e], sq);
          }
          sq += __shfl_xor_sync(0xffffffffu, sq, 1);
          sq += __shfl_xor_sync(0xffffffffu, sq, 2);
          ce[e] = sq;
        }
        double acc[NB][4][2];
#pragma unroll
        for (int bo = 0; bo < NB; ++bo)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[bo][e][0] = acc[bo][e][1] = 0.0;
#pragma unroll
        for (int kb = 0; kb < KB; ++kb) {
          double tf[NB];
#pragma unroll
          for (int bo = 0; bo < NB; ++bo) tf[bo] = Ts[(bo * KB + kb) * 32 + lane];
#pragma unroll
          for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int bo = 0; bo < NB; ++bo) {
              if (q.tall)
                dmma(acc[bo][e][0], acc[bo][e][1], x[kb][e], tf[bo]);
              else
                dmma(acc[bo][e][0], acc[bo][e][1], tf[bo], x[kb][e]);
            }
        }
        // W update (and O) at this lane's output positions
#pragma unroll
        for (int bo = 0; bo < NB; ++bo) {
          if (!q.tall) {
            // acc[bo][e][h] is column c + 8t + 4h + e of row 8 bo + g
            const int row = 8 * bo + g;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float o4[4], n4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                o4[e] = zero ? 0.f : (float)acc[bo][e][h];
                n4[e] = decay * fr.w[bo][h][e] - lr * o4[e];
              }
              const int64_t col0 = c + 8 * t + 4 * h;
              if (quad) {
                if (row < r && col0 < c_hi) {
                  st4(mt.W, q.off(row, col0), wdt, n4);
                  if (mt.upd) st4(mt.upd, q.off(row, col0), DT_FP32, o4);
                }
              } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  if (row < r && col0 + e < c_hi) {
                    st_elem(mt.W, q.off(row, col0 + e), wdt, n4[e]);
                    if (mt.upd) mt.upd[q.off(row, col0 + e)] = o4[e];
                  }
              }
            }
          } else {
            // acc[bo][e][h] is row 8 bo + 2t + h of column c + 8e + g
            const int row0 = 8 * bo + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int64_t col = c + 8 * e + g;
              float o2[2], n2[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                o2[h] = zero ? 0.f : (float)acc[bo][e][h];
                n2[h] = decay * fr.w[bo][h][e] - lr * o2[h];
              }
              if (pair && row0 + 1 < r && col < c_hi) {
                st2(mt.W, q.off(row0, col), wdt, n2[0], n2[1]);
                if (mt.upd) st2(mt.upd, q.off(row0, col), DT_FP32, o2[0], o2[1]);
              } else {
#pragma unroll
                for (int h = 0; h < 2; ++h)
                  if (row0 + h < r && col < c_hi) {
                    st_elem(mt.W, q.off(row0 + h, col), wdt, n2[h]);
                    if (mt.upd) mt.upd[q.off(row0 + h, col)] = o2[h];
                  }
              }
            }
          }
        }
        if (q.cond) {
          __syncwarp();  // every lane's read of these columns' previous energies is done
          if (t == 0)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int64_t col = col_of(c, e);
              if (col < c_hi) q.e_c[col] = ce[e];
            }
        }
      };
      stream_positions<Cf::DB, Frag>(c_lo + 32 * warp, 32 * TW, c_hi, load, step);
    } else {
      // RP == r <= 4: lane owns long-side columns c .. c + 3
      auto load = [&](Frag& fr, int64_t c) {
        const bool full = q.vec && c + 4 <= c_hi;
        if (full && q.tall) {
          float fm[4 * RP], fg[4 * RP], fw[4 * RP];
#pragma unroll
          for (int s = 0; s < RP; ++s) {
            ld4(mt.M, c * RP + 4 * s, mdt, &fm[4 * s]);
            if (nest) ld4(mt.G, c * RP + 4 * s, gdt, &fg[4 * s]);
            ld4(mt.W, c * RP + 4 * s, wdt, &fw[4 * s]);
          }
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              fr.m[i][e] = fm[e * RP + i];
              fr.g[i][e] = nest ? fg[e * RP + i] : 0.f;
              fr.w[i][0][e] = fw[e * RP + i];
            }
        } else if (full) {
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            ld4(mt.M, q.off(i, c), mdt, fr.m[i]);
            if (nest) {
              ld4(mt.G, q.off(i, c), gdt, fr.g[i]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) fr.g[i][e] = 0.f;
            }
            ld4(mt.W, q.off(i, c), wdt, fr.w[i][0]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const bool ok = c + e < c_hi;
              const int64_t o = ok ? q.off(i, c + e) : 0;
              fr.m[i][e] = ok ? ld_elem(mt.M, o, mdt) : 0.f;
              fr.g[i][e] = (ok && nest) ? ld_elem(mt.G, o, gdt) : 0.f;
              fr.w[i][0][e] = ok ? ld_elem(mt.W, o, wdt) : 0.f;
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) fr.ec[e] = (on && c + e < c_hi) ? q.e_c[c + e] : 0.f;
      };
      auto step = [&](Frag& fr, int64_t c) {
        const bool full = q.vec && c + 4 <= c_hi;
        float ov[RP][4], wv[RP][4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double w = on ? (c + e < c_hi ? (double)col_weight(fr.ec[e], inv_mc, eps) : 0.0) : 1.0;
          double x[RP];
          float sq = 0.f;
#pragma unroll
          for (int k = 0; k < RP; ++k) {
            const double m = (double)fr.m[k][e];
            x[k] = w * (nest ? fma((double)mu, m, (double)fr.g[k][e]) : m);
            sq = fmaf(fr.m[k][e], fr.m[k][e], sq);
          }
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            double y = 0.0;
#pragma unroll
            for (int k = 0; k < RP; ++k) y = fma(Ts[i * RP + k], x[k], y);
            ov[i][e] = zero ? 0.f : (float)y;
            wv[i][e] = decay * fr.w[i][0][e] - lr * ov[i][e];
          }
          if (q.cond && c + e < c_hi) q.e_c[c + e] = sq;  // this lane read it in load()
        }
        if (full && q.tall) {
          float fw[4 * RP], fo[4 * RP];
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              fw[e * RP + i] = wv[i][e];
              fo[e * RP + i] = ov[i][e];
            }
#pragma unroll
          for (int s = 0; s < RP; ++s) {
            st4(mt.W, c * RP + 4 * s, wdt, &fw[4 * s]);
            if (mt.upd) st4(mt.upd, c * RP + 4 * s, DT_FP32, &fo[4 * s]);
          }
        } else if (full) {
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            st4(mt.W, q.off(i, c), wdt, wv[i]);
            if (mt.upd) st4(mt.upd, q.off(i, c), DT_FP32, ov[i]);
          }
        } else {
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (c + e < c_hi) {
                st_elem(mt.W, q.off(i, c + e), wdt, wv[i][e]);
                if (mt.upd) mt.upd[q.off(i, c + e)] = ov[i][e];
              }
        }
      };
      stream_positions<Cf::DB, Frag>(c_lo + 4 * (lane + 32 * warp), 4 * TT, c_hi, load, step);
    }
  }
}

// ===========================================================================
// thin_fused: the whole step of one factor in one CTA, for r = RP = 2 when
// the factor's momentum (and, under Nesterov, its gradient) fits in shared
// memory.  Pass 1 streams G and M_{t-1} once: M_t (stored, and kept in
// shared memory), the Gram sums S_1, S_2 and the short-side energies; the
// block-reduced sums go through the r x r iteration on one warp; pass 2
// applies O = T (C^2 B) to the kept momentum and streams W once, writing the
// new long-side energies.  Per element the arithmetic is that of thin_gram /
// thin_apply (exactly rounded momentum, fp64 Gram sums and products);
// the HBM traffic is the algorithmic one (G 2, M 4 + 4, W 2 + 2 bytes per
// element with fp32 momentum), without the two-pass path's second read of
// M_t, and one launch replaces three.
// ===========================================================================
constexpr int FT = 128;  // threads of thin_fused (four CTAs per SM: 448 factors in one wave)
constexpr int FW = FT / 32;

// Four long-side columns c .. c + 3 of all RP rows, as v[row][column].
template <int RP>
__device__ __forceinline__ void load_cols(const void* base, int dt, const Geo& q, int64_t c,
                                          float v[RP][4]) {
  if (!q.tall) {
#pragma unroll
    for (int i = 0; i < RP; ++i) ld4(base, (int64_t)i * q.n + c, dt, v[i]);
  } else {
    float t[4 * RP];
#pragma unroll
    for (int k = 0; k < RP; ++k) ld4(base, c * RP + 4 * k, dt, &t[4 * k]);
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) v[i][e] = t[e * RP + i];
  }
}

template <int RP>
__device__ __forceinline__ void store_cols(void* base, int dt, const Geo& q, int64_t c,
                                           const float v[RP][4]) {
  if (!q.tall) {
#pragma unroll
    for (int i = 0; i < RP; ++i) st4(base, (int64_t)i * q.n + c, dt, v[i]);
  } else {
    float t[4 * RP];
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) t[e * RP + i] = v[i][e];
#pragma unroll
    for (int k = 0; k < RP; ++k) st4(base, c * RP + 4 * k, dt, &t[4 * k]);
  }
}

template <int RP>
__global__ void __launch_bounds__(FT, 4) thin_fused(const __grid_constant__ ThinParams p) {
  if (step_aborted(p.status)) return;  // an earlier launch of this step timed out
  extern __shared__ __align__(16) uint8_t fused_raw[];
  __shared__ WarpIterSmem<RP> it;
  __shared__ double red[FW][2][RP][RP];
  __shared__ float rede[FW][RP];
  __shared__ double Tsm[RP][RP];
  __shared__ int zsh;
  const int f = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const ThinMat mt = p.mats[f];
  const Geo q = geometry(mt, p.conditioned);
  const int64_t n = q.n;
  const bool nest = p.nesterov != 0;
  float* Ms = reinterpret_cast<float*>(fused_raw);  // M_t, [n][RP]
  float* Gs = Ms + (size_t)n * RP;                  // G under Nesterov, [n][RP]
  const double sc = p.fsc[4 * f], sr = p.fsc[4 * f + 1];
  const bool on = q.cond && sc > 0.0 && sr > 0.0;
  const float inv_mc = on ? (float)((double)n / sc) : 0.f;
  const float mu = p.mu, eps = p.eps;

  // ---- pass 1: momentum, Gram sums, short-side energies -------------------
  double s1[RP][RP], s2[RP][RP];
  float er[RP];
#pragma unroll
  for (int i = 0; i < RP; ++i) {
    er[i] = 0.f;
#pragma unroll
    for (int k = 0; k < RP; ++k) s1[i][k] = s2[i][k] = 0.0;
  }
  // each thread's next group of four columns is loaded before the current
  // one is processed (two groups of loads in flight per thread)
  float mv[RP][4], gv[RP][4];
  if (4 * (int64_t)tid < n) {
    load_cols<RP>(mt.M, mt.mdt, q, 4 * (int64_t)tid, mv);
    load_cols<RP>(mt.G, mt.gdt, q, 4 * (int64_t)tid, gv);
  }
  for (int64_t c = 4 * (int64_t)tid; c < n; c += 4 * FT) {
    float mn[RP][4], gn[RP][4];
    const bool more = c + 4 * FT < n;
    if (more) {
      load_cols<RP>(mt.M, mt.mdt, q, c + 4 * FT, mn);
      load_cols<RP>(mt.G, mt.gdt, q, c + 4 * FT, gn);
    }
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float m = momentum_value(mu, mv[i][e], gv[i][e], mt.mdt);
        mv[i][e] = m;
        er[i] = fmaf(m, m, er[i]);
      }
    store_cols<RP>(mt.M, mt.mdt, q, c, mv);
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int i = 0; i < RP; ++i) {
        Ms[(c + e) * RP + i] = mv[i][e];
        if (nest) Gs[(c + e) * RP + i] = gv[i][e];
      }
    double wd[4] = {1.0, 1.0, 1.0, 1.0};
    if (on) {
      const float4 e4 = *reinterpret_cast<const float4*>(q.e_c + c);
      wd[0] = (double)col_weight(e4.x, inv_mc, eps);
      wd[1] = (double)col_weight(e4.y, inv_mc, eps);
      wd[2] = (double)col_weight(e4.z, inv_mc, eps);
      wd[3] = (double)col_weight(e4.w, inv_mc, eps);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      double bx[RP];
#pragma unroll
      for (int k = 0; k < RP; ++k)
        bx[k] = nest ? fma((double)mu, (double)mv[k][e], (double)gv[k][e]) : (double)mv[k][e];
#pragma unroll
      for (int i = 0; i < RP; ++i)
#pragma unroll
        for (int k = i; k < RP; ++k) {
          const double xk = on ? wd[e] * bx[k] : bx[k];
          s1[i][k] = fma(bx[i], xk, s1[i][k]);
          if (on) s2[i][k] = fma(bx[i], wd[e] * xk, s2[i][k]);
        }
    }
    if (more) {
#pragma unroll
      for (int i = 0; i < RP; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          mv[i][e] = mn[i][e];
          gv[i][e] = gn[i][e];
        }
    }
  }

  // ---- block reduction (warps in order), then the r x r iteration ----------
#pragma unroll
  for (int i = 0; i < RP; ++i) {
#pragma unroll
    for (int k = i; k < RP; ++k) {
      const double a = warp_sum_d(s1[i][k]), b = warp_sum_d(s2[i][k]);
      if (lane == 0) {
        red[warp][0][i][k] = a;
        red[warp][1][i][k] = b;
      }
    }
    const float e = warp_sum(er[i]);
    if (lane == 0) rede[warp][i] = e;
  }
  __syncthreads();
  if (warp == 0) {
    for (int idx = lane; idx < RP * RP; idx += 32) {
      const int i = idx / RP, j = idx % RP;
      const int lo = i <= j ? i : j, hi = i <= j ? j : i;
      double g1 = 0.0, g2 = 0.0;
#pragma unroll
      for (int w = 0; w < FW; ++w) {
        g1 += red[w][0][lo][hi];
        g2 += red[w][1][lo][hi];
      }
      it.G[i][j] = g1;
      it.H[i][j] = g2;
    }
    __syncwarp();
    bool on_it;
    const double factor = iterate_factor_warp<RP>(p, f, mt, q, it, &on_it);
    // new short-side energies (R has been taken from the previous ones)
    if (q.cond && lane < q.r) {
      float e = 0.f;
#pragma unroll
      for (int w = 0; w < FW; ++w) e += rede[w][lane];
      q.e_r[lane] = e;
    }
    for (int idx = lane; idx < RP * RP; idx += 32) {
      const int i = idx / RP, j = idx % RP;
      Tsm[i][j] = factor * it.R[i] * it.P[i][j] * it.R[j];
    }
    if (lane == 0) zsh = factor == 0.0 ? 1 : 0;
  }
  __syncthreads();

  // ---- pass 2: O = T (C^2 B), W update, long-side energies -----------------
  double tm[RP][RP];
#pragma unroll
  for (int i = 0; i < RP; ++i)
#pragma unroll
    for (int k = 0; k < RP; ++k) tm[i][k] = Tsm[i][k];
  const bool zero = zsh != 0;
  const float lr = p.lr, decay = p.decay;
  float wv[RP][4];
  if (4 * (int64_t)tid < n) load_cols<RP>(mt.W, mt.wdt, q, 4 * (int64_t)tid, wv);
  for (int64_t c = 4 * (int64_t)tid; c < n; c += 4 * FT) {
    float wn[RP][4], ov[RP][4];
    const bool more = c + 4 * FT < n;
    if (more) load_cols<RP>(mt.W, mt.wdt, q, c + 4 * FT, wn);
    double wd[4] = {1.0, 1.0, 1.0, 1.0};
    if (on) {
      const float4 e4 = *reinterpret_cast<const float4*>(q.e_c + c);
      wd[0] = (double)col_weight(e4.x, inv_mc, eps);
      wd[1] = (double)col_weight(e4.y, inv_mc, eps);
      wd[2] = (double)col_weight(e4.z, inv_mc, eps);
      wd[3] = (double)col_weight(e4.w, inv_mc, eps);
    }
    float ce[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      double x[RP];
      float sq = 0.f;
#pragma unroll
      for (int k = 0; k < RP; ++k) {
        const float m = Ms[(c + e) * RP + k];
        const double bv = nest ? fma((double)mu, (double)m, (double)Gs[(c + e) * RP + k]) : (double)m;
        x[k] = on ? wd[e] * bv : bv;
        sq = fmaf(m, m, sq);
      }
      ce[e] = sq;
#pragma unroll
      for (int i = 0; i < RP; ++i) {
        double y = 0.0;
#pragma unroll
        for (int k = 0; k < RP; ++k) y = fma(tm[i][k], x[k], y);
        ov[i][e] = zero ? 0.f : (float)y;
        wv[i][e] = decay * wv[i][e] - lr * ov[i][e];
      }
    }
    store_cols<RP>(mt.W, mt.wdt, q, c, wv);
    if (mt.upd) store_cols<RP>(mt.upd, DT_FP32, q, c, ov);
    if (q.cond) *reinterpret_cast<float4*>(q.e_c + c) = make_float4(ce[0], ce[1], ce[2], ce[3]);
    if (more) {
#pragma unroll
      for (int i = 0; i < RP; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) wv[i][e] = wn[i][e];
    }
  }
}

template <typename K>
int resident_ctas(K kernel, int smem) {
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, TT, smem) != cudaSuccess || occ < 1)
    occ = 1;
  return occ;
}

template <int RP, typename T>
cudaError_t launch_iter_t(const ThinParams& p, cudaStream_t st) {
  const int iter_bytes = (int)sizeof(IterSmem<RP, T>);
  static DeviceOnce once;
  const cudaError_t e = device_once(once, nullptr, [&](int) {
    return cudaFuncSetAttribute(thin_iterate<RP, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                iter_bytes);
  });
  if (e != cudaSuccess) return e;
  thin_iterate<RP, T><<<p.count, IT, iter_bytes, st>>>(p);
  return cudaGetLastError();
}

template <int RP>
cudaError_t launch_iter_rp(const ThinParams& p, cudaStream_t st) {
  if constexpr (RP <= 8) {
    thin_iterate_warp<RP><<<(p.count + TW - 1) / TW, TT, 0, st>>>(p);
    return cudaGetLastError();
  } else {
    // the split-sum passes (bf16 tensor-core mode) feed an fp32 iteration
    if (p.split) return launch_iter_t<RP, float>(p, st);
    return launch_iter_t<RP, double>(p, st);
  }
}

template <int RP>
cudaError_t launch_rp(ThinParams& p, int nsm, cudaStream_t st) {
  static DeviceOnce once;
  static int occ_gram[MAX_DEVICES], occ_apply[MAX_DEVICES];
  int dev = 0;
  cudaError_t e = device_once(once, &dev, [](int d) {
    occ_gram[d] = resident_ctas(thin_gram<RP>, 0);
    occ_apply[d] = resident_ctas(thin_apply<RP>, 0);
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  p.grid_gram = std::min(p.units, nsm * occ_gram[dev]);
  p.grid_apply = std::min(p.units, nsm * occ_apply[dev]);
  thin_gram<RP><<<p.grid_gram, TT, 0, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_iter_rp<RP>(p, st);
  if (e != cudaSuccess) return e;
  thin_apply<RP><<<p.grid_apply, TT, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

int thin_part_doubles(int pad) {
  switch (pad) {
    case 1: return TCfg<1>::PART;
    case 2: return TCfg<2>::PART;
    case 3: return TCfg<3>::PART;
    case 4: return TCfg<4>::PART;
    case 8: return TCfg<8>::PART;
    case 16: return TCfg<16>::PART;
    default: return TCfg<32>::PART;
  }
}

int thin_slab(int pad) {
  switch (pad) {
    case 1: return TCfg<1>::SLAB;
    case 2: return TCfg<2>::SLAB;
    case 3: return TCfg<3>::SLAB;
    case 4: return TCfg<4>::SLAB;
    case 8: return TCfg<8>::SLAB;
    case 16: return TCfg<16>::SLAB;
    default: return TCfg<32>::SLAB;
  }
}

cudaError_t launch_thin_iterate(const ThinParams& p, cudaStream_t s) {
  switch (p.pad) {
    case 1: return launch_iter_rp<1>(p, s);
    case 2: return launch_iter_rp<2>(p, s);
    case 3: return launch_iter_rp<3>(p, s);
    case 4: return launch_iter_rp<4>(p, s);
    case 8: return launch_iter_rp<8>(p, s);
    case 16: return launch_iter_rp<16>(p, s);
    default: return launch_iter_rp<32>(p, s);
  }
}

namespace {
template <int RP>
cudaError_t launch_fused_rp(const ThinParams& p, size_t smem, cudaStream_t st) {
  static DeviceOnce once;
  const cudaError_t e = device_once(once, nullptr, [](int) {
    return cudaFuncSetAttribute(thin_fused<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)THIN_FUSED_MAX_SMEM);
  });
  if (e != cudaSuccess) return e;
  thin_fused<RP><<<p.count, FT, smem, st>>>(p);
  return cudaGetLastError();
}
}  // namespace

size_t thin_fused_smem(int pad, int64_t n, bool nesterov) {
  return (size_t)n * (size_t)pad * sizeof(float) * (nesterov ? 2 : 1);
}

cudaError_t launch_thin_fused(const ThinParams& p, size_t smem, cudaStream_t s) {
  if (p.count <= 0) return cudaSuccess;
  if (smem > THIN_FUSED_MAX_SMEM) return cudaErrorInvalidValue;
  if (p.pad != 2) return cudaErrorInvalidValue;
  return launch_fused_rp<2>(p, smem, s);
}

cudaError_t launch_thin_setup(const ThinSetupParams& p, cudaStream_t s) {
  if (p.count <= 0) return cudaSuccess;
  thin_setup<<<p.count, 256, 0, s>>>(p);
  return cudaGetLastError();
}

// All factors of one group share the padded short side p.pad (1, 2, 3, 4,
// 8, 16 or 32); their descriptors are in p.mats (written by thin_setup).
cudaError_t launch_thin(ThinParams& p, int nsm, cudaStream_t s) {
  if (p.count <= 0 || p.units <= 0) return cudaSuccess;
  switch (p.pad) {
    case 1: return launch_rp<1>(p, nsm, s);
    case 2: return launch_rp<2>(p, nsm, s);
    case 3: return launch_rp<3>(p, nsm, s);
    case 4: return launch_rp<4>(p, nsm, s);
    case 8: return launch_rp<8>(p, nsm, s);
    case 16: return launch_rp<16>(p, nsm, s);
    default: return launch_rp<32>(p, nsm, s);
  }
}

}  // namespace dm
