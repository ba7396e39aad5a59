// Whole Muon / Dimuon step for thin factors (short side r <= 32, e.g. LoRA A
// (r x n) and B (n x r)), one thread-block cluster per factor.
//
// The Newton-Schulz iterate is a left-multiple of the start matrix: each step
// X <- (aI + bA + cA^2) X with A = X X^T, so X_k = P_k X_0 with an r x r
// polynomial P_k in the Gram matrix A_0 = X_0 X_0^T; A_{k+1} = Q_k A_k Q_k.
// ("From PCG to Muon", section 6 "Muon's Gram Matrix": the orthogonaliser
// normalises the global Gram matrix G^T G; sitech.ge, "Instead of SVD -
// Newton-Schulz" for the iteration itself.)  The factor is streamed twice and
// the iteration runs in r x r space:
//   pass 1   M_t = mu M_{t-1} + G (stored), X_0 = R M_t C in fp64,
//            A_0 += X_0 X_0^T and H += X_0 C^2 X_0^T in fp64 (exact products),
//            row energies of M_t
//   reduce   Gram partials of the cluster's CTAs through distributed shared
//            memory, in rank order (deterministic)
//   iterate  rank 0: P <- Q P, A <- Q A Q in fp64; the Frobenius norms of
//            X_5 = P X_0 / s and Y = R X_5 C follow from A_0 and H; T = factor P
//   pass 2   reload M_t (L2-resident), O = R (T X_0) C, W update, column
//            energies of M_t
// The fp64 products (Gram matrices, r x r iteration, apply) run on the fp64
// tensor-core MMA (mma.sync m8n8k4) for r > 4; r <= 4 uses plain fp64 FMAs.
// Each CTA of the cluster owns a contiguous run of 4096-element chunks of the
// long side; the next chunk's loads are in flight during the current chunk's
// arithmetic.
// Dimuon conditioning, renormalisation, scale and decay follow "Dimuon: LoRA
// 에 맞춰 다시 짠 Muon" ("-1/4 power from both sides", "Why the *last*
// momentum", Problem 4) and "Muon Optimizer 정리" (eq. (1)-(3), "Scaling up").
#include <cooperative_groups.h>

#include "dm_common.cuh"

namespace cg = cooperative_groups;

namespace dm {
namespace {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int CHUNK_ELEMS = 4096;  // RP x CH elements per chunk
constexpr int VEC = 4;             // elements per vector access
constexpr int NVEC = CHUNK_ELEMS / VEC / THREADS;  // vectors per thread per chunk (4)

template <int RP>
struct Cfg {
  static constexpr bool MMA = RP >= 8;                // fp64 tensor-core path
  static constexpr int CH = CHUNK_ELEMS / RP;         // columns per chunk
  static constexpr int XLD = CH + 4;                  // padded fp64 row (8-bank shift)
  static constexpr int MLD = CH + 1;                  // padded fp32 row
  static constexpr int SLD = RP + 1;                  // padded r x r row
  static constexpr int NBD = RP / 8;                  // 8-row blocks (MMA path)
  static constexpr int NUB = NBD * (NBD + 1) / 2;     // upper-triangle 8x8 blocks
  // per-warp partials (MMA path: one RP x RP matrix per warp) or per-thread
  // partials (small path: two per thread)
  static constexpr int PARTN =
      WARPS * RP * RP > 2 * THREADS ? WARPS * RP * RP : 2 * THREADS;
};

template <int RP>
struct ThinSmem {
  union {
    struct {
      double xs[RP][Cfg<RP>::XLD];   // X_0 chunk (fp64)
      float ms[RP][Cfg<RP>::MLD];    // stored momentum chunk, then the update chunk
    } pass;
    double part[Cfg<RP>::PARTN];     // Gram / H partials
    struct {
      double G[RP][Cfg<RP>::SLD], H[RP][Cfg<RP>::SLD], P[RP][Cfg<RP>::SLD],
          A[RP][Cfg<RP>::SLD], Q[RP][Cfg<RP>::SLD], S[RP][Cfg<RP>::SLD];
    } it;
  } u;
  double Gc[RP * RP];  // this CTA's Gram partial (rank 0 reads it over DSMEM)
  double Hc[RP * RP];
  double T[RP][Cfg<RP>::SLD];  // factor * P, broadcast from rank 0
  float rowp[RP];              // row-energy partial of this CTA's slice
  float Rv[RP];
  float Cc[Cfg<RP>::CH];
  float red32[THREADS];
  double red[32];
  double sc[8];  // [0] slice sum of previous long-side energies, [1] factor, [4] ||X_0||^2
};

// D (8x8, two values per lane) += A (8x4) * B (4x8) in fp64.
// Lane l = 4g + t holds A[g][t], B[t][g], D[g][2t], D[g][2t+1].
__device__ __forceinline__ void dmma(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

// (relative energy + eps)^(-1/4) as 1 / sqrt(sqrt(.)).
__device__ __forceinline__ float cond_value(float rel_plus_eps) {
  return rsqrtf(sqrtf(rel_plus_eps));
}

// C = A * B for RP x RP fp64 matrices in shared memory (padded rows).
template <int RP>
__device__ __forceinline__ void mm(double (*C)[Cfg<RP>::SLD], double (*A)[Cfg<RP>::SLD],
                                   double (*B)[Cfg<RP>::SLD]) {
  if constexpr (Cfg<RP>::MMA) {
    constexpr int NBD = Cfg<RP>::NBD;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    for (int blk = warp; blk < NBD * NBD; blk += WARPS) {
      const int rb = blk / NBD, cb = blk % NBD;
      double d0 = 0.0, d1 = 0.0;
#pragma unroll
      for (int kb = 0; kb < RP / 4; ++kb)
        dmma(d0, d1, A[rb * 8 + g][kb * 4 + t], B[kb * 4 + t][cb * 8 + g]);
      C[rb * 8 + g][cb * 8 + 2 * t] = d0;
      C[rb * 8 + g][cb * 8 + 2 * t + 1] = d1;
    }
  } else {
    for (int idx = threadIdx.x; idx < RP * RP; idx += THREADS) {
      const int i = idx / RP, j = idx % RP;
      double s = 0.0;
#pragma unroll
      for (int k = 0; k < RP; ++k) s = fma(A[i][k], B[k][j], s);
      C[i][j] = s;
    }
  }
  __syncthreads();
}

// 4 consecutive elements (aligned) <-> floats.
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

template <int RP>
__global__ void __launch_bounds__(THREADS, 2) thin_step(const __grid_constant__ ThinParams p) {
  using Cf = Cfg<RP>;
  constexpr int CH = Cf::CH;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  ThinSmem<RP>& s = *reinterpret_cast<ThinSmem<RP>*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cs = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();

  const ThinMat& mt = p.mats[blockIdx.x / cs];
  const bool tall = mt.rows > mt.cols;
  const int r = (int)(tall ? mt.cols : mt.rows);
  const int64_t n = tall ? mt.rows : mt.cols;
  const int64_t nck = (n + CH - 1) / CH;  // chunks of the factor
  const int64_t k_lo = (nck * rank / cs) * CH;
  const int64_t k_hi = min(n, (nck * (rank + 1) / cs) * CH);
  float* e_r = tall ? mt.e_col : mt.e_row;  // energies along the short side
  float* e_c = tall ? mt.e_row : mt.e_col;  // energies along the long side
  const bool cond = p.conditioned && e_r != nullptr && e_c != nullptr;
  // Vector path: each 4-vector lies in one row (wide) or the chunk is one
  // contiguous run (tall with RP == r).
  // (tall r = 2 vectors span two columns: the long side must be even)
  const bool vec = mt.vec && (tall ? (RP == r && (RP >= 4 || n % 2 == 0)) : (n % VEC) == 0);

  // element (i, k) of X (short side i) in storage
  auto off = [&](int i, int64_t k) -> int64_t { return tall ? k * r + i : (int64_t)i * n + k; };
  // vector v of a chunk -> first element's (row, column); tall vectors run
  // along the flat (column-major in X) order
  auto vcoord = [&](int v, int& i, int& kk) {
    if (tall) {
      kk = (v * VEC) / RP;
      i = (v * VEC) % RP;
    } else {
      i = v / (CH / VEC);
      kk = (v % (CH / VEC)) * VEC;
    }
  };
  // element e (0..3) of a vector starting at (i, kk)
  auto ecoord = [&](int i, int kk, int e, int& ie, int& ke) {
    if (tall) {
      ie = (i + e) % RP;
      ke = kk + (i + e) / RP;
    } else {
      ie = i;
      ke = kk + e;
    }
  };

  // ---- means of the previous energies.  Every read of e_r / e_c for them
  //      happens before the first cluster barrier; in-place writes come later.
  double sr = 0.0, sl = 0.0;
  if (cond) {
    for (int i = tid; i < r; i += THREADS) sr += (double)e_r[i];
    for (int64_t k = k_lo + tid; k < k_hi; k += THREADS) sl += (double)e_c[k];
  }
  sr = block_sum_d(sr, s.red);
  sl = block_sum_d(sl, s.red);
  if (tid == 0) s.sc[0] = sl;
  cluster.sync();
  double sc_tot = 0.0;
  for (int q = 0; q < cs; ++q) sc_tot += *cluster.map_shared_rank(&s.sc[0], q);
  const bool on = cond && sr > 0.0 && sc_tot > 0.0;
  const float inv_mr = on ? (float)((double)r / sr) : 0.f;
  const float inv_mc = on ? (float)((double)n / sc_tot) : 0.f;
  if (tid < RP) {
    s.Rv[tid] = tid < r ? (on ? cond_value(e_r[tid] * inv_mr + p.eps) : 1.f) : 0.f;
    s.rowp[tid] = 0.f;
  }

  // previous long-side energies of a chunk ride along with its loads
  constexpr int ECP = (CH + THREADS - 1) / THREADS;
  float ecv[ECP];
  auto load_energies = [&](int64_t k0) {
#pragma unroll
    for (int q = 0; q < ECP; ++q) {
      const int kk = tid + THREADS * q;
      ecv[q] = (on && kk < CH && k0 + kk < k_hi) ? e_c[k0 + kk] : 0.f;
    }
  };
  auto conditioning_of_chunk = [&](int cw) {
#pragma unroll
    for (int q = 0; q < ECP; ++q) {
      const int kk = tid + THREADS * q;
      if (kk < CH) s.Cc[kk] = kk < cw ? (on ? cond_value(ecv[q] * inv_mc + p.eps) : 1.f) : 0.f;
    }
  };
  // loads of one chunk: a = first operand (G in pass 1, M in pass 2), b = second
  // (M in pass 1, W in pass 2)
  float av[NVEC][VEC], bv[NVEC][VEC];
  // second operand optional (with_b = false loads only pa)
  auto load_chunk_pair = [&](int64_t k0, const void* pa, int dta, const void* pb, int dtb,
                             float (&oa)[NVEC][VEC], float (&ob)[NVEC][VEC], bool with_b) {
    const int cw = (int)min((int64_t)CH, k_hi - k0);
#pragma unroll
    for (int q = 0; q < NVEC; ++q) {
      int i, kk;
      vcoord(tid + THREADS * q, i, kk);
      if (vec) {
        const bool ok = k0 < k_hi && i < r && kk < cw;  // vectors never straddle cw
        if (ok) {
          ld4(pa, off(i, k0 + kk), dta, oa[q]);
          if (with_b) ld4(pb, off(i, k0 + kk), dtb, ob[q]);
        } else {
#pragma unroll
          for (int e = 0; e < VEC; ++e) oa[q][e] = ob[q][e] = 0.f;
        }
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          int ie, ke;
          ecoord(i, kk, e, ie, ke);
          const bool ok = k0 < k_hi && ie < r && ke < cw;
          const int64_t o = ok ? off(ie, k0 + ke) : 0;
          oa[q][e] = ok ? ld_elem(pa, o, dta) : 0.f;
          ob[q][e] = (ok && with_b) ? ld_elem(pb, o, dtb) : 0.f;
        }
      }
    }
  };

  auto load_chunk = [&](int64_t k0, const void* pa, int dta, const void* pb, int dtb) {
    load_energies(k0);
    load_chunk_pair(k0, pa, dta, pb, dtb, av, bv, true);
  };

  // ---- pass 1 ----------------------------------------------------------------
  // MMA path: warps 0..3 accumulate A_0, warps 4..7 accumulate H, each over a
  // quarter of the chunk's 4-column steps; fragments are 8x8 upper blocks.
  double acc[Cf::MMA ? Cf::NUB : 1][2];
  // SIMT path (RP <= 4): thread t accumulates pair (t % (RP*RP)) over columns
  double sacc_g = 0.0, sacc_h = 0.0;
#pragma unroll
  for (int b = 0; b < (Cf::MMA ? Cf::NUB : 1); ++b) acc[b][0] = acc[b][1] = 0.0;

  load_chunk(k_lo, mt.G, mt.gdt, mt.M, mt.mdt);
  for (int64_t k0 = k_lo; k0 < k_hi; k0 += CH) {
    const int cw = (int)min((int64_t)CH, k_hi - k0);
    conditioning_of_chunk(cw);
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NVEC; ++q) {
      int i, kk;
      vcoord(tid + THREADS * q, i, kk);
      float m4[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        int ie, ke;
        ecoord(i, kk, e, ie, ke);
        const bool ok = ie < r && ke < cw;
        m4[e] = ok ? momentum_value(p.mu, bv[q][e], av[q][e], mt.mdt) : 0.f;
        s.u.pass.ms[ie][ke] = m4[e];
        // orthogonaliser input: M_t, or B_t = G + mu M_t under Nesterov
        const double b = p.nesterov ? fma((double)p.mu, (double)m4[e], (double)av[q][e])
                                    : (double)m4[e];
        s.u.pass.xs[ie][ke] = (double)s.Rv[ie] * b * (double)s.Cc[ke];
        if (!vec && ok) st_elem(mt.M, off(ie, k0 + ke), mt.mdt, m4[e]);
      }
      if (vec && i < r && kk < cw) st4(mt.M, off(i, k0 + kk), mt.mdt, m4);
    }
    load_chunk(k0 + CH, mt.G, mt.gdt, mt.M, mt.mdt);  // in flight during the Gram
    __syncthreads();
    if (cond) {  // row energies: THREADS / RP threads per row
      constexpr int TPR = THREADS / RP;
      const int i = tid / TPR;
      float e = 0.f;
      if (i < r)
        for (int kk = tid % TPR; kk < cw; kk += TPR) e = fmaf(s.u.pass.ms[i][kk], s.u.pass.ms[i][kk], e);
      s.red32[tid] = e;
    }
    if constexpr (Cf::MMA) {
      const int g = lane >> 2, t = lane & 3;
      const bool hpart = warp >= 4;
      for (int ks = warp & 3; ks < CH / 4; ks += 4) {
        const int kk = ks * 4 + t;
        const double c2 = hpart ? (double)s.Cc[kk] * (double)s.Cc[kk] : 1.0;
        double f[Cf::NBD];
#pragma unroll
        for (int b = 0; b < Cf::NBD; ++b) f[b] = s.u.pass.xs[b * 8 + g][kk];
        int ub = 0;
#pragma unroll
        for (int bi = 0; bi < Cf::NBD; ++bi)
#pragma unroll
          for (int bj = bi; bj < Cf::NBD; ++bj, ++ub) dmma(acc[ub][0], acc[ub][1], f[bi], f[bj] * c2);
      }
    } else {
      const int pr = tid % (RP * RP), i = pr / RP, j = pr % RP;
      for (int kk = tid / (RP * RP); kk < cw; kk += THREADS / (RP * RP)) {
        const double x = s.u.pass.xs[i][kk] * s.u.pass.xs[j][kk];
        sacc_g += x;
        sacc_h = fma(x, (double)s.Cc[kk] * (double)s.Cc[kk], sacc_h);
      }
    }
    __syncthreads();
    if (cond && tid < r) {
      constexpr int TPR = THREADS / RP;
      float e = 0.f;
      for (int q = 0; q < TPR; ++q) e += s.red32[tid * TPR + q];
      s.rowp[tid] += e;
    }
  }
  __syncthreads();

  // ---- CTA-level reduction of the Gram partials (fixed order) -----------------
  if constexpr (Cf::MMA) {
    const int g = lane >> 2, t = lane & 3;
    double* dst = s.u.part + warp * RP * RP;  // warps 0..3: A_0, warps 4..7: H
    int ub = 0;
#pragma unroll
    for (int bi = 0; bi < Cf::NBD; ++bi)
#pragma unroll
      for (int bj = bi; bj < Cf::NBD; ++bj, ++ub) {
        dst[(bi * 8 + g) * RP + bj * 8 + 2 * t] = acc[ub][0];
        dst[(bi * 8 + g) * RP + bj * 8 + 2 * t + 1] = acc[ub][1];
      }
    __syncthreads();
    for (int idx = tid; idx < RP * RP; idx += THREADS) {
      const int i = idx / RP, j = idx % RP;
      const int src = (i / 8 <= j / 8) ? idx : j * RP + i;  // lower blocks mirror upper ones
      double gs = 0.0, hs = 0.0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        gs += s.u.part[w * RP * RP + src];
        hs += s.u.part[(w + 4) * RP * RP + src];
      }
      s.Gc[idx] = gs;
      s.Hc[idx] = hs;
    }
  } else {
    s.u.part[tid] = sacc_g;
    s.u.part[THREADS + tid] = sacc_h;
    __syncthreads();
    for (int idx = tid; idx < RP * RP; idx += THREADS) {
      double gs = 0.0, hs = 0.0;
      for (int q = idx; q < THREADS; q += RP * RP) {
        gs += s.u.part[q];
        hs += s.u.part[THREADS + q];
      }
      s.Gc[idx] = gs;
      s.Hc[idx] = hs;
    }
  }
  cluster.sync();  // every CTA's Gc / Hc / rowp are final

  // ---- rank 0: cluster reduction and the r x r iteration -----------------------
  if (rank == 0) {
    for (int idx = tid; idx < RP * RP; idx += THREADS) {
      double gv[8], hv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        gv[q] = q < cs ? cluster.map_shared_rank(&s.Gc[0], q)[idx] : 0.0;
        hv[q] = q < cs ? cluster.map_shared_rank(&s.Hc[0], q)[idx] : 0.0;
      }
      double g = 0.0, h = 0.0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        g += gv[q];
        h += hv[q];
      }
      s.u.it.G[idx / RP][idx % RP] = g;
      s.u.it.H[idx / RP][idx % RP] = h;
    }
    if (cond && tid < r) {
      float e = 0.f;
      for (int q = 0; q < cs; ++q) e += cluster.map_shared_rank(&s.rowp[0], q)[tid];
      e_r[tid] = e;
    }
    __syncthreads();
    if (tid == 0) {
      double tr = 0.0;
      for (int i = 0; i < r; ++i) tr += s.u.it.G[i][i];
      s.sc[4] = tr;
    }
    __syncthreads();
    const double s2 = s.sc[4];
    const bool finite = isfinite(s2);
    const bool valid = finite && s2 >= NORM2_FLOOR;  // else the update is zero
    const double inv_s2 = valid ? 1.0 / s2 : 0.0;
    for (int idx = tid; idx < RP * RP; idx += THREADS) {
      const int i = idx / RP, j = idx % RP;
      s.u.it.A[i][j] = valid ? s.u.it.G[i][j] * inv_s2 : 0.0;
      s.u.it.P[i][j] = i == j ? 1.0 : 0.0;
    }
    __syncthreads();
    const double a = p.a, b = p.b, c = p.c;
    for (int it = 0; it < p.ns_steps; ++it) {
      mm<RP>(s.u.it.Q, s.u.it.A, s.u.it.A);  // Q = A A
      for (int idx = tid; idx < RP * RP; idx += THREADS) {
        const int i = idx / RP, j = idx % RP;
        s.u.it.Q[i][j] = c * s.u.it.Q[i][j] + b * s.u.it.A[i][j] + (i == j ? a : 0.0);
      }
      __syncthreads();
      mm<RP>(s.u.it.S, s.u.it.Q, s.u.it.P);  // P <- Q P
      for (int idx = tid; idx < RP * RP; idx += THREADS)
        s.u.it.P[idx / RP][idx % RP] = s.u.it.S[idx / RP][idx % RP];
      __syncthreads();
      mm<RP>(s.u.it.S, s.u.it.Q, s.u.it.A);  // A <- Q A Q
      mm<RP>(s.u.it.A, s.u.it.S, s.u.it.Q);
    }
    // ||X_5||^2 s^2 = tr(P A_0 P^T); ||R X_5 C||^2 s^2 = sum_i R_i^2 (P H P^T)_ii
    mm<RP>(s.u.it.S, s.u.it.P, s.u.it.G);
    double nx = 0.0;
    for (int idx = tid; idx < RP * RP; idx += THREADS)
      nx += s.u.it.S[idx / RP][idx % RP] * s.u.it.P[idx / RP][idx % RP];
    nx = block_sum_d(nx, s.red);
    mm<RP>(s.u.it.Q, s.u.it.P, s.u.it.H);
    double ny = 0.0;
    for (int idx = tid; idx < RP * RP; idx += THREADS) {
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
    for (int idx = tid; idx < RP * RP; idx += THREADS)
      s.T[idx / RP][idx % RP] = factor * s.u.it.P[idx / RP][idx % RP];
    if (tid == 0) s.sc[1] = factor;
  }
  cluster.sync();  // rank 0's T is final
  if (rank != 0) {
    const double* T0 = &cluster.map_shared_rank(&s.T[0][0], 0)[0];
    for (int idx = tid; idx < RP * Cf::SLD; idx += THREADS) (&s.T[0][0])[idx] = T0[idx];
    if (tid == 0) s.sc[1] = *cluster.map_shared_rank(&s.sc[1], 0);
  }
  cluster.sync();  // no CTA reads another CTA's shared memory after this point
  const bool zero_update = s.sc[1] == 0.0;

  // ---- pass 2 ----------------------------------------------------------------
  // Under Nesterov, X_0 needs G again: cv holds a chunk's G.
  float cv[NVEC][VEC];
  auto load_grad = [&](int64_t k0) {
    if (!p.nesterov) return;
    load_chunk_pair(k0, mt.G, mt.gdt, mt.G, mt.gdt, cv, cv, false);
  };
  load_grad(k_lo);
  load_chunk(k_lo, mt.M, mt.mdt, mt.W, mt.wdt);
  for (int64_t k0 = k_lo; k0 < k_hi; k0 += CH) {
    const int cw = (int)min((int64_t)CH, k_hi - k0);
    conditioning_of_chunk(cw);
    __syncthreads();
    float wcur[NVEC][VEC];
#pragma unroll
    for (int q = 0; q < NVEC; ++q) {
      int i, kk;
      vcoord(tid + THREADS * q, i, kk);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        int ie, ke;
        ecoord(i, kk, e, ie, ke);
        s.u.pass.ms[ie][ke] = av[q][e];
        const double b = p.nesterov ? fma((double)p.mu, (double)av[q][e], (double)cv[q][e])
                                    : (double)av[q][e];
        s.u.pass.xs[ie][ke] = (double)s.Rv[ie] * b * (double)s.Cc[ke];
        wcur[q][e] = bv[q][e];
      }
    }
    load_grad(k0 + CH);
    load_chunk(k0 + CH, mt.M, mt.mdt, mt.W, mt.wdt);  // in flight during the apply
    __syncthreads();
    if (cond) {
      for (int kk = tid; kk < cw; kk += THREADS) {
        float e = 0.f;
        for (int i = 0; i < r; ++i) e = fmaf(s.u.pass.ms[i][kk], s.u.pass.ms[i][kk], e);
        e_c[k0 + kk] = e;
      }
    }
    __syncthreads();
    if constexpr (Cf::MMA) {
      // O block (rb, cb) = sum_kb T[rb, kb] X[kb, cb]; one warp per 8 columns
      const int g = lane >> 2, t = lane & 3;
      for (int cb = warp; cb < CH / 8; cb += WARPS) {
        double o[Cf::NBD][2];
#pragma unroll
        for (int rb = 0; rb < Cf::NBD; ++rb) o[rb][0] = o[rb][1] = 0.0;
#pragma unroll
        for (int kb = 0; kb < RP / 4; ++kb) {
          const double xb = s.u.pass.xs[kb * 4 + t][cb * 8 + g];
#pragma unroll
          for (int rb = 0; rb < Cf::NBD; ++rb)
            dmma(o[rb][0], o[rb][1], s.T[rb * 8 + g][kb * 4 + t], xb);
        }
#pragma unroll
        for (int rb = 0; rb < Cf::NBD; ++rb)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int i = rb * 8 + g, kk = cb * 8 + 2 * t + h;
            s.u.pass.ms[i][kk] =
                zero_update ? 0.f : (float)((double)s.Rv[i] * o[rb][h] * (double)s.Cc[kk]);
          }
      }
    } else {
      for (int o = tid; o < CH; o += THREADS) {
        double x[RP];
#pragma unroll
        for (int j = 0; j < RP; ++j) x[j] = s.u.pass.xs[j][o];
#pragma unroll
        for (int i = 0; i < RP; ++i) {
          double acc2 = 0.0;
#pragma unroll
          for (int j = 0; j < RP; ++j) acc2 = fma(s.T[i][j], x[j], acc2);
          s.u.pass.ms[i][o] = zero_update ? 0.f : (float)((double)s.Rv[i] * acc2 * (double)s.Cc[o]);
        }
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NVEC; ++q) {
      int i, kk;
      vcoord(tid + THREADS * q, i, kk);
      float u4[VEC], w4[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        int ie, ke;
        ecoord(i, kk, e, ie, ke);
        u4[e] = s.u.pass.ms[ie][ke];
        w4[e] = p.decay * wcur[q][e] - p.lr * u4[e];
        if (!vec && ie < r && ke < cw) {
          const int64_t o = off(ie, k0 + ke);
          st_elem(mt.W, o, mt.wdt, w4[e]);
          if (mt.upd) mt.upd[o] = u4[e];
        }
      }
      if (vec && i < r && kk < cw) {
        st4(mt.W, off(i, k0 + kk), mt.wdt, w4);
        if (mt.upd) st4(mt.upd, off(i, k0 + kk), DT_FP32, u4);
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
    cudaError_t e =
        cudaFuncSetAttribute(thin_step<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    configured = dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.count * p.cluster), 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = (size_t)bytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, thin_step<RP>, p);
}

}  // namespace

// All factors of one launch share the padded short side p.pad (2..32) and
// the cluster size p.cluster (1..8 CTAs per factor).
cudaError_t launch_thin(const ThinParams& p, cudaStream_t s) {
  if (p.count <= 0) return cudaSuccess;
  switch (p.pad) {
    case 2: return launch_rp<2>(p, s);
    case 4: return launch_rp<4>(p, s);
    case 8: return launch_rp<8>(p, s);
    case 16: return launch_rp<16>(p, s);
    default: return launch_rp<32>(p, s);
  }
}

}  // namespace dm
