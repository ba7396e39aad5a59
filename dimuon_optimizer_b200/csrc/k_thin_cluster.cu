// Single-launch thin-factor step: one thread-block cluster per factor holds
// the whole factor in its shared memory.
//
// Same arithmetic as the Gram route of k_thin.cu / k_thin_bulk.cu ("From PCG
// to Muon", section 6 "Muon's Gram Matrix"; see k_thin.cu for the
// derivation): with b_j the long-side columns of B = M_t (G + mu M_t under
// Nesterov) and C_j^2 the Dimuon column weights,
//   S_1 = sum_j C_j^2 b_j b_j^T,  S_2 = sum_j C_j^4 b_j b_j^T,
//   O(:, j) = C_j^2 T b_j with T = f R P_5 R from the r x r iteration.
// Every CTA of the cluster owns a contiguous slice of the long side:
//   1. it issues bulk async copies (cp.async.bulk) of its slice of M_{t-1},
//      G and the previous long-side energies at once, so the whole slice is
//      in flight together, and sums the previous energies (all of them, in
//      the same order in every CTA of the cluster);
//   2. pass 1: M_t = mu M_{t-1} + G (exact value, one rounding) in place in shared
//      memory, S_1 / S_2 partial sums (fp64; fp64 tensor-core MMA for r = 8),
//      short-side energy partials; M_t goes back to global memory by a bulk
//      store, and the slice of W is fetched into the space G used (unless
//      Nesterov keeps G);
//   3. the CTAs' partial sums meet in the first CTA's shared memory
//      (distributed shared memory, one cluster barrier); every CTA sums them
//      in rank order and runs the r x r iteration itself, so all hold the
//      same T without a second exchange;
//   4. pass 2: O = C^2 T B for the slice, W updated in shared memory and
//      written back by a bulk store, the new long-side energies stored.
// HBM traffic per element is the algorithmic one (G, M_{t-1} read, M_t
// written, W read and written), one launch per group of factors, and no
// workspace.  Every mbarrier wait is bounded; every CTA passes every cluster
// barrier, whatever happened to its own copies.
#include <algorithm>

#include "dm_common.cuh"
#include "dm_sm100.cuh"
#include "dm_thin.cuh"

namespace dm {
namespace {

using namespace thin;
using namespace sm100;

#ifndef DM_CL_THREADS
#define DM_CL_THREADS 256
#endif
constexpr int CT = DM_CL_THREADS;  // threads per CTA
constexpr int CW = CT / 32;
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;

// ------------------------------ PTX pieces --------------------------------
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(gdst)),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until the bulk stores issued by this thread have read their shared
// memory source (the CTA may then end or reuse it).
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Orders this CTA's generic-proxy shared-memory accesses before later
// async-proxy ones (bulk copies reading or writing the same bytes).
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_f64(uint32_t addr, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(addr), "d"(v) : "memory");
}
__device__ __forceinline__ double ld_cluster_f64(uint32_t addr) {
  double v;
  asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Element access of the staged operands, converted to / from fp32.
template <typename T>
struct Ty;
template <>
struct Ty<float> {
  static constexpr int DT = DT_FP32;
  __device__ static float ld(const float* p) { return *p; }
  __device__ static void st(float* p, float v) { *p = v; }
};
template <>
struct Ty<__nv_bfloat16> {
  static constexpr int DT = DT_BF16;
  __device__ static float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ static void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// Bounded wait on a local mbarrier phase; false (and the timeout raised) after
// WAIT_NS.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 63u) == 0u && globaltimer_ns() - t0 > WAIT_NS) {
      raise_timeout(status);
      return false;
    }
  }
}

// Layout of one CTA's slice in dynamic shared memory.  Wide factors: RP rows
// of NC elements with a padded pitch (bank spread for the fragment reads);
// tall factors: the slice's NC x RP elements as stored.
template <int RP, typename TG, typename TM, typename TW>
struct Slice {
  int nc;                     // long-side columns of the slice
  int pm, pg, pw;             // row pitches (elements) of M, G, W (wide)
  uint32_t off_g, off_w, off_e, bytes;
  __device__ __host__ static Slice make(int nc, bool tall, bool nest) {
    Slice s;
    s.nc = nc;
    // wide rows padded by 16 bytes: the 8 rows of a fragment read then fall on
    // different banks (rows stay 16-byte aligned for the bulk copies)
    s.pm = tall ? nc : nc + 16 / (int)sizeof(TM);
    s.pg = tall ? nc : nc + 16 / (int)sizeof(TG);
    s.pw = tall ? nc : nc + 16 / (int)sizeof(TW);
    auto up = [](uint32_t x) { return (x + 127u) / 128u * 128u; };
    const uint32_t bm = up((uint32_t)(RP * s.pm) * (uint32_t)sizeof(TM));
    const uint32_t bg = up((uint32_t)(RP * s.pg) * (uint32_t)sizeof(TG));
    const uint32_t bw = up((uint32_t)(RP * s.pw) * (uint32_t)sizeof(TW));
    s.off_g = bm;
    // without Nesterov, W is fetched into the space G used (same element size)
    s.off_w = nest ? bm + bg : bm;
    s.off_e = nest ? bm + bg + bw : bm + (bg > bw ? bg : bw);
    s.bytes = s.off_e + up((uint32_t)nc * 4u);
    return s;
  }
};

// Doubles per CTA partial in the exchange: S_1, S_2 (fragment blocks for
// RP = 8, full RP x RP otherwise), RP short-side energies, one abort flag.
template <int RP>
struct Xch {
  static constexpr int PART = TCfg<RP>::MMA ? 64 * TCfg<RP>::NUB : RP * RP;
  static constexpr int WORDS = 2 * PART + RP + 1;
};
template <int RP>
__host__ __device__ constexpr uint32_t xch_bytes(int cs) {
  return ((uint32_t)cs * Xch<RP>::WORDS * 8u + 127u) / 128u * 128u;
}

template <int RP, typename TG, typename TM, typename TW>
__global__ void __launch_bounds__(CT) thin_cluster(const __grid_constant__ ThinClusterParams p) {
  static_assert(RP == 2 || RP == 4 || RP == 8, "ranks of the cluster kernel");
  using X = Xch<RP>;
  using SL = Slice<RP, TG, TM, TW>;
  extern __shared__ __align__(128) uint8_t cl_raw[];
  __shared__ double red[CW][2 * X::PART];
  __shared__ float rede[CW][RP];
  __shared__ WarpIterSmem<RP> it;
  __shared__ double Tsm[RP][RP + 1];
  __shared__ double red_d[32];
  __shared__ float erp[RP];  // previous short-side energies, this CTA's copy
  __shared__ __align__(8) uint64_t bar_in, bar_w;
  __shared__ int flag_sh[3];  // [0] slice in place, [1] write outputs, [2] zero update

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int CS = (int)cluster_size();  // CTAs per factor (1 without a cluster launch)
  const int rank = (int)cluster_rank();
  const int f = (int)blockIdx.x / CS;
  const ThinMat mt = p.mats[f];
  const Geo q = geometry(mt, p.conditioned);
  const int64_t n = q.n;
  const int nc = (int)(n / CS);
  const int64_t c0 = (int64_t)rank * nc;
  const bool nest = p.nesterov != 0;
  const SL sl = SL::make(nc, q.tall, nest);
  // dynamic shared memory: the rank slots of the exchange (read in the first
  // CTA only), then the slice
  double* xch = reinterpret_cast<double*>(cl_raw);
  uint8_t* slice = cl_raw + xch_bytes<RP>(CS);
  TM* Ms = reinterpret_cast<TM*>(slice);
  TG* Gs = reinterpret_cast<TG*>(slice + sl.off_g);
  TW* Ws = reinterpret_cast<TW*>(slice + sl.off_w);
  float* Es = reinterpret_cast<float*>(slice + sl.off_e);
  TM* Mg = reinterpret_cast<TM*>(mt.M);
  const TG* Gg = reinterpret_cast<const TG*>(mt.G);
  TW* Wg = reinterpret_cast<TW*>(mt.W);
  // An earlier launch of the step timed out: nothing of this factor is
  // written.  (Every CTA still takes part in the cluster barriers.)
  const bool skip = step_aborted(p.status);

  if (tid == 0) {
    mbar_init(&bar_in, 1);
    mbar_init(&bar_w, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // ---- 1. the whole slice in flight: M_{t-1}, G (and the energies) --------
  if (tid == 0 && !skip) {
    const uint32_t em = (uint32_t)nc * (uint32_t)sizeof(TM), eg = (uint32_t)nc * (uint32_t)sizeof(TG);
    uint32_t bytes = RP * (em + eg) + (q.cond ? (uint32_t)nc * 4u : 0u);
    mbar_arrive_expect_tx(&bar_in, bytes);
    if (!q.tall) {
      for (int i = 0; i < RP; ++i) {
        bulk_load(Ms + (size_t)i * sl.pm, Mg + (int64_t)i * n + c0, em, &bar_in);
        bulk_load(Gs + (size_t)i * sl.pg, Gg + (int64_t)i * n + c0, eg, &bar_in);
      }
    } else {
      bulk_load(Ms, Mg + c0 * RP, RP * em, &bar_in);
      bulk_load(Gs, Gg + c0 * RP, RP * eg, &bar_in);
    }
    if (q.cond) bulk_load(Es, q.e_c + c0, (uint32_t)nc * 4u, &bar_in);
  }
  // every CTA of the cluster has started before any writes into the first
  // one's shared memory (waited on just before those writes)
  __syncwarp();
  cluster_arrive();
  // previous energies: the whole long side summed in the same order by every
  // CTA of the cluster (so all agree on the mean), the short side read before
  // the first CTA replaces it
  double sc = 0.0, sr = 0.0;
  if (q.cond) {
    const float4* e4 = reinterpret_cast<const float4*>(q.e_c);
    for (int64_t k = tid; k < (n >> 2); k += CT) {
      const float4 v = e4[k];
      sc += ((double)v.x + (double)v.y) + ((double)v.z + (double)v.w);
    }
#pragma unroll
    for (int i = 0; i < RP; ++i) sr += (double)q.e_r[i];
    if (tid < RP) erp[tid] = q.e_r[tid];
  }
  sc = block_sum_d(sc, red_d);  // (its barriers also publish erp)
  const bool on = q.cond && sc > 0.0 && sr > 0.0;
  const float inv_mc = on ? (float)((double)n / sc) : 0.f;
  const float mu = p.mu, eps = p.eps;

  if (tid == 0) {
    flag_sh[0] = skip ? 0 : (wait_bar(&bar_in, 0, p.status) ? 1 : 0);
    if (!skip && !flag_sh[0]) mbar_wait_drain(&bar_in, 0, DRAIN_NS);
  }
  __syncthreads();
  const bool have = flag_sh[0] != 0;

  // ---- 2. pass 1: momentum, Gram partials, short-side energies -----------
  constexpr bool MMA = TCfg<RP>::MMA;
  double s1[MMA ? 2 : RP][MMA ? 1 : RP], s2[MMA ? 2 : RP][MMA ? 1 : RP];
#pragma unroll
  for (int i = 0; i < (MMA ? 2 : RP); ++i)
#pragma unroll
    for (int k = 0; k < (MMA ? 1 : RP); ++k) s1[i][k] = s2[i][k] = 0.0;
  float er[MMA ? 1 : RP];
#pragma unroll
  for (int i = 0; i < (MMA ? 1 : RP); ++i) er[i] = 0.f;
  auto mi = [&](int i, int j) -> int { return q.tall ? j * RP + i : i * sl.pm + j; };
  auto gi = [&](int i, int j) -> int { return q.tall ? j * RP + i : i * sl.pg + j; };
  auto wi = [&](int i, int j) -> int { return q.tall ? j * RP + i : i * sl.pw + j; };
  if (have) {
    if constexpr (MMA) {
      // warp w: groups of four columns 4 cg .. 4 cg + 3; lane (g, t) = row g
      // of column 4 cg + t, the DMMA's A[g][t] and B[t][g]
      const int g = lane >> 2, t = lane & 3;
      for (int cg = warp; cg < nc / 4; cg += CW) {
        const int j = 4 * cg + t;
        const float m = momentum_value(mu, Ty<TM>::ld(Ms + mi(g, j)), Ty<TG>::ld(Gs + gi(g, j)), Ty<TM>::DT);
        Ty<TM>::st(Ms + mi(g, j), m);
        er[0] = fmaf(m, m, er[0]);
        const double b = nest ? fma((double)mu, (double)m, (double)Ty<TG>::ld(Gs + gi(g, j))) : (double)m;
        const double w = on ? (double)col_weight(Es[j], inv_mc, eps) : 1.0;
        dmma(s1[0][0], s1[1][0], b, w * b);
        if (on) dmma(s2[0][0], s2[1][0], b, w * w * b);
      }
    } else {
      for (int j = tid; j < nc; j += CT) {
        double b[RP];
#pragma unroll
        for (int i = 0; i < RP; ++i) {
          const float g = Ty<TG>::ld(Gs + gi(i, j));
          const float m = momentum_value(mu, Ty<TM>::ld(Ms + mi(i, j)), g, Ty<TM>::DT);
          Ty<TM>::st(Ms + mi(i, j), m);
          er[i] = fmaf(m, m, er[i]);
          b[i] = nest ? fma((double)mu, (double)m, (double)g) : (double)m;
        }
        const double w = on ? (double)col_weight(Es[j], inv_mc, eps) : 1.0;
#pragma unroll
        for (int i = 0; i < RP; ++i)
#pragma unroll
          for (int k = i; k < RP; ++k) {
            const double xk = w * b[k];
            s1[i][k] = fma(b[i], xk, s1[i][k]);
            if (on) s2[i][k] = fma(b[i], w * xk, s2[i][k]);
          }
      }
    }
  }
  // per-warp partials to shared memory
  if constexpr (MMA) {
    const int g = lane >> 2, t = lane & 3;
    red[warp][g * 8 + 2 * t] = s1[0][0];
    red[warp][g * 8 + 2 * t + 1] = s1[1][0];
    red[warp][64 + g * 8 + 2 * t] = s2[0][0];
    red[warp][64 + g * 8 + 2 * t + 1] = s2[1][0];
    float e = er[0];
    e += __shfl_xor_sync(0xffffffffu, e, 1);
    e += __shfl_xor_sync(0xffffffffu, e, 2);
    if (t == 0) rede[warp][g] = e;
  } else {
#pragma unroll
    for (int i = 0; i < RP; ++i) {
#pragma unroll
      for (int k = 0; k < RP; ++k) {
        const double a = k >= i ? warp_sum_d(s1[i][k]) : 0.0;
        const double b = k >= i ? warp_sum_d(s2[i][k]) : 0.0;
        if (lane == 0) {
          red[warp][i * RP + k] = a;
          red[warp][X::PART + i * RP + k] = b;
        }
      }
      const float e = warp_sum(er[i]);
      if (lane == 0) rede[warp][i] = e;
    }
  }
  __syncthreads();
  // M_t back to global memory, and the W slice into the space G used
  if (tid == 0 && have) {
    fence_proxy_async();
    const uint32_t em = (uint32_t)nc * (uint32_t)sizeof(TM);
    if (!q.tall) {
      for (int i = 0; i < RP; ++i) bulk_store(Mg + (int64_t)i * n + c0, Ms + (size_t)i * sl.pm, em);
    } else {
      bulk_store(Mg + c0 * RP, Ms, RP * em);
    }
    bulk_commit();
    const uint32_t ew = (uint32_t)nc * (uint32_t)sizeof(TW);
    mbar_arrive_expect_tx(&bar_w, RP * ew);
    if (!q.tall) {
      for (int i = 0; i < RP; ++i) bulk_load(Ws + (size_t)i * sl.pw, Wg + (int64_t)i * n + c0, ew, &bar_w);
    } else {
      bulk_load(Ws, Wg + c0 * RP, RP * ew, &bar_w);
    }
  }
  // ---- 3. the cluster's partials meet in the first CTA --------------------
  __syncwarp();
  cluster_wait();
  const uint32_t slot = mapa_shared(smem_u32(xch + (size_t)rank * X::WORDS), 0);
  for (int idx = tid; idx < X::WORDS; idx += CT) {
    double v;
    if (idx < 2 * X::PART) {
      v = 0.0;
#pragma unroll
      for (int w = 0; w < CW; ++w) v += red[w][idx];
    } else if (idx < 2 * X::PART + RP) {
      float e = 0.f;
#pragma unroll
      for (int w = 0; w < CW; ++w) e += rede[w][idx - 2 * X::PART];
      v = (double)e;
    } else {
      v = have ? 0.0 : 1.0;
    }
    st_cluster_f64(slot + 8u * (uint32_t)idx, v);
  }
  __syncwarp();
  cluster_arrive();
  cluster_wait();
  // every CTA sums the slots in rank order and iterates itself
  if (warp == 0) {
    const uint32_t xch0 = mapa_shared(smem_u32(xch), 0);
    auto rd = [&](int r, int idx) -> double {
      return ld_cluster_f64(xch0 + 8u * (uint32_t)(r * X::WORDS + idx));
    };
    for (int idx = lane; idx < RP * RP; idx += 32) {
      const int i = idx / RP, j = idx % RP;
      int src;
      if constexpr (MMA) {
        src = i * 8 + j;
      } else {
        src = i <= j ? i * RP + j : j * RP + i;
      }
      double g1 = 0.0, g2 = 0.0;
      for (int r = 0; r < CS; ++r) {
        g1 += rd(r, src);
        g2 += rd(r, X::PART + src);
      }
      it.G[i][j] = g1;
      it.H[i][j] = g2;
    }
    int bad = 0;
    float er_new = 0.f;
    for (int r = 0; r < CS; ++r) {
      bad |= rd(r, X::WORDS - 1) != 0.0;
      if (lane < RP) er_new += (float)rd(r, 2 * X::PART + lane);
    }
    __syncwarp();
    cluster_arrive();  // done with the first CTA's slots
    IterIn in;
    in.sc = sc;
    in.sr = sr;
    in.cond = q.cond;
    in.r = RP;
    in.e_r = erp;
    in.eps = p.eps;
    in.coef = p.coef;
    in.ns_steps = p.ns_steps;
    in.kappa = mt.kappa;
    in.status = rank == 0 ? p.status : nullptr;
    bool on_it;
    const double factor = iterate_gram_warp<RP>(in, it, &on_it);
    for (int idx = lane; idx < RP * RP; idx += 32) {
      const int i = idx / RP, j = idx % RP;
      Tsm[i][j] = factor * it.R[i] * it.P[i][j] * it.R[j];
    }
    // the new short-side energies (the previous ones were read at the start
    // by every CTA of the cluster, before the barrier)
    if (rank == 0 && !bad && q.cond && lane < RP) q.e_r[lane] = er_new;
    if (lane == 0) {
      flag_sh[1] = bad ? 0 : 1;
      // a degenerate norm: O = 0 exactly (W only decayed), even where the
      // momentum is not finite
      flag_sh[2] = factor == 0.0 ? 1 : 0;
    }
  } else {
    cluster_arrive();
  }
  __syncthreads();
  const bool write = flag_sh[1] != 0;
  const bool zero = flag_sh[2] != 0;

  // ---- 4. pass 2: O = C^2 T B, W, long-side energies ---------------------
  bool have_w = false;
  if (write) {
    if (tid == 0) flag_sh[0] = wait_bar(&bar_w, 0, p.status) ? 1 : 0;
    __syncthreads();
    have_w = flag_sh[0] != 0;
  }
  const float lr = p.lr, decay = p.decay;
  if (have_w) {
    if constexpr (MMA) {
      // warp w: groups of eight columns; lane (g, t) supplies T[g][4 kb + t]
      // and X[4 kb + t][column g], and gets O[g][2 t], O[g][2 t + 1]
      const int g = lane >> 2, t = lane & 3;
      double ta[2];
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) ta[kb] = Tsm[g][4 * kb + t];
      for (int cg = warp; cg < nc / 8; cg += CW) {
        const int jc = 8 * cg + g;  // the column this lane supplies
        const double w = on ? (double)col_weight(Es[jc], inv_mc, eps) : 1.0;
        double d0 = 0.0, d1 = 0.0;
        float sq = 0.f;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          const int row = 4 * kb + t;
          const float m = Ty<TM>::ld(Ms + mi(row, jc));
          sq = fmaf(m, m, sq);
          const double b = nest ? fma((double)mu, (double)m, (double)Ty<TG>::ld(Gs + gi(row, jc))) : (double)m;
          dmma(d0, d1, ta[kb], w * b);
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        sq += __shfl_xor_sync(0xffffffffu, sq, 2);
        if (q.cond && t == 0) q.e_c[c0 + jc] = sq;
        const double o[2] = {d0, d1};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = 8 * cg + 2 * t + e;
          const float ov = zero ? 0.f : (float)o[e];
          TW* wp = Ws + wi(g, j);
          Ty<TW>::st(wp, decay * Ty<TW>::ld(wp) - lr * ov);
          if (mt.upd) mt.upd[q.tall ? (c0 + j) * RP + g : (int64_t)g * n + c0 + j] = ov;
        }
      }
    } else {
      double tm[RP][RP];
#pragma unroll
      for (int i = 0; i < RP; ++i)
#pragma unroll
        for (int k = 0; k < RP; ++k) tm[i][k] = Tsm[i][k];
      for (int j = tid; j < nc; j += CT) {
        const double w = on ? (double)col_weight(Es[j], inv_mc, eps) : 1.0;
        double x[RP];
        float sq = 0.f;
#pragma unroll
        for (int k = 0; k < RP; ++k) {
          const float m = Ty<TM>::ld(Ms + mi(k, j));
          sq = fmaf(m, m, sq);
          x[k] = w * (nest ? fma((double)mu, (double)m, (double)Ty<TG>::ld(Gs + gi(k, j))) : (double)m);
        }
        if (q.cond) q.e_c[c0 + j] = sq;
#pragma unroll
        for (int i = 0; i < RP; ++i) {
          double y = 0.0;
#pragma unroll
          for (int k = 0; k < RP; ++k) y = fma(tm[i][k], x[k], y);
          const float ov = zero ? 0.f : (float)y;
          TW* wp = Ws + wi(i, j);
          Ty<TW>::st(wp, decay * Ty<TW>::ld(wp) - lr * ov);
          if (mt.upd) mt.upd[q.tall ? (c0 + j) * RP + i : (int64_t)i * n + c0 + j] = ov;
        }
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    if (have_w) {
      fence_proxy_async();
      const uint32_t ew = (uint32_t)nc * (uint32_t)sizeof(TW);
      if (!q.tall) {
        for (int i = 0; i < RP; ++i) bulk_store(Wg + (int64_t)i * n + c0, Ws + (size_t)i * sl.pw, ew);
      } else {
        bulk_store(Wg + c0 * RP, Ws, RP * ew);
      }
      bulk_commit();
    } else if (have) {
      // W was fetched but is not written (timeout, or a peer had no data):
      // let the copy land before the CTA ends
      mbar_wait_drain(&bar_w, 0, DRAIN_NS);
    }
    bulk_wait_read();  // the stores have read their shared-memory sources
  }
  __syncwarp();
  cluster_wait();  // the first CTA's slots stay until all have read them
}

template <int RP, typename TG, typename TM, typename TW>
cudaError_t launch_cl(const ThinClusterParams& p, int cs, size_t smem, cudaStream_t st) {
  static DeviceOnce once;
  cudaError_t e = device_once(once, nullptr, [](int) {
    cudaError_t e = cudaFuncSetAttribute(thin_cluster<RP, TG, TM, TW>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)THIN_CL_MAX_SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(thin_cluster<RP, TG, TM, TW>,
                               cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return e;
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.count * cs), 1, 1);
  cfg.blockDim = dim3(CT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, thin_cluster<RP, TG, TM, TW>, p);
}

template <typename TG, typename TM, typename TW>
size_t smem_of(int pad, int cs, int64_t n, bool tall, bool nest) {
  const int nc = (int)(n / cs);
  switch (pad) {
    case 2: return xch_bytes<2>(cs) + Slice<2, TG, TM, TW>::make(nc, tall, nest).bytes;
    case 4: return xch_bytes<4>(cs) + Slice<4, TG, TM, TW>::make(nc, tall, nest).bytes;
    default: return xch_bytes<8>(cs) + Slice<8, TG, TM, TW>::make(nc, tall, nest).bytes;
  }
}

template <typename TG, typename TM, typename TW>
cudaError_t launch_types(const ThinClusterParams& p, int pad, int cs, size_t smem, cudaStream_t st) {
  switch (pad) {
    case 2: return launch_cl<2, TG, TM, TW>(p, cs, smem, st);
    case 4: return launch_cl<4, TG, TM, TW>(p, cs, smem, st);
    default: return launch_cl<8, TG, TM, TW>(p, cs, smem, st);
  }
}

}  // namespace

size_t thin_cluster_smem(int pad, int combo, int cs, int64_t n, bool tall, bool nest) {
  using bf = __nv_bfloat16;
  if (pad != 2 && pad != 4 && pad != 8) return 0;
  if (cs < 1 || cs > THIN_CL_MAX_CS || n % (8 * cs) != 0) return 0;
  switch (combo) {
    case 0: return smem_of<bf, float, bf>(pad, cs, n, tall, nest);
    case 1: return smem_of<bf, bf, bf>(pad, cs, n, tall, nest);
    case 2: return smem_of<float, float, float>(pad, cs, n, tall, nest);
    default: return 0;
  }
}

cudaError_t launch_thin_cluster(const ThinClusterParams& p, int pad, int combo, int cs, size_t smem,
                                cudaStream_t s) {
  if (p.count <= 0) return cudaSuccess;
  if (smem > THIN_CL_MAX_SMEM || cs < 1 || cs > THIN_CL_MAX_CS) return cudaErrorInvalidValue;
  using bf = __nv_bfloat16;
  switch (combo) {
    case 0: return launch_types<bf, float, bf>(p, pad, cs, smem, s);
    case 1: return launch_types<bf, bf, bf>(p, pad, cs, smem, s);
    case 2: return launch_types<float, float, float>(p, pad, cs, smem, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dm
