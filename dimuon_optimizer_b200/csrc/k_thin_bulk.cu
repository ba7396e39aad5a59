// Thin-factor streaming passes with shared-memory staging: the same
// arithmetic as thin_gram / thin_apply in k_thin.cu (Gram route, see there),
// for factors whose short side r equals the padded rank RP, whose long side
// is a multiple of 8 and whose buffers are 16-byte aligned, in one of the
// storage combinations (G, M, W) = (bf16, fp32, bf16), (bf16, bf16, bf16),
// (fp32, fp32, fp32).
//
// One producer warp per CTA takes slabs from the device counter and streams
// each slab through a ring of shared-memory stages with 1-D bulk async copies
// (cp.async.bulk, completion on an mbarrier): the copies of the next stages
// are in flight while four consumer warps work on the current one, so the
// loads need neither registers nor per-lane address arithmetic.  Consumers
// write their results (M_t, W, O, energies) straight to global memory.  Every
// wait is bounded; the slab-end reduction of the Gram partials synchronises
// the consumer warps through mbarriers, so a timeout can never leave a warp
// stuck at a hardware barrier.
#include <algorithm>

#include "dm_common.cuh"
#include "dm_sm100.cuh"
#include "dm_thin.cuh"

namespace dm {
namespace {

using namespace thin;
using namespace sm100;

constexpr int BT = 160;          // 4 consumer warps + 1 producer warp
constexpr int CW = 4;            // consumer warps
constexpr int ROWPAD = 64;       // bytes after each staged wide row (bank shift)
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;

// Element types of the staged operands.
template <typename T>
struct El;
template <>
struct El<float> {
  static constexpr int DT = DT_FP32;
  __device__ static float ld1(const float* p) { return *p; }
  __device__ static void ld2(const float* p, float& a, float& b) {
    const float2 f = *reinterpret_cast<const float2*>(p);
    a = f.x;
    b = f.y;
  }
  __device__ static void ld4(const float* p, float v[4]) {
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
  __device__ static void st1(float* p, float v) { *p = v; }
  __device__ static void st2(float* p, float a, float b) {
    *reinterpret_cast<float2*>(p) = make_float2(a, b);
  }
  __device__ static void st4(float* p, const float v[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <>
struct El<__nv_bfloat16> {
  using T = __nv_bfloat16;
  static constexpr int DT = DT_BF16;
  __device__ static float ld1(const T* p) { return __bfloat162float(*p); }
  __device__ static void ld2(const T* p, float& a, float& b) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    a = f.x;
    b = f.y;
  }
  __device__ static void ld4(const T* p, float v[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
  __device__ static void st1(T* p, float v) { *p = __float2bfloat16_rn(v); }
  __device__ static void st2(T* p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(a, b);
  }
  __device__ static void st4(T* p, const float v[4]) {
    uint2 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
    h[0] = __floats2bfloat162_rn(v[0], v[1]);
    h[1] = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = u;
  }
};

// Per-stage description written by the producer before it arms the stage.
struct StageInfo {
  ThinMat mt;
  int u, f, c0, c1;  // slab, factor, long-side columns [c0, c1)
  int first, last;   // first / last stage of the slab
  int on, zero;      // Dimuon conditioning on; zero update (apply pass)
  float inv_mc;      // n / sum of the previous long-side energies
  int pad_;
};

// Staged bytes of one operand: RP wide rows of CH elements at a padded pitch,
// or CH tall columns of RP elements back to back.
template <typename T>
__host__ __device__ constexpr int opnd_bytes(int rp, int ch) {
  return rp * (ch * (int)sizeof(T) + ROWPAD);
}
template <typename T>
__host__ __device__ constexpr int pitch_elems(int ch) {
  return ch + ROWPAD / (int)sizeof(T);
}

__device__ __forceinline__ void drain_stages(uint64_t* full, int ns, uint32_t armed,
                                             uint32_t armed_par) {
  for (int s = 0; s < ns; ++s)
    if (armed & (1u << s)) mbar_wait_drain(&full[s], (armed_par >> s) & 1u, DRAIN_NS);
}

// ---------------------------------------------------------------------------
// Producer: slabs from the counter, stages through the ring.  `kind` 0 =
// gram pass (M, G, E), 1 = apply pass (M, G under Nesterov, W, E).
// ---------------------------------------------------------------------------
template <int RP, int CH, int NS, typename TG, typename TM, typename TW, int KIND>
__device__ void produce(const ThinParams& p, uint8_t* stages, int stage_bytes, int offG, int offW,
                        int offE, StageInfo* info, uint64_t* full, uint64_t* empty,
                        volatile int* abort, int* counter) {
  const int lane = threadIdx.x & 31;
  int stage = 0;
  uint32_t ph = 0, armed = 0, armed_par = 0;
  bool ok = true;
  const int slab_cols = TCfg<RP>::SLAB;
  for (;;) {
    int u = 0;
    if (lane == 0) u = atomicAdd(counter, 1);
    u = __shfl_sync(0xffffffffu, u, 0);
    if (u >= p.units) break;
    const int f = p.unit_f[u];
    const int64_t c_lo = (int64_t)(u - p.starts[f]) * slab_cols;
    // per-slab values, lane 0 only
    ThinMat mt;
    Geo q;
    int64_t c_hi = 0;
    int on = 0, zero = 0;
    float inv_mc = 0.f;
    if (lane == 0) {
      mt = p.mats[f];
      q = geometry(mt, p.conditioned);
      c_hi = min(q.n, c_lo + slab_cols);
      if (KIND == 0) {
        on = q.cond && p.fsc[4 * f] > 0.0 && p.fsc[4 * f + 1] > 0.0;
      } else {
        on = p.fsc[4 * f + 2] != 0.0;
        zero = p.fsc[4 * f + 3] != 0.0;
      }
      inv_mc = on ? (float)((double)q.n / p.fsc[4 * f]) : 0.f;
    }
    for (int64_t c0 = c_lo;; c0 += CH) {
      int go = 1;
      if (lane == 0) {
        if (c0 >= c_hi) {
          go = 0;
        } else if (!mbar_wait_bounded(&empty[stage], ph ^ 1, abort, p.status, WAIT_NS)) {
          go = -1;
        } else {
          StageInfo& si = info[stage];
          si.mt = mt;
          si.u = u;
          si.f = f;
          si.c0 = (int)c0;
          si.c1 = (int)min(c0 + CH, c_hi);
          si.first = c0 == c_lo;
          si.last = si.c1 == c_hi;
          si.on = on;
          si.zero = zero;
          si.inv_mc = inv_mc;
          const int w = si.c1 - si.c0;
          uint32_t bytes = (uint32_t)(RP * w) * (uint32_t)sizeof(TM);
          if (KIND == 0 || p.nesterov) bytes += (uint32_t)(RP * w) * (uint32_t)sizeof(TG);
          if (KIND == 1) bytes += (uint32_t)(RP * w) * (uint32_t)sizeof(TW);
          if (si.on) bytes += (uint32_t)w * 4u;
          mbar_arrive_expect_tx(&full[stage], bytes);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (ph << stage);
        }
      }
      go = __shfl_sync(0xffffffffu, go, 0);
      if (go == 0) break;
      if (go < 0) {
        ok = false;
        break;
      }
      __syncwarp();
      // copies: lane i takes short-side row i (wide) or the whole run (tall)
      const StageInfo& si = info[stage];
      const Geo qs = geometry(si.mt, p.conditioned);
      const int w = si.c1 - si.c0;
      uint8_t* base = stages + (size_t)stage * stage_bytes;
      if (!qs.tall) {
        for (int i = lane; i < RP; i += 32) {
          const int64_t g0 = (int64_t)i * qs.n + si.c0;
          bulk_load(base + i * (CH * (int)sizeof(TM) + ROWPAD),
                    reinterpret_cast<const TM*>(si.mt.M) + g0, (uint32_t)(w * sizeof(TM)), &full[stage]);
          if (KIND == 0 || p.nesterov)
            bulk_load(base + offG + i * (CH * (int)sizeof(TG) + ROWPAD),
                      reinterpret_cast<const TG*>(si.mt.G) + g0, (uint32_t)(w * sizeof(TG)),
                      &full[stage]);
          if (KIND == 1)
            bulk_load(base + offW + i * (CH * (int)sizeof(TW) + ROWPAD),
                      reinterpret_cast<const TW*>(si.mt.W) + g0, (uint32_t)(w * sizeof(TW)),
                      &full[stage]);
        }
      } else if (lane == 0) {
        const int64_t g0 = (int64_t)si.c0 * RP;
        bulk_load(base, reinterpret_cast<const TM*>(si.mt.M) + g0, (uint32_t)(w * RP * sizeof(TM)),
                  &full[stage]);
        if (KIND == 0 || p.nesterov)
          bulk_load(base + offG, reinterpret_cast<const TG*>(si.mt.G) + g0,
                    (uint32_t)(w * RP * sizeof(TG)), &full[stage]);
        if (KIND == 1)
          bulk_load(base + offW, reinterpret_cast<const TW*>(si.mt.W) + g0,
                    (uint32_t)(w * RP * sizeof(TW)), &full[stage]);
      }
      if (si.on && lane == 1)
        bulk_load(base + offE, qs.e_c + si.c0, (uint32_t)(w * 4), &full[stage]);
      if (++stage == NS) {
        stage = 0;
        ph ^= 1;
      }
    }
    if (!ok) break;
  }
  if (lane == 0) {
    if (ok && mbar_wait_bounded(&empty[stage], ph ^ 1, abort, p.status, WAIT_NS)) {
      info[stage].u = -1;  // end of the work
      mbar_arrive(&full[stage]);
    }
    if (*abort) drain_stages(full, NS, armed, armed_par);
  }
}

// ===========================================================================
// thin_gram_bulk
// ===========================================================================
template <int RP, typename TG, typename TM>
struct GramBulk {
  static constexpr int CH = 2048 / RP;
  static constexpr int NS = 4;
  static constexpr int OFF_G = opnd_bytes<TM>(RP, CH);
  static constexpr int OFF_E = OFF_G + opnd_bytes<TG>(RP, CH);
  static constexpr int STAGE_BYTES = (OFF_E + CH * 4 + 127) / 128 * 128;
  static constexpr int RED_BYTES = CW * 2 * TCfg<RP>::PART * 8 + CW * RP * 4;
  static constexpr int SMEM = NS * STAGE_BYTES + NS * (int)sizeof(StageInfo) +
                              (2 * NS + 2) * 8 + 16 + RED_BYTES + 128;
};

template <int RP, typename TG, typename TM>
__global__ void __launch_bounds__(BT) thin_gram_bulk(const __grid_constant__ ThinParams p) {
  using L = GramBulk<RP, TG, TM>;
  using Cf = TCfg<RP>;
  constexpr int CH = L::CH, NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  uint8_t* stages = smem;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + NS * L::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(info + NS);
  uint64_t* empty = full + NS;
  uint64_t* redf = empty + NS;  // consumer warps wrote their partials
  uint64_t* redr = redf + 1;    // consumer warps read the partials
  volatile int* abort = reinterpret_cast<volatile int*>(redr + 1);
  double* red_s = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(redr + 1) + 16);
  float* red_e = reinterpret_cast<float*>(red_s + CW * 2 * Cf::PART);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    mbar_init(redf, CW);
    mbar_init(redr, CW);
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == CW) {
    produce<RP, CH, NS, TG, TM, TM, 0>(p, stages, L::STAGE_BYTES, L::OFF_G, 0, L::OFF_E, info, full,
                                       empty, abort, p.counters);
    return;
  }

  // ------------------------------- consumers -------------------------------
  const float mu = p.mu, eps = p.eps;
  constexpr int PM = pitch_elems<TM>(CH), PG = pitch_elems<TG>(CH);
  constexpr int NB = Cf::NB, NUB = Cf::NUB;
  constexpr int ROWS = Cf::MMA ? NB : RP;
  double s1[Cf::MMA ? NUB : RP][Cf::MMA ? 2 : RP], s2[Cf::MMA ? NUB : RP][Cf::MMA ? 2 : RP];
  float er[ROWS];
  int stage = 0;
  uint32_t ph = 0, nred = 0;
  for (;;) {
    if (!mbar_wait_bounded(&full[stage], ph, abort, p.status, WAIT_NS)) break;
    const StageInfo& si = info[stage];
    const int u = si.u;
    if (u < 0) break;
    const int c0 = si.c0, c1 = si.c1, first = si.first, last = si.last;
    const bool on = si.on != 0;
    const float inv_mc = si.inv_mc;
    const bool tall = si.mt.rows > si.mt.cols;
    const int64_t n = tall ? si.mt.rows : si.mt.cols;
    TM* Mg = reinterpret_cast<TM*>(si.mt.M);
    const bool cond = p.conditioned && si.mt.e_row != nullptr;
    const uint8_t* base = stages + (size_t)stage * L::STAGE_BYTES;
    const TM* Ms = reinterpret_cast<const TM*>(base);
    const TG* Gs = reinterpret_cast<const TG*>(base + L::OFF_G);
    const float* Es = reinterpret_cast<const float*>(base + L::OFF_E);
    if (first) {
#pragma unroll
      for (int a = 0; a < (Cf::MMA ? NUB : RP); ++a)
#pragma unroll
        for (int b = 0; b < (Cf::MMA ? 2 : RP); ++b) s1[a][b] = s2[a][b] = 0.0;
#pragma unroll
      for (int a = 0; a < ROWS; ++a) er[a] = 0.f;
    }

    if constexpr (Cf::MMA) {
      const int g = lane >> 2, t = lane & 3;
      // 16 columns per warp step: wide lane (g, t) at c + 4t + e, tall c + t + 4e
      for (int c = c0 + 16 * warp; c < c1; c += 16 * CW) {
        const int cs = c - c0;
        float mv[NB][4], gv[NB][4], ev[4];
        bool okc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = tall ? c + t + 4 * e : c + 4 * t + e;
          okc[e] = col < c1;
          ev[e] = (on && okc[e]) ? Es[col - c0] : 0.f;
        }
        if (!tall) {
          const bool ok = c + 4 * t < c1;  // (c1 - c0) is a multiple of 8
#pragma unroll
          for (int blk = 0; blk < NB; ++blk) {
            const int row = g + 8 * blk;
            if (ok) {
              El<TM>::ld4(Ms + row * PM + cs + 4 * t, mv[blk]);
              El<TG>::ld4(Gs + row * PG + cs + 4 * t, gv[blk]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) mv[blk][e] = gv[blk][e] = 0.f;
            }
          }
        } else {
#pragma unroll
          for (int blk = 0; blk < NB; ++blk)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int o = (cs + t + 4 * e) * RP + g + 8 * blk;
              mv[blk][e] = okc[e] ? El<TM>::ld1(Ms + o) : 0.f;
              gv[blk][e] = okc[e] ? El<TG>::ld1(Gs + o) : 0.f;
            }
        }
        double bx[NB][4];
#pragma unroll
        for (int blk = 0; blk < NB; ++blk)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float m = momentum_value(mu, mv[blk][e], gv[blk][e], El<TM>::DT);
            mv[blk][e] = m;
            bx[blk][e] = p.nesterov ? fma((double)mu, (double)m, (double)gv[blk][e]) : (double)m;
            er[blk] = fmaf(m, m, er[blk]);
          }
        if (!tall) {
          if (c + 4 * t < c1)
#pragma unroll
            for (int blk = 0; blk < NB; ++blk)
              El<TM>::st4(Mg + (int64_t)(g + 8 * blk) * n + c + 4 * t, mv[blk]);
        } else {
#pragma unroll
          for (int blk = 0; blk < NB; ++blk)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (okc[e]) El<TM>::st1(Mg + (int64_t)(c + t + 4 * e) * RP + g + 8 * blk, mv[blk][e]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double w = on ? (okc[e] ? (double)col_weight(ev[e], inv_mc, eps) : 0.0) : 1.0;
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
      }
    } else {
      // RP == r <= 4: lane owns columns c .. c + 3 (c1 - c0 is a multiple of 8)
      for (int c = c0 + 4 * (lane + 32 * warp); c < c1; c += 4 * 32 * CW) {
        const int cs = c - c0;
        float mv[RP][4], gv[RP][4], ev[4];
        if (!tall) {
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            El<TM>::ld4(Ms + i * PM + cs, mv[i]);
            El<TG>::ld4(Gs + i * PG + cs, gv[i]);
          }
        } else {
          float fm[4 * RP], fg[4 * RP];
#pragma unroll
          for (int s = 0; s < RP; ++s) {
            El<TM>::ld4(Ms + cs * RP + 4 * s, &fm[4 * s]);
            El<TG>::ld4(Gs + cs * RP + 4 * s, &fg[4 * s]);
          }
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              mv[i][e] = fm[e * RP + i];
              gv[i][e] = fg[e * RP + i];
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) ev[e] = on ? Es[cs + e] : 0.f;
        double bx[RP][4];
#pragma unroll
        for (int i = 0; i < RP; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float m = momentum_value(mu, mv[i][e], gv[i][e], El<TM>::DT);
            mv[i][e] = m;
            bx[i][e] = p.nesterov ? fma((double)mu, (double)m, (double)gv[i][e]) : (double)m;
            er[i] = fmaf(m, m, er[i]);
          }
        if (!tall) {
#pragma unroll
          for (int i = 0; i < RP; ++i) El<TM>::st4(Mg + (int64_t)i * n + c, mv[i]);
        } else {
          float fm[4 * RP];
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) fm[e * RP + i] = mv[i][e];
#pragma unroll
          for (int s = 0; s < RP; ++s) El<TM>::st4(Mg + (int64_t)c * RP + 4 * s, &fm[4 * s]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double w = on ? (double)col_weight(ev[e], inv_mc, eps) : 1.0;
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int k = i; k < RP; ++k) {
              const double xk = w * bx[k][e];
              s1[i][k] = fma(bx[i][e], xk, s1[i][k]);
              if (on) s2[i][k] = fma(bx[i][e], w * xk, s2[i][k]);
            }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage
    if (++stage == NS) {
      stage = 0;
      ph ^= 1;
    }

    if (last) {
      // slab-end reduction over the consumer warps (mbarrier-synchronised)
      if (!mbar_wait_bounded(redr, (nred & 1u) ^ 1u, abort, p.status, WAIT_NS)) break;
      double* mine = red_s + warp * 2 * Cf::PART;
      if constexpr (Cf::MMA) {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int ub = 0; ub < NUB; ++ub)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            mine[ub * 64 + g * 8 + 2 * t + h] = s1[ub][h];
            mine[Cf::PART + ub * 64 + g * 8 + 2 * t + h] = s2[ub][h];
          }
#pragma unroll
        for (int blk = 0; blk < NB; ++blk) {
          float e = er[blk];
          e += __shfl_xor_sync(0xffffffffu, e, 1);
          e += __shfl_xor_sync(0xffffffffu, e, 2);
          if (t == 0) red_e[warp * RP + g + 8 * blk] = e;
        }
      } else {
#pragma unroll
        for (int i = 0; i < RP; ++i) {
#pragma unroll
          for (int k = i; k < RP; ++k) {
            const double a = warp_sum_d(s1[i][k]), b = warp_sum_d(s2[i][k]);
            if (lane == 0) {
              mine[i * RP + k] = mine[k * RP + i] = a;
              mine[Cf::PART + i * RP + k] = mine[Cf::PART + k * RP + i] = b;
            }
          }
          const float e = warp_sum(er[i]);
          if (lane == 0) red_e[warp * RP + i] = e;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(redf);
      if (!mbar_wait_bounded(redf, nred & 1u, abort, p.status, WAIT_NS)) break;
      double* dst = p.part + (size_t)u * 2 * Cf::PART;
      for (int i = tid; i < 2 * Cf::PART; i += 32 * CW) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < CW; ++w) s += red_s[w * 2 * Cf::PART + i];
        dst[i] = s;
      }
      if (cond)
        for (int i = tid; i < RP; i += 32 * CW) {
          float s = 0.f;
#pragma unroll
          for (int w = 0; w < CW; ++w) s += red_e[w * RP + i];
          p.rpart[(size_t)u * RP + i] = s;
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(redr);
      ++nred;
    }
  }
}

// ===========================================================================
// thin_apply_bulk
// ===========================================================================
template <int RP, typename TG, typename TM, typename TW>
struct ApplyBulk {
  static constexpr int CH = (RP >= 32 ? 4096 : 2048) / RP;
  static constexpr int NS = 3;
  static constexpr int OFF_W = opnd_bytes<TM>(RP, CH);
  static constexpr int OFF_E = OFF_W + opnd_bytes<TW>(RP, CH);
  static constexpr int OFF_G = OFF_E + CH * 4;  // Nesterov only
  static constexpr int BYTES_NO_G = (OFF_G + 127) / 128 * 128;
  static constexpr int BYTES_G = (OFF_G + opnd_bytes<TG>(RP, CH) + 127) / 128 * 128;
  __host__ __device__ static constexpr int stage_bytes(bool nest) { return nest ? BYTES_G : BYTES_NO_G; }
  __host__ __device__ static constexpr int smem(bool nest) {
    return NS * stage_bytes(nest) + NS * (int)sizeof(StageInfo) + 2 * NS * 8 + 16 + 128;
  }
};

template <int RP, typename TG, typename TM, typename TW>
__global__ void __launch_bounds__(BT) thin_apply_bulk(const __grid_constant__ ThinParams p) {
  using L = ApplyBulk<RP, TG, TM, TW>;
  using Cf = TCfg<RP>;
  constexpr int CH = L::CH, NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  const int stage_bytes = L::stage_bytes(p.nesterov != 0);
  uint8_t* stages = smem;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + NS * stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(info + NS);
  uint64_t* empty = full + NS;
  volatile int* abort = reinterpret_cast<volatile int*>(empty + NS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    *abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == CW) {
    produce<RP, CH, NS, TG, TM, TW, 1>(p, stages, stage_bytes, L::OFF_G, L::OFF_W, L::OFF_E, info, full,
                                       empty, abort, p.counters + 1);
    return;
  }

  const float mu = p.mu, lr = p.lr, decay = p.decay, eps = p.eps;
  const bool nest = p.nesterov != 0;
  constexpr int PM = pitch_elems<TM>(CH), PG = pitch_elems<TG>(CH), PW = pitch_elems<TW>(CH);
  int stage = 0;
  uint32_t ph = 0;
  for (;;) {
    if (!mbar_wait_bounded(&full[stage], ph, abort, p.status, WAIT_NS)) break;
    const StageInfo& si = info[stage];
    if (si.u < 0) break;
    const int c0 = si.c0, c1 = si.c1, f = si.f;
    const bool on = si.on != 0, zero = si.zero != 0;
    const float inv_mc = si.inv_mc;
    const bool tall = si.mt.rows > si.mt.cols;
    const int64_t n = tall ? si.mt.rows : si.mt.cols;
    TW* Wg = reinterpret_cast<TW*>(si.mt.W);
    float* Ug = si.mt.upd;
    float* ecg = tall ? si.mt.e_row : si.mt.e_col;
    const bool cond = p.conditioned && ecg != nullptr;
    const uint8_t* base = stages + (size_t)stage * stage_bytes;
    const TM* Ms = reinterpret_cast<const TM*>(base);
    const TW* Ws = reinterpret_cast<const TW*>(base + L::OFF_W);
    const float* Es = reinterpret_cast<const float*>(base + L::OFF_E);
    const TG* Gs = reinterpret_cast<const TG*>(base + L::OFF_G);
    const double* Tg = p.T + (size_t)f * RP * RP;

    if constexpr (Cf::MMA) {
      constexpr int NB = Cf::NB, KB = Cf::KB;
      const int g = lane >> 2, t = lane & 3;
      // 32 columns per warp step; see thin_apply for the fragment layout
      for (int c = c0 + 32 * warp; c < c1; c += 32 * CW) {
        const int cs = c - c0;
        float mv[KB][4], gv[KB][4];
        bool okc[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) okc[e] = (tall ? c + 8 * e + g : c + 4 * g + e) < c1;
        if (!tall) {
          const bool ok = c + 4 * g < c1;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const int row = 4 * kb + t;
            if (ok) {
              El<TM>::ld4(Ms + row * PM + cs + 4 * g, mv[kb]);
              if (nest) El<TG>::ld4(Gs + row * PG + cs + 4 * g, gv[kb]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) mv[kb][e] = gv[kb][e] = 0.f;
            }
          }
        } else {
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int o = (cs + 8 * e + g) * RP + 4 * kb + t;
              mv[kb][e] = okc[e] ? El<TM>::ld1(Ms + o) : 0.f;
              if (nest) gv[kb][e] = okc[e] ? El<TG>::ld1(Gs + o) : 0.f;
            }
        }
        float ce[4];
        double x[KB][4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = tall ? c + 8 * e + g : c + 4 * g + e;
          const double w =
              on ? (okc[e] ? (double)col_weight(Es[col - c0], inv_mc, eps) : 0.0) : 1.0;
          float sq = 0.f;
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const double m = (double)mv[kb][e];
            x[kb][e] = w * (nest ? fma((double)mu, m, (double)gv[kb][e]) : m);
            sq = fmaf(mv[kb][e], mv[kb][e], sq);
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
          for (int bo = 0; bo < NB; ++bo) tf[bo] = __ldg(Tg + (bo * KB + kb) * 32 + lane);
#pragma unroll
          for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int bo = 0; bo < NB; ++bo) {
              if (tall)
                dmma(acc[bo][e][0], acc[bo][e][1], x[kb][e], tf[bo]);
              else
                dmma(acc[bo][e][0], acc[bo][e][1], tf[bo], x[kb][e]);
            }
        }
        if (!tall) {
          // acc[bo][e][h] is column c + 8t + 4h + e of row 8 bo + g
#pragma unroll
          for (int bo = 0; bo < NB; ++bo)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int row = 8 * bo + g, col0 = c + 8 * t + 4 * h;
              if (col0 < c1) {
                float w4[4], o4[4];
                El<TW>::ld4(Ws + row * PW + (col0 - c0), w4);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  o4[e] = zero ? 0.f : (float)acc[bo][e][h];
                  w4[e] = decay * w4[e] - lr * o4[e];
                }
                El<TW>::st4(Wg + (int64_t)row * n + col0, w4);
                if (Ug) El<float>::st4(Ug + (int64_t)row * n + col0, o4);
              }
            }
        } else {
          // acc[bo][e][h] is row 8 bo + 2t + h of column c + 8e + g
#pragma unroll
          for (int bo = 0; bo < NB; ++bo)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (!okc[e]) continue;
              const int col = c + 8 * e + g, row0 = 8 * bo + 2 * t;
              float w0, w1;
              El<TW>::ld2(Ws + (col - c0) * RP + row0, w0, w1);
              const float o0 = zero ? 0.f : (float)acc[bo][e][0];
              const float o1 = zero ? 0.f : (float)acc[bo][e][1];
              El<TW>::st2(Wg + (int64_t)col * RP + row0, decay * w0 - lr * o0, decay * w1 - lr * o1);
              if (Ug) El<float>::st2(Ug + (int64_t)col * RP + row0, o0, o1);
            }
        }
        if (cond && t == 0)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = tall ? c + 8 * e + g : c + 4 * g + e;
            if (okc[e]) ecg[col] = ce[e];
          }
      }
    } else {
      // RP == r <= 4: lane owns columns c .. c + 3
      for (int c = c0 + 4 * (lane + 32 * warp); c < c1; c += 4 * 32 * CW) {
        const int cs = c - c0;
        float mv[RP][4], gv[RP][4], wv[RP][4];
        if (!tall) {
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            El<TM>::ld4(Ms + i * PM + cs, mv[i]);
            if (nest) El<TG>::ld4(Gs + i * PG + cs, gv[i]);
            El<TW>::ld4(Ws + i * PW + cs, wv[i]);
          }
        } else {
          float fm[4 * RP], fg[4 * RP], fw[4 * RP];
#pragma unroll
          for (int s = 0; s < RP; ++s) {
            El<TM>::ld4(Ms + cs * RP + 4 * s, &fm[4 * s]);
            if (nest) El<TG>::ld4(Gs + cs * RP + 4 * s, &fg[4 * s]);
            El<TW>::ld4(Ws + cs * RP + 4 * s, &fw[4 * s]);
          }
#pragma unroll
          for (int i = 0; i < RP; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              mv[i][e] = fm[e * RP + i];
              gv[i][e] = nest ? fg[e * RP + i] : 0.f;
              wv[i][e] = fw[e * RP + i];
            }
        }
        float ov[RP][4], ce[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double w = on ? (double)col_weight(Es[cs + e], inv_mc, eps) : 1.0;
          double x[RP];
          float sq = 0.f;
#pragma unroll
          for (int k = 0; k < RP; ++k) {
            const double m = (double)mv[k][e];
            x[k] = w * (nest ? fma((double)mu, m, (double)gv[k][e]) : m);
            sq = fmaf(mv[k][e], mv[k][e], sq);
          }
          ce[e] = sq;
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            double y = 0.0;
#pragma unroll
            for (int k = 0; k < RP; ++k) y = fma(__ldg(Tg + i * RP + k), x[k], y);
            ov[i][e] = zero ? 0.f : (float)y;
            wv[i][e] = decay * wv[i][e] - lr * ov[i][e];
          }
        }
        if (!tall) {
#pragma unroll
          for (int i = 0; i < RP; ++i) {
            El<TW>::st4(Wg + (int64_t)i * n + c, wv[i]);
            if (Ug) El<float>::st4(Ug + (int64_t)i * n + c, ov[i]);
          }
        } else {
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
            El<TW>::st4(Wg + (int64_t)c * RP + 4 * s, &fw[4 * s]);
            if (Ug) El<float>::st4(Ug + (int64_t)c * RP + 4 * s, &fo[4 * s]);
          }
        }
        if (cond) El<float>::st4(ecg + c, ce);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);
    if (++stage == NS) {
      stage = 0;
      ph ^= 1;
    }
  }
}

template <typename K>
int resident(K kernel, int threads, int smem) {
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) != cudaSuccess ||
      occ < 1)
    occ = 1;
  return occ;
}

template <int RP, typename TG, typename TM, typename TW>
cudaError_t launch_bulk_rp(ThinParams& p, int nsm, cudaStream_t st) {
  using LG = GramBulk<RP, TG, TM>;
  using LA = ApplyBulk<RP, TG, TM, TW>;
  static int configured = -1;
  static int occ_g = 1, occ_a[2] = {1, 1};
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured != dev) {
    cudaError_t e = cudaFuncSetAttribute(thin_gram_bulk<RP, TG, TM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, LG::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(thin_apply_bulk<RP, TG, TM, TW>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, LA::smem(true));
    if (e != cudaSuccess) return e;
    occ_g = resident(thin_gram_bulk<RP, TG, TM>, BT, LG::SMEM);
    occ_a[0] = resident(thin_apply_bulk<RP, TG, TM, TW>, BT, LA::smem(false));
    occ_a[1] = resident(thin_apply_bulk<RP, TG, TM, TW>, BT, LA::smem(true));
    configured = dev;
  }
  const bool nest = p.nesterov != 0;
  p.grid_gram = std::min(p.units, nsm * occ_g);
  p.grid_apply = std::min(p.units, nsm * occ_a[nest ? 1 : 0]);
  thin_gram_bulk<RP, TG, TM><<<p.grid_gram, BT, LG::SMEM, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_thin_iterate(p, st);
  if (e != cudaSuccess) return e;
  thin_apply_bulk<RP, TG, TM, TW><<<p.grid_apply, BT, LA::smem(nest), st>>>(p);
  return cudaGetLastError();
}

template <typename TG, typename TM, typename TW>
cudaError_t launch_bulk_types(ThinParams& p, int nsm, cudaStream_t st) {
  switch (p.pad) {
    case 2: return launch_bulk_rp<2, TG, TM, TW>(p, nsm, st);
    case 4: return launch_bulk_rp<4, TG, TM, TW>(p, nsm, st);
    case 8: return launch_bulk_rp<8, TG, TM, TW>(p, nsm, st);
    case 16: return launch_bulk_rp<16, TG, TM, TW>(p, nsm, st);
    default: return launch_bulk_rp<32, TG, TM, TW>(p, nsm, st);
  }
}

}  // namespace

// Storage combination code of the staged path, or -1 when it has none.
int thin_bulk_combo(int gdt, int mdt, int wdt) {
  if (gdt == DT_BF16 && mdt == DT_FP32 && wdt == DT_BF16) return 0;
  if (gdt == DT_BF16 && mdt == DT_BF16 && wdt == DT_BF16) return 1;
  if (gdt == DT_FP32 && mdt == DT_FP32 && wdt == DT_FP32) return 2;
  return -1;
}

cudaError_t launch_thin_bulk(ThinParams& p, int combo, int nsm, cudaStream_t s) {
  if (p.count <= 0 || p.units <= 0) return cudaSuccess;
  using bf = __nv_bfloat16;
  switch (combo) {
    case 0: return launch_bulk_types<bf, float, bf>(p, nsm, s);
    case 1: return launch_bulk_types<bf, bf, bf>(p, nsm, s);
    default: return launch_bulk_types<float, float, float>(p, nsm, s);
  }
}

}  // namespace dm
