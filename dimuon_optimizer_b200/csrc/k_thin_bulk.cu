// Thin-factor streaming passes with shared-memory staging: the same
// arithmetic as thin_gram / thin_apply in k_thin.cu (Gram route, see there),
// for factors whose short side r equals the padded rank RP, whose long side
// is a multiple of 8 (any length for tall factors with r >= 8, whose staged
// rows are whole 16-byte groups) and whose buffers are 16-byte aligned, in one of the
// storage combinations (G, M, W) = (bf16, fp32, bf16), (bf16, bf16, bf16),
// (fp32, fp32, fp32).
//
// Each CTA owns a contiguous range of slabs (balanced to within one slab).
// Two producer warps stream it through a ring of shared-memory stages, taking
// alternate stages, with 1-D bulk async copies (cp.async.bulk, completion on
// an mbarrier): the copies of the next stages are in flight while the
// consumer warps (8; 4 for r = 32, 6 for r = 32 on the split path) work on
// the current one, so the loads need neither registers nor per-lane address
// arithmetic.  Sums: fp64 (FMA for r <= 4, DMMA for r >= 8), or for r = 32 in
// bf16 tensor-core mode bf16 tensor-core products of hi / lo split operands
// with fp32 accumulation (the SP kernels).  Full steps run
// branch-free code specialised on the layout (wide / tall), on whether Dimuon
// conditioning is on and on whether energies are written; partial steps at a
// factor's end take a predicated version.  Consumers write their results
// (M_t, W, O, energies) straight to global memory.  The Gram accumulators
// live across a run of consecutive slabs of one factor and are reduced once
// per run.  Every wait is bounded; the run-end reduction synchronises the
// consumer warps through mbarriers, so a timeout can never leave a warp stuck
// at a hardware barrier.
#include <algorithm>

#include "dm_common.cuh"
#include "dm_sm100.cuh"
#include "dm_thin.cuh"

namespace dm {
namespace {

using namespace thin;
using namespace sm100;

constexpr int ROWPAD = 64;       // bytes after each staged wide row (bank shift)
constexpr uint64_t WAIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_NS = 200000000ull;

// Bounded wait on an mbarrier phase whose try_wait carries a suspend-time
// hint, so a waiting warp sleeps in the barrier unit instead of spinning
// through issue slots the working warps need.  Same contract as
// mbar_wait_bounded: false after an abort or after WAIT_NS (then the abort
// flag and the timeout status are set).
constexpr uint32_t SLEEP_NS = 20000;
__device__ __forceinline__ bool try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(SLEEP_NS)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool wait_phase(uint64_t* bar, uint32_t parity, volatile int* abort,
                                           int* status) {
  if (try_wait_sleep(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (try_wait_sleep(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > WAIT_NS) {
      *abort = 1;
      raise_timeout(status);
      return false;
    }
  }
}

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
  int first, last;   // first / last stage of a run of slabs of one factor in this CTA
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

// Per-slab values the producer needs (and hands to the consumers).
struct SlabMeta {
  ThinMat mt;
  int f;
  int on, zero;
  float inv_mc;
  int64_t c_lo, c_hi;
};

template <int RP, int KIND>
__device__ __forceinline__ SlabMeta slab_meta(const ThinParams& p, int u) {
  SlabMeta m;
  m.f = p.unit_f[u];
  m.mt = p.mats[m.f];
  const Geo q = geometry(m.mt, p.conditioned);
  m.c_lo = (int64_t)(u - p.starts[m.f]) * TCfg<RP>::SLAB;
  m.c_hi = min(q.n, m.c_lo + TCfg<RP>::SLAB);
  const double sc = p.fsc[4 * m.f];
  if (KIND == 0) {
    m.on = q.cond && sc > 0.0 && p.fsc[4 * m.f + 1] > 0.0;
    m.zero = 0;
  } else {
    m.on = p.fsc[4 * m.f + 2] != 0.0;
    m.zero = p.fsc[4 * m.f + 3] != 0.0;
  }
  m.inv_mc = m.on ? (float)((double)q.n / sc) : 0.f;
  return m;
}

// ---------------------------------------------------------------------------
// Producer: slabs blockIdx.x, blockIdx.x + gridDim.x, ... (the next slab's
// descriptor is loaded while the current slab's stages are issued), stages
// through the ring.  KIND 0 = gram pass (M, G, E), 1 = apply pass (M, G
// under Nesterov, W, E).
// ---------------------------------------------------------------------------
template <int RP, int CH, int NS, typename TG, typename TM, typename TW, int KIND>
__device__ void produce(const ThinParams& p, uint8_t* stages, int stage_bytes, int offG, int offW,
                        int offE, StageInfo* info, uint64_t* full, uint64_t* empty,
                        volatile int* abort, int pw, int np) {
  // np producer warps walk the same stage sequence; warp pw fills the
  // stages whose ring index is pw modulo np (one warp's copy issue rate is
  // far below what the memory system takes)
  const int lane = threadIdx.x & 31;
  int stage = 0;
  uint32_t ph = 0, armed = 0, armed_par = 0;
  bool ok = true;
  // contiguous slab range of this CTA (balanced to within one slab), so a
  // CTA's slabs of one factor are consecutive and the Gram partials of such
  // a run are reduced once
  const int q = p.units / (int)gridDim.x, rem = p.units % (int)gridDim.x;
  const int u_begin = (int)blockIdx.x * q + min((int)blockIdx.x, rem);
  const int u_end = u_begin + q + ((int)blockIdx.x < rem ? 1 : 0);
  int u = u_begin;
  int prev_f = -1;
  SlabMeta cur;
  // every lane holds the slab values, so the loop control below is warp-uniform
  if (u < u_end) cur = slab_meta<RP, KIND>(p, u);
  while (u < u_end && ok) {
    const int un = u + 1;
    SlabMeta nxt;
    if (un < u_end) nxt = slab_meta<RP, KIND>(p, un);
    const bool run_first = cur.f != prev_f;
    const bool run_last = un >= u_end || nxt.f != cur.f;
    if (KIND == 0 && !run_last && pw == 0) {
      // this slab's partial slot holds zeros: the run's sum goes to its last slab
      constexpr int PART = TCfg<RP>::PART;
      double* dst = p.part + (size_t)u * 2 * PART;
      for (int i = lane; i < 2 * PART; i += 32) dst[i] = 0.0;
      if (cur.mt.e_row != nullptr && p.conditioned)
        for (int i = lane; i < RP; i += 32) p.rpart[(size_t)u * RP + i] = 0.f;
    }
    for (int64_t c0 = cur.c_lo;; c0 += CH) {
      if (c0 >= cur.c_hi) break;
      if (stage % np != pw) {  // another producer warp's stage
        if (++stage == NS) {
          stage = 0;
          ph ^= 1;
        }
        continue;
      }
      int go = 1;
      if (lane == 0) {
        if (!wait_phase(&empty[stage], ph ^ 1, abort, p.status)) {
          go = -1;
        } else {
          StageInfo& si = info[stage];
          si.mt = cur.mt;
          si.u = u;
          si.f = cur.f;
          si.c0 = (int)c0;
          si.c1 = (int)min(c0 + CH, cur.c_hi);
          si.first = run_first && c0 == cur.c_lo;
          si.last = run_last && si.c1 == cur.c_hi;
          si.on = cur.on;
          si.zero = cur.zero;
          si.inv_mc = cur.inv_mc;
          const int w = si.c1 - si.c0;
          uint32_t bytes = (uint32_t)(RP * w) * (uint32_t)sizeof(TM);
          if (KIND == 0 || p.nesterov) bytes += (uint32_t)(RP * w) * (uint32_t)sizeof(TG);
          if (KIND == 1) bytes += (uint32_t)(RP * w) * (uint32_t)sizeof(TW);
          if (cur.on) {
            // energies: whole 16-byte groups by bulk copy, the last w % 4
            // values (a ragged tall factor's end) by plain stores, made
            // visible to the consumers by this arrive's release
            const int wq = w & ~3;
            bytes += (uint32_t)wq * 4u;
            const float* ec = geometry(cur.mt, p.conditioned).e_c;
            float* es = reinterpret_cast<float*>(stages + (size_t)stage * stage_bytes + offE);
            if (wq < w) {
              for (int i = wq; i < w; ++i) es[i] = ec[si.c0 + i];
              // later bulk copies into this stage come after these writes
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
          }
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
      if (si.on && lane == 1 && (w & ~3) > 0)
        bulk_load(base + offE, qs.e_c + si.c0, (uint32_t)((w & ~3) * 4), &full[stage]);
      if (++stage == NS) {
        stage = 0;
        ph ^= 1;
      }
    }
    prev_f = cur.f;
    u = un;
    cur = nxt;
  }
  if (lane == 0) {
    if (ok && stage % np == pw && wait_phase(&empty[stage], ph ^ 1, abort, p.status)) {
      info[stage].u = -1;  // end of the work
      mbar_arrive(&full[stage]);
    }
    if (*abort) drain_stages(full, NS, armed, armed_par);
  }
}

// Column weights C_j^2 (and C_j^4) of the columns a consumer warp handles in
// the current stage, computed once per column: the warp's k-th step of SW
// columns starts at c0 + SW (warp + CW k); entry k SW + o holds column
// o of that step (zero past c1).
template <int SW, int CW, int NCOL>
__device__ __forceinline__ void stage_weights(double* wmine, const float* Es, int c0, int c1, int warp,
                                              int lane, float inv_mc, float eps) {
  for (int idx = lane; idx < NCOL; idx += 32) {
    const int k = idx / SW, o = idx % SW;
    const int col = c0 + SW * (warp + CW * k) + o;
    const double w = col < c1 ? (double)col_weight(Es[col - c0], inv_mc, eps) : 0.0;
    wmine[idx] = w;
    wmine[NCOL + idx] = w * w;
  }
  __syncwarp();
}

// ===========================================================================
// thin_gram_bulk: momentum, Gram partials, short-side energy partials
// ===========================================================================
// SP: the split bf16 tensor-core sums (r = 32, bf16 tensor-core mode), whose
// fp32 accumulators need fewer registers and half the reduction space: six
// consumer warps (one 16-column step each per stage of 96 columns) and three
// stages, two CTAs per SM.
template <int RP, typename TG, typename TM, bool SP = false>
struct GramBulk {
  static constexpr int CW = SP ? 6 : RP == 32 ? 4 : 8;  // consumer warps
  static constexpr int NP = 2;                          // producer warps
  static constexpr int BT = 32 * (CW + NP);
  static constexpr int MINB = SP ? 2 : RP == 8 || RP == 16 ? 3 : RP == 32 ? 2 : 1;  // resident CTAs
  static constexpr int CH = SP ? 96 : RP <= 4 ? 1024 : RP == 8 ? 256 : RP == 16 ? 128 : 64;
  static constexpr int NS = SP ? 3 : 4;
  static constexpr int PM = pitch_elems<TM>(CH), PG = pitch_elems<TG>(CH);
  static constexpr int OFF_G = opnd_bytes<TM>(RP, CH);
  static constexpr int OFF_E = OFF_G + opnd_bytes<TG>(RP, CH);
  static constexpr int STAGE_BYTES = (OFF_E + CH * 4 + 127) / 128 * 128;
  // per-warp Gram (fp64, or fp32 under SP) and energy partials for the
  // reduction at a run's end
  static constexpr int RED_S_BYTES = CW * 2 * TCfg<RP>::PART * (SP ? 4 : 8);
  static constexpr int RED_BYTES = RED_S_BYTES + CW * RP * 4;
  static constexpr int NCOL = TCfg<RP>::MMA ? CH / CW : 0;  // columns of one consumer warp per stage
  static constexpr int WS_BYTES = CW * 2 * NCOL * 8;
  static constexpr int SMEM = NS * STAGE_BYTES + NS * (int)sizeof(StageInfo) + (2 * NS + 2) * 8 + 16 +
                              RED_BYTES + WS_BYTES + 128;
};

// Accumulators of one consumer lane for one slab.
template <int RP>
struct GramAcc {
  static constexpr bool MMA = TCfg<RP>::MMA;
  double s1[MMA ? TCfg<RP>::NUB : RP][MMA ? 2 : RP];
  double s2[MMA ? TCfg<RP>::NUB : RP][MMA ? 2 : RP];
  float er[MMA ? TCfg<RP>::NB : RP];
};

// 16 long-side columns c .. c + 15, all inside the stage (RP >= 8).
// Lane (g, t) holds rows g + 8 blk at columns c + 4t + e (wide) or
// c + t + 4e (tall); the DMMA's k slot t is that column.
template <int RP, typename TG, typename TM, bool TALL, bool ON, bool NEST>
__device__ __forceinline__ void gram_step_mma(GramAcc<RP>& acc, const TM* Ms, const TG* Gs,
                                              const double* wrow, TM* Mg, int64_t n, int cs, int c,
                                              float mu, int g, int t) {
  using L = GramBulk<RP, TG, TM>;
  constexpr int NB = TCfg<RP>::NB;
  float mv[NB][4], gv[NB][4];
  if constexpr (!TALL) {
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      El<TM>::ld4(Ms + (g + 8 * blk) * L::PM + cs + 4 * t, mv[blk]);
      El<TG>::ld4(Gs + (g + 8 * blk) * L::PG + cs + 4 * t, gv[blk]);
    }
  } else {
#pragma unroll
    for (int blk = 0; blk < NB; ++blk)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int o = (cs + t + 4 * e) * RP + g + 8 * blk;
        mv[blk][e] = El<TM>::ld1(Ms + o);
        gv[blk][e] = El<TG>::ld1(Gs + o);
      }
  }
  double wd[4], w2d[4];
  if constexpr (ON) {
    constexpr int NCOL = L::NCOL;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int o = TALL ? t + 4 * e : 4 * t + e;
      wd[e] = wrow[o];
      w2d[e] = wrow[NCOL + o];
    }
  }
  double bx[NB][4];
#pragma unroll
  for (int blk = 0; blk < NB; ++blk)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float m = momentum_value(mu, mv[blk][e], gv[blk][e], El<TM>::DT);
      mv[blk][e] = m;
      bx[blk][e] = NEST ? fma((double)mu, (double)m, (double)gv[blk][e]) : (double)m;
      acc.er[blk] = fmaf(m, m, acc.er[blk]);
    }
  if constexpr (!TALL) {
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) El<TM>::st4(Mg + (int64_t)(g + 8 * blk) * n + c + 4 * t, mv[blk]);
  } else {
#pragma unroll
    for (int blk = 0; blk < NB; ++blk)
#pragma unroll
      for (int e = 0; e < 4; ++e) El<TM>::st1(Mg + (int64_t)(c + t + 4 * e) * RP + g + 8 * blk, mv[blk][e]);
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    double xw[NB], xw2[NB];
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      xw[blk] = ON ? wd[e] * bx[blk][e] : bx[blk][e];
      xw2[blk] = ON ? w2d[e] * bx[blk][e] : 0.0;
    }
    int ub = 0;
#pragma unroll
    for (int bi = 0; bi < NB; ++bi)
#pragma unroll
      for (int bj = bi; bj < NB; ++bj, ++ub) {
        dmma(acc.s1[ub][0], acc.s1[ub][1], bx[bi][e], xw[bj]);
        if constexpr (ON) dmma(acc.s2[ub][0], acc.s2[ub][1], bx[bi][e], xw2[bj]);
      }
  }
}

// Predicated version of gram_step_mma for a step that crosses the stage end.
template <int RP, typename TG, typename TM>
__device__ __noinline__ void gram_step_mma_tail(GramAcc<RP>& acc, const TM* Ms, const TG* Gs,
                                                const float* Es, TM* Mg, int64_t n, bool tall,
                                                bool on, int cs, int c, int c1, float mu,
                                                float inv_mc, float eps, bool nest, int g, int t) {
  using L = GramBulk<RP, TG, TM>;
  constexpr int NB = TCfg<RP>::NB;
  float mv[NB][4], gv[NB][4];
  bool okc[4];
  double wd[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int col = tall ? c + t + 4 * e : c + 4 * t + e;
    okc[e] = col < c1;
    wd[e] = on ? (okc[e] ? (double)col_weight(Es[col - c + cs], inv_mc, eps) : 0.0) : 1.0;
  }
#pragma unroll
  for (int blk = 0; blk < NB; ++blk)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int o = tall ? (cs + t + 4 * e) * RP + g + 8 * blk : (g + 8 * blk) * L::PM + cs + 4 * t + e;
      const int og = tall ? o : (g + 8 * blk) * L::PG + cs + 4 * t + e;
      mv[blk][e] = okc[e] ? El<TM>::ld1(Ms + o) : 0.f;
      gv[blk][e] = okc[e] ? El<TG>::ld1(Gs + og) : 0.f;
    }
  double bx[NB][4];
#pragma unroll
  for (int blk = 0; blk < NB; ++blk)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float m = momentum_value(mu, mv[blk][e], gv[blk][e], El<TM>::DT);
      mv[blk][e] = m;
      bx[blk][e] = nest ? fma((double)mu, (double)m, (double)gv[blk][e]) : (double)m;
      acc.er[blk] = fmaf(m, m, acc.er[blk]);
      const int col = tall ? c + t + 4 * e : c + 4 * t + e;
      if (okc[e])
        El<TM>::st1(Mg + (tall ? (int64_t)col * RP + g + 8 * blk : (int64_t)(g + 8 * blk) * n + col),
                    m);
    }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    double xw[NB], xw2[NB];
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      xw[blk] = wd[e] * bx[blk][e];
      xw2[blk] = wd[e] * xw[blk];
    }
    int ub = 0;
#pragma unroll
    for (int bi = 0; bi < NB; ++bi)
#pragma unroll
      for (int bj = bi; bj < NB; ++bj, ++ub) {
        dmma(acc.s1[ub][0], acc.s1[ub][1], bx[bi][e], xw[bj]);
        if (on) dmma(acc.s2[ub][0], acc.s2[ub][1], bx[bi][e], xw2[bj]);
      }
  }
}

// Four long-side columns c .. c + 3 owned by one lane (RP == r <= 4); the
// stage width is a multiple of 8, so every step is full.
template <int RP, typename TG, typename TM, bool TALL, bool ON, bool NEST>
__device__ __forceinline__ void gram_step_small(GramAcc<RP>& acc, const TM* Ms, const TG* Gs,
                                                const float* Es, TM* Mg, int64_t n, int cs, int c,
                                                float mu, float inv_mc, float eps) {
  using L = GramBulk<RP, TG, TM>;
  float mv[RP][4], gv[RP][4];
  if constexpr (!TALL) {
#pragma unroll
    for (int i = 0; i < RP; ++i) {
      El<TM>::ld4(Ms + i * L::PM + cs, mv[i]);
      El<TG>::ld4(Gs + i * L::PG + cs, gv[i]);
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
  double wd[4];
  if constexpr (ON) {
    const float4 e4 = *reinterpret_cast<const float4*>(Es + cs);
    wd[0] = (double)col_weight(e4.x, inv_mc, eps);
    wd[1] = (double)col_weight(e4.y, inv_mc, eps);
    wd[2] = (double)col_weight(e4.z, inv_mc, eps);
    wd[3] = (double)col_weight(e4.w, inv_mc, eps);
  }
  double bx[RP][4];
#pragma unroll
  for (int i = 0; i < RP; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float m = momentum_value(mu, mv[i][e], gv[i][e], El<TM>::DT);
      mv[i][e] = m;
      bx[i][e] = NEST ? fma((double)mu, (double)m, (double)gv[i][e]) : (double)m;
      acc.er[i] = fmaf(m, m, acc.er[i]);
    }
  if constexpr (!TALL) {
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
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
      for (int k = i; k < RP; ++k) {
        const double xk = ON ? wd[e] * bx[k][e] : bx[k][e];
        acc.s1[i][k] = fma(bx[i][e], xk, acc.s1[i][k]);
        if constexpr (ON) acc.s2[i][k] = fma(bx[i][e], wd[e] * xk, acc.s2[i][k]);
      }
  }
}

// ---------------------------------------------------------------------------
// Split bf16 tensor-core sums (RP = 32, bf16 tensor-core mode).  S_1 and S_2
// are Y Y^T products (K = long-side columns): m16n8k16 tiles with fp32
// accumulators, each operand split into bf16 hi + lo (three products per
// tile).  Only the tiles meeting the upper triangle are formed: 16-row tile
// mt against 8-column tile nt >= 2 mt.
// ---------------------------------------------------------------------------
template <int RP>
struct SCfg {
  static constexpr int NB = RP / 8;                      // 8-row blocks
  static constexpr int MT = RP / 16;                     // 16-row tiles
  static constexpr int NT = MT * NB - MT * (MT - 1);     // upper tiles
};

template <int RP>
struct SplitGramAcc {
  float s1[SCfg<RP>::NT][4];
  float s2[SCfg<RP>::NT][4];
  float er[SCfg<RP>::NB];
};

template <int RP, bool SP>
struct GramAccOf {
  using T = GramAcc<RP>;
};
template <int RP>
struct GramAccOf<RP, true> {
  using T = SplitGramAcc<RP>;
};

// Column factors of the split Gram sums, once per column and stage: entry
// k SW + o of the warp's k-th step holds C = (C^2)^(1/2) and C^2 of that
// column (zero past c1), so S_1 = sum (C b)(C b)^T and S_2 = sum (C^2 b)(C^2 b)^T.
template <int CW, int NCOL>
__device__ __forceinline__ void stage_col_factors(float* wmine, const float* Es, int c0, int c1,
                                                  int warp, int lane, float inv_mc, float eps) {
  for (int idx = lane; idx < NCOL; idx += 32) {
    const int k = idx / 16, o = idx % 16;
    const int col = c0 + 16 * (warp + CW * k) + o;
    const float w = col < c1 ? col_weight(Es[col - c0], inv_mc, eps) : 0.f;
    wmine[idx] = sqrtf(w);
    wmine[NCOL + idx] = w;
  }
  __syncwarp();
}

// A (= B) fragments of one 16-row tile of the split products: rows
// 16 mt + g (+ 8) at the lane's four k slots.
template <int NB>
__device__ __forceinline__ void split_rows(const float (&v)[NB][4], int mt, uint32_t (&h)[4],
                                           uint32_t (&l)[4]) {
  split_bf16x2(v[2 * mt][0], v[2 * mt][1], h[0], l[0]);
  split_bf16x2(v[2 * mt + 1][0], v[2 * mt + 1][1], h[1], l[1]);
  split_bf16x2(v[2 * mt][2], v[2 * mt][3], h[2], l[2]);
  split_bf16x2(v[2 * mt + 1][2], v[2 * mt + 1][3], h[3], l[3]);
}

// S += V V^T over the lane's 16 columns for the upper tiles (mt, nt >= 2 mt):
// the B fragment of 8-column tile nt is one half of the A fragment of
// 16-row tile nt / 2.
template <int RP>
__device__ __forceinline__ void syrk_split(float (*S)[4], const float (&v)[RP / 8][4]) {
  constexpr int NB = SCfg<RP>::NB, MT = SCfg<RP>::MT;
  uint32_t h[MT][4], l[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) split_rows<NB>(v, mt, h[mt], l[mt]);
  int ti = 0;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 2 * mt; nt < NB; ++nt, ++ti) {
      const int hn = nt & 1;
      const uint32_t bh[2] = {h[nt >> 1][hn], h[nt >> 1][2 + hn]};
      const uint32_t bl[2] = {l[nt >> 1][hn], l[nt >> 1][2 + hn]};
      hmma_split(S[ti], h[mt], l[mt], bh, bl);
    }
}

// 16 long-side columns c .. c + 15.  Lane (g, t) holds rows g + 8 b of the
// columns at k slots q = 0..3, i.e. c + 2t, c + 2t + 1, c + 2t + 8,
// c + 2t + 9 (the A and the B fragments of the m16n8k16 products use the
// same values).  FULL = false predicates the columns against c1.
template <int RP, typename TG, typename TM, bool TALL, bool ON, bool NEST, bool FULL>
__device__ __forceinline__ void gram_step_split(SplitGramAcc<RP>& acc, const TM* Ms, const TG* Gs,
                                                const float* wrow, TM* Mg, int64_t n, int cs, int c,
                                                int c1, float mu, int g, int t) {
  using L = GramBulk<RP, TG, TM, true>;
  constexpr int NB = SCfg<RP>::NB;
  const int off[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
  bool okc[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) okc[q] = FULL || c + off[q] < c1;
  float mv[NB][4], gv[NB][4];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    if constexpr (!TALL && FULL) {
      const TM* pm = Ms + (g + 8 * b) * L::PM + cs + 2 * t;
      const TG* pg = Gs + (g + 8 * b) * L::PG + cs + 2 * t;
      El<TM>::ld2(pm, mv[b][0], mv[b][1]);
      El<TM>::ld2(pm + 8, mv[b][2], mv[b][3]);
      El<TG>::ld2(pg, gv[b][0], gv[b][1]);
      El<TG>::ld2(pg + 8, gv[b][2], gv[b][3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int om = TALL ? (cs + off[q]) * RP + g + 8 * b : (g + 8 * b) * L::PM + cs + off[q];
        const int og = TALL ? om : (g + 8 * b) * L::PG + cs + off[q];
        mv[b][q] = okc[q] ? El<TM>::ld1(Ms + om) : 0.f;
        gv[b][q] = okc[q] ? El<TG>::ld1(Gs + og) : 0.f;
      }
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float m = momentum_value(mu, mv[b][q], gv[b][q], El<TM>::DT);
      mv[b][q] = m;
      acc.er[b] = fmaf(m, m, acc.er[b]);
      if constexpr (NEST) gv[b][q] = fmaf(mu, m, gv[b][q]);  // B = G + mu M_t
    }
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    if constexpr (!TALL && FULL) {
      TM* dst = Mg + (int64_t)(g + 8 * b) * n + c + 2 * t;
      El<TM>::st2(dst, mv[b][0], mv[b][1]);
      El<TM>::st2(dst + 8, mv[b][2], mv[b][3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (okc[q])
          El<TM>::st1(Mg + (TALL ? (int64_t)(c + off[q]) * RP + g + 8 * b
                                 : (int64_t)(g + 8 * b) * n + c + off[q]),
                      mv[b][q]);
    }
  }
  // the orthogonaliser's input columns b (B_t under Nesterov, else M_t)
  float (&bx)[NB][4] = NEST ? gv : mv;
  if constexpr (ON) {
    float cf[4], c2[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      cf[q] = wrow[off[q]];
      c2[q] = wrow[L::NCOL + off[q]];
    }
    float v[NB][4];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int q = 0; q < 4; ++q) v[b][q] = cf[q] * bx[b][q];
    syrk_split<RP>(acc.s1, v);
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int q = 0; q < 4; ++q) v[b][q] = c2[q] * bx[b][q];
    syrk_split<RP>(acc.s2, v);
  } else {
    syrk_split<RP>(acc.s1, bx);
  }
}

template <int RP, typename TG, typename TM, bool TALL, bool ON, bool NEST>
__device__ __forceinline__ void gram_stage_split(SplitGramAcc<RP>& acc, const TM* Ms, const TG* Gs,
                                                 const float* wmine, TM* Mg, int64_t n, int c0,
                                                 int c1, float mu, int warp, int g, int t) {
  constexpr int CW = GramBulk<RP, TG, TM, true>::CW;
  int k = 0;
  for (int c = c0 + 16 * warp; c < c1; c += 16 * CW, ++k) {
    if (c + 16 <= c1)
      gram_step_split<RP, TG, TM, TALL, ON, NEST, true>(acc, Ms, Gs, wmine + 16 * k, Mg, n, c - c0, c,
                                                        c1, mu, g, t);
    else
      gram_step_split<RP, TG, TM, TALL, ON, NEST, false>(acc, Ms, Gs, wmine + 16 * k, Mg, n, c - c0,
                                                         c, c1, mu, g, t);
  }
}

template <int RP, typename TG, typename TM, bool SP>
__global__ void __launch_bounds__(GramBulk<RP, TG, TM, SP>::BT, GramBulk<RP, TG, TM, SP>::MINB)
    thin_gram_bulk(const __grid_constant__ ThinParams p) {
  using L = GramBulk<RP, TG, TM, SP>;
  using Cf = TCfg<RP>;
  constexpr int CH = L::CH, NS = L::NS, CW = L::CW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  uint8_t* stages = smem;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + NS * L::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(info + NS);
  uint64_t* empty = full + NS;
  uint64_t* redf = empty + NS;  // run-end reduction: consumer warps wrote their partials
  uint64_t* redr = redf + 1;    // run-end reduction: consumer warps read the partials
  volatile int* abort = reinterpret_cast<volatile int*>(redr + 1);
  uint8_t* red_base = reinterpret_cast<uint8_t*>(redr + 1) + 16;
  double* red_s = reinterpret_cast<double*>(red_base);  // fp64 partials
  float* red_sf = reinterpret_cast<float*>(red_base);   // fp32 partials (SP)
  float* red_e = reinterpret_cast<float*>(red_base + L::RED_S_BYTES);
  double* wsm = reinterpret_cast<double*>(red_e + CW * RP);  // CW * RP is even
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    mbar_init(redf, CW);
    mbar_init(redr, CW);
    *abort = step_aborted(p.status) ? 1 : 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (*abort) return;  // an earlier launch of this step timed out

  if (warp >= CW) {
    produce<RP, CH, NS, TG, TM, TM, 0>(p, stages, L::STAGE_BYTES, L::OFF_G, 0, L::OFF_E, info, full,
                                       empty, abort, warp - CW, L::NP);
    return;
  }

  // ------------------------------- consumers -------------------------------
  const float mu = p.mu, eps = p.eps;
  const bool nest = p.nesterov != 0;
  const int g = lane >> 2, t = lane & 3;
  typename GramAccOf<RP, SP>::T acc;
  int stage = 0;
  uint32_t ph = 0, nred = 0;
  for (;;) {
    if (!wait_phase(&full[stage], ph, abort, p.status)) break;
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
      if constexpr (SP) {
#pragma unroll
        for (int a = 0; a < SCfg<RP>::NT; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc.s1[a][b] = acc.s2[a][b] = 0.f;
#pragma unroll
        for (int a = 0; a < SCfg<RP>::NB; ++a) acc.er[a] = 0.f;
      } else {
#pragma unroll
        for (int a = 0; a < (Cf::MMA ? Cf::NUB : RP); ++a)
#pragma unroll
          for (int b = 0; b < (Cf::MMA ? 2 : RP); ++b) acc.s1[a][b] = acc.s2[a][b] = 0.0;
#pragma unroll
        for (int a = 0; a < (Cf::MMA ? Cf::NB : RP); ++a) acc.er[a] = 0.f;
      }
    }

    if constexpr (SP) {
      float* wmine = reinterpret_cast<float*>(wsm + warp * 2 * L::NCOL);
      if (on) stage_col_factors<CW, L::NCOL>(wmine, Es, c0, c1, warp, lane, inv_mc, eps);
#define DM_GRAM_SPLIT(TALL_, ON_, NEST_) \
  gram_stage_split<RP, TG, TM, TALL_, ON_, NEST_>(acc, Ms, Gs, wmine, Mg, n, c0, c1, mu, warp, g, t)
      if (tall) {
        if (on) { if (nest) DM_GRAM_SPLIT(true, true, true); else DM_GRAM_SPLIT(true, true, false); }
        else { if (nest) DM_GRAM_SPLIT(true, false, true); else DM_GRAM_SPLIT(true, false, false); }
      } else {
        if (on) { if (nest) DM_GRAM_SPLIT(false, true, true); else DM_GRAM_SPLIT(false, true, false); }
        else { if (nest) DM_GRAM_SPLIT(false, false, true); else DM_GRAM_SPLIT(false, false, false); }
      }
#undef DM_GRAM_SPLIT
    } else if constexpr (Cf::MMA) {
      double* wmine = wsm + warp * 2 * L::NCOL;
      if (on) stage_weights<16, CW, L::NCOL>(wmine, Es, c0, c1, warp, lane, inv_mc, eps);
      int k = 0;
      for (int c = c0 + 16 * warp; c < c1; c += 16 * CW, ++k) {
        const int cs = c - c0;
        const double* wrow = wmine + 16 * k;
        if (c + 16 <= c1) {
#define DM_GRAM_MMA(TALL_, ON_, NEST_) \
  gram_step_mma<RP, TG, TM, TALL_, ON_, NEST_>(acc, Ms, Gs, wrow, Mg, n, cs, c, mu, g, t)
          if (tall) {
            if (on) { if (nest) DM_GRAM_MMA(true, true, true); else DM_GRAM_MMA(true, true, false); }
            else { if (nest) DM_GRAM_MMA(true, false, true); else DM_GRAM_MMA(true, false, false); }
          } else {
            if (on) { if (nest) DM_GRAM_MMA(false, true, true); else DM_GRAM_MMA(false, true, false); }
            else { if (nest) DM_GRAM_MMA(false, false, true); else DM_GRAM_MMA(false, false, false); }
          }
#undef DM_GRAM_MMA
        } else {
          gram_step_mma_tail<RP, TG, TM>(acc, Ms, Gs, Es, Mg, n, tall, on, cs, c, c1, mu, inv_mc, eps,
                                         nest, g, t);
        }
      }
    } else {
      for (int c = c0 + 4 * (lane + 32 * warp); c < c1; c += 4 * 32 * CW) {
        const int cs = c - c0;
#define DM_GRAM_SMALL(TALL_, ON_, NEST_) \
  gram_step_small<RP, TG, TM, TALL_, ON_, NEST_>(acc, Ms, Gs, Es, Mg, n, cs, c, mu, inv_mc, eps)
        if (tall) {
          if (on) { if (nest) DM_GRAM_SMALL(true, true, true); else DM_GRAM_SMALL(true, true, false); }
          else { if (nest) DM_GRAM_SMALL(true, false, true); else DM_GRAM_SMALL(true, false, false); }
        } else {
          if (on) { if (nest) DM_GRAM_SMALL(false, true, true); else DM_GRAM_SMALL(false, true, false); }
          else { if (nest) DM_GRAM_SMALL(false, false, true); else DM_GRAM_SMALL(false, false, false); }
        }
#undef DM_GRAM_SMALL
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[stage]);  // this warp is done with the stage
    if (++stage == NS) {
      stage = 0;
      ph ^= 1;
    }

    if (last) {
      // run-end reduction over the consumer warps: each writes its partials,
      // all meet on redf, the sums go to the run's last slab, all meet on
      // redr before the partial buffers are written again
      if (!wait_phase(redr, (nred & 1u) ^ 1u, abort, p.status)) break;
      double* mine = red_s + warp * 2 * Cf::PART;
      float* minef = red_sf + warp * 2 * Cf::PART;
      if constexpr (SP) {
        // tile (mt, nt) holds 8x8 blocks (2 mt, nt) and (2 mt + 1, nt) in the
        // DMMA accumulator layout (row g, columns 2t, 2t + 1); the upper ones
        // go to their packed slot
        constexpr int NB = SCfg<RP>::NB;
        int ti = 0;
#pragma unroll
        for (int mt = 0; mt < SCfg<RP>::MT; ++mt)
#pragma unroll
          for (int nt = 2 * mt; nt < NB; ++nt, ++ti)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int bi = 2 * mt + hh, bj = nt;
              if (bi > bj) continue;
              const int ub = bi * NB - bi * (bi - 1) / 2 + (bj - bi);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                minef[ub * 64 + g * 8 + 2 * t + h] = acc.s1[ti][2 * hh + h];
                minef[Cf::PART + ub * 64 + g * 8 + 2 * t + h] = acc.s2[ti][2 * hh + h];
              }
            }
#pragma unroll
        for (int blk = 0; blk < NB; ++blk) {
          float e = acc.er[blk];
          e += __shfl_xor_sync(0xffffffffu, e, 1);
          e += __shfl_xor_sync(0xffffffffu, e, 2);
          if (t == 0) red_e[warp * RP + g + 8 * blk] = e;
        }
      } else if constexpr (Cf::MMA) {
        constexpr int NB = Cf::NB, NUB = Cf::NUB;
#pragma unroll
        for (int ub = 0; ub < NUB; ++ub)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            mine[ub * 64 + g * 8 + 2 * t + h] = acc.s1[ub][h];
            mine[Cf::PART + ub * 64 + g * 8 + 2 * t + h] = acc.s2[ub][h];
          }
#pragma unroll
        for (int blk = 0; blk < NB; ++blk) {
          float e = acc.er[blk];
          e += __shfl_xor_sync(0xffffffffu, e, 1);
          e += __shfl_xor_sync(0xffffffffu, e, 2);
          if (t == 0) red_e[warp * RP + g + 8 * blk] = e;
        }
      } else {
#pragma unroll
        for (int i = 0; i < RP; ++i) {
#pragma unroll
          for (int k = i; k < RP; ++k) {
            const double a = warp_sum_d(acc.s1[i][k]), b = warp_sum_d(acc.s2[i][k]);
            if (lane == 0) {
              mine[i * RP + k] = mine[k * RP + i] = a;
              mine[Cf::PART + i * RP + k] = mine[Cf::PART + k * RP + i] = b;
            }
          }
          const float e = warp_sum(acc.er[i]);
          if (lane == 0) red_e[warp * RP + i] = e;
        }
      }
      double* dst = p.part + (size_t)u * 2 * Cf::PART;
      __syncwarp();
      if (lane == 0) mbar_arrive(redf);
      if (!wait_phase(redf, nred & 1u, abort, p.status)) break;
      for (int i = tid; i < 2 * Cf::PART; i += 32 * CW) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < CW; ++w)
          s += SP ? (double)red_sf[w * 2 * Cf::PART + i] : red_s[w * 2 * Cf::PART + i];
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
// thin_apply_bulk: O = C^2 T B, W update, long-side energies
// ===========================================================================
// SP: the split bf16 tensor-core apply (r = 32, bf16 tensor-core mode): six
// consumer warps, one 16-column step each per stage of 96 columns, three
// stages, two CTAs per SM.
template <int RP, typename TG, typename TM, typename TW, bool SP = false>
struct ApplyBulk {
  static constexpr int CW = SP ? 6 : RP == 32 ? 4 : 8;
  static constexpr int NP = 2;                 // producer warps
  static constexpr int BT = 32 * (CW + NP);
  static constexpr int MINB = SP || RP == 8 || RP == 2 || RP == 32 ? 2 : 1;  // resident CTAs
  static constexpr int CH = SP ? 96 : RP <= 4 ? 1024 : RP <= 16 ? 256 : 128;
  static constexpr int NS = SP || RP == 32 ? 3 : 4;
  static constexpr int PM = pitch_elems<TM>(CH), PG = pitch_elems<TG>(CH), PW = pitch_elems<TW>(CH);
  static constexpr int OFF_W = opnd_bytes<TM>(RP, CH);
  static constexpr int OFF_E = OFF_W + opnd_bytes<TW>(RP, CH);
  static constexpr int OFF_G = OFF_E + CH * 4;  // Nesterov only
  static constexpr int BYTES_NO_G = (OFF_G + 127) / 128 * 128;
  static constexpr int BYTES_G = (OFF_G + opnd_bytes<TG>(RP, CH) + 127) / 128 * 128;
  __host__ __device__ static constexpr int stage_bytes(bool nest) { return nest ? BYTES_G : BYTES_NO_G; }
  static constexpr int NCOL = TCfg<RP>::MMA ? CH / CW : 0;  // columns of one consumer warp per stage
  __host__ __device__ static constexpr int smem(bool nest) {
    return NS * stage_bytes(nest) + NS * (int)sizeof(StageInfo) + 2 * NS * 8 + 16 + CW * 2 * NCOL * 8 +
           128;
  }
};

// 32 long-side columns c .. c + 31 inside the stage (RP >= 8).  Lane (g, t)
// holds B rows 4 kb + t at column slots c + 4g + e (wide) or c + 8e + g
// (tall); wide computes D = T B (output rows 8 bo + g, columns c + 8t ..
// c + 8t + 7), tall D = B^T T^T (output rows 8 bo + 2t, +1 of column
// c + 8e + g).  FULL = false predicates the columns against c1.
template <int RP, typename TG, typename TM, typename TW, bool TALL, bool ON, bool COND, bool FULL,
          bool NEST>
__device__ __forceinline__ void apply_step_mma(const TM* Ms, const TG* Gs, const TW* Ws,
                                               const double* wrow, const double* Tg, TW* Wg, float* Ug,
                                               float* ecg, int64_t n, int cs, int c, int c1, float mu,
                                               float lr, float decay, float inv_mc, float eps,
                                               bool zero, int g, int t, int lane) {
  using L = ApplyBulk<RP, TG, TM, TW>;
  constexpr int NB = TCfg<RP>::NB, KB = TCfg<RP>::KB;
  bool okc[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) okc[e] = FULL || (TALL ? c + 8 * e + g : c + 4 * g + e) < c1;
  const bool okq = FULL || c + 4 * g < c1;  // wide: this lane's column quad is inside
  double wd[4];
  if constexpr (ON) {
#pragma unroll
    for (int e = 0; e < 4; ++e) wd[e] = wrow[TALL ? 8 * e + g : 4 * g + e];  // zero past c1
  }
  double acc[NB][4][2];
#pragma unroll
  for (int bo = 0; bo < NB; ++bo)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[bo][e][0] = acc[bo][e][1] = 0.0;
  float sq[4] = {0.f, 0.f, 0.f, 0.f};
  // k blocks one at a time: B rows 4 kb + t of this lane's four column slots
#pragma unroll
  for (int kb = 0; kb < KB; ++kb) {
    float mv[4], gv[4];
    if constexpr (!TALL) {
      if (okq) {
        El<TM>::ld4(Ms + (4 * kb + t) * L::PM + cs + 4 * g, mv);
        if (NEST) El<TG>::ld4(Gs + (4 * kb + t) * L::PG + cs + 4 * g, gv);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) mv[e] = gv[e] = 0.f;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int o = (cs + 8 * e + g) * RP + 4 * kb + t;
        mv[e] = okc[e] ? El<TM>::ld1(Ms + o) : 0.f;
        gv[e] = (NEST && okc[e]) ? El<TG>::ld1(Gs + o) : 0.f;
      }
    }
    double tf[NB];
#pragma unroll
    for (int bo = 0; bo < NB; ++bo) tf[bo] = __ldg(Tg + (bo * KB + kb) * 32 + lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const double m = (double)mv[e];
      const double bv = NEST ? fma((double)mu, m, (double)gv[e]) : m;
      const double x = ON ? wd[e] * bv : bv;
      if constexpr (COND) sq[e] = fmaf(mv[e], mv[e], sq[e]);
#pragma unroll
      for (int bo = 0; bo < NB; ++bo) {
        if constexpr (TALL)
          dmma(acc[bo][e][0], acc[bo][e][1], x, tf[bo]);
        else
          dmma(acc[bo][e][0], acc[bo][e][1], tf[bo], x);
      }
    }
  }
  float ce[4];
  if constexpr (COND) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float v = sq[e];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      ce[e] = v;
    }
  }
  if constexpr (!TALL) {
#pragma unroll
    for (int bo = 0; bo < NB; ++bo)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = 8 * bo + g, cl = cs + 8 * t + 4 * h;
        if (FULL || c + 8 * t + 4 * h < c1) {
          float w4[4], o4[4];
          El<TW>::ld4(Ws + row * L::PW + cl, w4);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            o4[e] = zero ? 0.f : (float)acc[bo][e][h];
            w4[e] = decay * w4[e] - lr * o4[e];
          }
          El<TW>::st4(Wg + (int64_t)row * n + c + 8 * t + 4 * h, w4);
          if (Ug) El<float>::st4(Ug + (int64_t)row * n + c + 8 * t + 4 * h, o4);
        }
      }
  } else {
#pragma unroll
    for (int bo = 0; bo < NB; ++bo)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (!okc[e]) continue;
        const int row0 = 8 * bo + 2 * t;
        float w0, w1;
        El<TW>::ld2(Ws + (cs + 8 * e + g) * RP + row0, w0, w1);
        const float o0 = zero ? 0.f : (float)acc[bo][e][0];
        const float o1 = zero ? 0.f : (float)acc[bo][e][1];
        const int64_t go = (int64_t)(c + 8 * e + g) * RP + row0;
        El<TW>::st2(Wg + go, decay * w0 - lr * o0, decay * w1 - lr * o1);
        if (Ug) El<float>::st2(Ug + go, o0, o1);
      }
  }
  if constexpr (COND) {
    if (t == 0) {
      if constexpr (!TALL) {
        if (FULL || c + 4 * g < c1) El<float>::st4(ecg + c + 4 * g, ce);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (okc[e]) ecg[c + 8 * e + g] = ce[e];
      }
    }
  }
}

// Four long-side columns c .. c + 3 owned by one lane (RP == r <= 4).
template <int RP, typename TG, typename TM, typename TW, bool TALL, bool ON, bool COND, bool NEST>
__device__ __forceinline__ void apply_step_small(const TM* Ms, const TG* Gs, const TW* Ws,
                                                 const float* Es, const double* Tg, TW* Wg, float* Ug,
                                                 float* ecg, int64_t n, int cs, int c, float mu,
                                                 float lr, float decay, float inv_mc, float eps,
                                                 bool zero) {
  using L = ApplyBulk<RP, TG, TM, TW>;
  float mv[RP][4], gv[RP][4], wv[RP][4];
  if constexpr (!TALL) {
#pragma unroll
    for (int i = 0; i < RP; ++i) {
      El<TM>::ld4(Ms + i * L::PM + cs, mv[i]);
      if (NEST) El<TG>::ld4(Gs + i * L::PG + cs, gv[i]);
      El<TW>::ld4(Ws + i * L::PW + cs, wv[i]);
    }
  } else {
    float fm[4 * RP], fg[4 * RP], fw[4 * RP];
#pragma unroll
    for (int s = 0; s < RP; ++s) {
      El<TM>::ld4(Ms + cs * RP + 4 * s, &fm[4 * s]);
      if (NEST) El<TG>::ld4(Gs + cs * RP + 4 * s, &fg[4 * s]);
      El<TW>::ld4(Ws + cs * RP + 4 * s, &fw[4 * s]);
    }
#pragma unroll
    for (int i = 0; i < RP; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        mv[i][e] = fm[e * RP + i];
        gv[i][e] = NEST ? fg[e * RP + i] : 0.f;
        wv[i][e] = fw[e * RP + i];
      }
  }
  double wd[4];
  if constexpr (ON) {
    const float4 e4 = *reinterpret_cast<const float4*>(Es + cs);
    wd[0] = (double)col_weight(e4.x, inv_mc, eps);
    wd[1] = (double)col_weight(e4.y, inv_mc, eps);
    wd[2] = (double)col_weight(e4.z, inv_mc, eps);
    wd[3] = (double)col_weight(e4.w, inv_mc, eps);
  }
  double tm[RP][RP];
#pragma unroll
  for (int i = 0; i < RP; ++i)
#pragma unroll
    for (int k = 0; k < RP; ++k) tm[i][k] = __ldg(Tg + i * RP + k);
  float ov[RP][4], ce[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    double x[RP];
    float sq = 0.f;
#pragma unroll
    for (int k = 0; k < RP; ++k) {
      const double m = (double)mv[k][e];
      const double bv = NEST ? fma((double)mu, m, (double)gv[k][e]) : m;
      x[k] = ON ? wd[e] * bv : bv;
      if constexpr (COND) sq = fmaf(mv[k][e], mv[k][e], sq);
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
  if constexpr (!TALL) {
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
  if constexpr (COND) El<float>::st4(ecg + c, ce);
}

// ---------------------------------------------------------------------------
// Split bf16 tensor-core apply (RP = 32, bf16 tensor-core mode): O = T X
// with X = C^2 B, K = the short side, m16n8k16 tiles, T and X split into
// bf16 hi + lo.  T's fragments stay in registers while the factor is the
// same.
// ---------------------------------------------------------------------------
template <int RP>
struct SplitT {
  static constexpr int MT = RP / 16, KT = RP / 16;
  uint32_t h[MT][KT][4], l[MT][KT][4];
};

// T is stored in the DMMA fragment order: T[i][k] at
// ((i / 8) (RP / 4) + k / 4) 32 + (i % 8) 4 + k % 4.
template <int RP>
__device__ __forceinline__ void load_split_t(SplitT<RP>& f, const double* Tg, int g, int t) {
  constexpr int KB = RP / 4;
  auto tv = [&](int i, int k) {
    return (float)__ldg(Tg + ((i >> 3) * KB + (k >> 2)) * 32 + (i & 7) * 4 + (k & 3));
  };
#pragma unroll
  for (int mt = 0; mt < SplitT<RP>::MT; ++mt)
#pragma unroll
    for (int kt = 0; kt < SplitT<RP>::KT; ++kt) {
      const int r0 = 16 * mt + g, r1 = r0 + 8, k0 = 16 * kt + 2 * t, k1 = k0 + 8;
      split_bf16x2(tv(r0, k0), tv(r0, k0 + 1), f.h[mt][kt][0], f.l[mt][kt][0]);
      split_bf16x2(tv(r1, k0), tv(r1, k0 + 1), f.h[mt][kt][1], f.l[mt][kt][1]);
      split_bf16x2(tv(r0, k1), tv(r0, k1 + 1), f.h[mt][kt][2], f.l[mt][kt][2]);
      split_bf16x2(tv(r1, k1), tv(r1, k1 + 1), f.h[mt][kt][3], f.l[mt][kt][3]);
    }
}

// 16 long-side columns c .. c + 15 as two 8-column tiles.  For tile nt,
// lane (g, t) supplies column c + 8 nt + g at rows 16 kt + {2t, 2t + 1,
// 2t + 8, 2t + 9} (the B fragment) and receives O rows 16 mt + g, + 8 at
// columns c + 8 nt + 2t, + 1.
template <int RP, typename TG, typename TM, typename TW, bool TALL, bool ON, bool COND, bool FULL,
          bool NEST>
__device__ __forceinline__ void apply_step_split(const SplitT<RP>& tf, const TM* Ms, const TG* Gs,
                                                 const TW* Ws, const double* wrow, TW* Wg, float* Ug,
                                                 float* ecg, int64_t n, int cs, int c, int c1,
                                                 float mu, float lr, float decay, bool zero, int g,
                                                 int t) {
  using L = ApplyBulk<RP, TG, TM, TW, true>;
  constexpr int MT = SplitT<RP>::MT, KT = SplitT<RP>::KT;
  const int off[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const int jl = 8 * nt + g;
    const bool okj = FULL || c + jl < c1;
    const float w = ON ? (float)wrow[jl] : 1.f;  // zero past c1
    uint32_t bh[KT][2], bl[KT][2];
    float sq = 0.f;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      float mv[4], gv[4];
      if constexpr (TALL) {
        const int o = (cs + jl) * RP + 16 * kt + 2 * t;
        if (okj) {
          El<TM>::ld2(Ms + o, mv[0], mv[1]);
          El<TM>::ld2(Ms + o + 8, mv[2], mv[3]);
          if (NEST) {
            El<TG>::ld2(Gs + o, gv[0], gv[1]);
            El<TG>::ld2(Gs + o + 8, gv[2], gv[3]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) mv[q] = gv[q] = 0.f;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int k = 16 * kt + off[q];
          mv[q] = okj ? El<TM>::ld1(Ms + k * L::PM + cs + jl) : 0.f;
          gv[q] = (NEST && okj) ? El<TG>::ld1(Gs + k * L::PG + cs + jl) : 0.f;
        }
      }
      float x[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if constexpr (COND) sq = fmaf(mv[q], mv[q], sq);
        const float bv = NEST ? fmaf(mu, mv[q], gv[q]) : mv[q];
        x[q] = ON ? w * bv : bv;
      }
      split_bf16x2(x[0], x[1], bh[kt][0], bl[kt][0]);
      split_bf16x2(x[2], x[3], bh[kt][1], bl[kt][1]);
    }
    float d[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      d[mt][0] = d[mt][1] = d[mt][2] = d[mt][3] = 0.f;
#pragma unroll
      for (int kt = 0; kt < KT; ++kt) hmma_split(d[mt], tf.h[mt][kt], tf.l[mt][kt], bh[kt], bl[kt]);
    }
    if constexpr (COND) {
      sq += __shfl_xor_sync(0xffffffffu, sq, 1);
      sq += __shfl_xor_sync(0xffffffffu, sq, 2);
      if (t == 0 && okj) ecg[c + jl] = sq;
    }
    const int col = 8 * nt + 2 * t;  // this lane's first output column
    const bool ok0 = FULL || c + col < c1, ok1 = FULL || c + col + 1 < c1;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = 16 * mt + g + 8 * hh;
        const float o0 = zero ? 0.f : d[mt][2 * hh], o1 = zero ? 0.f : d[mt][2 * hh + 1];
        if constexpr (!TALL) {
          if (ok0 && ok1) {
            float w0, w1;
            El<TW>::ld2(Ws + row * L::PW + cs + col, w0, w1);
            El<TW>::st2(Wg + (int64_t)row * n + c + col, decay * w0 - lr * o0, decay * w1 - lr * o1);
            if (Ug) El<float>::st2(Ug + (int64_t)row * n + c + col, o0, o1);
          } else if (ok0) {
            const float w0 = El<TW>::ld1(Ws + row * L::PW + cs + col);
            El<TW>::st1(Wg + (int64_t)row * n + c + col, decay * w0 - lr * o0);
            if (Ug) Ug[(int64_t)row * n + c + col] = o0;
          }
        } else {
          if (ok0) {
            const float w0 = El<TW>::ld1(Ws + (cs + col) * RP + row);
            El<TW>::st1(Wg + (int64_t)(c + col) * RP + row, decay * w0 - lr * o0);
            if (Ug) Ug[(int64_t)(c + col) * RP + row] = o0;
          }
          if (ok1) {
            const float w1 = El<TW>::ld1(Ws + (cs + col + 1) * RP + row);
            El<TW>::st1(Wg + (int64_t)(c + col + 1) * RP + row, decay * w1 - lr * o1);
            if (Ug) Ug[(int64_t)(c + col + 1) * RP + row] = o1;
          }
        }
      }
  }
}

template <int RP, typename TG, typename TM, typename TW, bool TALL, bool ON, bool COND, bool NEST>
__device__ __forceinline__ void apply_stage_split(const SplitT<RP>& tf, const TM* Ms, const TG* Gs,
                                                  const TW* Ws, const float* Es, double* wmine,
                                                  TW* Wg, float* Ug, float* ecg, int64_t n, int c0,
                                                  int c1, float mu, float lr, float decay,
                                                  float inv_mc, float eps, bool zero, int warp,
                                                  int lane) {
  using L = ApplyBulk<RP, TG, TM, TW, true>;
  constexpr int CW = L::CW;
  const int g = lane >> 2, t = lane & 3;
  if (ON) stage_weights<16, CW, L::NCOL>(wmine, Es, c0, c1, warp, lane, inv_mc, eps);
  int k = 0;
  for (int c = c0 + 16 * warp; c < c1; c += 16 * CW, ++k) {
    if (c + 16 <= c1)
      apply_step_split<RP, TG, TM, TW, TALL, ON, COND, true, NEST>(tf, Ms, Gs, Ws, wmine + 16 * k, Wg,
                                                                   Ug, ecg, n, c - c0, c, c1, mu, lr,
                                                                   decay, zero, g, t);
    else
      apply_step_split<RP, TG, TM, TW, TALL, ON, COND, false, NEST>(tf, Ms, Gs, Ws, wmine + 16 * k, Wg,
                                                                    Ug, ecg, n, c - c0, c, c1, mu, lr,
                                                                    decay, zero, g, t);
  }
}

template <int RP, typename TG, typename TM, typename TW, bool TALL, bool ON, bool COND, bool NEST>
__device__ __forceinline__ void apply_stage(const TM* Ms, const TG* Gs, const TW* Ws, const float* Es,
                                            double* wmine, const double* Tg, TW* Wg, float* Ug,
                                            float* ecg, int64_t n, int c0, int c1, float mu, float lr,
                                            float decay, float inv_mc, float eps, bool zero,
                                            int warp, int lane) {
  using L = ApplyBulk<RP, TG, TM, TW>;
  constexpr int CW = L::CW;
  if constexpr (TCfg<RP>::MMA) {
    const int g = lane >> 2, t = lane & 3;
    if (ON) stage_weights<32, CW, L::NCOL>(wmine, Es, c0, c1, warp, lane, inv_mc, eps);
    int k = 0;
    for (int c = c0 + 32 * warp; c < c1; c += 32 * CW, ++k) {
      if (c + 32 <= c1)
        apply_step_mma<RP, TG, TM, TW, TALL, ON, COND, true, NEST>(Ms, Gs, Ws, wmine + 32 * k, Tg, Wg, Ug, ecg,
                                                             n, c - c0, c, c1, mu, lr, decay, inv_mc, eps,
                                                             zero, g, t, lane);
      else
        apply_step_mma<RP, TG, TM, TW, TALL, ON, COND, false, NEST>(Ms, Gs, Ws, wmine + 32 * k, Tg, Wg, Ug,
                                                              ecg, n, c - c0, c, c1, mu, lr, decay, inv_mc,
                                                              eps, zero, g, t, lane);
    }
  } else {
    for (int c = c0 + 4 * (lane + 32 * warp); c < c1; c += 4 * 32 * CW)
      apply_step_small<RP, TG, TM, TW, TALL, ON, COND, NEST>(Ms, Gs, Ws, Es, Tg, Wg, Ug, ecg, n, c - c0, c, mu,
                                                       lr, decay, inv_mc, eps, zero);
  }
}

template <int RP, bool SP>
struct SplitTOf {
  struct T {};
};
template <int RP>
struct SplitTOf<RP, true> {
  using T = SplitT<RP>;
};

template <int RP, typename TG, typename TM, typename TW, bool SP>
__global__ void __launch_bounds__(ApplyBulk<RP, TG, TM, TW, SP>::BT, ApplyBulk<RP, TG, TM, TW, SP>::MINB)
    thin_apply_bulk(const __grid_constant__ ThinParams p) {
  using L = ApplyBulk<RP, TG, TM, TW, SP>;
  constexpr int CH = L::CH, NS = L::NS, CW = L::CW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  const int stage_bytes = L::stage_bytes(p.nesterov != 0);
  uint8_t* stages = smem;
  StageInfo* info = reinterpret_cast<StageInfo*>(smem + NS * stage_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(info + NS);
  uint64_t* empty = full + NS;
  volatile int* abort = reinterpret_cast<volatile int*>(empty + NS);
  double* wsm = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(empty + NS) + 16);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    *abort = step_aborted(p.status) ? 1 : 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (*abort) return;  // an earlier launch of this step timed out

  if (warp >= CW) {
    produce<RP, CH, NS, TG, TM, TW, 1>(p, stages, stage_bytes, L::OFF_G, L::OFF_W, L::OFF_E, info, full,
                                       empty, abort, warp - CW, L::NP);
    return;
  }

  const float mu = p.mu, lr = p.lr, decay = p.decay, eps = p.eps;
  const bool nest = p.nesterov != 0;
  int stage = 0;
  uint32_t ph = 0;
  typename SplitTOf<RP, SP>::T tfr;  // split T fragments of factor tf_f
  int tf_f = -1;
  for (;;) {
    if (!wait_phase(&full[stage], ph, abort, p.status)) break;
    const StageInfo& si = info[stage];
    if (si.u < 0) break;
    const int c0 = si.c0, c1 = si.c1;
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
    const double* Tg = p.T + (size_t)si.f * RP * RP;
    if constexpr (SP) {
      if (si.f != tf_f) {
        load_split_t<RP>(tfr, Tg, lane >> 2, lane & 3);
        tf_f = si.f;
      }
    }
#define DM_APPLY_STAGE(TALL_, ON_, COND_)                                                              \
  do {                                                                                                \
    if constexpr (SP) {                                                                               \
      if (nest)                                                                                       \
        apply_stage_split<RP, TG, TM, TW, TALL_, ON_, COND_, true>(                                   \
            tfr, Ms, Gs, Ws, Es, wsm + warp * 2 * L::NCOL, Wg, Ug, ecg, n, c0, c1, mu, lr, decay,     \
            inv_mc, eps, zero, warp, lane);                                                           \
      else                                                                                            \
        apply_stage_split<RP, TG, TM, TW, TALL_, ON_, COND_, false>(                                  \
            tfr, Ms, Gs, Ws, Es, wsm + warp * 2 * L::NCOL, Wg, Ug, ecg, n, c0, c1, mu, lr, decay,     \
            inv_mc, eps, zero, warp, lane);                                                           \
    } else if (nest)                                                                                  \
      apply_stage<RP, TG, TM, TW, TALL_, ON_, COND_, true>(Ms, Gs, Ws, Es, wsm + warp * 2 * L::NCOL, \
                                                           Tg, Wg, Ug, ecg, n, c0, c1, mu, lr, decay, \
                                                           inv_mc, eps, zero, warp, lane);            \
    else                                                                                              \
      apply_stage<RP, TG, TM, TW, TALL_, ON_, COND_, false>(Ms, Gs, Ws, Es, wsm + warp * 2 * L::NCOL, \
                                                            Tg, Wg, Ug, ecg, n, c0, c1, mu, lr, decay, \
                                                            inv_mc, eps, zero, warp, lane);           \
  } while (0)
    if (tall) {
      if (on) DM_APPLY_STAGE(true, true, true);
      else if (cond) DM_APPLY_STAGE(true, false, true);
      else DM_APPLY_STAGE(true, false, false);
    } else {
      if (on) DM_APPLY_STAGE(false, true, true);
      else if (cond) DM_APPLY_STAGE(false, false, true);
      else DM_APPLY_STAGE(false, false, false);
    }
#undef DM_APPLY_STAGE
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

template <int RP, typename TG, typename TM, typename TW, bool SP>
cudaError_t launch_bulk_sp(ThinParams& p, int nsm, cudaStream_t st) {
  using LG = GramBulk<RP, TG, TM, SP>;
  using LA = ApplyBulk<RP, TG, TM, TW, SP>;
  static DeviceOnce once;
  static int occ_g[MAX_DEVICES], occ_a[MAX_DEVICES][2];
  int dev = 0;
  cudaError_t e = device_once(once, &dev, [](int d) {
    cudaError_t e = cudaFuncSetAttribute(thin_gram_bulk<RP, TG, TM, SP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, LG::SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(thin_apply_bulk<RP, TG, TM, TW, SP>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, LA::smem(true));
    // shared memory over L1 for the staging rings
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(thin_gram_bulk<RP, TG, TM, SP>,
                               cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(thin_apply_bulk<RP, TG, TM, TW, SP>,
                               cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    occ_g[d] = resident(thin_gram_bulk<RP, TG, TM, SP>, LG::BT, LG::SMEM);
    occ_a[d][0] = resident(thin_apply_bulk<RP, TG, TM, TW, SP>, LA::BT, LA::smem(false));
    occ_a[d][1] = resident(thin_apply_bulk<RP, TG, TM, TW, SP>, LA::BT, LA::smem(true));
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  const bool nest = p.nesterov != 0;
  p.grid_gram = std::min(p.units, nsm * occ_g[dev]);
  p.grid_apply = std::min(p.units, nsm * occ_a[dev][nest ? 1 : 0]);
  thin_gram_bulk<RP, TG, TM, SP><<<p.grid_gram, LG::BT, LG::SMEM, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_thin_iterate(p, st);
  if (e != cudaSuccess) return e;
  thin_apply_bulk<RP, TG, TM, TW, SP><<<p.grid_apply, LA::BT, LA::smem(nest), st>>>(p);
  return cudaGetLastError();
}

template <int RP, typename TG, typename TM, typename TW>
cudaError_t launch_bulk_rp(ThinParams& p, int nsm, cudaStream_t st) {
  if constexpr (RP == 32) {
    if (p.split) return launch_bulk_sp<RP, TG, TM, TW, true>(p, nsm, st);
  }
  return launch_bulk_sp<RP, TG, TM, TW, false>(p, nsm, st);
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
