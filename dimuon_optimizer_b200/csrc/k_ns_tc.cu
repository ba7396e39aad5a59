// Tensor-core (tcgen05) products of the quintic Newton-Schulz iteration,
// precision mode DM_PREC_BF16_TC:
//   A  = X X^T             (symmetric: only tiles meeting the upper triangle)
//   B  = b A + c A A       (symmetric; A A = A A^T since A is symmetric)
//   X' = a X + B X         (last iteration: fused update / X_5 + norm partials)
// sitech.ge Muon post, "Instead of SVD - Newton-Schulz": X_next = aX +
// b(XX^T)X + c(XX^T)^2X, "efficient in bfloat16"; coefficients from
// "Muon Optimizer 정리", "Why orthogonalise".
//
// Structure (one CTA per SM, persistent over a static round-robin tile list):
//   warp 0      TMA producer: 64 x 64 bf16 boxes, 128-byte swizzle, 4 stages
//               of (128 x 64 A-operand, 256 x 64 B-operand) in shared memory
//   warp 1      one thread issues tcgen05.mma (M=128, N=256, K=16) into one of
//               two 256-column fp32 accumulators in tensor memory
//   warps 2..5  epilogue: tcgen05.ld -> registers -> fused epilogue -> global
// Operands may be K-major or MN-major per matrix (runtime descriptor bits),
// so wide matrices and tall matrices (handled transposed) need no copies.
// Every wait is bounded (see mbar_wait_bounded); no multicast loads are used.
#include "dm_common.cuh"
#include "dm_sm100.cuh"
#include "dm_tc_epilogue.cuh"
#include "dm_tiles.cuh"

namespace dm {
namespace {

using namespace sm100;
using namespace tcepi;

constexpr int STAGES = 4;
constexpr int BOX_BYTES = 64 * 64 * 2;
constexpr int A_BYTES = TC_BM * TC_BK * 2;      // 16 KB
constexpr int B_BYTES = TC_BN * TC_BK * 2;      // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int NUM_THREADS = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr uint32_t TMEM_COLS = 512;             // two 128 x 256 fp32 accumulators
constexpr int BAR_BYTES = 256;
// + one 32 x 32 bf16 staging tile per epilogue warp (coalesced epilogue)
constexpr int EPI_STAGE_BYTES = 8 * STAGE_TILE_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + EPI_STAGE_BYTES + 1024;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // any single wait > 2 s is a hang
constexpr uint64_t DRAIN_LIMIT_NS = 200000000ull;
constexpr uint64_t FORCED_LIMIT_NS = 20000000ull;   // forced-timeout hook: 20 ms

struct Tile {
  int g, lt, tm, tn;
};

__device__ __forceinline__ Tile decode_tile(const TcParams& p, int t) {
  Tile tl;
  tl.g = find_group(p.starts, p.count, t);
  tl.lt = t - p.starts[tl.g];
  gemm_tile_coord(p.mats[tl.g].g, tl.lt, TC_BM, TC_BN, tl.tm, tl.tn);
  return tl;
}

__global__ void __launch_bounds__(NUM_THREADS, 1) tc_ns_product(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* never = drain + 1;  // nothing ever arrives (forced-timeout hook)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    mbar_init(never, 1);
    // an earlier launch of this step gave up on a wait: leave without writing
    *abort = step_aborted(p.status) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (p.debug & DBG_FORCE_TIMEOUT) {
    // Test hook: one thread waits, with a short limit, on a barrier nothing
    // arrives on.  Its expiry takes the ordinary timeout path (abort flag,
    // status word) before any copy or product is issued, so every role then
    // leaves at its first abort check.
    if (threadIdx.x == 0) mbar_wait_bounded(never, 0, abort, p.status, FORCED_LIMIT_NS);
    __syncthreads();
  }

  if (warp == 0) {
    // ----------------------------- TMA producer -----------------------------
    if (lane == 0) {
      for (int g = 0; g < p.count; ++g) {
        tma_prefetch_map(&p.mats[g].ta);
        tma_prefetch_map(&p.mats[g].tb);
      }
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_par = 0;  // per-stage bits of the last armed phase
      for (int t = blockIdx.x; t < p.total_tiles && !*abort; t += gridDim.x) {
        const Tile tl = decode_tile(p, t);
        const TcMat& mt = p.mats[tl.g];
        const int a_mn = mt.g.flags & GF_A_MN, b_mn = mt.g.flags & GF_B_MN;
        const int m0 = tl.tm * TC_BM, n0 = tl.tn * TC_BN;
        const int nkb = (mt.g.K + TC_BK - 1) / TC_BK;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort, p.status, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          armed |= 1u << stage;
          armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          const int k0 = kb * TC_BK;
#pragma unroll
          for (int q = 0; q < TC_BM / 64; ++q) {
            if (a_mn)
              tma_load_2d(sa + q * BOX_BYTES, &mt.ta, &full[stage], m0 + 64 * q, k0);
            else
              tma_load_2d(sa + q * BOX_BYTES, &mt.ta, &full[stage], k0, m0 + 64 * q);
          }
#pragma unroll
          for (int q = 0; q < TC_BN / 64; ++q) {
            if (b_mn)
              tma_load_2d(sb + q * BOX_BYTES, &mt.tb, &full[stage], n0 + 64 * q, k0);
            else
              tma_load_2d(sb + q * BOX_BYTES, &mt.tb, &full[stage], k0, n0 + 64 * q);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      if (*abort) {
        // Let the copies already in flight land before the CTA exits.
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s))
            mbar_wait_drain(&full[s], (armed_par >> s) & 1u, DRAIN_LIMIT_NS);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int t = blockIdx.x; t < p.total_tiles && !*abort; t += gridDim.x, ++local) {
        const Tile tl = decode_tile(p, t);
        const GemmMat& g = p.mats[tl.g].g;
        const int a_mn = (g.flags & GF_A_MN) ? 1 : 0, b_mn = (g.flags & GF_B_MN) ? 1 : 0;
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort, p.status, WAIT_LIMIT_NS)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TC_BN);
        const uint32_t idesc = idesc_bf16(TC_BM, TC_BN, a_mn, b_mn);
        const int nkb = (g.K + TC_BK - 1) / TC_BK;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort, p.status, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < TC_BK / 16; ++kk) {
            const uint64_t ad = a_mn ? smem_desc(sa + kk * 2048, BOX_BYTES, 1024)
                                     : smem_desc(sa + kk * 32, 16, 1024);
            const uint64_t bd = b_mn ? smem_desc(sb + kk * 2048, BOX_BYTES, 1024)
                                     : smem_desc(sb + kk * 32, 16, 1024);
            mma_bf16(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit(&tfull[acc]);
      }
      // Every MMA this thread issued has completed once `drain` flips.
      mma_commit(drain);
      mbar_wait_drain(drain, 0, DRAIN_LIMIT_NS);
    }
  } else {
    // ------------------------------- epilogue -------------------------------
    // Warps 2..9: two warps per TMEM lane quarter, each taking half of the
    // accumulator's columns.
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const int half = ew >> 2;
    const int row_in_half = quarter * 32 + lane;
    int local = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++local) {
      const Tile tl = decode_tile(p, t);
      const GemmMat& g = p.mats[tl.g].g;
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const int r = tl.tm * TC_BM + row_in_half;
      const int nch = min(TC_BN, g.N - tl.tn * TC_BN + 31) / 32;  // chunks holding columns < N
      constexpr int CH_PER = TC_BN / 32 / 2;
      // the first chunk's aux is in flight while the products run
      AuxPrefetch pf;
      fetch_scalars(g, pf);
      fetch_aux(g, r, r < g.M, tl.tn * TC_BN, half * CH_PER, half * CH_PER + CH_PER, nch, pf);
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort, p.status, WAIT_LIMIT_NS)) break;
      tc_fence_after();
      float sx = 0.f, sy = 0.f;
      epilogue_row(g, p.lr, p.decay, r, r < g.M, tl.tn * TC_BN,
                   tmem_base + (uint32_t)(acc * TC_BN) + ((uint32_t)(quarter * 32) << 16),
                   half * CH_PER, half * CH_PER + CH_PER, nch, sx, sy,
                   reinterpret_cast<__nv_bfloat16*>(smem + STAGES * STAGE_BYTES + BAR_BYTES) +
                       ew * (STAGE_TILE_BYTES / 2),
                   pf);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[acc]);
      }
      if (g.epi == EPI_FINAL_DIMUON) {
        // one (sum x^2, sum y^2) pair per epilogue warp; no barrier needed
        sx = warp_sum(sx);
        sy = warp_sum(sy);
        if (lane == 0) {
          const int slot = (tl.tm * g.tiles_n + tl.tn) * 8 + ew;
          g.part[2 * slot] = sx;
          g.part[2 * slot + 1] = sy;
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

int tc_smem_bytes() { return SMEM_BYTES; }

cudaError_t launch_tc(const TcParams& p, int grid, cudaStream_t s) {
  if (p.total_tiles <= 0 || grid <= 0) return cudaSuccess;
  static DeviceOnce once;
  const cudaError_t e = device_once(once, nullptr, [](int) {
    return cudaFuncSetAttribute(tc_ns_product, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES);
  });
  if (e != cudaSuccess) return e;
  tc_ns_product<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(p);
  return cudaGetLastError();
}

}  // namespace dm
