// Tensor-core Newton-Schulz products on CTA pairs (tcgen05 cta_group::2):
// the same three products and fused epilogues as tc_ns_product
//   A = X X^T, B = b A + c A A (symmetric), X' = a X + B X
// (sitech.ge Muon post, "Instead of SVD - Newton-Schulz"; coefficients from
// "Muon Optimizer 정리", "Why orthogonalise"), with 256 x 256 output tiles
// computed by a pair of CTAs (a cluster of 2 on two SMs):
//   - each CTA loads its own 128 rows of the A operand and its own 128
//     columns of the B operand for k blocks of 128 (TMA, 128-byte swizzle,
//     no multicast; one 32 KB copy per operand slab through chunked 3-D
//     maps: 2 chunks of 64 k x 128 rows for K-major slabs, 2 chunks of 64
//     columns x 128 k for MN-major ones), 64 KB per stage, 3 stages; both
//     CTAs' loads complete on the leader's "full" barrier;
//   - one thread of the leader issues tcgen05.mma.cta_group::2 with M = 256,
//     N = 256: the accumulator's rows 0..127 live in the leader's tensor
//     memory, rows 128..255 in the peer's; per k-block the MMA reads half of
//     B from each CTA, so each SM streams 2/3 of the bytes a 128 x 256 tile
//     needs per flop;
//   - the MMA's completion frees the stage in both CTAs and hands each CTA's
//     epilogue warps its half of the accumulator;
//   - the peer's epilogue warps report a drained accumulator to the leader.
// Every wait is bounded; the kernel ends with a cluster barrier so neither
// CTA leaves while the other still addresses its shared memory.
#include "dm_common.cuh"
#include "dm_sm100.cuh"
#include "dm_tc_epilogue.cuh"
#include "dm_tiles.cuh"

namespace dm {
namespace {

using namespace sm100;
using namespace tcepi;

constexpr int PAIR_BM = 256;                     // output tile rows (both CTAs)
constexpr int PAIR_BN = 256;                     // output tile columns
constexpr int HALF = 128;                        // rows (A) / columns (B) per CTA
// k per stage.  128 (3 stages of 64 KB) measured faster than 64 (6 stages of
// 32 KB) on every workload tried: one 32 KB copy per operand slab keeps the
// copy engine well below its per-copy limit (large batch 39.0 -> 35.6 ms per
// step).  The code also takes BK = 64.
constexpr int BK = 128;
constexpr int STAGES = BK == 64 ? 6 : 3;
constexpr int CHUNK_BYTES = HALF * 64 * 2;       // 128 rows x 64 k (K-major) or 64 k x 64 (MN-major), 16 KB
constexpr int BOX_BYTES = 64 * 64 * 2;
constexpr int A_BYTES = HALF * BK * 2;
constexpr int B_BYTES = HALF * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // 32 or 64 KB per CTA
constexpr int NUM_THREADS = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr uint32_t TMEM_COLS = 512;              // two 128-lane x 256-column accumulators
constexpr int BAR_BYTES = 256;
// + one 32 x 32 bf16 staging tile per epilogue warp (coalesced epilogue)
constexpr int EPI_STAGE_BYTES = 8 * STAGE_TILE_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + EPI_STAGE_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 200000000ull;
constexpr uint64_t FORCED_LIMIT_NS = 20000000ull;   // forced-timeout hook: 20 ms
constexpr uint16_t PAIR_MASK = 0x3;

struct Tile {
  int g, lt, tm, tn;
};

__device__ __forceinline__ Tile decode_tile(const TcParams& p, int t) {
  Tile tl;
  tl.g = find_group(p.starts, p.count, t);
  tl.lt = t - p.starts[tl.g];
  gemm_tile_coord(p.mats[tl.g].g, tl.lt, PAIR_BM, PAIR_BN, tl.tm, tl.tn);
  return tl;
}

// One CTA's operand slab (128 rows or columns x BK k) of one stage.
//   K-major, chunked map (box 64 k x 128 rows x 2 k chunks): one copy;
//   K-major, 2-D map (box 64 x 128): one copy per 64-k chunk;
//   MN-major, chunked map (box 64 x BK k rows x 2 chunks): one copy;
//   MN-major, 2-D map (box 64 x 64): one copy per 64 x 64 block.
__device__ __forceinline__ void load_slab(uint8_t* s, const CUtensorMap* map, uint32_t bar, int mn,
                                          int chunked, int k0, int r0) {
  if (!mn) {
    if (chunked) {
      tma_load_3d_pair(s, map, bar, 0, r0, k0 / 64);
    } else {
#pragma unroll
      for (int c = 0; c < BK / 64; ++c) tma_load_2d_pair(s + c * CHUNK_BYTES, map, bar, k0 + 64 * c, r0);
    }
  } else if (chunked) {
    tma_load_3d_pair(s, map, bar, 0, k0, r0 / 64);
  } else {
#pragma unroll
    for (int c = 0; c < HALF / 64; ++c)
#pragma unroll
      for (int j = 0; j < BK / 64; ++j)
        tma_load_2d_pair(s + c * (BK * 128) + j * BOX_BYTES, map, bar, r0 + 64 * c, k0 + 64 * j);
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1) tc_ns_product_pair(const __grid_constant__ TcParams p) {
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
  const uint32_t rank = cluster_rank();  // 0 = leader, 1 = peer
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // leader: its own arrive.expect_tx; peer: unused
      mbar_init(&empty[s], 1);  // one multicast commit per consumed stage
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 16);  // leader: 8 local + 8 peer epilogue warps
    }
    mbar_init(drain, 1);
    mbar_init(never, 1);
    // An earlier launch of this step gave up on a wait: leave without
    // writing.  Both CTAs of the pair read the abort word at their start; it
    // only changes when some wait of this launch has run for its full limit,
    // long after both have read it.  (Were they ever to disagree, the CTA
    // that goes on ends in its own bounded waits.)
    *abort = step_aborted(p.status) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 1) {  // the same warp of both CTAs allocates collectively
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised in both CTAs, TMEM address published
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (p.debug & DBG_FORCE_TIMEOUT) {
    // Test hook: one leader thread waits, with a short limit, on a barrier
    // nothing arrives on.  Its expiry takes the ordinary timeout path (abort
    // flag, status word); the abort is copied into the peer before the
    // cluster barrier, so no copy or product is issued in either CTA and
    // every role leaves at its first abort check.
    if (threadIdx.x == 0 && rank == 0) {
      mbar_wait_bounded(never, 0, abort, p.status, FORCED_LIMIT_NS);
      st_cluster_u32(mapa_shared(smem_u32(const_cast<int*>(abort)), 1), 1u);
    }
    cluster_sync_all();
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
      uint32_t armed = 0, armed_par = 0;
      for (int t = pair; t < p.total_tiles && !*abort; t += npairs) {
        const Tile tl = decode_tile(p, t);
        const TcMat& mt = p.mats[tl.g];
        const int a_mn = mt.g.flags & GF_A_MN, b_mn = mt.g.flags & GF_B_MN;
        const int a3 = mt.g.flags & GF_A_BOX3, b3 = mt.g.flags & GF_B_BOX3;
        const int m0 = tl.tm * PAIR_BM + (int)rank * HALF;
        const int n0 = tl.tn * PAIR_BN + (int)rank * HALF;
        const int nkb = (mt.g.K + BK - 1) / BK;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort, p.status, WAIT_LIMIT_NS)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          if (rank == 0) {
            mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);  // both CTAs' bytes
            armed |= 1u << stage;
            armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          const int k0 = kb * BK;
          // one copy per operand slab where the map allows (the copy
          // engine's per-copy cost makes 8 KB boxes too slow to feed the
          // tensor pipe).  Stage layout per operand: K-major [k chunk][128
          // rows][64 k]; MN-major [64-wide chunk][BK k rows][64].
          load_slab(sa, &mt.ta, bar, a_mn, a3, k0, m0);
          load_slab(sb, &mt.tb, bar, b_mn, b3, k0, n0);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      if (*abort && rank == 0) {
        // Both CTAs' copies in flight complete on the leader's barriers.
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s))
            mbar_wait_drain(&full[s], (armed_par >> s) & 1u, DRAIN_LIMIT_NS);
      }
    }
  } else if (warp == 1) {
    // ------------------------- MMA issuer (leader only) -------------------------
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      for (int t = pair; t < p.total_tiles && !*abort; t += npairs, ++local) {
        const Tile tl = decode_tile(p, t);
        const GemmMat& g = p.mats[tl.g].g;
        const int a_mn = (g.flags & GF_A_MN) ? 1 : 0, b_mn = (g.flags & GF_B_MN) ? 1 : 0;
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort, p.status, WAIT_LIMIT_NS)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * PAIR_BN);
        const uint32_t idesc = idesc_bf16(PAIR_BM, PAIR_BN, a_mn, b_mn);
        const int nkb = (g.K + BK - 1) / BK;
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
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major: k chunk kk / 4, 32 bytes per k step inside it;
            // MN-major: 16 k rows of 128 bytes per k step, chunks BK rows apart
            const uint32_t koff = (uint32_t)((kk >> 2) * CHUNK_BYTES + (kk & 3) * 32);
            const uint64_t ad = a_mn ? smem_desc(sa + kk * 2048, BK * 128, 1024)
                                     : smem_desc(sa + koff, 16, 1024);
            const uint64_t bd = b_mn ? smem_desc(sb + kk * 2048, BK * 128, 1024)
                                     : smem_desc(sb + koff, 16, 1024);
            mma_bf16_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit_pair(&empty[stage], PAIR_MASK);  // frees the stage in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc], PAIR_MASK);  // accumulator ready in both CTAs
      }
      mma_commit_pair(drain, 0x1);
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
    for (int t = pair; t < p.total_tiles; t += npairs, ++local) {
      const Tile tl = decode_tile(p, t);
      const GemmMat& g = p.mats[tl.g].g;
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      const int r = tl.tm * PAIR_BM + (int)rank * HALF + row_in_half;
      const int nch = min(PAIR_BN, g.N - tl.tn * PAIR_BN + 31) / 32;  // chunks holding columns < N
      constexpr int CH_PER = PAIR_BN / 32 / 2;
      // the first chunk's aux is in flight while the products run
      AuxPrefetch pf;
      fetch_scalars(g, pf);
      fetch_aux(g, r, r < g.M, tl.tn * PAIR_BN, half * CH_PER, half * CH_PER + CH_PER, nch, pf);
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort, p.status, WAIT_LIMIT_NS)) break;
      tc_fence_after();
      float sx = 0.f, sy = 0.f;
      epilogue_row(g, p.lr, p.decay, r, r < g.M, tl.tn * PAIR_BN,
                   tmem_base + (uint32_t)(acc * PAIR_BN) + ((uint32_t)(quarter * 32) << 16),
                   half * CH_PER, half * CH_PER + CH_PER, nch, sx, sy,
                   reinterpret_cast<__nv_bfloat16*>(smem + STAGES * STAGE_BYTES + BAR_BYTES) +
                       ew * (STAGE_TILE_BYTES / 2),
                   pf);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(&tempty[acc]);
        else
          mbar_arrive_remote(mapa_shared(smem_u32(&tempty[acc]), 0));
      }
      if (g.epi == EPI_FINAL_DIMUON) {
        // one (sum x^2, sum y^2) pair per epilogue warp; no barrier needed
        sx = warp_sum(sx);
        sy = warp_sum(sy);
        if (lane == 0) {
          const int slot = (tl.tm * g.tiles_n + tl.tn) * 16 + (int)rank * 8 + ew;
          g.part[2 * slot] = sx;
          g.part[2 * slot + 1] = sy;
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA of the pair is still addressed by the other
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace

int tc_pair_smem_bytes() { return SMEM_BYTES; }
int tc_pair_bk() { return BK; }

cudaError_t launch_tc_pair(const TcParams& p, int pairs, cudaStream_t s) {
  if (p.total_tiles <= 0 || pairs <= 0) return cudaSuccess;
  static DeviceOnce once;
  const cudaError_t e = device_once(once, nullptr, [](int) {
    return cudaFuncSetAttribute(tc_ns_product_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES);
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = (size_t)SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_ns_product_pair, p);
}

}  // namespace dm
