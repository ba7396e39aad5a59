// Host side of libdimuon.so: argument validation, workspace layout, launch
// planning and the C ABI declared in include/dimuon.h.
//
// Step order (one stream, no host synchronisation):
//   status word cleared
//   thin factors (short side <= DM_THIN_MAX): thin_gram, thin_iterate,
//        thin_apply per padded short side (Gram route, whole step)
//   other matrices:
//     K0   (Dimuon) R, C from the previous momentum's energies
//     K1   momentum, X_0 = R M_t C, partial norms / energies
//     K1b  energies of M_t, ||X_0||_F scalars
//     ns_steps x { A = X X^T ; B = b_k A + c_k A^2 ; X <- a_k X + BX }  (tensor cores
//          in DM_PREC_BF16_TC, fp32 SIMT in DM_PREC_FP32); the last product
//          applies the Muon update or emits X_5
//     K3a, K3 (Dimuon) renormalise Y = R X_5 C, scale, decay, apply
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "dimuon.h"
#include "dm_internal.h"
#include "dm_tiles.cuh"

namespace dm {
namespace {

constexpr size_t HEADER_BYTES = 1024;
constexpr int64_t MAX_DIM = int64_t(1) << 24;
constexpr int64_t MAX_ELEMS = (int64_t(1) << 31) - 1;

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

struct MatPlan {
  int idx;
  bool thin;
  int64_t rows, cols;
  int m, n;
  bool tall;
  int64_t ldx, ldm;
  int k1_rt, k1_ct;
  int n_part;
  size_t off_scal, off_R, off_C, off_psum, off_perow, off_pecol, off_pfin;
  size_t off_X[2], off_A, off_B;
};

// One group of thin factors launched together (same padded short side).
struct ThinLaunch {
  int pad;
  int combo;                // storage combination of the staged path, -1 = register path
  int cs = 0;               // CTAs per factor of the single-launch cluster kernel, 0 = not used
  bool fused = false;       // r = 2 single-pass kernel (one CTA per factor)
  size_t fused_smem = 0;
  std::vector<int> idx;     // matrix indices
  std::vector<int> starts;  // first slab of each factor, plus the total
  size_t off_mats, off_starts, off_unit_f, off_part, off_rpart, off_T, off_fsc;
};

// Header of the workspace: the device status word at 0, the thin slab
// counters (two per group) from THIN_CTR_OFFSET; zeroed at the start of a step.
constexpr size_t THIN_CTR_OFFSET = 64;

int thin_pad(int r) { return r <= 4 ? r : r <= 8 ? 8 : r <= 16 ? 16 : 32; }

// Shared memory per CTA the cluster kernel's slices may take: with the
// kernel's static arrays four to five CTAs stay resident per SM.
#ifndef DM_THIN_CL_BUDGET_KB
#define DM_THIN_CL_BUDGET_KB 40
#endif
constexpr size_t THIN_CL_BUDGET = DM_THIN_CL_BUDGET_KB * 1024;

struct Layout {
  std::vector<MatPlan> mats;
  std::vector<ThinLaunch> thin;
  std::vector<uint32_t> canary;  // checked mode: 256-byte canary blocks (offset / 256)
  size_t bytes = 0;
  bool tc = false;
  bool cond = false;
};

dm_status_t validate(const dm_matrix_t* mats, int n, const dm_hparams_t* hp, int cond) {
  if (n < 0 || (n > 0 && !mats) || !hp) return DM_ERR_INVALID_ARG;
  if (hp->ns_steps < 1 || hp->ns_steps > DM_MAX_NS_STEPS) return DM_ERR_INVALID_ARG;
  if (hp->ns_coeffs)
    for (int i = 0; i < 3 * hp->ns_steps; ++i) {
      const float v = hp->ns_coeffs[i];
      if (!(v == v) || v > 3.0e38f || v < -3.0e38f) return DM_ERR_INVALID_ARG;
    }
  if (hp->precision != DM_PREC_FP32 && hp->precision != DM_PREC_BF16_TC) return DM_ERR_INVALID_ARG;
  if (hp->scale_mode != DM_SCALE_NONE && hp->scale_mode != DM_SCALE_MOONSHOT &&
      hp->scale_mode != DM_SCALE_JORDAN && hp->scale_mode != DM_SCALE_BERNSTEIN)
    return DM_ERR_INVALID_ARG;
  const float scalars[] = {hp->mu, hp->lr, hp->weight_decay, hp->a, hp->b, hp->c, hp->cond_eps,
                           hp->scale_coef};
  for (float v : scalars)
    if (!(v == v) || v > 3.0e38f || v < -3.0e38f) return DM_ERR_INVALID_ARG;
  if (cond && !(hp->cond_eps >= 0.f)) return DM_ERR_INVALID_ARG;
  if (hp->nesterov != 0 && hp->nesterov != 1) return DM_ERR_INVALID_ARG;
  if (hp->reserved[0] || hp->reserved[1] || hp->reserved[2]) return DM_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const dm_matrix_t& m = mats[i];
    if (m.rows < 1 || m.cols < 1 || m.rows > MAX_DIM || m.cols > MAX_DIM ||
        m.rows * m.cols > MAX_ELEMS)
      return DM_ERR_INVALID_ARG;
    if (!m.weight || !m.grad || !m.momentum) return DM_ERR_INVALID_ARG;
    const int32_t dts[] = {m.weight_dtype, m.grad_dtype, m.momentum_dtype};
    for (int32_t d : dts)
      if (d != DM_BF16 && d != DM_FP32) return DM_ERR_UNSUPPORTED;
    if (cond && (!m.row_energy || !m.col_energy)) return DM_ERR_INVALID_ARG;
  }
  return DM_OK;
}

Layout make_layout(const dm_matrix_t* mats, int n, const dm_hparams_t* hp, int cond) {
  Layout L;
  L.tc = hp->precision == DM_PREC_BF16_TC;
  L.cond = cond != 0;
  const size_t esz = L.tc ? 2 : 4;
  const bool canaries = (hp->debug_flags & DM_DBG_CANARY) != 0;
  size_t cur = HEADER_BYTES;
  // checked mode: a 256-byte canary after the header and after every region
  auto guard = [&]() {
    if (!canaries) return;
    cur = round_up(cur, 256);
    L.canary.push_back((uint32_t)(cur / 256));
    cur += 256;
  };
  guard();
  auto take = [&](size_t bytes, size_t align) {
    cur = round_up(cur, align);
    const size_t o = cur;
    cur += round_up(bytes, 16);
    guard();
    return o;
  };
  for (int i = 0; i < n; ++i) {
    MatPlan p{};
    p.idx = i;
    p.rows = mats[i].rows;
    p.cols = mats[i].cols;
    p.tall = p.rows > p.cols;
    p.m = (int)std::min(p.rows, p.cols);
    p.n = (int)std::max(p.rows, p.cols);
    p.thin = p.m <= DM_THIN_MAX && !(hp->debug_flags & DM_DBG_NO_THIN);
    if (!p.thin) {
      // rows padded to whole 64-element chunks, so a chunked (3-D) operand
      // map never reads past the end of a row
      p.ldx = (int64_t)round_up((size_t)p.cols, 64);
      p.ldm = (int64_t)round_up((size_t)p.m, 64);
      p.k1_rt = (int)ceil_div(p.rows, K1_ROWS);
      p.k1_ct = (int)ceil_div(p.cols, K1_COLS);
      if (L.tc)  // enough (sum x^2, sum y^2) slots for either tensor-core kernel
        p.n_part = (int)std::max(ceil_div(p.rows, TC_BM) * ceil_div(p.cols, TC_BN) * 8,
                                 ceil_div(p.rows, TC2_BM) * ceil_div(p.cols, TC2_BN) * 16);
      else  // fp32 products: one (sum x^2, sum y^2) per tile, tiles of 64 at the most
        p.n_part = (int)(ceil_div(p.rows, 64) * ceil_div(p.cols, 64));
      p.off_scal = take(SC_COUNT * sizeof(float), 256);
      p.off_psum = take((size_t)p.k1_rt * p.k1_ct * sizeof(float), 256);
      if (L.cond) {
        p.off_R = take((size_t)p.rows * sizeof(float), 256);
        p.off_C = take((size_t)p.cols * sizeof(float), 256);
        p.off_perow = take((size_t)p.k1_ct * p.rows * sizeof(float), 256);
        p.off_pecol = take((size_t)p.k1_rt * p.cols * sizeof(float), 256);
        p.off_pfin = take((size_t)p.n_part * 2 * sizeof(float), 256);
      }
      for (int b = 0; b < 2; ++b) p.off_X[b] = take((size_t)p.rows * p.ldx * esz, 1024);
      p.off_A = take((size_t)p.m * p.ldm * esz, 1024);
      p.off_B = take((size_t)p.m * p.ldm * esz, 1024);
    }
    L.mats.push_back(p);
  }
  // thin factors: one launch group per padded short side and path (staged
  // path for r == pad, long side a multiple of 8 (any length for tall factors
  // with r >= 8: each staged row is then whole 16-byte groups), 16-byte
  // aligned buffers and a supported storage combination; register path
  // otherwise)
  auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  std::vector<std::pair<int, int>> pads;
  std::vector<std::vector<int>> members;
  for (const MatPlan& p : L.mats) {
    if (!p.thin) continue;
    const int pad = thin_pad(p.m);
    const dm_matrix_t& um = mats[p.idx];
    int combo = thin_bulk_combo(um.grad_dtype, um.momentum_dtype, um.weight_dtype);
    const bool ok = p.m == pad && pad >= 2 && pad != 3 && (p.n % 8 == 0 || (p.tall && pad >= 8)) &&
                    al16(um.grad) &&
                    al16(um.momentum) && al16(um.weight) && al16(um.update_out) &&
                    (!cond || (al16(um.row_energy) && al16(um.col_energy)));
    if (!ok || (hp->debug_flags & DM_DBG_THIN_REGS)) combo = -1;
    const std::pair<int, int> key(pad, combo);
    size_t g = 0;
    while (g < pads.size() && pads[g] != key) ++g;
    if (g == pads.size()) {
      pads.push_back(key);
      members.emplace_back();
    }
    members[g].push_back(p.idx);
  }
  for (size_t g = 0; g < pads.size(); ++g) {
    ThinLaunch tl;
    tl.pad = pads[g].first;
    tl.combo = pads[g].second;
    tl.idx = members[g];
    const int slab = thin_slab(tl.pad);
    tl.starts.push_back(0);
    for (int i : tl.idx) tl.starts.push_back(tl.starts.back() + (int)ceil_div(L.mats[i].n, slab));
    const size_t units = (size_t)tl.starts.back(), count = tl.idx.size();
    tl.off_mats = take(count * sizeof(ThinMat), 256);
    tl.off_starts = take((count + 1) * sizeof(int), 256);
    tl.off_unit_f = take(units * sizeof(int), 256);
    tl.off_part = take(units * 2 * thin_part_doubles(tl.pad) * sizeof(double), 256);
    tl.off_rpart = take(units * tl.pad * sizeof(float), 256);
    tl.off_T = take(count * tl.pad * tl.pad * sizeof(double), 256);
    tl.off_fsc = take(count * 4 * sizeof(double), 256);
    // single-launch cluster kernel: the smallest cluster whose per-CTA slice
    // of every factor of the group fits the budget.  By default for r <= 4;
    // at r = 8 the two-pass staged kernels measured faster on the LoRA batch
    // (448 factors of width 4096: 0.109 against 0.150 ms per step), so the
    // cluster kernel takes r = 8 only under DM_DBG_THIN_CLUSTER.
    const bool cl_pad = tl.pad == 2 || tl.pad == 4 ||
                        (tl.pad == 8 && (hp->debug_flags & DM_DBG_THIN_CLUSTER));
    if (tl.combo >= 0 && cl_pad && !(hp->debug_flags & (DM_DBG_THIN_STAGED | DM_DBG_THIN_REGS))) {
      for (int cs = 1; cs <= THIN_CL_MAX_CS && !tl.cs; cs *= 2) {
        bool ok = true;
        for (int i : tl.idx) {
          const MatPlan& p = L.mats[i];
          const size_t b = thin_cluster_smem(tl.pad, tl.combo, cs, p.n, p.tall, hp->nesterov != 0);
          ok = ok && b > 0 && b <= THIN_CL_BUDGET;
        }
        if (ok) tl.cs = cs;
      }
    }
    // else r = 2 on the staged layout whose momentum (and Nesterov gradient)
    // fits one CTA's shared memory: the single-pass kernel
    if (!tl.cs) {
      int64_t max_n = 0;
      for (int i : tl.idx) max_n = std::max<int64_t>(max_n, L.mats[i].n);
      tl.fused_smem = thin_fused_smem(tl.pad, max_n, hp->nesterov != 0);
      tl.fused = tl.combo >= 0 && tl.pad == 2 && tl.fused_smem <= THIN_FUSED_MAX_SMEM &&
                 !(hp->debug_flags & DM_DBG_THIN_STAGED);
    }
    L.thin.push_back(std::move(tl));
  }
  L.bytes = round_up(cur, 1024);
  return L;
}

// ------------------------------ tensor maps -------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 matrix [outer][inner] with leading dimension ld (elements); boxes of
// 64 inner x `rows` outer elements with the 128-byte swizzle the UMMA
// descriptors expect (64 x 64 for the single-CTA kernel, 64 x 128 for one
// CTA's K-major operand slab in the pair kernel).
bool make_map(CUtensorMap* map, void* ptr, int64_t inner, int64_t outer, int64_t ld, int rows = 64) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same matrix seen as 64-element chunks of its rows: dims (element in
// chunk, row, chunk), box 64 x `rows` rows x `chunks` chunks, laid out
// [chunk][row][64] in shared memory (the layout 64-wide 2-D boxes stacked
// chunk by chunk give).  Used for one CTA's operand slab in one copy:
// MN-major slabs (2 chunks of 64 output rows/columns x BK k rows) and
// K-major slabs (BK / 64 chunks of k x 128 rows).  Needs ld >= the chunk
// count x 64 (rows are padded to whole chunks); the padding is read, so a
// K-major (chunks along k) map is only built when the inner extent is a
// multiple of 64.  Returns false if the driver does not take the map; the
// caller then falls back to 2-D boxes.
bool make_map3(CUtensorMap* map, void* ptr, int64_t inner, int64_t outer, int64_t ld, int rows,
               int chunks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || ld < (int64_t)round_up((size_t)inner, 64)) return false;
  cuuint64_t dims[3] = {64, (cuuint64_t)outer, (cuuint64_t)ceil_div(inner, 64)};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), 128};
  cuuint32_t box[3] = {64, (cuuint32_t)rows, (cuuint32_t)chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Operand maps of one matrix's buffers (X[0], X[1], A, B): 64 x 64 boxes,
// 64 x 128 boxes, chunked 3-D maps for MN-major slabs (valid when has3) and
// for K-major slabs of 128 k (valid when hask3[b]).
struct MatMaps {
  CUtensorMap m64[4], m128[4], m3[4], k3[4];
  bool has3, hask3[4];
};

std::mutex g_cache_mu;
std::unordered_map<std::string, std::vector<MatMaps>> g_map_cache;

std::string cache_key(const Layout& L, const void* ws, int dev) {
  std::string k;
  auto put = [&](const void* p, size_t n) { k.append(reinterpret_cast<const char*>(p), n); };
  put(&ws, sizeof(ws));
  put(&dev, sizeof(dev));
  for (const MatPlan& p : L.mats) {
    if (p.thin) continue;
    put(&p.rows, sizeof(p.rows));
    put(&p.cols, sizeof(p.cols));
    put(&p.off_X[0], sizeof(size_t));
  }
  return k;
}

bool get_maps(const Layout& L, uint8_t* ws, int dev, std::vector<MatMaps>& out) {
  const std::string key = cache_key(L, ws, dev);
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    auto it = g_map_cache.find(key);
    if (it != g_map_cache.end()) {
      out = it->second;
      return true;
    }
  }
  out.assign(L.mats.size(), MatMaps{});
  for (size_t i = 0; i < L.mats.size(); ++i) {
    const MatPlan& p = L.mats[i];
    if (p.thin) continue;
    MatMaps& mm = out[i];
    mm.has3 = true;
    for (int b = 0; b < 4; ++b) {
      uint8_t* base = ws + (b < 2 ? p.off_X[b] : b == 2 ? p.off_A : p.off_B);
      const int64_t inner = b < 2 ? p.cols : p.m, outer = b < 2 ? p.rows : p.m;
      const int64_t ld = b < 2 ? p.ldx : p.ldm;
      if (!make_map(&mm.m64[b], base, inner, outer, ld, 64)) return false;
      if (!make_map(&mm.m128[b], base, inner, outer, ld, 128)) return false;
      const int bk = tc_pair_bk();
      mm.has3 = mm.has3 && make_map3(&mm.m3[b], base, inner, outer, ld, bk, 2);
      mm.hask3[b] = bk == 128 && inner % 64 == 0 && make_map3(&mm.k3[b], base, inner, outer, ld, 128, 2);
    }
  }
  std::lock_guard<std::mutex> lk(g_cache_mu);
  if (g_map_cache.size() > 64) g_map_cache.clear();
  g_map_cache[key] = out;
  return true;
}

int sm_count(int dev) {
  static std::mutex mu;
  static std::unordered_map<int, int> cache;
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    v = 148;
  cache[dev] = v;
  return v;
}

// ---------------------------- product plans -------------------------------
enum Phase { PH_SYRK = 0, PH_POLY = 1, PH_GEMM = 2 };

// (a, b, c) of Newton-Schulz iteration k (1-based): the caller's schedule
// when it gave one, else the fixed quintic.
struct Coef {
  float a, b, c;
};
Coef coef_of(const dm_hparams_t* hp, int k) {
  if (!hp->ns_coeffs) return {hp->a, hp->b, hp->c};
  const float* q = hp->ns_coeffs + 3 * (k - 1);
  return {q[0], q[1], q[2]};
}

// Fills the epilogue / shape part of one product; operand sources are set by
// the caller (tensor maps or pointers).  Returns operand-source descriptors.
struct OperandSrc {
  int a_buf, b_buf;   // 0/1 = X buffer, 2 = A, 3 = B
};

OperandSrc fill_gemm(GemmMat& g, const MatPlan& p, const dm_matrix_t& um, const dm_hparams_t* hp,
                     uint8_t* ws, int phase, int k, bool cond, float kappa, int bm, int bn) {
  std::memset(&g, 0, sizeof(g));
  const int ns = hp->ns_steps;
  const int xin = (k - 1) & 1, xout = k & 1;
  float* scal = reinterpret_cast<float*>(ws + p.off_scal);
  g.scal = scal;
  g.scal_idx = -1;
  OperandSrc src{};
  if (phase == PH_SYRK) {
    g.M = g.N = p.m;
    g.K = p.n;
    g.flags = GF_SYM | (p.tall ? (GF_A_MN | GF_B_MN) : 0);
    g.out = ws + p.off_A;
    g.ldo = (int)p.ldm;
    g.epi = EPI_SYRK;
    if (k == 1) g.scal_idx = SC_INV_S2;
    src = {xin, xin};
  } else if (phase == PH_POLY) {
    g.M = g.N = p.m;
    g.K = p.m;
    g.flags = GF_SYM;
    g.out = ws + p.off_B;
    g.ldo = (int)p.ldm;
    g.aux = ws + p.off_A;
    g.ldaux = (int)p.ldm;
    g.epi = EPI_POLY;
    g.coef_acc = coef_of(hp, k).c;
    g.coef_aux = coef_of(hp, k).b;
    src = {2, 2};
  } else {
    g.M = (int)p.rows;
    g.N = (int)p.cols;
    g.K = p.m;
    if (p.tall) {
      g.flags = GF_N_FAST;
      src = {xin, 3};
    } else {
      g.flags = GF_B_MN;
      src = {3, xin};
    }
    g.aux = ws + p.off_X[xin];
    g.ldaux = (int)p.ldx;
    g.coef_aux = coef_of(hp, k).a;
    if (k == 1) g.scal_idx = SC_INV_S;
    if (k < ns) {
      g.epi = EPI_GEMM;
      g.out = ws + p.off_X[xout];
      g.ldo = (int)p.ldx;
    } else if (!cond) {
      g.epi = EPI_FINAL_MUON;
      g.W = um.weight;
      g.wdt = um.weight_dtype;
      g.ldw = (int)p.cols;
      g.upd = um.update_out;
      g.kappa = kappa;
    } else {
      g.epi = EPI_FINAL_DIMUON;
      g.out = ws + p.off_X[xout];
      g.ldo = (int)p.ldx;
      g.R = reinterpret_cast<const float*>(ws + p.off_R);
      g.C = reinterpret_cast<const float*>(ws + p.off_C);
      g.part = reinterpret_cast<float*>(ws + p.off_pfin);
    }
  }
  g.tiles_m = (int)ceil_div(g.M, bm);
  g.tiles_n = (int)ceil_div(g.N, bn);
  return src;
}

// Per-matrix update scale (dm_scale_t), rows x cols in the caller's orientation.
float kappa_of(const dm_hparams_t* hp, int64_t rows, int64_t cols) {
  switch (hp->scale_mode) {
    case DM_SCALE_MOONSHOT:
      return (float)((double)hp->scale_coef * std::sqrt((double)std::max(rows, cols)));
    case DM_SCALE_JORDAN:
      return (float)std::sqrt(std::max(1.0, (double)rows / (double)cols));
    case DM_SCALE_BERNSTEIN:
      return (float)std::sqrt((double)rows / (double)cols);
    default:
      return 1.f;
  }
}

#define DM_CUDA(x)                          \
  do {                                      \
    if ((x) != cudaSuccess) return DM_ERR_CUDA; \
  } while (0)

dm_status_t run_body(const dm_matrix_t* mats, int n, const dm_hparams_t* hp, const Layout& L,
                     uint8_t* ws, cudaStream_t s, int cond, int dev);

dm_status_t run_step(const dm_matrix_t* mats, int n, const dm_hparams_t* hp, void* workspace,
                     size_t ws_bytes, void* stream_v, int cond) {
  dm_status_t st = validate(mats, n, hp, cond);
  if (st != DM_OK) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DM_ERR_WORKSPACE;
  const Layout L = make_layout(mats, n, hp, cond);
  if (ws_bytes < L.bytes) return DM_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream_v);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  int dev = 0;
  DM_CUDA(cudaGetDevice(&dev));

  // status word and thin slab counters
  const bool canaries = !L.canary.empty();
  DM_CUDA(cudaMemsetAsync(ws, 0, THIN_CTR_OFFSET + 2 * sizeof(int) * L.thin.size(), s));
  auto canary_pass = [&](int mode) -> cudaError_t {
    static thread_local CanaryParams cp;
    for (size_t b = 0; b < L.canary.size(); b += CANARY_MAX) {
      cp.count = (int)std::min<size_t>(CANARY_MAX, L.canary.size() - b);
      cp.mode = mode;
      cp.plant = (hp->debug_flags & DM_DBG_CANARY_SELFTEST) != 0 && b == 0;
      cp.status = status;
      std::memcpy(cp.blk, L.canary.data() + b, sizeof(uint32_t) * cp.count);
      const cudaError_t e = launch_canary(cp, s);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  };
  if (canaries) DM_CUDA(canary_pass(0));
  const dm_status_t body = run_body(mats, n, hp, L, ws, s, cond, dev);
  if (body != DM_OK) return body;
  if (canaries) DM_CUDA(canary_pass(1));
  return DM_OK;
}

// The step's kernels (between the header clear and the canary check).
dm_status_t run_body(const dm_matrix_t* mats, int n, const dm_hparams_t* hp, const Layout& L,
                     uint8_t* ws, cudaStream_t s, int cond, int dev) {
  int* status = reinterpret_cast<int*>(ws);
  const float decay = 1.f - hp->lr * hp->weight_decay;
  if (n == 0) return DM_OK;

  // ---------------------------- thin factors -------------------------------
  for (size_t gi = 0; gi < L.thin.size(); ++gi) {
    const ThinLaunch& tl = L.thin[gi];
    auto thin_desc = [&](int idx) {
      const dm_matrix_t& um = mats[idx];
      ThinMat t;
      std::memset(&t, 0, sizeof(t));
      t.G = um.grad;
      t.M = um.momentum;
      t.W = um.weight;
      t.upd = um.update_out;
      t.e_row = cond ? um.row_energy : nullptr;
      t.e_col = cond ? um.col_energy : nullptr;
      t.rows = (int32_t)um.rows;
      t.cols = (int32_t)um.cols;
      t.gdt = (uint8_t)um.grad_dtype;
      t.mdt = (uint8_t)um.momentum_dtype;
      t.wdt = (uint8_t)um.weight_dtype;
      t.kappa = kappa_of(hp, um.rows, um.cols);
      auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
      t.vec = (uint8_t)(al16(um.grad) && al16(um.momentum) && al16(um.weight) && al16(um.update_out));
      return t;
    };
    if (tl.cs > 0) {
      // one launch per THIN_CL_MAX factors, no set-up launch, no workspace
      const int count = (int)tl.idx.size();
      for (int first = 0; first < count; first += THIN_CL_MAX) {
        static thread_local ThinClusterParams cp;
        std::memset(&cp, 0, sizeof(cp));
        cp.count = std::min(THIN_CL_MAX, count - first);
        cp.conditioned = cond;
        cp.nesterov = hp->nesterov;
        cp.ns_steps = hp->ns_steps;
        cp.mu = hp->mu;
        cp.lr = hp->lr;
        cp.decay = decay;
        cp.eps = hp->cond_eps;
        for (int k = 1; k <= hp->ns_steps; ++k) {
          const Coef q = coef_of(hp, k);
          cp.coef[k - 1][0] = q.a;
          cp.coef[k - 1][1] = q.b;
          cp.coef[k - 1][2] = q.c;
        }
        cp.status = status;
        size_t smem = 0;
        for (int q = 0; q < cp.count; ++q) {
          const int i = tl.idx[first + q];
          cp.mats[q] = thin_desc(i);
          smem = std::max(smem, thin_cluster_smem(tl.pad, tl.combo, tl.cs, L.mats[i].n, L.mats[i].tall,
                                                  hp->nesterov != 0));
        }
        DM_CUDA(launch_thin_cluster(cp, tl.pad, tl.combo, tl.cs, smem, s));
      }
      continue;
    }
    ThinMat* mats_dev = reinterpret_cast<ThinMat*>(ws + tl.off_mats);
    int* starts_dev = reinterpret_cast<int*>(ws + tl.off_starts);
    double* fsc = reinterpret_cast<double*>(ws + tl.off_fsc);
    const int count = (int)tl.idx.size();
    for (int first = 0; first < count; first += THIN_MAX) {
      static thread_local ThinSetupParams sp;
      std::memset(&sp, 0, sizeof(sp));
      sp.count = std::min(THIN_MAX, count - first);
      sp.first = first;
      sp.conditioned = cond;
      sp.mats_dst = mats_dev;
      sp.starts_dst = starts_dev;
      sp.unit_f_dst = reinterpret_cast<int*>(ws + tl.off_unit_f);
      sp.fsc = fsc;
      for (int q = 0; q <= sp.count; ++q) sp.starts[q] = tl.starts[first + q];
      for (int q = 0; q < sp.count; ++q) sp.mats[q] = thin_desc(tl.idx[first + q]);
      DM_CUDA(launch_thin_setup(sp, s));
    }
    ThinParams tp;
    std::memset(&tp, 0, sizeof(tp));
    tp.count = count;
    tp.pad = tl.pad;
    tp.units = tl.starts.back();
    tp.conditioned = cond;
    tp.nesterov = hp->nesterov;
    tp.ns_steps = hp->ns_steps;
    // bf16 tensor-core mode: the staged r = 32 passes take their sums on
    // bf16 tensor cores (split operands, fp32 accumulation) and the r x r
    // iteration in fp32; fp32 mode and the register path keep fp64
    tp.split = L.tc && tl.pad == 32 && tl.combo >= 0 && !tl.fused && !tl.cs ? 1 : 0;
    tp.mu = hp->mu;
    tp.lr = hp->lr;
    tp.decay = decay;
    for (int k = 1; k <= hp->ns_steps; ++k) {
      const Coef q = coef_of(hp, k);
      tp.coef[k - 1][0] = q.a;
      tp.coef[k - 1][1] = q.b;
      tp.coef[k - 1][2] = q.c;
    }
    tp.eps = hp->cond_eps;
    tp.status = status;
    tp.mats = mats_dev;
    tp.starts = starts_dev;
    tp.unit_f = reinterpret_cast<const int*>(ws + tl.off_unit_f);
    tp.part = reinterpret_cast<double*>(ws + tl.off_part);
    tp.rpart = reinterpret_cast<float*>(ws + tl.off_rpart);
    tp.T = reinterpret_cast<double*>(ws + tl.off_T);
    tp.fsc = fsc;
    tp.counters = reinterpret_cast<int*>(ws + THIN_CTR_OFFSET) + 2 * gi;
    if (tl.fused)
      DM_CUDA(launch_thin_fused(tp, tl.fused_smem, s));
    else if (tl.combo >= 0)
      DM_CUDA(launch_thin_bulk(tp, tl.combo, sm_count(dev), s));
    else
      DM_CUDA(launch_thin(tp, sm_count(dev), s));
  }

  // -------------------------- Newton-Schulz path ---------------------------
  std::vector<const MatPlan*> big;
  for (const MatPlan& p : L.mats)
    if (!p.thin) big.push_back(&p);
  if (big.empty()) return DM_OK;
  // heaviest products first, so the persistent grid ends with small tiles
  std::stable_sort(big.begin(), big.end(), [](const MatPlan* a, const MatPlan* b) {
    return (double)a->m * a->m * a->n > (double)b->m * b->m * b->n;
  });
  const int xdt = L.tc ? DT_BF16 : DT_FP32;

  // K0
  if (cond) {
    static thread_local K0Params p0;
    for (size_t b = 0; b < big.size(); b += K0_MAX) {
      std::memset(&p0, 0, sizeof(p0));
      p0.eps = hp->cond_eps;
      for (size_t q = b; q < std::min(big.size(), b + K0_MAX); ++q) {
        const MatPlan& p = *big[q];
        const dm_matrix_t& um = mats[p.idx];
        K0Mat& k = p0.mats[p0.count++];
        k.e_row = um.row_energy;
        k.e_col = um.col_energy;
        k.R = reinterpret_cast<float*>(ws + p.off_R);
        k.C = reinterpret_cast<float*>(ws + p.off_C);
        k.rows = p.rows;
        k.cols = p.cols;
      }
      DM_CUDA(launch_k0(p0, s));
    }
  }
  // K1
  {
    static thread_local K1Params p1;
    for (size_t b = 0; b < big.size(); b += K1_MAX) {
      std::memset(&p1, 0, sizeof(p1));
      p1.mu = hp->mu;
      p1.nesterov = hp->nesterov;
      p1.status = status;
      int tiles = 0;
      for (size_t q = b; q < std::min(big.size(), b + K1_MAX); ++q) {
        const MatPlan& p = *big[q];
        const dm_matrix_t& um = mats[p.idx];
        p1.starts[p1.count] = tiles;
        K1Mat& k = p1.mats[p1.count++];
        k.G = um.grad;
        k.M = um.momentum;
        k.X0 = ws + p.off_X[0];
        k.R = cond ? reinterpret_cast<const float*>(ws + p.off_R) : nullptr;
        k.C = cond ? reinterpret_cast<const float*>(ws + p.off_C) : nullptr;
        k.part_sumsq = reinterpret_cast<float*>(ws + p.off_psum);
        k.part_erow = cond ? reinterpret_cast<float*>(ws + p.off_perow) : nullptr;
        k.part_ecol = cond ? reinterpret_cast<float*>(ws + p.off_pecol) : nullptr;
        k.rows = p.rows;
        k.cols = p.cols;
        k.ldx = p.ldx;
        k.gdt = um.grad_dtype;
        k.mdt = um.momentum_dtype;
        k.xdt = xdt;
        k.vec = (p.cols % 8 == 0) && !(reinterpret_cast<uintptr_t>(um.grad) & 15u) &&
                !(reinterpret_cast<uintptr_t>(um.momentum) & 15u);
        k.n_rt = p.k1_rt;
        k.n_ct = p.k1_ct;
        tiles += p.k1_rt * p.k1_ct;
      }
      p1.starts[p1.count] = tiles;
      DM_CUDA(launch_k1(p1, tiles, s));
    }
  }
  // K1b
  {
    static thread_local K1bParams pb;
    for (size_t b = 0; b < big.size(); b += K1B_MAX) {
      std::memset(&pb, 0, sizeof(pb));
      pb.status = status;
      int blocks = 0;
      for (size_t q = b; q < std::min(big.size(), b + K1B_MAX); ++q) {
        const MatPlan& p = *big[q];
        const dm_matrix_t& um = mats[p.idx];
        pb.starts[pb.count] = blocks;
        K1bMat& k = pb.mats[pb.count++];
        k.part_sumsq = reinterpret_cast<const float*>(ws + p.off_psum);
        k.part_erow = cond ? reinterpret_cast<const float*>(ws + p.off_perow) : nullptr;
        k.part_ecol = cond ? reinterpret_cast<const float*>(ws + p.off_pecol) : nullptr;
        k.e_row = cond ? um.row_energy : nullptr;
        k.e_col = cond ? um.col_energy : nullptr;
        k.scal = reinterpret_cast<float*>(ws + p.off_scal);
        k.rows = p.rows;
        k.cols = p.cols;
        k.n_rt = p.k1_rt;
        k.n_ct = p.k1_ct;
        blocks += 1 + (cond ? (int)ceil_div(p.rows + p.cols, K1B_THREADS) : 0);
      }
      pb.starts[pb.count] = blocks;
      DM_CUDA(launch_k1b(pb, blocks, s));
    }
  }
  // Newton-Schulz products
  std::vector<int> final_npart(n, 0);  // partial slots the last product wrote
  if (L.tc) {
    std::vector<MatMaps> maps;
    if (!get_maps(L, ws, dev, maps)) return DM_ERR_CUDA;
    const int nsm = sm_count(dev);
    static thread_local TcParams pt;
    auto build = [&](size_t b, int ph, int k, int bm, int bn, bool pair) {
      std::memset(&pt, 0, sizeof(pt));
      pt.status = status;
      pt.lr = hp->lr;
      pt.decay = decay;
      pt.debug = hp->debug_flags;
      int tiles = 0;
      for (size_t q = b; q < std::min(big.size(), b + TC_MAX); ++q) {
        const MatPlan& p = *big[q];
        TcMat& tm = pt.mats[pt.count];
        const OperandSrc src = fill_gemm(tm.g, p, mats[p.idx], hp, ws, ph, k, cond != 0,
                                         kappa_of(hp, p.rows, p.cols), bm, bn);
        const MatMaps& mm = maps[p.idx];
        // single-CTA kernel: 64 x 64 boxes; pair kernel: one copy per slab
        // (chunked maps) where the maps allow, else 64 x 128 boxes (K-major)
        // or 64 x 64 boxes (MN-major)
        auto pick = [&](int buf, bool mn, int box3_flag) -> const CUtensorMap& {
          if (!pair) return mm.m64[buf];
          if (!mn) {
            if (mm.hask3[buf]) {
              tm.g.flags |= box3_flag;
              return mm.k3[buf];
            }
            return mm.m128[buf];
          }
          if (mm.has3) {
            tm.g.flags |= box3_flag;
            return mm.m3[buf];
          }
          return mm.m64[buf];
        };
        tm.ta = pick(src.a_buf, (tm.g.flags & GF_A_MN) != 0, GF_A_BOX3);
        tm.tb = pick(src.b_buf, (tm.g.flags & GF_B_MN) != 0, GF_B_BOX3);
        pt.starts[pt.count++] = tiles;
        tiles += gemm_tile_count(tm.g, bm, bn);
      }
      pt.starts[pt.count] = tiles;
      pt.total_tiles = tiles;
      return tiles;
    };
    for (int k = 1; k <= hp->ns_steps; ++k)
      for (int ph = 0; ph < 3; ++ph)
        for (size_t b = 0; b < big.size(); b += TC_MAX) {
          const int pair_tiles = build(b, ph, k, TC2_BM, TC2_BN, true);
          // CTA pairs (256 x 256 tiles) measured at least as fast as single
          // CTAs on every workload tried, including one 1024^2 matrix
          bool pair = true;
          if (hp->debug_flags & DM_DBG_TC_PAIR) pair = true;
          if (hp->debug_flags & DM_DBG_TC_SINGLE) pair = false;
          if (pair) {
            DM_CUDA(launch_tc_pair(pt, std::min(pair_tiles, nsm / 2), s));
          } else {
            const int tiles = build(b, ph, k, TC_BM, TC_BN, false);
            DM_CUDA(launch_tc(pt, std::min(tiles, nsm), s));
          }
          if (k == hp->ns_steps && ph == PH_GEMM)
            for (size_t q = b; q < std::min(big.size(), b + TC_MAX); ++q) {
              const MatPlan& p = *big[q];
              final_npart[p.idx] =
                  pair ? (int)(ceil_div(p.rows, TC2_BM) * ceil_div(p.cols, TC2_BN) * 16)
                       : (int)(ceil_div(p.rows, TC_BM) * ceil_div(p.cols, TC_BN) * 8);
            }
        }
  } else {
    static thread_local SimtParams ps;
    const int nsm = sm_count(dev);
    auto build_simt = [&](size_t b, int ph, int k, int tb) {
          std::memset(&ps, 0, sizeof(ps));
          ps.lr = hp->lr;
          ps.decay = decay;
          ps.status = status;
          int tiles = 0;
          for (size_t q = b; q < std::min(big.size(), b + SIMT_MAX); ++q) {
            const MatPlan& p = *big[q];
            SimtMat& sm = ps.mats[ps.count];
            const OperandSrc src = fill_gemm(sm.g, p, mats[p.idx], hp, ws, ph, k, cond != 0,
                                             kappa_of(hp, p.rows, p.cols), tb, tb);
            auto ptr = [&](int buf) -> const float* {
              return reinterpret_cast<const float*>(
                  ws + (buf < 2 ? p.off_X[buf] : (buf == 2 ? p.off_A : p.off_B)));
            };
            auto ld = [&](int buf) -> int { return (int)(buf < 2 ? p.ldx : p.ldm); };
            sm.a = ptr(src.a_buf);
            sm.b = ptr(src.b_buf);
            sm.lda = ld(src.a_buf);
            sm.ldb = ld(src.b_buf);
            ps.starts[ps.count++] = tiles;
            tiles += gemm_tile_count(sm.g, tb, tb);
          }
          ps.starts[ps.count] = tiles;
          return tiles;
    };
    for (int k = 1; k <= hp->ns_steps; ++k)
      for (int ph = 0; ph < 3; ++ph)
        for (size_t b = 0; b < big.size(); b += SIMT_MAX) {
          // 128 x 128 tiles, or 64 x 64 when those would leave SMs idle
          int tb = 128;
          int tiles = build_simt(b, ph, k, tb);
          if (tiles < 2 * nsm) {
            tb = 64;
            tiles = build_simt(b, ph, k, tb);
          }
          DM_CUDA(launch_simt(ps, tiles, tb, s));
          if (k == hp->ns_steps && ph == PH_GEMM)
            for (size_t q = b; q < std::min(big.size(), b + SIMT_MAX); ++q) {
              const MatPlan& p = *big[q];
              final_npart[p.idx] = (int)(ceil_div(p.rows, tb) * ceil_div(p.cols, tb));
            }
        }
  }
  // K3a / K3
  if (cond) {
    static thread_local K3Params p3;
    for (size_t b = 0; b < big.size(); b += K3_MAX) {
      std::memset(&p3, 0, sizeof(p3));
      p3.lr = hp->lr;
      p3.decay = decay;
      p3.status = status;
      int tiles = 0;
      for (size_t q = b; q < std::min(big.size(), b + K3_MAX); ++q) {
        const MatPlan& p = *big[q];
        const dm_matrix_t& um = mats[p.idx];
        p3.starts[p3.count] = tiles;
        K3Mat& k = p3.mats[p3.count++];
        k.X5 = ws + p.off_X[hp->ns_steps & 1];
        k.W = um.weight;
        k.upd = um.update_out;
        k.R = reinterpret_cast<const float*>(ws + p.off_R);
        k.C = reinterpret_cast<const float*>(ws + p.off_C);
        k.part = reinterpret_cast<const float*>(ws + p.off_pfin);
        k.scal = reinterpret_cast<float*>(ws + p.off_scal);
        k.rows = p.rows;
        k.cols = p.cols;
        k.ldx = p.ldx;
        k.xdt = xdt;
        k.wdt = um.weight_dtype;
        k.vec = (p.cols % 8 == 0) && !(reinterpret_cast<uintptr_t>(um.weight) & 15u) &&
                !(reinterpret_cast<uintptr_t>(um.update_out) & 15u);
        k.n_part = final_npart[p.idx];
        k.n_rt = p.k1_rt;
        k.n_ct = p.k1_ct;
        k.kappa = kappa_of(hp, p.rows, p.cols);
        tiles += p.k1_rt * p.k1_ct;
      }
      p3.starts[p3.count] = tiles;
      DM_CUDA(launch_k3a(p3, s));
      DM_CUDA(launch_k3(p3, tiles, s));
    }
  }
  return DM_OK;
}

// Kernel launches run_step enqueues for this layout (the header memset is
// not a kernel).
int64_t count_launches(const Layout& L, const dm_hparams_t* hp, int cond) {
  auto chunks = [](int64_t count, int64_t per) { return (count + per - 1) / per; };
  int64_t k = 0;
  for (const ThinLaunch& tl : L.thin) {
    const int64_t count = (int64_t)tl.idx.size();
    if (tl.cs > 0)
      k += chunks(count, THIN_CL_MAX);
    else
      k += chunks(count, THIN_MAX) + (tl.fused ? 1 : 3);
  }
  k += 2 * (int64_t)((L.canary.size() + CANARY_MAX - 1) / CANARY_MAX);
  int64_t big = 0;
  for (const MatPlan& p : L.mats) big += p.thin ? 0 : 1;
  if (big == 0) return k;
  if (cond) k += chunks(big, K0_MAX);
  k += chunks(big, K1_MAX) + chunks(big, K1B_MAX);
  k += (int64_t)hp->ns_steps * 3 * chunks(big, L.tc ? TC_MAX : SIMT_MAX);
  if (cond) k += 2 * chunks(big, K3_MAX);
  return k;
}

}  // namespace
}  // namespace dm

extern "C" {

void dm_default_hparams(dm_hparams_t* hp) {
  if (!hp) return;
  hp->mu = 0.95f;
  hp->lr = 0.02f;
  hp->weight_decay = 0.f;
  hp->ns_steps = 5;
  hp->a = 3.4445f;
  hp->b = -4.7750f;
  hp->c = 2.0315f;
  hp->cond_eps = 1e-4f;
  hp->scale_mode = DM_SCALE_NONE;
  hp->scale_coef = 0.2f;
  hp->precision = DM_PREC_BF16_TC;
  hp->debug_flags = 0;
  hp->nesterov = 0;
  hp->reserved[0] = hp->reserved[1] = hp->reserved[2] = 0;
  hp->ns_coeffs = nullptr;
}

dm_status_t dm_workspace_size(const dm_matrix_t* mats, int n, const dm_hparams_t* hp,
                              int conditioned, size_t* bytes) {
  if (!bytes) return DM_ERR_INVALID_ARG;
  try {
    const dm_status_t st = dm::validate(mats, n, hp, conditioned);
    if (st != DM_OK) return st;
    *bytes = dm::make_layout(mats, n, hp, conditioned).bytes;
    return DM_OK;
  } catch (...) {
    return DM_ERR_INVALID_ARG;
  }
}

dm_status_t dm_step_launches(const dm_matrix_t* mats, int n, const dm_hparams_t* hp,
                             int conditioned, int64_t* launches) {
  if (!launches) return DM_ERR_INVALID_ARG;
  try {
    const dm_status_t st = dm::validate(mats, n, hp, conditioned);
    if (st != DM_OK) return st;
    *launches = dm::count_launches(dm::make_layout(mats, n, hp, conditioned), hp, conditioned);
    return DM_OK;
  } catch (...) {
    return DM_ERR_INVALID_ARG;
  }
}

dm_status_t dm_muon_step(const dm_matrix_t* mats, int n, const dm_hparams_t* hp, void* workspace,
                         size_t workspace_bytes, void* stream) {
  try {
    return dm::run_step(mats, n, hp, workspace, workspace_bytes, stream, 0);
  } catch (...) {
    return DM_ERR_CUDA;
  }
}

dm_status_t dm_dimuon_step(const dm_matrix_t* mats, int n, const dm_hparams_t* hp,
                           void* workspace, size_t workspace_bytes, void* stream) {
  try {
    return dm::run_step(mats, n, hp, workspace, workspace_bytes, stream, 1);
  } catch (...) {
    return DM_ERR_CUDA;
  }
}

dm_status_t dm_read_device_status(const void* workspace, void* stream, int32_t* out) {
  if (!workspace || !out) return DM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DM_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DM_ERR_CUDA;
  *out = v;
  return DM_OK;
}

const char* dm_status_string(int32_t status) {
  switch (status) {
    case DM_OK: return "ok";
    case DM_ERR_INVALID_ARG: return "invalid argument";
    case DM_ERR_UNSUPPORTED: return "unsupported dtype or mode";
    case DM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DM_ERR_CUDA: return "CUDA call failed";
    case DM_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case DM_ERR_NONFINITE: return "non-finite Frobenius norm (update set to zero)";
    case DM_ERR_CANARY: return "workspace canary overwritten";
    default: return "unknown status";
  }
}

const char* dm_version(void) { return "0.2.0"; }

}  // extern "C"
