// Internal (non-ABI) definitions of libdimuon: kernel parameter blocks,
// workspace scalar slots and the launch entry points of each kernel file.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace dm {

// One-time set-up of a launcher (kernel attributes, occupancy queries), run
// once per device with that device current, safe under concurrent callers.
// Each launcher keeps its own static DeviceOnce; a failed set-up is
// remembered and returned on every later call on that device.
constexpr int MAX_DEVICES = 64;
struct DeviceOnce {
  std::once_flag flag[MAX_DEVICES];
  cudaError_t err[MAX_DEVICES] = {};
};
template <class F>
inline cudaError_t device_once(DeviceOnce& once, int* dev_out, F&& init) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  std::call_once(once.flag[dev], [&] { once.err[dev] = init(dev); });
  if (dev_out) *dev_out = dev;
  return once.err[dev];
}

enum { DT_BF16 = 0, DT_FP32 = 1 };

// Per-matrix scalar slots (float[SC_COUNT] in the workspace).
enum {
  SC_SUMSQ = 0,   // ||X_0||_F^2 of the stored X_0
  SC_INV_S = 1,   // 1 / max(||X_0||_F, 1e-30)
  SC_INV_S2 = 2,  // its square
  SC_VALID = 3,   // 1 when ||X_0||_F is finite, else 0 (update forced to 0)
  SC_FINAL = 4,   // Dimuon: kappa * ||X_5||_F / ||R X_5 C||_F (0 if invalid)
  SC_COUNT = 16
};

// Device status codes (mirror dm_status_t).
enum { ST_OK = 0, ST_TIMEOUT = 5, ST_NONFINITE = 6, ST_CANARY = 7 };
// int32 index, after the status word, of the step's abort word (set with
// ST_TIMEOUT; both live in the workspace header that each step clears).
constexpr int STATUS_ABORT_WORD = 1;

// debug_flags bit read inside the tensor-core kernels (mirrors the public
// DM_DBG_FORCE_TIMEOUT).
constexpr unsigned DBG_FORCE_TIMEOUT = 0x8u;

// ------------------------------- K0 ---------------------------------------
// Dimuon conditioning vectors R, C from the previous momentum's energies.
struct K0Mat {
  const float* e_row;
  const float* e_col;
  float* R;
  float* C;
  int64_t rows, cols;
};
constexpr int K0_MAX = 256;
struct K0Params {
  int count;
  float eps;
  K0Mat mats[K0_MAX];
};

// ------------------------------- K1 ---------------------------------------
// Momentum update, X_0 = R M_t C (or M_t), partial sums of squares, partial
// row / column energies.  Tiles of K1_ROWS x K1_COLS.
constexpr int K1_ROWS = 64;
constexpr int K1_COLS = 256;
struct K1Mat {
  const void* G;
  void* M;
  void* X0;
  const float* R;          // null: no conditioning
  const float* C;
  float* part_sumsq;       // [n_rt * n_ct]
  float* part_erow;        // [n_ct][rows], null: energies not needed
  float* part_ecol;        // [n_rt][cols]
  int64_t rows, cols, ldx;
  int gdt, mdt, xdt, vec;
  int n_rt, n_ct;
};
constexpr int K1_MAX = 200;
struct K1Params {
  int count;
  float mu;
  int* status;
  int nesterov;           // X_0 from B_t = G + mu M_t instead of M_t
  int starts[K1_MAX + 1];
  K1Mat mats[K1_MAX];
};

// ------------------------------- K1b --------------------------------------
// Reduction of the K1 partials: energies of M_t and the norm scalars.
constexpr int K1B_THREADS = 256;
struct K1bMat {
  const float* part_sumsq;
  const float* part_erow;
  const float* part_ecol;
  float* e_row;            // user output, null in Muon mode
  float* e_col;
  float* scal;
  int64_t rows, cols;
  int n_rt, n_ct;
};
constexpr int K1B_MAX = 200;
struct K1bParams {
  int count;
  int* status;
  int starts[K1B_MAX + 1];  // blocks per matrix: 1 + energy blocks
  K1bMat mats[K1B_MAX];
};

// --------------------------- NS products ----------------------------------
enum {
  EPI_SYRK = 0,          // out = S * acc                       (symmetric)
  EPI_POLY = 1,          // out = c * acc + b * aux             (symmetric)
  EPI_GEMM = 2,          // out = S * (acc + a * aux)
  EPI_FINAL_MUON = 3,    // W <- decay W - lr kappa S (acc + a aux), upd = O
  EPI_FINAL_DIMUON = 4   // out = S (acc + a aux) = X_5, plus norm partials
};

// One product of one matrix.  Output tile grid tiles_m x tiles_n; `sym`
// enumerates only tiles that meet the upper triangle and mirrors them.
struct GemmMat {
  void* out;
  const void* aux;
  const float* scal;      // per-matrix scalar slots
  void* W;                // final epilogues
  float* upd;
  const float* R;         // Dimuon final: user-orientation R and C
  const float* C;
  float* part;            // Dimuon final: per-tile (sum x^2, sum y^2)
  int ldo, ldaux, ldw;
  int M, N, K;
  int tiles_m, tiles_n;
  int flags;              // bit0 a_mn, bit1 b_mn, bit2 sym, bit3 n-fast raster
  int epi;                // EPI_*
  int scal_idx;           // slot multiplying the result, -1 for none
  int wdt;                // weight dtype
  float coef_acc, coef_aux, kappa;
};
// GF_A_BOX3 / GF_B_BOX3: the pair kernel's operand map is a chunked 3-D map
// (one copy per operand slab of a stage)
enum { GF_A_MN = 1, GF_B_MN = 2, GF_SYM = 4, GF_N_FAST = 8, GF_A_BOX3 = 16, GF_B_BOX3 = 32 };

// fp32 SIMT products
constexpr int SIMT_MAX = 120;
// A operand element (i, k) at a_mn ? a[k*lda + i] : a[i*lda + k];
// B operand element (j, k) at b_mn ? b[k*ldb + j] : b[j*ldb + k].
struct SimtMat {
  GemmMat g;
  const float* a;
  const float* b;
  int lda, ldb;
};
struct SimtParams {
  int count;
  float lr, decay;
  int* status;
  int starts[SIMT_MAX + 1];
  SimtMat mats[SIMT_MAX];
};

// tcgen05 products (bf16 operands, fp32 accumulation in TMEM)
constexpr int TC_BM = 128, TC_BN = 256, TC_BK = 64;
struct TcMat {
  CUtensorMap ta;   // A-operand map, bf16, 128-byte swizzle (box per kernel: see the host)
  CUtensorMap tb;   // B-operand map
  GemmMat g;
};
constexpr int TC_MAX = 76;
struct TcParams {
  int count;
  int total_tiles;
  float lr, decay;
  int* status;
  unsigned debug;
  int starts[TC_MAX + 1];
  TcMat mats[TC_MAX];
};

// ------------------------------- K3 ---------------------------------------
struct K3Mat {
  const void* X5;
  void* W;
  float* upd;
  const float* R;
  const float* C;
  const float* part;
  float* scal;
  int64_t rows, cols, ldx;
  int xdt, wdt, vec, n_part;
  int n_rt, n_ct;
  float kappa;
};
constexpr int K3_MAX = 200;
struct K3Params {
  int count;
  float lr, decay;
  int* status;
  int starts[K3_MAX + 1];
  K3Mat mats[K3_MAX];
};

// ------------------------------ thin --------------------------------------
// Whole step of short-side <= 32 factors (Gram route): per padded short
// side, thin_setup copies the factor descriptors into the workspace (up to
// THIN_MAX per launch) and sums the previous energies; thin_gram,
// thin_iterate and thin_apply then cover every factor of that padded side,
// the streaming two in slabs of thin_slab(pad) long-side columns (handed out
// by a device counter in the register kernels, as contiguous per-CTA ranges
// in the staged ones).
struct ThinMat {           // 64 bytes
  const void* G;
  void* M;
  void* W;
  float* upd;
  float* e_row;           // user orientation, null in Muon mode
  float* e_col;
  int32_t rows, cols;
  uint8_t gdt, mdt, wdt;
  uint8_t vec;            // G, M, W, upd all 16-byte aligned
  float kappa;
};
constexpr int THIN_MAX = 448;  // descriptors per setup launch (kernel parameter space)
struct ThinSetupParams {
  int count;              // factors in this launch (<= THIN_MAX)
  int first;              // their first index in the group
  int conditioned;
  ThinMat* mats_dst;      // group descriptor table (device)
  int* starts_dst;        // group slab starts (device), count + 1 entries written
  int* unit_f_dst;        // group slab -> factor table (device)
  double* fsc;            // group per-factor scalars (device)
  int starts[THIN_MAX + 1];
  ThinMat mats[THIN_MAX];
};
struct ThinParams {
  int count;              // factors in the group
  int pad;                // padded short side (1, 2, 3, 4, 8, 16, 32)
  int units;              // slabs over all factors
  int grid_gram, grid_apply;  // persistent grid sizes
  int conditioned;
  int nesterov;
  int ns_steps;
  int split;              // r = 32 staged passes: Gram and apply sums on bf16 tensor
                          // cores with hi / lo split operands (bf16 tensor-core mode)
  float mu, lr, decay, eps;
  float coef[64][3];      // (a_k, b_k, c_k) of Newton-Schulz iteration k < ns_steps
  int* status;
  const ThinMat* mats;    // [count]
  const int* starts;      // [count + 1]: first slab of each factor
  const int* unit_f;      // [units]: factor of each slab
  double* part;           // [units][2][thin_part_doubles(pad)]: S_1, S_2 slab partials
  float* rpart;           // [units][pad]: short-side energy partials
  double* T;              // [count][pad * pad]: apply matrices
  double* fsc;            // [count][4]: sums of the previous long- / short-side
                          // energies, conditioning on, zero update
  int* counters;          // [2]: next slab of thin_gram / thin_apply (zero at the start)
};
static_assert(sizeof(ThinMat) == 64, "ThinMat packing");
static_assert(sizeof(ThinSetupParams) <= 32764, "kernel parameter space");
int thin_part_doubles(int pad);
// Single-pass thin step (one CTA per factor, r = pad = 2, the factor's
// momentum and, under Nesterov, gradient kept in shared memory).
constexpr size_t THIN_FUSED_MAX_SMEM = 96 * 1024;
size_t thin_fused_smem(int pad, int64_t n, bool nesterov);
cudaError_t launch_thin_fused(const ThinParams& p, size_t smem, cudaStream_t s);
int thin_slab(int pad);

// ----------------------------- canaries -----------------------------------
// Checked-workspace mode: 256-byte canaries (64 words) at the listed 256-byte
// blocks of the workspace.  mode 0 (step start): fill; mode 1 (step end):
// check.  `plant` (self-test hook) leaves the first word of the first canary
// wrong at the fill.
constexpr uint32_t CANARY_FILL = 0xA5C3A5C3u;
constexpr int CANARY_MAX = 7000;          // canaries per launch
struct CanaryParams {
  int count;
  int mode;
  int plant;
  int* status;                // the workspace base (status word first)
  uint32_t blk[CANARY_MAX];   // canary offsets / 256
};
static_assert(sizeof(CanaryParams) <= 32764, "kernel parameter space");
cudaError_t launch_canary(const CanaryParams& p, cudaStream_t s);

// ------------------------------ launches ----------------------------------
cudaError_t launch_k0(const K0Params& p, cudaStream_t s);
cudaError_t launch_k1(const K1Params& p, int total_tiles, cudaStream_t s);
cudaError_t launch_k1b(const K1bParams& p, int total_blocks, cudaStream_t s);
cudaError_t launch_k3a(const K3Params& p, cudaStream_t s);
cudaError_t launch_k3(const K3Params& p, int total_tiles, cudaStream_t s);
// tile: 128 (128 x 128 tiles) or 64 (64 x 64 tiles)
cudaError_t launch_simt(const SimtParams& p, int total_tiles, int tile, cudaStream_t s);
cudaError_t launch_tc(const TcParams& p, int grid, cudaStream_t s);
int tc_smem_bytes();
constexpr int TC2_BM = 256, TC2_BN = 256;  // CTA-pair output tile
cudaError_t launch_tc_pair(const TcParams& p, int pairs, cudaStream_t s);
int tc_pair_smem_bytes();
int tc_pair_bk();  // k per stage of the pair kernel (box shapes of its maps)
cudaError_t launch_thin_setup(const ThinSetupParams& p, cudaStream_t s);
cudaError_t launch_thin(ThinParams& p, int nsm, cudaStream_t s);
cudaError_t launch_thin_iterate(const ThinParams& p, cudaStream_t s);
// shared-memory staged thin path (k_thin_bulk.cu)
int thin_bulk_combo(int gdt, int mdt, int wdt);
cudaError_t launch_thin_bulk(ThinParams& p, int combo, int nsm, cudaStream_t s);
// single-launch cluster path (k_thin_cluster.cu): one cluster of cs CTAs per
// factor, the factor held in the cluster's shared memory; r = pad in {2, 4, 8},
// long side a multiple of 8 cs, staged storage combinations and alignment
constexpr int THIN_CL_MAX = 448;      // factors per launch (kernel parameter space)
constexpr int THIN_CL_MAX_CS = 8;     // portable cluster size
constexpr size_t THIN_CL_MAX_SMEM = 200 * 1024;
struct ThinClusterParams {
  int count;              // factors (clusters) in this launch
  int conditioned;
  int nesterov;
  int ns_steps;
  float mu, lr, decay, eps;
  float coef[64][3];      // (a_k, b_k, c_k) of Newton-Schulz iteration k
  int* status;
  ThinMat mats[THIN_CL_MAX];
};
static_assert(sizeof(ThinClusterParams) <= 32764, "kernel parameter space");
// Dynamic shared memory of one CTA (0 if this (pad, combo, cs, n) has no kernel).
size_t thin_cluster_smem(int pad, int combo, int cs, int64_t n, bool tall, bool nest);
cudaError_t launch_thin_cluster(const ThinClusterParams& p, int pad, int combo, int cs, size_t smem,
                                cudaStream_t s);

}  // namespace dm
