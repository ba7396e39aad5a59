/*
 * dimuon.h - C ABI of libdimuon.so: the Muon optimizer step for 2-D hidden
 * weight matrices, with Dimuon's diagonal conditioning as an optional mode,
 * on one NVIDIA B200 (sm_100a).
 *
 * The step, per matrix (sources: web pages, cited by title and section):
 *   1. M_t = mu M_{t-1} + G
 *        "Muon Optimizer 정리" (dongju923.github.io), "Update rule", eq. (1).
 *      With hp.nesterov the orthogonaliser's input is B_t = G + mu M_t in
 *      place of M_t below (M_t is still what is stored).
 *   2. Dimuon only: R = diag((e_row/mean(e_row) + eps)^(-1/4)),
 *      C = diag((e_col/mean(e_col) + eps)^(-1/4)) from the row / column sums
 *      of squares of the PREVIOUS momentum M_{t-1}; X_0 = R M_t C.
 *      Muon: X_0 = M_t.
 *        "Dimuon: LoRA 에 맞춰 다시 짠 Muon" (lameproof.com optim-book),
 *        "-1/4 power from both sides", "Why the *last* momentum", Problem 4.
 *   3. X <- X_0 / ||X_0||_F, then ns_steps times
 *      X <- a X + b (X X^T) X + c (X X^T)^2 X, (a,b,c) = (3.4445,-4.7750,2.0315),
 *      on the short side of the matrix (tall matrices are handled transposed).
 *        sitech.ge Muon post, "Instead of SVD - Newton-Schulz";
 *        "Muon Optimizer 정리", "Why orthogonalise".
 *      Optionally iteration k uses its own (a_k, b_k, c_k) (hp.ns_coeffs): the
 *      Dimuon page's toy orthogonalises with Polar Express, an iteration of
 *      this form whose quintic changes from one iteration to the next
 *      ("16 columns with input size 0.1 to 10").
 *   4. Dimuon only: Y = R X C rescaled to ||X||_F ("the norm is fixed
 *      afterwards", Dimuon page, Problem 4 (c)).  Muon: Y = X.
 *   5. O = kappa Y, kappa = 1 (DM_SCALE_NONE) or
 *      scale_coef * sqrt(max(rows, cols)) (DM_SCALE_MOONSHOT, RMS matched to
 *      AdamW: sitech.ge, "From speedrun to real training"), or one of the
 *      two other rules that section names without formulas (dm_scale_t).
 *   6. W_t = (1 - lr * weight_decay) W_{t-1} - lr O   (decoupled decay:
 *      "Muon Optimizer 정리", "Scaling up"; eq. (3)).
 *
 * Conventions
 *   - Every matrix is row-major and contiguous (leading dimension == cols).
 *   - All pointers in dm_matrix_t and the workspace are DEVICE pointers on the
 *     current CUDA device; hyper-parameters are host values.
 *   - The caller owns every buffer.  The library allocates no device memory
 *     and keeps no state between calls apart from a host-side cache of
 *     launch plans keyed by the workspace pointer and the matrix shapes.
 *   - dm_muon_step / dm_dimuon_step validate their arguments synchronously and
 *     return an error before launching anything; otherwise they enqueue all
 *     work on `stream` (a cudaStream_t; NULL = legacy default stream) and
 *     return without synchronising.  No C++ exception crosses this ABI.
 *   - Streams are passed as void* (a cudaStream_t cast to void*) so that the
 *     header needs no CUDA header; device status values are returned as
 *     int32_t holding a dm_status_t code, for a fixed width across
 *     compilers.
 *   - Conditions found on the device (a non-finite Frobenius norm, a bounded
 *     wait that ran out) are written to a status word inside the workspace;
 *     dm_read_device_status synchronises the stream and reads it.  Each step
 *     clears the word at its start.
 *   - After a bounded wait has run out (DM_ERR_DEVICE_TIMEOUT), every later
 *     launch of the same step returns without writing: the weights, updates,
 *     momenta and energies those launches cover keep their values, so no
 *     weight is updated from intermediate buffers that the timed-out launch
 *     left half written.  Only the launch that timed out may have written
 *     part of its own outputs (in Muon mode, the last Newton-Schulz product
 *     writes W).
 *   - Calls are re-entrant for distinct workspaces.  Two steps that share a
 *     workspace must be ordered on the device (same stream, or events).
 *   - The enqueued work contains no host synchronisation and no allocation,
 *     so a step can be captured into a CUDA graph by the caller.
 */
#ifndef DIMUON_H_
#define DIMUON_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DM_OK = 0,
  DM_ERR_INVALID_ARG = 1,     /* null pointer, non-positive shape, bad enum  */
  DM_ERR_UNSUPPORTED = 2,     /* dtype / mode combination not provided       */
  DM_ERR_WORKSPACE = 3,       /* workspace null, misaligned or too small      */
  DM_ERR_CUDA = 4,            /* a CUDA runtime / driver call failed          */
  DM_ERR_DEVICE_TIMEOUT = 5,  /* device status: a bounded wait gave up        */
  DM_ERR_NONFINITE = 6,       /* device status: non-finite ||X_0||_F; that
                                 matrix got O = 0 (its W was only decayed).
                                 A norm below 1e-15 also gives O = 0, without
                                 a status (nothing to normalise).             */
  DM_ERR_CANARY = 7           /* device status (DM_DBG_CANARY only): a canary
                                 word between workspace regions was changed
                                 during the step                              */
} dm_status_t;

typedef enum { DM_BF16 = 0, DM_FP32 = 1 } dm_dtype_t;

/* Arithmetic of the Newton-Schulz products for matrices whose short side is
 * larger than DM_THIN_MAX.  Matrices with a short side <= DM_THIN_MAX take the
 * thin-factor path (Gram iteration): fp64 sums and fp64 r x r iteration in
 * both modes, except factors of rank exactly 32 on the staged layout in
 * DM_PREC_BF16_TC mode, whose Gram and apply sums run on bf16 tensor cores
 * with hi / lo split operands (about 2^-16 relative per term) and whose r x r
 * iteration runs in fp32 (tf32 tensor cores, split operands); their update
 * agrees with the fp64 result to about 1e-5 on well-conditioned factors and
 * to about 1e-3 on factors whose column scales span many orders of
 * magnitude, inside the mode's 3e-2. */
typedef enum {
  DM_PREC_FP32 = 0,     /* fp32 SIMT products, fp32 intermediates           */
  DM_PREC_BF16_TC = 1   /* bf16 operands on tcgen05 tensor cores, fp32
                           accumulation in tensor memory                      */
} dm_precision_t;

/* Per-matrix update scale kappa; rows x cols is the matrix as the caller
 * stores it (rows = output features of an (out, in) weight).  The sitech.ge
 * post ("From speedrun to real training") names Jordan's, Moonshot's and
 * Bernstein's rules as different without printing the first and the last;
 * DM_SCALE_JORDAN and DM_SCALE_BERNSTEIN follow those authors' published
 * rules (Jordan's Muon: sqrt(max(1, out / in)); Bernstein's spectral
 * scaling: sqrt(out / in)).  scale_coef is used by DM_SCALE_MOONSHOT only. */
typedef enum {
  DM_SCALE_NONE = 0,      /* kappa = 1                                   */
  DM_SCALE_MOONSHOT = 1,  /* kappa = scale_coef * sqrt(max(rows, cols))  */
  DM_SCALE_JORDAN = 2,    /* kappa = sqrt(max(1, rows / cols))           */
  DM_SCALE_BERNSTEIN = 3  /* kappa = sqrt(rows / cols)                   */
} dm_scale_t;

#define DM_THIN_MAX 32
#define DM_MAX_NS_STEPS 64   /* largest accepted hp.ns_steps */

/* One matrix of the group.  Orientation: rows x cols as stored by the caller.
 *   weight      in/out  rows x cols, weight_dtype
 *   grad        in      rows x cols, grad_dtype
 *   momentum    in/out  rows x cols, momentum_dtype; all zero before step 1
 *   row_energy  in/out  fp32[rows]; Dimuon only (ignored by dm_muon_step):
 *                       in = row sums of squares of M_{t-1} (zeros before
 *                       step 1), out = those of the stored M_t
 *   col_energy  in/out  fp32[cols]; as row_energy, for columns
 *   update_out  out     optional fp32 rows x cols (NULL to skip): O_t       */
typedef struct {
  int64_t rows;
  int64_t cols;
  void* weight;
  int32_t weight_dtype;
  int32_t grad_dtype;
  const void* grad;
  void* momentum;
  int32_t momentum_dtype;
  int32_t reserved0;
  float* row_energy;
  float* col_energy;
  float* update_out;
} dm_matrix_t;

typedef struct {
  float mu;             /* momentum coefficient                         */
  float lr;             /* eta                                          */
  float weight_decay;   /* lambda (decoupled)                           */
  int32_t ns_steps;     /* Newton-Schulz iterations, >= 1               */
  float a, b, c;        /* quintic coefficients                         */
  float cond_eps;       /* Dimuon damping, default 1e-4                 */
  int32_t scale_mode;   /* dm_scale_t                                   */
  float scale_coef;     /* DM_SCALE_MOONSHOT coefficient, default 0.2   */
  int32_t precision;    /* dm_precision_t                               */
  uint32_t debug_flags; /* 0 in production; bits below are test hooks   */
  int32_t nesterov;     /* 1: orthogonalise B_t = G + mu M_t instead of
                           M_t ("From PCG to Muon", section 3: the
                           momentum-and-Nesterov combination)           */
  int32_t reserved[3];  /* must be zero                                 */
  const float* ns_coeffs; /* NULL: (a, b, c) above in every iteration.
                           Else a HOST array of 3 * ns_steps floats:
                           iteration k (0-based) uses (a_k, b_k, c_k) =
                           ns_coeffs[3k], ns_coeffs[3k + 1],
                           ns_coeffs[3k + 2], and a, b, c are ignored.
                           Read during the call only: the values are
                           copied into the enqueued launches (a captured
                           graph keeps them), so the array may be
                           released when the call returns.  Non-finite
                           entries are rejected with DM_ERR_INVALID_ARG. */
} dm_hparams_t;

/* debug_flags bits (test hooks; none of them changes the arithmetic) */
#define DM_DBG_NO_THIN 0x1u       /* send short-side <= DM_THIN_MAX matrices
                                     down the Newton-Schulz path as well   */
#define DM_DBG_TC_SINGLE 0x2u     /* tensor-core products on single CTAs
                                     (128 x 256 tiles) only                */
#define DM_DBG_TC_PAIR 0x4u       /* tensor-core products on CTA pairs
                                     (256 x 256 tiles) only                */
#define DM_DBG_THIN_REGS 0x10u    /* thin factors always take the register
                                     path (no shared-memory staging)       */
#define DM_DBG_THIN_STAGED 0x20u  /* thin factors take the two-pass staged
                                     kernels instead of the single-launch
                                     ones (one cluster per factor, or for
                                     r = 2 one CTA per factor)             */
#define DM_DBG_THIN_CLUSTER 0x80u /* thin factors of r = 8 take the
                                     single-launch cluster kernel as well
                                     (by default only r <= 4 does; r = 8
                                     takes the two-pass staged kernels)   */
#define DM_DBG_CANARY 0x40u      /* checked workspace: 256 canary bytes
                                     after the header and after every
                                     workspace region (dm_workspace_size
                                     grows accordingly; pass the flag to
                                     both calls).  The step fills them at
                                     its start and checks them all at its
                                     end; a changed byte sets
                                     DM_ERR_CANARY.
                                     Costs two small launches; the
                                     arithmetic is unchanged.              */
#define DM_DBG_CANARY_SELFTEST 0x100u /* checker self-test hook (with
                                     DM_DBG_CANARY): the fill leaves one
                                     canary word wrong, so the step must
                                     end with DM_ERR_CANARY                */
#define DM_DBG_FORCE_TIMEOUT 0x8u /* failure-detection hook: each
                                     tensor-core product launch makes one
                                     bounded wait run out (20 ms, on a
                                     barrier nothing arrives on) before it
                                     issues any copy or product; the launch
                                     then leaves without writing and the
                                     device status reads
                                     DM_ERR_DEVICE_TIMEOUT.  Every later
                                     launch of the step then returns at
                                     once, so W and update_out of the
                                     Newton-Schulz matrices stay as they
                                     were (their momenta, written before
                                     the first product, are updated).      */

/* Fills *hp with the defaults: mu 0.95, lr 0.02, wd 0, ns_steps 5,
 * (a,b,c) = (3.4445, -4.7750, 2.0315), cond_eps 1e-4, DM_SCALE_NONE,
 * scale_coef 0.2, DM_PREC_BF16_TC, debug_flags 0, nesterov 0,
 * ns_coeffs NULL. */
void dm_default_hparams(dm_hparams_t* hp);

/* Bytes of device workspace a step over `mats[0..n)` needs with these
 * hyper-parameters; `conditioned` = 0 for dm_muon_step, 1 for
 * dm_dimuon_step.  Host-only; touches no device memory.  The workspace must
 * be 256-byte aligned; its contents need no initialisation. */
dm_status_t dm_workspace_size(const dm_matrix_t* mats, int n,
                              const dm_hparams_t* hp, int conditioned,
                              size_t* bytes);

/* Number of kernel launches one step over `mats[0..n)` enqueues with these
 * hyper-parameters (conditioned = 0: dm_muon_step, 1: dm_dimuon_step), for
 * sizing CUDA graphs or checking a profile.  Host-only; validates like
 * dm_workspace_size. */
dm_status_t dm_step_launches(const dm_matrix_t* mats, int n, const dm_hparams_t* hp,
                             int conditioned, int64_t* launches);

/* One Muon step over the group (steps 1, 3, 5, 6 above; row_energy and
 * col_energy are ignored).  Asynchronous on `stream`. */
dm_status_t dm_muon_step(const dm_matrix_t* mats, int n,
                         const dm_hparams_t* hp, void* workspace,
                         size_t workspace_bytes, void* stream);

/* One Dimuon step over the group (steps 1-6).  row_energy / col_energy must
 * be non-null for every matrix.  Asynchronous on `stream`. */
dm_status_t dm_dimuon_step(const dm_matrix_t* mats, int n,
                           const dm_hparams_t* hp, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Synchronises `stream`, then reads the device status word of the last step
 * that used `workspace` into *out (DM_OK, DM_ERR_NONFINITE or
 * DM_ERR_DEVICE_TIMEOUT).  Returns DM_ERR_CUDA if the synchronisation or the
 * copy fails. */
dm_status_t dm_read_device_status(const void* workspace, void* stream,
                                  int32_t* out);

/* Size of the scratch array behind dm_step_noalloc: 32 MiB per GPU that
 * loads the library, held until the process exits. */
#define DM_NOALLOC_MAX_BYTES (32u * 1024u * 1024u)

/* The step (conditioned = 0: as dm_muon_step, 1: as dm_dimuon_step) without
 * a caller-provided workspace.  The pages have no counterpart: this exists
 * for callers that cannot allocate device memory, such as code running
 * inside a framework whose caching allocator has reserved the whole device,
 * or a latency-critical path where cudaMalloc / cudaFree would synchronise
 * the device.  Its scratch memory is one fixed array of
 * DM_NOALLOC_MAX_BYTES in the library's device code; the caller still passes
 * every input and output.
 *   - Groups whose dm_workspace_size exceeds DM_NOALLOC_MAX_BYTES are
 *     rejected with DM_ERR_WORKSPACE before any device work.  Thin factors
 *     (short side <= DM_THIN_MAX) need a little scratch per 512-2048 long-side
 *     columns (fp64 Gram partials) and per factor; 448 LoRA factors of rank
 *     32 and width 4096 need about 22 MB.
 *   - The first call on a device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress); make that first call before
 *     any stream capture.
 *   - Every call shares the one array and leaves its contents behind; the step
 *     zeroes its header (status word, slab counters) itself and needs nothing
 *     else zeroed.  Calls whose
 *     device work overlaps (different streams or threads without ordering)
 *     race on the array: order them on the device.
 *   - device_status_out (nullable, device int32) receives the step's device
 *     status word (as dm_read_device_status would report it), asynchronously.
 *   - Calls no allocating routine (no cudaMalloc, cudaFree or library
 *     allocator). */
dm_status_t dm_step_noalloc(const dm_matrix_t* mats, int n,
                            const dm_hparams_t* hp, int conditioned,
                            int32_t* device_status_out, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* dm_status_string(int32_t status);

/* Library version, "major.minor.patch". */
const char* dm_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DIMUON_H_ */
