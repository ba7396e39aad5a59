"""Plain fp64 CPU oracle for the Muon / Dimuon optimizer step.

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously-correct
restatement of the method that the CUDA library is checked against.  Only the
test-suite, the package smoke check and the benchmark's CPU-baseline leg may
import it.  It shares no code with the CUDA path and imports nothing from it.

Sources (web pages; titles as printed, sections translated):
  [Dimuon]    "Dimuon: LoRA 에 맞춰 다시 짠 Muon" (lameproof.com optim-book,
              section "Dimuon: diagonal conditioning")
  [MuonNote]  "Muon Optimizer 정리" (dongju923.github.io)
  [Sitech]    "Muon. What happens when an LLM optimizer treats a weight matrix
              as a matrix" (sitech.ge blog)
  [PCG2Muon]  "From PCG to Muon: Preconditioner와 Optimizer의 기하학"
              (hwan-h-heo.github.io)

Every floating-point operation is carried out in numpy float64.  Rounding to a
storage dtype happens only where the step stores a tensor (the momentum M_t
and the weight W_t), using round-to-nearest-even written out below from the
bf16 format definition.

Readings taken where the pages are silent or garbled (each is listed again in
the repository's design notes):
  * The Dimuon display formula is missing from the extracted page.  The page
    says the same diagonal matrices multiply before and after
    orthogonalisation, so the step direction is R . NS(R M C) . C with one R and
    one C ([Dimuon], "-1/4 power from both sides").
  * "Relative energy" = row (column) sum of squares divided by the mean row
    (column) sum of squares.
  * R and C come from the stored previous momentum M_{t-1} itself (not from
    mu*M_{t-1}); when M_{t-1} is all zero the conditioning is off (R = C = I)
    ([Dimuon], "Why the *last* momentum").
  * "The norm is fixed afterwards" ([Dimuon], Problem 4 (c)): the conditioned
    step Y = R X_5 C is rescaled to the Frobenius norm of X_5.
  * The RMS-matching scale is kappa = coef * sqrt(max(m, n)) (coef 0.2) and is
    applied after that renormalisation ([Sitech], "From speedrun to real
    training"; [MuonNote], "Scaling up").
  * Weight decay is decoupled: W_t = (1 - lr*wd) W_{t-1} - lr * O_t
    ([MuonNote], "Scaling up": AdamW's weight decay).
  * Tall matrices are orthogonalised on their short side: X is transposed so
    that rows <= cols; R and C swap roles; the result is transposed back.
  * Degenerate norms: when ||X_0||_F is non-finite the update O_t is zero,
    W is only decayed and a flag is reported.  Below 1e-15 the update is zero
    too: that floor is not a reading of the pages (they are silent) but the
    CUDA library's implementation limit (it carries 1/||X_0||^2 as an fp32
    scalar, which overflows below it); the oracle applies the same floor so
    that the two agree.
  * Hyper-parameters reach the CUDA library as float32; the oracle rounds each
    scalar through float32 before using it in fp64 arithmetic.
  * Nesterov (optional, off by default): the matrix fed to the
    orthogonaliser is B_t = G + mu M_t, with M_t the stored momentum
    ([PCG2Muon], section 3 "Adam and Muon Optimizer": the orthogonaliser
    takes the momentum-and-Nesterov combination B_t; its formula is not
    printed, this is the standard look-ahead form).  M_t itself, and the
    energies Dimuon reads, are unchanged.
  * 1-D variables ([PCG2Muon], section 6 "Muon Reshaping"): the vector keeps
    its order in a row-major ceil(L/w) x w matrix with the cells past the end
    zero; "restored after the update" is read as keeping the first L cells.

Parity pins for every function here live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# Newton-Schulz quintic coefficients ([MuonNote], "Why orthogonalise";
# [Sitech], "Instead of SVD - Newton-Schulz").
NS_A = 3.4445
NS_B = -4.7750
NS_C = 2.0315
NS_STEPS = 5
COND_EPS = 1e-4          # [Dimuon], Problem 4: (relative energy + 1e-4)^(-1/4)
MOONSHOT_COEF = 0.2      # RMS-matching coefficient (see module docstring)
NORM_FLOOR = 1e-15      # ||X_0||_F below this: zero update (library limit, see docstring)

SCALE_NONE = 0
SCALE_MOONSHOT = 1
SCALE_JORDAN = 2
SCALE_BERNSTEIN = 3


def f32(x: float) -> float:
    """The value a Python float takes after passing through a C float."""
    return float(np.float32(x))


@dataclass
class HParams:
    """Step hyper-parameters, mirroring the C struct field by field."""
    mu: float = 0.95
    lr: float = 0.02
    weight_decay: float = 0.0
    ns_steps: int = NS_STEPS
    a: float = NS_A
    b: float = NS_B
    c: float = NS_C
    cond_eps: float = COND_EPS
    scale_mode: int = SCALE_NONE
    scale_coef: float = MOONSHOT_COEF
    nesterov: bool = False
    # Per-iteration (a_k, b_k, c_k), one triple per Newton-Schulz iteration;
    # None: the fixed (a, b, c) every iteration (see newton_schulz).
    ns_coeffs: tuple | None = None

    def as_f32(self) -> "HParams":
        coeffs = None
        if self.ns_coeffs is not None:
            coeffs = tuple((f32(a), f32(b), f32(c)) for (a, b, c) in self.ns_coeffs)
        return HParams(mu=f32(self.mu), lr=f32(self.lr),
                       weight_decay=f32(self.weight_decay),
                       ns_steps=int(self.ns_steps), a=f32(self.a),
                       b=f32(self.b), c=f32(self.c),
                       cond_eps=f32(self.cond_eps),
                       scale_mode=int(self.scale_mode),
                       scale_coef=f32(self.scale_coef), nesterov=bool(self.nesterov),
                       ns_coeffs=coeffs)


# ----------------------------------------------------------------------------
# Storage rounding (bf16 format: 1 sign bit, 8 exponent bits, 7 fraction bits,
# the exponent range of IEEE binary32).  Round to nearest, ties to even.
# ----------------------------------------------------------------------------
_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
_BF16_MIN_EXP = -133          # exponent of the smallest subnormal: 2^-126 * 2^-7


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, copy=True)
    finite = np.isfinite(x) & (x != 0.0)
    xf = x[finite]
    _, e = np.frexp(xf)                  # xf = m * 2^e, 0.5 <= |m| < 1
    # 8 significant bits: quantum 2^(e-8), never below the subnormal quantum.
    q_exp = np.maximum(e - 8, _BF16_MIN_EXP)
    q = np.ldexp(1.0, q_exp)
    r = np.rint(xf / q) * q              # np.rint rounds half to even
    r = np.where(np.abs(r) > _BF16_MAX, np.copysign(np.inf, r), r)
    out[finite] = r
    return out


def store_round(x, dtype: str) -> np.ndarray:
    """Round to the storage dtype ("bf16" or "fp32"); returned as float64."""
    if dtype == "bf16":
        return round_bf16(x)
    if dtype == "fp32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(f"unknown storage dtype {dtype!r}")


# ----------------------------------------------------------------------------
# Method steps.
# ----------------------------------------------------------------------------
def momentum_update(M_prev, G, mu: float) -> np.ndarray:
    """M_t = mu * M_{t-1} + grad ([MuonNote], "Update rule", eq. (1)).

    The stored momentum is the exact value of mu M_{t-1} + G rounded once to
    its storage type.  mu, M_{t-1} and G are float32 (or bf16) values, so the
    product is exact in float64 and the sum is exact as the float64 pair
    (s, e) of a two-sum.  The value returned is s rounded to odd with e as
    the sticky part: s itself when e = 0, else whichever of s and its float64
    neighbour on the side of e has an odd last bit.  With at least two more
    bits than the storage type, one later round-to-nearest-even to float32 or
    bf16 of this value is the correctly rounded exact value (rounding to odd
    carries the information a second rounding needs); rounding the float64
    sum s directly would round twice."""
    M_prev = np.asarray(M_prev, np.float64)
    G = np.asarray(G, np.float64)
    p = mu * M_prev                      # exact: 24-bit times 24-bit significands
    s = p + G
    bb = s - p
    e = (p - (s - bb)) + (G - bb)        # s + e = p + G exactly (two-sum)
    inexact = (e != 0.0) & np.isfinite(s)
    odd = (s.view(np.int64) & 1) == 1
    toward = np.nextafter(s, np.where(e > 0.0, np.inf, -np.inf))
    return np.where(inexact & ~odd, toward, s)


def energies(M) -> tuple[np.ndarray, np.ndarray]:
    """Row and column sums of squares of a matrix ([Dimuon], "Why the *last*
    momentum": the statistics are read from the stored momentum)."""
    M = np.asarray(M, np.float64)
    return (M * M).sum(axis=1), (M * M).sum(axis=0)


def conditioning(e_prev, eps: float = COND_EPS):
    """Diagonal of R (or C): (relative energy + eps)^(-1/4).

    [Dimuon], "-1/4 power from both sides" and Problem 4 (a).  Relative
    energy is the energy divided by the mean energy of the same vector.  A
    vector whose energies are all zero (first step, M_{t-1} = 0) switches the
    conditioning off and yields None (identity).
    """
    e = np.asarray(e_prev, np.float64)
    total = e.sum()
    if not total > 0.0:
        return None
    rel = e / (total / e.size)
    with np.errstate(divide="ignore"):
        return np.power(rel + eps, -0.25)


def frobenius_normalise(X):
    """X / ||X||_F ([Sitech], "Instead of SVD - Newton-Schulz")."""
    X = np.asarray(X, np.float64)
    nrm = math.sqrt(float((X * X).sum()))
    return (X / nrm if nrm > 0.0 else X), nrm


def newton_schulz(X, steps: int = NS_STEPS, a: float = NS_A, b: float = NS_B,
                  c: float = NS_C, coeffs=None) -> np.ndarray:
    """Quintic Newton-Schulz iteration on an already normalised X.

    Each step: A = X X^T; B = b A + c A A; X <- a X + B X, i.e.
    X <- aX + b(XX^T)X + c(XX^T)^2 X ([Sitech], "Instead of SVD -
    Newton-Schulz"; coefficients from [MuonNote], "Why orthogonalise").

    `coeffs`, when given, is a schedule: one (a_k, b_k, c_k) per iteration,
    `steps` of them, used in place of the fixed (a, b, c).  The Dimuon
    page's toy orthogonalises with Polar Express ([Dimuon], "16 columns with
    input size 0.1 to 10"), an iteration of this same form whose quintic
    changes from one iteration to the next; the page prints no
    coefficients, so only the mechanism is restated here.
    """
    X = np.asarray(X, np.float64)
    if coeffs is not None and len(coeffs) != steps:
        raise ValueError("one (a, b, c) triple per iteration")
    for k in range(steps):
        ak, bk, ck = (a, b, c) if coeffs is None else coeffs[k]
        A = X @ X.T
        B = bk * A + ck * (A @ A)
        X = ak * X + B @ X
    return X


def scale_factor(mode: int, coef: float, rows: int, cols: int) -> float:
    """Per-matrix update scale kappa, rows x cols as the caller stores the
    matrix (rows = output features).  MOONSHOT: RMS matched to AdamW
    ([Sitech], "From speedrun to real training").  That section names
    Jordan's and Bernstein's rules as different ones without formulas; they
    are read as those authors' published rules: Jordan's Muon scales by
    sqrt(max(1, rows / cols)), Bernstein's spectral scaling by
    sqrt(rows / cols).  Parity of these two is unpinned to the pages."""
    if mode == SCALE_NONE:
        return 1.0
    if mode == SCALE_MOONSHOT:
        return coef * math.sqrt(max(rows, cols))
    if mode == SCALE_JORDAN:
        return math.sqrt(max(1.0, rows / cols))
    if mode == SCALE_BERNSTEIN:
        return math.sqrt(rows / cols)
    raise ValueError(f"unknown scale mode {mode}")


@dataclass
class StepResult:
    W: np.ndarray            # W_t after storage rounding (float64 array)
    M: np.ndarray            # M_t after storage rounding
    O: np.ndarray            # the update O_t (fp64, user orientation)
    e_row: np.ndarray | None = None   # energies of the stored M_t (Dimuon)
    e_col: np.ndarray | None = None
    nonfinite: bool = False
    extras: dict = field(default_factory=dict)


def optimizer_step(W_prev, G, M_prev, hp: HParams, *, conditioned: bool,
                   e_row_prev=None, e_col_prev=None,
                   momentum_dtype: str = "fp32", weight_dtype: str = "fp32",
                   hp_through_f32: bool = True) -> StepResult:
    """One Muon (conditioned=False) or Dimuon (conditioned=True) step on one
    matrix, in the page's order:

      1. M_t = mu M_{t-1} + G, stored                ([MuonNote] eq. (1));
         with Nesterov the orthogonaliser's input is B_t = G + mu M_t
      2. orient so rows <= cols
      3. Dimuon: R, C from the energies of M_{t-1}; X_0 = R M_t C  ([Dimuon])
      4. X <- X_0 / ||X_0||_F                          ([Sitech])
      5. ns_steps quintic iterations                   ([Sitech], [MuonNote])
      6. Dimuon: Y = R X C, rescaled to ||X||_F        ([Dimuon], Problem 4)
      7. O = kappa Y                                   ([Sitech], [MuonNote])
      8. W_t = (1 - lr wd) W_{t-1} - lr O, stored      ([MuonNote] eq. (3))
    """
    if hp_through_f32:
        hp = hp.as_f32()
    W_prev = np.asarray(W_prev, np.float64)
    G = np.asarray(G, np.float64)
    M_prev = np.asarray(M_prev, np.float64)
    rows, cols = G.shape

    M_t = store_round(momentum_update(M_prev, G, hp.mu), momentum_dtype)

    R = C = None
    if conditioned:
        R = conditioning(e_row_prev, hp.cond_eps)
        C = conditioning(e_col_prev, hp.cond_eps)
        # Conditioning is switched off as a whole when M_{t-1} was zero; the
        # row and column energies of one matrix are zero together.
        if R is None or C is None:
            R = C = None

    B_t = G + hp.mu * M_t if hp.nesterov else M_t
    X0 = B_t if R is None else R[:, None] * B_t * C[None, :]
    transposed = rows > cols
    if transposed:
        X0 = X0.T

    X, nrm = frobenius_normalise(X0)
    nonfinite = not math.isfinite(nrm)
    if nonfinite or nrm < NORM_FLOOR:
        Y = np.zeros_like(X0)
    else:
        X5 = newton_schulz(X, hp.ns_steps, hp.a, hp.b, hp.c, hp.ns_coeffs)
        if R is None:
            Y = X5
        else:
            Rn, Cn = (C, R) if transposed else (R, C)
            Y = Rn[:, None] * X5 * Cn[None, :]
            ny = math.sqrt(float((Y * Y).sum()))
            nx = math.sqrt(float((X5 * X5).sum()))
            Y = Y * (nx / ny) if ny > 0.0 else np.zeros_like(Y)
    if transposed:
        Y = Y.T

    kappa = scale_factor(hp.scale_mode, hp.scale_coef, rows, cols)
    O = kappa * Y
    W_t = store_round((1.0 - hp.lr * hp.weight_decay) * W_prev - hp.lr * O,
                      weight_dtype)
    res = StepResult(W=W_t, M=M_t, O=O, nonfinite=nonfinite)
    if conditioned:
        res.e_row, res.e_col = energies(M_t)
    return res


def muon_step(W_prev, G, M_prev, hp: HParams, **kw) -> StepResult:
    """Muon step ([MuonNote], "Update rule", eq. (1)-(3))."""
    return optimizer_step(W_prev, G, M_prev, hp, conditioned=False, **kw)


def dimuon_step(W_prev, G, M_prev, e_row_prev, e_col_prev, hp: HParams,
                **kw) -> StepResult:
    """Dimuon step: Muon with diagonal conditioning from the previous
    momentum's energies ([Dimuon])."""
    return optimizer_step(W_prev, G, M_prev, hp, conditioned=True,
                          e_row_prev=e_row_prev, e_col_prev=e_col_prev, **kw)


# ----------------------------------------------------------------------------
# Reference quantities used by the pins (not part of the step itself).
# ----------------------------------------------------------------------------
# Muon on a 1-D variable ([PCG2Muon] section 6, "Muon Reshaping")
# ----------------------------------------------------------------------------
def vector_matrix_shape(length: int, width: int) -> tuple[int, int]:
    """Shape of the matrix a length-`length` vector is laid out in at a given
    width: rows = ceil(length / width), the variables kept in their order
    (row-major), the cells past the end zero."""
    if length < 1 or width < 1:
        raise ValueError("length and width must be positive")
    return -(-length // width), width


def vector_to_matrix(v, width: int) -> np.ndarray:
    """The vector in row-major order in a rows x width matrix, zero-padded
    ([PCG2Muon] section 6: the remaining cells are padded with 0)."""
    v = np.asarray(v, np.float64).reshape(-1)
    rows, cols = vector_matrix_shape(v.size, width)
    X = np.zeros(rows * cols)
    X[:v.size] = v
    return X.reshape(rows, cols)


def matrix_to_vector(X, length: int) -> np.ndarray:
    """The first `length` cells in row-major order: the padding is dropped
    after the update ([PCG2Muon] section 6: restored after the update)."""
    return np.asarray(X, np.float64).reshape(-1)[:length].copy()


def vector_step(w_prev, g, m_prev, width: int, hp: HParams, *, conditioned: bool = False,
                e_row_prev=None, e_col_prev=None, momentum_dtype: str = "fp32",
                weight_dtype: str = "fp32") -> StepResult:
    """One step on a 1-D variable: lay W, G and M out at the given width with
    zero padding, run optimizer_step on the matrices, return the first
    len(w) entries of W_t, M_t and O_t.  The padded gradient cells are zero,
    so the padded momentum cells stay zero; the padded weight cells are
    dropped.  Dimuon energies (when conditioned) belong to the padded matrix
    and are returned for it."""
    w_prev = np.asarray(w_prev, np.float64).reshape(-1)
    L = w_prev.size
    res = optimizer_step(vector_to_matrix(w_prev, width), vector_to_matrix(g, width),
                         vector_to_matrix(m_prev, width), hp, conditioned=conditioned,
                         e_row_prev=e_row_prev, e_col_prev=e_col_prev,
                         momentum_dtype=momentum_dtype, weight_dtype=weight_dtype)
    return StepResult(W=matrix_to_vector(res.W, L), M=matrix_to_vector(res.M, L),
                      O=matrix_to_vector(res.O, L), e_row=res.e_row, e_col=res.e_col,
                      nonfinite=res.nonfinite,
                      extras={"matrix": res, "padded_M": res.M.reshape(-1)[L:].copy()})


# ----------------------------------------------------------------------------
def polar_factor_svd(X) -> np.ndarray:
    """U V^T from a LAPACK SVD: the exact orthogonal polar factor that the
    iteration approximates ([MuonNote], "Newton-Schulz orthogonalisation":
    (M M^T)^(-1/2) M = U V^T)."""
    U, _, Vt = np.linalg.svd(np.asarray(X, np.float64), full_matrices=False)
    return U @ Vt


def top_column_share(O, cols) -> float:
    """Share of the step's squared Frobenius norm held by the given columns
    ([Dimuon], "16 columns with input size 0.1 to 10")."""
    O = np.asarray(O, np.float64)
    tot = float((O * O).sum())
    return float((O[:, cols] ** 2).sum()) / tot
