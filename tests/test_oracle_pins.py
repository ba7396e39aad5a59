"""Pins that tie the fp64 oracle to what the pages and the mathematics fix.

Each test states the passage it follows.  None of them re-derives a value by
re-typing the oracle's own formula: they use values printed on the pages
(tests/golden), closed forms from the spectral calculus (SVD / eigh),
invariants of the method, library routines (torch's bf16 cast) and
pure-Python brute force on tiny inputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle as orc
import workloads
from rounding_cases import crafted_bf16_tie, crafted_fp32_tie

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# --------------------------------------------------------------------------
# helpers that are independent of the oracle
# --------------------------------------------------------------------------
def quintic_scalar(x, a, b, c, steps):
    """The scalar odd polynomial p(x) = a x + b x^3 + c x^5 applied `steps`
    times (Muon Optimizer 정리, 'Why orthogonalise')."""
    for _ in range(steps):
        x = a * x + b * x ** 3 + c * x ** 5
    return x


def bf_matmul(A, B):
    n, k = len(A), len(A[0])
    m = len(B[0])
    return [[sum(A[i][p] * B[p][j] for p in range(k)) for j in range(m)]
            for i in range(n)]


def bf_transpose(A):
    return [list(r) for r in zip(*A)]


def brute_force_step(W, G, M, mu, lr, wd, a, b, c, steps, eps, kappa_coef,
                     moonshot, e_row=None, e_col=None, nesterov=False, coeffs=None):
    """Pure-Python restatement of one step on a tiny matrix (lists of floats).
    Orientation is handled by transposing when rows > cols.  `coeffs`: one
    (a, b, c) per iteration in place of the fixed triple."""
    rows, cols = len(G), len(G[0])
    # the stored momentum (fp32 storage) is what the rest of the step reads
    Mt = [[float(np.float32(mu * M[i][j] + G[i][j])) for j in range(cols)]
          for i in range(rows)]
    Rv = Cv = None
    if e_row is not None and sum(e_row) > 0:
        mr = sum(e_row) / rows
        mc = sum(e_col) / cols
        Rv = [(e / mr + eps) ** -0.25 for e in e_row]
        Cv = [(e / mc + eps) ** -0.25 for e in e_col]
    Bt = [[G[i][j] + mu * Mt[i][j] if nesterov else Mt[i][j] for j in range(cols)]
          for i in range(rows)]
    X0 = [[Bt[i][j] * (Rv[i] * Cv[j] if Rv else 1.0) for j in range(cols)]
          for i in range(rows)]
    tall = rows > cols
    if tall:
        X0 = bf_transpose(X0)
    nrm = math.sqrt(sum(v * v for r in X0 for v in r))
    X = [[v / nrm for v in r] for r in X0]
    for it in range(steps):
        if coeffs is not None:
            a, b, c = coeffs[it]
        A = bf_matmul(X, bf_transpose(X))
        AA = bf_matmul(A, A)
        Bm = [[b * A[i][j] + c * AA[i][j] for j in range(len(A))]
              for i in range(len(A))]
        BX = bf_matmul(Bm, X)
        X = [[a * X[i][j] + BX[i][j] for j in range(len(X[0]))]
             for i in range(len(X))]
    if tall:
        X = bf_transpose(X)
    if Rv:
        Y = [[Rv[i] * X[i][j] * Cv[j] for j in range(cols)] for i in range(rows)]
        nx = math.sqrt(sum(v * v for r in X for v in r))
        ny = math.sqrt(sum(v * v for r in Y for v in r))
        Y = [[v * nx / ny for v in r] for r in Y]
    else:
        Y = X
    kappa = kappa_coef * math.sqrt(max(rows, cols)) if moonshot else 1.0
    O = [[kappa * v for v in r] for r in Y]
    Wn = [[(1 - lr * wd) * W[i][j] - lr * O[i][j] for j in range(cols)]
          for i in range(rows)]
    er = [sum(v * v for v in r) for r in Mt]
    ec = [sum(Mt[i][j] ** 2 for i in range(rows)) for j in range(cols)]
    return Wn, Mt, O, er, ec


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------
def test_bf16_rounding_matches_torch_cast():
    """Round-to-nearest-even to bf16 agrees with torch's fp32->bf16 cast on
    fp32 inputs (ties, subnormals, large values, signs)."""
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8),
                  2.0 ** -130, 3 * 2.0 ** -134, 3.3e38, -3.3e38, 0.0, -0.0]),
        # exact ties between neighbouring bf16 values
        (np.arange(1, 2000) * 2.0 + 1.0) * 2.0 ** -9,
    ]).astype(np.float32)
    want = torch.from_numpy(vals).bfloat16().float().numpy().astype(np.float64)
    got = orc.round_bf16(vals.astype(np.float64))
    np.testing.assert_array_equal(got, want)


# --------------------------------------------------------------------------
# conditioning (Dimuon page, Problem 4)
# --------------------------------------------------------------------------
def _energies_with_relative(rel):
    # append one filler entry so that the mean of the vector is exactly 1
    rel = list(rel)
    filler = (len(rel) + 1) - sum(rel)
    return np.array(rel + [filler])


def test_conditioning_values_problem4(golden):
    g = golden("conditioning_problem4.json")
    e = _energies_with_relative(g["relative_energy"])
    R = orc.conditioning(e, 1e-4)[: len(g["relative_energy"])]
    np.testing.assert_allclose(np.round(R, g["printed_decimals"]), g["with_eps"],
                               atol=0)
    R0 = orc.conditioning(e, 0.0)[: len(g["relative_energy"])]
    want = [float(v) if v != "inf" else math.inf for v in g["without_eps"]]
    assert math.isinf(R0[-1])
    np.testing.assert_allclose(np.round(R0[:-1], g["printed_decimals"]), want[:-1],
                               atol=0)


def test_conditioning_caps(golden):
    """Per-side gain <= 10, per-entry gain <= 100; a row whose previous
    energy was zero gets exactly the cap (Problem 4 (b), (c))."""
    g = golden("conditioning_problem4.json")
    rng = np.random.default_rng(3)
    for _ in range(50):
        e_r = rng.exponential(1.0, 37) * (rng.random(37) < 0.7)
        e_c = rng.exponential(1.0, 53) ** 4
        if e_r.sum() == 0:
            continue
        R = orc.conditioning(e_r)
        C = orc.conditioning(e_c)
        assert R.max() <= g["per_side_cap"] * (1 + 1e-12)
        assert (R[:, None] * C[None, :]).max() <= g["max_entry_gain"] * (1 + 1e-12)
        np.testing.assert_allclose(R[e_r == 0], g["per_side_cap"], rtol=1e-12)


def test_conditioning_off_when_previous_momentum_zero():
    """'Why the *last* momentum': at step 1 M_0 = 0 and conditioning is off."""
    assert orc.conditioning(np.zeros(8)) is None


# --------------------------------------------------------------------------
# the toy (Dimuon page, '16 columns with input size 0.1 to 10')
# --------------------------------------------------------------------------
def test_toy_column_norms(golden):
    g = golden("toy_lora_4x16.json")
    G, s = workloads.toy_lora_factor()
    assert G.shape == tuple(g["shape"])
    norms = np.linalg.norm(G, axis=0)
    assert round(norms.min(), 3) == g["col_norm_min"]
    assert round(norms.max()) == g["col_norm_max"]


def test_toy_muon_top4_share(golden):
    g = golden("toy_lora_4x16.json")
    G, _ = workloads.toy_lora_factor()
    r = orc.muon_step(np.zeros_like(G), G, np.zeros_like(G), orc.HParams())
    share = orc.top_column_share(r.O, [12, 13, 14, 15])
    assert round(share, 2) == g["muon_top4_share"]


def test_adam_sign_share(golden):
    g = golden("adam_first_step.json")
    G, _ = workloads.toy_lora_factor()
    assert orc.top_column_share(np.sign(G), [12, 13, 14, 15]) == g["top4_share"]


def test_toy_dimuon_moves_energy_off_large_columns(golden):
    """Step 2 of the toy is conditioned by step 1's momentum; the share of
    the 4 largest-input columns falls far below Muon's and below Adam's
    sign step (the page prints 19 %, from a different orthogonaliser)."""
    g = golden("toy_lora_4x16.json")
    G, _ = workloads.toy_lora_factor()
    hp = orc.HParams()
    Z = np.zeros_like(G)
    s1 = orc.dimuon_step(Z, G, Z, np.zeros(4), np.zeros(16), hp)
    s2 = orc.dimuon_step(s1.W, G, s1.M, s1.e_row, s1.e_col, hp)
    share1 = orc.top_column_share(s1.O, [12, 13, 14, 15])
    share2 = orc.top_column_share(s2.O, [12, 13, 14, 15])
    assert round(share1, 2) == g["muon_top4_share"]
    assert share2 < g["adam_sign_top4_share"]
    sv = np.linalg.svd(s2.O, compute_uv=False)
    assert sv[0] / sv[-1] > 2.0     # singular values no longer equal


# --------------------------------------------------------------------------
# Newton-Schulz (Muon Optimizer 정리; sitech.ge 'Instead of SVD')
# --------------------------------------------------------------------------
def test_coefficients_match_pages(golden):
    g = golden("ns5_coefficients.json")
    assert (orc.NS_A, orc.NS_B, orc.NS_C, orc.NS_STEPS) == (g["a"], g["b"], g["c"],
                                                            g["iterations"])


@pytest.mark.parametrize("shape", [(5, 9), (9, 9), (16, 40), (3, 70)])
def test_ns_equals_spectral_closed_form(golden, shape):
    """The matrix iteration acts on singular values only:
    NS(X) = U p^5(Sigma / ||X||_F) V^T with the page's scalar polynomial."""
    g = golden("ns5_coefficients.json")
    rng = np.random.default_rng(sum(shape))
    X = rng.standard_normal(shape) * np.logspace(-2, 0, shape[1])[None, :]
    Xn, _ = orc.frobenius_normalise(X)
    got = orc.newton_schulz(Xn, g["iterations"], g["a"], g["b"], g["c"])
    U, S, Vt = np.linalg.svd(X, full_matrices=False)
    want = U @ np.diag(quintic_scalar(S / np.linalg.norm(X), g["a"], g["b"],
                                      g["c"], g["iterations"])) @ Vt
    np.testing.assert_allclose(got, want, atol=1e-12, rtol=0)


def test_ns_tall_route_equals_short_side_route():
    """q(X X^T) X = X q(X^T X): orthogonalising the long side (a large Gram)
    gives the same matrix as transposing to the short side."""
    rng = np.random.default_rng(11)
    X, _ = orc.frobenius_normalise(rng.standard_normal((30, 7)))
    long_side = orc.newton_schulz(X)
    short_side = orc.newton_schulz(X.T).T
    np.testing.assert_allclose(long_side, short_side, atol=1e-12)


def test_worked_example_sitech(golden):
    """U diag(20, 3, 0.2) V^T -> approximately U diag(1, 1, 1) V^T: the
    singular vectors are kept and the singular values land in NS5's band."""
    g = golden("worked_example_sitech.json")
    rng = np.random.default_rng(5)
    U, _ = np.linalg.qr(rng.standard_normal((3, 3)))
    V, _ = np.linalg.qr(rng.standard_normal((6, 3)))
    X = U @ np.diag(g["singular_values_in"]) @ V.T
    out = orc.newton_schulz(orc.frobenius_normalise(X)[0])
    U2, S2, V2t = np.linalg.svd(out, full_matrices=False)
    assert np.all((S2 > 0.6) & (S2 < 1.25)), S2
    # each input direction maps to itself: U^T out V is diagonal, positive
    D = U.T @ out @ V
    np.testing.assert_allclose(D - np.diag(np.diag(D)), 0, atol=1e-12)
    assert np.all(np.diag(D) > 0.6)
    np.testing.assert_allclose(np.abs(np.diag(D) - 1.0).max() < 0.35, True)


@pytest.mark.parametrize("shape", [(64, 64), (32, 96), (128, 40), (16, 200)])
def test_polar_direction(shape):
    """NS5 approximates the orthogonal polar factor U V^T (Muon Optimizer 정리,
    'Newton-Schulz orthogonalisation'; From PCG to Muon, section 3)."""
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    G = rng.standard_normal(shape)
    X5 = orc.newton_schulz(orc.frobenius_normalise(G)[0])
    P = orc.polar_factor_svd(G)
    cos = (X5 * P).sum() / (np.linalg.norm(X5) * np.linalg.norm(P))
    assert cos >= 0.95


def test_polar_factor_nuclear_norm_identity():
    """<G, U V^T> = ||G||_* (From PCG to Muon, section 4, line search note);
    the nuclear norm is taken here from the eigenvalues of G^T G."""
    rng = np.random.default_rng(2)
    for shape in [(20, 8), (8, 20), (15, 15)]:
        G = rng.standard_normal(shape)
        lam = np.linalg.eigvalsh(G.T @ G if shape[0] >= shape[1] else G @ G.T)
        nuclear = np.sqrt(np.clip(lam, 0, None)).sum()
        assert abs((G * orc.polar_factor_svd(G)).sum() - nuclear) < 1e-10 * nuclear


@pytest.mark.parametrize("n", [1, 2, 8])
def test_gram_route_polar(n):
    """Q = G (G^T G)^(-1/2) for a tall N x n gradient (From PCG to Muon,
    'Muon's Gram Matrix'), via eigh, equals the SVD polar factor."""
    rng = np.random.default_rng(n)
    G = rng.standard_normal((300, n))
    lam, V = np.linalg.eigh(G.T @ G)
    Q = G @ (V @ np.diag(lam ** -0.5) @ V.T)
    np.testing.assert_allclose(orc.polar_factor_svd(G), Q, atol=1e-12)


def test_width_one_vector(golden):
    """Width 1 normalises the whole vector (From PCG to Muon, 'Muon
    Reshaping'): NS5 of an n x 1 matrix is p^5(1) g / ||g||."""
    g = golden("ns5_coefficients.json")
    rng = np.random.default_rng(9)
    v = rng.standard_normal((50, 1))
    got = orc.newton_schulz(orc.frobenius_normalise(v)[0])
    k = quintic_scalar(1.0, g["a"], g["b"], g["c"], g["iterations"])
    np.testing.assert_allclose(got, k * v / np.linalg.norm(v), atol=1e-14)
    got_row = orc.newton_schulz(orc.frobenius_normalise(v.T)[0])
    np.testing.assert_allclose(got_row, k * v.T / np.linalg.norm(v), atol=1e-14)


# --------------------------------------------------------------------------
# whole step
# --------------------------------------------------------------------------
@pytest.mark.parametrize("shape,moonshot,wd", [((4, 16), False, 0.0),
                                               ((6, 3), True, 0.1),
                                               ((5, 5), True, 0.05)])
def test_step_brute_force(shape, moonshot, wd):
    """Pure-Python loops reproduce the whole Muon and Dimuon step."""
    rng = np.random.default_rng(shape[0] * 10 + shape[1])
    W = rng.standard_normal(shape) * 0.02
    G = rng.standard_normal(shape)
    M = rng.standard_normal(shape)
    e_r = rng.exponential(1.0, shape[0]); e_r[0] = 0.0
    e_c = rng.exponential(1.0, shape[1])
    hp = orc.HParams(mu=0.9, lr=0.03, weight_decay=wd,
                     scale_mode=orc.SCALE_MOONSHOT if moonshot else orc.SCALE_NONE)
    h = hp.as_f32()
    for cond in (False, True):
        want = brute_force_step(W.tolist(), G.tolist(), M.tolist(), h.mu, h.lr,
                                h.weight_decay, h.a, h.b, h.c, h.ns_steps,
                                h.cond_eps, h.scale_coef, moonshot,
                                e_r.tolist() if cond else None,
                                e_c.tolist() if cond else None)
        got = orc.optimizer_step(W, G, M, hp, conditioned=cond, e_row_prev=e_r,
                                 e_col_prev=e_c, momentum_dtype="fp32",
                                 weight_dtype="fp32")
        # compare against the brute force with the same fp32 storage rounding
        np.testing.assert_allclose(got.M, np.float32(want[1]), rtol=0, atol=0)
        np.testing.assert_allclose(got.O, want[2], rtol=1e-10, atol=1e-13)
        Wb = np.float32(np.array(want[0]))
        assert np.abs(got.W - Wb).max() <= np.spacing(np.abs(Wb).max(), dtype=np.float32) * 4
        if cond:
            er, ec = orc.energies(got.M)
            np.testing.assert_allclose(got.e_row, er)
            Mt = np.array(want[1], np.float32).astype(np.float64)
            np.testing.assert_allclose(got.e_row, (Mt ** 2).sum(1), rtol=1e-12)
            np.testing.assert_allclose(got.e_col, (Mt ** 2).sum(0), rtol=1e-12)


def exact_round(x, bits, qmin, maxval):
    """Nearest binary float with `bits` significand bits to the rational x
    (ties to even; quantum never below 2^qmin; beyond maxval -> inf), by
    exact integer arithmetic."""
    from fractions import Fraction
    x = Fraction(x)
    if x == 0:
        return 0.0
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1                                   # 2^e <= a < 2^(e+1)
    q = Fraction(2) ** max(e - bits + 1, qmin)
    n = a / q
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = fl * q
    out = math.inf if v > maxval else float(v)
    return out if x > 0 else -out


FP32_FMT = (24, -149, (2 - 2.0 ** -23) * 2.0 ** 127)
BF16_FMT = (8, -133, (2 - 2.0 ** -7) * 2.0 ** 127)


def exact_momentum(mu, m, g, fmt):
    from fractions import Fraction
    return exact_round(Fraction(mu) * Fraction(m) + Fraction(g), *fmt)


def double_rounded_momentum(mu, m, g, dtype):
    """The float64 sum rounded again to the storage type (two roundings)."""
    v = np.float64(mu) * np.float64(m) + np.float64(g)
    return float(orc.store_round(v, dtype))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_momentum_is_the_correctly_rounded_exact_value(dtype):
    """[MuonNote] 'Update rule', eq. (1): M_t = mu M_{t-1} + G, stored once.
    Brute force with exact rational arithmetic over random draws whose
    magnitudes differ by up to 2^60 (where the float64 sum itself rounds)."""
    rng = np.random.default_rng(11)
    fmt = BF16_FMT if dtype == "bf16" else FP32_FMT
    n = 400
    M = rng.standard_normal(n) * np.exp2(rng.integers(-30, 30, n))
    G = rng.standard_normal(n) * np.exp2(rng.integers(-30, 30, n))
    M = orc.store_round(M, dtype)
    G = orc.store_round(G, dtype)
    for mu in (float(np.float32(0.95)), float(np.float32(0.9)), 0.75):
        got = orc.store_round(orc.momentum_update(M, G, mu), dtype)
        for i in range(n):
            assert got[i] == exact_momentum(mu, M[i], G[i], fmt), (mu, M[i], G[i])


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_momentum_double_rounding_case(dtype):
    """A constructed case where rounding the float64 sum to the storage type
    differs from rounding the exact value: the oracle gives the latter."""
    mu, m, g = crafted_fp32_tie() if dtype == "fp32" else crafted_bf16_tie()
    fmt = FP32_FMT if dtype == "fp32" else BF16_FMT
    for v in (mu, m, g):
        assert float(orc.store_round(v, "fp32")) == v   # all float32 values
    exact = exact_momentum(mu, m, g, fmt)
    assert double_rounded_momentum(mu, m, g, dtype) != exact
    got = orc.store_round(orc.momentum_update(np.array([m]), np.array([g]), mu), dtype)
    assert got[0] == exact


def test_first_step_dimuon_equals_muon():
    """'Why the *last* momentum': with M_0 = 0 the first Dimuon step is
    exactly the Muon step."""
    rng = np.random.default_rng(4)
    for shape in [(4, 16), (12, 5)]:
        W = rng.standard_normal(shape); G = rng.standard_normal(shape)
        Z = np.zeros(shape)
        hp = orc.HParams(weight_decay=0.1, scale_mode=orc.SCALE_MOONSHOT)
        d = orc.dimuon_step(W, G, Z, np.zeros(shape[0]), np.zeros(shape[1]), hp)
        m = orc.muon_step(W, G, Z, hp)
        np.testing.assert_array_equal(d.W, m.W)
        np.testing.assert_array_equal(d.O, m.O)


def test_mu_zero_still_conditioned_by_previous_momentum():
    """'Why the *last* momentum': with beta set to 0 between steps the new
    momentum holds only G_2, yet the step still depends on M_1."""
    rng = np.random.default_rng(8)
    G1 = rng.standard_normal((4, 16)) * np.logspace(-1, 1, 16)[None, :] ** 2
    G2 = rng.standard_normal((4, 16))
    Z = np.zeros_like(G1)
    s1 = orc.dimuon_step(Z, G1, Z, np.zeros(4), np.zeros(16), orc.HParams())
    hp0 = orc.HParams(mu=0.0)
    s2 = orc.dimuon_step(s1.W, G2, s1.M, s1.e_row, s1.e_col, hp0)
    plain = orc.muon_step(s1.W, G2, s1.M, hp0)
    assert np.abs(s2.O - plain.O).max() > 1e-3
    h = hp0.as_f32()
    want = brute_force_step(s1.W.tolist(), G2.tolist(), s1.M.tolist(), 0.0, h.lr,
                            0.0, h.a, h.b, h.c, 5, h.cond_eps, 0.2, False,
                            ((s1.M ** 2).sum(1)).tolist(), ((s1.M ** 2).sum(0)).tolist())
    np.testing.assert_allclose(s2.O, want[2], rtol=1e-9, atol=1e-12)


def test_uniform_conditioning_reduces_to_muon():
    """R = C = k I cancels between the Frobenius normalisation and the
    renormalisation, so uniform energies give the Muon step."""
    rng = np.random.default_rng(6)
    W = rng.standard_normal((8, 20)); G = rng.standard_normal((8, 20))
    M = rng.standard_normal((8, 20))
    hp = orc.HParams()
    d = orc.dimuon_step(W, G, M, np.full(8, 3.0), np.full(20, 0.5), hp)
    m = orc.muon_step(W, G, M, hp)
    np.testing.assert_allclose(d.O, m.O, atol=1e-12)


def test_moonshot_scale_rms_near_adamw():
    """With the Moonshot rule the update RMS of a square matrix sits near the
    0.2 coefficient (sitech.ge, 'From speedrun to real training': update
    RMS matched to AdamW's)."""
    rng = np.random.default_rng(12)
    for n in (64, 256):
        G = rng.standard_normal((n, n))
        r = orc.muon_step(np.zeros((n, n)), G, np.zeros((n, n)),
                          orc.HParams(scale_mode=orc.SCALE_MOONSHOT))
        rms = math.sqrt((r.O ** 2).mean())
        assert 0.12 < rms < 0.26


def test_nonfinite_gradient_only_decays():
    G = np.ones((3, 5)); G[1, 2] = np.inf
    W = np.full((3, 5), 2.0)
    r = orc.muon_step(W, G, np.zeros((3, 5)),
                      orc.HParams(lr=0.5, weight_decay=0.5))
    assert r.nonfinite
    decay = 1.0 - 0.5 * 0.5          # lr and wd are exact in float32
    np.testing.assert_array_equal(r.W, decay * W)
    np.testing.assert_array_equal(r.O, 0.0)


def test_negligible_norm_zero_update():
    """A momentum whose Frobenius norm is below the 1e-15 floor gives a zero
    update rather than an amplified one."""
    rng = np.random.default_rng(21)
    W = rng.standard_normal((6, 9))
    r = orc.muon_step(W, 1e-20 * rng.standard_normal((6, 9)), np.zeros((6, 9)), orc.HParams())
    assert not r.nonfinite
    np.testing.assert_array_equal(r.O, 0.0)
    r = orc.muon_step(W, 1e-12 * rng.standard_normal((6, 9)), np.zeros((6, 9)), orc.HParams())
    assert np.abs(r.O).max() > 0.01


def test_zero_gradient_zero_update():
    W = np.full((3, 5), 2.0)
    r = orc.muon_step(W, np.zeros((3, 5)), np.zeros((3, 5)), orc.HParams())
    assert not r.nonfinite
    np.testing.assert_array_equal(r.O, 0.0)
    np.testing.assert_array_equal(r.W, W)


@pytest.mark.parametrize("cond", [False, True])
def test_nesterov_brute_force(cond):
    """Nesterov: the orthogonaliser takes B_t = G + mu M_t (From PCG to Muon,
    section 3, momentum-and-Nesterov combination); M_t and the energies are
    those of the plain momentum."""
    rng = np.random.default_rng(31)
    shape = (5, 8)
    W = rng.standard_normal(shape) * 0.02
    G = rng.standard_normal(shape)
    M = rng.standard_normal(shape)
    e_r = rng.exponential(1.0, shape[0])
    e_c = rng.exponential(1.0, shape[1])
    hp = orc.HParams(mu=0.9, lr=0.03, nesterov=True)
    h = hp.as_f32()
    want = brute_force_step(W.tolist(), G.tolist(), M.tolist(), h.mu, h.lr, 0.0, h.a, h.b,
                            h.c, h.ns_steps, h.cond_eps, h.scale_coef, False,
                            e_r.tolist() if cond else None, e_c.tolist() if cond else None,
                            nesterov=True)
    got = orc.optimizer_step(W, G, M, hp, conditioned=cond, e_row_prev=e_r, e_col_prev=e_c)
    np.testing.assert_allclose(got.O, want[2], rtol=1e-10, atol=1e-13)
    plain = orc.optimizer_step(W, G, M, orc.HParams(mu=0.9, lr=0.03), conditioned=cond,
                               e_row_prev=e_r, e_col_prev=e_c)
    np.testing.assert_array_equal(got.M, plain.M)
    assert np.abs(got.O - plain.O).max() > 1e-3


def test_nesterov_without_momentum_is_plain():
    """With mu = 0, B_t = G = M_t: Nesterov changes nothing."""
    rng = np.random.default_rng(32)
    W = rng.standard_normal((6, 9))
    G = rng.standard_normal((6, 9)).astype(np.float32).astype(np.float64)  # = stored M_t
    Z = np.zeros((6, 9))
    a = orc.muon_step(W, G, Z, orc.HParams(mu=0.0, nesterov=True))
    b = orc.muon_step(W, G, Z, orc.HParams(mu=0.0))
    np.testing.assert_array_equal(a.O, b.O)


# --------------------------------------------------------------------------
# Muon on a 1-D variable (From PCG to Muon, section 6 "Muon Reshaping")
# --------------------------------------------------------------------------
@pytest.mark.parametrize("width,length", [(1, 37), (2, 37), (8, 37), (32, 37), (128, 37), (5, 40)])
def test_vector_layout_brute_force(width, length):
    """Row-major layout with zero padding and the padding dropped after the
    update, checked against the pure-Python step on a matrix filled by hand;
    the padded momentum cells stay exactly zero."""
    rng = np.random.default_rng(width * 100 + length)
    w = rng.standard_normal(length) * 0.02
    g = rng.standard_normal(length)
    m = rng.standard_normal(length)
    rows = (length + width - 1) // width

    def by_hand(v):
        return [[float(v[i * width + j]) if i * width + j < length else 0.0 for j in range(width)]
                for i in range(rows)]

    hp = orc.HParams(mu=0.9, lr=0.05, weight_decay=0.01)
    h = hp.as_f32()
    want = brute_force_step(by_hand(w), by_hand(g), by_hand(m), h.mu, h.lr, h.weight_decay,
                            h.a, h.b, h.c, h.ns_steps, h.cond_eps, h.scale_coef, False)
    flat = lambda X: np.array(X, np.float64).reshape(-1)[:length]  # noqa: E731
    got = orc.vector_step(w, g, m, width, hp)
    np.testing.assert_array_equal(got.M, np.float32(flat(want[1])))
    np.testing.assert_allclose(got.O, flat(want[2]), rtol=1e-10, atol=1e-13)
    assert np.all(got.extras["padded_M"] == 0.0)
    assert got.W.shape == (length,) and got.O.shape == (length,)


@pytest.mark.parametrize("width", [1, 4096])
def test_vector_width_one_closed_form(width, golden):
    """A width-1 layout (and a single row, width >= length) normalises the whole
    vector: O = kappa p^5(1) B / ||B|| with B = G + mu M_t under Nesterov
    (From PCG to Muon, section 6: width 1 normalises the vector; momentum
    and Nesterov stay in the step)."""
    g5 = golden("ns5_coefficients.json")
    rng = np.random.default_rng(41)
    L = 1000
    w, g, m = rng.standard_normal(L) * 0.02, rng.standard_normal(L), rng.standard_normal(L)
    hp = orc.HParams(mu=0.95, lr=0.02, nesterov=True)
    h = hp.as_f32()
    got = orc.vector_step(w, g, m, width, hp)
    Mt = np.float32(h.mu * m + g).astype(np.float64)
    B = g + h.mu * Mt
    # the step carries its coefficients through float32 like the library
    assert (h.a, h.b, h.c) == tuple(float(np.float32(g5[k])) for k in "abc")
    k = quintic_scalar(1.0, h.a, h.b, h.c, g5["iterations"])
    np.testing.assert_array_equal(got.M, Mt)
    np.testing.assert_allclose(got.O, k * B / np.linalg.norm(B), rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------
# Jordan / Bernstein scale rules (named, not printed, by [Sitech] "From
# speedrun to real training"; read as those authors' published rules).
# Parity of the two formulas is unpinned to the pages; what is pinned is how
# the scale enters the step: O is exactly kappa times the unscaled update,
# and the orientation (rows = output features) decides which side counts.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(96, 40), (40, 96), (64, 64)])
def test_scale_rules_closed_forms(shape):
    r, c = shape
    assert orc.scale_factor(orc.SCALE_JORDAN, 0.2, r, c) == pytest.approx(max(1.0, r / c) ** 0.5)
    assert orc.scale_factor(orc.SCALE_BERNSTEIN, 0.2, r, c) == pytest.approx((r / c) ** 0.5)
    # Jordan's rule never shrinks the update; Bernstein's shrinks it for wide matrices
    assert orc.scale_factor(orc.SCALE_JORDAN, 0.2, r, c) >= 1.0
    assert (orc.scale_factor(orc.SCALE_BERNSTEIN, 0.2, r, c) < 1.0) == (r < c)


@pytest.mark.parametrize("mode", [orc.SCALE_JORDAN, orc.SCALE_BERNSTEIN])
@pytest.mark.parametrize("shape", [(48, 20), (20, 48)])
def test_scale_rules_scale_the_update_only(mode, shape):
    rng = np.random.default_rng(77)
    W = 0.02 * rng.standard_normal(shape)
    G = rng.standard_normal(shape)
    M = rng.standard_normal(shape)
    base = orc.muon_step(W, G, M, orc.HParams(weight_decay=0.01))
    got = orc.muon_step(W, G, M, orc.HParams(weight_decay=0.01, scale_mode=mode))
    kappa = orc.scale_factor(mode, orc.MOONSHOT_COEF, *shape)
    np.testing.assert_array_equal(got.M, base.M)
    np.testing.assert_allclose(got.O, kappa * base.O, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------
# Per-iteration coefficient schedules.  The Dimuon page's toy ("16 columns
# with input size 0.1 to 10") orthogonalises with Polar Express, whose
# quintic changes from iteration to iteration; the page prints none of its
# coefficients, so what is pinned is the mechanism: iteration k applies its
# own odd quintic p_k to the singular values.
# ---------------------------------------------------------------------------
# five distinct quintics; their composition maps [0, 1] into [0, 1]
SCHEDULE = ((3.4445, -4.7750, 2.0315), (3.0, -3.2, 1.2), (2.5, -2.2, 0.7),
            (1.875, -1.25, 0.375), (1.5, -0.5, 0.0))


@pytest.mark.parametrize("shape", [(5, 9), (9, 9), (16, 40), (3, 70)])
def test_schedule_equals_composed_spectral_closed_form(shape):
    """NS with a schedule = U (p_K o ... o p_1)(Sigma / ||X||_F) V^T, each p_k
    the scalar quintic of its own triple (LAPACK SVD on the other side)."""
    rng = np.random.default_rng(sum(shape) + 5)
    X = rng.standard_normal(shape) * np.logspace(-2, 0, shape[1])[None, :]
    Xn, _ = orc.frobenius_normalise(X)
    got = orc.newton_schulz(Xn, len(SCHEDULE), coeffs=SCHEDULE)
    U, S, Vt = np.linalg.svd(X, full_matrices=False)
    s = S / np.linalg.norm(X)
    for (a, b, c) in SCHEDULE:
        s = quintic_scalar(s, a, b, c, 1)
    np.testing.assert_allclose(got, U @ np.diag(s) @ Vt, atol=1e-12, rtol=0)
    # the order of the iterations matters: the reversed schedule differs
    rev = orc.newton_schulz(Xn, len(SCHEDULE), coeffs=SCHEDULE[::-1])
    assert np.abs(rev - got).max() > 1e-3


def test_constant_schedule_is_the_fixed_step():
    """A schedule that repeats (a, b, c) is the fixed-coefficient step, bit
    for bit, through the whole Muon and Dimuon step."""
    rng = np.random.default_rng(21)
    shape = (24, 40)
    W, G, M = 0.02 * rng.standard_normal(shape), rng.standard_normal(shape), rng.standard_normal(shape)
    er, ec = rng.exponential(1.0, shape[0]), rng.exponential(1.0, shape[1])
    fixed = orc.HParams(ns_steps=4)
    sched = orc.HParams(ns_steps=4, ns_coeffs=((orc.NS_A, orc.NS_B, orc.NS_C),) * 4)
    for cond in (False, True):
        a = orc.optimizer_step(W, G, M, fixed, conditioned=cond, e_row_prev=er, e_col_prev=ec)
        b = orc.optimizer_step(W, G, M, sched, conditioned=cond, e_row_prev=er, e_col_prev=ec)
        np.testing.assert_array_equal(a.O, b.O)
        np.testing.assert_array_equal(a.W, b.W)


def _taylor_quintic():
    """Coefficients of x (1 + u/2 + 3u^2/8), u = 1 - x^2: the second-order
    binomial series of x (1 - u)^(-1/2) = x / |x|, written from the series'
    coefficients binom(-1/2, k) (-1)^k, k = 0, 1, 2."""
    t = [1.0, 0.5, 0.375]
    # x (t0 + t1 (1 - x^2) + t2 (1 - x^2)^2) = a x + b x^3 + c x^5
    return (t[0] + t[1] + t[2], -(t[1] + 2 * t[2]), t[2])


def test_schedule_ending_in_taylor_steps_reaches_the_polar_factor():
    """Five page iterations followed by Taylor steps (fixed point 1 with zero
    slope) drive every singular value to 1: the result is the LAPACK polar
    factor U V^T to 1e-9 ([MuonNote], 'Why orthogonalise')."""
    a, b, c = _taylor_quintic()
    assert (a, b, c) == (1.875, -1.25, 0.375)
    sched = ((orc.NS_A, orc.NS_B, orc.NS_C),) * 5 + ((a, b, c),) * 6
    rng = np.random.default_rng(8)
    X = rng.standard_normal((20, 50))   # well conditioned: sigma_min / ||X|| ~ 0.1
    Xn, _ = orc.frobenius_normalise(X)
    got = orc.newton_schulz(Xn, len(sched), coeffs=sched)
    np.testing.assert_allclose(got, orc.polar_factor_svd(X), atol=1e-9, rtol=0)


@pytest.mark.parametrize("shape", [(4, 7), (7, 4)])
def test_schedule_brute_force_step(shape):
    """Pure-Python loops with a per-iteration schedule reproduce the oracle's
    Muon and Dimuon step (wide and tall)."""
    rng = np.random.default_rng(shape[0] * 7 + shape[1])
    W = 0.02 * rng.standard_normal(shape)
    G = rng.standard_normal(shape)
    M = rng.standard_normal(shape)
    e_r, e_c = rng.exponential(1.0, shape[0]), rng.exponential(1.0, shape[1])
    hp = orc.HParams(mu=0.9, lr=0.03, weight_decay=0.02, ns_steps=len(SCHEDULE),
                     ns_coeffs=SCHEDULE)
    h = hp.as_f32()
    for cond in (False, True):
        want = brute_force_step(W.tolist(), G.tolist(), M.tolist(), h.mu, h.lr,
                                h.weight_decay, h.a, h.b, h.c, h.ns_steps, h.cond_eps,
                                h.scale_coef, False, e_r.tolist() if cond else None,
                                e_c.tolist() if cond else None, coeffs=h.ns_coeffs)
        got = orc.optimizer_step(W, G, M, hp, conditioned=cond, e_row_prev=e_r,
                                 e_col_prev=e_c, momentum_dtype="fp32", weight_dtype="fp32")
        np.testing.assert_allclose(got.O, want[2], rtol=1e-10, atol=1e-13)


# ---------------------------------------------------------------------------
# torch.optim.Muon (a library implementation of the same step) pins the
# Jordan and Moonshot scale rules and the update's structure.  Its momentum
# is an average, buf <- mu buf + (1 - mu) g; with G = (1 - mu) g the
# oracle's M_t = mu M_{t-1} + G is that buffer, and its Nesterov input
# g + mu (buf - g) is the oracle's B_t = G + mu M_t.  Its adjustment
# "original" is kappa = sqrt(max(1, rows / cols)) and "match_rms_adamw" is
# kappa = 0.2 sqrt(max(rows, cols)).  It orthogonalises in bf16, hence the
# bf16 tolerance on the update.  (Bernstein's rule has no such library
# counterpart and stays unpinned.)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("shape", [(96, 40), (40, 96), (64, 64)])
def test_scale_rules_match_torch_muon_adjustment(shape):
    from torch.optim import _muon
    assert orc.scale_factor(orc.SCALE_JORDAN, 0.2, *shape) == pytest.approx(
        _muon._adjust_lr(1.0, "original", torch.Size(shape)), rel=1e-15)
    assert orc.scale_factor(orc.SCALE_MOONSHOT, 0.2, *shape) == pytest.approx(
        _muon._adjust_lr(1.0, "match_rms_adamw", torch.Size(shape)), rel=1e-15)


@pytest.mark.parametrize("shape", [(48, 20), (20, 48)])
@pytest.mark.parametrize("rule", ["original", "match_rms_adamw"])
@pytest.mark.parametrize("nesterov", [False, True])
def test_step_matches_torch_muon(shape, rule, nesterov):
    mode = orc.SCALE_JORDAN if rule == "original" else orc.SCALE_MOONSHOT
    mu, lr, wd = 0.9, 0.05, 0.1
    rng = np.random.default_rng(shape[0] + 3 * shape[1] + nesterov)
    W0 = 0.02 * rng.standard_normal(shape)
    p = torch.nn.Parameter(torch.from_numpy(W0.astype(np.float32)))
    opt = torch.optim.Muon([p], lr=lr, weight_decay=wd, momentum=mu, nesterov=nesterov,
                           adjust_lr_fn=rule)
    W, M = np.float32(W0).astype(np.float64), np.zeros(shape)
    hp = orc.HParams(mu=mu, lr=lr, weight_decay=wd, scale_mode=mode, nesterov=nesterov)
    for t in range(3):
        g = rng.standard_normal(shape).astype(np.float32)
        p.grad = torch.from_numpy(g)
        opt.step()
        res = orc.muon_step(W, (1.0 - np.float32(mu)) * g.astype(np.float64), M, hp,
                            momentum_dtype="fp32", weight_dtype="fp32")
        Wt = p.detach().numpy().astype(np.float64)
        # the update part of W, relative to its size (bf16 orthogonalisation)
        dw_t, dw_o = Wt - (1 - lr * wd) * W, res.W - (1 - lr * wd) * W
        assert np.linalg.norm(dw_t - dw_o) <= 3e-2 * np.linalg.norm(dw_o), t
        # teacher forcing: continue both from torch's state
        W = Wt
        M = opt.state[p]["momentum_buffer"].numpy().astype(np.float64)
