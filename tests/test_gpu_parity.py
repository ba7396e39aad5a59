"""GPU parity: the CUDA library against the fp64 oracle, element by element,
on the same seeded inputs (teacher-forced every step), through the C ABI.

Tolerances (written here, derived from the method's arithmetic):
  O_t          relative Frobenius <= 1e-5 (fp32 mode, thin path),
               <= 3e-2 (bf16 tensor-core mode)
  sing. values of O_t / kappa within 0.05
  M_t          <= 1 storage ulp per element
  W_t          <= 1 storage ulp of (1 - lr wd) W_{t-1} - lr O_t (GPU's own O_t)
  energies     relative 2e-5 of the sums of squares of the stored M_t
"""
import numpy as np
import pytest
import torch

import dimuon_optimizer_b200 as dm
import oracle as orc
import workloads
from rounding_cases import crafted_bf16_tie, crafted_fp32_tie
from gpu_harness import (TOL_BF16, TOL_FP32, TOL_THIN_SPLIT_ILL, Group, oracle_hp, rel_fro,
                         run_gpu_step, step_and_compare, thin_tol, to_dev, to_host)

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

BF, F32 = dm.DM_BF16, dm.DM_FP32


def gaussian(shapes, seed, scale_cols=False):
    rng = np.random.default_rng(seed)
    out = []
    for (r, c) in shapes:
        g = rng.standard_normal((r, c))
        if scale_cols:
            g *= rng.lognormal(0.0, 1.0, c)[None, :]
        out.append(g)
    return out


def hparams(precision, **kw):
    return dm.dm_default_hparams(precision=precision, **kw)


# --------------------------------------------------------------------------
# Newton-Schulz path, fp32 SIMT products
# --------------------------------------------------------------------------
NS_SHAPES = [(64, 96), (130, 200), (300, 140), (257, 513), (40, 33)]


@pytest.mark.parametrize("cond", [False, True])
@pytest.mark.parametrize("dts", [(BF, BF, BF), (F32, F32, F32), (BF, BF, F32)])
def test_fp32_mode_ns_path(cond, dts):
    wdt, gdt, mdt = dts
    grp = Group(NS_SHAPES, wdt, gdt, mdt, cond=cond, seed=11)
    hp = hparams(dm.DM_PREC_FP32, weight_decay=0.05, scale_mode=dm.DM_SCALE_MOONSHOT)
    ws = None
    for t in range(3):
        _, ws = step_and_compare(grp, gaussian(NS_SHAPES, 100 + t, scale_cols=True), hp,
                                 TOL_FP32, ws=ws)


# --------------------------------------------------------------------------
# Newton-Schulz path, bf16 tcgen05 products
# --------------------------------------------------------------------------
TC_SHAPES = [(384, 640), (700, 260), (257, 513), (40, 100), (128, 256), (520, 136)]


@pytest.mark.parametrize("kernel", [0, dm.DM_DBG_TC_SINGLE, dm.DM_DBG_TC_PAIR])
@pytest.mark.parametrize("cond", [False, True])
def test_tc_mode_ns_path(cond, kernel):
    """Tensor-core products: the planner's choice, single-CTA 128 x 256 tiles
    and CTA-pair 256 x 256 tiles."""
    grp = Group(TC_SHAPES, BF, BF, BF, cond=cond, seed=12)
    hp = hparams(dm.DM_PREC_BF16_TC, weight_decay=0.1, scale_mode=dm.DM_SCALE_MOONSHOT,
                 debug_flags=kernel)
    ws = None
    for t in range(3):
        rep, ws = step_and_compare(grp, gaussian(TC_SHAPES, 200 + t, scale_cols=True), hp,
                                   TOL_BF16, ws=ws)
    assert max(rep.o_err) < 2e-2


def test_tc_mode_fp32_storage():
    shapes = [(300, 520), (520, 300)]
    grp = Group(shapes, F32, F32, F32, cond=True, seed=13)
    hp = hparams(dm.DM_PREC_BF16_TC)
    ws = None
    for t in range(2):
        _, ws = step_and_compare(grp, gaussian(shapes, 300 + t), hp, TOL_BF16, ws=ws)


@pytest.mark.parametrize("ns_steps", [1, 2, 6])
def test_ns_step_counts(ns_steps):
    shapes = [(200, 330), (330, 200)]
    for prec, tol, dbg in ((dm.DM_PREC_FP32, TOL_FP32, 0), (dm.DM_PREC_BF16_TC, TOL_BF16, 0),
                           (dm.DM_PREC_BF16_TC, TOL_BF16, dm.DM_DBG_TC_PAIR)):
        grp = Group(shapes, BF, BF, F32, cond=True, seed=14)
        hp = hparams(prec, ns_steps=ns_steps, debug_flags=dbg)
        ws = None
        for t in range(2):
            _, ws = step_and_compare(grp, gaussian(shapes, 400 + t), hp, tol, ws=ws)


# --------------------------------------------------------------------------
# thin factors (Gram route).  Shapes with r in {2, 4, 8, 16, 32} and a long
# side divisible by 8 (any long side for tall factors with r >= 8) take the
# shared-memory staged kernels (r = 2: the single-pass kernel unless
# DM_DBG_THIN_STAGED), the rest (and everything under DM_DBG_THIN_REGS) the
# register kernels.  The ragged tall ones end their last stage on a partial
# group of four energies.
# --------------------------------------------------------------------------
THIN_SHAPES = [(4, 16), (2, 100), (8, 4096), (4096, 8), (17, 333), (32, 4096), (4096, 32),
               (1, 50), (50, 1), (31, 31), (16, 1000), (2, 2056), (3000, 4), (8, 24),
               (1001, 8), (4099, 16), (777, 32), (13, 8), (2, 5128), (5128, 2), (4, 4096),
               (4096, 4), (32, 1032), (1032, 32)]


# default: the cluster kernel for r <= 4 (r = 2 factors whose long side is an
# odd multiple of 8 above 2560, such as 5128, take the one-CTA single-pass
# kernel), the staged kernels for r = 8 .. 32; cluster: r = 8 on the cluster
# kernel too
@pytest.mark.parametrize("path", [0, dm.DM_DBG_THIN_STAGED, dm.DM_DBG_THIN_REGS,
                                  dm.DM_DBG_THIN_CLUSTER],
                         ids=["default", "staged", "regs", "cluster"])
@pytest.mark.parametrize("cond", [False, True])
@pytest.mark.parametrize("mdt", [F32, BF])
def test_thin_path(cond, mdt, path):
    grp = Group(THIN_SHAPES, BF, BF, mdt, cond=cond, seed=15)
    hp = hparams(dm.DM_PREC_BF16_TC, weight_decay=0.01, debug_flags=path)
    ws = None
    for t in range(3):
        _, ws = step_and_compare(grp, gaussian(THIN_SHAPES, 500 + t, scale_cols=True), hp,
                                 thin_tol(True), ws=ws)


@pytest.mark.parametrize("prec", [dm.DM_PREC_FP32, dm.DM_PREC_BF16_TC], ids=["fp32", "bf16"])
@pytest.mark.parametrize("cond", [False, True])
def test_thin_path_fp32_storage(cond, prec):
    """fp32 gradients, momentum and weights (the third staged combination),
    with Nesterov; in bf16 mode the rank-32 factors take the split sums."""
    shapes = [(8, 512), (512, 16), (32, 256), (256, 32), (4, 96), (2, 40)]
    grp = Group(shapes, F32, F32, F32, cond=cond, seed=17)
    hp = hparams(prec, nesterov=1)
    ws = None
    for t in range(3):
        _, ws = step_and_compare(grp, gaussian(shapes, 700 + t, scale_cols=True), hp,
                                 thin_tol(prec == dm.DM_PREC_BF16_TC), ws=ws)


def test_thin_threshold_hook_matches_ns_path():
    """The same thin factors through the Newton-Schulz kernels (test hook)
    agree with the oracle too."""
    shapes = [(8, 300), (300, 8), (32, 257)]
    grp = Group(shapes, F32, F32, F32, cond=True, seed=16)
    hp = hparams(dm.DM_PREC_FP32, debug_flags=dm.DM_DBG_NO_THIN)
    ws = None
    for t in range(2):
        _, ws = step_and_compare(grp, gaussian(shapes, 600 + t, scale_cols=True), hp, TOL_FP32,
                                 ws=ws)


@pytest.mark.parametrize("prec,tol", [(dm.DM_PREC_FP32, TOL_FP32), (dm.DM_PREC_BF16_TC, TOL_BF16)])
@pytest.mark.parametrize("cond", [False, True])
def test_nesterov(prec, tol, cond):
    """B_t = G + mu M_t feeds the orthogonaliser on every path (Newton-Schulz
    and thin)."""
    shapes = [(200, 330), (330, 200), (8, 600), (600, 16), (32, 600), (600, 32)]
    grp = Group(shapes, BF, BF, F32, cond=cond, seed=21)
    hp = hparams(prec, nesterov=1, weight_decay=0.02)
    ws = None
    thin = thin_tol(prec == dm.DM_PREC_BF16_TC)

    def tol_of(shape):  # Newton-Schulz matrices at the mode's tolerance, thin factors at theirs
        if min(shape) > 32:
            return tol
        return thin(shape) if callable(thin) else thin

    for t in range(3):
        _, ws = step_and_compare(grp, gaussian(shapes, 900 + t, scale_cols=True), hp, tol_of,
                                 ws=ws)


@pytest.mark.parametrize("prec,tol", [(dm.DM_PREC_FP32, TOL_FP32), (dm.DM_PREC_BF16_TC, TOL_BF16)])
@pytest.mark.parametrize("mode", [dm.DM_SCALE_JORDAN, dm.DM_SCALE_BERNSTEIN])
def test_scale_rules(mode, prec, tol):
    """Jordan's and Bernstein's per-matrix scale on every path (Newton-Schulz
    wide and tall, thin wide and tall)."""
    shapes = [(200, 330), (330, 200), (8, 600), (600, 16)]
    grp = Group(shapes, BF, BF, F32, cond=False, seed=23)
    hp = hparams(prec, scale_mode=mode, weight_decay=0.02)
    ws = None
    for t in range(2):
        _, ws = step_and_compare(grp, gaussian(shapes, 950 + t, scale_cols=True), hp, tol, ws=ws)


# --------------------------------------------------------------------------
# invariants and edge cases
# --------------------------------------------------------------------------
def test_first_dimuon_step_equals_muon():
    """'Why the *last* momentum': with M_0 = 0 the conditioning is off."""
    shapes = [(96, 160), (16, 300)]
    g = gaussian(shapes, 700)
    outs = []
    for cond in (False, True):
        grp = Group(shapes, F32, F32, F32, cond=cond, seed=17)
        run_gpu_step(grp, g, hparams(dm.DM_PREC_FP32))
        outs.append([to_host(u) for u in grp.upd])
    for a, b in zip(*outs):
        assert rel_fro(b, a) < 1e-6


def test_nonfinite_gradient_reports_and_only_decays():
    # Newton-Schulz, thin (fp64 sums) and rank-32 thin (split sums in bf16 mode)
    shapes = [(64, 128), (8, 256), (32, 256), (256, 32)]
    g = gaussian(shapes, 800)
    g[0][3, 5] = np.inf
    g[1][2, 7] = np.nan
    g[2][30, 200] = -np.inf
    g[3][100, 31] = np.nan
    grp = Group(shapes, F32, F32, F32, cond=False, seed=18)
    W0 = [to_host(w) for w in grp.W]
    hp = hparams(dm.DM_PREC_BF16_TC, weight_decay=0.5, lr=0.1)
    ws, _ = run_gpu_step(grp, g, hp)
    assert dm.dm_read_device_status(ws) == dm.DM_ERR_NONFINITE
    decay = np.float32(1) - np.float32(0.1) * np.float32(0.5)
    for w0, w in zip(W0, grp.W):
        np.testing.assert_allclose(to_host(w), np.float32(decay) * w0.astype(np.float32),
                                   rtol=1e-7)
    # a clean step on the same workspace clears the status word
    grp2 = Group(shapes, F32, F32, F32, cond=False, seed=18)
    run_gpu_step(grp2, gaussian(shapes, 801), hp, ws)
    assert dm.dm_read_device_status(ws) == dm.DM_OK


def test_zero_gradient_gives_zero_update():
    shapes = [(64, 128), (4, 64), (32, 96), (96, 32)]
    for prec in (dm.DM_PREC_FP32, dm.DM_PREC_BF16_TC):
        for cond in (False, True):
            grp = Group(shapes, F32, F32, F32, cond=cond, seed=19)
            W0 = [to_host(w) for w in grp.W]
            ws, _ = run_gpu_step(grp, [np.zeros(s) for s in shapes], hparams(prec))
            assert dm.dm_read_device_status(ws) == dm.DM_OK
            for w0, w, u in zip(W0, grp.W, grp.upd):
                assert np.all(to_host(u) == 0.0)
                np.testing.assert_array_equal(to_host(w), w0)


def test_empty_group():
    hp = hparams(dm.DM_PREC_BF16_TC)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    assert dm.dm_muon_step([], hp, ws) == dm.DM_OK
    assert dm.dm_read_device_status(ws) == dm.DM_OK


def test_cuda_graph_capture_matches_eager():
    shapes = [(256, 384), (384, 256), (8, 512), (32, 512), (512, 32)]
    g = gaussian(shapes, 900)
    hp = hparams(dm.DM_PREC_BF16_TC)
    eager = Group(shapes, BF, BF, BF, cond=True, seed=20)
    graphed = Group(shapes, BF, BF, BF, cond=True, seed=20)
    ws_e, _ = run_gpu_step(eager, g, hp)
    G = [to_dev(x, BF) for x in g]
    mats = graphed.matrices(G)
    ws = torch.empty(dm.dm_workspace_size(mats, hp, 1), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        dm.check(dm.dm_dimuon_step(mats, hp, ws, stream=s))
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager.W, graphed.W):
        assert torch.equal(a, b)
    for a, b in zip(eager.er, graphed.er):
        assert torch.equal(a, b)


# --------------------------------------------------------------------------
# the workloads
# --------------------------------------------------------------------------
def test_toy_lora_factor_two_steps():
    """4x16 fp32 toy: step 1 unconditioned (71 % top-4 share printed on the
    Dimuon page), step 2 conditioned by step 1's momentum."""
    G, _ = workloads.toy_lora_factor()
    grp = Group([(4, 16)], F32, F32, F32, cond=True, seed=0)
    hp = dm.dm_default_hparams(precision=dm.DM_PREC_FP32)
    shares = []
    for t in range(2):
        step_and_compare(grp, [G], hp, TOL_FP32)
        shares.append(orc.top_column_share(to_host(grp.upd[0]), [12, 13, 14, 15]))
    assert round(shares[0], 2) == 0.71
    assert shares[1] < 0.25


@pytest.mark.parametrize("prec,tol", [(dm.DM_PREC_FP32, TOL_FP32), (dm.DM_PREC_BF16_TC, TOL_BF16)])
def test_square_1024(prec, tol):
    shapes = workloads.single_square_shapes()
    grp = Group(shapes, BF, BF, BF, cond=False, seed=1)
    step_and_compare(grp, workloads.gaussian_grads(shapes, 1), hparams(prec), tol)


def test_gpt2_small_group():
    shapes = workloads.gpt2_small_shapes()
    grads = workloads.gpt2_small_grads()
    grp = Group(shapes, BF, BF, BF, cond=False, seed=2)
    hp = hparams(dm.DM_PREC_BF16_TC, weight_decay=0.1, scale_mode=dm.DM_SCALE_MOONSHOT)
    rep, _ = step_and_compare(grp, grads, hp, TOL_BF16, sample=list(range(12)))
    assert len(rep.o_err) == 12


# one matrix of each orientation of the large batch: 4096^2 (K-major
# operands), 4096 x 14336 (wide: B operand MN-major, X X^T over k = 14336)
# and 14336 x 4096 (tall: both X X^T operands MN-major)
LARGE_SAMPLE = [0, 8, 15]


@pytest.mark.slow
def test_large_batch_sampled():
    """The full large batch in one grouped call, in the launch configuration
    the benchmark times; the oracle checks one matrix of each orientation,
    singular values included."""
    shapes = workloads.large_batch_shapes()
    rng = np.random.default_rng(3)
    grads = [rng.standard_normal(s, dtype=np.float32) for s in shapes]
    grp = Group(shapes, BF, BF, BF, cond=False, seed=3)
    hp = hparams(dm.DM_PREC_BF16_TC)
    rep, _ = step_and_compare(grp, grads, hp, TOL_BF16, sample=LARGE_SAMPLE)
    assert len(rep.sv_err) == len(LARGE_SAMPLE)
    assert max(rep.o_err) < 2e-2


@pytest.mark.slow
def test_large_batch_dimuon_sampled():
    """The large batch through the Dimuon path (conditioning kernels, the
    last product's per-tile norm partials at 16 x 56 tiles, renormalisation
    and apply), two steps so that the second is conditioned by the first
    step's energies; one matrix of each orientation against the oracle."""
    shapes = workloads.large_batch_shapes()
    rng = np.random.default_rng(33)
    grp = Group(shapes, BF, BF, BF, cond=True, seed=3)
    hp = hparams(dm.DM_PREC_BF16_TC, weight_decay=0.01)
    ws = None
    for t in range(2):
        grads = [rng.standard_normal(s, dtype=np.float32) * rng.lognormal(0.0, 1.0, s[1])[None, :]
                 for s in shapes]
        rep, ws = step_and_compare(grp, grads, hp, TOL_BF16, ws=ws, sample=LARGE_SAMPLE,
                                   check_sv=t == 1)
        assert max(rep.o_err) < 2e-2
    assert len(rep.sv_err) == len(LARGE_SAMPLE)


@pytest.mark.parametrize("r,path", [(2, 0), (8, 0), (8, dm.DM_DBG_THIN_CLUSTER), (32, 0)],
                         ids=["r2", "r8", "r8-cluster", "r32"])
def test_lora_batch_twenty_steps(r, path):
    """224 projections (A r x 4096, B 4096 x r), fp32 momentum, bf16 weights,
    Dimuon, 20 steps: teacher-forced parity on a sample each step, dead rows
    of B capped at a 10x per-side gain, and a free-running oracle rerun of
    one projection at the end."""
    shapes = workloads.lora_shapes(r)
    stream = workloads.LoraGradStream(r)
    grp = Group(shapes, BF, BF, F32, cond=True, seed=4)
    lr = {2: 0.018, 8: 0.010, 32: 0.010}[r]
    hp = hparams(dm.DM_PREC_BF16_TC, lr=lr, debug_flags=path)
    ws = None
    h = orc.HParams(lr=lr)
    free = None
    for t in range(1, 21):
        grads = stream.step(t)
        er_prev = to_host(grp.er[1])
        if free is None:
            free = dict(W=to_host(grp.W[1]), M=to_host(grp.M[1]), er=np.zeros(shapes[1][0]),
                        ec=np.zeros(shapes[1][1]))
        g1 = to_host(to_dev(grads[1], BF))
        fr = orc.dimuon_step(free["W"], g1, free["M"], free["er"], free["ec"], h,
                             momentum_dtype="fp32", weight_dtype="bf16")
        free = dict(W=fr.W, M=fr.M, er=fr.e_row, ec=fr.e_col)
        sample = [0, 1, 2 * 111, 2 * 111 + 1, len(shapes) - 1]
        _, ws = step_and_compare(grp, grads, hp, thin_tol(True, TOL_THIN_SPLIT_ILL), ws=ws,
                                 sample=sample)
        dead = stream.dead[0]
        if t <= 5:
            # the dead rows of B stay out of the momentum and the update
            assert np.all(to_host(grp.er[1])[dead] == 0.0)
            assert np.all(to_host(grp.upd[1])[dead] == 0.0)
        if t == 6:
            assert np.all(er_prev[dead] == 0.0)
            gain = dead_row_gain(to_host(grp.upd[1]), to_host(grp.M[1]), er_prev, dead,
                                 float(np.float32(h.cond_eps)))
            # R = (0 + eps)^(-1/4) = 10 on each side of X_5: O gains R^2 = 100
            assert abs(gain / 100.0 - 1.0) < 1e-3, gain
    assert rel_fro(to_host(grp.W[1]), free["W"]) < 3e-2


# tensor-core path (K1), fp32 path, thin staged / cluster / register kernels
ROUNDING_SHAPES = [(64, 96), (8, 512), (512, 8), (2, 512), (32, 256), (8, 24), (5, 40)]


@pytest.mark.parametrize("mdt", [BF, F32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("prec", [dm.DM_PREC_BF16_TC, dm.DM_PREC_FP32], ids=["tc", "fp32"])
def test_momentum_rounds_the_exact_value_once(mdt, prec):
    """Inputs built so that rounding the float64 sum mu M + G to the storage
    type would round twice and differ from the exact value rounded once
    ("Muon Optimizer 정리", Update rule, eq. (1)): every kernel that forms
    M_t stores the correctly rounded value, bit-equal to the oracle."""
    mu, m, g = crafted_bf16_tie() if mdt == BF else crafted_fp32_tie()
    # (W, G, M) all bf16 or all fp32: storage combinations of every thin kernel
    grp = Group(ROUNDING_SHAPES, mdt, mdt, mdt, cond=False, seed=61)
    rng = np.random.default_rng(62)
    grads = []
    for i, s in enumerate(ROUNDING_SHAPES):
        M0 = rng.standard_normal(s)
        G0 = rng.standard_normal(s)
        M0.flat[::7] = m
        G0.flat[::7] = g
        grp.M[i].copy_(to_dev(M0, mdt))
        grads.append(G0)
    hp = hparams(prec, mu=mu)
    step_and_compare(grp, grads, hp, TOL_BF16 if prec == dm.DM_PREC_BF16_TC else TOL_FP32,
                     check_sv=False)
    # the constructed entries took the exact value's rounding
    want = orc.store_round(orc.momentum_update(np.array([m]), np.array([g]), np.float32(mu)),
                           "bf16" if mdt == BF else "fp32")[0]
    for i in range(len(ROUNDING_SHAPES)):
        assert np.all(to_host(grp.M[i]).flat[::7] == want)


def dead_row_gain(O, M, e_prev, dead, eps):
    """Gain the kernel gave the rows of a tall factor whose previous energy
    was zero, measured from its own output.  For a tall factor the conditioned
    update is O = s R^2 M K with one r x r matrix K = C q(X_0^T X_0) C for all
    rows ([Dimuon], '-1/4 power from both sides'), so row i is R_i^2 (M K)_i.
    K s is fitted on the live rows with R from the previous energies; the
    dead rows' O over their M (K s) is then their R^2."""
    live = np.setdiff1d(np.arange(O.shape[0]), dead)
    R = (e_prev / e_prev.mean() + eps) ** -0.25
    Ks, *_ = np.linalg.lstsq(M[live], O[live] / (R[live] ** 2)[:, None], rcond=None)
    pred = M[dead] @ Ks
    return float((O[dead] * pred).sum() / (pred * pred).sum())


# --------------------------------------------------------------------------
# 1-D parameters laid out at widths 1 .. 128 ("From PCG to Muon", section 6)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("width", [1, 2, 8, 32, 128])
def test_vector_reshape(width):
    """Vectors of ragged lengths at each width, Muon with momentum and
    Nesterov: the first `length` cells of M_t, O_t, W_t match the oracle's
    vector step (teacher-forced, three steps) and the padded momentum cells
    stay exactly zero."""
    lengths = [1000, 4099, 65537]
    shapes = [dm.vector_matrix_shape(L, width) for L in lengths]
    grp = Group(shapes, BF, BF, F32, cond=False, seed=31 + width)
    prec = dm.DM_PREC_FP32  # width 128 takes the fp32 Newton-Schulz kernels
    hp = hparams(prec, nesterov=1, weight_decay=0.01)
    h = oracle_hp(hp)
    rng = np.random.default_rng(width)
    ws = None
    for step in range(3):
        grads = []
        for (r, c), L in zip(shapes, lengths):
            g = np.zeros(r * c)
            g[:L] = rng.standard_normal(L)
            grads.append(g.reshape(r, c))
        before = [(to_host(grp.W[i]).reshape(-1)[:L], to_host(grp.M[i]).reshape(-1)[:L])
                  for i, L in enumerate(lengths)]
        ws, G = run_gpu_step(grp, grads, hp, ws)
        for i, L in enumerate(lengths):
            w0, m0 = before[i]
            g_host = to_host(G[i]).reshape(-1)[:L]
            res = orc.vector_step(w0, g_host, m0, width, h, momentum_dtype="fp32",
                                  weight_dtype="bf16")
            Mg = to_host(grp.M[i]).reshape(-1)
            Og = to_host(grp.upd[i]).reshape(-1)[:L]
            np.testing.assert_array_equal(Mg[:L], res.M)
            assert np.all(Mg[L:] == 0.0)
            assert rel_fro(Og, res.O) <= TOL_FP32, (width, L, rel_fro(Og, res.O))


# --------------------------------------------------------------------------
# per-iteration coefficient schedules (the mechanism Polar Express needs;
# "Dimuon: LoRA 에 맞춰 다시 짠 Muon", "16 columns with input size 0.1 to 10")
# --------------------------------------------------------------------------
# five distinct quintics; their composition maps [0, 1] into [0, 1]
SCHEDULE = ((3.4445, -4.7750, 2.0315), (3.0, -3.2, 1.2), (2.5, -2.2, 0.7),
            (1.875, -1.25, 0.375), (1.5, -0.5, 0.0))
SCHED_SHAPES = [(384, 640), (700, 260), (40, 100), (8, 4096), (4096, 8), (2, 2056),
                (32, 4096), (17, 333)]


@pytest.mark.parametrize("prec,dbg,tol", [
    (dm.DM_PREC_BF16_TC, 0, TOL_BF16), (dm.DM_PREC_BF16_TC, dm.DM_DBG_TC_SINGLE, TOL_BF16),
    (dm.DM_PREC_FP32, 0, TOL_FP32), (dm.DM_PREC_FP32, dm.DM_DBG_THIN_STAGED, TOL_FP32),
    (dm.DM_PREC_FP32, dm.DM_DBG_THIN_REGS, TOL_FP32),
    (dm.DM_PREC_FP32, dm.DM_DBG_THIN_CLUSTER, TOL_FP32)],
    ids=["tc-pair", "tc-single", "simt+thin-default", "simt+thin-staged", "simt+thin-regs",
         "simt+thin-cluster"])
@pytest.mark.parametrize("cond", [False, True])
def test_coefficient_schedule(prec, dbg, tol, cond):
    """Iteration k applies its own (a_k, b_k, c_k) on every path: tensor-core
    and fp32 products, and the thin factors' r x r iteration (single-pass,
    staged and register kernels)."""
    grp = Group(SCHED_SHAPES, BF, BF, F32, cond=cond, seed=41)
    hp = hparams(prec, weight_decay=0.01, debug_flags=dbg, ns_coeffs=SCHEDULE)
    assert hp.ns_steps == len(SCHEDULE)
    ws = None
    for t in range(2):
        thin_tol = TOL_FP32 if prec == dm.DM_PREC_FP32 else tol
        _, ws = step_and_compare(grp, gaussian(SCHED_SHAPES, 1100 + t, scale_cols=True), hp,
                                 max(tol, thin_tol), ws=ws)


@pytest.mark.parametrize("prec", [dm.DM_PREC_FP32, dm.DM_PREC_BF16_TC])
def test_constant_schedule_is_bitwise_the_fixed_step(prec):
    """A schedule repeating the default (a, b, c) gives the default step bit
    for bit (weights, momentum, energies, update)."""
    g = gaussian(SCHED_SHAPES, 1200)
    fixed = Group(SCHED_SHAPES, BF, BF, F32, cond=True, seed=42)
    sched = Group(SCHED_SHAPES, BF, BF, F32, cond=True, seed=42)
    hp = hparams(prec)
    run_gpu_step(fixed, g, hp)
    run_gpu_step(sched, g, hparams(prec, ns_coeffs=[(hp.a, hp.b, hp.c)] * hp.ns_steps))
    for name in ("W", "M", "er", "ec", "upd"):
        for a, b in zip(getattr(fixed, name), getattr(sched, name)):
            assert torch.equal(a, b), name


# --------------------------------------------------------------------------
# resume: a step continued from state saved to the host and reloaded into
# fresh buffers (and a fresh workspace) equals the uninterrupted run bit for
# bit (the library keeps no state of its own between calls)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("prec", [dm.DM_PREC_FP32, dm.DM_PREC_BF16_TC])
def test_resume_from_saved_state_is_bitwise(prec):
    shapes = [(256, 384), (384, 256), (8, 4096), (4096, 16), (2, 2056), (40, 100)]
    hp = hparams(prec, weight_decay=0.01, scale_mode=dm.DM_SCALE_MOONSHOT)
    grads = [gaussian(shapes, 1300 + t, scale_cols=True) for t in range(4)]
    run = Group(shapes, BF, BF, F32, cond=True, seed=43)
    ws = None
    saved = None
    for t in range(4):
        ws, _ = run_gpu_step(run, grads[t], hp, ws)
        if t == 1:  # checkpoint after two steps: weights, momentum, energies
            saved = {k: [x.detach().cpu().clone() for x in getattr(run, k)]
                     for k in ("W", "M", "er", "ec")}
    resumed = Group(shapes, BF, BF, F32, cond=True, seed=99)  # other initial values
    for k, host in saved.items():
        for dst, src in zip(getattr(resumed, k), host):
            dst.copy_(src.cuda())
    ws2 = None
    for t in (2, 3):
        ws2, _ = run_gpu_step(resumed, grads[t], hp, ws2)
    for k in ("W", "M", "er", "ec", "upd"):
        for a, b in zip(getattr(run, k), getattr(resumed, k)):
            assert torch.equal(a, b), k
