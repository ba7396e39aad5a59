"""Helpers for the GPU parity tests: build device buffers from seeded host
arrays, run one library step through the C ABI, and compare it element by
element with the fp64 oracle run on the same (teacher-forced) state."""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

import dimuon_optimizer_b200 as dm
import oracle as orc

TOL_FP32 = 1e-5      # relative Frobenius error of O_t, fp32 mode / thin path
TOL_BF16 = 3e-2      # relative Frobenius error of O_t, bf16 tensor-core mode
TOL_SV = 0.05        # singular values of O_t / kappa
# staged r = 32 thin factors in bf16 tensor-core mode: Gram and apply sums on
# bf16 tensor cores with hi / lo split operands (about 2^-16 relative per
# term, fp32 accumulation) instead of fp64.  The Gram route squares the
# factor's condition number, so the error grows with it: a few 1e-6 on
# Gaussian factors (1e-4 bound here), up to 1.2e-3 on the first, unconditioned
# step of the LoRA batch whose column scales span 1e-2 .. 1e6 (5e-3 bound);
# both well inside the bf16 mode's 3e-2.
TOL_THIN_SPLIT = 1e-4
TOL_THIN_SPLIT_ILL = 5e-3


def thin_tol(precision_bf16, split_tol=TOL_THIN_SPLIT):
    """Tolerance of O_t for a thin-factor group: fp64 sums everywhere except
    the r = 32 factors in bf16 tensor-core mode."""
    if not precision_bf16:
        return TOL_FP32
    return lambda shape: split_tol if min(shape) == 32 else TOL_FP32


def tdtype(code):
    return torch.bfloat16 if code == dm.DM_BF16 else torch.float32


def sname(code):
    return "bf16" if code == dm.DM_BF16 else "fp32"


def to_dev(x, code):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(tdtype(code)).cuda()


def to_host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@dataclass
class Group:
    shapes: list
    wdt: int = dm.DM_BF16
    gdt: int = dm.DM_BF16
    mdt: int = dm.DM_BF16
    cond: bool = False
    seed: int = 0
    W: list = field(default_factory=list)
    M: list = field(default_factory=list)
    er: list = field(default_factory=list)
    ec: list = field(default_factory=list)
    upd: list = field(default_factory=list)

    def __post_init__(self):
        rng = np.random.default_rng(self.seed + 1000)
        for (r, c) in self.shapes:
            self.W.append(to_dev(0.02 * rng.standard_normal((r, c)), self.wdt))
            self.M.append(torch.zeros((r, c), dtype=tdtype(self.mdt), device="cuda"))
            self.er.append(torch.zeros(r, dtype=torch.float32, device="cuda"))
            self.ec.append(torch.zeros(c, dtype=torch.float32, device="cuda"))
            self.upd.append(torch.zeros((r, c), dtype=torch.float32, device="cuda"))

    def matrices(self, G):
        return [dm.dm_matrix(self.W[i], G[i], self.M[i],
                             self.er[i] if self.cond else None,
                             self.ec[i] if self.cond else None, self.upd[i])
                for i in range(len(self.shapes))]


def run_gpu_step(grp: Group, grads_host, hp, ws=None):
    G = [to_dev(g, grp.gdt) for g in grads_host]
    mats = grp.matrices(G)
    need = dm.dm_workspace_size(mats, hp, int(grp.cond))
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    fn = dm.dm_dimuon_step if grp.cond else dm.dm_muon_step
    dm.check(fn(mats, hp, ws))
    torch.cuda.synchronize()
    return ws, G


def oracle_hp(hp):
    coeffs = None
    if hp.ns_coeffs:
        coeffs = tuple((hp.ns_coeffs[3 * k], hp.ns_coeffs[3 * k + 1], hp.ns_coeffs[3 * k + 2])
                       for k in range(hp.ns_steps))
    return orc.HParams(mu=hp.mu, lr=hp.lr, weight_decay=hp.weight_decay, ns_steps=hp.ns_steps,
                       a=hp.a, b=hp.b, c=hp.c, cond_eps=hp.cond_eps, scale_mode=hp.scale_mode,
                       scale_coef=hp.scale_coef, nesterov=bool(hp.nesterov), ns_coeffs=coeffs)


def rel_fro(x, y):
    ny = np.linalg.norm(y)
    return np.linalg.norm(x - y) / (ny if ny > 0 else 1.0)


def storage_ulp(x, code):
    """Spacing of the storage format at |x| (bf16: 8 significant bits)."""
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1e-300)))
    bits = 7 if code == dm.DM_BF16 else 23
    return np.where(a > 0, 2.0 ** (e - bits), 2.0 ** -133)


@dataclass
class StepReport:
    o_err: list
    sv_err: list
    m_mismatch: list


def step_and_compare(grp: Group, grads_host, hp, o_tol, *, ws=None, check_sv=True,
                     sample=None):
    """One teacher-forced step: snapshot state, run the GPU step, run the
    oracle on the snapshot, compare.  `sample` limits the oracle to a subset
    of matrix indices (full-size groups)."""
    idx = range(len(grp.shapes)) if sample is None else sample
    before = {i: (to_host(grp.W[i]), to_host(grp.M[i]), to_host(grp.er[i]), to_host(grp.ec[i]))
              for i in idx}
    ws, G = run_gpu_step(grp, grads_host, hp, ws)
    h = oracle_hp(hp)
    rep = StepReport([], [], [])
    for i in idx:
        W0, M0, er0, ec0 = before[i]
        g_host = to_host(G[i])
        res = orc.optimizer_step(W0, g_host, M0, h, conditioned=grp.cond, e_row_prev=er0,
                                 e_col_prev=ec0, momentum_dtype=sname(grp.mdt),
                                 weight_dtype=sname(grp.wdt))
        Mg, Wg, Og = to_host(grp.M[i]), to_host(grp.W[i]), to_host(grp.upd[i])
        # momentum: both sides round the exact value of mu M + G once -> equal
        dM = np.abs(Mg - res.M)
        rep.m_mismatch.append(int((dM > 0).sum()))
        assert rep.m_mismatch[-1] == 0, (i, dM.max())
        # the update
        e = rel_fro(Og, res.O)
        rep.o_err.append(e)
        tol = o_tol(grp.shapes[i]) if callable(o_tol) else o_tol
        assert e <= tol, (i, grp.shapes[i], e)
        # the apply: W_t = (1 - lr wd) W_{t-1} - lr O_t with the GPU's own O_t
        decay = np.float32(1.0) - np.float32(hp.lr) * np.float32(hp.weight_decay)
        Wexp = store_round_np(float(decay) * W0 - float(np.float32(hp.lr)) * Og, grp.wdt)
        dW = np.abs(Wg - Wexp)
        assert np.all(dW <= storage_ulp(Wexp, grp.wdt) * 1.0001 + 1e-7), (i, dW.max())
        if grp.cond:
            Mt = Mg
            np.testing.assert_allclose(to_host(grp.er[i]), (Mt * Mt).sum(1), rtol=2e-5, atol=1e-30)
            np.testing.assert_allclose(to_host(grp.ec[i]), (Mt * Mt).sum(0), rtol=2e-5, atol=1e-30)
        # singular values of both updates (fp64 LAPACK; seconds up to a
        # 4096-wide short side)
        if check_sv and min(grp.shapes[i]) <= 4096 and np.linalg.norm(res.O) > 0:
            kap = orc.scale_factor(hp.scale_mode, orc.f32(hp.scale_coef), *grp.shapes[i])
            sg = np.linalg.svd(Og / kap, compute_uv=False)
            so = np.linalg.svd(res.O / kap, compute_uv=False)
            d = float(np.abs(sg - so).max())
            rep.sv_err.append(d)
            assert d <= TOL_SV, (i, d)
    return rep, ws


def store_round_np(x, code):
    return orc.store_round(x, sname(code))
