"""Checked-workspace mode (DM_DBG_CANARY): 256 canary bytes after the
workspace header and after every workspace region, filled at a step's start
and checked at its end.  Stand-in for a memory sanitizer, which this pool
does not offer: every path's kernels must leave all canaries intact, with
results bit-equal to the unchecked mode, and a changed canary must be
reported."""
import numpy as np
import pytest
import torch

import dimuon_optimizer_b200 as dm
from gpu_harness import Group, to_dev

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

BF, F32 = dm.DM_BF16, dm.DM_FP32
# tensor-core / fp32 products (wide, tall, ragged) and thin factors of every
# thin kernel (cluster, staged, register)
SHAPES = [(384, 640), (700, 260), (40, 100), (8, 4096), (4096, 8), (2, 2056), (32, 4096),
          (17, 333), (1001, 8), (4, 16)]


def grads(seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal(s) for s in SHAPES]


@pytest.mark.parametrize("prec,path", [(dm.DM_PREC_BF16_TC, 0), (dm.DM_PREC_FP32, 0),
                                       (dm.DM_PREC_BF16_TC, dm.DM_DBG_THIN_STAGED),
                                       (dm.DM_PREC_BF16_TC, dm.DM_DBG_THIN_REGS),
                                       (dm.DM_PREC_BF16_TC, dm.DM_DBG_THIN_CLUSTER)],
                         ids=["tc", "fp32", "thin-staged", "thin-regs", "thin-cluster"])
@pytest.mark.parametrize("cond", [False, True])
def test_checked_mode_leaves_canaries_and_results(prec, path, cond):
    plain = Group(SHAPES, BF, BF, F32, cond=cond, seed=81)
    checked = Group(SHAPES, BF, BF, F32, cond=cond, seed=81)
    hp = dm.dm_default_hparams(precision=prec, weight_decay=0.01, debug_flags=path)
    hpc = dm.dm_default_hparams(precision=prec, weight_decay=0.01,
                                debug_flags=path | dm.DM_DBG_CANARY)
    fn = dm.dm_dimuon_step if cond else dm.dm_muon_step
    ws = wsc = None
    for step in range(3):
        G = [to_dev(g, BF) for g in grads(90 + step)]
        mp, mc = plain.matrices(G), checked.matrices(G)
        if ws is None:
            ws = torch.empty(dm.dm_workspace_size(mp, hp, int(cond)), dtype=torch.uint8,
                             device="cuda")
            wsc = torch.empty(dm.dm_workspace_size(mc, hpc, int(cond)), dtype=torch.uint8,
                              device="cuda")
            assert wsc.numel() > ws.numel()
        dm.check(fn(mp, hp, ws))
        dm.check(fn(mc, hpc, wsc))
        assert dm.dm_read_device_status(wsc) == dm.DM_OK
        assert dm.dm_read_device_status(ws) == dm.DM_OK
        for name in ("W", "M", "upd") + (("er", "ec") if cond else ()):
            for a, b in zip(getattr(plain, name), getattr(checked, name)):
                assert torch.equal(a, b), name


def test_changed_canary_is_reported():
    """The checker's self-test hook leaves one canary word wrong at the fill:
    the step must end with DM_ERR_CANARY, and the next checked step (which
    refills the canaries) reads clean again, with the same results as an
    unchecked step."""
    grp = Group(SHAPES[:4], BF, BF, F32, cond=True, seed=82)
    ref = Group(SHAPES[:4], BF, BF, F32, cond=True, seed=82)
    hp = dm.dm_default_hparams(debug_flags=dm.DM_DBG_CANARY)
    bad = dm.dm_default_hparams(debug_flags=dm.DM_DBG_CANARY | dm.DM_DBG_CANARY_SELFTEST)
    G = [to_dev(g, BF) for g in grads(95)[:4]]
    mats = grp.matrices(G)
    ws = torch.empty(dm.dm_workspace_size(mats, hp, 1), dtype=torch.uint8, device="cuda")
    dm.check(dm.dm_dimuon_step(mats, bad, ws))
    assert dm.dm_read_device_status(ws) == dm.DM_ERR_CANARY
    dm.check(dm.dm_dimuon_step(mats, hp, ws))
    assert dm.dm_read_device_status(ws) == dm.DM_OK
    # the hook changes a canary, not the arithmetic
    hp0 = dm.dm_default_hparams()
    mref = ref.matrices(G)
    ws0 = torch.empty(dm.dm_workspace_size(mref, hp0, 1), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        dm.check(dm.dm_dimuon_step(mref, hp0, ws0))
    for name in ("W", "M", "er", "ec", "upd"):
        for a, b in zip(getattr(grp, name), getattr(ref, name)):
            assert torch.equal(a, b), name
