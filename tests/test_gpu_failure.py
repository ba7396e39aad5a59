"""Failure detection on the GPU without a fault: the tensor-core kernels'
bounded waits.  The DM_DBG_FORCE_TIMEOUT hook makes one wait per product
launch run out (20 ms, on a barrier nothing arrives on) before any copy or
product is issued; the test checks that the expiry reaches the host as
DM_ERR_DEVICE_TIMEOUT through the device status word, that the step ends in
bounded time, and that the context stays usable: the next ordinary step on
the same device matches the oracle."""
import time

import numpy as np
import pytest
import torch

import dimuon_optimizer_b200 as dm
import workloads
from gpu_harness import TOL_BF16, Group, run_gpu_step, step_and_compare

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

SHAPES = [(384, 640), (640, 384)]


@pytest.mark.parametrize("kernel", [dm.DM_DBG_TC_SINGLE, dm.DM_DBG_TC_PAIR],
                         ids=["single", "pair"])
@pytest.mark.parametrize("cond", [False, True], ids=["muon", "dimuon"])
def test_forced_timeout_is_reported_and_context_survives(kernel, cond):
    grads = workloads.gaussian_grads(SHAPES, seed=71)
    bad = Group(SHAPES, cond=cond, seed=71)
    hp = dm.dm_default_hparams(debug_flags=kernel | dm.DM_DBG_FORCE_TIMEOUT)
    t0 = time.monotonic()
    ws, _ = run_gpu_step(bad, grads, hp)
    status = dm.dm_read_device_status(ws)
    elapsed = time.monotonic() - t0
    assert status == dm.DM_ERR_DEVICE_TIMEOUT, dm.dm_status_string(status)
    # 5 iterations x 3 products, each launch giving up after 20 ms
    assert elapsed < 10.0, elapsed

    # the same workspace and device, an ordinary step: parity with the oracle
    good = Group(SHAPES, cond=cond, seed=72)
    hp_ok = dm.dm_default_hparams(debug_flags=kernel)
    step_and_compare(good, grads, hp_ok, TOL_BF16, ws=ws)
    assert dm.dm_read_device_status(ws) == dm.DM_OK
    # and a second one on its state (momentum, energies carried over)
    step_and_compare(good, workloads.gaussian_grads(SHAPES, seed=73), hp_ok, TOL_BF16, ws=ws)
    assert dm.dm_read_device_status(ws) == dm.DM_OK


def test_status_cleared_by_next_step():
    """A step clears the status word at its start: after a forced timeout an
    ordinary step on the same workspace reads back DM_OK."""
    grads = workloads.gaussian_grads(SHAPES[:1], seed=74)
    grp = Group(SHAPES[:1], seed=74)
    ws, _ = run_gpu_step(grp, grads, dm.dm_default_hparams(debug_flags=dm.DM_DBG_FORCE_TIMEOUT))
    assert dm.dm_read_device_status(ws) == dm.DM_ERR_DEVICE_TIMEOUT
    ws, _ = run_gpu_step(grp, grads, dm.dm_default_hparams(), ws)
    assert dm.dm_read_device_status(ws) == dm.DM_OK
    # the momentum was still updated by the aborted step (it precedes the
    # products), so it stays finite
    assert np.isfinite(grp.M[0].float().cpu().numpy()).all()
