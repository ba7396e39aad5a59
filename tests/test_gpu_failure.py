"""Failure detection on the GPU without a fault: the tensor-core kernels'
bounded waits.  The DM_DBG_FORCE_TIMEOUT hook makes one wait per product
launch run out (20 ms, on a barrier nothing arrives on) before any copy or
product is issued; the test checks that the expiry reaches the host as
DM_ERR_DEVICE_TIMEOUT through the device status word, that the step ends in
bounded time, that no later launch of the step wrote a weight or an update
(the timed-out product left its buffers half written), and that the context
stays usable: the next ordinary step on the same device matches the
oracle."""
import time

import numpy as np
import pytest
import torch

import dimuon_optimizer_b200 as dm
import workloads
from gpu_harness import TOL_BF16, Group, run_gpu_step, step_and_compare, to_host

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

SHAPES = [(384, 640), (640, 384)]


@pytest.mark.parametrize("kernel", [dm.DM_DBG_TC_SINGLE, dm.DM_DBG_TC_PAIR],
                         ids=["single", "pair"])
@pytest.mark.parametrize("cond", [False, True], ids=["muon", "dimuon"])
def test_forced_timeout_is_reported_and_context_survives(kernel, cond):
    grads = workloads.gaussian_grads(SHAPES, seed=71)
    bad = Group(SHAPES, cond=cond, seed=71)
    W0 = [w.clone() for w in bad.W]
    hp = dm.dm_default_hparams(debug_flags=kernel | dm.DM_DBG_FORCE_TIMEOUT)
    t0 = time.monotonic()
    ws, _ = run_gpu_step(bad, grads, hp)
    status = dm.dm_read_device_status(ws)
    elapsed = time.monotonic() - t0
    assert status == dm.DM_ERR_DEVICE_TIMEOUT, dm.dm_status_string(status)
    # the first product launch gives up after 20 ms; every later one leaves
    assert elapsed < 10.0, elapsed
    # no weight or update was written from the half-computed products
    for w0, w, u in zip(W0, bad.W, bad.upd):
        assert torch.equal(w, w0)
        assert not bool(u.any())

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
    W0 = grp.W[0].clone()
    ws, _ = run_gpu_step(grp, grads, dm.dm_default_hparams(debug_flags=dm.DM_DBG_FORCE_TIMEOUT))
    assert dm.dm_read_device_status(ws) == dm.DM_ERR_DEVICE_TIMEOUT
    # the aborted step left W as it was (its momentum update precedes the
    # products and stays: M_1 = G)
    assert torch.equal(grp.W[0], W0)
    np.testing.assert_array_equal(to_host(grp.M[0]),
                                  to_host(torch.from_numpy(grads[0].astype(np.float32))
                                          .to(grp.M[0].dtype)))
    ws, _ = run_gpu_step(grp, grads, dm.dm_default_hparams(), ws)
    assert dm.dm_read_device_status(ws) == dm.DM_OK
    assert np.isfinite(grp.M[0].float().cpu().numpy()).all()
    assert not torch.equal(grp.W[0], W0)
