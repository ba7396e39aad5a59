"""dm_step_noalloc: the step for callers that cannot allocate device memory
(for example code inside a framework whose caching allocator holds the whole
device, or a latency-critical path where cudaMalloc would synchronise).  Its
scratch memory is the library's own fixed 32 MiB device array, so its results
must match the workspace-taking entry points on the same inputs, call after
call, even though every call reuses what the previous one left in the array.

Neither side may depend on scratch contents it did not write: the reference
workspace is filled with 0xFF bytes (NaN as fp32 / bf16) before every call,
and before the compared calls the array is left holding another group's
results (other shapes, the other mode).
"""
import numpy as np
import pytest
import torch

import dimuon_optimizer_b200 as dm
from gpu_harness import TOL_FP32, Group, rel_fro, storage_ulp, to_dev, to_host

SHAPES = [(256, 384), (300, 200), (8, 512), (40, 100), (32, 256)]
FOREIGN = [(520, 136), (2, 2056), (64, 96), (4096, 32)]


def grads(step):
    rng = np.random.default_rng(50 + step)
    return [rng.standard_normal(s) for s in SHAPES]


def test_oversize_group_rejected_before_device_work():
    """A group whose workspace would exceed the fixed array is refused with
    DM_ERR_WORKSPACE; this check is host-only."""
    m = dm.dm_matrix_t()
    m.rows = m.cols = 4096
    m.weight, m.grad, m.momentum = 0x1000, 0x2000, 0x3000
    hp = dm.dm_default_hparams()
    assert dm.dm_workspace_size([m], hp, 0) > dm.DM_NOALLOC_MAX_BYTES
    assert dm.dm_step_noalloc([m], hp, 0, stream=0) == dm.DM_ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
@pytest.mark.parametrize("conditioned", [0, 1])
def test_noalloc_matches_workspace_entry_point(conditioned):
    hp = dm.dm_default_hparams(precision=dm.DM_PREC_BF16_TC, weight_decay=0.1,
                               scale_mode=dm.DM_SCALE_MOONSHOT)
    ref = Group(SHAPES, dm.DM_BF16, dm.DM_BF16, dm.DM_FP32, cond=bool(conditioned), seed=31)
    new = Group(SHAPES, dm.DM_BF16, dm.DM_BF16, dm.DM_FP32, cond=bool(conditioned), seed=31)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ws = None
    step_fn = dm.dm_dimuon_step if conditioned else dm.dm_muon_step
    # another group, in the other mode, leaves its results in the array
    other = Group(FOREIGN, dm.DM_BF16, dm.DM_BF16, dm.DM_FP32, cond=not conditioned, seed=32)
    rng = np.random.default_rng(60)
    for _ in range(2):
        Gf = [to_dev(rng.standard_normal(s), dm.DM_BF16) for s in FOREIGN]
        dm.check(dm.dm_step_noalloc(other.matrices(Gf), hp, 1 - conditioned, status))
    torch.cuda.synchronize()
    assert int(status.item()) == dm.DM_OK
    for step in range(2):  # two calls in a row on the shared array
        G = [to_dev(g, dm.DM_BF16) for g in grads(step)]
        mats_ref = ref.matrices(G)
        if ws is None:
            ws = torch.empty(dm.dm_workspace_size(mats_ref, hp, conditioned), dtype=torch.uint8,
                             device="cuda")
        assert dm.dm_workspace_size(mats_ref, hp, conditioned) <= dm.DM_NOALLOC_MAX_BYTES
        ws.fill_(0xFF)  # poison: a read of scratch the step did not write shows up as NaN
        dm.check(step_fn(mats_ref, hp, ws))
        dm.check(dm.dm_step_noalloc(new.matrices(G), hp, conditioned, status))
        torch.cuda.synchronize()
        assert int(status.item()) == dm.DM_OK
        assert dm.dm_read_device_status(ws) == dm.DM_OK
        for i in range(len(SHAPES)):
            assert rel_fro(to_host(new.upd[i]), to_host(ref.upd[i])) <= TOL_FP32
            np.testing.assert_array_equal(to_host(new.M[i]), to_host(ref.M[i]))
            Wr = to_host(ref.W[i])
            assert np.all(np.abs(to_host(new.W[i]) - Wr)
                          <= storage_ulp(Wr, dm.DM_BF16) * 1.0001)
            if conditioned:
                np.testing.assert_allclose(to_host(new.er[i]), to_host(ref.er[i]), rtol=2e-5)
                np.testing.assert_allclose(to_host(new.ec[i]), to_host(ref.ec[i]), rtol=2e-5)
