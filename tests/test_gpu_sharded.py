"""The sharded step's GPU leg at one rank: the library updates the owned
matrices in place inside the flat weight buffer; with a single rank this must
equal the ordinary step on separately allocated buffers, bit for bit, with
the gradients given as separate tensors or in the flat gradient layout."""
import numpy as np
import pytest
import torch

import dimuon_optimizer_b200 as dm
import workloads
from dimuon_optimizer_b200 import sharded

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]


@pytest.mark.parametrize("prebuilt", [False, True], ids=["per_call", "prebuilt"])
@pytest.mark.parametrize("flat_grads", [False, True], ids=["grad_list", "grad_flat"])
@pytest.mark.parametrize("cond", [False, True])
def test_sharded_single_rank_matches_plain_step(cond, flat_grads, prebuilt):
    shapes = workloads.gpt2_small_shapes(layers=1) + workloads.lora_shapes(8, projections=3)
    plan = sharded.plan_shards(shapes, 1)
    sw = sharded.ShardedWeights(plan, dtype=torch.bfloat16, device="cuda")
    rng = np.random.default_rng(3)
    W0 = [torch.from_numpy(0.02 * rng.standard_normal(s)).to(torch.bfloat16).cuda() for s in shapes]
    G = [torch.from_numpy(rng.standard_normal(s)).to(torch.bfloat16).cuda() for s in shapes]
    for v, w in zip(sw.views, W0):
        v.copy_(w)
    Wp = [w.clone() for w in W0]
    M1 = {i: torch.zeros(s, dtype=torch.float32, device="cuda") for i, s in enumerate(shapes)}
    M2 = [torch.zeros(s, dtype=torch.float32, device="cuda") for s in shapes]
    er1 = {i: torch.zeros(s[0], device="cuda") for i, s in enumerate(shapes)}
    ec1 = {i: torch.zeros(s[1], device="cuda") for i, s in enumerate(shapes)}
    er2 = [torch.zeros(s[0], device="cuda") for s in shapes]
    ec2 = [torch.zeros(s[1], device="cuda") for s in shapes]
    hp = dm.dm_default_hparams(weight_decay=0.01)
    nb = sharded.workspace_bytes(sw, 0, G, M1, hp, cond, er1, ec1)
    ws1 = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mats = [dm.dm_matrix(Wp[i], G[i], M2[i], er2[i] if cond else None, ec2[i] if cond else None)
            for i in range(len(shapes))]
    ws2 = torch.empty(dm.dm_workspace_size(mats, hp, int(cond)), dtype=torch.uint8, device="cuda")
    grads = G
    if flat_grads:
        grads = sharded.ShardedGrads(plan, dtype=torch.bfloat16, device="cuda")
        for v, g in zip(grads.views, G):
            v.copy_(g)
    owned = (sharded.owned_matrices(sw, 0, grads, M1, conditioned=cond, row_energy=er1,
                                    col_energy=ec1) if prebuilt else None)
    for _ in range(2):
        sharded.sharded_step(sw, 0, grads, M1, hp, ws1, conditioned=cond, row_energy=er1,
                             col_energy=ec1, mats=owned)
        dm.check((dm.dm_dimuon_step if cond else dm.dm_muon_step)(mats, hp, ws2))
    torch.cuda.synchronize()
    for i in range(len(shapes)):
        assert torch.equal(sw.views[i], Wp[i]), i
        assert torch.equal(M1[i], M2[i]), i
