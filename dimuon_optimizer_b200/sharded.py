"""Whole-matrix sharding of one optimizer step over data-parallel ranks.

Each matrix's update depends on that matrix alone ("Muon Optimizer 정리",
eq. (1)-(3); "Dimuon: LoRA 에 맞춰 다시 짠 Muon": the conditioning is per
matrix), so a step over many matrices splits by matrix: every rank updates
the matrices it owns (its momentum and energy buffers exist only there) and
the updated weights are then exchanged so every rank holds all of them.

Layout.  All weights live in one flat buffer, rank by rank: the matrices a rank
owns sit back to back (in their original order, each start aligned to 128
elements so the library's vector and bulk-copy paths stay aligned) in that
rank's slice, and every slice has the same padded length.  The exchange is
then a single all-gather of the slices into the same buffer (NCCL over
NVLink / NVSwitch on a GPU node; gloo on CPU for the tests).  Gradients can
use the same layout (ShardedGrads): the data-parallel gradient reduction then
becomes one reduce-scatter that leaves each rank the averaged gradients of
exactly the matrices it owns (ZeRO-style: no rank needs the others' reduced
gradients).

Ownership.  A greedy longest-processing-time assignment by estimated cost:
algorithmic Newton-Schulz flops 5 (3 m^2 n + m^3) at the measured bf16 rate
for matrices with a short side above 32, streamed bytes (14 per element) at
the measured HBM rate for thin factors.

This module is host plumbing (torch.distributed); every step of the
arithmetic runs in libdimuon through the binding.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import DM_THIN_MAX

ALIGN_ELEMS = 128
_NS_RATE = 1.3e15   # bf16 tensor-core flop/s (sustained, measured order of magnitude)
_HBM_RATE = 6.5e12  # bytes/s


def matrix_cost(rows: int, cols: int, ns_steps: int = 5) -> float:
    """Estimated seconds of one step on one matrix (used only to balance)."""
    m, n = min(rows, cols), max(rows, cols)
    if m <= DM_THIN_MAX:
        return 14.0 * m * n / _HBM_RATE
    return ns_steps * (3.0 * m * m * n + m ** 3) / _NS_RATE + 10.0 * m * n / _HBM_RATE


def _align(x: int) -> int:
    return (x + ALIGN_ELEMS - 1) // ALIGN_ELEMS * ALIGN_ELEMS


@dataclass(frozen=True)
class ShardPlan:
    shapes: tuple            # (rows, cols) per matrix, in the caller's order
    world: int
    owner: tuple             # rank owning each matrix
    offset: tuple            # element offset of each matrix in the flat buffer
    slice_elems: int         # padded elements per rank slice

    def owned(self, rank: int) -> list:
        """Indices of the matrices rank `rank` updates, in the caller's order."""
        return [i for i, o in enumerate(self.owner) if o == rank]

    @property
    def total_elems(self) -> int:
        return self.world * self.slice_elems

    def load(self, rank: int) -> float:
        return sum(matrix_cost(*self.shapes[i]) for i in self.owned(rank))


def plan_shards(shapes, world: int) -> ShardPlan:
    """Deterministic balanced ownership and the flat layout (see module doc)."""
    shapes = tuple((int(r), int(c)) for r, c in shapes)
    if world < 1:
        raise ValueError("world must be >= 1")
    costs = [matrix_cost(r, c) for r, c in shapes]
    order = sorted(range(len(shapes)), key=lambda i: (-costs[i], i))
    load = [0.0] * world
    owner = [0] * len(shapes)
    for i in order:
        k = min(range(world), key=lambda q: (load[q], q))
        owner[i] = k
        load[k] += costs[i]
    used = [0] * world
    local = [0] * len(shapes)
    for i, (r, c) in enumerate(shapes):
        local[i] = used[owner[i]]
        used[owner[i]] += _align(r * c)
    slice_elems = max(used + [ALIGN_ELEMS])
    offset = tuple(owner[i] * slice_elems + local[i] for i in range(len(shapes)))
    return ShardPlan(shapes, world, tuple(owner), offset, slice_elems)


class ShardedWeights:
    """The flat weight buffer of a plan and one view per matrix."""

    def __init__(self, plan: ShardPlan, dtype=torch.bfloat16, device="cuda"):
        self.plan = plan
        self.flat = torch.zeros(plan.total_elems, dtype=dtype, device=device)
        self.views = [self.flat[o:o + r * c].view(r, c) for o, (r, c) in zip(plan.offset, plan.shapes)]

    def my_slice(self, rank: int) -> torch.Tensor:
        s = self.plan.slice_elems
        return self.flat[rank * s:(rank + 1) * s]

    def gather(self, rank: int, group=None):
        """Every rank's slice to every rank, in place (the step's one exchange)."""
        import torch.distributed as dist
        if self.plan.world == 1:
            return
        s = self.plan.slice_elems
        if dist.get_backend(group) == "nccl":
            dist.all_gather_into_tensor(self.flat, self.my_slice(rank).clone(), group=group)
        else:
            parts = [self.flat[q * s:(q + 1) * s] for q in range(self.plan.world)]
            dist.all_gather(parts, self.my_slice(rank).clone(), group=group)


class ShardedGrads:
    """Flat gradient buffer in a plan's layout.  Each rank's backward writes its
    local gradients into `views`; reduce() then leaves, in the views of the
    matrices this rank owns, the mean (or sum) over ranks of those gradients,
    with one reduce-scatter of the slices (the other views keep local values)."""

    def __init__(self, plan: ShardPlan, dtype=torch.bfloat16, device="cuda"):
        self.plan = plan
        self.flat = torch.zeros(plan.total_elems, dtype=dtype, device=device)
        self.views = [self.flat[o:o + r * c].view(r, c) for o, (r, c) in zip(plan.offset, plan.shapes)]
        self._recv = torch.empty(plan.slice_elems, dtype=dtype, device=device)

    def reduce(self, rank: int, group=None, average: bool = True):
        import torch.distributed as dist
        if self.plan.world == 1:
            return
        s = self.plan.slice_elems
        dist.reduce_scatter_tensor(self._recv, self.flat, group=group)
        if average:
            self._recv.div_(self.plan.world)
        self.flat[rank * s:(rank + 1) * s].copy_(self._recv)


def owned_matrices(weights: ShardedWeights, rank: int, grads, momenta, *, conditioned=False,
                   row_energy=None, col_energy=None, update_out=None):
    """The library's matrix descriptors for the matrices `rank` owns, built
    once: pass them to sharded_step as `mats` while the same tensors are used
    step after step (the descriptors hold their addresses).  `grads` as in
    sharded_step (a ShardedGrads: its views)."""
    from . import _array, dm_matrix
    views = grads.views if isinstance(grads, ShardedGrads) else grads
    idx = weights.plan.owned(rank)
    mats = [dm_matrix(weights.views[i], views[i], momenta[i],
                      row_energy[i] if conditioned else None,
                      col_energy[i] if conditioned else None,
                      update_out.get(i) if update_out else None) for i in idx]
    return _array(mats)[0] if mats else None


def sharded_step(weights: ShardedWeights, rank: int, grads, momenta, hp, workspace, *,
                 conditioned=False, row_energy=None, col_energy=None, update_out=None,
                 stream=None, group=None, mats=None):
    """One sharded step: the library updates this rank's matrices in place in
    the flat buffer, then the slices are all-gathered.

    grads:    a ShardedGrads holding this rank's local gradients (reduced here
              by one reduce-scatter, averaged over ranks), or one tensor per
              matrix of the plan holding the already reduced gradient (only the
              owned ones are read)
    momenta / row_energy / col_energy / update_out: dicts from matrix index to
              tensor, for the owned matrices only
    workspace: device buffer of at least workspace_bytes(...) for the owned set
    mats:     optional descriptors from owned_matrices (skips rebuilding them)
    """
    from . import dm_dimuon_step, dm_matrix, dm_muon_step, check
    if isinstance(grads, ShardedGrads):
        grads.reduce(rank, group)  # on the current stream
        grads = grads.views
        if stream is not None:
            stream.wait_stream(torch.cuda.current_stream())
    if mats is None:
        idx = weights.plan.owned(rank)
        mats = [dm_matrix(weights.views[i], grads[i], momenta[i],
                          row_energy[i] if conditioned else None,
                          col_energy[i] if conditioned else None,
                          update_out.get(i) if update_out else None) for i in idx]
    if mats is not None and len(mats):
        fn = dm_dimuon_step if conditioned else dm_muon_step
        check(fn(mats, hp, workspace, stream=stream))
    if stream is not None:
        torch.cuda.current_stream().wait_stream(stream)
    weights.gather(rank, group)


def workspace_bytes(weights: ShardedWeights, rank: int, grads, momenta, hp, conditioned=False,
                    row_energy=None, col_energy=None) -> int:
    """Workspace the owned set of `rank` needs (host-only query)."""
    from . import dm_matrix, dm_workspace_size
    idx = weights.plan.owned(rank)
    if not idx:
        return 1
    mats = [dm_matrix(weights.views[i], grads[i], momenta[i],
                      row_energy[i] if conditioned else None,
                      col_energy[i] if conditioned else None) for i in idx]
    return dm_workspace_size(mats, hp, int(conditioned))
