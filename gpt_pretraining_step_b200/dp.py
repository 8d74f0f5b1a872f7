"""Data-parallel plumbing around the step library (host side only).

Each rank trains on its own batch; the mean-loss gradients of the ranks are
averaged (one all-reduce of the contiguous fp32 gradient span) before the
optimizer runs replicated on every rank, so N ranks with B rows each compute
the same update as one rank with N*B rows.  "¿Cómo Entrenar Tu Propio ChatGPT
por $50?" (frequently asked questions) states that single-GPU and 8-GPU runs
give almost identical results; this is the exact form of that equivalence.

Sharded optimizer ("¿Cómo Entrenar Tu Propio ChatGPT por $50?", section
"Entrenamiento distribuido": ZeRO-2 style sharding in three asynchronous
phases).  Rank r owns a contiguous range of layers (every block matrix kind
of those layers).  Phase 1 starts, for every owner, a reduce of its layers'
gradients to it, and an all-reduce of the embedding and lm_head gradients
(AdamW stays replicated: it is 0.5 ms of a d20 step); phase 2 waits, runs
Muon on the rank's own layers and AdamW, and starts the broadcasts of every
owner's new bf16 working copies; phase 3 waits for them.  Each matrix's
update depends only on its own gradient and state, so the result is the
replicated one, while each rank orthogonalises only its share of the
matrices.  The fp32 masters, momenta and NorMuon state of a layer stay
current only on its owner (the others never read them while sharding is
on); `sync_masters` also broadcasts the masters, e.g. before a checkpoint.
"""
from __future__ import annotations


def average_gradients(flat, group=None):
    """In-place mean over ranks of a gradient tensor (SUM then divide: every backend)."""
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return flat
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    flat.div_(dist.get_world_size(group))
    return flat


def max_over_ranks(value: float, device="cpu", group=None) -> float:
    """The slowest rank's value (step times are reported as the max over ranks)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct per rank, stable across runs."""
    return base + 100 * rank


def layer_shards(n_layer: int, world: int):
    """Contiguous layer ranges [(l0, l1)] of the ranks: sizes differ by at
    most one, the larger ranges first, every layer in exactly one range."""
    base, extra = divmod(n_layer, world)
    out, start = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((start, start + n))
        start += n
    return out


BLOCK_KINDS = 4   # fused q|k|v, attention output, MLP up, MLP down
REGION_MASTER, REGION_BF16, REGION_GRAD = 0, 1, 2


def sharded_optimizer_step(st, n_layer, muon=(0.02, 0.95, 0.0), adam=(3e-3, 0.8, 0.95, 1e-10, 0.0),
                           normuon_beta2=-1.0, group=None, sync_masters=False):
    """One optimizer step of a data-parallel rank, its Muon share only (see
    the module header).  st provides block_region(what, kind, l0, l1) and
    adamw_grad_view() (tensor views the collectives read and write in place),
    muon_step_layers(l0, l1, lr, momentum, wd, normuon_beta2) and
    adamw_step(lr, beta1, beta2, eps, wd).  Every rank issues the same
    collectives in the same order."""
    import torch.distributed as dist
    lr, momentum, wd = muon
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        st.muon_step_layers(0, n_layer, lr, momentum, wd, normuon_beta2)
        st.adamw_step(*adam)
        return
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    shards = layer_shards(n_layer, world)

    def glob(r):
        return dist.get_global_rank(group, r) if group is not None else r

    # phase 1: gradients of each owner's layers to the owner, AdamW gradients everywhere
    work = [dist.all_reduce(st.adamw_grad_view(), op=dist.ReduceOp.SUM, group=group, async_op=True)]
    for owner, (a, b) in enumerate(shards):
        if b <= a:
            continue
        for kind in range(BLOCK_KINDS):
            work.append(dist.reduce(st.block_region(REGION_GRAD, kind, a, b), dst=glob(owner),
                                    op=dist.ReduceOp.SUM, group=group, async_op=True))
    for w in work:
        w.wait()
    # phase 2: mean gradients, this rank's Muon share and the replicated AdamW,
    # then every owner's new working copies (and masters) to the others
    l0, l1 = shards[rank]
    st.adamw_grad_view().div_(world)
    if l1 > l0:
        for kind in range(BLOCK_KINDS):
            st.block_region(REGION_GRAD, kind, l0, l1).div_(world)
        st.muon_step_layers(l0, l1, lr, momentum, wd, normuon_beta2)
    st.adamw_step(*adam)
    work = []
    for owner, (a, b) in enumerate(shards):
        if b <= a:
            continue
        for kind in range(BLOCK_KINDS):
            work.append(dist.broadcast(st.block_region(REGION_BF16, kind, a, b), src=glob(owner), group=group,
                                       async_op=True))
            if sync_masters:
                work.append(dist.broadcast(st.block_region(REGION_MASTER, kind, a, b), src=glob(owner),
                                           group=group, async_op=True))
    # phase 3: the parameters are current everywhere once the broadcasts land
    for w in work:
        w.wait()
