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


# --- overlapped exchange with AdamW sharded by rows ------------------------------
#
# The same three phases, with the two refinements the pages' ZeRO-2 scheme has:
# the reduce of a gradient bucket starts as soon as the backward has completed
# that bucket (the library records a CUDA event per bucket; the collectives of
# the bucket wait for it on a communication stream, so they run while the rest
# of the backward does), and the AdamW state of the embedding and lm_head is
# split by rows (a reduce-scatter of their gradients, each rank's AdamW on its
# rows, an all-gather of the new bf16 rows).  Buckets, in the order the
# backward completes them: 0 lm_head, 1..4 the block matrix kinds over every
# layer, 5 the embedding and the extras.

EMBED_ID, LM_HEAD_ID = 0, 1


def adamw_rows_shardable(vocab: int, d_model: int, world: int) -> bool:
    """Equal row shares of the embedding [vocab, d] and lm_head [d, vocab]
    (what reduce-scatter and all-gather of equal chunks need)."""
    return vocab % world == 0 and d_model % world == 0


class ShardedExchange:
    """One data-parallel rank's optimizer step with the exchange overlapped
    with the backward.

    st: a GPTStep (or any object with the same methods): grad_bucket(i),
    tensor_region(what, id, r0, r1), block_region(what, kind, l0, l1),
    set_grad_events(events), fwd_bwd(tok, tgt), muon_step_layers(...),
    adamw_step_shard(part, nparts, ...), adamw_step(...).
    On GPUs the bucket collectives are issued from a side stream that waits on
    each bucket's event; without CUDA (gloo tests) they run after fwd_bwd.
    Every rank issues the same collectives in the same order.
    """

    def __init__(self, st, n_layer, vocab, d_model, group=None, use_cuda=None):
        import torch
        import torch.distributed as dist
        self.st, self.n_layer, self.vocab, self.d = st, n_layer, vocab, d_model
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.shards = layer_shards(n_layer, self.world)
        self.shard_adam = adamw_rows_shardable(vocab, d_model, self.world)
        self.cuda = torch.cuda.is_available() if use_cuda is None else use_cuda
        self.events = None
        self.comm = None
        if self.cuda:
            self.comm = torch.cuda.Stream()
            self.events = [torch.cuda.Event() for _ in range(6)]
            st.set_grad_events(self.events)

    def _glob(self, r):
        import torch.distributed as dist
        return dist.get_global_rank(self.group, r) if self.group is not None else r

    def _rows(self, n_rows):
        return n_rows * self.rank // self.world, n_rows * (self.rank + 1) // self.world

    def _reduce_scatter_rows(self, tid, n_rows, work):
        """Sum of tensor tid's gradient over the ranks, into this rank's rows."""
        import torch.distributed as dist
        full = self.st.tensor_region(REGION_GRAD, tid, 0, n_rows)
        r0, r1 = self._rows(n_rows)
        mine = self.st.tensor_region(REGION_GRAD, tid, r0, r1)
        out = mine.clone()
        work.append((dist.reduce_scatter_tensor(out, full, op=dist.ReduceOp.SUM, group=self.group,
                                                async_op=True), out, mine))

    def _bucket_collectives(self, i, work):
        import torch.distributed as dist
        st = self.st
        if i == 0:
            if self.shard_adam:
                self._reduce_scatter_rows(LM_HEAD_ID, self.d, work)
            else:
                work.append((dist.all_reduce(st.grad_bucket(0), group=self.group, async_op=True), None, None))
        elif 1 <= i <= 4:
            for owner, (a, b) in enumerate(self.shards):
                if b > a:
                    work.append((dist.reduce(st.block_region(REGION_GRAD, i - 1, a, b), dst=self._glob(owner),
                                             op=dist.ReduceOp.SUM, group=self.group, async_op=True), None, None))
        else:
            bucket = st.grad_bucket(5)
            if self.shard_adam:
                self._reduce_scatter_rows(EMBED_ID, self.vocab, work)
                n_emb = self.vocab * self.d
                if bucket.numel() > n_emb:   # the extras' gradients, replicated
                    work.append((dist.all_reduce(bucket[n_emb:], group=self.group, async_op=True), None, None))
            else:
                work.append((dist.all_reduce(bucket, group=self.group, async_op=True), None, None))

    def step(self, tok, tgt, muon=(0.02, 0.95, 0.0), adam=(3e-3, 0.8, 0.95, 1e-10, 0.0), normuon_beta2=-1.0,
             sync_masters=False):
        """fwd_bwd, then the three phases; returns fwd_bwd's loss."""
        import torch
        import torch.distributed as dist
        st, world = self.st, self.world
        loss = st.fwd_bwd(tok, tgt)
        # phase 1: each bucket's reduce as soon as the backward has completed it
        work = []
        if self.cuda:
            with torch.cuda.stream(self.comm):
                for i in range(6):
                    self.comm.wait_event(self.events[i])
                    self._bucket_collectives(i, work)
        else:
            for i in range(6):
                self._bucket_collectives(i, work)
        for w, out, mine in work:
            w.wait()
            if out is not None:
                mine.copy_(out)
        # phase 2: mean gradients of this rank's share, its Muon layers and AdamW rows
        l0, l1 = self.shards[self.rank]
        lr, momentum, wd = muon
        if self.shard_adam:
            for tid, n_rows in ((EMBED_ID, self.vocab), (LM_HEAD_ID, self.d)):
                st.tensor_region(REGION_GRAD, tid, *self._rows(n_rows)).div_(world)
            n_emb = self.vocab * self.d
            extras = st.grad_bucket(5)[n_emb:]
            if extras.numel():
                extras.div_(world)
        else:
            st.grad_bucket(0).div_(world)
            st.grad_bucket(5).div_(world)
        if l1 > l0:
            for kind in range(BLOCK_KINDS):
                st.block_region(REGION_GRAD, kind, l0, l1).div_(world)
            st.muon_step_layers(l0, l1, lr, momentum, wd, normuon_beta2)
        if self.shard_adam:
            st.adamw_step_shard(self.rank, world, *adam)
        else:
            st.adamw_step(*adam)
        # phase 3: every owner's new bf16 rows and matrices to the others
        work = []
        if self.shard_adam:
            for tid, n_rows in ((EMBED_ID, self.vocab), (LM_HEAD_ID, self.d)):
                whats = (REGION_BF16, REGION_MASTER) if sync_masters else (REGION_BF16,)
                for what in whats:
                    full = st.tensor_region(what, tid, 0, n_rows)
                    mine = st.tensor_region(what, tid, *self._rows(n_rows)).clone()
                    work.append(dist.all_gather_into_tensor(full, mine, group=self.group, async_op=True))
        for owner, (a, b) in enumerate(self.shards):
            if b <= a:
                continue
            for kind in range(BLOCK_KINDS):
                work.append(dist.broadcast(st.block_region(REGION_BF16, kind, a, b), src=self._glob(owner),
                                           group=self.group, async_op=True))
                if sync_masters:
                    work.append(dist.broadcast(st.block_region(REGION_MASTER, kind, a, b), src=self._glob(owner),
                                               group=self.group, async_op=True))
        for w in work:
            w.wait()
        return loss


# --- ranks that leave between steps -----------------------------------------------

class RankLeft(RuntimeError):
    """Raised on the ranks that remain when another rank did not join a step."""

    def __init__(self, step, missing):
        super().__init__(f"rank(s) {missing} did not join step {step}")
        self.step, self.missing = step, missing


def join_step(store, step: int, rank: int, world: int, timeout_s: float = 5.0):
    """Host-side check before a step's first launch: every rank announces it
    in the key-value store and waits (up to timeout_s) for the others.  A rank
    that has left (exited between steps, or never returns) is found here, on
    the host, before any kernel or collective of the step is issued: the
    remaining ranks get RankLeft naming it, instead of a collective that never
    completes."""
    import datetime
    store.set(f"join/{step}/{rank}", "1")
    keys = [f"join/{step}/{r}" for r in range(world)]
    try:
        store.wait(keys, datetime.timedelta(seconds=timeout_s))
    except Exception:
        missing = [r for r in range(world) if not store.check([keys[r]])]
        if not missing:
            return
        raise RankLeft(step, missing) from None
