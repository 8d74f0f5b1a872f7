"""Data-parallel host logic on CPU with two gloo ranks.

Two ranks each compute the fp64 oracle gradients of half a batch; the
helpers bench.py uses for N GPUs (gradient averaging, max over ranks, per-rank
seeds) must turn them into exactly the full-batch gradients.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import synthetic as syn
    from gpt_pretraining_step_b200 import dp
    from oracle import model as om

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    s = syn.make_shape(depth=1, d_model=128, vocab=64, batch=2 * world, seq_len=8)
    params = syn.init_params(s, seed=0, std=0.05)
    tok, tgt = syn.tokens(s, seed=1), syn.targets(s, seed=2)
    rows = slice(2 * rank, 2 * rank + 2)           # each rank: its own 2 sequences
    _, grads, _ = om.fwd_bwd(params, tok[rows], tgt[rows], s.depth)
    names = [n for n, *_ in syn.param_specs(s)]
    flat = torch.tensor(np.concatenate([grads[n].ravel() for n in names]))
    dp.average_gradients(flat)
    slowest = dp.max_over_ranks(1.0 + rank)
    np.save(os.path.join(outdir, f"rank{rank}.npy"), flat.numpy())
    np.save(os.path.join(outdir, f"max{rank}.npy"), np.array([slowest]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_average_equals_full_batch(tmp_path):
    import sys
    sys.path.insert(0, ROOT)
    import synthetic as syn
    from oracle import model as om

    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    s = syn.make_shape(depth=1, d_model=128, vocab=64, batch=2 * world, seq_len=8)
    params = syn.init_params(s, seed=0, std=0.05)
    _, grads, _ = om.fwd_bwd(params, syn.tokens(s, seed=1), syn.targets(s, seed=2), s.depth)
    names = [n for n, *_ in syn.param_specs(s)]
    full = np.concatenate([grads[n].ravel() for n in names])
    for r in range(world):
        avg = np.load(tmp_path / f"rank{r}.npy")
        assert np.allclose(avg, full, rtol=1e-10, atol=1e-14)
        assert float(np.load(tmp_path / f"max{r}.npy")[0]) == float(world)


def test_rank_seeds_distinct_and_stable():
    import sys
    sys.path.insert(0, ROOT)
    from gpt_pretraining_step_b200 import dp
    seeds = [dp.rank_seed(1, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds == [dp.rank_seed(1, r) for r in range(8)]


def test_single_process_helpers_are_identity():
    import sys
    sys.path.insert(0, ROOT)
    from gpt_pretraining_step_b200 import dp
    t = torch.arange(5, dtype=torch.float32)
    assert torch.equal(dp.average_gradients(t.clone()), t)
    assert dp.max_over_ranks(3.5) == 3.5


# --- sharded optimizer (three-phase, layer ranges per rank) ---------------------

D_FAKE, L_FAKE, V_FAKE = 8, 4, 16


def _fake_shapes():
    d = D_FAKE
    return [(d, 3 * d), (d, d), (d, 4 * d), (4 * d, d)]


class _FakeStep:
    """Host stand-in for GPTStep with the same optimizer-side interface; the
    update of each matrix is the fp64 oracle's."""

    def __init__(self, seed):
        from oracle import optim as oo
        self.oo = oo
        rng = np.random.default_rng(seed)
        d = D_FAKE
        self.shapes = _fake_shapes()
        self.master = [torch.tensor(rng.standard_normal((L_FAKE, r, c)) * 0.02, dtype=torch.float32)
                       for r, c in self.shapes]
        self.bf16 = [m.to(torch.bfloat16) for m in self.master]
        self.mom = [torch.zeros_like(m) for m in self.master]
        self.emb = torch.tensor(rng.standard_normal((V_FAKE + d, d)) * 0.02, dtype=torch.float32)
        self.m = torch.zeros_like(self.emb)
        self.v = torch.zeros_like(self.emb)
        self.t = 0
        n_emb = self.emb.numel()
        self.grad = torch.zeros(n_emb + sum(L_FAKE * r * c for r, c in self.shapes), dtype=torch.float32)
        self.offs = []
        o = n_emb
        for r, c in self.shapes:
            self.offs.append(o)
            o += L_FAKE * r * c
        self.n_emb = n_emb

    def set_grads(self, seed):
        self.grad.copy_(torch.tensor(np.random.default_rng(seed).standard_normal(self.grad.numel()),
                                     dtype=torch.float32))

    def block_region(self, what, kind, l0, l1):
        r, c = self.shapes[kind]
        if what == 2:
            return self.grad[self.offs[kind] + l0 * r * c:self.offs[kind] + l1 * r * c]
        t = self.master[kind] if what == 0 else self.bf16[kind]
        return t.view(-1)[l0 * r * c:l1 * r * c]

    def adamw_grad_view(self):
        return self.grad[:self.n_emb]

    def muon_step_layers(self, l0, l1, lr, momentum, wd, normuon_beta2):
        for kind, (r, c) in enumerate(self.shapes):
            g = self.block_region(2, kind, 0, L_FAKE).view(L_FAKE, r, c)
            for l in range(l0, l1):
                W, M = self.oo.muon_step(self.master[kind][l].double().numpy(), g[l].double().numpy(),
                                         self.mom[kind][l].double().numpy(), lr, momentum, wd)
                self.master[kind][l] = torch.tensor(W, dtype=torch.float32)
                self.mom[kind][l] = torch.tensor(M, dtype=torch.float32)
                self.bf16[kind][l] = self.master[kind][l].to(torch.bfloat16)

    def adamw_step(self, lr, beta1, beta2, eps, wd):
        self.t += 1
        p, m, v = self.oo.adamw_step(self.emb.double().numpy(), self.adamw_grad_view().view_as(self.emb).double().numpy(),
                                     self.m.double().numpy(), self.v.double().numpy(), self.t, lr, beta1, beta2, eps, wd)
        self.emb = torch.tensor(p, dtype=torch.float32)
        self.m = torch.tensor(m, dtype=torch.float32)
        self.v = torch.tensor(v, dtype=torch.float32)


def _shard_worker(rank, world, port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from gpt_pretraining_step_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    st = _FakeStep(seed=5)                      # identical parameters on every rank
    for step in range(2):
        st.set_grads(seed=100 * step + rank)    # each rank: its own batch's gradients
        dp.sharded_optimizer_step(st, L_FAKE, muon=(0.02, 0.95, 0.01), adam=(3e-3, 0.8, 0.95, 1e-10, 0.0),
                                  sync_masters=(step == 1))
    out = {f"bf16_{k}": st.bf16[k].float().numpy() for k in range(4)}
    out.update({f"master_{k}": st.master[k].numpy() for k in range(4)})
    out["emb"] = st.emb.numpy()
    np.savez(os.path.join(outdir, f"shard{rank}.npz"), **out)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_sharded_optimizer_equals_replicated(tmp_path):
    """Three ranks over four layers (uneven shards): after two sharded steps
    every rank holds the parameters one replicated step sequence on the mean
    gradients gives (bf16 copies identical on every rank)."""
    import sys
    sys.path.insert(0, ROOT)
    world = 3
    mp.start_processes(_shard_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    ref = _FakeStep(seed=5)
    for step in range(2):
        gs = []
        for r in range(world):
            ref.set_grads(seed=100 * step + r)
            gs.append(ref.grad.clone())
        ref.grad.copy_(sum(gs) / world)
        ref.muon_step_layers(0, L_FAKE, 0.02, 0.95, 0.01, -1.0)
        ref.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.0)
    res = [np.load(tmp_path / f"shard{r}.npz") for r in range(world)]
    for k in range(4):
        for r in range(world):
            assert np.array_equal(res[r][f"bf16_{k}"], res[0][f"bf16_{k}"]), (k, r)
            # masters were broadcast by their owners on the last step
            assert np.allclose(res[r][f"master_{k}"], ref.master[k].numpy(), rtol=1e-5, atol=1e-7), (k, r)
        assert np.allclose(res[0][f"bf16_{k}"], ref.bf16[k].float().numpy(), rtol=1e-2, atol=1e-6), k
    for r in range(world):
        assert np.allclose(res[r]["emb"], ref.emb.numpy(), rtol=1e-6, atol=1e-9)


def test_layer_shards_cover_and_balance():
    import sys
    sys.path.insert(0, ROOT)
    from gpt_pretraining_step_b200 import dp
    for n_layer in (1, 4, 20, 26):
        for world in (1, 2, 3, 8):
            sh = dp.layer_shards(n_layer, world)
            assert len(sh) == world and sh[0][0] == 0 and sh[-1][1] == n_layer
            assert all(a <= b for a, b in sh) and all(sh[i][1] == sh[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in sh]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


# --- overlapped exchange, AdamW sharded by rows ------------------------------------

V2, D2, L2 = 24, 8, 4   # vocab 24, width 8: row-shardable over 2 and 3 ranks


class _FakeStep2:
    """Host stand-in for GPTStep with the library's gradient layout (lm_head,
    embedding, blocks) and its sharding interface; every update is the fp64
    oracle's."""

    def __init__(self, seed, vocab=V2, d=D2):
        from oracle import optim as oo
        self.oo = oo
        rng = np.random.default_rng(seed)
        self.V, self.d = vocab, d
        self.shapes = [(d, 3 * d), (d, d), (d, 4 * d), (4 * d, d)]
        self.w = {0: torch.tensor(rng.standard_normal((vocab, d)) * 0.02, dtype=torch.float32),
                  1: torch.tensor(rng.standard_normal((d, vocab)) * 0.02, dtype=torch.float32)}
        self.wb = {k: v.to(torch.bfloat16) for k, v in self.w.items()}
        self.m = {k: torch.zeros_like(v) for k, v in self.w.items()}
        self.v = {k: torch.zeros_like(v) for k, v in self.w.items()}
        self.master = [torch.tensor(rng.standard_normal((L2, r, c)) * 0.02, dtype=torch.float32)
                       for r, c in self.shapes]
        self.bf16 = [mm.to(torch.bfloat16) for mm in self.master]
        self.mom = [torch.zeros_like(mm) for mm in self.master]
        self.t = 0
        n_lm, n_emb = d * vocab, vocab * d
        self.off = {1: 0, 0: n_lm}
        o = n_lm + n_emb
        self.boff = []
        for r, c in self.shapes:
            self.boff.append(o)
            o += L2 * r * c
        self.grad = torch.zeros(o, dtype=torch.float32)

    # the step's gradients come from the "batch" (a seed)
    def fwd_bwd(self, tok, tgt):
        self.grad.copy_(torch.tensor(np.random.default_rng(int(tok)).standard_normal(self.grad.numel()),
                                     dtype=torch.float32))
        return 0.0

    def set_grad_events(self, events):
        pass

    def grad_bucket(self, i):
        if i == 0:
            return self.grad[:self.d * self.V]
        if i == 5:
            return self.grad[self.off[0]:self.boff[0]]
        return self.block_region(2, i - 1, 0, L2)

    def tensor_region(self, what, tid, r0, r1):
        rows, cols = self.w[tid].shape
        if what == 2:
            return self.grad[self.off[tid] + r0 * cols:self.off[tid] + r1 * cols]
        t = self.w[tid] if what == 0 else self.wb[tid]
        return t.view(-1)[r0 * cols:r1 * cols]

    def block_region(self, what, kind, l0, l1):
        r, c = self.shapes[kind]
        if what == 2:
            return self.grad[self.boff[kind] + l0 * r * c:self.boff[kind] + l1 * r * c]
        t = self.master[kind] if what == 0 else self.bf16[kind]
        return t.view(-1)[l0 * r * c:l1 * r * c]

    def muon_step_layers(self, l0, l1, lr, momentum, wd, normuon_beta2):
        for kind, (r, c) in enumerate(self.shapes):
            g = self.block_region(2, kind, 0, L2).view(L2, r, c)
            for l in range(l0, l1):
                W, M = self.oo.muon_step(self.master[kind][l].double().numpy(), g[l].double().numpy(),
                                         self.mom[kind][l].double().numpy(), lr, momentum, wd)
                self.master[kind][l] = torch.tensor(W, dtype=torch.float32)
                self.mom[kind][l] = torch.tensor(M, dtype=torch.float32)
                self.bf16[kind][l] = self.master[kind][l].to(torch.bfloat16)

    def _adam_rows(self, tid, r0, r1, lr, beta1, beta2, eps, wd):
        cols = self.w[tid].shape[1]
        g = self.tensor_region(2, tid, r0, r1).view(r1 - r0, cols)
        p, m, v = self.oo.adamw_step(self.w[tid][r0:r1].double().numpy(), g.double().numpy(),
                                     self.m[tid][r0:r1].double().numpy(), self.v[tid][r0:r1].double().numpy(),
                                     self.t, lr, beta1, beta2, eps, wd)
        self.w[tid][r0:r1] = torch.tensor(p, dtype=torch.float32)
        self.m[tid][r0:r1] = torch.tensor(m, dtype=torch.float32)
        self.v[tid][r0:r1] = torch.tensor(v, dtype=torch.float32)
        self.wb[tid][r0:r1] = self.w[tid][r0:r1].to(torch.bfloat16)

    def adamw_step_shard(self, part, nparts, lr, beta1, beta2, eps, wd):
        self.t += 1
        for tid in (0, 1):
            rows = self.w[tid].shape[0]
            self._adam_rows(tid, rows * part // nparts, rows * (part + 1) // nparts, lr, beta1, beta2, eps, wd)

    def adamw_step(self, lr, beta1, beta2, eps, wd):
        self.t += 1
        for tid in (0, 1):
            self._adam_rows(tid, 0, self.w[tid].shape[0], lr, beta1, beta2, eps, wd)


def _exchange_worker(rank, world, port, outdir, vocab, d):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from gpt_pretraining_step_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    st = _FakeStep2(seed=5, vocab=vocab, d=d)   # identical parameters on every rank
    ex = dp.ShardedExchange(st, L2, vocab, d, use_cuda=False)
    for step in range(2):
        ex.step(100 * step + rank, None, muon=(0.02, 0.95, 0.01), adam=(3e-3, 0.8, 0.95, 1e-10, 0.01),
                sync_masters=(step == 1))
    out = {f"bf16_{k}": st.bf16[k].float().numpy() for k in range(4)}
    out.update({f"master_{k}": st.master[k].numpy() for k in range(4)})
    out.update({f"w{t}": st.w[t].numpy() for t in (0, 1)})
    out.update({f"wb{t}": st.wb[t].float().numpy() for t in (0, 1)})
    out["sharded"] = np.array([ex.shard_adam])
    np.savez(os.path.join(outdir, f"ex{rank}.npz"), **out)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,vocab,d", [(2, V2, D2), (3, V2, 12), (3, 20, D2)])
def test_overlapped_exchange_equals_replicated(tmp_path, world, vocab, d):
    """Two steps of the bucketed exchange (AdamW rows reduce-scattered and
    all-gathered when the rows split evenly, all-reduced otherwise; Muon by
    layer ranges) give every rank the parameters the replicated optimizer
    gives on the mean gradients."""
    import sys
    sys.path.insert(0, ROOT)
    mp.start_processes(_exchange_worker, args=(world, _free_port(), str(tmp_path), vocab, d), nprocs=world,
                       join=True, start_method="spawn")
    ref = _FakeStep2(seed=5, vocab=vocab, d=d)
    for step in range(2):
        gs = []
        for r in range(world):
            ref.fwd_bwd(100 * step + r, None)
            gs.append(ref.grad.clone())
        ref.grad.copy_(sum(gs) / world)
        ref.muon_step_layers(0, L2, 0.02, 0.95, 0.01, -1.0)
        ref.adamw_step(3e-3, 0.8, 0.95, 1e-10, 0.01)
    res = [np.load(tmp_path / f"ex{r}.npz") for r in range(world)]
    assert bool(res[0]["sharded"][0]) == (vocab % world == 0 and d % world == 0)
    for r in range(world):
        for k in range(4):
            assert np.array_equal(res[r][f"bf16_{k}"], res[0][f"bf16_{k}"]), (k, r)
            assert np.allclose(res[r][f"master_{k}"], ref.master[k].numpy(), rtol=1e-5, atol=1e-7), (k, r)
        for t in (0, 1):
            assert np.array_equal(res[r][f"wb{t}"], res[0][f"wb{t}"]), (t, r)
            assert np.allclose(res[r][f"w{t}"], ref.w[t].numpy(), rtol=1e-6, atol=1e-9), (t, r)
            assert np.allclose(res[r][f"wb{t}"], ref.wb[t].float().numpy(), rtol=1e-2, atol=1e-6), (t, r)


def _leave_worker(rank, world, port, store_port, outdir):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from gpt_pretraining_step_b200 import dp

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    store = dist.TCPStore("127.0.0.1", store_port, world, rank == 0, timeout=datetime.timedelta(seconds=30))
    st = _FakeStep2(seed=5)
    ex = dp.ShardedExchange(st, L2, V2, D2, use_cuda=False)
    result = "done"
    for step in range(2):
        if rank == world - 1 and step == 1:
            result = "left"
            break                                  # this rank leaves between steps
        try:
            dp.join_step(store, step, rank, world, timeout_s=2.0)
        except dp.RankLeft as e:
            result = f"rank-left:{e.step}:{e.missing}"
            break
        ex.step(100 * step + rank, None)
    with open(os.path.join(outdir, f"leave{rank}.txt"), "w") as f:
        f.write(result)
    if rank == 0:
        # the store's server lives in rank 0: keep it up until the others wrote their result
        for r in range(1, world):
            store.wait([f"done/{r}"], datetime.timedelta(seconds=30))
    else:
        store.set(f"done/{rank}", "1")


@pytest.mark.timeout(300)
def test_rank_leaving_between_steps_is_found_on_the_host(tmp_path):
    """Three ranks; the last leaves after the first step.  The others learn it
    on the host, before they issue any collective of the second step, and
    raise RankLeft naming it (no collective is left waiting)."""
    import sys
    sys.path.insert(0, ROOT)
    world = 3
    mp.start_processes(_leave_worker, args=(world, _free_port(), _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = [open(tmp_path / f"leave{r}.txt").read() for r in range(world)]
    assert got[world - 1] == "left"
    for r in range(world - 1):
        assert got[r] == f"rank-left:1:[{world - 1}]", got
