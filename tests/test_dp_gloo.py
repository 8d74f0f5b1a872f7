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
