"""The multi-rank host path of bench.py on CPU: two gloo ranks (no GPU).

Each rank decodes its own disjoint slice of the seeded batch (weak scaling, no collective on
the data path); the job time is the slowest rank's.  Here every rank runs the CPU oracle on
its slice of a tiny workload; the gathered per-sequence replay scores must equal a single
process replaying the whole batch, and the timing reduction must return the maximum.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, B: int, T: int, out_dir: str):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from bench import max_over_ranks, rank_sequences
    from oracle import RLTOracle
    from workloads import TINY, make_tokens, make_weights

    wl = TINY.with_batch(B, T)
    seqs = rank_sequences(rank, B)
    tok = make_tokens(wl, seqs)
    score, _, _, _ = RLTOracle(wl.model, make_weights(wl.model)).replay(tok, 4, 1.0)
    gathered = [torch.zeros(B, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(gathered, torch.from_numpy(score))
    slowest = max_over_ranks(10.0 * (rank + 1))
    if rank == 0:
        np.save(os.path.join(out_dir, "scores.npy"), torch.cat(gathered).numpy())
        np.save(os.path.join(out_dir, "slowest.npy"), np.array([slowest]))
        np.save(os.path.join(out_dir, "seqs.npy"), np.array([list(rank_sequences(r, B)) for r in range(world)]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_sequences_and_take_the_slowest_time(tmp_path):
    from oracle import RLTOracle
    from workloads import TINY, make_tokens, make_weights

    world, B, T = 2, 2, 10
    mp.spawn(_rank_main, args=(world, _free_port(), B, T, str(tmp_path)), nprocs=world, join=True)
    seqs = np.load(tmp_path / "seqs.npy")
    assert sorted(seqs.ravel().tolist()) == list(range(world * B))          # disjoint, covering
    wl = TINY.with_batch(world * B, T)
    full = RLTOracle(wl.model, make_weights(wl.model)).replay(make_tokens(wl), 4, 1.0)[0]
    np.testing.assert_allclose(np.load(tmp_path / "scores.npy"), full, rtol=0, atol=1e-12)
    assert float(np.load(tmp_path / "slowest.npy")[0]) == 20.0
