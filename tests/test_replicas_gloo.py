"""The N-GPU path's host logic, run as world_size-2 gloo ranks on CPU: each rank
solves its own problem (own seed, no data-path collective), the job time is the
slowest rank's, and the job throughput counts every rank's units.  The per-rank
problem here is a tiny HSA step computed by the oracle, so the test also checks that
a rank's result equals the same problem solved in a single process."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from linear_attention_paged_b200 import replicas, workloads as W

TINY = W.C0.with_(name="tiny", T_p=256, n_c=4, Nq=130, K_p=2, r=16)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _solve(rank):
    from oracle import hsa_oracle as O
    cfg = TINY.with_(seed=replicas.rank_seed(TINY.seed, rank))
    inp = W.make_inputs(cfg, device="cpu")
    return O.hsa_step(inp, cfg.B, cfg.K_p)["o"]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, lr = replicas.env_ranks()
    assert (r, w, lr) == (rank, world, rank)
    replicas.init(w, "gloo", timeout_s=60.0)
    try:
        out = _solve(r)
        replicas.barrier(w)
        # stand-in device times: rank 1 is the slower one
        mine = 10.0 + 5.0 * r
        slowest = replicas.max_over_ranks(mine, w)
        units = 3.0
        thr = replicas.job_throughput(units, w, slowest / 1000.0)
        np.save(os.path.join(out_dir, f"out{r}.npy"), out)
        np.save(os.path.join(out_dir, f"stats{r}.npy"), np.array([slowest, thr]))
    finally:
        replicas.shutdown(w)


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    outs = [np.load(tmp_path / f"out{r}.npy") for r in range(world)]
    stats = [np.load(tmp_path / f"stats{r}.npy") for r in range(world)]
    # every rank agrees on the slowest time and the job throughput
    for st in stats:
        assert st[0] == pytest.approx(15.0)
        assert st[1] == pytest.approx(world * 3.0 / 0.015)
    # independent problems: different seeds give different results ...
    assert not np.allclose(outs[0], outs[1])
    # ... and each rank's result is the single-process result of its problem
    for r in range(world):
        np.testing.assert_array_equal(outs[r], _solve(r))


def test_single_process_helpers():
    assert replicas.rank_seed(7, 0) == 7
    assert len({replicas.rank_seed(7, r) for r in range(8)}) == 8
    assert replicas.max_over_ranks(3.5, 1) == 3.5
    assert replicas.job_throughput(3.0, 4, 0.5) == pytest.approx(24.0)
    replicas.barrier(1)
    replicas.init(1, "gloo")      # no process group for one rank
    assert not torch.distributed.is_initialized()
