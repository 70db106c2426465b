"""Probe-parallel CD-RGE across processes (gloo, CPU): each rank evaluates its
probe slice (here with the fp64 oracle as the per-rank computation), the
scalar losses are all-gathered, and every rank applies the same update.  The
result must equal the single-process update exactly."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from zero_order_recurrent_b200.probe_parallel import gather_losses, probe_slice


@pytest.mark.parametrize("n,world", [(8, 2), (7, 2), (5, 3), (2, 4), (1, 2)])
def test_probe_slices_partition_the_probes(n, world):
    slices = [probe_slice(n, r, world) for r in range(world)]
    covered = [i for b, c in slices for i in range(b, b + c)]
    assert covered == list(range(n))
    counts = [c for _, c in slices]
    assert max(counts) - min(counts) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, n, out_path):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import oracle as O
    import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        cfg = W.CONFIGS["tiny"]
        spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
        theta = W.init_theta(cfg)
        tok, tgt = W.batch_for(cfg)
        seed = W.step_seed(3)
        begin, count = probe_slice(n, rank, world)
        lp_l, lm_l = O.probe_losses(theta, spec, seed, n, cfg.eps, tok, tgt,
                                    probes=range(begin, begin + count))
        lp, lm = gather_losses(torch.from_numpy(np.asarray(lp_l, dtype=np.float64)),
                               torch.from_numpy(np.asarray(lm_l, dtype=np.float64)), n)
        c = O.coefficients(lp.numpy(), lm.numpy(), n, cfg.eps, cfg.eta)
        new = O.update(theta, spec, seed, n, c)
        np.save(out_path.format(rank=rank), np.concatenate([lp.numpy(), lm.numpy(), new]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n,world", [(8, 2), (7, 2)])
def test_sharded_update_equals_single_process(tmp_path, n, world):
    out = str(tmp_path / "rank{rank}.npy")
    mp.start_processes(_worker, args=(world, _free_port(), n, out), nprocs=world, join=True,
                       start_method="spawn")
    import oracle as O
    import workloads as W
    cfg = W.CONFIGS["tiny"]
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg)
    seed = W.step_seed(3)
    lp, lm = O.probe_losses(theta, spec, seed, n, cfg.eps, tok, tgt)
    new = O.update(theta, spec, seed, n, O.coefficients(lp, lm, n, cfg.eps, cfg.eta))
    want = np.concatenate([lp, lm, new])
    results = [np.load(out.format(rank=r)) for r in range(world)]
    for r in results:
        assert np.array_equal(r, want)
