"""Failure detection and recovery without a GPU fault.

* Bounded device waits: a tensor-core kernel whose producer issues nothing
  (zo_debug_cell_stall) must give up after its wait limit, report
  ZO_ERR_TIMEOUT through zo_sync_status and leave the context usable.
* Host-side fault injection (ZO_FAULT=alloc|launch): the allocation-failure
  and launch-failure returns of the C ABI, with nothing changed on the device.
* The probe-parallel step (probe slices, a gloo all-gather of the scalar
  losses, the same update on every rank) run as two processes on the one
  device: theta after two steps must equal the single-process step bit for
  bit.
* Checkpoint and resume of the training driver: a run interrupted after two
  steps and resumed from its checkpoint ends with the same theta as the
  uninterrupted run."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch

import workloads as W
import zero_order_recurrent_b200 as zo

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def library():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from zero_order_recurrent_b200 import build
    build.build()
    zo.load_library()


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bf16_setup():
    V, E, H, L, B, T, n = 50, 64, 64, 2, 256, 3, 2
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L, dtype="bf16")
    theta = dev(W.init_theta(cfg, seed=1))
    tok, tgt = W.markov_batch(B, T, step=0, vocab=V)
    return zo.Context(V, E, H, L, "bf16", B, T, n), theta, dev(tok), dev(tgt), n


def _losses(ctx, theta, tok, tgt, n):
    lp = torch.empty(n, device="cuda")
    lm = torch.empty(n, device="cuda")
    zo.zo_probe_losses(ctx, theta, 5, n, 1e-3, tok, tgt, lp, lm)
    return lp, lm


@pytest.mark.parametrize("kind", [0, 1], ids=["pair_cell_kernel", "single_cta_loss_kernel"])
def test_bounded_wait_runs_out_and_the_context_recovers(kind):
    ctx, theta, tok, tgt, n = _bf16_setup()
    with ctx:
        lp0, lm0 = _losses(ctx, theta, tok, tgt, n)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        zo.zo_debug_cell_stall(ctx, kind, 1_000_000)          # 1 ms per wait
        assert zo.zo_sync_status(ctx) == zo.ZO_ERR_TIMEOUT
        assert zo.zo_sync_status(ctx) == zo.ZO_OK              # the latch was cleared
        lp1, lm1 = _losses(ctx, theta, tok, tgt, n)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        assert torch.equal(lp0, lp1) and torch.equal(lm0, lm1)


def test_stall_hook_rejects_bad_arguments():
    ctx, *_ = _bf16_setup()
    with ctx:
        for kind, ns in ((2, 1_000_000), (0, 10), (1, 10**11)):
            with pytest.raises(zo.ZOError) as e:
                zo.zo_debug_cell_stall(ctx, kind, ns)
            assert e.value.status == zo.ZO_ERR_INVALID_ARG
    with zo.Context(10, 16, 32, 1, "f32", 8, 21, 0) as c32:
        with pytest.raises(zo.ZOError) as e:
            zo.zo_debug_cell_stall(c32, 0, 1_000_000)
        assert e.value.status == zo.ZO_ERR_UNSUPPORTED


def test_injected_allocation_failure(monkeypatch):
    free0 = torch.cuda.mem_get_info()[0]
    monkeypatch.setenv("ZO_FAULT", "alloc")
    for dtype in ("f32", "bf16"):
        with pytest.raises(zo.ZOError) as e:
            zo.Context(50, 64, 64, 2, dtype, 256, 3, 2)
        assert e.value.status == zo.ZO_ERR_OOM
    monkeypatch.delenv("ZO_FAULT")
    assert torch.cuda.mem_get_info()[0] >= free0 - (64 << 20)   # nothing kept
    ctx, theta, tok, tgt, n = _bf16_setup()
    with ctx:
        _losses(ctx, theta, tok, tgt, n)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK


def test_injected_launch_failure(monkeypatch):
    ctx, theta, tok, tgt, n = _bf16_setup()
    with ctx:
        lp0, lm0 = _losses(ctx, theta, tok, tgt, n)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        before = theta.clone()
        c = torch.zeros(n, device="cuda")
        monkeypatch.setenv("ZO_FAULT", "launch")
        launches = zo.zo_kernel_launches()
        for call in (lambda: _losses(ctx, theta, tok, tgt, n),
                     lambda: zo.zo_coeffs(ctx, lp0, lm0, n, 1e-3, 1e-3, c),
                     lambda: zo.zo_update(ctx, theta, 5, n, lp0)):
            with pytest.raises(zo.ZOError) as e:
                call()
            assert e.value.status == zo.ZO_ERR_CUDA
        hp = torch.empty(n).pin_memory()
        hm = torch.empty(n).pin_memory()
        with pytest.raises(zo.ZOError):
            zo.zo_step_host(ctx, theta, 5, n, 1e-3, 1e-3, tok.cpu(), tgt.cpu(), hp, hm)
        assert zo.zo_kernel_launches() == launches              # nothing was enqueued
        monkeypatch.delenv("ZO_FAULT")
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        assert torch.equal(theta, before)
        lp1, lm1 = _losses(ctx, theta, tok, tgt, n)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        assert torch.equal(lp0, lp1) and torch.equal(lm0, lm1)


# ---------------------------------------------------------------------------
# the probe-parallel step, two processes on the one device (gloo)
# ---------------------------------------------------------------------------
def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _shard_problem(name):
    if name == "tiny":
        cfg = W.CONFIGS["tiny"]
        tok, tgt = W.batch_for(cfg)
        return cfg, (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers, "f32", cfg.batch, cfg.seq, 0), \
            W.init_theta(cfg), tok, tgt, cfg.n_pert
    cfg = W.small_config(vocab=50, embed=64, hidden=64, layers=2, dtype="bf16")
    tok, tgt = W.markov_batch(256, 3, step=1, vocab=50)
    return cfg, (50, 64, 64, 2, "bf16", 256, 3, 3), W.init_theta(cfg, seed=2), tok, tgt, 7


def _shard_worker(rank, world, port, name, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    from datetime import timedelta

    import torch.distributed as dist

    import zero_order_recurrent_b200 as zo
    from zero_order_recurrent_b200.probe_parallel import cdrge_step_sharded
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        zo.load_library()
        cfg, ctx_args, theta, tok, tgt, n = _shard_problem(name)
        th = torch.from_numpy(theta).cuda()
        coef = torch.empty(n, device="cuda")
        with zo.Context(*ctx_args) as ctx:
            for step in range(2):
                cdrge_step_sharded(ctx, th, W.step_seed(step), n, 1e-3, 1e-3,
                                   torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda(), coef)
            torch.cuda.synchronize()
            assert zo.zo_sync_status(ctx) == zo.ZO_OK
        np.save(out.format(rank=rank), th.cpu().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["tiny", "bf16"])
def test_sharded_step_in_two_processes_matches_single_process(name):
    import torch.multiprocessing as mp
    cfg, ctx_args, theta, tok, tgt, n = _shard_problem(name)
    th = dev(theta)
    lp = torch.empty(n, device="cuda")
    lm = torch.empty(n, device="cuda")
    coef = torch.empty(n, device="cuda")
    with zo.Context(*ctx_args) as ctx:
        for step in range(2):
            zo.cdrge_step(ctx, th, W.step_seed(step), n, 1e-3, 1e-3, dev(tok), dev(tgt), lp, lm, coef)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
    want = th.cpu().numpy()
    with tempfile.TemporaryDirectory() as d:
        out = os.path.join(d, "theta_{rank}.npy")
        mp.spawn(_shard_worker, args=(2, _free_port(), name, out), nprocs=2, join=True)
        for r in range(2):
            assert np.array_equal(np.load(out.format(rank=r)), want), r


# ---------------------------------------------------------------------------
# checkpoint and resume
# ---------------------------------------------------------------------------
def test_resumed_training_run_repeats_the_uninterrupted_run():
    from zero_order_recurrent_b200 import checkpoint as ckpt
    from zero_order_recurrent_b200.train import train
    kw = dict(task="copy", n_pert=16, eps=1e-3, eta=0.05, eval_lengths=(11,), log_every=1, seed=3)
    full = train(steps=4, **kw)["theta"].cpu().numpy()
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "run.npz")
        train(steps=2, checkpoint=path, **kw)
        th, step, run_seed, meta = ckpt.load(path)
        assert step == 2 and run_seed == 3 and meta["task"] == "copy"
        resumed = train(steps=4, theta=torch.from_numpy(th).cuda(), start_step=step, **kw)
    assert np.array_equal(resumed["theta"].cpu().numpy(), full)
    assert not np.array_equal(th, full)
