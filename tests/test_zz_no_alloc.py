"""zo_probe_losses_static: the entry point for callers that cannot call
cudaMalloc where they need the losses (a memory manager owns the whole device
heap, or the loop must not take cudaMalloc's implicit synchronisation).  It
runs the fp32 probe-loss path with its scratch in a fixed device array instead
of a context's workspace; its losses must equal those of zo_probe_losses.

This file is collected last so that a run stopping at the first failure has
already run every other test; it needs nothing from them."""
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


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _context_losses(cfg, theta, seed, tok, tgt):
    n = cfg.n_pert
    lp = torch.empty(n, device="cuda")
    lm = torch.empty(n, device="cuda")
    with zo.Context.for_config(cfg) as ctx:
        zo.zo_probe_losses(ctx, theta, seed, n, cfg.eps, _dev(tok), _dev(tgt), lp, lm)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
    return lp.cpu().numpy(), lm.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "overfit"])
def test_static_entry_matches_context_entry_on_two_calls(name):
    cfg = W.CONFIGS[name]
    theta = _dev(W.init_theta(cfg))
    tok, tgt = W.batch_for(cfg)
    spec = zo.ModelSpec(cfg.vocab, cfg.embed, cfg.hidden, cfg.layers, zo.ZO_DTYPE_FP32, 0, 0, 0)
    # two calls in a row with different probe seeds: the second must not see
    # anything the first left in the shared scratch
    for step in (0, 1):
        seed = W.step_seed(step)
        want_p, want_m = _context_losses(cfg, theta, seed, tok, tgt)
        lp = torch.full((cfg.n_pert,), float("nan"), device="cuda")
        lm = torch.full((cfg.n_pert,), float("nan"), device="cuda")
        st = zo.zo_probe_losses_static(spec, theta, seed, cfg.n_pert, cfg.eps, _dev(tok),
                                       _dev(tgt), lp, lm)
        assert st == zo.ZO_OK, zo.status_string(st)
        torch.cuda.synchronize()
        assert np.allclose(lp.cpu().numpy(), want_p, rtol=1e-5, atol=0)
        assert np.allclose(lm.cpu().numpy(), want_m, rtol=1e-5, atol=0)


def test_static_entry_rejects_requests_beyond_its_scratch():
    cfg = W.CONFIGS["tiny"]
    theta = _dev(W.init_theta(cfg))
    spec = zo.ModelSpec(cfg.vocab, cfg.embed, cfg.hidden, cfg.layers, zo.ZO_DTYPE_FP32, 0, 0, 0)
    B = 64
    n = zo.ZO_STATIC_SCRATCH_FLOATS // (2 * B) + 1
    tok, tgt = W.random_batch(B, 3, cfg.vocab, seed=1)
    lp = torch.empty(n, device="cuda")
    lm = torch.empty(n, device="cuda")
    st = zo.zo_probe_losses_static(spec, theta, 1, n, cfg.eps, _dev(tok), _dev(tgt), lp, lm)
    assert st == zo.ZO_ERR_INVALID_ARG
    bf16 = zo.ModelSpec(cfg.vocab, 64, 64, 1, zo.ZO_DTYPE_BF16, 0, 0, 0)
    st = zo.zo_probe_losses_static(bf16, theta, 1, 2, cfg.eps, _dev(tok), _dev(tgt), lp, lm)
    assert st == zo.ZO_ERR_INVALID_ARG
