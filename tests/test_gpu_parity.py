"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Tolerances: probe signs bit-exact; losses 1e-5 relative
(fp32 path) and 1e-2 relative (bf16 path); update 1e-6 relative to
|theta'| + sum|c|; sign(L+ - L-) agreement >= 95%; cos(g_gpu, g_oracle) >= 0.99."""
import math

import numpy as np
import pytest
import torch

import oracle as O
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


def spec_of(cfg):
    return (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)


def gpu_losses(ctx, theta, seed, n, eps, tok, tgt, rows=False):
    B = tok.shape[0]
    th = dev(theta)
    lp = torch.empty(n, device="cuda")
    lm = torch.empty(n, device="cuda")
    rl = torch.empty(n * 2 * B, device="cuda") if rows else None
    zo.zo_probe_losses(ctx, th, seed, n, eps, dev(tok), dev(tgt), lp, lm, row_loss=rl)
    assert zo.zo_sync_status(ctx) == zo.ZO_OK
    out = (lp.cpu().numpy().astype(np.float64), lm.cpu().numpy().astype(np.float64))
    if rows:
        out = out + (rl.cpu().numpy().reshape(n, 2, B).astype(np.float64),)
    return out


def sign_agreement(lp_a, lm_a, lp_b, lm_b):
    return float(np.mean(np.sign(np.asarray(lp_a) - lm_a) == np.sign(np.asarray(lp_b) - lm_b)))


def estimate_cosine(spec, seed, probes, lp_a, lm_a, lp_b, lm_b):
    G = O.probe_gram(spec, seed, probes)
    return O.gram_cosine(np.asarray(lp_a) - lm_a, np.asarray(lp_b) - lm_b, G)


# ---------------------------------------------------------------------------
# a1: probe signs
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [W.step_seed(0), 0, (1 << 64) - 1, 0x0123456789ABCDEF])
@pytest.mark.parametrize("probe,q0", [(0, 0), (1, 1000), (511, 12345), (65535, (1 << 32) - 3),
                                      ((1 << 31) - 1, 7)])
def test_sign_words_bit_exact(seed, probe, q0):
    n = 67
    out = torch.zeros(4 * n, dtype=torch.int32, device="cuda")
    zo.zo_sign_words(seed, probe, q0, n, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().view(np.uint32).reshape(n, 4)
    want = O.sign_words(seed, probe, q0, n)
    assert np.array_equal(got, want)


# ---------------------------------------------------------------------------
# a5 / a6: coefficients and update
# ---------------------------------------------------------------------------
def _check_update(cfg, n, theta, seed, coeffs, ctx, idx=None):
    th = dev(theta)
    c = dev(coeffs.astype(np.float32))
    zo.zo_update(ctx, th, seed, n, c)
    assert zo.zo_sync_status(ctx) == zo.ZO_OK
    got = th.cpu().numpy().astype(np.float64)
    c64 = coeffs.astype(np.float32).astype(np.float64)
    if idx is None:
        want = O.update(theta, spec_of(cfg), seed, n, c64)
        mask = O.real_mask(*spec_of(cfg))
        assert np.array_equal(got[~mask], theta[~mask])
    else:
        want = O.update_at(theta, seed, n, c64, idx)
        got = got[idx]
    err = np.abs(got - want)
    csum = np.abs(c64).sum()
    assert np.all(err <= 1e-6 * (np.abs(want) + csum))
    # where theta' outweighs the coefficient mass, the plain relative bound
    big = np.abs(want) >= csum
    if np.any(big):
        rel = float(np.max(err[big] / np.abs(want[big])))
        print(f"update n={n}: max relative error {rel:.3e} on {int(big.sum())} elements "
              f"with |theta'| >= sum|c|")
        assert rel <= 1e-6
    return th


# every probe-group count the update kernels compile (1 and 2 groups of four
# probes up to 8 probes, 16 groups per pass above 64; 2, 4 and 8 groups of
# eight for 9..64 probes), counts that leave a group partly empty, and
# several passes
@pytest.mark.parametrize("name,n", [("tiny", 8), ("tiny", 1), ("tiny", 3), ("overfit", 512),
                                    ("overfit", 37), ("overfit", 5), ("overfit", 9),
                                    ("overfit", 13),
                                    ("overfit", 16), ("overfit", 17), ("overfit", 29),
                                    ("overfit", 32), ("overfit", 33), ("overfit", 48),
                                    ("overfit", 64), ("overfit", 65), ("overfit", 100),
                                    ("tiny", 24), ("tiny", 57)])
def test_update_matches_oracle(name, n):
    cfg = W.CONFIGS[name]
    theta = W.init_theta(cfg)
    seed = W.step_seed(5)
    coeffs = np.random.default_rng(n).standard_normal(n) * 1e-3
    with zo.Context.for_config(cfg) as ctx:
        _check_update(cfg, n, theta, seed, coeffs, ctx)


@pytest.mark.parametrize("kind", ["tiny", "overfit", "bf16", "bf16_vocab"])
def test_unperturbed_loss_matches_oracle(kind):
    """zo_loss: the forward at radius 0 on every forward path (per-probe fp32,
    probe-column fp32, bf16 tensor cores, bf16 with the vocabulary table)."""
    if kind in ("tiny", "overfit"):
        cfg = W.CONFIGS[kind]
        theta = W.init_theta(cfg)
        tok, tgt = W.batch_for(cfg)
        ctx = zo.Context.for_config(cfg)
        rtol = 1e-5
    else:
        E = 64 if kind == "bf16" else 512
        cfg = W.small_config(vocab=50, embed=E, hidden=64, layers=2, dtype="bf16")
        theta = W.init_theta(cfg, seed=4)
        tok, tgt = W.random_batch(256, 3, 50, seed=6, ignore_frac=0.2)
        ctx = zo.Context(50, E, 64, 2, "bf16", 256, 3, 0)
        rtol = 1e-2
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    with ctx:
        out = torch.full((1,), float("nan"), device="cuda")
        zo.zo_loss(ctx, dev(theta), dev(tok), dev(tgt), out)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        got = float(out.cpu())
    assert math.isclose(got, O.loss_at(theta, spec, tok, tgt), rel_tol=rtol)


def test_forward_coefficients_match_formula():
    n = 257
    rng = np.random.default_rng(4)
    lp = (2.3 + 1e-3 * rng.standard_normal(n)).astype(np.float32)
    l0 = np.float32(2.3)
    with zo.Context(10, 16, 32, 1) as ctx:
        out = torch.empty(n, device="cuda")
        zo.zo_coeffs_forward(ctx, dev(lp), dev(np.array([l0])), n, 1e-3, 5e-2, out)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        want = O.coefficients_forward(lp, float(l0), n, 1e-3, 5e-2)
        assert np.allclose(out.cpu().numpy(), want, rtol=1e-6, atol=0)


def test_update_rejects_too_many_probes():
    cfg = W.CONFIGS["tiny"]
    n = zo.ZO_MAX_UPDATE_PROBES + 1
    th = dev(W.init_theta(cfg))
    c = torch.zeros(n, device="cuda")
    with zo.Context.for_config(cfg) as ctx:
        with pytest.raises(zo.ZOError) as e:
            zo.zo_update(ctx, th, 1, n, c)
        assert e.value.status == zo.ZO_ERR_INVALID_ARG
        assert torch.equal(th, dev(W.init_theta(cfg)))


@pytest.mark.parametrize("n", [64, 32, 21, 12])
def test_update_bf16_context_sampled_and_shadow(n):
    """charlm-size theta (many spans per warp): sampled indices against the
    oracle; the bf16 shadow the update writes equals a fresh cast of theta'
    (losses bit-identical)."""
    cfg = W.CONFIGS["charlm"]
    theta = W.init_theta(cfg)
    seed = W.step_seed(1)
    coeffs = np.random.default_rng(0).standard_normal(n) * 1e-4
    rng = np.random.default_rng(1)
    mask = O.real_mask(*spec_of(cfg))
    idx = np.sort(rng.choice(np.nonzero(mask)[0], 20000, replace=False))
    with zo.Context.for_config(cfg, max_batch=128, max_seq=2, chunk=2) as ctx:
        th = _check_update(cfg, n, theta, seed, coeffs, ctx, idx)
        tok, tgt = W.markov_batch(128, 2, step=3)
        lp1 = torch.empty(2, device="cuda")
        lm1 = torch.empty(2, device="cuda")
        zo.zo_probe_losses(ctx, th, seed, 2, cfg.eps, dev(tok), dev(tgt), lp1, lm1)
        zo.zo_invalidate_shadow(ctx)
        lp2 = torch.empty(2, device="cuda")
        lm2 = torch.empty(2, device="cuda")
        zo.zo_probe_losses(ctx, th, seed, 2, cfg.eps, dev(tok), dev(tgt), lp2, lm2)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        assert torch.equal(lp1, lp2) and torch.equal(lm1, lm2)


def test_coefficients_match_formula():
    n = 300
    rng = np.random.default_rng(2)
    lp = (2.3 + 1e-3 * rng.standard_normal(n)).astype(np.float32)
    lm = (2.3 + 1e-3 * rng.standard_normal(n)).astype(np.float32)
    with zo.Context(10, 16, 32, 1) as ctx:
        out = torch.empty(n, device="cuda")
        zo.zo_coeffs(ctx, dev(lp), dev(lm), n, 1e-3, 5e-4, out)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        want = O.coefficients(lp, lm, n, 1e-3, 5e-4)
        assert np.allclose(out.cpu().numpy(), want, rtol=1e-6, atol=0)


# ---------------------------------------------------------------------------
# a0-a4 on the fp32 path (tiny, overfit)
# ---------------------------------------------------------------------------
def test_fp32_tiny_full_step_matches_oracle():
    cfg = W.CONFIGS["tiny"]
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg)
    seed = W.step_seed(0)
    with zo.Context.for_config(cfg) as ctx:
        lp, lm = gpu_losses(ctx, theta, seed, cfg.n_pert, cfg.eps, tok, tgt)
    olp, olm = O.probe_losses(theta, spec_of(cfg), seed, cfg.n_pert, cfg.eps, tok, tgt)
    assert np.allclose(lp, olp, rtol=1e-5, atol=0)
    assert np.allclose(lm, olm, rtol=1e-5, atol=0)
    assert sign_agreement(lp, lm, olp, olm) >= 0.95
    assert estimate_cosine(spec_of(cfg), seed, range(cfg.n_pert), lp, lm, olp, olm) >= 0.99


def test_fp32_overfit_full_launch_sampled_probes():
    """overfit config as benchmarked (512 probes, T = 100); the oracle checks a
    sample of 24 probes spread over the range."""
    cfg = W.CONFIGS["overfit"]
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg)
    seed = W.step_seed(0)
    with zo.Context.for_config(cfg) as ctx:
        lp, lm = gpu_losses(ctx, theta, seed, cfg.n_pert, cfg.eps, tok, tgt)
    probes = list(range(0, 512, 23)) + [511]
    olp, olm = O.probe_losses(theta, spec_of(cfg), seed, cfg.n_pert, cfg.eps, tok, tgt, probes=probes)
    assert np.allclose(lp[probes], olp, rtol=1e-5, atol=0)
    assert np.allclose(lm[probes], olm, rtol=1e-5, atol=0)
    assert sign_agreement(lp[probes], lm[probes], olp, olm) >= 0.95
    assert estimate_cosine(spec_of(cfg), seed, probes, lp[probes], lm[probes], olp, olm) >= 0.99


@pytest.mark.parametrize("V,E,H,L,B,T,n,chunk,frac", [
    (7, 5, 6, 3, 5, 4, 3, 0, 0.3),      # three layers, odd widths
    (13, 8, 24, 2, 9, 3, 7, 3, 0.5),    # ragged row blocks, several chunks
    (11, 12, 40, 1, 1, 1, 1, 0, 0.0),   # T = 1, one probe
    (9, 4, 8, 2, 3, 5, 2, 0, 1.0),      # nothing scored: loss 0
    # widths that are multiples of 32 take the probe-column kernel (four
    # probes per CTA, rows across lanes):
    (50, 32, 32, 1, 3, 4, 6, 0, 0.3),   # inputs split over warps, a CTA with 2 of 4 probes
    (65, 64, 64, 2, 2, 3, 5, 2, 0.0),   # 65 logits (two row blocks), split inputs, chunks
    (40, 96, 96, 3, 1, 5, 9, 0, 0.5),   # three layers, 6 row blocks, 3 input words
])
def test_fp32_edge_cases(V, E, H, L, B, T, n, chunk, frac):
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L)
    theta = W.init_theta(cfg, seed=3)
    tok, tgt = W.random_batch(B, T, V, seed=4, ignore_frac=frac)
    seed = W.step_seed(2)
    with zo.Context(V, E, H, L, "f32", B, T, chunk) as ctx:
        lp, lm, rows = gpu_losses(ctx, theta, seed, n, 1e-3, tok, tgt, rows=True)
    olp, olm, orp, orm = O.probe_losses(theta, (V, E, H, L), seed, n, 1e-3, tok, tgt, return_rows=True)
    assert np.allclose(lp, olp, rtol=1e-5, atol=1e-7)
    assert np.allclose(lm, olm, rtol=1e-5, atol=1e-7)
    assert np.allclose(rows[:, 0], orp, rtol=1e-5, atol=1e-6)
    assert np.allclose(rows[:, 1], orm, rtol=1e-5, atol=1e-6)


def test_deterministic_repeat():
    cfg = W.CONFIGS["tiny"]
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg)
    with zo.Context.for_config(cfg) as ctx:
        a = gpu_losses(ctx, theta, 7, 8, cfg.eps, tok, tgt)
        b = gpu_losses(ctx, theta, 7, 8, cfg.eps, tok, tgt)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ---------------------------------------------------------------------------
# error reporting
# ---------------------------------------------------------------------------
def test_token_out_of_range_is_reported():
    cfg = W.CONFIGS["tiny"]
    tok, tgt = W.batch_for(cfg)
    tok = tok.copy()
    tok[3, 4] = 10
    with zo.Context.for_config(cfg) as ctx:
        th = dev(W.init_theta(cfg))
        lp = torch.empty(2, device="cuda")
        lm = torch.empty(2, device="cuda")
        zo.zo_probe_losses(ctx, th, 1, 2, 1e-3, dev(tok), dev(tgt), lp, lm)
        assert zo.zo_sync_status(ctx) == zo.ZO_ERR_BOUNDS
        assert zo.zo_sync_status(ctx) == zo.ZO_OK   # cleared


@pytest.mark.parametrize("t_bad", [0, 2])
def test_token_out_of_range_is_reported_on_the_vocabulary_path(t_bad):
    """bf16 model whose first layer takes its input term from the vocabulary
    table: a bad token at t = 0 (first-step kernel) or later (cell epilogue)."""
    V, E, H, L, B, T = 50, 512, 64, 1, 256, 3
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L, dtype="bf16")
    tok, tgt = W.random_batch(B, T, V, seed=1)
    tok = tok.copy()
    tok[7, t_bad] = V
    with zo.Context(V, E, H, L, "bf16", B, T, 0) as ctx:
        th = dev(W.init_theta(cfg))
        lp = torch.empty(2, device="cuda")
        lm = torch.empty(2, device="cuda")
        zo.zo_probe_losses(ctx, th, 1, 2, 1e-3, dev(tok), dev(tgt), lp, lm)
        assert zo.zo_sync_status(ctx) == zo.ZO_ERR_BOUNDS
        assert zo.zo_sync_status(ctx) == zo.ZO_OK


def test_nonfinite_loss_keeps_theta():
    cfg = W.CONFIGS["tiny"]
    theta = W.init_theta(cfg)
    theta[5] = np.nan
    tok, tgt = W.batch_for(cfg)
    with zo.Context.for_config(cfg) as ctx:
        th = dev(theta)
        lp = torch.empty(3, device="cuda")
        lm = torch.empty(3, device="cuda")
        c = torch.empty(3, device="cuda")
        zo.cdrge_step(ctx, th, 11, 3, 1e-3, 1e-3, dev(tok), dev(tgt), lp, lm, c)
        assert zo.zo_sync_status(ctx) == zo.ZO_ERR_NONFINITE
        got = th.cpu().numpy()
        assert np.array_equal(np.isnan(got), np.isnan(theta))
        assert np.array_equal(got[~np.isnan(theta)], theta[~np.isnan(theta)])


@pytest.mark.parametrize("n,bad", [(3, float("nan")), (12, float("inf")), (24, float("nan")),
                                   (64, float("-inf")), (100, float("nan"))])
def test_update_nonfinite_coefficient_keeps_theta(n, bad):
    """A non-finite coefficient leaves theta (and its bf16 shadow) unchanged and
    latches ZO_ERR_NONFINITE, in each update kernel (four-probe tables, two,
    four and eight eight-probe tables, four-probe passes)."""
    cfg = W.CONFIGS["charlm"]
    theta = W.init_theta(cfg)
    coeffs = (np.random.default_rng(n).standard_normal(n) * 1e-3).astype(np.float32)
    coeffs[n // 2] = bad
    tok, tgt = W.markov_batch(128, 2, step=3)
    with zo.Context.for_config(cfg, max_batch=128, max_seq=2, chunk=2) as ctx:
        th = dev(theta)
        lp0 = torch.empty(2, device="cuda")
        lm0 = torch.empty(2, device="cuda")
        zo.zo_probe_losses(ctx, th, 5, 2, cfg.eps, dev(tok), dev(tgt), lp0, lm0)
        zo.zo_update(ctx, th, 5, n, dev(coeffs))
        assert zo.zo_sync_status(ctx) == zo.ZO_ERR_NONFINITE
        assert np.array_equal(th.cpu().numpy(), theta)
        # the shadow still matches theta: the losses repeat bit for bit
        lp1 = torch.empty(2, device="cuda")
        lm1 = torch.empty(2, device="cuda")
        zo.zo_probe_losses(ctx, th, 5, 2, cfg.eps, dev(tok), dev(tgt), lp1, lm1)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        assert torch.equal(lp0, lp1) and torch.equal(lm0, lm1)


def test_host_step_matches_device_step():
    cfg = W.CONFIGS["tiny"]
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg)
    seed = W.step_seed(4)
    with zo.Context.for_config(cfg) as ctx:
        a = dev(theta)
        lp = torch.empty(8, device="cuda")
        lm = torch.empty(8, device="cuda")
        c = torch.empty(8, device="cuda")
        zo.cdrge_step(ctx, a, seed, 8, cfg.eps, cfg.eta, dev(tok), dev(tgt), lp, lm, c)
        b = dev(theta)
        hp = np.zeros(8, np.float32)
        hm = np.zeros(8, np.float32)
        zo.zo_step_host(ctx, b, seed, 8, cfg.eps, cfg.eta, tok, tgt, hp, hm)
        assert torch.equal(a, b)
        assert np.array_equal(hp, lp.cpu().numpy()) and np.array_equal(hm, lm.cpu().numpy())


# ---------------------------------------------------------------------------
# bf16 tensor-core path
# ---------------------------------------------------------------------------
def _bf16(x):
    """Round fp32 to bf16 (round to nearest even), returned as fp32."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("B,E,H", [(200, 64, 64), (128, 128, 128), (300, 256, 1024)])
@pytest.mark.parametrize("xp", [0, 1, 2, 3, 4, 5], ids=["single", "single_exact_eps", "pair",
                                                       "pair_exact_eps", "pair_direct_w",
                                                       "single_epi8"])
def test_tc_cell_preactivation_matches_emulation(B, E, H, xp):
    """One tensor-core cell step (layer 0, t = 0) against an fp64 evaluation of
    the same bf16 operands: x = bf16(E +- eps p) and either
    W = bf16(bf16(W) +- bf16(eps) p) or, with the exact-eps variant, the sum of
    the products with bf16(W) and with +-bf16(eps) p."""
    V, n = 50, 2
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=1, dtype="bf16")
    theta = W.init_theta(cfg, seed=8)
    tok, _ = W.random_batch(B, 1, V, seed=9)
    seed = W.step_seed(6)
    eps = np.float32(1e-3)
    segs, _ = O.layout(V, E, H, 1)
    offE, offW, offb = segs[0][3], segs[1][3], segs[2][3]
    with zo.Context(V, E, H, 1, "bf16", B, 1, n) as ctx:
        zo.zo_debug_cell_variant(ctx, xp)
        out = torch.full((2 * n, B, 4 * H), float("nan"), device="cuda")
        zo.zo_debug_cell_preact(ctx, dev(theta), seed, 0, n, float(eps), dev(tok), out)
        assert zo.zo_sync_status(ctx) == zo.ZO_OK
        got = out.cpu().numpy()
    Wt = theta[offW:offW + 4 * H * (E + H)].reshape(4 * H, E + H)[:, :E]
    for i in range(n):
        pE = O.probe_signs(seed, i, offE, V * E).reshape(V, E).astype(np.float32)
        pW = O.probe_signs(seed, i, offW, 4 * H * (E + H)).reshape(4 * H, E + H)[:, :E].astype(np.float32)
        pb = O.probe_signs(seed, i, offb, 4 * H).astype(np.float32)
        for s, sg in ((0, 1.0), (1, -1.0)):
            x = _bf16((theta[offE:offE + V * E].reshape(V, E) + np.float32(sg) * eps * pE)[tok[:, 0]])
            if xp in (zo.ZO_CELL_SINGLE_EXACT_EPS, zo.ZO_CELL_PAIR_EXACT_EPS):
                Wp = _bf16(Wt).astype(np.float64) + \
                    float(sg) * float(_bf16(np.float32(eps))) * pW.astype(np.float64)
            else:
                Wp = _bf16(_bf16(Wt) + np.float32(sg) * _bf16(np.float32(eps)) * pW)
            bias = (theta[offb:offb + 4 * H] + np.float32(sg) * eps * pb).astype(np.float64)
            want = x.astype(np.float64) @ Wp.astype(np.float64).T + bias
            g = got[2 * i + s]
            err = np.abs(g - want)
            assert np.all(err <= 1e-4 * (np.abs(x).astype(np.float64) @ np.abs(Wp).T + 1e-3)), \
                (i, s, float(err.max()))


@pytest.mark.parametrize("xp", [0, 1, 2, 3, 4, 5], ids=["single", "single_exact_eps", "pair",
                                                       "pair_exact_eps", "pair_direct_w",
                                                       "single_epi8"])
@pytest.mark.parametrize("V,E,H,L,B,T,n", [(50, 64, 64, 2, 200, 4, 4), (50, 128, 256, 1, 128, 3, 3),
                                           (50, 512, 64, 2, 256, 3, 2)])
def test_bf16_small_matches_oracle(V, E, H, L, B, T, n, xp):
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L, dtype="bf16")
    theta = W.init_theta(cfg, seed=1)
    tok, tgt = W.markov_batch(B, T, step=0, vocab=V)
    seed = W.step_seed(3)
    with zo.Context(V, E, H, L, "bf16", B, T, n) as ctx:
        zo.zo_debug_cell_variant(ctx, xp)
        lp, lm, rows = gpu_losses(ctx, theta, seed, n, 1e-3, tok, tgt, rows=True)
    olp, olm, orp, orm = O.probe_losses(theta, (V, E, H, L), seed, n, 1e-3, tok, tgt, return_rows=True)
    assert np.allclose(lp, olp, rtol=1e-2) and np.allclose(lm, olm, rtol=1e-2)
    assert np.allclose(rows[:, 0], orp, rtol=1e-2, atol=1e-3)
    assert np.allclose(rows[:, 1], orm, rtol=1e-2, atol=1e-3)


_NATIVE = None


def native_oracle():
    """The C++ fp64 oracle (built on first use)."""
    global _NATIVE
    if _NATIVE is None:
        from oracle import native
        _NATIVE = native.Oracle()
    return _NATIVE


def _row_slice_gate(cfg, theta, tok, tgt, seed, rows_gpu, probes, rows):
    """The GPU's per-row loss sums of a full launch (rows_gpu [n, 2, B]) against
    the C++ oracle on `probes` x `rows`: every row sum within 1e-2 relative;
    over the slice, sign(L+ - L-) agreement >= 95% and cos(g_gpu, g_oracle)
    >= 0.99 (from the probe Gram matrix).  Returns (agreement, cosine)."""
    NO = native_oracle()
    spec = spec_of(cfg)
    orl, orc = NO.probe_row_losses(theta, spec, seed, probes, cfg.eps, tok, tgt, rows=rows)
    g = rows_gpu[probes][:, :, rows]
    assert np.allclose(g, orl, rtol=1e-2), float(np.max(np.abs(g - orl) / np.abs(orl)))
    cnt = orc.sum()
    glp, glm = g[:, 0].sum(axis=1) / cnt, g[:, 1].sum(axis=1) / cnt
    olp, olm = orl[:, 0].sum(axis=1) / cnt, orl[:, 1].sum(axis=1) / cnt
    assert np.allclose(glp, olp, rtol=1e-2) and np.allclose(glm, olm, rtol=1e-2)
    agree = sign_agreement(glp, glm, olp, olm)
    cos = O.gram_cosine(glp - glm, olp - olm, NO.probe_gram(spec, seed, probes))
    print(f"{cfg.name}: {len(probes)} probes x {len(rows)} rows: sign agreement {agree:.4f}, "
          f"cosine {cos:.5f}")
    assert agree >= 0.95, agree
    assert cos >= 0.99, cos
    return agree, cos


def test_bf16_charlm_full_size_all_probes_on_32_rows():
    """charlm exactly as benchmarked (64 probes, batch 1024, T = 10); the C++
    oracle evaluates all 64 probes on batch rows 0..31 (each row's forward is
    independent of the others), compared per row and through the slice's
    sign agreement and estimate cosine over the 64 probes."""
    cfg = W.CONFIGS["charlm"]
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg, step=0)
    seed = W.step_seed(0)
    with zo.Context.for_config(cfg) as ctx:
        lp, lm, rows = gpu_losses(ctx, theta, seed, cfg.n_pert, cfg.eps, tok, tgt, rows=True)
    _row_slice_gate(cfg, theta, tok, tgt, seed, rows, list(range(cfg.n_pert)), np.arange(32))
    n_all = (tgt >= 0).sum()
    assert np.allclose(lp, rows[:, 0].sum(axis=1) / n_all, rtol=1e-5)
    assert np.allclose(lm, rows[:, 1].sum(axis=1) / n_all, rtol=1e-5)


@pytest.mark.slow
@pytest.mark.parametrize("name,n_probes,n_rows", [("lstm270m", 8, 32), ("lstm1b", 2, 32),
                                                  ("lstm4b", 1, 8)])
def test_bf16_large_full_launch_sampled_rows(name, n_probes, n_rows):
    """270M / 1.1B / 4.3B exactly as benchmarked (all probes, batch 1024,
    T = 10); the C++ oracle evaluates probes 0..n_probes-1 on batch rows
    0..n_rows-1, compared per row, plus (with two probes or more) the slice's
    sign agreement and estimate cosine.  The full-batch losses are the means of
    the GPU's own row sums."""
    cfg = W.CONFIGS[name]
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg, step=0)
    seed = W.step_seed(0)
    with zo.Context.for_config(cfg) as ctx:
        lp, lm, rows = gpu_losses(ctx, theta, seed, cfg.n_pert, cfg.eps, tok, tgt, rows=True)
    assert np.all(np.isfinite(lp)) and np.all(np.isfinite(lm))
    probes, sl = list(range(n_probes)), np.arange(n_rows)
    if n_probes >= 2:
        _row_slice_gate(cfg, theta, tok, tgt, seed, rows, probes, sl)
    else:
        orl, _ = native_oracle().probe_row_losses(theta, spec_of(cfg), seed, probes, cfg.eps, tok,
                                                  tgt, rows=sl)
        assert np.allclose(rows[probes][:, :, sl], orl, rtol=1e-2)
    n_all = (tgt >= 0).sum()
    assert np.allclose(lp, rows[:, 0].sum(axis=1) / n_all, rtol=1e-5)
    assert np.allclose(lm, rows[:, 1].sum(axis=1) / n_all, rtol=1e-5)


@pytest.mark.parametrize("name,slices", [("tiny", [(0, 3), (3, 5)]), ("charlm", [(0, 2), (5, 1), (62, 2)])])
def test_probe_slices_match_full_call(name, slices):
    """zo_probe_losses_slice(probe_begin, n) returns entries probe_begin ..
    probe_begin + n - 1 of zo_probe_losses, bit for bit (the unit of the
    probe-parallel scheme)."""
    cfg = W.CONFIGS[name]
    theta = dev(W.init_theta(cfg))
    B = min(cfg.batch, 128)
    tok, tgt = W.batch_for(cfg)
    tok, tgt = dev(tok[:B]), dev(tgt[:B])
    n = cfg.n_pert
    with zo.Context.for_config(cfg, max_batch=B, chunk=8 if cfg.dtype == "bf16" else None) as ctx:
        lp = torch.empty(n, device="cuda")
        lm = torch.empty(n, device="cuda")
        zo.zo_probe_losses(ctx, theta, 9, n, cfg.eps, tok, tgt, lp, lm)
        for b0, c in slices:
            sp = torch.empty(c, device="cuda")
            sm = torch.empty(c, device="cuda")
            zo.zo_probe_losses_slice(ctx, theta, 9, b0, c, cfg.eps, tok, tgt, sp, sm)
            assert zo.zo_sync_status(ctx) == zo.ZO_OK
            assert torch.equal(sp, lp[b0:b0 + c]) and torch.equal(sm, lm[b0:b0 + c])


@pytest.mark.parametrize("V,E,H,L,B,T,n,chunk,frac", [
    (50, 128, 64, 3, 300, 3, 3, 0, 0.0),    # three layers, E != H, ragged 256-row tiles
    (64, 64, 128, 2, 257, 2, 5, 2, 0.2),    # V = 64 (all logit columns), 3 chunks (2, 2, 1)
    (2, 64, 64, 1, 1, 4, 2, 0, 0.0),        # V = 2, a single batch row
    (33, 64, 64, 2, 128, 1, 4, 0, 0.0),     # T = 1 (no recurrent input at all)
    (50, 64, 64, 1, 100, 3, 2, 0, 1.0),     # nothing scored: losses 0
    # E >= 512 and >= 256 batch rows: layer 0's input term from the per-chunk
    # vocabulary table (t = 0 from the table alone, later steps add it to the
    # recurrent K stages in the epilogue)
    (50, 512, 64, 2, 256, 3, 3, 0, 0.2),    # two layers, ignored targets
    (64, 512, 128, 1, 300, 1, 2, 0, 0.0),   # T = 1: the first-step kernel only, ragged rows
    (17, 1024, 64, 2, 260, 2, 3, 2, 0.3),   # two chunks, V = 17
])
def test_bf16_edge_cases(V, E, H, L, B, T, n, chunk, frac):
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L, dtype="bf16")
    theta = W.init_theta(cfg, seed=2)
    tok, tgt = W.random_batch(B, T, V, seed=5, ignore_frac=frac)
    seed = W.step_seed(8)
    with zo.Context(V, E, H, L, "bf16", B, T, chunk) as ctx:
        lp, lm, rows = gpu_losses(ctx, theta, seed, n, 1e-3, tok, tgt, rows=True)
    olp, olm, orp, orm = O.probe_losses(theta, (V, E, H, L), seed, n, 1e-3, tok, tgt,
                                        return_rows=True)
    if frac == 1.0:
        assert np.all(lp == 0) and np.all(lm == 0) and np.all(rows == 0)
        return
    assert np.allclose(lp, olp, rtol=1e-2) and np.allclose(lm, olm, rtol=1e-2)
    assert np.allclose(rows[:, 0], orp, rtol=1e-2, atol=1e-3)
    assert np.allclose(rows[:, 1], orm, rtol=1e-2, atol=1e-3)


def test_bf16_shape_limits_are_reported():
    for V, E, H in ((65, 64, 64), (50, 48, 64), (50, 64, 96)):
        with pytest.raises(zo.ZOError) as e:
            zo.Context(V, E, H, 1, "bf16", 8, 2, 1)
        assert e.value.status == zo.ZO_ERR_UNSUPPORTED
