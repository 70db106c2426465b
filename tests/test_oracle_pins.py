"""Pins for the fp64 oracle: each test ties an oracle function to something
other than itself (published known-answer values, a library routine, a closed
form, an exact identity, or brute force on a tiny input)."""
import ctypes
import ctypes.util
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# Philox4x32-10
# ---------------------------------------------------------------------------
def test_philox_known_answers():
    """Random123's published known-answer vectors for Philox4x32-10."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = O.philox4x32_10(*v[:6])
        assert [int(x) for x in out] == v[6:10]


def _curand_host():
    for name in ("/usr/local/cuda/lib64/libcurand.so", ctypes.util.find_library("curand")):
        if name and os.path.exists(name):
            try:
                return ctypes.CDLL(name)
            except OSError:
                pass
    return None


def test_philox_against_curand_host_generator():
    """cuRAND's CPU-side Philox4_32_10 generator (a library routine) emits output
    block k from counter (k / 65536, 0, k % 65536, 0) with key = seed.  With the
    oracle's counter (q, 0, probe, 0) this is probe k % 65536, block q = k / 65536,
    so its stream reproduces the oracle's sign words bit for bit."""
    lib = _curand_host()
    if lib is None:
        pytest.skip("libcurand not available")
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), 161) == 0   # PHILOX4_32_10
    seed = W.step_seed(7)
    assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
    nblk = 2 * 65536 + 64
    out = np.zeros(4 * nblk, dtype=np.uint32)
    assert lib.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(out.size)) == 0
    lib.curandDestroyGenerator(gen)
    out = out.reshape(-1, 4)
    for probe in (0, 1, 5, 511, 4097, 65535):
        for q in (0, 1):
            k = q * 65536 + probe
            if k >= nblk:
                continue
            w = O.sign_words(seed, probe, q, 1)[0]
            assert list(w) == list(out[k]), (probe, q)
    # block 2 for the first probes
    for probe in range(64):
        assert list(O.sign_words(seed, probe, 2, 1)[0]) == list(out[2 * 65536 + probe])


def test_sign_mapping_and_signs_at():
    """probe_signs (block decode) and signs_at (per-index decode) agree, and the
    sign of element j is bit (e>>1) + 16*(e&1) of word (j>>5)&3, e = j&31."""
    seed = W.step_seed(3)
    s = O.probe_signs(seed, 9, 100, 1000)
    assert np.array_equal(s, O.signs_at(seed, 9, np.arange(100, 1100)))
    words = O.sign_words(seed, 9, 0, 9)
    for j in (100, 101, 127, 128, 129, 160, 161, 1099):
        e = j & 31
        bit = (int(words[j >> 7][(j >> 5) & 3]) >> ((e >> 1) + 16 * (e & 1))) & 1
        assert s[j - 100] == 1 - 2 * bit


def test_rademacher_statistics():
    """pith.science review, "Assumptions": E[p] = 0 and E[p p^T] = I.
    Over 2^22 signs per probe: mean, lag-1 correlation and cross-probe
    correlation all within 5 standard errors of 0."""
    seed = W.step_seed(11)
    n = 1 << 22
    P = np.stack([O.probe_signs(seed, i, 0, n).astype(np.float64) for i in range(4)])
    se = 5.0 / math.sqrt(n)
    assert np.all(np.abs(P.mean(axis=1)) < se)
    assert np.all(np.abs((P[:, 1:] * P[:, :-1]).mean(axis=1)) < se)
    C = P @ P.T / n
    assert np.allclose(np.diag(C), 1.0)
    off = C[~np.eye(4, dtype=bool)]
    assert np.all(np.abs(off) < se)
    # every bit position of every word is balanced
    w = O.sign_words(seed, 0, 0, 1 << 16)
    bits = (w[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
    frac = bits.mean(axis=0)
    assert np.all(np.abs(frac - 0.5) < 5 * 0.5 / math.sqrt(1 << 16))


# ---------------------------------------------------------------------------
# Layout
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name,d_real,d_pad", [
    ("tiny", 6762, 7040), ("overfit", 240050, 240128),
    ("charlm", 13703730, 13703808), ("lstm270m", 268877874, None),
    ("lstm1b", 1074626610, None)])
def test_layout_sizes(name, d_real, d_pad):
    """Parameter counts: E V*E + sum_l 4H(in_l+H) + 4H per layer + V*H + V."""
    c = W.CONFIGS[name]
    V, E, H, L = c.vocab, c.embed, c.hidden, c.layers
    closed = V * E + sum(4 * H * ((E if l == 0 else H) + H) + 4 * H for l in range(L)) + V * H + V
    assert closed == d_real
    segs, dp = O.layout(V, E, H, L)
    assert sum(r * cc for _, r, cc, _ in segs) == d_real
    assert all(off % 128 == 0 for *_, off in segs)
    assert W.segments(V, E, H, L) == (segs, dp)
    if d_pad is not None:
        assert dp == d_pad


# ---------------------------------------------------------------------------
# Forward and loss against torch (library routines, fp64)
# ---------------------------------------------------------------------------
def torch_row_losses(theta, spec, tokens, targets):
    V, E, H, L = spec
    P = O.unpack(np.asarray(theta, dtype=np.float64), V, E, H, L)
    emb = torch.nn.Embedding(V, E, dtype=torch.float64)
    lstm = torch.nn.LSTM(E, H, num_layers=L, batch_first=True, dtype=torch.float64)
    lin = torch.nn.Linear(H, V, dtype=torch.float64)
    with torch.no_grad():
        emb.weight.copy_(torch.from_numpy(P["E"]))
        for l in range(L):
            in_l = E if l == 0 else H
            Wl = torch.from_numpy(P[f"W{l + 1}"])
            getattr(lstm, f"weight_ih_l{l}").copy_(Wl[:, :in_l])
            getattr(lstm, f"weight_hh_l{l}").copy_(Wl[:, in_l:])
            getattr(lstm, f"bias_ih_l{l}").copy_(torch.from_numpy(P[f"b{l + 1}"]))
            getattr(lstm, f"bias_hh_l{l}").zero_()
        lin.weight.copy_(torch.from_numpy(P["Wout"]))
        lin.bias.copy_(torch.from_numpy(P["bout"]))
        out, _ = lstm(emb(torch.from_numpy(tokens.astype(np.int64))))
        logits = lin(out)
        tg = torch.from_numpy(targets.astype(np.int64))
        ce = torch.nn.functional.cross_entropy(logits.reshape(-1, V), tg.reshape(-1),
                                               ignore_index=-1, reduction="none")
        return ce.reshape(tokens.shape).sum(dim=1).numpy()


@pytest.mark.parametrize("V,E,H,L,B,T,frac", [
    (10, 16, 32, 1, 8, 21, 0.0), (50, 64, 128, 2, 1, 30, 0.0), (7, 5, 6, 3, 4, 9, 0.3),
    (13, 8, 24, 2, 5, 7, 0.5)])
def test_forward_matches_torch_lstm(V, E, H, L, B, T, frac):
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L)
    theta = W.init_theta(cfg, seed=5)
    tokens, targets = W.random_batch(B, T, V, seed=3, ignore_frac=frac)
    P = O.unpack(theta.astype(np.float64), V, E, H, L)
    rl, rc = O.lstm_row_losses(P, L, tokens, targets)
    ref = torch_row_losses(theta, (V, E, H, L), tokens, targets)
    assert np.allclose(rl, ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(rc, (targets >= 0).sum(axis=1))


def test_tiny_copy_batch_format():
    tok, tgt = W.copy_batch(8, 10, seed=0)
    assert tok.shape == (8, 21) and tgt.shape == (8, 21)
    assert np.all((tok[:, :10] >= 1) & (tok[:, :10] <= 8))
    assert np.all(tok[:, 10] == 9) and np.all(tok[:, 11:] == 0)
    assert np.all(tgt[:, :11] == -1) and np.array_equal(tgt[:, 11:], tok[:, :10])


# ---------------------------------------------------------------------------
# Estimator algebra on a quadratic (closed forms)
# ---------------------------------------------------------------------------
def _all_signs(d):
    idx = np.arange(1 << d)[:, None]
    return (1 - 2 * ((idx >> np.arange(d)) & 1)).astype(np.float64)


def test_quadratic_all_sign_vectors_give_exact_gradient():
    """Method check 1 (exactness): on L = 1/2 x^T A x + b^T x + k, averaging the central
    difference over all 2^d Rademacher vectors returns the gradient exactly
    (the cubic remainder vanishes and sum_p p p^T = 2^d I).  With eta = eps the
    update is theta' = theta - eps * grad."""
    d = 10
    rng = np.random.default_rng(0)
    M = rng.standard_normal((d, d))
    A = M @ M.T
    b = rng.standard_normal(d)
    theta = rng.standard_normal(d)
    loss = lambda x: 0.5 * x @ A @ x + b @ x + 3.0
    eps = 0.25
    P = _all_signs(d)
    lp = np.array([loss(theta + eps * p) for p in P])
    lm = np.array([loss(theta - eps * p) for p in P])
    c = O.coefficients(lp, lm, len(P), eps, eps)
    new = O.update_with_probes(theta, P, c)
    grad = A @ theta + b
    assert np.allclose((theta - new) / eps, grad, rtol=1e-12, atol=1e-12)
    assert np.allclose(O.estimate(lp, lm, eps, P), grad, rtol=1e-12, atol=1e-12)
    # eta != eps: the step scales by eta
    c2 = O.coefficients(lp, lm, len(P), eps, 0.5)
    assert np.allclose((theta - O.update_with_probes(theta, P, c2)) / 0.5, grad, rtol=1e-12)


def test_single_probe_error_identity():
    """pith.science referee, major comment 1: a single Rademacher probe has
    E||g_i - grad||^2 = (d - 1) ||grad||^2 (exact over all 2^d sign vectors)."""
    d = 9
    rng = np.random.default_rng(1)
    M = rng.standard_normal((d, d))
    A = M + M.T
    b = rng.standard_normal(d)
    theta = rng.standard_normal(d)
    loss = lambda x: 0.5 * x @ A @ x + b @ x
    eps = float(np.float32(1e-2))      # the oracle promotes eps from fp32
    grad = A @ theta + b
    errs = []
    for p in _all_signs(d):
        g = O.estimate([loss(theta + eps * p)], [loss(theta - eps * p)], eps, p[None, :])
        errs.append(np.sum((g - grad) ** 2))
    assert math.isclose(np.mean(errs), (d - 1) * np.sum(grad ** 2), rel_tol=1e-9)


def test_app_c_antithetic_forward_difference_equals_central_difference():
    """pith.science review, Appendix C: the antithetic forward-difference
    estimator 1/(2K) sum_i [(L(t+e p)-L(t))/e p + (L(t-e p)-L(t))/e (-p)] equals
    the central-difference estimator.  Checked on the oracle's own LSTM losses."""
    cfg = W.small_config(vocab=5, embed=3, hidden=4, layers=1)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg, seed=2)
    tok, tgt = W.random_batch(3, 5, cfg.vocab, seed=1)
    seed, K, eps = W.step_seed(4), 6, 1e-3
    lp, lm = O.probe_losses(theta, spec, seed, K, eps, tok, tgt)
    l0 = O.loss_at(theta, spec, tok, tgt)
    P = O.probe_matrix(spec, seed, K).astype(np.float64)
    e = float(np.float32(eps))
    fd = sum(((lp[i] - l0) / e) * P[i] + ((lm[i] - l0) / e) * (-P[i]) for i in range(K)) / (2 * K)
    cd = O.estimate(lp, lm, eps, P)
    assert np.allclose(fd, cd, rtol=1e-9, atol=1e-12)


def test_forward_coefficients_over_antithetic_set_give_the_central_update():
    """Forward-difference coefficients (eta (L+ - L0)/(eps n)) over the
    antithetic set {p_i, -p_i} (n = 2K; L(theta - eps p_i) is the + loss of
    -p_i) move theta exactly as the central coefficients over {p_i} (n = K):
    the Appendix C identity on the coefficients.  Plus one value by hand."""
    assert O.coefficients_forward([3.0], 2.0, 2, 0.5, 0.25)[0] == 0.25
    cfg = W.small_config(vocab=5, embed=3, hidden=4, layers=1)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg, seed=2)
    tok, tgt = W.random_batch(3, 5, cfg.vocab, seed=1)
    seed, K, eps, eta = W.step_seed(6), 5, 1e-3, 3e-2
    lp, lm = O.probe_losses(theta, spec, seed, K, eps, tok, tgt)
    l0 = O.loss_at(theta, spec, tok, tgt)
    P = O.probe_matrix(spec, seed, K).astype(np.float64)
    cf = O.coefficients_forward(np.concatenate([lp, lm]), l0, 2 * K, eps, eta)
    fwd = cf[:K] @ P + cf[K:] @ (-P)
    cen = O.coefficients(lp, lm, K, eps, eta) @ P
    assert np.allclose(fwd, cen, rtol=1e-12, atol=1e-15)


def test_antisymmetry_negated_probe_negates_coefficient():
    """Method check 2 (antisymmetry): replacing p_i by -p_i swaps L+ and L-, so c_i -> -c_i
    exactly (IEEE subtraction is antisymmetric)."""
    cfg = W.CONFIGS["tiny"]
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg)
    seed = W.step_seed(0)
    lp, lm = O.probe_losses(theta, spec, seed, 3, cfg.eps, tok, tgt)
    np_, nm = O.probe_losses(theta, spec, seed, 3, cfg.eps, tok, tgt, probe_scale=-1)
    assert np.array_equal(np_, lm) and np.array_equal(nm, lp)
    c = O.coefficients(lp, lm, 3, cfg.eps, cfg.eta)
    cn = O.coefficients(np_, nm, 3, cfg.eps, cfg.eta)
    assert np.array_equal(cn, -c)


# ---------------------------------------------------------------------------
# Central difference vs autograd, and convergence of the estimator
# ---------------------------------------------------------------------------
def _autograd_gradient(theta, spec, tokens, targets):
    """d L / d theta via torch fp64 autograd on the same flat layout."""
    V, E, H, L = spec
    segs, d_pad = O.layout(V, E, H, L)
    th = torch.tensor(np.asarray(theta, dtype=np.float64), requires_grad=True)
    P = {}
    for name, r, c, off in segs:
        a = th[off:off + r * c]
        P[name] = a if r == 1 else a.reshape(r, c)
    B, T = tokens.shape
    h = [torch.zeros(B, H, dtype=torch.float64) for _ in range(L)]
    cs = [torch.zeros(B, H, dtype=torch.float64) for _ in range(L)]
    tot = 0.0
    n = int((targets >= 0).sum())
    for t in range(T):
        x = P["E"][torch.from_numpy(tokens[:, t].astype(np.int64))]
        for l in range(L):
            G = torch.cat([x, h[l]], 1) @ P[f"W{l + 1}"].T + P[f"b{l + 1}"]
            i, f, g, o = G.split(H, dim=1)
            cs[l] = torch.sigmoid(f) * cs[l] + torch.sigmoid(i) * torch.tanh(g)
            h[l] = torch.sigmoid(o) * torch.tanh(cs[l])
            x = h[l]
        logits = x @ P["Wout"].T + P["bout"]
        tg = torch.from_numpy(targets[:, t].astype(np.int64))
        tot = tot + torch.nn.functional.cross_entropy(logits, tg, ignore_index=-1, reduction="sum")
    (tot / n).backward()
    return th.grad.numpy()


def test_central_difference_matches_directional_derivative():
    """(L+ - L-)/(2 eps) = grad . p + O(eps^2) (review: bias O(eps^2));
    grad from torch fp64 autograd.  The error must also shrink ~4x when eps halves."""
    cfg = W.small_config(vocab=6, embed=4, hidden=5, layers=2)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg, seed=3)
    tok, tgt = W.random_batch(3, 6, cfg.vocab, seed=2)
    g = _autograd_gradient(theta, spec, tok, tgt)
    seed = W.step_seed(1)
    P = O.probe_matrix(spec, seed, 4).astype(np.float64)
    errs = []
    for eps in (4e-3, 2e-3):
        lp, lm = O.probe_losses(theta, spec, seed, 4, eps, tok, tgt)
        e = float(np.float32(eps))
        cd = (lp - lm) / (2 * e)
        dd = P @ g
        errs.append(np.abs(cd - dd))
        assert np.allclose(cd, dd, rtol=1e-3, atol=1e-5)
    assert np.all(errs[1] < 0.4 * errs[0] + 1e-12)


def test_coordinate_cd_matches_autograd():
    """The brute-force coordinate CD gradient is grad + O(eps^2) (torch fp64 autograd)."""
    cfg = W.small_config(vocab=4, embed=2, hidden=3, layers=1)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg, seed=4).astype(np.float64)
    tok, tgt = W.random_batch(2, 4, cfg.vocab, seed=5)
    mask = O.real_mask(*spec)
    g_ad = _autograd_gradient(theta, spec, tok, tgt)
    g_cd = O.coordinate_cd_gradient(lambda t: O.loss_at(t, spec, tok, tgt), theta, 1e-4,
                                    index=np.nonzero(mask)[0])
    assert np.allclose(g_cd[mask], g_ad[mask], rtol=1e-6, atol=1e-9)


def test_estimator_converges_to_coordinate_cd_gradient():
    """Method check 3 (convergence): with K >> d probes, g_hat_K (Philox probes, oracle
    losses) approaches the coordinate CD gradient; for Rademacher probes
    E cos ~ sqrt(K / (K + d - 1))."""
    cfg = W.small_config(vocab=3, embed=2, hidden=2, layers=1)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg, seed=6)
    tok, tgt = W.random_batch(2, 4, cfg.vocab, seed=7)
    mask = O.real_mask(*spec)
    d = int(mask.sum())
    eps = 1e-3
    e = float(np.float32(eps))
    g_cd = O.coordinate_cd_gradient(lambda t: O.loss_at(t, spec, tok, tgt),
                                    theta.astype(np.float64), e, index=np.nonzero(mask)[0])
    K = 4000
    seed = W.step_seed(9)
    lp, lm = O.probe_losses(theta, spec, seed, K, eps, tok, tgt)
    P = O.probe_matrix(spec, seed, K).astype(np.float64)
    g = O.estimate(lp, lm, eps, P)
    cos = float(g @ g_cd / (np.linalg.norm(g) * np.linalg.norm(g_cd)))
    expect = math.sqrt(K / (K + d - 1))
    assert cos >= 0.99
    assert abs(cos - expect) < 0.01
    # and a small K is visibly worse, as the variance bound says
    g8 = O.estimate(lp[:8], lm[:8], eps, P[:8])
    cos8 = float(g8 @ g_cd / (np.linalg.norm(g8) * np.linalg.norm(g_cd)))
    assert cos8 < 0.9


def test_update_replays_probes():
    """update() (seed replay) equals the explicit sum with probe_matrix, and
    update_at() equals update() at sampled indices; padding is untouched."""
    cfg = W.CONFIGS["tiny"]
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg)
    seed = W.step_seed(2)
    c = np.random.default_rng(0).standard_normal(cfg.n_pert) * 1e-3
    new = O.update(theta, spec, seed, cfg.n_pert, c)
    P = O.probe_matrix(spec, seed, cfg.n_pert)
    ref = O.update_with_probes(theta, P, c)
    assert np.allclose(new, ref, rtol=0, atol=1e-15)
    mask = O.real_mask(*spec)
    assert np.array_equal(new[~mask], theta[~mask].astype(np.float64))
    idx = np.nonzero(mask)[0][::37]
    assert np.allclose(O.update_at(theta, seed, cfg.n_pert, c, idx), new[idx], rtol=0, atol=1e-15)


# ---------------------------------------------------------------------------
# The cosine gate of the GPU tests: probe Gram matrix and cos(g_a, g_b)
# ---------------------------------------------------------------------------
def test_probe_gram_matches_explicit_products():
    """probe_gram (per-segment sign products over the real parameters) equals
    P P^T of the explicit probe matrix (padding columns 0) for a subset of
    probes in any order; its diagonal is d_real (closed form)."""
    cfg = W.small_config(vocab=5, embed=3, hidden=7, layers=2)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    seed = W.step_seed(8)
    P = O.probe_matrix(spec, seed, 6).astype(np.int64)
    sel = [4, 1, 5]
    G = O.probe_gram(spec, seed, sel)
    assert np.array_equal(G, (P @ P.T)[np.ix_(sel, sel)])
    d_real = cfg.vocab * cfg.embed + sum(4 * cfg.hidden * ((cfg.embed if l == 0 else cfg.hidden)
                                                           + cfg.hidden) + 4 * cfg.hidden
                                         for l in range(cfg.layers)) + cfg.vocab * cfg.hidden + cfg.vocab
    assert np.all(np.diag(G) == d_real)


def test_gram_cosine_hand_values():
    """cos(sum a_i p_i, sum b_i p_i) from the Gram matrix.  Orthonormal probes
    (G = I): orthogonal coefficients give 0, proportional 1, opposite -1,
    (3, 4) vs (4, 3) gives 24/25.  Probes (1,1,1) and (1,1,-1) (G = [[3,1],[1,3]]):
    the two probes themselves have cosine 1/3."""
    I = np.eye(2)
    assert O.gram_cosine([1, 0], [0, 1], I) == 0.0
    assert math.isclose(O.gram_cosine([1, 2], [2, 4], I), 1.0, rel_tol=1e-15)
    assert math.isclose(O.gram_cosine([1, 2], [-1, -2], I), -1.0, rel_tol=1e-15)
    assert math.isclose(O.gram_cosine([3, 4], [4, 3], I), 24 / 25, rel_tol=1e-15)
    G = np.array([[3.0, 1.0], [1.0, 3.0]])
    assert math.isclose(O.gram_cosine([1, 0], [0, 1], G), 1 / 3, rel_tol=1e-15)
    assert math.isclose(O.gram_cosine([2, 0], [0, 5], G), 1 / 3, rel_tol=1e-15)


def test_gram_cosine_equals_cosine_of_explicit_estimates():
    """On Philox probes, gram_cosine(a, b, probe_gram) is the plain cosine of the
    explicit vectors sum a_i p_i and sum b_i p_i built from the probe matrix."""
    cfg = W.CONFIGS["tiny"]
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    seed = W.step_seed(5)
    n = 6
    rng = np.random.default_rng(2)
    a = rng.standard_normal(n)
    b = a + 0.3 * rng.standard_normal(n)
    P = O.probe_matrix(spec, seed, n).astype(np.float64)
    ga, gb = a @ P, b @ P
    want = float(ga @ gb / (np.linalg.norm(ga) * np.linalg.norm(gb)))
    got = O.gram_cosine(a, b, O.probe_gram(spec, seed, range(n)))
    assert math.isclose(got, want, rel_tol=1e-12)
