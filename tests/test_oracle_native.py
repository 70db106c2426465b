"""Pins for the plain C++ fp64 oracle (oracle/zo_oracle_cpu.cpp).  Each ties it
to something other than itself: the published Philox known-answer vectors,
torch fp64 (nn.LSTM + cross_entropy, autograd), closed forms, and the
independently written numpy oracle.  The last test compiles copies of the C++
source with planted mistakes and checks that a pin catches every one."""
import math
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle as O
import workloads as W
from oracle import native
from tests import test_oracle_pins as pins

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def N():
    return native.Oracle()


# ---------------------------------------------------------------------------
# pins, each a function of an oracle instance (reused on the mutants below)
# ---------------------------------------------------------------------------
def pin_philox_known_answers(N):
    """Random123's published known-answer vectors for Philox4x32-10."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        assert list(N.philox4x32_10(*v[:6])) == v[6:10]


def pin_signs_match_numpy_oracle(N):
    """Sign words and decoded signs against the numpy oracle (written
    separately) over several seeds, probes and block offsets (q >= 2^32)."""
    for seed in (W.step_seed(0), 0, (1 << 64) - 1):
        for probe, q0 in ((0, 0), (7, 1000), (65535, (1 << 32) - 2)):
            assert np.array_equal(N.sign_words(seed, probe, q0, 5), O.sign_words(seed, probe, q0, 5))
        assert np.array_equal(N.probe_signs(seed, 3, 77, 1000), O.probe_signs(seed, 3, 77, 1000))


def pin_forward_matches_torch(N):
    """The unperturbed forward (eps = 0) against torch fp64 nn.LSTM +
    Embedding + Linear + cross_entropy, per row, incl. 3 layers and ignored
    targets."""
    for V, E, H, L, B, T, frac in ((10, 16, 32, 1, 8, 21, 0.0), (7, 5, 6, 3, 4, 9, 0.3),
                                   (13, 8, 24, 2, 5, 7, 0.5)):
        cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L)
        theta = W.init_theta(cfg, seed=5)
        tok, tgt = W.random_batch(B, T, V, seed=3, ignore_frac=frac)
        rl, rc = N.probe_row_losses(theta, (V, E, H, L), 0, [0], 0.0, tok, tgt, threads=2)
        ref = pins.torch_row_losses(theta, (V, E, H, L), tok, tgt)
        assert np.allclose(rl[0, 0], ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(rl[0, 1], ref, rtol=1e-12, atol=1e-12)
        assert np.array_equal(rc, (tgt >= 0).sum(axis=1))


def pin_perturbed_forward_matches_torch(N):
    """L(theta +- eps p_i) against torch fp64 at the explicitly perturbed
    point theta +- eps p_i, p_i from the numpy oracle's sign matrix."""
    V, E, H, L, B, T = 9, 6, 8, 2, 4, 6
    spec = (V, E, H, L)
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L)
    theta = W.init_theta(cfg, seed=8)
    tok, tgt = W.random_batch(B, T, V, seed=4, ignore_frac=0.2)
    seed, eps = W.step_seed(12), 0.05     # a large radius so that a sign error shows
    e = float(np.float32(eps))
    Pm = O.probe_matrix(spec, seed, 3).astype(np.float64)
    rl, _ = N.probe_row_losses(theta, spec, seed, [0, 2], eps, tok, tgt, threads=2)
    for k, i in enumerate((0, 2)):
        for s, sg in ((0, 1.0), (1, -1.0)):
            ref = pins.torch_row_losses(theta.astype(np.float64) + sg * e * Pm[i], spec, tok, tgt)
            assert np.allclose(rl[k, s], ref, rtol=1e-12, atol=1e-12)


def pin_central_difference_matches_autograd(N):
    """(L+ - L-)/(2 eps) = grad . p + O(eps^2), grad from torch fp64 autograd."""
    V, E, H, L = 6, 4, 5, 2
    spec = (V, E, H, L)
    cfg = W.small_config(vocab=V, embed=E, hidden=H, layers=L)
    theta = W.init_theta(cfg, seed=3)
    tok, tgt = W.random_batch(3, 6, V, seed=2)
    g = pins._autograd_gradient(theta, spec, tok, tgt)
    seed, eps = W.step_seed(1), 2e-3
    lp, lm = N.probe_losses(theta, spec, seed, 4, eps, tok, tgt, threads=2)
    P = O.probe_matrix(spec, seed, 4).astype(np.float64)
    cd = (lp - lm) / (2 * float(np.float32(eps)))
    assert np.allclose(cd, P @ g, rtol=1e-3, atol=1e-5)


def pin_coefficients_closed_form(N):
    """c_i = eta (L+ - L-)/(2 eps n): hand values; forward: eta (L+ - L0)/(eps n)."""
    assert N.coefficients([3.0, 1.0], [1.0, 3.0], 2, 0.5, 0.25).tolist() == [0.25, -0.25]
    assert N.coefficients_forward([3.0], 2.0, 2, 0.5, 0.25).tolist() == [0.25]
    lp = np.random.default_rng(0).standard_normal(7)
    lm = np.random.default_rng(1).standard_normal(7)
    assert np.allclose(N.coefficients(lp, lm, 7, 1e-3, 3e-2),
                       float(np.float32(3e-2)) * (lp - lm) / (2 * float(np.float32(1e-3)) * 7),
                       rtol=1e-15)


def pin_update_matches_explicit_sum(N):
    """theta' = theta - sum_i c_i p_i with the probes replayed from the seed,
    against the explicit product with the numpy oracle's probe matrix; padding
    unchanged; update_at equals update at sampled indices."""
    cfg = W.small_config(vocab=7, embed=9, hidden=10, layers=2)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg, seed=2)
    seed, n = W.step_seed(4), 13
    c = np.random.default_rng(3).standard_normal(n) * 1e-3
    new = N.update(theta, spec, seed, n, c, threads=3)
    ref = theta.astype(np.float64) - c @ O.probe_matrix(spec, seed, n).astype(np.float64)
    assert np.allclose(new, ref, rtol=0, atol=1e-15)
    mask = O.real_mask(*spec)
    assert np.array_equal(new[~mask], theta[~mask].astype(np.float64))
    idx = np.nonzero(mask)[0][::11]
    assert np.allclose(N.update_at(theta, spec, seed, n, c, idx), new[idx], rtol=0, atol=1e-15)
    for j0, j1 in ((0, len(theta)), (5, 300), (200, 201), (130, 130)):
        assert np.array_equal(N.update_range(theta, spec, seed, n, c, j0, j1, threads=2), new[j0:j1])


def pin_gram_matches_explicit(N):
    """G_ik = p_i . p_k over the real parameters: the explicit product of the
    numpy oracle's probe matrix (padding columns 0), diagonal = d_real."""
    cfg = W.small_config(vocab=5, embed=3, hidden=7, layers=2)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    seed = W.step_seed(8)
    P = O.probe_matrix(spec, seed, 6).astype(np.int64)
    G = N.probe_gram(spec, seed, [5, 0, 3], threads=2)
    sel = [5, 0, 3]
    assert np.array_equal(G, (P @ P.T)[np.ix_(sel, sel)].astype(np.float64))
    d_real = int(O.real_mask(*spec).sum())
    assert np.all(np.diag(G) == d_real)


PINS = [pin_philox_known_answers, pin_signs_match_numpy_oracle, pin_forward_matches_torch,
        pin_perturbed_forward_matches_torch, pin_central_difference_matches_autograd,
        pin_coefficients_closed_form, pin_update_matches_explicit_sum, pin_gram_matches_explicit]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_native_oracle_pin(pin, N):
    pin(N)


# ---------------------------------------------------------------------------
# agreement with the numpy oracle on the workloads' own shapes
# ---------------------------------------------------------------------------
def test_native_matches_numpy_oracle_on_tiny_step(N):
    """The full tiny COPY step: all probe losses, coefficients and the update."""
    cfg = W.CONFIGS["tiny"]
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg)
    seed = W.step_seed(0)
    lp, lm = N.probe_losses(theta, spec, seed, cfg.n_pert, cfg.eps, tok, tgt)
    olp, olm = O.probe_losses(theta, spec, seed, cfg.n_pert, cfg.eps, tok, tgt)
    assert np.allclose(lp, olp, rtol=1e-13) and np.allclose(lm, olm, rtol=1e-13)
    c = N.coefficients(lp, lm, cfg.n_pert, cfg.eps, cfg.eta)
    assert np.allclose(c, O.coefficients(olp, olm, cfg.n_pert, cfg.eps, cfg.eta), rtol=1e-9)
    assert np.allclose(N.update(theta, spec, seed, cfg.n_pert, c),
                       O.update(theta, spec, seed, cfg.n_pert, c), rtol=0, atol=1e-15)
    assert math.isclose(N.loss_at(theta, spec, tok, tgt), O.loss_at(theta, spec, tok, tgt),
                        rel_tol=1e-13)


def test_native_matches_numpy_oracle_on_row_slices(N):
    """Row subsets of a Markov batch on a 2-layer bf16-sized shape (probes
    taken out of order; each row's forward is independent of the others)."""
    cfg = W.small_config(vocab=50, embed=64, hidden=64, layers=2)
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg, seed=1)
    tok, tgt = W.markov_batch(40, 4, step=0, vocab=50)
    rows = np.array([3, 0, 39, 17])
    seed = W.step_seed(3)
    a = N.probe_losses(theta, spec, seed, 9, 1e-3, tok, tgt, probes=[8, 2], rows=rows,
                       return_rows=True)
    b = O.probe_losses(theta, spec, seed, 9, 1e-3, tok, tgt, probes=[8, 2], rows=rows,
                       return_rows=True)
    for x, y in zip(a, b):
        assert np.allclose(x, y, rtol=1e-13, atol=1e-13)


def test_native_rejects_out_of_range_inputs(N):
    cfg = W.CONFIGS["tiny"]
    spec = (cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    theta = W.init_theta(cfg)
    tok, tgt = W.batch_for(cfg)
    bad = tok.copy()
    bad[0, 0] = cfg.vocab
    with pytest.raises(ValueError):
        N.probe_losses(theta, spec, 1, 2, 1e-3, bad, tgt)
    badt = tgt.copy()
    badt[1, 3] = -2
    with pytest.raises(ValueError):
        N.probe_losses(theta, spec, 1, 2, 1e-3, tok, badt)
    with pytest.raises(ValueError):
        N.probe_losses(theta[:-1], spec, 1, 2, 1e-3, tok, tgt)


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------
MUTATIONS = {
    "swap_i_f_gates": ("const double ig = sigmoid(g[u]);\n          const double fg = sigmoid(g[H + u]);",
                       "const double ig = sigmoid(g[H + u]);\n          const double fg = sigmoid(g[u]);"),
    "drop_cell_bias": ("G[(size_t)b * 4 * H + r] = acc[b] + bias;", "G[(size_t)b * 4 * H + r] = acc[b];"),
    "no_recurrent_input": ("a[(size_t)(in + k) * nb + b] = h[l][(size_t)b * H + k];",
                           "a[(size_t)(in + k) * nb + b] = 0.0;"),
    "philox_no_key_bump": ("key0 += 0x9E3779B9u;", ""),
    "philox_swapped_multipliers": ("(uint64_t)0xD2511F53u * x[0]", "(uint64_t)0xCD9E8D57u * x[0]"),
    "plain_bit_order": ("return (e >> 1) + 16 * (e & 1);", "return e;"),
    "missing_factor_two": ("/ (2.0 * (double)eps * n)", "/ ((double)eps * n)"),
    "wrong_update_sign": ("out[j0 - j0_all + k] -= coeffs[i] * p[k];",
                          "out[j0 - j0_all + k] += coeffs[i] * p[k];"),
    "perturb_ignores_sign": ("const double step[2] = {s_eps, -s_eps};",
                             "const double step[2] = {s_eps, s_eps};"),
    "lse_without_max": ("row_loss[b] += mx + std::log(se) - zb[tg];",
                        "row_loss[b] += std::log(se) - zb[tg];"),
    "gram_counts_padding": ("const int64_t n_real = std::min<int64_t>(128, len - qq * 128);",
                            "const int64_t n_real = 128;"),
}


def _mutant(name, tmpdir):
    old, new = MUTATIONS[name]
    src = open(native.SRC).read()
    assert src.count(old) == 1, name
    path = os.path.join(tmpdir, f"{name}.cpp")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmpdir, f"{name}.so")
    native.build(force=True, src=path, out=so)
    return native.Oracle(native.load(so, rebuild=False))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_native_pins_catch_planted_mistake(name):
    with tempfile.TemporaryDirectory() as d:
        mod = _mutant(name, d)
        caught = []
        for pin in PINS:
            try:
                with np.errstate(all="ignore"):
                    pin(mod)
            except Exception:
                caught.append(pin.__name__)
        assert caught, f"no pin caught mutation {name}"


def test_native_unmutated_copy_builds_and_passes():
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "copy.cpp")
        with open(path, "w") as f:
            f.write(open(native.SRC).read())
        so = os.path.join(d, "copy.so")
        native.build(force=True, src=path, out=so)
        mod = native.Oracle(native.load(so, rebuild=False))
        for pin in PINS:
            pin(mod)
