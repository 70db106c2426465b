"""fp64 CPU oracle for central-difference random-vector gradient estimation
(CD-RGE) on multi-layer LSTMs.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never calls it, and it shares no code with the library.

Two independent implementations of the same method live in this package: the
plain C++17 one (``zo_oracle_cpu.cpp`` via ``native.py``), which the
full-size GPU parity gates and the timed CPU baseline use, and this numpy one,
written separately, which pins the C++ one (the two must agree to rounding)
and serves the small GPU parity cases and the estimator-algebra pins.

Sources ("Scaling Recurrent Neural Networks to a Billion Parameters with
Zero-Order Optimization", Chaubard & Kochenderfer, arXiv 2505.17852):

* pith.science review, "What carries the argument": the update
      Theta' = Theta - 1/(2 n_pert) * sum_i (L(Theta + eps p_i) - L(Theta - eps p_i)) p_i
  with Rademacher p_i in {-1,+1}^d and the step size tied to eps (eta = eps).
* alex-wiki source page, "Method": the estimator
      g_hat = 1/K * sum_i (L(theta + eps u_i) - L(theta - eps u_i)) / (2 eps) * u_i,
  with Rademacher directions, reconstructible random seeds and chunked
  perturbations.  The update is theta - eta * g_hat, which is the review's
  formula when eta = eps.
* pith.science review, "Assumptions": E[p] = 0 and E[p p^T] = I.

Readings where the pages are silent:

1. Model: textbook LSTM, gate blocks in the order i, f, g, o, one bias per
   layer, h0 = c0 = 0, no forget-gate offset; token embedding in front and a
   linear output layer on top of the last layer.
2. Loss: natural-log softmax cross-entropy from the top layer at every
   timestep, averaged over every (row, step) whose target is >= 0.
3. Every parameter is perturbed (embedding, weights, biases, output layer);
   the zero padding between segments is not a parameter.
4. Probe signs ("reconstructible random seeds"): Philox4x32-10 (Salmon,
   Moraes, Dror & Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11)
   with key = (seed lo, seed hi) and counter = (q lo, q hi, probe, 0) for the
   128-element block q = j >> 7.  Element j reads output word (j >> 5) & 3,
   at bit position (e >> 1) + 16 * (e & 1) with e = j & 31, so elements 2m and
   2m+1 of a word sit at bits m and m + 16.  Bit 0 gives p = +1, bit 1 gives
   p = -1.
5. eps is an fp32 value; the oracle promotes exactly that value to double.
6. With no scored target the loss is defined as 0.

Every floating-point computation here is fp64.  Parity: pinned (see the
``-m "not gpu"`` tests under tests/ for what pins each function).
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# Philox4x32-10 (SC'11, Philox-4x32 with 10 rounds)
# ---------------------------------------------------------------------------
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_M32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32-10 block function on arrays (or scalars) of uint32 values.

    One round maps (c0, c1, c2, c3) with key (k0, k1) to
        (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0));
    the key is bumped by the Weyl constants (W0, W1) between rounds.
    Returns four uint32 arrays.
    """
    c0 = np.asarray(c0, dtype=np.uint64) & _M32
    c1 = np.asarray(c1, dtype=np.uint64) & _M32
    c2 = np.asarray(c2, dtype=np.uint64) & _M32
    c3 = np.asarray(c3, dtype=np.uint64) & _M32
    k0 = int(k0) & 0xFFFFFFFF
    k1 = int(k1) & 0xFFFFFFFF
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + PHILOX_W0) & 0xFFFFFFFF
            k1 = (k1 + PHILOX_W1) & 0xFFFFFFFF
        p0 = c0 * np.uint64(PHILOX_M0)
        p1 = c2 * np.uint64(PHILOX_M1)
        hi0, lo0 = p0 >> np.uint64(32), p0 & _M32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _M32
        c0, c1, c2, c3 = hi1 ^ c1 ^ np.uint64(k0), lo1, hi0 ^ c3 ^ np.uint64(k1), lo0
    return tuple(x.astype(np.uint32) for x in (c0, c1, c2, c3))


def sign_words(step_seed: int, probe: int, q_first: int, n_blocks: int) -> np.ndarray:
    """Philox output words [n_blocks, 4] for blocks q_first.. of one probe."""
    q = np.arange(q_first, q_first + n_blocks, dtype=np.uint64)
    k0 = step_seed & 0xFFFFFFFF
    k1 = (step_seed >> 32) & 0xFFFFFFFF
    w = philox4x32_10(q & _M32, q >> np.uint64(32), np.uint64(probe), np.uint64(0), k0, k1)
    return np.stack(w, axis=1)


# element e (0..31) of a word reads bit position (e >> 1) + 16 * (e & 1)
_BITPOS = np.array([(e >> 1) + 16 * (e & 1) for e in range(32)], dtype=np.int64)


def probe_signs(step_seed: int, probe: int, j0: int, count: int) -> np.ndarray:
    """Rademacher signs p_{probe, j} for j in [j0, j0 + count), as int8 +-1."""
    if count <= 0:
        return np.zeros(0, dtype=np.int8)
    q0 = j0 >> 7
    q1 = (j0 + count - 1) >> 7
    words = sign_words(step_seed, probe, q0, q1 - q0 + 1)          # [nq, 4] uint32
    bits = np.unpackbits(words.view(np.uint8).reshape(-1, 4, 4), axis=2, bitorder="little")
    bits = bits.reshape(-1, 4, 32)[:, :, _BITPOS].reshape(-1)       # element order
    start = j0 - (q0 << 7)
    b = bits[start:start + count].astype(np.int8)
    return (1 - 2 * b).astype(np.int8)


# ---------------------------------------------------------------------------
# Parameter layout
# ---------------------------------------------------------------------------
def layout(vocab: int, embed: int, hidden: int, layers: int):
    """Segments of the flat parameter vector as a list of
    (name, rows, cols, offset), plus the padded length.  Order: E[V x E];
    per layer W_l[4H x (in_l + H)], b_l[4H]; W_out[V x H]; b_out[V].  Each
    segment starts on a multiple of 128 elements."""
    segs = []
    off = 0
    shapes = [("E", vocab, embed)]
    for l in range(layers):
        in_l = embed if l == 0 else hidden
        shapes.append((f"W{l + 1}", 4 * hidden, in_l + hidden))
        shapes.append((f"b{l + 1}", 1, 4 * hidden))
    shapes.append(("Wout", vocab, hidden))
    shapes.append(("bout", 1, vocab))
    for name, r, c in shapes:
        segs.append((name, r, c, off))
        off += r * c
        off = -(-off // 128) * 128
    return segs, off


def real_mask(vocab, embed, hidden, layers) -> np.ndarray:
    """Boolean [d_pad]: True where the element is a parameter (not padding)."""
    segs, d_pad = layout(vocab, embed, hidden, layers)
    m = np.zeros(d_pad, dtype=bool)
    for _, r, c, off in segs:
        m[off:off + r * c] = True
    return m


def unpack(theta: np.ndarray, vocab, embed, hidden, layers) -> dict:
    """Views of the flat vector as the model's matrices (fp64 copies)."""
    segs, d_pad = layout(vocab, embed, hidden, layers)
    assert theta.shape[-1] == d_pad
    out = {}
    for name, r, c, off in segs:
        a = np.asarray(theta[off:off + r * c], dtype=np.float64)
        out[name] = a.reshape(c) if r == 1 else a.reshape(r, c)
    return out


# ---------------------------------------------------------------------------
# Forward pass and loss
# ---------------------------------------------------------------------------
def _sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def lstm_row_losses(P: dict, layers: int, tokens: np.ndarray, targets: np.ndarray):
    """Forward of embedding -> `layers` LSTM layers -> linear -> softmax CE.

    Returns (per-row sum of CE over scored steps [B], per-row scored count [B]).
    Cell: G = [x_t | h_{t-1}] W^T + b; i, f, o = sigmoid; g = tanh on the gate
    blocks [i | f | g | o]; c_t = f*c_{t-1} + i*g; h_t = o*tanh(c_t).
    """
    B, T = tokens.shape
    H = P["b1"].shape[0] // 4
    h = [np.zeros((B, H)) for _ in range(layers)]
    c = [np.zeros((B, H)) for _ in range(layers)]
    loss = np.zeros(B)
    count = np.zeros(B, dtype=np.int64)
    rows = np.arange(B)
    for t in range(T):
        x = P["E"][tokens[:, t]]
        for l in range(layers):
            W = P[f"W{l + 1}"]
            G = np.concatenate([x, h[l]], axis=1) @ W.T + P[f"b{l + 1}"]
            i = _sigmoid(G[:, 0:H])
            f = _sigmoid(G[:, H:2 * H])
            g = np.tanh(G[:, 2 * H:3 * H])
            o = _sigmoid(G[:, 3 * H:4 * H])
            c[l] = f * c[l] + i * g
            h[l] = o * np.tanh(c[l])
            x = h[l]
        logits = x @ P["Wout"].T + P["bout"]
        m = logits.max(axis=1, keepdims=True)
        lse = m[:, 0] + np.log(np.exp(logits - m).sum(axis=1))
        tgt = targets[:, t]
        valid = tgt >= 0
        ce = lse - logits[rows, np.where(valid, tgt, 0)]
        loss += np.where(valid, ce, 0.0)
        count += valid
    return loss, count


def mean_loss(row_loss, row_count) -> float:
    n = int(np.sum(row_count))
    return float(np.sum(row_loss) / n) if n > 0 else 0.0


def perturbed(theta: np.ndarray, spec, step_seed: int, probe: int, sign: float, eps: float,
              probe_scale: int = 1) -> np.ndarray:
    """theta + sign * eps * p_probe over every parameter (padding stays 0), fp64.

    `probe_scale` = -1 replaces p by -p (used to test antisymmetry)."""
    V, E, H, L = spec
    segs, d_pad = layout(V, E, H, L)
    out = np.zeros(d_pad, dtype=np.float64)
    e = float(np.float32(eps))
    chunk = 1 << 22
    for _, r, c, off in segs:
        n = r * c
        for a in range(0, n, chunk):
            m = min(chunk, n - a)
            p = probe_signs(step_seed, probe, off + a, m).astype(np.float64) * probe_scale
            out[off + a:off + a + m] = theta[off + a:off + a + m].astype(np.float64) + sign * e * p
    return out


def probe_losses(theta, spec, step_seed, n_pert, eps, tokens, targets, probes=None,
                 rows=None, probe_scale=1, return_rows=False):
    """L(theta + eps p_i) and L(theta - eps p_i) for each probe i.

    pith.science review, "What carries the argument": each probe needs two
    complete forwards at the two perturbed points.  `probes` selects a subset
    of probe indices (default all n_pert) and `rows` a subset of batch rows;
    the probe signs depend only on (step_seed, i), never on the subset.
    """
    V, E, H, L = spec
    probes = list(range(n_pert)) if probes is None else list(probes)
    tok = tokens if rows is None else tokens[rows]
    tgt = targets if rows is None else targets[rows]
    lp, lm, rp, rm = [], [], [], []
    for i in probes:
        for sgn, acc, racc in ((+1.0, lp, rp), (-1.0, lm, rm)):
            th = perturbed(theta, spec, step_seed, i, sgn, eps, probe_scale)
            P = unpack(th, V, E, H, L)
            del th
            rl, rc = lstm_row_losses(P, L, tok, tgt)
            acc.append(mean_loss(rl, rc))
            racc.append(rl)
    if return_rows:
        return np.array(lp), np.array(lm), np.array(rp), np.array(rm)
    return np.array(lp), np.array(lm)


def loss_at(theta, spec, tokens, targets) -> float:
    """L(theta), unperturbed."""
    V, E, H, L = spec
    P = unpack(np.asarray(theta, dtype=np.float64), V, E, H, L)
    rl, rc = lstm_row_losses(P, L, tokens, targets)
    return mean_loss(rl, rc)


# ---------------------------------------------------------------------------
# Coefficients and update
# ---------------------------------------------------------------------------
def coefficients(loss_plus, loss_minus, n_pert: int, eps: float, eta: float) -> np.ndarray:
    """c_i = eta * (L+_i - L-_i) / (2 eps n_pert).

    alex-wiki "Method": theta' = theta - eta * g_hat with
    g_hat = 1/K sum_i (L+_i - L-_i)/(2 eps) u_i, i.e. theta' = theta - sum_i c_i u_i.
    With eta = eps this is the review's 1/(2 n_pert) (L+ - L-) factor."""
    lp = np.asarray(loss_plus, dtype=np.float64)
    lm = np.asarray(loss_minus, dtype=np.float64)
    e = float(np.float32(eps))
    h = float(np.float32(eta))
    return h * (lp - lm) / (2.0 * e * n_pert)


def coefficients_forward(loss_plus, loss0, n_pert: int, eps: float, eta: float) -> np.ndarray:
    """Forward-difference coefficients c_i = eta * (L+_i - L0) / (eps n_pert),
    L0 = L(theta): the one-sided estimator g_hat = 1/n sum_i (L(theta + eps u_i)
    - L(theta))/eps u_i.  Over an antithetic set {u_i, -u_i} it equals the
    central difference (pith.science review, "Circularity Check": the
    Appendix C identity)."""
    lp = np.asarray(loss_plus, dtype=np.float64)
    e = float(np.float32(eps))
    h = float(np.float32(eta))
    return h * (lp - float(loss0)) / (e * n_pert)


def update_with_probes(theta, probes: np.ndarray, coeffs) -> np.ndarray:
    """theta' = theta - sum_i c_i p_i with explicit probe vectors [n, d]."""
    th = np.asarray(theta, dtype=np.float64)
    return th - np.asarray(coeffs, dtype=np.float64) @ np.asarray(probes, dtype=np.float64)


def update(theta, spec, step_seed: int, n_pert: int, coeffs) -> np.ndarray:
    """theta' = theta - sum_i c_i p_i with p_i replayed from (step_seed, i)
    (review, "What carries the argument"; alex-wiki "reconstructible random
    seeds").  Padding is left unchanged."""
    V, E, H, L = spec
    segs, d_pad = layout(V, E, H, L)
    th = np.asarray(theta, dtype=np.float64).copy()
    c = np.asarray(coeffs, dtype=np.float64)
    for _, r, cc, off in segs:
        n = r * cc
        acc = np.zeros(n)
        for i in range(n_pert):
            acc += c[i] * probe_signs(step_seed, i, off, n)
        th[off:off + n] -= acc
    return th


def estimate(loss_plus, loss_minus, eps, probes: np.ndarray) -> np.ndarray:
    """g_hat = 1/K sum_i (L+_i - L-_i)/(2 eps) u_i (alex-wiki "Method")."""
    lp = np.asarray(loss_plus, dtype=np.float64)
    lm = np.asarray(loss_minus, dtype=np.float64)
    K = len(lp)
    return ((lp - lm) / (2.0 * float(np.float32(eps)) * K)) @ np.asarray(probes, dtype=np.float64)


def coordinate_cd_gradient(loss_fn, theta, eps, index=None) -> np.ndarray:
    """Brute-force coordinate central differences
    g_j = (L(theta + eps e_j) - L(theta - eps e_j)) / (2 eps)."""
    th = np.asarray(theta, dtype=np.float64)
    idx = range(th.size) if index is None else index
    g = np.zeros(th.size)
    for j in idx:
        a = th.copy()
        a[j] += eps
        b = th.copy()
        b[j] -= eps
        g[j] = (loss_fn(a) - loss_fn(b)) / (2.0 * eps)
    return g


def probe_matrix(spec, step_seed: int, n_pert: int) -> np.ndarray:
    """All probes as an int8 matrix [n_pert, d_pad] (padding columns 0)."""
    V, E, H, L = spec
    segs, d_pad = layout(V, E, H, L)
    P = np.zeros((n_pert, d_pad), dtype=np.int8)
    for i in range(n_pert):
        for _, r, c, off in segs:
            P[i, off:off + r * c] = probe_signs(step_seed, i, off, r * c)
    return P


def gram_cosine(c_a, c_b, gram) -> float:
    """cos(sum_i a_i p_i, sum_i b_i p_i) from the probe Gram matrix G_ik = p_i . p_k."""
    a = np.asarray(c_a, dtype=np.float64)
    b = np.asarray(c_b, dtype=np.float64)
    num = a @ gram @ b
    den = math.sqrt(max(a @ gram @ a, 0.0) * max(b @ gram @ b, 0.0))
    return float(num / den) if den > 0 else 0.0


def probe_gram(spec, step_seed: int, probes) -> np.ndarray:
    """p_i . p_k over the real parameters, via popcount of the sign differences."""
    V, E, H, L = spec
    segs, _ = layout(V, E, H, L)
    probes = list(probes)
    n = len(probes)
    G = np.zeros((n, n))
    for _, r, c, off in segs:
        cnt = r * c
        S = np.stack([probe_signs(step_seed, i, off, cnt).astype(np.int64) for i in probes])
        G += S @ S.T
    return G


def signs_at(step_seed: int, probe: int, index) -> np.ndarray:
    """p_{probe, j} for an arbitrary array of element indices j (int8 +-1)."""
    j = np.asarray(index, dtype=np.int64)
    q = (j >> 7).astype(np.uint64)
    k0 = step_seed & 0xFFFFFFFF
    k1 = (step_seed >> 32) & 0xFFFFFFFF
    w = np.stack(philox4x32_10(q & _M32, q >> np.uint64(32), np.uint64(probe), np.uint64(0), k0, k1),
                 axis=-1)
    word = w[np.arange(j.size), (j >> 5) & 3]
    bit = (word >> _BITPOS[j & 31].astype(np.uint32)) & np.uint32(1)
    return (1 - 2 * bit.astype(np.int8)).astype(np.int8)


def update_at(theta, step_seed: int, n_pert: int, coeffs, index) -> np.ndarray:
    """theta'_j = theta_j - sum_i c_i p_ij at the given (parameter) indices only."""
    j = np.asarray(index, dtype=np.int64)
    c = np.asarray(coeffs, dtype=np.float64)
    acc = np.zeros(j.size)
    for i in range(n_pert):
        acc += c[i] * signs_at(step_seed, i, j)
    return np.asarray(theta, dtype=np.float64)[j] - acc
