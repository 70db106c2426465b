"""Seeded synthetic workloads for CD-RGE on multi-layer LSTMs.

This module only makes inputs: model shapes, initial parameters, token and
target arrays, and per-step seeds.  It holds none of the method's arithmetic
(no probe signs, no forward pass, no loss, no update), so that both the fp64
oracle under ``oracle/`` and the CUDA library can be fed the very same arrays
without sharing any computation.

Workload shapes follow "Scaling Recurrent Neural Networks to a Billion
Parameters with Zero-Order Optimization" as summarised on the pith.science
review and the alex-wiki source page ("Evidence And Limits"):

* tiny     - COPY transduction (train lengths up to 10), batch 8, 1-layer LSTM.
* overfit  - single-batch overfitting on one random length-100 sequence,
             batch 1, up to 512 perturbations per update.
* charlm / lstm270m / lstm1b - character-level language modelling with batch
             1024 and sequence length 10; Penn Treebank is replaced by a seeded
             first-order Markov chain with Dirichlet(0.1) rows over 50 symbols.

Everything is drawn from ``numpy.random.default_rng`` with fixed seeds.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

MASK64 = (1 << 64) - 1


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    vocab: int
    embed: int
    hidden: int
    layers: int
    dtype: str          # "f32" or "bf16" (bf16 operands, fp32 master parameters)
    batch: int
    seq: int            # input/target pairs per sequence
    n_pert: int
    eps: float
    eta: float
    task: str           # "copy", "overfit" or "markov"
    chunk: int = 0      # probes per pass on the GPU, 0 = library default


CONFIGS = {
    "tiny": Config("tiny", 10, 16, 32, 1, "f32", 8, 21, 8, 1e-3, 1e-3, "copy"),
    "overfit": Config("overfit", 50, 64, 128, 2, "f32", 1, 100, 512, 1e-3, 1e-3, "overfit"),
    "charlm": Config("charlm", 50, 256, 1024, 2, "bf16", 1024, 10, 64, 1e-3, 1e-3, "markov"),
    "lstm270m": Config("lstm270m", 50, 4096, 4096, 2, "bf16", 1024, 10, 32, 1e-3, 1e-3, "markov"),
    "lstm1b": Config("lstm1b", 50, 8192, 8192, 2, "bf16", 1024, 10, 16, 1e-3, 1e-3, "markov", 16),
    # the pages' single-device feasibility scale (~4.3B parameters, 17 GB fp32)
    "lstm4b": Config("lstm4b", 50, 16384, 16384, 2, "bf16", 1024, 10, 16, 1e-3, 1e-3, "markov", 16),
}

INIT_SEED = 1
RUN_SEED = 0


def segments(vocab: int, embed: int, hidden: int, layers: int):
    """Flat parameter layout: list of (name, rows, cols, offset).

    Order: embedding E[V x E]; per layer l: W_l[4H x (in_l + H)] (gate blocks
    i, f, g, o stacked by rows, columns [input | recurrent]), b_l[4H]; then the
    output projection W_out[V x H] and b_out[V].  Every segment starts on a
    multiple of 128 elements; the gaps are zero padding.
    """
    out = []
    off = 0

    def add(name, rows, cols):
        nonlocal off
        out.append((name, rows, cols, off))
        off += rows * cols
        off = (off + 127) // 128 * 128

    add("E", vocab, embed)
    for layer in range(layers):
        in_l = embed if layer == 0 else hidden
        add(f"W{layer + 1}", 4 * hidden, in_l + hidden)
        add(f"b{layer + 1}", 1, 4 * hidden)
    add("Wout", vocab, hidden)
    add("bout", 1, vocab)
    return out, off


def init_theta(cfg: Config, seed: int = INIT_SEED) -> np.ndarray:
    """Initial fp32 parameter vector (padding zero).

    The pages give no initialisation.  Embedding rows are N(0, 1); every LSTM
    and output weight and bias is U(-1/sqrt(H), 1/sqrt(H)), the usual LSTM
    default.
    """
    segs, d_pad = segments(cfg.vocab, cfg.embed, cfg.hidden, cfg.layers)
    rng = np.random.default_rng(seed)
    theta = np.zeros(d_pad, dtype=np.float32)
    bound = 1.0 / math.sqrt(cfg.hidden)
    for name, rows, cols, off in segs:
        n = rows * cols
        if name == "E":
            theta[off:off + n] = rng.standard_normal(n, dtype=np.float32)
        else:
            u = rng.random(n, dtype=np.float32)
            theta[off:off + n] = (2.0 * u - 1.0) * np.float32(bound)
    return theta


def splitmix64(x: int) -> int:
    """One SplitMix64 output for state x (Steele, Lea & Flood, OOPSLA 2014)."""
    z = (x + 0x9E3779B97F4A7C15) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def step_seed(step: int, run_seed: int = RUN_SEED) -> int:
    """Per-update probe seed; probes of step s are reproducible from (run_seed, s)."""
    return splitmix64((run_seed ^ step) & MASK64)


def copy_batch(batch: int = 8, length: int = 10, seed: int = 0):
    """COPY task: data digits 1..8, delimiter 9, blank 0.

    Input  = x_1..x_L, 9, 0 x L          (2L + 1 positions)
    Target = -1 x (L + 1), x_1..x_L      (-1 = position not scored)
    """
    rng = np.random.default_rng(seed)
    data = rng.integers(1, 9, size=(batch, length), dtype=np.int32)
    T = 2 * length + 1
    tokens = np.zeros((batch, T), dtype=np.int32)
    targets = np.full((batch, T), -1, dtype=np.int32)
    tokens[:, :length] = data
    tokens[:, length] = 9
    targets[:, length + 1:] = data
    return tokens, targets


def task_length(task: str, length: int) -> int:
    """Positions of one example of a transduction task with `length` data digits."""
    return 3 * length + 3 if task == "add" else 2 * length + 1


def transduction_batch(task: str, lengths, T: int, seed: int = 0):
    """One batch of a transduction task (the pages' COPY / REVERSE / ADD
    workloads; they give the lengths only, the formats are readings), each row
    padded with blanks (token 0, target -1) to T positions.

    Tokens: data digits 1..8, delimiter 9, blank 0; target -1 = not scored.
      copy:    x_1..x_L, 9, 0 x L        -> targets -1 x (L+1), x_1..x_L
      reverse: x_1..x_L, 9, 0 x L        -> targets -1 x (L+1), x_L..x_1
      add:     a_1..a_L, 9, b_1..b_L, 9, 0 x (L+1)  (base-8 digits, least
               significant first, token = digit + 1)
               -> targets -1 x (2L+2), then the L+1 digits of a + b
    """
    rng = np.random.default_rng(seed)
    lengths = np.asarray(lengths, dtype=np.int64)
    B = len(lengths)
    tokens = np.zeros((B, T), dtype=np.int32)
    targets = np.full((B, T), -1, dtype=np.int32)
    for r, L in enumerate(lengths):
        L = int(L)
        if task_length(task, L) > T:
            raise ValueError(f"{task} of length {L} needs {task_length(task, L)} > {T} positions")
        if task in ("copy", "reverse"):
            x = rng.integers(1, 9, size=L, dtype=np.int32)
            tokens[r, :L] = x
            tokens[r, L] = 9
            targets[r, L + 1:2 * L + 1] = x if task == "copy" else x[::-1]
        elif task == "add":
            a = rng.integers(0, 8, size=L)
            b = rng.integers(0, 8, size=L)
            tokens[r, :L] = a + 1
            tokens[r, L] = 9
            tokens[r, L + 1:2 * L + 1] = b + 1
            tokens[r, 2 * L + 1] = 9
            carry = 0
            for i in range(L + 1):
                s = carry + (int(a[i]) + int(b[i]) if i < L else 0)
                targets[r, 2 * L + 2 + i] = s % 8 + 1
                carry = s // 8
        else:
            raise ValueError(f"unknown task {task}")
    return tokens, targets


def overfit_batch(vocab: int = 50, length: int = 100, seed: int = 0):
    """One uniform random sequence of length+1 tokens, batch 1."""
    rng = np.random.default_rng(seed)
    seq = rng.integers(0, vocab, size=length + 1, dtype=np.int32)
    return seq[None, :-1].copy(), seq[None, 1:].copy()


def markov_transitions(vocab: int = 50, alpha: float = 0.1, seed: int = 1) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.dirichlet(np.full(vocab, alpha), size=vocab)


def markov_batch(batch: int, seq: int, step: int = 0, vocab: int = 50, seed: int = 1):
    """B rows of seq+1 tokens from the Markov chain; tokens = [:, :T], targets = [:, 1:]."""
    P = markov_transitions(vocab, seed=seed)
    cdf = np.cumsum(P, axis=1)
    cdf[:, -1] = 1.0
    rng = np.random.default_rng((seed, step))
    x = np.empty((batch, seq + 1), dtype=np.int32)
    x[:, 0] = rng.integers(0, vocab, size=batch)
    for t in range(1, seq + 1):
        u = rng.random(batch)
        rows = cdf[x[:, t - 1]]
        x[:, t] = np.minimum((u[:, None] > rows).sum(axis=1), vocab - 1)
    return x[:, :-1].copy(), x[:, 1:].copy()


def batch_for(cfg: Config, step: int = 0):
    if cfg.task == "copy":
        return copy_batch(cfg.batch, (cfg.seq - 1) // 2, seed=0)
    if cfg.task == "overfit":
        return overfit_batch(cfg.vocab, cfg.seq, seed=0)
    return markov_batch(cfg.batch, cfg.seq, step=step, vocab=cfg.vocab, seed=1)


def small_config(name="micro", vocab=7, embed=5, hidden=6, layers=1, batch=3, seq=4,
                 n_pert=4, dtype="f32"):
    """A toy model for tests."""
    return Config(name, vocab, embed, hidden, layers, dtype, batch, seq, n_pert, 1e-3, 1e-3, "markov")


def random_batch(batch: int, seq: int, vocab: int, seed: int = 0, ignore_frac: float = 0.0):
    """Uniform tokens and targets; a fraction of targets set to -1 (not scored)."""
    rng = np.random.default_rng(seed)
    tokens = rng.integers(0, vocab, size=(batch, seq), dtype=np.int32)
    targets = rng.integers(0, vocab, size=(batch, seq), dtype=np.int32)
    if ignore_frac > 0:
        targets[rng.random((batch, seq)) < ignore_frac] = -1
    return tokens, targets
