"""ctypes binding of the plain C++17 fp64 oracle (``zo_oracle_cpu.cpp``).

TEST INFRASTRUCTURE ONLY, like the numpy oracle beside it: only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may use it.  The functions mirror the numpy oracle's
names and return values; the arithmetic is the C++ file's.  Threads default
to the CPUs this process may run on (``os.sched_getaffinity``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "zo_oracle_cpu.cpp")
LIB = os.path.join(HERE, "libzo_oracle.so")
CXXFLAGS = ["-O3", "-std=c++17", "-fPIC", "-shared", "-pthread"]

_lib = None


def build(force: bool = False, src: str = SRC, out: str = LIB) -> str:
    """Compile the C++ oracle with the host compiler (g++)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp"
    r = subprocess.run(["g++", *CXXFLAGS, src, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("g++ failed building the C++ oracle:\n" + r.stdout + r.stderr)
    os.replace(tmp, out)
    return out


def cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _declare(lib):
    P, I32, I64, U32, U64, F, D = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                   ctypes.c_uint64, ctypes.c_float, ctypes.c_double)
    sig = {
        "zoo_d_pad": ([I32, I32, I32, I32], I64),
        "zoo_philox4x32_10": ([U32, U32, U32, U32, U32, U32, P], None),
        "zoo_sign_words": ([U64, U32, U64, I64, P], None),
        "zoo_signs": ([U64, U32, I64, I64, P], None),
        "zoo_probe_row_losses": ([P, I32, I32, I32, I32, U64, P, I32, F, P, P, I32, I32, P, I32,
                                  I32, P, P], I32),
        "zoo_coefficients": ([P, P, I32, F, F, P], None),
        "zoo_coefficients_forward": ([P, D, I32, F, F, P], None),
        "zoo_update": ([P, I32, I32, I32, I32, U64, I32, P, P, I64, I32, P], I32),
        "zoo_update_range": ([P, I32, I32, I32, I32, U64, I32, P, I64, I64, I32, P], I32),
        "zoo_probe_gram": ([I32, I32, I32, I32, U64, P, I32, I32, P], I32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


def load(path: str = LIB, rebuild: bool = True):
    """Load (building first if missing or stale) the C++ oracle."""
    global _lib
    if _lib is not None and path == LIB:
        return _lib
    if rebuild and path == LIB:
        build()
    lib = _declare(ctypes.CDLL(path))
    if path == LIB:
        _lib = lib
    return lib


def _p(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


class Oracle:
    """The C++ oracle behind the numpy oracle's function names."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else load()

    def d_pad(self, spec):
        return int(self.lib.zoo_d_pad(*spec))

    def philox4x32_10(self, c0, c1, c2, c3, k0, k1):
        out = np.zeros(4, dtype=np.uint32)
        self.lib.zoo_philox4x32_10(c0, c1, c2, c3, k0, k1, _p(out))
        return tuple(int(x) for x in out)

    def sign_words(self, step_seed, probe, q_first, n_blocks):
        out = np.zeros((n_blocks, 4), dtype=np.uint32)
        self.lib.zoo_sign_words(step_seed, probe, q_first, n_blocks, _p(out))
        return out

    def probe_signs(self, step_seed, probe, j0, count):
        out = np.zeros(max(count, 0), dtype=np.int8)
        if count > 0:
            self.lib.zoo_signs(step_seed, probe, j0, count, _p(out))
        return out

    def _theta(self, theta, spec):
        th = np.ascontiguousarray(theta, dtype=np.float32)
        if th.shape != (self.d_pad(spec),):
            raise ValueError(f"theta has shape {th.shape}, the spec needs ({self.d_pad(spec)},)")
        return th

    def probe_row_losses(self, theta, spec, step_seed, probes, eps, tokens, targets, rows=None,
                         threads=None):
        """Row sums [len(probes), 2, n_rows] of the cross-entropy over scored
        steps, and the scored counts [n_rows]."""
        V, E, H, L = spec
        th = self._theta(theta, spec)
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        tgt = np.ascontiguousarray(targets, dtype=np.int32)
        B, T = tok.shape
        pr = np.ascontiguousarray(list(probes), dtype=np.int32)
        rw = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
        nb = B if rw is None else len(rw)
        rl = np.zeros((len(pr), 2, nb))
        rc = np.zeros(nb, dtype=np.int64)
        st = self.lib.zoo_probe_row_losses(_p(th), V, E, H, L, step_seed, _p(pr), len(pr), eps,
                                           _p(tok), _p(tgt), B, T, _p(rw), nb,
                                           threads or cores(), _p(rl), _p(rc))
        if st == 2:
            raise ValueError("token or target out of range")
        if st != 0:
            raise ValueError("bad arguments to the C++ oracle")
        return rl, rc

    def probe_losses(self, theta, spec, step_seed, n_pert, eps, tokens, targets, probes=None,
                     rows=None, return_rows=False, threads=None):
        probes = list(range(n_pert)) if probes is None else list(probes)
        rl, rc = self.probe_row_losses(theta, spec, step_seed, probes, eps, tokens, targets, rows,
                                       threads)
        n = int(rc.sum())
        lp = rl[:, 0].sum(axis=1) / n if n > 0 else np.zeros(len(probes))
        lm = rl[:, 1].sum(axis=1) / n if n > 0 else np.zeros(len(probes))
        if return_rows:
            return lp, lm, rl[:, 0], rl[:, 1]
        return lp, lm

    def loss_at(self, theta, spec, tokens, targets, threads=None):
        rl, rc = self.probe_row_losses(theta, spec, 0, [0], 0.0, tokens, targets, None, threads)
        n = int(rc.sum())
        return float(rl[0, 0].sum() / n) if n > 0 else 0.0

    def coefficients(self, loss_plus, loss_minus, n_pert, eps, eta):
        lp = np.ascontiguousarray(loss_plus, dtype=np.float64)
        lm = np.ascontiguousarray(loss_minus, dtype=np.float64)
        out = np.zeros(len(lp))
        self.lib.zoo_coefficients(_p(lp), _p(lm), n_pert, eps, eta, _p(out))
        return out

    def coefficients_forward(self, loss_plus, loss0, n_pert, eps, eta):
        lp = np.ascontiguousarray(loss_plus, dtype=np.float64)
        out = np.zeros(len(lp))
        self.lib.zoo_coefficients_forward(_p(lp), float(loss0), n_pert, eps, eta, _p(out))
        return out

    def update(self, theta, spec, step_seed, n_pert, coeffs, threads=None):
        V, E, H, L = spec
        th = self._theta(theta, spec)
        c = np.ascontiguousarray(coeffs, dtype=np.float64)
        out = np.zeros(th.size)
        if self.lib.zoo_update(_p(th), V, E, H, L, step_seed, n_pert, _p(c), None, 0,
                               threads or cores(), _p(out)):
            raise ValueError("bad arguments to the C++ oracle")
        return out

    def update_range(self, theta, spec, step_seed, n_pert, coeffs, j0, j1, threads=None):
        """theta' on the contiguous elements j0 <= j < j1."""
        V, E, H, L = spec
        th = self._theta(theta, spec)
        c = np.ascontiguousarray(coeffs, dtype=np.float64)
        out = np.zeros(max(j1 - j0, 0))
        if self.lib.zoo_update_range(_p(th), V, E, H, L, step_seed, n_pert, _p(c), j0, j1,
                                     threads or cores(), _p(out)):
            raise ValueError("bad arguments to the C++ oracle")
        return out

    def update_at(self, theta, spec, step_seed, n_pert, coeffs, index, threads=None):
        V, E, H, L = spec
        th = self._theta(theta, spec)
        c = np.ascontiguousarray(coeffs, dtype=np.float64)
        idx = np.ascontiguousarray(index, dtype=np.int64)
        out = np.zeros(idx.size)
        if self.lib.zoo_update(_p(th), V, E, H, L, step_seed, n_pert, _p(c), _p(idx), idx.size,
                               threads or cores(), _p(out)):
            raise ValueError("bad arguments to the C++ oracle")
        return out

    def probe_gram(self, spec, step_seed, probes, threads=None):
        V, E, H, L = spec
        pr = np.ascontiguousarray(list(probes), dtype=np.int32)
        G = np.zeros((len(pr), len(pr)))
        if self.lib.zoo_probe_gram(V, E, H, L, step_seed, _p(pr), len(pr), threads or cores(),
                                   _p(G)):
            raise ValueError("bad arguments to the C++ oracle")
        return G
