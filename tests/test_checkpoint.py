"""Checkpoint files of a CD-RGE run (CPU): theta, the next step and the run
seed round-trip exactly; a malformed theta is refused; a write replaces the
previous checkpoint only once it is complete."""
import os

import numpy as np
import pytest

import workloads as W
from zero_order_recurrent_b200 import checkpoint as ckpt


def test_round_trip(tmp_path):
    theta = W.init_theta(W.CONFIGS["tiny"])
    p = str(tmp_path / "c.npz")
    ckpt.save(p, theta, 17, (1 << 64) - 1, task="copy", eta=0.05)
    th, step, seed, meta = ckpt.load(p)
    assert th.dtype == np.float32 and np.array_equal(th, theta)
    assert step == 17 and seed == (1 << 64) - 1 and meta == {"task": "copy", "eta": 0.05}


def test_rejects_non_flat_or_non_fp32(tmp_path):
    p = str(tmp_path / "c.npz")
    with pytest.raises(ValueError):
        ckpt.save(p, np.zeros((2, 3), dtype=np.float32), 0, 0)
    with pytest.raises(ValueError):
        ckpt.save(p, np.zeros(6), 0, 0)
    assert not os.path.exists(p)


def test_overwrite_keeps_a_complete_file(tmp_path):
    p = str(tmp_path / "c.npz")
    ckpt.save(p, np.ones(8, dtype=np.float32), 1, 5)
    ckpt.save(p, np.full(8, 2.0, dtype=np.float32), 2, 5)
    th, step, _, _ = ckpt.load(p)
    assert step == 2 and np.all(th == 2.0)
    assert sorted(os.listdir(tmp_path)) == ["c.npz"]
