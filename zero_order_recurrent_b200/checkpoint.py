"""Checkpoint and resume of a CD-RGE run.

The state of a run is theta and the step counter.  Every probe of step s is
regenerated from (run seed, s) - the pages' "reconstructible random seeds"
(alex-wiki source page, "Method") - and the update keeps no moments, so a
checkpoint holds theta (fp32, the flat layout of include/zo.h), the next step
and the run seed, and a resumed run repeats the uninterrupted one bit for bit.
Files are written to a temporary name and renamed, so a crash mid-write
leaves the previous checkpoint intact.
"""
from __future__ import annotations

import json
import os

import numpy as np


def save(path: str, theta, step: int, run_seed: int, **meta) -> None:
    """Write theta (torch tensor or numpy array), the next step and the run seed."""
    th = theta.detach().cpu().numpy() if hasattr(theta, "detach") else np.asarray(theta)
    if th.dtype != np.float32 or th.ndim != 1:
        raise ValueError("theta must be a flat fp32 vector")
    tmp = path + ".tmp.npz"
    np.savez(tmp, theta=th, step=np.int64(step), run_seed=np.uint64(run_seed),
             meta=np.array(json.dumps(meta)))
    os.replace(tmp, path)


def load(path: str):
    """(theta fp32 numpy, next step, run seed, meta dict) from a checkpoint."""
    with np.load(path) as z:
        return (z["theta"].copy(), int(z["step"]), int(z["run_seed"]),
                json.loads(str(z["meta"])))
