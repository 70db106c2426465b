"""Training on the transduction tasks with CD-RGE through the C ABI.

The pages train small recurrent models on COPY-style transduction tasks with
zero-order updates only (alex-wiki, "Evidence And Limits": training on short
sequences, evaluation on longer ones) and sweep the step size against the
perturbation radius (pith.science review, "Referee Report": eta and eps).
This driver runs that loop on one GPU: every step draws a fresh batch of
lengths 1..max_len, calls zo_probe_losses / zo_coeffs / zo_update (the
probes are replayed from the step seed, never stored), and records the loss
at theta estimated as the mean of (L+ + L-)/2 over the probes (O(eps^2) from
L(theta)).  After training, each evaluation length is scored by zo_loss, the
unperturbed forward.

    python -m zero_order_recurrent_b200.train --task copy --steps 2000 --eta 0.05
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np


def _repo_root():
    return os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def train(task: str = "copy", steps: int = 1000, n_pert: int = 64, eps: float = 1e-3,
          eta: float = 1e-3, batch: int = 8, max_len: int = 10, eval_lengths=(11, 20, 40, 60),
          embed: int = 16, hidden: int = 32, layers: int = 1, seed: int = 0,
          log_every: int = 100, theta=None, estimator: str = "central", start_step: int = 0,
          checkpoint: str = None, checkpoint_every: int = 0):
    """Runs zero-order updates start_step .. steps-1; returns the loss history,
    the evaluation losses per length, the device time per step and the final
    theta (device).  Each step's batch and probes depend only on (seed, step),
    so a run resumed from a checkpoint (theta and start_step, see
    checkpoint.py) repeats the uninterrupted run exactly; with `checkpoint`
    set, theta and the next step are saved every `checkpoint_every` steps and
    at the end.
    estimator "central": c_i = eta (L+_i - L-_i)/(2 eps n) (CD-RGE);
    "forward": c_i = eta (L+_i - L(theta))/(eps n) with L(theta) from zo_loss."""
    if estimator not in ("central", "forward"):
        raise ValueError(f"unknown estimator {estimator}")
    import torch
    if _repo_root() not in sys.path:
        sys.path.insert(0, _repo_root())
    import workloads as W
    import zero_order_recurrent_b200 as zo

    V = 10
    T_train = W.task_length(task, max_len)
    T_eval = max([W.task_length(task, L) for L in eval_lengths] + [T_train])
    cfg = W.small_config(vocab=V, embed=embed, hidden=hidden, layers=layers)
    if theta is None:
        theta = torch.from_numpy(W.init_theta(cfg)).cuda()
    dev = theta.device
    lp = torch.empty(n_pert, device=dev)
    lm = torch.empty(n_pert, device=dev)
    coef = torch.empty(n_pert, device=dev)
    l0 = torch.empty(1, device=dev)
    from zero_order_recurrent_b200 import checkpoint as ckpt
    history = []
    ms = 0.0
    with zo.Context(V, embed, hidden, layers, "f32", batch, T_eval, 0) as ctx:
        for step in range(start_step, steps):
            lengths = np.random.default_rng((seed, 7, step)).integers(1, max_len + 1, size=batch)
            tok, tgt = W.transduction_batch(task, lengths, T_train, seed=seed * 1000003 + step)
            tok_d = torch.from_numpy(tok).to(dev)
            tgt_d = torch.from_numpy(tgt).to(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            sseed = W.step_seed(step, run_seed=seed)
            if estimator == "central":
                zo.cdrge_step(ctx, theta, sseed, n_pert, eps, eta, tok_d, tgt_d, lp, lm, coef)
            else:
                zo.zo_loss(ctx, theta, tok_d, tgt_d, l0)
                zo.zo_probe_losses(ctx, theta, sseed, n_pert, eps, tok_d, tgt_d, lp, lm)
                zo.zo_coeffs_forward(ctx, lp, l0, n_pert, eps, eta, coef)
                zo.zo_update(ctx, theta, sseed, n_pert, coef)
            e1.record()
            if step % log_every == 0 or step == steps - 1:
                torch.cuda.synchronize()
                st = zo.zo_sync_status(ctx)
                if st != zo.ZO_OK:
                    raise RuntimeError(f"step {step}: {zo.status_string(st)}")
                history.append((step, float(((lp + lm) * 0.5).mean())))
            torch.cuda.synchronize()
            ms += e0.elapsed_time(e1)
            if checkpoint and ((checkpoint_every and (step + 1) % checkpoint_every == 0)
                               or step == steps - 1):
                ckpt.save(checkpoint, theta, step + 1, seed, task=task, n_pert=n_pert, eps=eps,
                          eta=eta, estimator=estimator)
        evals = {}
        for L in eval_lengths:
            tok, tgt = W.transduction_batch(task, [L] * batch, W.task_length(task, L),
                                            seed=seed * 1000003 + 10**9 + L)
            zo.zo_loss(ctx, theta, torch.from_numpy(tok).to(dev), torch.from_numpy(tgt).to(dev),
                       lp[:1])
            torch.cuda.synchronize()
            evals[int(L)] = float(lp[0])
        st = zo.zo_sync_status(ctx)
        if st != zo.ZO_OK:
            raise RuntimeError(f"evaluation: {zo.status_string(st)}")
    return {"task": task, "estimator": estimator, "steps": steps, "n_pert": n_pert, "eps": eps,
            "eta": eta,
            "max_len": max_len, "history": history, "eval": evals,
            "ms_per_step": ms / max(steps - start_step, 1), "theta": theta}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--task", default="copy", choices=["copy", "reverse", "add"])
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--n-pert", type=int, default=64)
    ap.add_argument("--eps", type=float, default=1e-3)
    ap.add_argument("--eta", type=float, nargs="+", default=[1e-3],
                    help="one or more step sizes (a sweep against eps)")
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--max-len", type=int, default=10)
    ap.add_argument("--eval-lengths", type=int, nargs="*", default=[11, 20, 40, 60])
    ap.add_argument("--hidden", type=int, default=32)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--log-every", type=int, default=100)
    ap.add_argument("--estimator", default="central", choices=["central", "forward"])
    ap.add_argument("--checkpoint", default=None, help="save theta and the next step here")
    ap.add_argument("--checkpoint-every", type=int, default=0)
    ap.add_argument("--resume", default=None, help="start from this checkpoint")
    args = ap.parse_args(argv)
    theta0, start = None, 0
    if args.resume:
        import torch

        from zero_order_recurrent_b200 import checkpoint as ckpt
        th, start, run_seed, _ = ckpt.load(args.resume)
        if run_seed != args.seed:
            raise SystemExit(f"checkpoint is of run seed {run_seed}, not {args.seed}")
        theta0 = torch.from_numpy(th).cuda()
    for eta in args.eta:
        r = train(task=args.task, steps=args.steps, n_pert=args.n_pert, eps=args.eps, eta=eta,
                  batch=args.batch, max_len=args.max_len, eval_lengths=args.eval_lengths,
                  hidden=args.hidden, seed=args.seed, log_every=args.log_every,
                  estimator=args.estimator, theta=None if theta0 is None else theta0.clone(),
                  start_step=start, checkpoint=args.checkpoint,
                  checkpoint_every=args.checkpoint_every)
        r.pop("theta")
        print(json.dumps(r), flush=True)


if __name__ == "__main__":
    main()
