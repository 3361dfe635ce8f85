"""Host-side schedules of the optimizer's scalar hyper-parameters.

* Momentum warm-up (modded-nanogpt 2024-11-10 record write-up, section
  "核心改动二学习率翻倍"): over the first `steps` steps the Muon momentum
  moves linearly from `start` to `end`; frac = min(step / steps, 1),
  mu = (1 - frac) start + frac end (500 steps, 0.85 -> 0.95 on the page).
* WSD learning-rate multiplier (Track 3 Aurora write-up, section on the
  hyper-parameter placement): flat at 1 for the first (1 - cooldown_frac)
  of training, then linear to 0 at the last step (cooldown_frac 0.7).
* Linear warm-down (2024-11-10 record write-up, hyper-parameter table):
  flat for num_iterations - warmdown_iters steps, then linear to 0.

These run on the host and produce the per-step scalars passed to the
library; they are plain functions of the step number.
"""
from __future__ import annotations


def momentum_warmup(step: int, steps: int = 500, start: float = 0.85, end: float = 0.95) -> float:
    frac = min(max(step, 0) / float(steps), 1.0) if steps > 0 else 1.0
    return (1.0 - frac) * start + frac * end


def wsd_multiplier(step: int, total_steps: int, cooldown_frac: float = 0.7) -> float:
    """1 during the stable phase, then linear decay reaching 0 at `total_steps`."""
    if total_steps <= 0:
        return 1.0
    x = min(max(step, 0) / float(total_steps), 1.0)
    if x < 1.0 - cooldown_frac:
        return 1.0
    return max((1.0 - x) / cooldown_frac, 0.0) if cooldown_frac > 0 else 0.0


def warmdown_multiplier(step: int, num_iterations: int, warmdown_iters: int, warmup_iters: int = 0) -> float:
    """Linear warm-up over warmup_iters, flat, then linear warm-down to 0 over the last warmdown_iters."""
    if warmup_iters > 0 and step < warmup_iters:
        return (step + 1) / float(warmup_iters)
    if step < num_iterations - warmdown_iters:
        return 1.0
    return max((num_iterations - step) / float(warmdown_iters), 0.0) if warmdown_iters > 0 else 0.0
