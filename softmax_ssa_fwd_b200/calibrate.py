"""Skip-softmax threshold calibration helpers (host side).

"Skip-Softmax Sparse Attention for Diffusion Models" (Model-Optimizer
examples/diffusers/sparsity README), intro and "Threshold Modes": a calibrated
exponential model gives ``scale_factor = a * exp(b * target_sparsity)``; the
backend turns it into the kernel threshold ``threshold = scale_factor / seq_k``
(the kernel then works with log2(threshold)); fitting in log space is
recommended when scale factors span orders of magnitude.  The config export
example on the same page prints a prefill fit ``a = 1443.49, b = 4.30``.

The mapping from the fitted scale factor to this library's lambda is the one
reading taken here: ``lambda = scale_factor / Lk``.

``sweep`` measures the achieved tile-skip fraction of the CUDA kernel for a
list of thresholds on given inputs (the pages' calibration uses real model
activations and a dataset; here any tensors can be passed), and ``fit_logspace``
fits ``(a, b)`` to (target sparsity, scale factor) pairs by least squares on
``log(scale_factor) = log(a) + b * sparsity``.
"""
from __future__ import annotations

import math
from typing import Iterable, Sequence

# Fixed-threshold default of the pages ("Threshold Modes", static lambda row).
DEFAULT_LAMBDA = 0.1
# Prefill fit printed in the config export example.
EXAMPLE_FIT = {"a": 1443.49, "b": 4.30}
# Threshold trials of the calibration ("Attention Sparsity for HuggingFace
# Models", custom configuration: optional ``threshold_trials``).
DEFAULT_TRIALS = (1e-4, 5e-4, 1e-3, 5e-3, 1e-2, 2e-2, 5e-2, 1e-1, 2e-1, 3e-1, 5e-1, 7e-1)


def scale_factor(a: float, b: float, target_sparsity: float) -> float:
    """scale_factor = a * exp(b * target_sparsity)."""
    return a * math.exp(b * target_sparsity)


def lambda_from_target(a: float, b: float, target_sparsity: float, seq_k: int) -> float:
    """Kernel threshold for a target sparsity: scale_factor / seq_k."""
    if seq_k <= 0:
        raise ValueError("seq_k must be positive")
    if not 0.0 <= target_sparsity <= 1.0:
        raise ValueError("target_sparsity must lie in [0, 1]")
    return scale_factor(a, b, target_sparsity) / seq_k


def fit_logspace(sparsities: Sequence[float], scale_factors: Sequence[float]) -> dict:
    """Least-squares fit of log(scale_factor) = log(a) + b * sparsity.

    Pairs with a non-positive scale factor are dropped.  Returns {"a", "b"}."""
    pts = [(float(s), math.log(float(f))) for s, f in zip(sparsities, scale_factors) if f > 0]
    if len(pts) < 2:
        raise ValueError("need at least two points with a positive scale factor")
    n = len(pts)
    mx = sum(s for s, _ in pts) / n
    my = sum(y for _, y in pts) / n
    sxx = sum((s - mx) ** 2 for s, _ in pts)
    if sxx == 0.0:
        raise ValueError("sparsities must not all be equal")
    b = sum((s - mx) * (y - my) for s, y in pts) / sxx
    return {"a": math.exp(my - b * mx), "b": b}


def sweep(q, k, v, lambdas: Iterable[float], *, causal: bool = True, Br: int = 128,
          Bc: int = 128, scale: float | None = None):
    """Achieved fraction of visited key tiles skipped by the CUDA kernel for each
    lambda, on the given bf16 CUDA tensors.  Returns [(lambda, fraction)]."""
    from . import ssa
    B, Lq, Hq, d = q.shape
    Lk = k.shape[1]
    visited = ssa.ssa_visited_tiles(causal, Lq, Lk, Br, Bc) * B * Hq
    out = []
    for lam in lambdas:
        _, _, cnt = ssa.attention(q, k, v, causal=causal, scale=scale, mode=ssa.MODE_SKIP,
                                  lam=float(lam), Br=Br, Bc=Bc)
        st = ssa.ssa_device_status()
        if st != ssa.SSA_OK:
            raise RuntimeError(ssa.status_string(st))
        out.append((float(lam), int(cnt.sum().item()) / visited))
    return out


def calibrate(q, k, v, target_sparsity: float, *, trials: Sequence[float] = DEFAULT_TRIALS,
              causal: bool = True, scale: float | None = None) -> dict:
    """Sweep the trials on (q, k, v), fit (a, b) in log space and return the fit
    with the lambda it gives for ``target_sparsity`` at this key length."""
    Lk = k.shape[1]
    pts = sweep(q, k, v, trials, causal=causal, scale=scale)
    fit = fit_from_sweep(pts, Lk)
    fit["lambda"] = lambda_from_target(fit["a"], fit["b"], target_sparsity, Lk)
    fit["points"] = pts
    return fit


def skip_enabled(step: int, initial_disabled_steps: int) -> bool:
    """Step gating of diffusion models: skip-softmax stays off (dense mode) for
    the first ``initial_disabled_steps`` denoising steps (the config example's
    ``initial_disabled_steps``)."""
    return step >= initial_disabled_steps


def skip_enabled_at_timestep(timestep: float, disabled_until_timestep: float | None) -> bool:
    """Timestep cutoff of diffusion models ("Refactor Skip Softmax Attention
    Interface", summary item 5: a normalized-timestep cutoff,
    ``disabled_until_timestep``).  The page names the knob only; the reading
    taken: the denoising timestep is normalized to [0, 1] and falls over the
    run, skip-softmax stays off while it is above the cutoff and is on from the
    first step at or below it.  ``None`` means no cutoff."""
    if not 0.0 <= timestep <= 1.0:
        raise ValueError("timestep must be normalized to [0, 1]")
    if disabled_until_timestep is None:
        return True
    if not 0.0 <= disabled_until_timestep <= 1.0:
        raise ValueError("disabled_until_timestep must lie in [0, 1]")
    return timestep <= disabled_until_timestep


def skip_phase(step: int, timestep: float | None = None, *, initial_disabled_steps: int = 0,
               disabled_until_timestep: float | None = None) -> bool:
    """True when a denoising step runs skip-softmax, False when it runs dense:
    both gates (step count and timestep cutoff) must let it through.  The phase
    decides the ``mode`` passed to the kernel, and a CUDA graph captured in one
    phase replays that phase, so captured graphs are keyed by it (the same page
    keys graphs by the resolved phase)."""
    if not skip_enabled(step, initial_disabled_steps):
        return False
    if timestep is None:
        if disabled_until_timestep is not None:
            raise ValueError("a timestep cutoff needs the step's timestep")
        return True
    return skip_enabled_at_timestep(timestep, disabled_until_timestep)


def fit_from_sweep(points: Sequence[tuple], seq_k: int) -> dict:
    """Fit (a, b) from sweep output: each lambda becomes a scale factor
    lambda * seq_k at its achieved sparsity; points with zero or full sparsity
    carry no information about the slope and are dropped."""
    use = [(s, lam * seq_k) for lam, s in points if 0.0 < s < 1.0]
    return fit_logspace([s for s, _ in use], [f for _, f in use])
