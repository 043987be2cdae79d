"""Calibration helpers: the pages' worked fit, the log-space fit, and (GPU) a
threshold sweep of the kernel on a stress input."""
import json
import math
import os

import pytest

from softmax_ssa_fwd_b200 import calibrate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "calibration_example.json")


def test_pages_example_fit():
    g = json.load(open(GOLDEN))
    sf = calibrate.scale_factor(g["a"], g["b"], g["target_sparsity"])
    assert sf == pytest.approx(g["scale_factor"], rel=1e-7)
    lam = calibrate.lambda_from_target(g["a"], g["b"], g["target_sparsity"], g["seq_k"])
    assert lam == pytest.approx(g["lambda"], rel=1e-6)
    assert calibrate.EXAMPLE_FIT == {"a": g["a"], "b": g["b"]}


def test_lambda_grows_with_target_and_shrinks_with_length():
    a, b = 1443.49, 4.30
    assert calibrate.lambda_from_target(a, b, 0.6, 8192) > calibrate.lambda_from_target(a, b, 0.5, 8192)
    assert calibrate.lambda_from_target(a, b, 0.5, 16384) == pytest.approx(
        calibrate.lambda_from_target(a, b, 0.5, 8192) / 2)
    with pytest.raises(ValueError):
        calibrate.lambda_from_target(a, b, 1.5, 8192)
    with pytest.raises(ValueError):
        calibrate.lambda_from_target(a, b, 0.5, 0)


def test_fit_logspace_recovers_exact_model():
    a, b = 37.5, 6.25
    s = [0.1, 0.3, 0.45, 0.7, 0.9]
    f = [a * math.exp(b * x) for x in s]
    fit = calibrate.fit_logspace(s, f)
    assert fit["a"] == pytest.approx(a, rel=1e-10) and fit["b"] == pytest.approx(b, rel=1e-10)


def test_fit_from_sweep_drops_uninformative_points():
    seq_k = 4096
    a, b = 2.0, 5.0
    pts = [(a * math.exp(b * s) / seq_k, s) for s in (0.2, 0.4, 0.6)] + [(1e-9, 0.0), (10.0, 1.0)]
    fit = calibrate.fit_from_sweep(pts, seq_k)
    assert fit["a"] == pytest.approx(a, rel=1e-9) and fit["b"] == pytest.approx(b, rel=1e-9)


@pytest.mark.gpu
def test_sweep_on_stress_input_is_monotone_and_fits():
    from softmax_ssa_fwd_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["llama8k"].with_(L=2048, Hq=8, Hkv=2, sink_coef=12.0)
    q, k, v = make_inputs(w, "cuda")
    lams = [1e-6, 1e-5, 1e-4, 1e-3, 1e-2, 1e-1]
    pts = calibrate.sweep(q, k, v, lams, scale=w.scale)
    fr = [s for _, s in pts]
    assert all(x <= y for x, y in zip(fr, fr[1:]))
    assert fr[-1] > 0.0
    fit = calibrate.fit_from_sweep(pts, w.L)
    assert fit["a"] > 0


def test_default_trials_and_step_gating():
    assert calibrate.DEFAULT_TRIALS[0] == 1e-4 and calibrate.DEFAULT_TRIALS[-1] == 7e-1
    assert list(calibrate.DEFAULT_TRIALS) == sorted(calibrate.DEFAULT_TRIALS)
    assert not calibrate.skip_enabled(0, 5) and not calibrate.skip_enabled(4, 5)
    assert calibrate.skip_enabled(5, 5) and calibrate.skip_enabled(0, 0)


@pytest.mark.gpu
def test_calibrate_hits_its_own_fit():
    from softmax_ssa_fwd_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["llama8k"].with_(L=2048, Hq=8, Hkv=2, sink_coef=9.0)
    q, k, v = make_inputs(w, "cuda")
    fit = calibrate.calibrate(q, k, v, 0.5, scale=w.scale)
    assert fit["a"] > 0 and math.isfinite(fit["b"])
    assert fit["lambda"] == pytest.approx(fit["a"] * math.exp(fit["b"] * 0.5) / w.L)


def test_timestep_cutoff_gate():
    from softmax_ssa_fwd_b200.calibrate import skip_enabled_at_timestep
    assert skip_enabled_at_timestep(0.9, None)
    assert not skip_enabled_at_timestep(0.9, 0.5)
    assert skip_enabled_at_timestep(0.5, 0.5)       # on from the first step at the cutoff
    assert skip_enabled_at_timestep(0.1, 0.5)
    # over a run with falling timesteps the gate switches on once and stays on
    ts = [1.0 - i / 49 for i in range(50)]
    on = [skip_enabled_at_timestep(t, 0.3) for t in ts]
    first = on.index(True)
    assert not any(on[:first]) and all(on[first:]) and ts[first] <= 0.3 < ts[first - 1]
    for bad in ((1.5, 0.5), (-0.1, 0.5), (0.5, 1.2)):
        with pytest.raises(ValueError):
            skip_enabled_at_timestep(*bad)


def test_skip_phase_needs_both_gates():
    from softmax_ssa_fwd_b200.calibrate import skip_phase
    assert skip_phase(0)
    assert not skip_phase(2, initial_disabled_steps=3)
    assert skip_phase(3, initial_disabled_steps=3)
    assert not skip_phase(10, 0.8, initial_disabled_steps=3, disabled_until_timestep=0.5)
    assert not skip_phase(1, 0.2, initial_disabled_steps=3, disabled_until_timestep=0.5)
    assert skip_phase(10, 0.2, initial_disabled_steps=3, disabled_until_timestep=0.5)
    with pytest.raises(ValueError):
        skip_phase(10, None, disabled_until_timestep=0.5)

