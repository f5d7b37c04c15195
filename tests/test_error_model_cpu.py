"""The rounding-error model behind the GPU parity tolerances, checked against
the roundings themselves (torch's bf16, f16 and float8 conversions, round to
nearest even) rather than against the formula that states it.

Each step of the model is an rms relative error; these tests draw values whose
significands are spread log-uniformly (as the model assumes), perform the
step's actual rounding and compare the measured rms relative error with the
model's figure. A mistake in the model's constant, in a unit roundoff or in how
a two-term split composes would show here.
"""

import math

import numpy as np
import torch

from harness import MODEL_STEPS, RHO, U, model_rel_rms

E4M3, E5M2 = torch.float8_e4m3fn, torch.float8_e5m2


def _loguniform(n, lo, hi, seed):
    rng = np.random.default_rng(seed)
    return np.exp(rng.uniform(math.log(lo), math.log(hi), n)) * rng.choice([-1.0, 1.0], n)


def _rms_rel(got, x):
    return float(np.sqrt(np.mean(((got - x) / x) ** 2)))


def test_rho_is_the_rms_relative_error_of_round_to_nearest():
    x = _loguniform(400000, 1e-3, 1e3, 0)
    t = torch.tensor(x, dtype=torch.float64)
    for dtype, u in ((torch.bfloat16, U["bf16"]), (torch.float16, U["f16"])):
        got = t.float().to(dtype).double().numpy()
        assert abs(_rms_rel(got, x) / u - RHO) < 0.01
        # and u bounds every single rounding
        assert np.all(np.abs(got - x) <= u * np.abs(x) * (1 + 1e-6) + 1e-30)


def test_query_split_step_matches_the_model():
    x = _loguniform(400000, 2.0 ** -5, 400.0, 1)
    q = torch.tensor(x, dtype=torch.float32)
    hi = q.to(E4M3).to(torch.float32)
    lo = (q - hi).to(E5M2).to(torch.float32)
    got = (hi + lo).double().numpy()
    model = MODEL_STEPS["fp8"]["query"]
    assert abs(_rms_rel(got, q.double().numpy()) / model - 1.0) < 0.05


def test_p_split_step_matches_the_model():
    # P' in [1/4, 448]: f16, then hi = e4m3, lo = e4m3 of the exact f16 residual
    x = np.abs(_loguniform(400000, 0.25, 448.0, 2))
    h = torch.tensor(x, dtype=torch.float32).to(torch.float16)
    hi = h.to(E4M3).to(torch.float16)
    lo = (h - hi).to(E4M3).to(torch.float16)
    got = hi.double().numpy() + lo.double().numpy()
    model = MODEL_STEPS["fp8"]["p"]
    assert abs(_rms_rel(got, x) / model - 1.0) < 0.05


def test_bf16_steps_and_total():
    s = MODEL_STEPS["bf16"]
    assert s["query"] == s["p"] == s["o_lat"] == RHO * 2.0 ** -8
    assert s["partials"] == RHO * 2.0 ** -11
    # the stated bf16 bound (5e-3) is 1.50x the model's rms
    assert abs(5e-3 / model_rel_rms("bf16") - 1.504) < 0.01
    # the FP8 path's model is below the bf16 one
    assert model_rel_rms("fp8") < model_rel_rms("bf16")
