"""The FP8 path's two-term operand splits, emulated with torch's own float8
conversions (round to nearest even), against the precision the design states
for them.

* The absorbed query: q = e4m3(q) + e5m2(q - e4m3(q)), residual taken in fp32.
  Within 2^-7 of |q| wherever e4m3 is normal.
* P' = 2^kp * P * s_t: rounded to f16, then hi = e4m3(x) and lo = e4m3(x - hi),
  the difference exact in f16. Within 2^-8 of x for x >= 1/4, and within an
  absolute 2^-10 below that; f16's own rounding adds 2^-11 of x.
* kp, the largest integer with 2^kp * s_max <= 56, keeps P' = P * s * 2^kp
  at most 448 (e4m3's largest finite value) while P <= 2^3 (the lazy max), and
  puts every weight P >= (s_max / s) / 112 at P' >= 1/4, where the split keeps
  8 significant bits.

These are host-side checks of the scheme's arithmetic; the CUDA kernels are
checked against the oracle by the GPU parity tests.
"""

import math

import numpy as np
import torch

E4M3, E5M2 = torch.float8_e4m3fn, torch.float8_e5m2


def _loguniform(rng, lo, hi, n):
    return np.exp(rng.uniform(math.log(lo), math.log(hi), n))


def test_query_split_keeps_seven_bits():
    rng = np.random.default_rng(0)
    x = _loguniform(rng, 2.0 ** -6, 440.0, 200000) * rng.choice([-1.0, 1.0], 200000)
    q = torch.tensor(x, dtype=torch.float32)
    hi = q.to(E4M3).to(torch.float32)
    lo = (q - hi).to(E5M2).to(torch.float32)
    err = (hi + lo - q).abs().double().numpy()
    assert np.all(err <= 2.0 ** -7 * np.abs(x) * (1 + 1e-6))
    # one term alone is four bits: the correction is what buys the rest
    assert np.max((hi - q).abs().double().numpy() / np.abs(x)) > 2.0 ** -6


def _p_split(x):
    h = torch.tensor(x, dtype=torch.float32).to(torch.float16)
    hi = h.to(E4M3).to(torch.float16)
    res = h - hi                                  # exact in f16
    lo = res.to(E4M3).to(torch.float16)
    return h.double().numpy(), (hi.double() + lo.double()).numpy()


def test_p_split_keeps_eight_bits_above_a_quarter():
    rng = np.random.default_rng(1)
    x = _loguniform(rng, 0.25, 440.0, 200000)
    h, got = _p_split(x)
    assert np.all(np.abs(h - x) <= 2.0 ** -11 * x)
    assert np.all(np.abs(got - h) <= 2.0 ** -8 * x * (1 + 1e-6))


def test_p_split_small_weights_have_a_bounded_absolute_error():
    rng = np.random.default_rng(2)
    x = np.concatenate([_loguniform(rng, 2.0 ** -14, 0.25, 200000), [0.0]])
    h, got = _p_split(x)
    assert np.all(np.abs(got - h) <= 2.0 ** -10 * (1 + 1e-6))


def _kp(s):
    y = np.float32(56.0) / np.float32(s)
    return int((np.float32(y).view(np.uint32) >> 23) & 0xFF) - 127     # floor(log2 y), y normal


def test_p_scale_exponent_bounds_the_split_operand():
    rng = np.random.default_rng(3)
    s_max = np.concatenate([_loguniform(rng, 1e-6, 1e4, 100000), [56.0, 28.0, 1.75, 56.0 * 2.0 ** -20]])
    for s in s_max:
        kp = _kp(s)
        assert kp == math.floor(math.log2(56.0 / float(s)))
        assert 2.0 ** kp * s <= 56.0 < 2.0 ** (kp + 1) * s
        assert 2.0 ** 3 * 2.0 ** kp * s <= 448.0    # P <= 2^3 under the lazy max


def test_p_scale_puts_ordinary_weights_where_the_split_keeps_eight_bits():
    # the FP8 workload's token scales span a factor 2 (s in [1/48, 1/24])
    rng = np.random.default_rng(4)
    s = rng.uniform(1 / 48, 1 / 24, 4096)
    s_max = s.max()
    kp = _kp(s_max)
    p_min = (s_max / s) / 112.0
    assert np.all(p_min <= 1 / 56 + 1e-12)
    x = (2.0 ** kp) * p_min * s                   # the smallest weight that qualifies
    assert np.all(x >= 0.25 * (1 - 1e-6))
    # weights in [P_min, 2^3] split with a relative error of at most 2^-8 (+ f16's 2^-11)
    P = np.exp(rng.uniform(math.log(1 / 56), math.log(8.0), 4096))
    xs = (2.0 ** kp) * P * s
    h, got = _p_split(xs)
    assert np.all(np.abs(got - xs) <= (2.0 ** -8 + 2.0 ** -11) * xs * (1 + 1e-6))
