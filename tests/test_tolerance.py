"""The parity metric itself (CPU): it must reject real errors, apply the bf16 bar to the raw
difference, and take off the output's own rounding only where a test asks for it."""
import numpy as np
import torch

from tolerance import err, half_ulp_bf16


def test_half_ulp():
    assert half_ulp_bf16(np.array([1.0]))[0] == 2.0 ** -8
    assert half_ulp_bf16(np.array([1.5]))[0] == 2.0 ** -8
    assert half_ulp_bf16(np.array([0.25]))[0] == 2.0 ** -10
    assert half_ulp_bf16(np.array([0.0]))[0] == 0.0


def test_raw_bar_by_default():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(10000) ** 3          # heavy tails: rounding alone is large vs rms
    exact = torch.tensor(ref, dtype=torch.float32).bfloat16()
    e, raw = err(exact, ref, torch.bfloat16)
    assert e == raw and raw > 0.0                   # no allowance unless asked for
    e, raw = err(exact, ref, torch.bfloat16, rounding_floor=True)
    assert e == 0.0 and raw > 0.0                   # the rounding floor removes exact rounding


def test_metric_rejects_errors():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(10000) ** 3
    bad = ref.copy()
    bad[17] += 0.05 * np.sqrt(np.mean(ref ** 2))   # a 5%-of-rms arithmetic error
    g = torch.tensor(bad, dtype=torch.float32).bfloat16()
    assert err(g, ref, torch.bfloat16)[0] > 2e-2
    assert err(g, ref, torch.bfloat16, rounding_floor=True)[0] > 2e-2
    e, _ = err(torch.tensor(ref * (1 + 2e-4)), ref, torch.float32)
    assert e > 1e-4


def test_light_tailed_bf16_rounding_passes_raw_bar():
    """Outputs with max/rms near 4-5 (the linear, MLP and chunked layers): exact bf16
    rounding stays inside the raw 2e-2 bar -- at most half an ulp at the largest value
    (2^2 * 2^-8 for values in [4, 8)) over the RMS."""
    rng = np.random.default_rng(1)
    ref = rng.standard_normal(200000)
    e, raw = err(torch.tensor(ref, dtype=torch.float32).bfloat16(), ref, torch.bfloat16)
    rms = np.sqrt(np.mean(ref ** 2))
    assert e == raw and raw <= 2.0 ** (2 - 8) / rms < 2e-2


def test_auto_floor_only_where_exact_rounding_fails_the_bar():
    from tolerance import rounding_alone
    rng = np.random.default_rng(2)
    light = rng.standard_normal(100000)              # rounding alone ~1.2e-2: raw bar stands
    heavy = rng.standard_normal(100000) ** 3         # rounding alone far above 2e-2
    assert rounding_alone(light) < 2e-2 < rounding_alone(heavy)
    g = torch.tensor(light, dtype=torch.float32).bfloat16()
    e, raw = err(g, light, torch.bfloat16, rounding_floor="auto")
    assert e == raw
    g = torch.tensor(heavy, dtype=torch.float32).bfloat16()
    e, raw = err(g, heavy, torch.bfloat16, rounding_floor="auto")
    assert e < 1e-6 < raw  # exact rounding (via fp32) is all the difference there is
