"""The parity metric itself (CPU): it must reject real errors and accept exact bf16 rounding."""
import numpy as np
import torch

from tolerance import err, half_ulp_bf16


def test_half_ulp():
    assert half_ulp_bf16(np.array([1.0]))[0] == 2.0 ** -8
    assert half_ulp_bf16(np.array([1.5]))[0] == 2.0 ** -8
    assert half_ulp_bf16(np.array([0.25]))[0] == 2.0 ** -10
    assert half_ulp_bf16(np.array([0.0]))[0] == 0.0


def test_metric_accepts_rounding_and_rejects_errors():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(10000) ** 3          # heavy tails: rounding alone is large vs rms
    exact = torch.tensor(ref, dtype=torch.float32).bfloat16()
    e, raw = err(exact, ref, torch.bfloat16)
    assert e == 0.0 and raw > 0.0
    bad = ref.copy()
    bad[17] += 0.05 * np.sqrt(np.mean(ref ** 2))   # a 5%-of-rms arithmetic error
    e, _ = err(torch.tensor(bad, dtype=torch.float32).bfloat16(), ref, torch.bfloat16)
    assert e > 2e-2
    e, _ = err(torch.tensor(ref * (1 + 2e-4)), ref, torch.float32)
    assert e > 1e-4
