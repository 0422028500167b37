"""CPU checks of the parity helpers themselves."""
import numpy as np
import torch

from tests._parity import half_ulp


def test_half_ulp_bf16():
    # bf16 keeps 8 significant bits: spacing 2^-7 in [1, 2), 2^-5 in [4, 8)
    assert half_ulp(np.array([1.5]), torch.bfloat16)[0] == 2.0 ** -8
    assert half_ulp(np.array([-4.49]), torch.bfloat16)[0] == 2.0 ** -6
    x = torch.tensor([4.4885], dtype=torch.float64)
    r = x.to(torch.bfloat16).double()
    assert abs(float(r - x)) <= half_ulp(x.numpy(), torch.bfloat16)[0]


def test_half_ulp_matches_rounding_everywhere():
    rng = np.random.default_rng(0)
    for dt in (torch.bfloat16, torch.float16):
        x = rng.standard_normal(20000) * 4
        x32 = torch.tensor(x, dtype=torch.float32)  # the kernel casts from fp32
        r = x32.to(dt).double().numpy()
        assert np.all(np.abs(r - x32.double().numpy()) <= half_ulp(x, dt) * (1 + 1e-9))
