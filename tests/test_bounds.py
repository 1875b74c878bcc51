"""The ulp-aware bound the wide-value GPU tests use, pinned on the CPU:
half an ulp of the 16-bit output formats at known magnitudes, and the
rounding error of torch's own float32 -> fp16 / bf16 casts never above it."""
import numpy as np
import torch

from helpers import half_ulp, ulp_aware_bound


def test_half_ulp_known_spacings():
    # bf16 keeps 7 fraction bits: spacing 2^-5 on [4, 8), 2^-7 on [1, 2)
    assert half_ulp(5.0, "bf16") == 2 ** -6 and half_ulp(1.5, "bf16") == 2 ** -8
    assert half_ulp(-7.99, "bf16") == 2 ** -6
    # fp16 keeps 10: spacing 2^-10 on [1, 2); subnormal spacing 2^-24
    assert half_ulp(1.5, "f16") == 2 ** -11 and half_ulp(2 ** -20, "f16") == 2 ** -25
    assert half_ulp(0.0, "f16") == 2 ** -25


def test_half_ulp_covers_round_to_nearest_casts():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * 4).astype(np.float32)
    for dt, td in (("bf16", torch.bfloat16), ("f16", torch.float16)):
        r = torch.from_numpy(x).to(td).double().numpy()
        err = np.abs(r - x.astype(np.float64))
        assert (err <= half_ulp(x, dt)).all(), dt
        # and the bound is tight: some casts use more than half of it
        assert (err > 0.5 * half_ulp(x, dt)).any(), dt


def test_bound_is_the_tolerance_below_the_crossover():
    # bf16: half an ulp passes 1e-2 only from 4 (2^-7 below 4, 2^-6 on [4, 8))
    assert ulp_aware_bound(1.0, "bf16", 1e-2) == 1e-2
    assert ulp_aware_bound(5.0, "bf16", 1e-2) > 2 ** -6
    assert ulp_aware_bound(0.3, "f16", 2e-3) == 2e-3
