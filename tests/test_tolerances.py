"""The bf16 bound of the parity tests: the stated 2e-2 of the output RMS,
widened only where the correctly rounded bf16 output itself misses it."""
import numpy as np
import torch

from tolerances import TOL_BF16, err_bf16, tol_bf16_for


def test_bound_is_the_stated_one_for_ordinary_outputs():
    o = np.random.default_rng(1).standard_normal(4096)
    assert tol_bf16_for(o) == TOL_BF16


def test_bound_follows_correct_rounding_for_heavy_tailed_outputs():
    # RMS ~ 0.05, one output just above a power of two: its bf16 rounding error
    # (half an ulp, ~2^-8 relative) is ~0.0039 * 0.5 / 0.05 ~ 0.04 of the RMS
    o = np.full(4096, 0.05)
    o[7] = 0.5 * (1 + 2.0 ** -8 * 0.999)
    r = err_bf16(torch.from_numpy(o).to(torch.bfloat16), o)
    assert r > TOL_BF16
    assert abs(tol_bf16_for(o) - 1.05 * r) < 1e-12
    # a result past both bf16 neighbours of o[7] is outside the widened bound
    g = torch.from_numpy(o).to(torch.bfloat16).to(torch.float64).numpy()
    g[7] += 2 * 2.0 ** -8
    assert err_bf16(g, o) > tol_bf16_for(o)
