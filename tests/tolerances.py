"""Error metrics and tolerances of the parity tests (the oracle is fp64).

fp32 path:  max_i |g_i - o_i| / max(|o_i|, 1e-2 * RMS(o)) <= 1e-4
            (relative error per element; the floor keeps outputs near zero
            from dividing by almost nothing)
bf16 path:  max_i |g_i - o_i| / RMS(o) <= 2e-2, or, for an output whose
            correctly rounded bf16 form already misses that bound (rounding
            costs up to 2^-8 |o_i|, so outputs with max |o| / RMS(o) above ~5
            can), within 5% of that rounding's own error (tol_bf16_for)
state:      max |S_gpu - S_oracle| / max |S_oracle| <= 1e-5
bf16 gradients (backward pass; no tolerance is stated for it, this one is
            derived from the arithmetic): max_i |g_i - o_i| / max(|o_i|, RMS(o))
            <= 1e-2.  Gradients are heavy-tailed (max/RMS ~ 10: tokens with a
            small denominator weigh 1/den^2), so the output metric above is
            below the rounding error of a correctly rounded bf16 result; per
            element, rounding to bf16 costs <= 2^-9 ~ 2e-3 and the fp32 sums far
            less, which leaves a margin of 5.  fp32 gradients use the fp32 metric.
"""
import numpy as np
import torch

TOL_F32 = 1e-4
TOL_BF16 = 2e-2
TOL_STATE = 1e-5
TOL_BF16_GRAD = 1e-2


def as_np(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def err_f32(g, o):
    g, o = as_np(g), as_np(o)
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    den = np.maximum(np.abs(o), 1e-2 * rms)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(np.abs(g - o) / den)) if o.size else 0.0


def err_bf16(g, o):
    g, o = as_np(g), as_np(o)
    rms = float(np.sqrt(np.mean(o * o))) if o.size else 0.0
    if rms == 0.0:
        return float(np.max(np.abs(g - o))) if o.size else 0.0
    return float(np.max(np.abs(g - o)) / rms)


def tol_bf16_for(o):
    """The bf16 bound for the oracle output o: TOL_BF16, unless rounding o to
    bf16 (the best any bf16 result can do) already exceeds it; then 5% above
    that rounding's error."""
    o = as_np(o)
    r = torch.from_numpy(o).to(torch.bfloat16)
    return max(TOL_BF16, 1.05 * err_bf16(r, o))


def err_out(g, o, dtype):
    return err_f32(g, o) if dtype == torch.float32 else err_bf16(g, o)


def tol_out(dtype):
    return TOL_F32 if dtype == torch.float32 else TOL_BF16


def err_state(g, o):
    g, o = as_np(g), as_np(o)
    m = float(np.max(np.abs(o)))
    return float(np.max(np.abs(g - o))) / (m if m > 0 else 1.0)


def err_bf16_grad(g, o):
    g, o = as_np(g), as_np(o)
    if not o.size:
        return 0.0
    rms = float(np.sqrt(np.mean(o * o)))
    den = np.maximum(np.abs(o), rms)
    den = np.where(den > 0, den, 1.0)
    return float(np.max(np.abs(g - o) / den))


def err_grad(g, o, dtype):
    return err_f32(g, o) if dtype == torch.float32 else err_bf16_grad(g, o)


def tol_grad(dtype):
    return TOL_F32 if dtype == torch.float32 else TOL_BF16_GRAD
