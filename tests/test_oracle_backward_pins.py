"""Pins of the oracle's backward pass (CPU).

The pages give only the forward recurrence ("Nvidia, MIT ve diğerleri video
yapay zeka devrimini başlattı", section "Sabit Bellekli KV önbelleğe alma
mekanizması"); the backward is its derivative, for block-autoregressive
training.  The oracle's backward (chain rule through the recurrence) is
pinned against two things that share none of its code:

- central finite differences of the oracle's own forward, in fp64;
- torch autograd through a brute-force O(N^2) restatement of the definition
  (block-causal mask, ratio form, RoPE on the numerator only), in fp64;

plus closed-form special cases.  Inputs stay away from 0 so that no finite
difference step crosses the ReLU kink.
"""
import math

import numpy as np
import pytest
import torch

EPS = 1e-6


def away_from_zero(shape, seed, lo=0.2):
    g = torch.Generator().manual_seed(seed)
    r = torch.randn(shape, generator=g, dtype=torch.float64)
    return torch.sign(r) * (lo + r.abs())


def loss(orc, q, k, v, dout, L, rope):
    return float((orc.full_forward(q, k, v, L, rope=rope, eps=EPS) * dout.numpy()).sum())


def finite_diff(orc, q, k, v, dout, L, rope, h=1e-5):
    grads = []
    for which in range(3):
        xs = [q.clone(), k.clone(), v.clone()]
        g = np.zeros(tuple(q.shape))
        flat = xs[which].view(-1)
        for i in range(flat.numel()):
            x0 = float(flat[i])
            flat[i] = x0 + h
            lp = loss(orc, *xs, dout, L, rope)
            flat[i] = x0 - h
            lm = loss(orc, *xs, dout, L, rope)
            flat[i] = x0
            g.reshape(-1)[i] = (lp - lm) / (2 * h)
        grads.append(g)
    return grads


def rope_angles(N, d, Hg, Wg, dims, base, t_offset=0):
    """[N, d/2] angle of every feature pair of every token (interleaved pairs,
    sections frame / row / column), written from the stated convention."""
    t = torch.arange(N)
    per = Hg * Wg
    pos = {0: t // per + t_offset, 1: (t % per) // Wg, 2: t % Wg}
    cols = []
    for ax, D in enumerate(dims):
        for i in range(D // 2):
            cols.append(pos[ax].to(torch.float64) * base ** (-2.0 * i / D))
    return torch.stack(cols, 1)


def rotate(x, ang):
    """x [B, N, H, d]; ang [N, d/2]."""
    c, s = torch.cos(ang)[None, :, None, :], torch.sin(ang)[None, :, None, :]
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = torch.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def brute_torch(q, k, v, L, ang):
    """out_i = sum_{j: blk(j) <= blk(i)} (psi q_i . psi k_j) v_j / (sum_j phi q_i . phi k_j + eps)."""
    N = q.shape[1]
    blk = torch.arange(N) // (L if L > 0 else N)
    mask = (blk[None, :] <= blk[:, None]).to(torch.float64)          # [i, j]
    fq, fk = torch.relu(q), torch.relu(k)
    pq, pk = (rotate(fq, ang), rotate(fk, ang)) if ang is not None else (fq, fk)
    a_num = torch.einsum("bihd,bjhd->bhij", pq, pk) * mask
    a_den = torch.einsum("bihd,bjhd->bhij", fq, fk) * mask
    num = torch.einsum("bhij,bjhd->bihd", a_num, v)
    den = a_den.sum(-1).permute(0, 2, 1)[..., None]                   # [b, i, h, 1]
    return num / (den + EPS)


CASES = [  # (B, N, H, d, L, rope dims or None)
    (1, 7, 2, 4, 3, None),
    (1, 6, 1, 4, 0, None),
    (2, 5, 1, 4, 1, None),
    (1, 7, 2, 8, 3, (2, 2, 4)),
    (1, 8, 1, 8, 4, (4, 2, 2)),
]


@pytest.mark.parametrize("case", CASES)
def test_backward_matches_finite_differences(orc, case):
    B, N, H, d, L, dims = case
    q, k, v, dout = (away_from_zero((B, N, H, d), 100 + i + 7 * N) for i in range(4))
    rope = orc.make_rope(Hg=2, Wg=2, t_offset=1, dims=dims) if dims else None
    got = orc.full_backward(q, k, v, dout, L, rope=rope, eps=EPS)
    want = finite_diff(orc, q, k, v, dout, L, rope)
    for g, w in zip(got, want):
        scale = np.abs(w).max()
        assert np.abs(g - w).max() <= 1e-7 * scale + 1e-9


@pytest.mark.parametrize("case", CASES)
def test_backward_matches_autograd_of_brute_definition(orc, case):
    B, N, H, d, L, dims = case
    q, k, v, dout = (away_from_zero((B, N, H, d), 200 + i + 7 * N) for i in range(4))
    rope = orc.make_rope(Hg=2, Wg=2, t_offset=1, dims=dims) if dims else None
    ang = rope_angles(N, d, 2, 2, dims, 10000.0, t_offset=1) if dims else None
    xs = [t.clone().requires_grad_(True) for t in (q, k, v)]
    out = brute_torch(*xs, L, ang)
    # the forward restatement agrees with the oracle's forward first
    assert np.abs(out.detach().numpy() - orc.full_forward(q, k, v, L, rope=rope, eps=EPS)).max() <= 1e-12 * max(
        1.0, float(out.detach().abs().max()))
    (out * dout).sum().backward()
    got = orc.full_backward(q, k, v, dout, L, rope=rope, eps=EPS)
    for g, x in zip(got, xs):
        w = x.grad.numpy()
        assert np.abs(g - w).max() <= 1e-11 * max(1.0, np.abs(w).max())


def test_backward_zero_upstream_gives_zero(orc):
    q, k, v = (away_from_zero((1, 9, 2, 4), 300 + i) for i in range(3))
    for g in orc.full_backward(q, k, v, torch.zeros_like(q), 4, eps=EPS):
        assert not g.any()


def test_backward_all_queries_nonpositive(orc):
    """phi(q) = 0 everywhere: out = 0/eps = 0 whatever k, v, so every gradient is 0."""
    q = -away_from_zero((1, 9, 2, 4), 310).abs()
    k, v, dout = (away_from_zero((1, 9, 2, 4), 311 + i) for i in range(3))
    for g in orc.full_backward(q, k, v, dout, 4, eps=EPS):
        assert not g.any()


def test_backward_single_token_closed_form(orc):
    """One token, one block, d = 1, q, k > 0: out = q k v / (q k + eps), so
    dv = dout q k / (q k + eps), dq = dout k v eps / (q k + eps)^2 and dk =
    dout q v eps / (q k + eps)^2 (eps = 0.25 keeps the difference that forms
    dq well conditioned)."""
    qv, kv_, vv, do, eps = 0.7, 1.3, -0.4, 2.0, 0.25
    t = lambda x: torch.tensor([[[[x]]]], dtype=torch.float64)
    dq, dk, dv = (float(g.reshape(-1)[0]) for g in orc.full_backward(t(qv), t(kv_), t(vv), t(do), 0, eps=eps))
    den = qv * kv_ + eps
    assert math.isclose(dv, do * qv * kv_ / den, rel_tol=1e-14)
    assert math.isclose(dq, do * kv_ * vv * eps / den ** 2, rel_tol=1e-13)
    assert math.isclose(dk, do * qv * vv * eps / den ** 2, rel_tol=1e-13)
