"""Pins of the oracle's depthwise 3D convolution (Mix-FFN), CPU.

The pages name the operation only (a 1x3x3 spatial and a 3x1x1 temporal
convolution alternating in the MLP, "Nvidia, MIT ve diğerleri video yapay zeka
devrimini başlattı", section "Verimli doğrusal DiT"); the oracle's reading is
a depthwise convolution with zero padding.  Pinned against torch's grouped
conv3d (a library implementation of the same definition) in fp64, and by
closed forms: the identity kernel, and the count of in-range taps for ones.
"""
import numpy as np
import pytest
import torch

SHAPES = [(1, 3, 5, 7, 8), (2, 4, 3, 6, 16), (1, 1, 1, 1, 8), (1, 5, 1, 9, 24)]
KERNELS = [(1, 3, 3), (3, 1, 1), (3, 3, 3), (1, 1, 1)]


def reference(x, w, bias):
    """torch conv3d, groups = C, on [B, C, T, H, W]."""
    xt = torch.as_tensor(x, dtype=torch.float64).permute(0, 4, 1, 2, 3)
    wt = torch.as_tensor(w, dtype=torch.float64)[:, None]
    pad = tuple(k // 2 for k in w.shape[1:])
    y = torch.nn.functional.conv3d(xt, wt, None if bias is None else torch.as_tensor(bias, dtype=torch.float64),
                                   padding=pad, groups=x.shape[-1])
    return y.permute(0, 2, 3, 4, 1).numpy()


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("ks", KERNELS)
def test_dwconv_matches_library(orc, shape, ks):
    g = torch.Generator().manual_seed(sum(shape) + 10 * sum(ks))
    x = torch.randn(shape, generator=g, dtype=torch.float64)
    w = torch.randn((shape[-1],) + ks, generator=g, dtype=torch.float64).numpy()
    b = torch.randn(shape[-1], generator=g, dtype=torch.float64).numpy()
    got = orc.dwconv3d(x, w, b)
    want = reference(x.numpy(), w, b)
    assert np.abs(got - want).max() <= 1e-12 * max(1.0, np.abs(want).max())


@pytest.mark.parametrize("ks", [(1, 3, 3), (3, 1, 1)])
def test_dwconv_identity_kernel(orc, ks):
    x = torch.randn(2, 3, 4, 5, 8, dtype=torch.float64)
    w = np.zeros((8,) + ks)
    w[:, ks[0] // 2, ks[1] // 2, ks[2] // 2] = 1.0
    assert np.array_equal(orc.dwconv3d(x, w), x.numpy())


def test_dwconv_ones_count_taps(orc):
    """All-ones input and weights: each output is the number of in-range taps
    (zero padding), e.g. 4 at a frame corner and 9 inside for 1x3x3."""
    T, H, W = 3, 4, 5
    x = torch.ones(1, T, H, W, 8, dtype=torch.float64)
    y = orc.dwconv3d(x, np.ones((8, 1, 3, 3)))
    for h in range(H):
        for w_ in range(W):
            nh = 1 + (h > 0) + (h < H - 1)
            nw = 1 + (w_ > 0) + (w_ < W - 1)
            assert np.all(y[0, :, h, w_, :] == nh * nw)
    yt = orc.dwconv3d(x, np.ones((8, 3, 1, 1)))
    for t in range(T):
        assert np.all(yt[0, t] == 1 + (t > 0) + (t < T - 1))


def test_dwconv_depthwise_channels_do_not_mix(orc):
    x = torch.zeros(1, 3, 3, 3, 8, dtype=torch.float64)
    x[..., 5] = 1.0
    y = orc.dwconv3d(x, np.ones((8, 3, 3, 3)))
    assert not np.delete(y, 5, axis=-1).any() and y[..., 5].any()
