"""GPU parity of the Mix-FFN depthwise convolution (la_dwconv3d) against the
fp64 oracle: both kernel shapes (1x3x3 spatial, 3x1x1 temporal), bf16 and fp32,
ragged grids, tiled and untiled TMA shapes, with and without bias, element by element (fp32: per-element
relative 1e-4 with an RMS floor; bf16: max error / RMS 2e-2); a full-size
latent grid checked on sampled channels; bitwise determinism."""
import numpy as np
import pytest
import torch

from tolerances import err_out, tol_out

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_causal_linear_b200 import build

    build.build()
    from block_causal_linear_b200 import la as _la

    return _la


def draw(shape, ks, dtype, seed, with_bias=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g).to(dtype)
    w = (torch.randn((shape[-1],) + ks, generator=g) / 3.0).to(torch.float32)
    b = torch.randn(shape[-1], generator=g).to(torch.float32) if with_bias else None
    return x, w, b


CASES = [  # shape [B, T, Hg, Wg, C], kernel, dtype, bias
    ((1, 3, 5, 7, 8), (1, 3, 3), torch.bfloat16, True),
    ((2, 4, 3, 6, 24), (3, 1, 1), torch.bfloat16, False),
    ((1, 5, 9, 11, 2056), (1, 3, 3), torch.bfloat16, True),     # channel vectors past one CTA, ragged
    ((1, 7, 4, 5, 2056), (3, 1, 1), torch.float32, True),
    ((1, 2, 1, 1, 16), (1, 3, 3), torch.float32, True),          # 1x1 frames: only the centre tap
    ((1, 1, 6, 6, 16), (3, 1, 1), torch.bfloat16, True),         # one frame: only the centre tap
    # bf16 with C >= 64 runs on TMA tiles (64 channels, halo zero-filled by the copy):
    ((2, 7, 4, 5, 2056), (3, 1, 1), torch.bfloat16, True),      # ragged last channel tile, two batches
    ((2, 3, 300, 5, 64), (1, 3, 3), torch.bfloat16, True),      # frame split into row tiles
    ((1, 2, 3, 300, 128), (1, 3, 3), torch.bfloat16, False),    # rows split into column tiles
    ((2, 300, 2, 40, 64), (3, 1, 1), torch.bfloat16, True),     # frame tiles and column tiles
]


@pytest.mark.parametrize("case", CASES)
def test_dwconv_matches_oracle(la, orc, case):
    shape, ks, dtype, with_bias = case
    x, w, b = draw(shape, ks, dtype, seed=sum(shape) + sum(ks))
    y = la.dwconv3d(x.cuda(), w.cuda(), None if b is None else b.cuda())
    torch.cuda.synchronize()
    ref = orc.dwconv3d(x, w.double().numpy(), None if b is None else b.double().numpy())
    assert err_out(y, ref, dtype) <= tol_out(dtype)


def test_dwconv_fullsize_sampled(la, orc):
    """480p latent grid (21 x 15 x 26 tokens), 5120 channels, both shapes; the
    oracle on 64 sampled channels (channels are independent)."""
    shape = (1, 21, 15, 26, 5120)
    for ks in ((1, 3, 3), (3, 1, 1)):
        x, w, b = draw(shape, ks, torch.bfloat16, seed=7 + ks[0])
        y = la.dwconv3d(x.cuda(), w.cuda(), b.cuda()).cpu()
        ch = torch.arange(0, 5120, 80)
        ref = orc.dwconv3d(x[..., ch].contiguous(), w[ch].double().numpy(), b[ch].double().numpy())
        assert err_out(y[..., ch], ref, torch.bfloat16) <= tol_out(torch.bfloat16)


def test_dwconv_deterministic(la):
    x, w, b = draw((1, 6, 7, 9, 256), (1, 3, 3), torch.bfloat16, seed=3)
    xc, wc, bc = x.cuda(), w.cuda(), b.cuda()
    a = la.dwconv3d(xc, wc, bc).clone()
    c = la.dwconv3d(xc, wc, bc)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))
