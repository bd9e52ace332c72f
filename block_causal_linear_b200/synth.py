"""Seeded synthetic inputs and the five workload shapes.

This module draws numbers and describes shapes; it holds none of the attention
arithmetic.  Both the CUDA path (tests, benchmark) and the fp64 oracle take
their inputs from here, so the two always see identical q, k, v.

Recipe (one generator per workload, seeded with the workload's seed):
for each block in order, for each denoising pass in order, draw q, then k, then
v, each ``[B, N_blk, H, d]`` in row-major order, as
``torch.randn(..., dtype=float64) * scale + bias``, rounded to fp32 and then,
for bf16 workloads, to bf16 (round to nearest even).  The generator is torch's
generator of the device the tensors are made on: the CPU generator for the
small cases the oracle runs whole, the CUDA (Philox) generator for full-size
cases; the oracle then reads the device tensors copied back to the host.

Shapes follow the latent grids of the SANA-Video pages: 32x spatial / 4x
temporal DC-AE-V compression for 480p, 8x VAE + 2x2 patchify for 720p, 64
heads of d = 32 ("Nvidia, MIT ve diğerleri video yapay zeka devrimini
başlattı", section "Derin sıkıştırmalı otomatik kodlayıcı (DC-AE-V)").
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Iterator, Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "f32" or "bf16": storage type of q, k, v, out
    B: int
    H: int
    d: int
    frames: int           # latent frames per block
    Hg: int               # latent rows per frame
    Wg: int               # latent columns per frame
    n_blocks: int
    passes: int = 1       # denoising passes per block; the last one commits
    mode: str = "stream"  # "stream": la_block_forward per pass; "full": one la_full_forward
    rope: bool = False
    rope_dims: Tuple[int, int, int] = (8, 12, 12)
    rope_base: float = 10000.0
    seed: int = 0
    scale: float = 1.0
    bias: float = 0.0
    eps: float = 1e-6

    @property
    def n_blk(self) -> int:
        """Tokens per block."""
        return self.frames * self.Hg * self.Wg

    @property
    def n_total(self) -> int:
        return self.n_blk * self.n_blocks

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def calls(self) -> int:
        return self.n_blocks * self.passes if self.mode == "stream" else 1

    @property
    def token_heads(self) -> int:
        """Token-heads processed by the whole workload (every pass counts)."""
        return self.B * self.n_total * self.H * self.passes

    @property
    def alg_bytes(self) -> int:
        """Algorithmic HBM bytes: read q, k, v and write out once per token-head
        and pass (4 * d * elem bytes), plus the fp32 state read and written per
        streaming call.  Workspace traffic is overhead and not counted."""
        per_th = 4 * self.d * self.elem_bytes
        state = 0
        if self.mode == "stream":
            state = self.calls * 2 * self.B * self.H * (self.d * self.d + self.d) * 4
        return self.token_heads * per_th + state

    def shrink(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    1: Workload("tiny-fp32-3x48", "f32", B=1, H=2, d=32, frames=2, Hg=4, Wg=6, n_blocks=3,
                mode="stream", seed=0),
    2: Workload("480p-single-block-8190", "bf16", B=1, H=64, d=32, frames=21, Hg=15, Wg=26,
                n_blocks=1, mode="full", seed=1),
    3: Workload("720p-single-block-75600", "bf16", B=1, H=64, d=32, frames=21, Hg=45, Wg=80,
                n_blocks=1, mode="full", seed=2, scale=0.5, bias=0.1),
    4: Workload("480p-1min-stream-24x15600", "bf16", B=1, H=64, d=32, frames=10, Hg=30, Wg=52,
                n_blocks=24, mode="stream", seed=3),
    5: Workload("720p-B4-7x10800-4pass-rope", "bf16", B=4, H=64, d=32, frames=3, Hg=45, Wg=80,
                n_blocks=7, passes=4, mode="stream", rope=True, seed=4),
}


def _draw(w: Workload, g: torch.Generator, n: int, device) -> torch.Tensor:
    x = torch.randn((w.B, n, w.H, w.d), generator=g, dtype=torch.float64, device=device)
    if w.scale != 1.0 or w.bias != 0.0:
        x = x * w.scale + w.bias
    x = x.to(torch.float32)
    if w.dtype == "bf16":
        x = x.to(torch.bfloat16)
    return x


def generator(w: Workload, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    return g


def stream(w: Workload, device="cpu", blocks: Optional[int] = None
           ) -> Iterator[Tuple[int, int, torch.Tensor, torch.Tensor, torch.Tensor]]:
    """Yield (block, pass, q, k, v) in draw order; each tensor [B, n_blk, H, d]."""
    g = generator(w, device)
    nb = w.n_blocks if blocks is None else blocks
    for blk in range(nb):
        for p in range(w.passes):
            q = _draw(w, g, w.n_blk, device)
            k = _draw(w, g, w.n_blk, device)
            v = _draw(w, g, w.n_blk, device)
            yield blk, p, q, k, v


def full_sequence(w: Workload, device="cpu"):
    """q, k, v of the whole sequence [B, n_total, H, d] (blocks concatenated
    along tokens).  Only for one-pass workloads."""
    assert w.passes == 1
    qs, ks, vs = [], [], []
    for _, _, q, k, v in stream(w, device):
        qs.append(q), ks.append(k), vs.append(v)
    if len(qs) == 1:
        return qs[0], ks[0], vs[0]
    return torch.cat(qs, 1), torch.cat(ks, 1), torch.cat(vs, 1)


def upstream_grad(w: Workload, device="cpu") -> torch.Tensor:
    """dout for a backward pass over the whole sequence of a workload: the same
    recipe as the inputs, from the workload's seed + 7919, drawn after nothing
    else (so it does not change the inputs' draws)."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed + 7919)
    return _draw(w, g, w.n_blk * w.n_blocks, device)


def to_e4m3(x: torch.Tensor):
    """FP8 inputs for the E4M3 path: per-tensor amax scaling, scale =
    max|x| / 448 in fp32 (448 is the largest E4M3 magnitude), codes = x / scale
    rounded to nearest even E4M3 (torch float8_e4m3fn).  Returns (uint8 codes,
    scale).  Input preparation only."""
    xf = x.to(torch.float32)
    amax = float(xf.abs().max()) if xf.numel() else 0.0
    scale = float(torch.tensor(amax / 448.0 if amax > 0 else 1.0, dtype=torch.float32))
    codes = (xf / scale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale


_E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)   # magnitudes of E2M1 codes 0..7


def to_nvfp4(x: torch.Tensor):
    """NVFP4 inputs (two-level scaling, the usual recipe): a per-tensor fp32
    scale s = max|x| / (6 * 448); per 16 consecutive elements of the last axis
    an E4M3 block scale, max|block| / 6 / s rounded to nearest even E4M3; each
    element x / (s * block scale) rounded to the nearest E2M1 value (ties to
    the even code), saturated at 6.  Returns (uint8 codes [..., d/2] with
    element 2i in the low nibble, uint8 block scales [..., d/16], s).  Input
    preparation only."""
    d = x.shape[-1]
    if d % 16:
        raise ValueError("the last axis must be a multiple of 16")
    xf = x.to(torch.float64)
    amax = float(xf.abs().max()) if xf.numel() else 0.0
    s = float(torch.tensor(amax / (6.0 * 448.0) if amax > 0 else 1.0, dtype=torch.float32))
    blocks = xf.reshape(*xf.shape[:-1], d // 16, 16)
    bmax = blocks.abs().amax(dim=-1)
    sf = (bmax / 6.0 / s).to(torch.float32).clamp(max=448.0).to(torch.float8_e4m3fn)
    sfv = sf.to(torch.float64)
    denom = (sfv * s).unsqueeze(-1)
    y = torch.where(denom > 0, blocks / torch.where(denom > 0, denom, torch.ones_like(denom)),
                    torch.zeros_like(blocks))
    mag = y.abs().clamp(max=6.0)
    grid = torch.tensor(_E2M1_GRID, dtype=torch.float64, device=x.device)
    up = torch.searchsorted(grid, mag.contiguous(), right=False).clamp(max=7)   # first grid value >= mag
    lo = (up - 1).clamp(min=0)
    dl, du = mag - grid[lo], grid[up] - mag
    pick_up = (du < dl) | ((du == dl) & (up % 2 == 0))
    code = torch.where(pick_up, up, lo)
    code = code | torch.where((y < 0) & (code > 0), 8, 0)
    code = code.reshape(*xf.shape[:-1], d).to(torch.uint8)
    packed = code[..., 0::2] | (code[..., 1::2] << 4)
    return packed.contiguous(), sf.view(torch.uint8).contiguous(), s


def random_qkv(B, N, H, d, seed, dtype=torch.float32, device="cpu", scale=1.0, bias=0.0):
    """Free-form seeded draw for edge-case tests (same recipe, any shape):
    fp64 normal draws rounded to fp32, then converted to ``dtype``."""
    w = Workload("adhoc", "f32", B=B, H=H, d=d, frames=1, Hg=1, Wg=max(N, 1), n_blocks=1,
                 seed=seed, scale=scale, bias=bias)
    g = generator(w, device)
    return tuple(_draw(w, g, N, device).to(dtype) for _ in range(3))
