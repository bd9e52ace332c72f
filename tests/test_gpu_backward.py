"""GPU parity of the backward pass (la_full_backward) against the fp64 oracle.

dq, dk, dv of sum(full_forward(q, k, v) * dout) on the same seeded inputs,
element by element: fp32 path, per-element relative error with a 1e-2 RMS
floor, 1e-4 (as the forward); bf16 path, per-element relative error with an
RMS floor, 1e-2 (derived from the arithmetic, tests/tolerances.py: the
gradients are heavy-tailed, so the forward's max-error-over-RMS metric would
sit below the rounding of a correctly rounded bf16 result).  Shapes span several tiles and splits with
ragged tails, one and many blocks, with and without RoPE, on the CUDA-core
and the tensor-core state paths; plus bitwise determinism and a full-size
case checked on a sample of heads.
"""
import pytest
import torch

from block_causal_linear_b200 import synth
from tolerances import err_grad, tol_grad

pytestmark = pytest.mark.gpu
EPS = 1e-6


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_causal_linear_b200 import build

    build.build()
    from block_causal_linear_b200 import la as _la

    return _la


def inputs(B, N, H, dtype, seed):
    q, k, v = synth.random_qkv(B, N, H, 32, seed=seed, dtype=dtype)
    dout = synth.random_qkv(B, N, H, 32, seed=seed + 1, dtype=dtype)[0]
    return q, k, v, dout


CASES = [  # dtype, B, N, H, tokens_per_block, rope
    (torch.float32, 1, 200, 2, 64, False),
    (torch.float32, 2, 130, 3, 0, False),
    (torch.bfloat16, 1, 300, 8, 128, False),      # tensor-core state path (H % 4 == 0)
    (torch.bfloat16, 1, 517, 4, 0, False),
    (torch.bfloat16, 2, 250, 6, 100, False),      # CUDA-core path (H % 4 != 0)
    (torch.bfloat16, 1, 240, 4, 60, True),
    (torch.float32, 1, 180, 2, 45, True),
    (torch.bfloat16, 1, 1000, 8, 250, True),     # RoPE: key side on the tensor cores, ragged tiles
    (torch.bfloat16, 2, 777, 4, 300, True),      # RoPE: two batches, a short last block
    (torch.bfloat16, 1, 2100, 16, 0, True),      # RoPE: one block, many tiles per split
]


@pytest.mark.parametrize("case", CASES)
def test_backward_matches_oracle(la, orc, case):
    dtype, B, N, H, L, use_rope = case
    q, k, v, dout = inputs(B, N, H, dtype, seed=40 + N)
    rope = la.make_rope(Hg=3, Wg=5, t_offset=2) if use_rope else None
    orope = orc.make_rope(Hg=3, Wg=5, t_offset=2) if use_rope else None
    got = la.full_backward(q.cuda(), k.cuda(), v.cuda(), dout.cuda(), L, rope=rope, eps=EPS)
    torch.cuda.synchronize()
    la.device_status()
    if use_rope and dtype == torch.bfloat16 and H % 4 == 0:
        assert la.la_last_path() == "bwd(tc state, tc keys)"   # key side on the tensor cores
    want = orc.full_backward(q, k, v, dout, L, rope=orope, eps=EPS)
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        e = err_grad(g, w, dtype)
        assert e <= tol_grad(dtype), (name, e)


def test_backward_deterministic(la):
    q, k, v, dout = (t.cuda() for t in inputs(1, 1000, 8, torch.bfloat16, seed=7))
    a = [t.clone() for t in la.full_backward(q, k, v, dout, 256, eps=EPS)]
    b = la.full_backward(q, k, v, dout, 256, eps=EPS)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_backward_zero_upstream(la):
    q, k, v, _ = (t.cuda() for t in inputs(1, 300, 4, torch.bfloat16, seed=9))
    for g in la.full_backward(q, k, v, torch.zeros_like(q), 100, eps=EPS):
        assert not g.float().abs().max().item()


def test_backward_fullsize_sampled_heads(la, orc):
    """Two 480p streaming blocks (2 x 15,600 tokens, 64 heads, bf16): heads are
    independent, so the oracle runs on a sample of heads of the same inputs."""
    w = synth.WORKLOADS[4]
    N = 2 * w.n_blk
    q, k, v, dout = (t.cuda() for t in inputs(1, N, 64, torch.bfloat16, seed=11))
    got = la.full_backward(q, k, v, dout, w.n_blk, eps=EPS)
    torch.cuda.synchronize()
    la.device_status()
    heads = [0, 13, 38, 63]
    idx = torch.tensor(heads, device="cuda")
    sub = [t.index_select(2, idx).contiguous().cpu() for t in (q, k, v, dout)]
    want = orc.full_backward(*sub, w.n_blk, eps=EPS)
    for name, g, wt in zip(("dq", "dk", "dv"), got, want):
        e = err_grad(g.index_select(2, idx).cpu(), wt, torch.bfloat16)
        assert e <= tol_grad(torch.bfloat16), (name, e)


def test_backward_rope_deterministic_and_fullsize_sampled(la, orc):
    """RoPE backward on two 720p B4 blocks (2 x 10,800 tokens, 3 x 45 x 80
    latent frames each, 64 heads): repeated calls give the same bits, and a
    sample of heads matches the oracle (heads are independent)."""
    w = synth.WORKLOADS[5]
    B, N = 1, 2 * w.n_blk
    q, k, v, dout = (t.cuda() for t in inputs(B, N, 64, torch.bfloat16, seed=13))
    rope = la.make_rope(Hg=w.Hg, Wg=w.Wg, t_offset=0)
    got = [t.clone() for t in la.full_backward(q, k, v, dout, w.n_blk, rope=rope, eps=EPS)]
    again = la.full_backward(q, k, v, dout, w.n_blk, rope=rope, eps=EPS)
    torch.cuda.synchronize()
    la.device_status()
    for x, y in zip(got, again):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    heads = [0, 29, 63]
    idx = torch.tensor(heads, device="cuda")
    sub = [t.index_select(2, idx).contiguous().cpu() for t in (q, k, v, dout)]
    want = orc.full_backward(*sub, w.n_blk, rope=orc.make_rope(Hg=w.Hg, Wg=w.Wg, t_offset=0), eps=EPS)
    for name, g, wt in zip(("dq", "dk", "dv"), got, want):
        e = err_grad(g.index_select(2, idx).cpu(), wt, torch.bfloat16)
        assert e <= tol_grad(torch.bfloat16), (name, e)
