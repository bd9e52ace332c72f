"""The five workload shapes and the input recipe, pinned on the CPU.

The benchmark's throughput and roofline denominators (token-heads and
algorithmic bytes per step) and every parity case draw on
`block_causal_linear_b200/synth.py`; these tests fix its shapes to the latent
grids the pages give (480p under 32x spatial / 4x temporal compression, 720p
under an 8x VAE plus 2x2 patchify, 64 heads of d = 32) and its draw order, so
that a silent change to either shows up here."""
import torch

from block_causal_linear_b200 import synth


def test_workload_shapes_and_sizes():
    w = synth.WORKLOADS
    # (tokens per block, blocks, passes, B, H, dtype, rope, seed)
    assert (w[1].n_blk, w[1].n_blocks, w[1].passes, w[1].B, w[1].H, w[1].dtype) == (48, 3, 1, 1, 2, "f32")
    assert (w[2].n_blk, w[2].n_blocks, w[2].mode) == (21 * 15 * 26, 1, "full") == (8190, 1, "full")
    assert (w[3].n_blk, w[3].n_blocks, w[3].scale, w[3].bias) == (75600, 1, 0.5, 0.1)
    assert (w[4].n_blk, w[4].n_blocks, w[4].mode) == (15600, 24, "stream")
    assert (w[5].n_blk, w[5].n_blocks, w[5].passes, w[5].B, w[5].rope) == (10800, 7, 4, 4, True)
    assert w[5].rope_dims == (8, 12, 12) and w[5].rope_base == 10000.0
    assert [w[c].seed for c in range(1, 6)] == [0, 1, 2, 3, 4]
    for c in range(2, 6):
        assert (w[c].H, w[c].d, w[c].dtype, w[c].eps) == (64, 32, "bf16", 1e-6)
    # token-heads and algorithmic bytes per step: q, k, v read and out written
    # (4 x 64 B per token-head in bf16), plus the fp32 state read and written
    # per streaming call
    assert w[2].token_heads == 8190 * 64 and w[2].alg_bytes == 8190 * 64 * 256
    assert w[3].alg_bytes == 75600 * 64 * 256
    state = 2 * 64 * (32 * 32 + 32) * 4          # per batch element and call
    assert w[4].alg_bytes == 24 * 15600 * 64 * 256 + 24 * state
    assert w[5].token_heads == 4 * 10800 * 7 * 4 * 64
    assert w[5].alg_bytes == w[5].token_heads * 256 + 28 * 4 * state
    assert abs(w[5].token_heads * 256 / 1e9 - 19.82) < 0.01


def test_draw_order_and_rounding():
    w = synth.WORKLOADS[1]
    draws = list(synth.stream(w))
    assert [(b, p) for b, p, *_ in draws] == [(0, 0), (1, 0), (2, 0)]
    # q, then k, then v of each block, from one generator seeded with the
    # workload's seed, drawn in fp64 and rounded to fp32
    g = torch.Generator().manual_seed(0)
    for _, _, q, k, v in draws:
        for t in (q, k, v):
            want = torch.randn((1, 48, 2, 32), generator=g, dtype=torch.float64).to(torch.float32)
            assert t.dtype == torch.float32 and torch.equal(t, want)
    # bf16 workloads round the fp32 value to nearest even bf16; config 3 scales
    # and shifts in fp64 first
    w3 = synth.WORKLOADS[3].shrink(frames=1, Hg=2, Wg=3, H=2)
    _, _, q, _, _ = next(synth.stream(w3))
    g = torch.Generator().manual_seed(2)
    want = (torch.randn((1, 6, 2, 32), generator=g, dtype=torch.float64) * 0.5 + 0.1).to(torch.float32)
    assert q.dtype == torch.bfloat16 and torch.equal(q, want.to(torch.bfloat16))


def test_passes_draw_fresh_inputs():
    w = synth.WORKLOADS[5].shrink(frames=1, Hg=2, Wg=2, H=4, B=1, n_blocks=2)
    draws = list(synth.stream(w))
    assert [(b, p) for b, p, *_ in draws] == [(b, p) for b in range(2) for p in range(4)]
    ks = [k for *_, k, _ in draws]
    assert all(not torch.equal(ks[i], ks[j]) for i in range(len(ks)) for j in range(i))
