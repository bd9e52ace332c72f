"""Pins of the fp64 oracle against facts that do not come from the oracle.

Each test pins the oracle to a hand-worked example, a closed form, a property
the pages state (token-split equivalence, block causality, streamed equals
one-shot, constant state size) or a library second opinion.  A plausible slip in
the oracle -- a dropped term, a transposed state, a wrong sign, a missing ReLU, an
off-by-one block edge, a wrong RoPE frequency or section -- fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from block_causal_linear_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
EPS = 1e-6


def _t(a, dtype=torch.float64):
    """[N, d] list -> [1, N, 1, d] tensor."""
    return torch.tensor(a, dtype=dtype).reshape(1, len(a), 1, len(a[0]))


def rel(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------- golden, by hand

def test_golden_two_blocks_every_entry_point(orc):
    g = json.load(open(os.path.join(GOLD, "hand_two_blocks_d2.json")))
    q, k, v = _t(g["q"]), _t(g["k"]), _t(g["v"])
    L = g["tokens_per_block"]
    want = np.array(g["numerator"], float) / (np.array(g["denominator_without_eps"], float)[:, None] + EPS)
    want = want.reshape(1, 4, 1, 2)
    # definition form
    np.testing.assert_allclose(orc.brute(q, k, v, L, eps=EPS), want, rtol=1e-14, atol=0)
    # recurrence, one shot
    np.testing.assert_allclose(orc.full_forward(q, k, v, L, eps=EPS), want, rtol=1e-14, atol=0)
    # the block reduction itself
    KV0, z0 = orc.block_kv(k, v, 0, 2)
    KV1, z1 = orc.block_kv(k, v, 2, 4)
    np.testing.assert_array_equal(KV0[0, 0], np.array(g["KV_block0"], float))
    np.testing.assert_array_equal(z0[0, 0], np.array(g["z_block0"], float))
    np.testing.assert_array_equal(KV1[0, 0], np.array(g["KV_block1"], float))
    np.testing.assert_array_equal(z1[0, 0], np.array(g["z_block1"], float))
    # streaming, block by block with commit
    st = orc.State(1, 1, 2)
    o0 = orc.block_forward(q[:, :2], k[:, :2], v[:, :2], st, commit=True, eps=EPS)
    o1 = orc.block_forward(q[:, 2:], k[:, 2:], v[:, 2:], st, commit=True, eps=EPS)
    np.testing.assert_allclose(np.concatenate([o0, o1], 1), want, rtol=1e-14, atol=0)
    np.testing.assert_array_equal(st.S[0, 0], np.array([[3, -2], [2, 1]], float))
    np.testing.assert_array_equal(st.Z[0, 0], np.array([3, 3], float))
    # apply alone, on the committed state, for token 3 of block 1
    o3 = orc.apply(q[:, 2:], st.S, st.Z, toks=[1], eps=EPS)
    np.testing.assert_allclose(o3[0, 0, 0], want[0, 3, 0], rtol=1e-14)


def test_golden_rope_sign_and_pairing(orc):
    g = json.load(open(os.path.join(GOLD, "hand_rope_sign_d2.json")))
    q, k, v = _t(g["q"]), _t(g["k"]), _t(g["v"])
    s1 = math.sin(1.0)
    num = np.array([[a + b * s1 for a, b in row] for row in g["numerator_in_terms_of_sin1"]])
    want = (num / (np.array(g["denominator_without_eps"], float)[:, None] + EPS)).reshape(1, 2, 1, 2)
    rope = orc.make_rope(Hg=1, Wg=1, t_offset=0, dims=(2, 0, 0))
    np.testing.assert_allclose(orc.brute(q, k, v, 0, rope=rope, eps=EPS), want, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(orc.full_forward(q, k, v, 0, rope=rope, eps=EPS), want, rtol=1e-14, atol=1e-15)


def test_bf16_and_fp32_inputs_widen_exactly(orc):
    # one token, q = k = e0: out = v * 1/(1+eps); v holds exactly representable values
    vals = [1.5, -5.0, 0.0078125, -3.0e38, 1.0e-38, 65504.0]
    d = len(vals)
    q = torch.zeros(1, 1, 1, d)
    q[..., 0] = 1.0
    v = torch.tensor(vals).reshape(1, 1, 1, d)
    for dt in (torch.float32, torch.bfloat16):
        vv = v.to(dt)
        out = orc.brute(q.to(dt), q.to(dt), vv, eps=EPS)
        np.testing.assert_allclose(out.ravel(), vv.double().numpy().ravel() / (1 + EPS), rtol=1e-15)
    # the bf16 bit patterns themselves: 0x3FC0 = 1.5, 0xC0A0 = -5.0
    bits = torch.tensor([0x3FC0, -16224], dtype=torch.int16)      # -16224 is 0xC0A0
    vb = bits.view(torch.bfloat16).reshape(1, 1, 1, 2)
    qb = torch.tensor([1.0, 0.0]).to(torch.bfloat16).reshape(1, 1, 1, 2)
    out = orc.brute(qb, qb, vb, eps=0.0)
    np.testing.assert_array_equal(out.ravel(), [1.5, -5.0])


# ---------------------------------------------------------------- closed forms

def test_single_token_gives_scaled_v(orc):
    q, k, v = synth.random_qkv(1, 1, 3, 32, seed=11, dtype=torch.float64)
    q, k = q.abs() + 0.1, k.abs() + 0.1              # phi = identity on these
    a = (q * k).sum(-1, keepdim=True)
    want = (v * a / (a + EPS)).numpy()
    np.testing.assert_allclose(orc.brute(q, k, v, eps=EPS), want, rtol=1e-13)
    np.testing.assert_allclose(orc.full_forward(q, k, v, eps=EPS), want, rtol=1e-13)


def test_identical_keys_give_prefix_mean_of_v(orc):
    B, N, H, d, L = 1, 13, 2, 8, 4
    q, _, v = synth.random_qkv(B, N, H, d, seed=12, dtype=torch.float64)
    q = q.abs()
    k = torch.rand(1, 1, H, d, dtype=torch.float64).expand(B, N, H, d).contiguous()
    out = orc.full_forward(q, k, v, L, eps=EPS)
    for i in range(N):
        vis = min((i // L + 1) * L, N)
        a = (q[0, i] * k[0, 0]).sum(-1, keepdim=True).numpy()             # [H,1]
        want = v[0, :vis].sum(0).numpy() * a / (vis * a + EPS)
        np.testing.assert_allclose(out[0, i], want, rtol=1e-12)


def test_nonpositive_q_or_k_gives_zero(orc):
    q, k, v = synth.random_qkv(2, 9, 3, 32, seed=13, dtype=torch.float64)
    out = orc.full_forward(-q.abs(), k, v, 3, eps=EPS)
    assert np.all(out == 0.0)
    out = orc.brute(q, -k.abs(), v, 3, eps=EPS)
    assert np.all(out == 0.0)


def test_rope_frequencies_sections_and_positions_closed_form(orc):
    # d = 32 split 8/12/12; token j at frame j // 12, row (j % 12) // 4, column j % 4.
    # q at token 0 and every k are the same one-hot pair start e_{lo+2i}; v_j = e_j.
    # Then out_0[c] = cos(delta_axis(c) * base^(-2i/D)) / (N + eps), exactly.
    Hg, Wg, frames, d, base = 3, 4, 2, 32, 10000.0
    N = frames * Hg * Wg
    sections = [(0, 8, lambda j: j // (Hg * Wg)), (8, 12, lambda j: (j % (Hg * Wg)) // Wg),
                (20, 12, lambda j: j % Wg)]
    rope = orc.make_rope(Hg=Hg, Wg=Wg, t_offset=0, dims=(8, 12, 12), base=base)
    v = torch.zeros(1, N, 1, d, dtype=torch.float64)
    for j in range(N):
        v[0, j, 0, j] = 1.0
    for lo, D, axis in sections:
        for i in range(D // 2):
            e = torch.zeros(d, dtype=torch.float64)
            e[lo + 2 * i] = 1.0
            q = e.expand(1, N, 1, d).contiguous()
            k = q.clone()
            out = orc.full_forward(q, k, v, 0, rope=rope, eps=EPS)
            theta = base ** (-2.0 * i / D)
            want = np.array([math.cos((axis(c) - axis(0)) * theta) for c in range(N)]) / (N + EPS)
            np.testing.assert_allclose(out[0, 0, 0, :N], want, rtol=0, atol=1e-14)
            assert np.all(out[0, 0, 0, N:] == 0.0)


def test_rope_at_position_zero_is_identity(orc):
    q, k, v = synth.random_qkv(1, 12, 2, 32, seed=14, dtype=torch.float64)
    # a grid of 12 rows and a single column: every token has column 0, and only
    # the column section (all 32 dims) rotates, so every rotation is the identity
    rope = orc.make_rope(Hg=12, Wg=1, t_offset=0, dims=(0, 0, 32))
    np.testing.assert_allclose(orc.full_forward(q, k, v, 5, rope=rope, eps=EPS),
                               orc.full_forward(q, k, v, 5, eps=EPS), rtol=1e-14, atol=1e-15)


# ---------------------------------------------------------------- invariants

SHAPES = [  # B, N, H, d, tokens_per_block
    (1, 1, 1, 2, 0), (2, 17, 3, 4, 5), (1, 20, 2, 32, 7), (2, 12, 1, 32, 1), (1, 16, 2, 32, 16),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("use_rope", [False, True])
@pytest.mark.parametrize("dtype", [torch.float64, torch.float32, torch.bfloat16])
def test_brute_equals_recurrence(orc, shape, use_rope, dtype):
    B, N, H, d, L = shape
    q, k, v = synth.random_qkv(B, N, H, d, seed=100 + N, dtype=torch.float32)
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    rope = None
    if use_rope:
        dims = {2: (2, 0, 0), 4: (2, 2, 0), 32: (8, 12, 12)}[d]
        rope = orc.make_rope(Hg=2, Wg=3, t_offset=3, dims=dims)
    a = orc.brute(q, k, v, L, rope=rope, eps=EPS)
    b = orc.full_forward(q, k, v, L, rope=rope, eps=EPS)
    assert rel(b, a) < 1e-12


def test_library_second_opinion_numpy_einsum(orc):
    # test-only second opinion written with numpy masks and einsum
    B, N, H, d, L = 2, 23, 3, 32, 6
    q, k, v = synth.random_qkv(B, N, H, d, seed=21, dtype=torch.float64)
    fq, fk, vv = np.maximum(q.numpy(), 0), np.maximum(k.numpy(), 0), v.numpy()
    blk = np.arange(N) // L
    mask = (blk[None, :] <= blk[:, None]).astype(np.float64)       # [i, j]
    A = np.einsum("bihe,bjhe->bhij", fq, fk) * mask
    want = np.einsum("bhij,bjhe->bihe", A, vv) / (A.sum(-1).transpose(0, 2, 1)[..., None] + EPS)
    assert rel(orc.brute(q, k, v, L, eps=EPS), want) < 1e-12
    assert rel(orc.full_forward(q, k, v, L, eps=EPS), want) < 1e-12


def test_token_split_is_equivalent(orc):
    # KV_{1-2} = KV_1 + KV_2 along any cut of the token order
    q, k, v = synth.random_qkv(2, 31, 3, 32, seed=22, dtype=torch.float32)
    rope = orc.make_rope(Hg=2, Wg=4, t_offset=1)
    for r in (None, rope):
        KV, z = orc.block_kv(k, v, 0, 31, rope=r)
        for cut in (1, 8, 30):
            KVa, za = orc.block_kv(k, v, 0, cut, rope=r)
            KVb, zb = orc.block_kv(k, v, cut, 31, rope=r)
            assert rel(KVa + KVb, KV) < 1e-13 and rel(za + zb, z) < 1e-13


def test_block_causality_bitwise(orc):
    B, N, H, d, L = 1, 21, 2, 32, 7
    q, k, v = synth.random_qkv(B, N, H, d, seed=23, dtype=torch.float32)
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    q2[:, 14:] += 3.0
    k2[:, 14:] *= -2.0
    v2[:, 14:] += 1.0
    for f in (lambda *a: orc.brute(*a, L, eps=EPS), lambda *a: orc.full_forward(*a, L, eps=EPS)):
        a, b = f(q, k, v), f(q2, k2, v2)
        assert np.array_equal(a[:, :14], b[:, :14])
        assert not np.array_equal(a[:, 14:], b[:, 14:])


def test_streamed_equals_one_shot_and_commit_semantics(orc):
    B, H, d, L, nb = 2, 3, 32, 10, 4
    q, k, v = synth.random_qkv(B, L * nb, H, d, seed=24, dtype=torch.float32)
    rope = orc.make_rope(Hg=2, Wg=5, t_offset=0)
    for r in (None, rope):
        one = orc.full_forward(q, k, v, L, rope=r, eps=EPS)
        st = orc.State(B, H, d)
        outs = []
        for n in range(nb):
            sl = slice(n * L, (n + 1) * L)
            S0, Z0 = st.S.copy(), st.Z.copy()
            ro = orc.block_forward(q[:, sl], k[:, sl], v[:, sl], st, commit=False, rope=r, eps=EPS,
                                   tok_base=n * L)
            assert np.array_equal(st.S, S0) and np.array_equal(st.Z, Z0)     # read-only pass
            o = orc.block_forward(q[:, sl], k[:, sl], v[:, sl], st, commit=True, rope=r, eps=EPS,
                                  tok_base=n * L)
            assert np.array_equal(o, ro)
            KV, z = orc.block_kv(k[:, sl], v[:, sl], rope=r, tok_base=n * L)
            assert np.array_equal(st.S, S0 + KV) and np.array_equal(st.Z, Z0 + z)
            outs.append(o)
        assert rel(np.concatenate(outs, 1), one) < 1e-13


def test_state_size_is_constant(orc):
    st = orc.State(1, 2, 32)
    size0 = st.nbytes()
    for n in range(12):
        q, k, v = synth.random_qkv(1, 8, 2, 32, seed=300 + n)
        orc.block_forward(q, k, v, st, commit=True, eps=EPS)
        assert st.nbytes() == size0 == 2 * (32 * 32 + 32) * 8


def test_rope_depends_on_relative_position_only(orc):
    q, k, v = synth.random_qkv(1, 24, 2, 32, seed=25, dtype=torch.float32)
    a = orc.full_forward(q, k, v, 8, rope=orc.make_rope(Hg=2, Wg=3, t_offset=0), eps=EPS)
    b = orc.full_forward(q, k, v, 8, rope=orc.make_rope(Hg=2, Wg=3, t_offset=57), eps=EPS)
    c = orc.full_forward(q, k, v, 8, eps=EPS)
    assert rel(a, b) < 1e-12
    assert rel(a, c) > 1e-3                        # and RoPE does change the result


def test_permuting_tokens_inside_a_block_permutes_outputs(orc):
    q, k, v = synth.random_qkv(1, 18, 2, 32, seed=26, dtype=torch.float64)
    perm = torch.cat([torch.randperm(6, generator=torch.Generator().manual_seed(1)) + 6 * b for b in range(3)])
    a = orc.full_forward(q, k, v, 6, eps=EPS)
    b = orc.full_forward(q[:, perm], k[:, perm], v[:, perm], 6, eps=EPS)
    assert rel(b, a[:, perm.numpy()]) < 1e-13


def test_linear_in_v(orc):
    q, k, v1 = synth.random_qkv(1, 15, 2, 32, seed=27, dtype=torch.float64)
    v2 = synth.random_qkv(1, 15, 2, 32, seed=28, dtype=torch.float64)[2]
    a = orc.full_forward(q, k, v1 + 2 * v2, 4, eps=EPS)
    b = orc.full_forward(q, k, v1, 4, eps=EPS) + 2 * orc.full_forward(q, k, v2, 4, eps=EPS)
    assert rel(a, b) < 1e-13


def test_rejects_bad_arguments(orc):
    q, k, v = synth.random_qkv(1, 4, 1, 6, seed=29, dtype=torch.float64)
    bad = orc.make_rope(Hg=1, Wg=1, dims=(2, 2, 1))   # odd section
    with pytest.raises(ValueError):
        orc.brute(q, k, v, rope=bad)
    with pytest.raises(ValueError):
        orc.block_kv(k, v, 3, 2)


def test_recurrence_cost_is_linear_in_tokens(orc):
    # The method's cost is O(N) in tokens (a fixed-size state per head): four
    # times the tokens must cost about four times the time, far from the 16x
    # of the quadratic brute form.  Median of three runs each.
    import time

    def t(N):
        q, k, v = synth.random_qkv(1, N, 2, 32, seed=24, dtype=torch.float32)
        ts = []
        for _ in range(3):
            t0 = time.perf_counter()
            orc.full_forward(q, k, v, 0, eps=EPS)
            ts.append(time.perf_counter() - t0)
        return sorted(ts)[1]

    ratio = t(32768) / t(8192)
    assert 1.5 < ratio < 8.0, ratio
