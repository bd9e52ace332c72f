"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs, element by element, at sizes the oracle finishes in
seconds that still span several tiles and a ragged tail; plus the invariants
of the method checked on the GPU itself."""
import numpy as np
import pytest
import torch

from block_causal_linear_b200 import synth
from tolerances import TOL_STATE, err_out, err_state, tol_out

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


def orc_rope(orc, r):
    if r is None:
        return None
    return orc.make_rope(Hg=r.Hg, Wg=r.Wg, t_offset=r.t_offset, dims=(r.dt, r.dh, r.dw), base=r.base)


def expect_path(la, dtype, H, rope):
    """bf16 with H % 4 == 0 runs the tensor-core kernels (with RoPE too: every
    RoPE grid here fits their cos/sin table), the rest the FFMA ones."""
    want = "tc" if (dtype == torch.bfloat16 and H % 4 == 0 and la.tc_enabled()) else "ffma"
    assert la.la_last_path() == want


# ---------------------------------------------------------------- configuration 1

def test_config1_tiny_fp32_streamed_and_one_shot(la, orc):
    w = synth.WORKLOADS[1]
    blocks = list(synth.stream(w, "cpu"))
    q = torch.cat([b[2] for b in blocks], 1)
    k = torch.cat([b[3] for b in blocks], 1)
    v = torch.cat([b[4] for b in blocks], 1)
    ref = orc.brute(q, k, v, w.n_blk, eps=w.eps)                       # definition form
    # one shot
    g = la.full_forward(q.cuda(), k.cuda(), v.cuda(), w.n_blk, eps=w.eps)
    assert err_out(g, ref, torch.float32) <= 1e-4
    # streamed with commit after every block, state against the oracle's state
    st = la.State(w.B, w.H)
    ost = orc.State(w.B, w.H, w.d)
    outs = []
    for n, (_, _, qb, kb, vb) in enumerate(blocks):
        outs.append(la.block_forward(qb.cuda(), kb.cuda(), vb.cuda(), st, commit=True, eps=w.eps))
        orc.block_forward(qb, kb, vb, ost, commit=True, eps=w.eps)
        assert err_state(st.S, ost.S) <= TOL_STATE and err_state(st.Z, ost.Z) <= TOL_STATE
    assert err_out(torch.cat(outs, 1), ref, torch.float32) <= 1e-4
    assert st.blocks_committed == 3
    la.device_status()


# ---------------------------------------------------------------- small shapes, every path

CASES = [  # B, N, H, tokens_per_block, dtype, rope
    (1, 1, 4, 0, torch.bfloat16, False),
    (1, 63, 4, 0, torch.bfloat16, False),
    (2, 129, 8, 0, torch.bfloat16, False),
    (1, 1000, 8, 0, torch.bfloat16, False),
    (2, 777, 4, 300, torch.bfloat16, False),
    (1, 1000, 8, 128, torch.bfloat16, False),
    (2, 700, 8, 0, torch.bfloat16, True),
    (1, 900, 4, 250, torch.bfloat16, True),
    (1, 500, 6, 0, torch.bfloat16, False),       # H not a multiple of 4
    (1, 333, 2, 100, torch.bfloat16, True),
    (1, 3000, 64, 0, torch.bfloat16, True),      # RoPE: every head group split over many CTAs
    (3, 2000, 12, 700, torch.bfloat16, True),    # RoPE: 3 blocks, the last one short, B 3
    (2, 2100, 16, 1000, torch.bfloat16, True),   # RoPE: a last block of 100 tokens
    (2, 300, 3, 64, torch.float32, False),
    (1, 257, 4, 0, torch.float32, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}N{c[1]}H{c[2]}L{c[3]}{str(c[4])[6:]}{'R' if c[5] else ''}")
def test_full_forward_matches_oracle(la, orc, case):
    B, N, H, L, dtype, use_rope = case
    q, k, v = synth.random_qkv(B, N, H, 32, seed=1000 + N + H, dtype=dtype)
    rope = la.make_rope(Hg=3, Wg=5, t_offset=2) if use_rope else None
    g = la.full_forward(q.cuda(), k.cuda(), v.cuda(), L, rope=rope, eps=EPS)
    torch.cuda.synchronize()
    expect_path(la, dtype, H, use_rope)
    ref = orc.full_forward(q, k, v, L, rope=orc_rope(orc, rope), eps=EPS)
    assert err_out(g, ref, dtype) <= tol_out(dtype)
    la.device_status()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("use_rope", [False, True])
def test_streaming_commit_and_read_only_passes(la, orc, dtype, use_rope):
    B, H, n_blk, nb = 2, 8, 450, 3
    rope = la.make_rope(Hg=3, Wg=50, T=3, t_offset=-1) if use_rope else None
    o_rope = (lambda t0: orc.make_rope(Hg=3, Wg=50, t_offset=t0)) if use_rope else (lambda t0: None)
    st = la.State(B, H)
    ost = orc.State(B, H, 32)
    for n in range(nb):
        for p in range(2):
            q, k, v = synth.random_qkv(B, n_blk, H, 32, seed=2000 + 10 * n + p, dtype=dtype)
            commit = p == 1
            S0, Z0 = st.S.clone(), st.Z.clone()
            g = la.block_forward(q.cuda(), k.cuda(), v.cuda(), st, commit=commit, rope=rope, eps=EPS)
            ref = orc.block_forward(q, k, v, ost, commit=commit, rope=o_rope(3 * n), eps=EPS)
            assert err_out(g, ref, dtype) <= tol_out(dtype)
            if not commit:
                assert torch.equal(st.S, S0) and torch.equal(st.Z, Z0)   # read-only pass
            else:
                assert err_state(st.S, ost.S) <= TOL_STATE and err_state(st.Z, ost.Z) <= TOL_STATE
    assert st.blocks_committed == nb
    assert st.t_next == (3 * nb if use_rope else 0)
    la.device_status()


# ---------------------------------------------------------------- invariants on the GPU

def test_deterministic_bitwise(la):
    q, k, v = (t.cuda() for t in synth.random_qkv(2, 2000, 8, 32, seed=31, dtype=torch.bfloat16))
    outs, states = [], []
    for _ in range(2):
        st = la.State(2, 8)
        la.block_forward(q, k, v, st, commit=True, eps=EPS)
        outs.append(la.block_forward(q, k, v, st, commit=True, eps=EPS))
        states.append((st.S.clone(), st.Z.clone()))
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(states[0][0], states[1][0]) and torch.equal(states[0][1], states[1][1])
    a = la.full_forward(q, k, v, 300, eps=EPS)
    b = la.full_forward(q, k, v, 300, eps=EPS)
    assert torch.equal(a, b)


def test_block_causality_bitwise(la):
    q, k, v = (t.cuda() for t in synth.random_qkv(1, 1200, 8, 32, seed=32, dtype=torch.bfloat16))
    a = la.full_forward(q, k, v, 400, eps=EPS)
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    q2[:, 800:] += 1
    k2[:, 800:] *= -1
    v2[:, 800:] += 2
    b = la.full_forward(q2, k2, v2, 400, eps=EPS)
    assert torch.equal(a[:, :800], b[:, :800])
    assert not torch.equal(a[:, 800:], b[:, 800:])


def test_streamed_equals_one_shot(la, orc):
    """Streaming 4 blocks with commit (each call a single block) gives the
    one-shot 4-block result: both match the oracle, and they differ from each
    other by at most the bf16 rounding of their outputs (2 ulp)."""
    B, H, L, nb = 1, 8, 640, 4
    qc, kc, vc = synth.random_qkv(B, L * nb, H, 32, seed=33, dtype=torch.bfloat16)
    q, k, v = qc.cuda(), kc.cuda(), vc.cuda()
    one = la.full_forward(q, k, v, L, eps=EPS)
    st = la.State(B, H)
    streamed = torch.cat([la.block_forward(q[:, i * L:(i + 1) * L].contiguous(), k[:, i * L:(i + 1) * L].contiguous(),
                                           v[:, i * L:(i + 1) * L].contiguous(), st, commit=True, eps=EPS)
                          for i in range(nb)], 1)
    ref = orc.full_forward(qc, kc, vc, L, eps=EPS)
    assert err_out(one, ref, torch.bfloat16) <= tol_out(torch.bfloat16)
    assert err_out(streamed, ref, torch.bfloat16) <= tol_out(torch.bfloat16)
    a, b = streamed.double(), one.double()
    rms = float((b * b).mean().sqrt())
    assert bool(((a - b).abs() <= 2.0 ** -6 * torch.maximum(a.abs(), b.abs()) + 1e-3 * rms).all())


def test_zero_feature_map_gives_zero(la):
    q, k, v = (t.cuda() for t in synth.random_qkv(1, 500, 8, 32, seed=34, dtype=torch.bfloat16))
    out = la.full_forward(-q.abs(), k, v, 0, eps=EPS)
    assert torch.count_nonzero(out) == 0
    out = la.full_forward(q, -k.abs(), v, 0, eps=EPS)
    assert torch.count_nonzero(out) == 0


def test_constant_memory_while_streaming(la):
    B, H, n_blk = 1, 8, 1000
    st = la.State(B, H)
    ws = la.alloc_workspace(B, n_blk, H, 32, n_blk)
    q, k, v = (t.cuda() for t in synth.random_qkv(B, n_blk, H, 32, seed=35, dtype=torch.bfloat16))
    out = torch.empty_like(q)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    alloc0 = torch.cuda.memory_allocated()
    for _ in range(24):
        la.block_forward(q, k, v, st, commit=True, eps=EPS, ws=ws, out=out)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    assert st.nbytes() == B * H * (32 * 32 + 32) * 4
    assert st.blocks_committed == 24


def test_runtime_errors_are_reported(la):
    q, k, v = (t.cuda() for t in synth.random_qkv(1, 64, 4, 32, seed=36, dtype=torch.bfloat16))
    with pytest.raises(la.LAError):
        la.full_forward(q, k, v, 0, eps=EPS, ws=torch.empty(16, dtype=torch.uint8, device="cuda"))
    la.device_status()



def test_one_workspace_serves_calls_of_different_shapes(la, orc):
    """A workspace sized for the largest call is reused, without clearing, by
    calls of other shapes and block counts in turn."""
    big = la.alloc_workspace(2, 3000, 8, 32, 0)
    for (B, N, H, L) in [(1, 3000, 8, 0), (2, 1000, 8, 0), (1, 129, 4, 0), (2, 2000, 8, 700), (2, 3000, 8, 0)]:
        q, k, v = synth.random_qkv(B, N, H, 32, seed=40 + N, dtype=torch.bfloat16)
        assert la.la_workspace_size(B, N, H, 32, L) <= big.numel()
        g = la.full_forward(q.cuda(), k.cuda(), v.cuda(), L, eps=EPS, ws=big)
        torch.cuda.synchronize()
        la.device_status()
        ref = orc.full_forward(q, k, v, L, eps=EPS)
        assert err_out(g, ref, torch.bfloat16) <= tol_out(torch.bfloat16)


def test_rope_grid_beyond_the_table(la, orc):
    """A RoPE grid whose cos/sin records do not fit the tensor-core kernels'
    8 KiB table (3 x 200 per frame: 200 column positions x 48 bytes alone)
    takes the CUDA-core kernels, which compute the angles per element, and
    matches the oracle; the E4M3 and NVFP4 calls, which have no CUDA-core
    path, refuse it with LA_EUNSUPPORTED before enqueueing anything."""
    B, N, H = 1, 1200, 8
    q, k, v = synth.random_qkv(B, N, H, 32, seed=77)
    rope = la.make_rope(Hg=3, Wg=200, t_offset=1)
    g = la.full_forward(q.cuda(), k.cuda(), v.cuda(), 0, rope=rope, eps=EPS)
    torch.cuda.synchronize()
    la.device_status()
    assert la.la_last_path() == "ffma"
    ref = orc.full_forward(q, k, v, 0, rope=orc_rope(orc, rope), eps=EPS)
    assert err_out(g, ref, torch.bfloat16) <= tol_out(torch.bfloat16)
    codes = [synth.to_e4m3(t) for t in (q, k, v)]
    with pytest.raises(la.LAError) as e:
        la.full_forward_e4m3(*[c.cuda() for c, _ in codes], [s_ for _, s_ in codes], 0, eps=EPS, rope=rope)
    assert e.value.status == la.LA_EUNSUPPORTED
    fp4 = [synth.to_nvfp4(t) for t in (q, k, v)]
    with pytest.raises(la.LAError) as e:
        la.full_forward_nvfp4(*[(c.cuda(), sf.cuda(), s_) for c, sf, s_ in fp4], 0, eps=EPS, rope=rope)
    assert e.value.status == la.LA_EUNSUPPORTED
