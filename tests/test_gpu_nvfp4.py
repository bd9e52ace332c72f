"""GPU parity of the NVFP4 path (la_full_forward_nvfp4, la_block_forward_nvfp4)
against the fp64 oracle run on the decoded inputs (oracle.nvfp4_decode: E2M1
code values times their E4M3 block scale times the per-tensor scale), element
by element, bf16-output tolerance (max |g - o| / RMS(o) <= 2e-2); the state
after commit within the state tolerance; bitwise determinism; argument
errors."""
import pytest
import torch

from block_causal_linear_b200 import synth
from tolerances import TOL_STATE, err_bf16, err_state, tol_bf16_for, TOL_BF16

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


def fp4_inputs(B, N, H, seed, scale=1.0, bias=0.0):
    q, k, v = synth.random_qkv(B, N, H, 32, seed=seed, scale=scale, bias=bias)
    return [synth.to_nvfp4(t) for t in (q, k, v)]


def on_gpu(qkv):
    return [(c.cuda(), sf.cuda(), s) for c, sf, s in qkv]


def decoded(orc, qkv):
    return [orc.nvfp4_decode(c, sf, s) for c, sf, s in qkv]


# (1, 517, 8, 0): 9 reduce splits, a separate combine; (2, 300, 8, 0): 5 splits
# combined inside the reduce (a cluster); (2, 300, 8, 128) and (1, 1000, 16,
# 250): several blocks with a ragged last one; (1, 33, 24, 0): one partial
# tile, 6 head groups (the last group's scales at the end of a 48-byte row);
# (1, 4099, 64, 0) and (1, 8190, 64, 0): the 480p head count, the second the
# 480p single-block workload itself.
@pytest.mark.parametrize("B,N,H,L", [(1, 517, 8, 0), (2, 300, 8, 0), (2, 300, 8, 128), (1, 1000, 16, 250),
                                     (1, 33, 24, 0), (1, 4099, 64, 0), (1, 8190, 64, 0)])
def test_full_forward_nvfp4_matches_oracle(la, orc, B, N, H, L):
    qkv = fp4_inputs(B, N, H, seed=160 + N + H)
    g = la.full_forward_nvfp4(*on_gpu(qkv), L, eps=EPS)
    torch.cuda.synchronize()
    la.device_status()
    assert la.la_last_path() == "tc_nvfp4"
    ref = orc.full_forward(*decoded(orc, qkv), L, eps=EPS)
    assert err_bf16(g, ref) <= TOL_BF16


def test_block_forward_nvfp4_streaming(la, orc):
    B, H, Nb, nb = 1, 8, 400, 3
    st = la.State(B, H)
    ost = orc.State(B, H, 32)
    for i in range(nb):
        qkv = fp4_inputs(B, Nb, H, seed=180 + i, scale=0.7, bias=0.05)
        commit = i != 1          # the middle call is read-only
        S0, Z0 = st.S.clone(), st.Z.clone()
        g = la.block_forward_nvfp4(*on_gpu(qkv), st, commit=commit, eps=EPS)
        ref = orc.block_forward(*decoded(orc, qkv), ost, commit=commit, eps=EPS)
        torch.cuda.synchronize()
        assert err_bf16(g, ref) <= TOL_BF16
        if commit:
            assert err_state(st.S, ost.S) <= TOL_STATE and err_state(st.Z, ost.Z) <= TOL_STATE
        else:
            assert torch.equal(st.S, S0) and torch.equal(st.Z, Z0)
    assert st.blocks_committed == 2
    la.device_status()


def test_nvfp4_state_shared_with_bf16_calls(la, orc):
    """The state is fp32 in real units: an NVFP4 block, then a bf16 block on
    the same state, equals the oracle's stream over the decoded and the bf16
    values."""
    B, H, Nb = 1, 8, 300
    st = la.State(B, H)
    ost = orc.State(B, H, 32)
    qkv = fp4_inputs(B, Nb, H, seed=191)
    la.block_forward_nvfp4(*on_gpu(qkv), st, commit=True, eps=EPS)
    orc.block_forward(*decoded(orc, qkv), ost, commit=True, eps=EPS)
    q, k, v = synth.random_qkv(B, Nb, H, 32, seed=192, dtype=torch.bfloat16)
    g = la.block_forward(q.cuda(), k.cuda(), v.cuda(), st, commit=True, eps=EPS)
    ref = orc.block_forward(q, k, v, ost, commit=True, eps=EPS)
    torch.cuda.synchronize()
    assert err_bf16(g, ref) <= TOL_BF16
    assert err_state(st.S, ost.S) <= TOL_STATE and err_state(st.Z, ost.Z) <= TOL_STATE
    la.device_status()


def test_nvfp4_deterministic(la):
    qkv = on_gpu(fp4_inputs(1, 3000, 8, seed=193))
    a = la.full_forward_nvfp4(*qkv, 700, eps=EPS).clone()
    b = la.full_forward_nvfp4(*qkv, 700, eps=EPS)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_nvfp4_argument_errors(la):
    qkv = on_gpu(fp4_inputs(1, 64, 8, seed=194))
    with pytest.raises(la.LAError) as e:     # H not a multiple of 8
        la.full_forward_nvfp4(*on_gpu(fp4_inputs(1, 64, 4, seed=195)), 0, eps=EPS)
    assert e.value.status == la.LA_EUNSUPPORTED
    bad = [qkv[0], qkv[1], (qkv[2][0], qkv[2][1], 0.0)]   # a per-tensor scale that is not > 0
    with pytest.raises(la.LAError) as e:
        la.full_forward_nvfp4(*bad, 0, eps=EPS)
    assert e.value.status == la.LA_EINVAL
    la.device_status()


def orc_rope(orc, r):
    return orc.make_rope(Hg=r.Hg, Wg=r.Wg, t_offset=r.t_offset, dims=(r.dt, r.dh, r.dw), base=r.base)


# RoPE on the NVFP4 path (the stream-K RoPE kernels decoding codes and block
# scales): ragged tails, multi-block scans, two batches, 2..8 head groups (H 24:
# the last group's scales at the end of a 48-byte row)
@pytest.mark.parametrize("B,N,H,L,grid", [(1, 517, 8, 0, (3, 5)), (2, 300, 8, 128, (3, 5)),
                                          (1, 1000, 24, 250, (4, 10)), (1, 4099, 64, 0, (7, 9)),
                                          (2, 2700, 16, 900, (9, 20))])
def test_full_forward_nvfp4_rope_matches_oracle(la, orc, B, N, H, L, grid):
    qkv = fp4_inputs(B, N, H, seed=260 + N + H)
    rope = la.make_rope(Hg=grid[0], Wg=grid[1], t_offset=2)
    g = la.full_forward_nvfp4(*on_gpu(qkv), L, eps=EPS, rope=rope)
    torch.cuda.synchronize()
    la.device_status()
    assert la.la_last_path() == "tc_nvfp4"
    ref = orc.full_forward(*decoded(orc, qkv), L, rope=orc_rope(orc, rope), eps=EPS)
    assert err_bf16(g, ref) <= tol_bf16_for(ref)


def test_block_forward_nvfp4_rope_streaming(la, orc):
    """Streamed blocks with RoPE positions from the state (t_offset < 0), a
    read-only pass in the middle; outputs and committed state against the
    oracle, t_next advanced by the committed blocks' frames; repeated calls
    give the same bits."""
    B, H, Hg, Wg, F, nb = 2, 8, 3, 50, 3, 3
    Nb = F * Hg * Wg
    st = la.State(B, H)
    ost = orc.State(B, H, 32)
    rope = la.make_rope(Hg=Hg, Wg=Wg, T=F, t_offset=-1)
    frames = 0
    for i in range(nb):
        qkv = fp4_inputs(B, Nb, H, seed=280 + i, scale=0.7, bias=0.05)
        commit = i != 1
        g = la.block_forward_nvfp4(*on_gpu(qkv), st, commit=commit, eps=EPS, rope=rope)
        ref = orc.block_forward(*decoded(orc, qkv), ost, commit=commit, rope=orc.make_rope(Hg=Hg, Wg=Wg, t_offset=frames),
                                eps=EPS)
        torch.cuda.synchronize()
        la.device_status()
        assert err_bf16(g, ref) <= tol_bf16_for(ref)
        assert err_state(st.S, ost.S) <= TOL_STATE and err_state(st.Z, ost.Z) <= TOL_STATE
        if commit:
            frames += F
    assert st.blocks_committed == 2 and st.t_next == 2 * F
    qkv = on_gpu(fp4_inputs(1, 3000, 8, seed=299))
    r2 = la.make_rope(Hg=6, Wg=10, t_offset=0)
    a = la.full_forward_nvfp4(*qkv, 700, eps=EPS, rope=r2).clone()
    b = la.full_forward_nvfp4(*qkv, 700, eps=EPS, rope=r2)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
