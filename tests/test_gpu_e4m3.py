"""GPU parity of the FP8 E4M3 path (la_full_forward_e4m3, la_block_forward_e4m3)
against the fp64 oracle run on the decoded inputs (oracle.e4m3_decode: code
values times the per-tensor scale), element by element, bf16-output
tolerance (max |g - o| / RMS(o) <= 2e-2); the state after commit within the
state tolerance; bitwise determinism."""
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


def fp8_inputs(B, N, H, seed, scale=1.0, bias=0.0):
    q, k, v = synth.random_qkv(B, N, H, 32, seed=seed, scale=scale, bias=bias)
    return [synth.to_e4m3(t) for t in (q, k, v)]


def decoded(orc, qkv):
    return [orc.e4m3_decode(c, s) for c, s in qkv]


# (2, 300, 8, 0): one block of 5 splits per head group, combined inside the reduce (a cluster)
@pytest.mark.parametrize("B,N,H,L", [(1, 517, 4, 0), (2, 300, 8, 128), (1, 1000, 12, 250), (1, 4099, 64, 0),
                                     (2, 300, 8, 0)])
def test_full_forward_e4m3_matches_oracle(la, orc, B, N, H, L):
    qkv = fp8_inputs(B, N, H, seed=60 + N)
    codes = [c.cuda() for c, _ in qkv]
    scales = [s for _, s in qkv]
    g = la.full_forward_e4m3(*codes, scales, L, eps=EPS)
    torch.cuda.synchronize()
    la.device_status()
    assert la.la_last_path() == "tc_e4m3"
    ref = orc.full_forward(*decoded(orc, qkv), L, eps=EPS)
    assert err_bf16(g, ref) <= TOL_BF16


def test_block_forward_e4m3_streaming(la, orc):
    B, H, Nb, nb = 1, 8, 400, 3
    st = la.State(B, H)
    ost = orc.State(B, H, 32)
    for i in range(nb):
        qkv = fp8_inputs(B, Nb, H, seed=80 + i, scale=0.7, bias=0.05)
        codes = [c.cuda() for c, _ in qkv]
        commit = i != 1          # the middle call is read-only
        g = la.block_forward_e4m3(*codes, [s for _, s in qkv], st, commit=commit, eps=EPS)
        ref = orc.block_forward(*decoded(orc, qkv), ost, commit=commit, eps=EPS)
        torch.cuda.synchronize()
        assert err_bf16(g, ref) <= TOL_BF16
        assert err_state(st.S, ost.S) <= TOL_STATE and err_state(st.Z, ost.Z) <= TOL_STATE
    assert st.blocks_committed == 2


def test_e4m3_deterministic(la):
    qkv = fp8_inputs(1, 3000, 8, seed=91)
    codes = [c.cuda() for c, _ in qkv]
    scales = [s for _, s in qkv]
    a = la.full_forward_e4m3(*codes, scales, 700, eps=EPS).clone()
    b = la.full_forward_e4m3(*codes, scales, 700, eps=EPS)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def orc_rope(orc, r):
    return orc.make_rope(Hg=r.Hg, Wg=r.Wg, t_offset=r.t_offset, dims=(r.dt, r.dh, r.dw), base=r.base)


# RoPE on the E4M3 path (the stream-K RoPE kernels on codes): several tiles and
# a ragged tail, multi-block scans, two batches, head counts of 1..16 groups
@pytest.mark.parametrize("B,N,H,L,grid", [(1, 517, 4, 0, (3, 5)), (2, 300, 8, 128, (3, 5)),
                                          (1, 1000, 12, 250, (4, 10)), (1, 4099, 64, 0, (7, 9)),
                                          (2, 2700, 8, 900, (9, 20))])
def test_full_forward_e4m3_rope_matches_oracle(la, orc, B, N, H, L, grid):
    qkv = fp8_inputs(B, N, H, seed=160 + N)
    codes = [c.cuda() for c, _ in qkv]
    scales = [s for _, s in qkv]
    rope = la.make_rope(Hg=grid[0], Wg=grid[1], t_offset=2)
    g = la.full_forward_e4m3(*codes, scales, L, eps=EPS, rope=rope)
    torch.cuda.synchronize()
    la.device_status()
    assert la.la_last_path() == "tc_e4m3"
    ref = orc.full_forward(*decoded(orc, qkv), L, rope=orc_rope(orc, rope), eps=EPS)
    assert err_bf16(g, ref) <= tol_bf16_for(ref)


def test_block_forward_e4m3_rope_streaming(la, orc):
    """Streamed blocks with RoPE positions from the state (t_offset < 0), a
    read-only pass in the middle; outputs and committed state against the
    oracle, and t_next advanced by the committed blocks' frames."""
    B, H, Hg, Wg, F, nb = 2, 8, 3, 50, 3, 3
    Nb = F * Hg * Wg
    st = la.State(B, H)
    ost = orc.State(B, H, 32)
    rope = la.make_rope(Hg=Hg, Wg=Wg, T=F, t_offset=-1)
    frames = 0
    for i in range(nb):
        qkv = fp8_inputs(B, Nb, H, seed=180 + i, scale=0.7, bias=0.05)
        codes = [c.cuda() for c, _ in qkv]
        commit = i != 1
        g = la.block_forward_e4m3(*codes, [s for _, s in qkv], st, commit=commit, eps=EPS, rope=rope)
        ref = orc.block_forward(*decoded(orc, qkv), ost, commit=commit, rope=orc.make_rope(Hg=Hg, Wg=Wg, t_offset=frames),
                                eps=EPS)
        torch.cuda.synchronize()
        la.device_status()
        assert err_bf16(g, ref) <= tol_bf16_for(ref)
        assert err_state(st.S, ost.S) <= TOL_STATE and err_state(st.Z, ost.Z) <= TOL_STATE
        if commit:
            frames += F
    assert st.blocks_committed == 2 and st.t_next == 2 * F


def test_e4m3_rope_deterministic(la, orc):
    """Repeated E4M3 RoPE calls over a 5-block scan give the same bits, and
    match the oracle on the decoded values."""
    qkv = fp8_inputs(1, 3000, 8, seed=191)
    codes = [c.cuda() for c, _ in qkv]
    scales = [s for _, s in qkv]
    rope = la.make_rope(Hg=6, Wg=10, t_offset=0)
    a = la.full_forward_e4m3(*codes, scales, 700, eps=EPS, rope=rope).clone()
    b = la.full_forward_e4m3(*codes, scales, 700, eps=EPS, rope=rope)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    dec = [orc.e4m3_decode(c, s) for c, s in qkv]
    ref = orc.full_forward(*dec, 700, rope=orc_rope(orc, rope), eps=EPS)
    assert err_bf16(a, ref) <= tol_bf16_for(ref)
