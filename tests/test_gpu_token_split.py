"""GPU parity of the token split of one block over R ranks (la_block_reduce,
la_block_apply), emulated on one GPU by running the R ranks' calls one after
another (no kernel waits on another): the concatenated outputs match the
oracle's unsplit block (bf16 2e-2 / fp32 1e-4 metrics), every emulated rank
commits the same state bit for bit, and that state matches the oracle's."""
import numpy as np
import pytest
import torch

from block_causal_linear_b200 import ranks, synth
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


CASES = [  # dtype, B, N, H, R, rope (Hg, Wg) or None
    (torch.bfloat16, 1, 1000, 8, 3, None),
    (torch.bfloat16, 2, 777, 4, 4, None),
    (torch.float32, 1, 500, 2, 2, None),
    (torch.bfloat16, 1, 6 * 15, 4, 3, (3, 5)),      # 6 frames of 3 x 5, two frames per rank
]


@pytest.mark.parametrize("case", CASES)
def test_token_split_matches_unsplit_block(la, orc, case):
    dtype, B, N, H, R, grid = case
    prior = synth.random_qkv(B, 300, H, 32, seed=5, dtype=dtype)      # one committed block first
    q, k, v = synth.random_qkv(B, N, H, 32, seed=6 + N, dtype=dtype)
    orope = orc.make_rope(Hg=grid[0], Wg=grid[1], t_offset=0) if grid else None
    ost = orc.State(B, H, 32)
    if grid:
        # the prior block: 300 tokens are 20 frames of 3 x 5
        orc.block_forward(*prior, ost, commit=True, rope=orope, eps=EPS)
        orope2 = orc.make_rope(Hg=grid[0], Wg=grid[1], t_offset=300 // (grid[0] * grid[1]))
    else:
        orc.block_forward(*prior, ost, commit=True, eps=EPS)
        orope2 = None
    ref = orc.block_forward(q, k, v, ost, commit=True, rope=orope2, eps=EPS)

    states, outs, partials = [], [], []
    align = grid[0] * grid[1] if grid else 1
    frames0 = 300 // align if grid else 0
    for r in range(R):
        st = la.State(B, H)
        rp = la.make_rope(Hg=grid[0], Wg=grid[1], T=300 // align, t_offset=0) if grid else None
        la.block_forward(*(t.cuda() for t in prior), st, commit=True, rope=rp, eps=EPS)
        states.append(st)
    for r in range(R):
        t0, t1 = ranks.token_slice(N, R, r, align)
        rp = la.make_rope(Hg=grid[0], Wg=grid[1], t_offset=frames0 + t0 // align) if grid else None
        partials.append(la.block_reduce(k[:, t0:t1].contiguous().cuda(), v[:, t0:t1].contiguous().cuda(), rope=rp))
    gathered = torch.stack(partials).contiguous()
    for r in range(R):
        t0, t1 = ranks.token_slice(N, R, r, align)
        rp = la.make_rope(Hg=grid[0], Wg=grid[1], T=N // align, t_offset=frames0 + t0 // align) if grid else None
        outs.append(la.block_apply(q[:, t0:t1].contiguous().cuda(), gathered, states[r], commit=True, rope=rp,
                                   eps=EPS))
    torch.cuda.synchronize()
    la.device_status()
    g = torch.cat(outs, 1)
    assert err_out(g, ref, dtype) <= tol_out(dtype)
    for st in states[1:]:
        assert torch.equal(st.S, states[0].S) and torch.equal(st.Z, states[0].Z)
    assert err_state(states[0].S, ost.S) <= TOL_STATE and err_state(states[0].Z, ost.Z) <= TOL_STATE
    assert all(st.blocks_committed == 2 for st in states)


def test_split_partial_bytes(la):
    assert la.la_split_partial_bytes(2, 64, 32) == 2 * 64 * 1056 * 4
    assert la.la_split_partial_bytes(1, 1, 16) == 0
