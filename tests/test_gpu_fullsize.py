"""Full-size parity: the five workloads at their full sizes, in the launch
configuration the benchmark times (block_causal_linear_b200.runner), against
the fp64 oracle on sampled heads.  Heads are independent in this method, so
the oracle runs the same call sequence on a subset of heads with its own
fp64 state; every token of those heads is compared."""
import numpy as np
import pytest
import torch

from block_causal_linear_b200 import synth
from tolerances import TOL_STATE, err_out, err_state, tol_out

pytestmark = pytest.mark.gpu

SAMPLED_HEADS = {1: None, 2: None, 3: [0, 13, 31, 47, 63], 4: [1, 22, 40, 63], 5: [5, 58]}


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_causal_linear_b200 import build

    build.build()
    from block_causal_linear_b200 import la as _la

    return _la


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_workload_full_size(la, orc, cfg):
    from block_causal_linear_b200.runner import Runner, host_heads

    w = synth.WORKLOADS[cfg]
    heads = SAMPLED_HEADS[cfg] or list(range(w.H))
    dtype = w.torch_dtype
    r = Runner(w, "cuda")
    r.step()
    torch.cuda.synchronize()
    la.device_status()
    H = len(heads)
    ost = orc.State(w.B, H, w.d)
    worst = 0.0
    for i, (blk, p, q, k, v) in enumerate(r.calls):
        qh, kh, vh = host_heads(q, heads), host_heads(k, heads), host_heads(v, heads)
        gh = host_heads(r.outs[i], heads)
        if w.mode == "full":
            rope = orc.make_rope(Hg=w.Hg, Wg=w.Wg, t_offset=0, dims=w.rope_dims, base=w.rope_base) if w.rope else None
            ref = orc.full_forward(qh, kh, vh, r.tokens_per_block, rope=rope, eps=w.eps)
        else:
            rope = orc.make_rope(Hg=w.Hg, Wg=w.Wg, t_offset=blk * w.frames, dims=w.rope_dims,
                                 base=w.rope_base) if w.rope else None
            ref = orc.block_forward(qh, kh, vh, ost, commit=(p == w.passes - 1), rope=rope, eps=w.eps)
        e = err_out(gh, ref, dtype)
        worst = max(worst, e)
        assert e <= tol_out(dtype), f"call {i} (block {blk}, pass {p}): error {e}"
    if w.mode == "stream":
        hs = torch.as_tensor(heads, device="cuda")
        assert err_state(r.state.S.index_select(1, hs), ost.S) <= TOL_STATE
        assert err_state(r.state.Z.index_select(1, hs), ost.Z) <= TOL_STATE
        assert r.state.blocks_committed == w.n_blocks
    print(f"config {cfg} ({w.name}): worst error {worst:.3e} over {len(r.calls)} calls, {H} heads")
