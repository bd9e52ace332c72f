"""Checkpoint and resume of a stream through the C ABI (la_state_save,
la_state_restore).  The fixed-size state is the method's whole memory of the
past ("Nvidia, MIT ve diğerleri video yapay zeka devrimini başlattı", section
"Sabit Bellekli KV önbelleğe alma mekanizması"), so streaming 24 blocks must
give, bit for bit, what streaming 12 blocks, saving S, Z and the counters to
pinned host memory, restoring them into fresh device buffers and streaming 12
more gives.  With RoPE the restored t_next places the later blocks' frames."""
import pytest
import torch

from block_causal_linear_b200 import synth

pytestmark = pytest.mark.gpu
EPS = 1e-6
NB = 24


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_causal_linear_b200 import build

    build.build()
    from block_causal_linear_b200 import la as _la

    return _la


@pytest.mark.parametrize("dtype,H,use_rope", [
    (torch.bfloat16, 8, True),      # tensor cores, RoPE positions from t_next
    (torch.bfloat16, 64, False),    # tensor cores, the benchmark's head count
    (torch.float32, 2, False),      # CUDA cores
])
def test_stream_resumes_bitwise_from_a_checkpoint(la, dtype, H, use_rope):
    B, T, Hg, Wg = 1, 3, 5, 20
    n_blk = T * Hg * Wg
    rope = la.make_rope(Hg=Hg, Wg=Wg, T=T, t_offset=-1) if use_rope else None
    blocks = [tuple(t.cuda() for t in synth.random_qkv(B, n_blk, H, 32, seed=900 + n, dtype=dtype))
              for n in range(NB)]

    def stream_blocks(st, idx):
        return [la.block_forward(*blocks[n], st, commit=True, rope=rope, eps=EPS) for n in idx]

    ref_state = la.State(B, H)
    ref_out = stream_blocks(ref_state, range(NB))

    st = la.State(B, H)
    stream_blocks(st, range(NB // 2))
    S_host = torch.empty(st.S.shape, dtype=torch.float32).pin_memory()
    Z_host = torch.empty(st.Z.shape, dtype=torch.float32).pin_memory()
    counters = st.save(S_host, Z_host)
    torch.cuda.synchronize()
    assert counters.blocks_committed == NB // 2
    assert counters.t_next == (NB // 2) * T if use_rope else counters.t_next == 0
    del st

    resumed = la.State(B, H)           # fresh buffers, zero state, counters 0
    resumed.restore(S_host, Z_host, counters)
    assert resumed.blocks_committed == NB // 2
    out = stream_blocks(resumed, range(NB // 2, NB))
    torch.cuda.synchronize()
    la.device_status()
    for i, n in enumerate(range(NB // 2, NB)):
        assert torch.equal(out[i], ref_out[n]), f"block {n}"
    assert torch.equal(resumed.S, ref_state.S)
    assert torch.equal(resumed.Z, ref_state.Z)
    assert resumed.blocks_committed == ref_state.blocks_committed == NB
    assert resumed.t_next == ref_state.t_next
