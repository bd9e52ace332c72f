"""The allocation-free entry point, la_full_forward_static_ws.

It serves callers that cannot allocate device memory themselves (a plug-in
inside a framework that owns every allocation and cannot hand it a
workspace).  Its scratch is a static device array inside the library.  These
tests call it through the C ABI and compare it with la_full_forward (which
takes a caller-allocated workspace) on two calls in a row, with different
inputs, so that a stale scratch from the first call would show up in the
second.  Both entry points run the same plan and the same kernels on the same
inputs, so their outputs must agree bit for bit; one case is also checked
against the fp64 oracle.  This file is collected last on purpose, so that a
run that stops at its first failure has run every other test before it.

The no-allocation check compares the device's free memory before and after a
call (and torch's reserved pool); it assumes that nothing else allocates on
the device meanwhile, as on a GPU leased to this test run alone, and retries
once after a synchronize if the figures moved.
"""
import ctypes

import pytest
import torch

from block_causal_linear_b200 import synth
from tolerances import err_out, tol_out

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


def _static_call(la, q, k, v, out, L, rope=None):
    B, N, H, d = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return la.la_full_forward_static_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        la._dtype_code(q), B, N, H, d, L, rope, EPS, stream)


@pytest.mark.parametrize("dtype,H,L,use_rope", [
    (torch.bfloat16, 64, 0, False),      # the 480p single-block shape of the benchmark
    (torch.bfloat16, 8, 300, True),
    (torch.float32, 4, 100, False),
])
def test_static_scratch_matches_workspace_entry_point_twice(la, orc, dtype, H, L, use_rope):
    N = 8190 if H == 64 else 1000
    rope = la.make_rope(Hg=5, Wg=20, t_offset=1) if use_rope else None
    for call in range(2):
        q, k, v = (t.cuda() for t in synth.random_qkv(1, N, H, 32, seed=500 + 7 * call + H, dtype=dtype))
        want = la.full_forward(q, k, v, L, rope=rope, eps=EPS)
        got = torch.empty_like(q)
        torch.cuda.synchronize()

        def memory():
            return torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()

        before = memory()
        rc = _static_call(la, q, k, v, got, L, rope)
        assert rc == la.LA_OK, la.la_status_string(rc)
        torch.cuda.synchronize()
        if call == 1:
            # the array was set up by the first call; later calls allocate nothing
            after = memory()
            if after != before:          # someone else's allocation: measure once more
                before = memory()
                assert _static_call(la, q, k, v, got, L, rope) == la.LA_OK
                torch.cuda.synchronize()
                after = memory()
            assert after == before
        la.device_status()
        # same plan, same kernels, same inputs: the same bits
        assert torch.equal(got, want), f"call {call}: static scratch differs from the workspace call"
        if H == 64 and call == 1:
            ref = orc.full_forward(q.cpu(), k.cpu(), v.cpu(), L, rope=None, eps=EPS)
            assert err_out(got.cpu(), ref, dtype) <= tol_out(dtype)


def test_static_scratch_rejects_shapes_beyond_its_size(la):
    # 64 x 2000 tokens x 64 heads in blocks of 100: its workspace is far above 16 MiB
    B, N, H, L = 64, 2000, 64, 100
    assert la.la_workspace_size(B, N, H, 32, L) > la.LA_STATIC_WS_BYTES
    q = torch.zeros(B, N, H, 32, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    rc = _static_call(la, q, q, q, out, L)
    assert rc == la.LA_EWORKSPACE
