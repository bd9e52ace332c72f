"""The bounded waits on the GPU: a kernel whose mbarrier wait can never
complete (la_selftest_bounded_wait: nothing arrives at its barrier) gives up
after the waits' time limit, raises the device flag and returns; the host
reads LA_ETIMEOUT from la_device_status, the flag is cleared, and the
context stays usable (a forward call afterwards matches the oracle).  No
fault, trap or hang is involved."""
import time

import pytest
import torch

from block_causal_linear_b200 import synth
from tolerances import err_bf16, TOL_BF16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def la():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_causal_linear_b200 import build

    build.build()
    from block_causal_linear_b200 import la as _la

    return _la


def test_wait_gives_up_and_is_reported(la, orc):
    la.device_status()   # nothing pending before the test
    t0 = time.monotonic()
    la.selftest_bounded_wait()
    with pytest.raises(la.LAError) as e:
        la.device_status()
    waited = time.monotonic() - t0
    assert e.value.status == la.LA_ETIMEOUT
    assert 1.0 < waited < 60.0   # the wait's own limit (2 s), not a hang
    la.device_status()   # the flag was cleared

    # the context is still usable
    q, k, v = synth.random_qkv(1, 300, 4, 32, seed=5, dtype=torch.bfloat16)   # tensor-core path
    out = la.full_forward(q.cuda(), k.cuda(), v.cuda(), 0)
    torch.cuda.synchronize()
    la.device_status()
    ref = orc.full_forward(q.float(), k.float(), v.float(), 0)
    assert err_bf16(out, ref) <= TOL_BF16
