"""The bounded-wait error path on the GPU: a wait on a barrier that nothing
completes gives up after its limit (about one second), records bit 0 of the
library's error word, and leaves the context usable, so that a decode right
after it matches the oracle.  The failure is made on purpose the safe way: a
barrier nothing arrives on, no trap, no bad address."""
import time

import numpy as np
import pytest
import torch

import fp8_kv_paged_kvq_b200 as kvq
from tests import oracle_side as OS
from tests.test_gpu_parity import SPECS, assert_decode_close, build_both

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    torch.cuda.synchronize()
    kvq.device_error()                              # start from a clear word
    flag = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    t0 = time.monotonic()
    kvq.wait_timeout_check(flag)
    torch.cuda.synchronize()
    dt = time.monotonic() - t0
    assert int(flag.item()) == 1
    assert 0.9 < dt < 30.0, dt
    assert kvq.device_error() & 1
    assert kvq.device_error() == 0                  # read and cleared
    for name in ("tiny", "wide_ps64"):
        wl, db, oc = build_both(SPECS[name], seed=21)
        out, lse = db.step(check_tags=False)
        torch.cuda.synchronize()
        ro, rl = OS.decode(wl, oc)
        assert_decode_close(out, lse, ro.reshape(out.shape), rl.reshape(lse.shape), name)
    assert kvq.device_error() == 0
