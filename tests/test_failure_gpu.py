"""Failure detection on the device without a fault: a bounded wait that runs out records
its error bit, the host reads it through sol_device_errors, and the context stays usable
(sol_selftest_wait_timeout waits on an mbarrier phase that can never complete, with the
same bounded helper the kernels use for their own copies)."""
from __future__ import annotations

import pytest
import torch

from dit_block_b200 import sol, workloads as wl
from parity_util import assert_close, to_f64, to_oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_stays_usable(oracle_mod):
    sol.lib()
    assert sol.device_errors(clear=True) & 4 == 0
    sol.selftest_wait_timeout(polls=8)
    torch.cuda.synchronize()
    flags = sol.device_errors()
    assert flags & 4, f"the wait did not give up (flags {flags:#x})"
    assert sol.device_errors(clear=True) & 4 and sol.device_errors() == 0
    # the context is intact: an op still runs and matches the oracle
    w = wl.WORKLOADS["tiny"]
    u = wl.activation(w, "u", 32, 2 * w.inner, "cuda")
    out = torch.empty((32, w.inner), dtype=u.dtype, device="cuda")
    sol.swiglu(out, u, inner=w.inner)
    torch.cuda.synchronize()
    assert_close(to_f64(out), oracle_mod.swiglu(to_oracle(u), w.inner), u.dtype, "swiglu after the self-test")
    assert sol.device_errors() == 0
