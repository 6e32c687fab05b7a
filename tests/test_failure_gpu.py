"""Failure detection without a GPU fault.

Every wait of the library's kernels on an mbarrier is bounded; when a wait
gives up it records where in a device error word and the kernel unwinds.
blasst_selftest_wait_timeout launches a kernel whose wait cannot complete
(nothing arrives at the barrier) with a short limit; the host must then see
BLASST_ERR_TIMEOUT naming that wait, the error word must clear on reading,
and the context must stay usable for a normal decode call.  Nothing traps or
hangs.
"""
import math

import pytest
import torch

from synth import config_seed, planted_gap

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import dynamic_block_sparse_fa_b200 as m
    st, where = m.blasst_check_device_error()
    assert st == 0
    m.blasst_selftest_wait_timeout(2_000_000)  # ~1 ms of SM clock
    st, where = m.blasst_check_device_error()
    assert st == 5, "the bounded wait did not report a timeout"
    assert str(where).startswith("99"), where
    # the error word was cleared by reading it
    st, _ = m.blasst_check_device_error()
    assert st == 0
    # and the context still runs kernels correctly
    x = planted_gap(1, 8, 2, 1, 2048, 128, decode=True, block=64,
                    seed=config_seed(1, 99), device="cuda")
    o, lse = m.blasst_decode(x.q, x.k, x.v, ln_lambda=-4.0)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    assert m.blasst_check_device_error()[0] == 0


def test_selftest_rejects_bad_limits():
    import dynamic_block_sparse_fa_b200 as m
    with pytest.raises(m.BlasstError, match="INVALID_ARG"):
        m.blasst_selftest_wait_timeout(0)
    with pytest.raises(m.BlasstError, match="INVALID_ARG"):
        m.blasst_selftest_wait_timeout(10 ** 12)
