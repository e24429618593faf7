"""Failure detection on the GPU without a fault: a bounded in-kernel wait that runs out is
reported to the host as FA_ERR_TIMEOUT, and the context stays usable afterwards.

Two forms. The self-test kernel waits on a barrier that nothing completes. The attention
kernels themselves are driven into their give-up path through the library's test hook
(fa_debug_stall_next): in one launch the TMA producer of every CTA leaves out one tile, so the
MMA warp's wait for it runs out after a short limit; the kernel must then let what it issued
finish, free its tensor memory and return with FA_ERR_TIMEOUT. The next ordinary call on the
same context must give correct results, which it could not if tensor memory had been left
allocated or a copy left in flight."""

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import make_inputs
from parity import assert_fwd_ok, assert_grad_ok, fwd_errors, to64

pytestmark = pytest.mark.gpu


def test_timed_out_wait_is_reported_and_cleared():
    fa.fa_check_status()  # clean start
    fa.fa_selftest_timeout(limit_us=20000)  # a barrier nothing arrives at; gives up after 20 ms
    with pytest.raises(fa.FaError) as e:
        fa.fa_check_status()
    assert e.value.status == 5  # FA_ERR_TIMEOUT
    fa.fa_check_status()  # the word was cleared: no error now


def test_context_usable_after_timeout():
    fa.fa_selftest_timeout(limit_us=5000)
    with pytest.raises(fa.FaError):
        fa.fa_check_status()
    x = make_inputs(1, 1, 256, 64, seed=3, with_do=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v)
    fa.fa_check_status()
    assert torch.isfinite(o).all()


def _expect_timeout():
    with pytest.raises(fa.FaError) as e:
        fa.fa_check_status()
    assert e.value.status == 5, e.value
    fa.fa_check_status()  # cleared


def _check_fwd(x, d, causal, o, lse):
    o_ref, lse_ref = oracle.attention_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]),
                                              fa.default_scale(d), causal)
    assert_fwd_ok(fwd_errors(o, lse, o_ref, lse_ref), f"after timeout d={d}")


@pytest.mark.parametrize("d,causal,skip", [(128, True, 1), (64, False, 0), (128, False, 4)])
def test_forward_kernel_timeout_unwinds(d, causal, skip):
    """fa_fwd_kernel: a K/V tile never arrives; the call reports FA_ERR_TIMEOUT, and the next
    forward on the same context matches the oracle."""
    fa.fa_check_status()
    x = make_inputs(1, 1, 384, d, seed=40 + d + skip, with_do=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    fa.fa_debug_stall_next(0, skip=skip, limit_us=20000)
    fa.attention_forward(q, k, v, causal=causal)
    _expect_timeout()
    o, lse = fa.attention_forward(q, k, v, causal=causal)
    fa.fa_check_status()
    _check_fwd(x, d, causal, o, lse)


@pytest.mark.parametrize("d,causal,skip", [(128, True, 0), (128, False, 1), (64, True, 0),
                                           (64, False, 2), (256, True, 0), (256, False, 1)])
def test_backward_kernel_timeout_unwinds(d, causal, skip):
    """The backward main kernel (the 128-row kernel at d = 128, the 64-row one at d = 64, the dV
    pass at d = 256): a query tile never arrives; the call reports FA_ERR_TIMEOUT, and the next
    backward on the same context matches the oracle."""
    fa.fa_check_status()
    x = make_inputs(1, 2, 384, d, seed=50 + d + skip)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=causal)
    fa.fa_check_status()
    fa.fa_debug_stall_next(2, skip=skip, limit_us=20000)
    fa.attention_backward(q, k, v, o, do, lse, causal=causal)
    _expect_timeout()
    dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, causal=causal)
    fa.fa_check_status()
    ref = oracle.attention_backward(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["do"]),
                                    fa.default_scale(d), causal)
    for g, r, n in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
        assert_grad_ok(g, r, f"after timeout d={d} {n}")


def test_noalloc_backward_timeout_is_readable():
    """fa_bwd_noalloc records a timed-out wait in the status word built into the library;
    fa_check_status reads and clears it too."""
    fa.fa_check_status()
    x = make_inputs(1, 2, 384, 128, seed=60)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    fa.fa_check_status()
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    fa.fa_debug_stall_next(2, skip=0, limit_us=20000)
    fa.fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal=True)
    _expect_timeout()
    fa.fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal=True)
    fa.fa_check_status()
    ref = oracle.attention_backward(to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["do"]),
                                    fa.default_scale(128), True)
    for g, r, n in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
        assert_grad_ok(g, r, f"noalloc after timeout {n}")


def test_stall_hook_is_disarmed_by_one_launch():
    fa.fa_check_status()
    x = make_inputs(1, 1, 256, 64, seed=61, with_do=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    fa.fa_debug_stall_next(0, skip=0, limit_us=5000)
    fa.attention_forward(q, k, v)
    _expect_timeout()
    o, lse = fa.attention_forward(q, k, v)  # disarmed: runs normally
    fa.fa_check_status()
    _check_fwd(x, 64, False, o, lse)
    fa.fa_debug_stall_next(0, skip=0, limit_us=5000)
    fa.fa_debug_stall_next(-1)  # disarm without a launch
    fa.attention_forward(q, k, v)
    fa.fa_check_status()
