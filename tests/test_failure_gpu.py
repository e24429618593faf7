"""Failure detection on the GPU without a fault: a bounded in-kernel wait that runs out is
reported to the host as FA_ERR_TIMEOUT, and the context stays usable afterwards."""

import pytest
import torch

from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import make_inputs

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
