"""The longest single head the tests run: B = H = 1, N = 2^20, d = 128, causal, forward and
backward in the bench's launch configuration. O, lse and dQ are compared with the oracle on
sampled rows (each row costs the oracle O(N d)); dV and dK, which would need the oracle's full
N x N forward, are checked through an identity that holds at any size and, through the oracle,
at the last key, which only the last query sees."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import make_inputs
from parity import TOL_GRAD_REL, assert_fwd_ok, fwd_errors, grad_rel_error, to64

pytestmark = pytest.mark.gpu

N, D = 1 << 20, 128


def test_max_length_forward_backward():
    x = make_inputs(1, 1, N, D, seed=2024)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, causal=True)
    fa.fa_check_status()
    for t in (o, lse, dq, dk, dv):
        assert torch.isfinite(t).all()
    scale = fa.default_scale(D)
    rng = np.random.Generator(np.random.PCG64(77))
    idx = sorted(set(rng.choice(N, size=40, replace=False).tolist()) | {0, 1, 4095, N - 1})
    rows = [(0, 0, i) for i in idx]
    qn, kn, vn, don = (x[n].float().numpy() for n in ("q", "k", "v", "do"))
    o_r, lse_r, dq_r = oracle.attention_rows(qn, kn, vn, scale, True, rows, do=don)
    o64, lse64, dq64 = to64(o)[0, 0], to64(lse)[0, 0], to64(dq)[0, 0]
    assert_fwd_ok(fwd_errors(o64[idx], lse64[idx], o_r, lse_r), "N = 2^20 sampled rows")
    assert grad_rel_error(dq64[idx], dq_r) <= TOL_GRAD_REL

    # Rows of P sum to 1, so sum_j dV_j = sum_i dO_i; with bf16 probabilities and outputs each
    # term carries a relative error of about 2^-9, far inside 1e-2 of the sum's magnitude.
    dv_sum = to64(dv)[0, 0].sum(axis=0)
    do_sum = x["do"][0, 0].double().sum(dim=0).numpy()
    assert np.abs(dv_sum - do_sum).max() <= 1e-2 * np.abs(do_sum).max()

    # The last key is seen by the last query only, so the oracle's dK and dV of that key need
    # only row N - 1's output and lse, which attention_rows has just computed.
    t = idx.index(N - 1)
    o_stats = np.full((N, D), np.nan)
    lse_stats = np.full(N, np.nan)
    o_stats[N - 1], lse_stats[N - 1] = o_r[t], lse_r[t]
    dk_last, dv_last = oracle.attention_keys(qn, kn, vn, don, scale, True, (0, 0), [N - 1],
                                             stats=(o_stats, lse_stats))
    assert grad_rel_error(to64(dv)[0, 0, N - 1:], dv_last) <= TOL_GRAD_REL
    assert grad_rel_error(to64(dk)[0, 0, N - 1:], dk_last) <= TOL_GRAD_REL
