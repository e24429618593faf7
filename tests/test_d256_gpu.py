"""Head dimension 256 against the fp64 oracle: forward and backward compared in full on small
ragged, grouped-head and bottom-right shapes (rows that see no key give O = 0, lse = -inf and
dQ = 0; keys that no query sees give dK = dV = 0), sampled rows and keys of a B=2 H=16 N=8192
causal workload, the causal exactness properties, and the rejections of the paths that do not
support d = 256 (dropout, the FP8 forward)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import (WORKLOADS, make_inputs_ex, sampled_keys, sampled_rows,
                                              workload_inputs)
from parity import TOL_GRAD_REL, assert_fwd_ok, assert_grad_ok, fwd_errors, grad_rel_error, to64

pytestmark = pytest.mark.gpu

CASES = [  # (B, H, H_kv, N_q, N_kv, mask)
    (1, 1, 1, 1, 1, False),
    (1, 2, 2, 300, 300, False),
    (1, 2, 2, 300, 300, True),
    (2, 4, 2, 513, 513, True),
    (1, 2, 1, 100, 700, "bottom_right"),
    (1, 2, 2, 700, 300, "bottom_right"),
    (1, 3, 1, 1, 1000, "bottom_right"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%dh%dkv%dq%dk%d-%s" % c)
def test_d256_forward_against_oracle(case):
    B, H, H_kv, N_q, N_kv, mask = case
    x = make_inputs_ex(B, H, H_kv, N_q, N_kv, 256, seed=3000 + N_q + N_kv)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, causal=mask)
    fa.fa_check_status()
    o_r, lse_r = oracle.attention_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]),
                                          fa.default_scale(256), mask)
    o64, l64 = to64(o), to64(lse)
    empty = np.isneginf(lse_r)
    assert np.all(o64[empty] == 0) and np.all(np.isneginf(l64[empty]))
    assert_fwd_ok(fwd_errors(o64[~empty], l64[~empty], o_r[~empty], lse_r[~empty]), str(case))


def test_d256_full_size_sampled_rows():
    w = WORKLOADS["causal_fwd_b2h16n8192d256"]
    x = workload_inputs(w)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    fa.fa_check_status()
    rows = sampled_rows(w, w.row_samples)
    qn, kn, vn = (x[n].float().numpy() for n in ("q", "k", "v"))
    o_r, lse_r = oracle.attention_rows(qn, kn, vn, w.scale, True, rows)
    idx = tuple(np.array(rows).T)
    assert_fwd_ok(fwd_errors(to64(o)[idx], to64(lse)[idx], o_r, lse_r), "B2 H16 N8192 d256 rows")


def test_d256_causal_masked_keys_have_no_effect():
    x = make_inputs_ex(1, 2, 2, 384, 384, 256, seed=31)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = fa.attention_forward(q, k, v, causal=True)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 200:] = torch.randn_like(k2[:, :, 200:].float()).to(torch.bfloat16) * 4
    v2[:, :, 200:] = torch.randn_like(v2[:, :, 200:].float()).to(torch.bfloat16) * 4
    o2, l2 = fa.attention_forward(q, k2, v2, causal=True)
    fa.fa_check_status()
    assert torch.equal(o1[:, :, :200], o2[:, :, :200]) and torch.equal(l1[:, :, :200], l2[:, :, :200])
    assert torch.equal(o1[0, 0, 0], v[0, 0, 0])  # row 0 sees key 0 only


BWD_CASES = CASES + [  # (B, H, H_kv, N_q, N_kv, mask)
    (1, 2, 2, 200, 600, True),      # key tiles 2..4 seen by no query
    (1, 2, 2, 1000, 1000, False),   # several tiles in both directions, ragged
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "b%dh%dkv%dq%dk%d-%s" % c)
def test_d256_backward_against_oracle(case):
    B, H, H_kv, N_q, N_kv, mask = case
    x = make_inputs_ex(B, H, H_kv, N_q, N_kv, 256, seed=3100 + N_q + N_kv + H)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=mask)
    dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, causal=mask)
    fa.fa_check_status()
    dq_r, dk_r, dv_r, _, lse_r = oracle.attention_backward(
        to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["do"]), fa.default_scale(256), mask,
        return_forward=True)
    dq64, dk64, dv64 = to64(dq), to64(dk), to64(dv)
    empty_rows = np.isneginf(lse_r)  # rows that see no key
    assert np.all(dq64[empty_rows] == 0.0), "dQ of rows that see no key must be 0"
    unseen = np.all(dk_r == 0.0, axis=-1) & np.all(dv_r == 0.0, axis=-1)
    assert np.all(dk64[unseen] == 0.0) and np.all(dv64[unseen] == 0.0)
    for g, r, n in ((dq64, dq_r, "dQ"), (dk64, dk_r, "dK"), (dv64, dv_r, "dV")):
        if np.abs(r).max() == 0.0:
            # e.g. N = 1: P = 1 and dS = dP - D = 0 exactly, so dQ = dK = 0; the kernels form
            # dP on the tensor core and D in the preprocess, two fp32 sums of the same products
            # in different orders, so what is left is their rounding difference
            assert np.abs(g).max() <= 1e-4, f"{case} {n}: {np.abs(g).max():.3e}"
        else:
            assert_grad_ok(g, r, f"{case} {n}")


def test_d256_backward_full_size_sampled():
    """B=2, H=16, N=8192, d=256 causal in the bench's launch configuration: dQ on 256 sampled
    rows, dK and dV on 64 sampled keys of 2 seeded heads."""
    w = WORKLOADS["causal_train_b2h16n8192d256"]
    x = workload_inputs(w)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, causal=True)
    fa.fa_check_status()
    for g in (dq, dk, dv):
        assert torch.isfinite(g).all()
    qn, kn, vn, don = (x[n].float().numpy() for n in ("q", "k", "v", "do"))
    rows = sampled_rows(w, w.row_samples)
    _, _, dq_r = oracle.attention_rows(qn, kn, vn, w.scale, True, rows, do=don)
    idx = tuple(np.array(rows).T)
    assert grad_rel_error(to64(dq)[idx], dq_r) <= TOL_GRAD_REL
    keys = sampled_keys(w, w.key_samples, max_heads=2)
    dk64, dv64 = to64(dk), to64(dv)
    for head in sorted({(b, h) for b, h, _ in keys}):
        js = [jj for b, h, jj in keys if (b, h) == head]
        dk_r, dv_r = oracle.attention_keys(qn, kn, vn, don, w.scale, True, head, js)
        assert grad_rel_error(dk64[head][js], dk_r) <= TOL_GRAD_REL, f"dK head {head}"
        assert grad_rel_error(dv64[head][js], dv_r) <= TOL_GRAD_REL, f"dV head {head}"


def test_d256_causal_masked_queries_have_no_effect():
    """Changing Q and dO rows i < j0 leaves dK and dV rows >= j0 bit-identical."""
    x = make_inputs_ex(1, 2, 2, 640, 640, 256, seed=33)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    _, dk1, dv1 = fa.attention_backward(q, k, v, o, do, lse, causal=True)
    j0 = 333
    q2, do2 = q.clone(), do.clone()
    q2[:, :, :j0] = torch.randn_like(q2[:, :, :j0].float()).to(torch.bfloat16) * 2
    do2[:, :, :j0] = torch.randn_like(do2[:, :, :j0].float()).to(torch.bfloat16) * 2
    _, dk2, dv2 = fa.attention_backward(q2, k, v, o, do2, lse, causal=True)
    fa.fa_check_status()
    assert torch.equal(dk1[:, :, j0:], dk2[:, :, j0:])
    assert torch.equal(dv1[:, :, j0:], dv2[:, :, j0:])
    assert not torch.equal(dk1[:, :, :j0], dk2[:, :, :j0])


def test_d256_rejected_where_unsupported():
    x = make_inputs_ex(1, 1, 1, 128, 128, 256, seed=32)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v)
    assert fa.fa_bwd_ex_workspace_size(1, 1, 1, 128, 128, 256) > 0
    with pytest.raises(fa.FaError, match="dropout"):
        fa.attention_forward(q, k, v, dropout=(0.1, 1, 0))
    with pytest.raises(fa.FaError, match="dropout"):
        fa.attention_backward(q, k, v, o, do, lse, dropout=(0.1, 1, 0))
    fa.fa_check_status()
