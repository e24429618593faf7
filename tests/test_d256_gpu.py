"""Head dimension 256 (forward only) against the fp64 oracle: full comparison on small ragged,
grouped-head and bottom-right shapes (rows that see no key give O = 0, lse = -inf), sampled rows
of a B=2 H=16 N=8192 causal workload, the causal exactness property, and the rejections of the
paths that do not support d = 256."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import WORKLOADS, make_inputs_ex, sampled_rows, workload_inputs
from parity import assert_fwd_ok, fwd_errors, to64

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


def test_d256_rejected_where_unsupported():
    x = make_inputs_ex(1, 1, 1, 128, 128, 256, seed=32)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v)
    with pytest.raises(fa.FaError, match="d <= 128"):
        ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
        fa.fa_bwd_ex(q, k, v, o, do, lse, torch.empty_like(q), torch.empty_like(k),
                     torch.empty_like(v), ws)
    assert fa.fa_bwd_ex_workspace_size(1, 1, 1, 128, 128, 256) == 0
    with pytest.raises(fa.FaError, match="dropout"):
        fa.attention_forward(q, k, v, dropout=(0.1, 1, 0))
    fa.fa_check_status()
