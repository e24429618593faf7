"""Dropout on the GPU against the oracle (through fa_fwd_ex / fa_bwd_ex).

The keep decisions are checked exactly: with V (or dO) one-hot per key (or query) block, each
entry of O (or dV) is a single kept-or-dropped probability, so its zero pattern is the keep mask,
which must equal the oracle's Philox mask bit for bit. Values are held to the tolerances without
dropout (the O bounds multiplied by the keep scale r = 256/(256 - p8), which multiplies every
kept weight and its rounding error), on small shapes in full and on the causal B=4 H=16 N=4096
d=128 training workload on sampled rows and keys."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import (WORKLOADS, make_inputs_ex, sampled_keys,
                                              sampled_rows, workload_inputs)
from parity import (TOL_GRAD_REL, assert_fwd_ok, assert_grad_ok, fwd_errors, grad_rel_error,
                    to64)

pytestmark = pytest.mark.gpu

SEED = (0x5EED << 32) | 0x1234  # high word non-zero: both key words matter


def _visible(n_q, n_kv, mode):
    i = np.arange(n_q)[:, None]
    j = np.arange(n_kv)[None, :]
    if mode in (False, "none"):
        return np.ones((n_q, n_kv), bool)
    off = n_kv - n_q if mode == "bottom_right" else 0
    return j <= i + off


@pytest.mark.parametrize("mode", [False, True, "bottom_right"])
@pytest.mark.parametrize("d", [64, 128])
def test_keep_mask_exact_forward(mode, d):
    """O with V one-hot per key block: O[i, j - 128c] == 0 exactly where the oracle drops (i, j)
    or j is not visible to i."""
    B, H, H_kv, N_q, N_kv = 1, 2, 1, 200, 300 if mode == "bottom_right" else 200
    p, off = 0.3, 5
    x = make_inputs_ex(B, H, H_kv, N_q, N_kv, d, seed=900 + d)
    q, k = x["q"].cuda(), x["k"].cuda()
    p8 = oracle.dropout_p8(p)
    vis = _visible(N_q, N_kv, mode)
    for c0 in range(0, N_kv, d):
        v = torch.zeros(B, H_kv, N_kv, d, dtype=torch.bfloat16)
        n = min(d, N_kv - c0)
        v[:, :, c0:c0 + n, :n] = torch.eye(n, dtype=torch.bfloat16)
        o, _ = fa.attention_forward(q, k, v.cuda(), causal=mode, dropout=(p, SEED, off))
        fa.fa_check_status()
        o = o.float().cpu().numpy()
        for h in range(H):
            z = oracle.dropout_keep(h, range(N_q), np.arange(c0, c0 + n), p8, SEED, off)
            expect_nonzero = z & vis[:, c0:c0 + n]
            got_nonzero = o[0, h, :, :n] != 0
            bad = np.argwhere(got_nonzero != expect_nonzero)
            assert bad.size == 0, f"head {h} block {c0}: {len(bad)} mismatches, first {bad[:4]}"


@pytest.mark.parametrize("d", [64, 128])
def test_keep_mask_exact_backward(d):
    """dV with dO one-hot per query block: dV[j, i - 64c] == 0 exactly where (i, j) is dropped
    or masked."""
    B, H, N, p, off = 1, 1, 192, 0.5, 11
    x = make_inputs_ex(B, H, H, N, N, d, seed=950 + d)
    q, k, v = (x[t].cuda() for t in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, causal=True, dropout=(p, SEED, off))
    p8 = oracle.dropout_p8(p)
    vis = _visible(N, N, True)
    for c0 in range(0, N, d):
        do = torch.zeros(B, H, N, d, dtype=torch.bfloat16)
        n = min(d, N - c0)
        do[:, :, c0:c0 + n, :n] = torch.eye(n, dtype=torch.bfloat16)
        _, _, dv = fa.attention_backward(q, k, v, o, do.cuda(), lse, causal=True,
                                         dropout=(p, SEED, off))
        fa.fa_check_status()
        dv = dv.float().cpu().numpy()[0, 0]  # [N keys, d]
        z = oracle.dropout_keep(0, np.arange(c0, c0 + n), N, p8, SEED, off)  # [n queries, N]
        expect = (z & vis[c0:c0 + n]).T  # [N keys, n]
        got = dv[:, :n] != 0
        assert np.array_equal(got, expect), f"block {c0}: {(got != expect).sum()} mismatches"


CASES = [  # (B, H, H_kv, N_q, N_kv, d, mask, p)
    (1, 2, 2, 256, 256, 64, False, 0.1),
    (2, 4, 2, 333, 333, 128, True, 0.25),
    (1, 2, 2, 100, 700, 128, "bottom_right", 0.5),
    (1, 4, 1, 513, 513, 64, True, 0.17),
    (1, 2, 1, 640, 130, 128, False, 0.9),
    (1, 2, 2, 300, 300, 96, True, 0.2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%dh%dkv%dq%dk%dd%d-%s-p%s" % c)
def test_dropout_against_oracle(case):
    B, H, H_kv, N_q, N_kv, d, mask, p = case
    dr = (p, SEED, 3)
    x = make_inputs_ex(B, H, H_kv, N_q, N_kv, d, seed=1000 + N_q + N_kv + d)
    q, k, v, do = (x[t].cuda() for t in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=mask, dropout=dr)
    dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, causal=mask, dropout=dr)
    fa.fa_check_status()
    scale = fa.default_scale(d)
    dq_r, dk_r, dv_r, o_r, lse_r = oracle.attention_backward(
        to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["do"]), scale, mask,
        return_forward=True, dropout=dr)
    r_keep = oracle.keep_scale(oracle.dropout_p8(p))
    assert_fwd_ok(fwd_errors(o, lse, o_r, lse_r), str(case), keep_scale=r_keep)
    for g, r, n in zip((dq, dk, dv), (dq_r, dk_r, dv_r), ("dQ", "dK", "dV")):
        assert_grad_ok(g, r, f"{case} {n}")


def test_dropout_zero_probability_is_no_dropout():
    x = make_inputs_ex(1, 2, 2, 300, 300, 128, seed=5)
    q, k, v, do = (x[t].cuda() for t in ("q", "k", "v", "do"))
    o1, l1 = fa.attention_forward(q, k, v, causal=True)
    o2, l2 = fa.attention_forward(q, k, v, causal=True, dropout=(0.0, 7, 0))
    g1 = fa.attention_backward(q, k, v, o1, do, l1, causal=True)
    g2 = fa.attention_backward(q, k, v, o2, do, l2, causal=True, dropout=(0.0, 7, 0))
    fa.fa_check_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_dropout_deterministic_and_offset_sensitive():
    x = make_inputs_ex(1, 2, 2, 256, 256, 64, seed=6)
    q, k, v = (x[t].cuda() for t in ("q", "k", "v"))
    a, la = fa.attention_forward(q, k, v, dropout=(0.2, 42, 0))
    b, lb = fa.attention_forward(q, k, v, dropout=(0.2, 42, 0))
    c, lc = fa.attention_forward(q, k, v, dropout=(0.2, 42, 1))
    fa.fa_check_status()
    assert torch.equal(a, b) and torch.equal(la, lb)
    assert not torch.equal(a, c)
    assert torch.equal(la, lc)  # lse is that of the undropped softmax


def test_dropout_full_size_sampled():
    """Causal B=4 H=16 N=4096 d=128 with p = 0.1: O, lse and dQ on sampled rows, dK and dV on
    sampled keys, against the oracle's per-row and per-key dropout paths."""
    w = WORKLOADS["causal_train_b4h16n4096d128"]
    dr = (0.1, SEED, 17)
    x = workload_inputs(w)
    q, k, v, do = (x[t].cuda() for t in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=True, dropout=dr)
    dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, causal=True, dropout=dr)
    fa.fa_check_status()
    qn, kn, vn, don = (x[t].float().numpy() for t in ("q", "k", "v", "do"))
    rows = sampled_rows(w, 256)
    o_r, lse_r, dq_r = oracle.attention_rows(qn, kn, vn, w.scale, True, rows, do=don, dropout=dr)
    idx = tuple(np.array(rows).T)
    assert_fwd_ok(fwd_errors(to64(o)[idx], to64(lse)[idx], o_r, lse_r), "N4096 dropout rows",
                  keep_scale=oracle.keep_scale(oracle.dropout_p8(0.1)))
    assert grad_rel_error(to64(dq)[idx], dq_r) <= TOL_GRAD_REL
    sel = sampled_keys(w, 32, max_heads=1)
    b, h = sel[0][:2]
    keys = [j for (_, _, j) in sel]
    dk_r, dv_r = oracle.attention_keys(qn, kn, vn, don, w.scale, True, (b, h), keys, dropout=dr)
    assert grad_rel_error(to64(dk)[b, h, keys], dk_r) <= TOL_GRAD_REL
    assert grad_rel_error(to64(dv)[b, h, keys], dv_r) <= TOL_GRAD_REL
