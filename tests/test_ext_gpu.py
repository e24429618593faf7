"""Parity of the extended shapes against the fp64 oracle, through fa_fwd_ex / fa_bwd_ex:
grouped key/value heads (H a multiple of H_kv, H_kv = 1 included), unequal query and key
lengths, and the causal mask aligned at the top left or at the bottom right.

A query row that sees no key (bottom-right alignment with N_q > N_kv) must give exactly O = 0,
lse = -inf and dQ = 0, and a key that no query sees exactly dK = dV = 0; every other element is
held to the same tolerances as the square case."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import make_inputs_ex
from parity import assert_fwd_ok, assert_grad_ok, fwd_errors, to64

pytestmark = pytest.mark.gpu

CASES = [  # (B, H, H_kv, N_q, N_kv, d, mask)
    (1, 4, 1, 300, 300, 64, False),             # one shared K/V head
    (1, 4, 1, 300, 300, 64, True),
    (2, 8, 2, 513, 513, 128, True),             # grouped heads, ragged
    (1, 6, 3, 200, 200, 128, False),
    (1, 2, 2, 100, 700, 128, "bottom_right"),   # new queries over a longer context
    (1, 2, 1, 1, 1000, 64, "bottom_right"),     # one decoded query
    (1, 1, 1, 257, 1025, 128, "bottom_right"),
    (1, 2, 2, 700, 300, 64, "bottom_right"),    # rows 0..399 see no key
    (1, 1, 1, 300, 1, 128, "bottom_right"),     # only the last row sees the single key
    (1, 2, 2, 200, 600, 64, True),              # keys 200.. seen by no query
    (1, 2, 2, 600, 200, 128, True),
    (1, 3, 1, 130, 900, 128, False),
    (1, 2, 2, 384, 128, 64, False),
    (1, 2, 2, 300, 300, 96, False),             # d = 96: the d = 128 kernels, zero-filled
    (2, 4, 2, 513, 513, 96, True),
    (1, 2, 1, 100, 700, 96, "bottom_right"),
    (1, 2, 2, 200, 600, 128, True),             # d = 128: key tiles 2..4 seen by no query
    (1, 2, 1, 130, 520, 96, True),              # d = 96, grouped: keys 130.. seen by no query
]


def _ids(c):
    return "b%dh%dkv%dq%dk%dd%d-%s" % c


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_ext_fwd_bwd_against_oracle(case):
    B, H, H_kv, N_q, N_kv, d, mask = case
    x = make_inputs_ex(B, H, H_kv, N_q, N_kv, d, seed=500 + N_q + 3 * N_kv + d + H)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=mask)
    dq, dk, dv = fa.attention_backward(q, k, v, o, do, lse, causal=mask)
    fa.fa_check_status()
    scale = fa.default_scale(d)
    dq_r, dk_r, dv_r, o_r, lse_r = oracle.attention_backward(
        to64(x["q"]), to64(x["k"]), to64(x["v"]), to64(x["do"]), scale, mask,
        return_forward=True)

    empty = np.isneginf(lse_r)  # rows that see no key
    o64, lse64, dq64 = to64(o), to64(lse), to64(dq)
    assert np.all(o64[empty] == 0.0), "O of rows that see no key must be 0"
    assert np.all(np.isneginf(lse64[empty])), "lse of rows that see no key must be -inf"
    assert np.all(dq64[empty] == 0.0), "dQ of rows that see no key must be 0"
    live = ~empty
    if live.any():
        assert_fwd_ok(fwd_errors(o64[live], lse64[live], o_r[live], lse_r[live]), _ids(case))
        assert_grad_ok(dq64[live], dq_r[live], f"{_ids(case)} dQ")
    # keys seen by no query: the oracle's dK, dV are exactly 0 there, and so must ours be
    unseen = np.all(dk_r == 0.0, axis=-1) & np.all(dv_r == 0.0, axis=-1)
    dk64, dv64 = to64(dk), to64(dv)
    assert np.all(dk64[unseen] == 0.0) and np.all(dv64[unseen] == 0.0)
    assert_grad_ok(dk64, dk_r, f"{_ids(case)} dK")
    assert_grad_ok(dv64, dv_r, f"{_ids(case)} dV")


def test_ext_square_matches_plain_entry_points():
    """fa_fwd_ex / fa_bwd_ex with H_kv = H, N_q = N_kv and the top-left mask run the same
    kernels as fa_fwd / fa_bwd: the results are bitwise equal."""
    x = make_inputs_ex(2, 3, 3, 333, 333, 128, seed=77)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o1 = torch.empty_like(q)
    l1 = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    fa.fa_fwd(q, k, v, o1, l1, causal=True)
    o2, l2 = fa.attention_forward(q, k, v, causal="top_left")
    ws = torch.empty(fa.fa_bwd_workspace_size(2, 3, 333, 128), dtype=torch.uint8, device=q.device)
    g1 = [torch.empty_like(q) for _ in range(3)]
    fa.fa_bwd(q, k, v, o1, do, l1, *g1, ws, causal=True)
    g2 = fa.attention_backward(q, k, v, o2, do, l2, causal="top_left")
    fa.fa_check_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_ext_bottom_right_equals_top_left_when_square():
    x = make_inputs_ex(1, 2, 2, 200, 200, 64, seed=78)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = fa.attention_forward(q, k, v, causal="top_left")
    o2, l2 = fa.attention_forward(q, k, v, causal="bottom_right")
    fa.fa_check_status()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
