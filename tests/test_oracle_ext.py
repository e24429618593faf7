"""Pins for the oracle's extended cases (CPU only): unequal query/key lengths with the
bottom-right causal alignment, query rows that see no key, and grouped key/value heads.

Independent references: torch's fp64 scaled_dot_product_attention with enable_gqa and with
the causal_lower_right bias (library special cases, with autograd for the gradients), closed
reductions to the already-pinned modes, pure-Python brute force, finite differences and a
hand-worked fixture. Planted mistakes (wrong head mapping, flipped offset) must fail a pin.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest

from oracle import attention_backward, attention_forward, attention_keys, attention_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _close(a, b, tol, what):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = np.max(np.abs(a - b) / (1 + np.abs(b))) if a.size else 0.0
    assert err <= tol, f"{what}: {err:.3e}"


def _torch_ref(q, k, v, do, scale, mode):
    import torch
    import torch.nn.functional as F
    from torch.nn.attention.bias import causal_lower_right, causal_upper_left

    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    group = q.shape[1] // k.shape[1]
    kk, vv = tk.repeat_interleave(group, 1), tv.repeat_interleave(group, 1)
    if mode == "none":
        o = F.scaled_dot_product_attention(tq, tk, tv, scale=scale, enable_gqa=True)
    else:
        bias = (causal_lower_right if mode == "bottom_right" else causal_upper_left)(
            q.shape[2], k.shape[2])
        o = F.scaled_dot_product_attention(tq, kk, vv, attn_mask=bias, scale=scale)
    o.backward(torch.tensor(do))
    return (o.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy())


def _impl_oracle(q, k, v, do, scale, mode):
    o, _ = attention_forward(q, k, v, scale, mode)
    dq, dk, dv = attention_backward(q, k, v, do, scale, mode)
    return o, dq, dk, dv


@pytest.mark.parametrize("mode", ["none", "top_left", "bottom_right"])
@pytest.mark.parametrize("hq,hkv,nq,nk", [(4, 2, 9, 13), (4, 1, 13, 13), (2, 2, 5, 11), (6, 3, 1, 7)])
def test_torch_sdpa_grouped_heads_and_masks(mode, hq, hkv, nq, nk):
    if mode == "top_left" and nq != nk:
        pytest.skip("top-left alignment is defined here for N_q = N_k")
    q, do = _rand((2, hq, nq, 8), 1), _rand((2, hq, nq, 8), 2)
    k, v = _rand((2, hkv, nk, 8), 3), _rand((2, hkv, nk, 8), 4)
    ref = _torch_ref(q, k, v, do, 0.3, mode)
    got = _impl_oracle(q, k, v, do, 0.3, mode)
    for g, r, n in zip(got, ref, ("O", "dQ", "dK", "dV")):
        _close(g, r, 1e-11, f"{mode} {n}")


def test_bottom_right_with_empty_rows_matches_torch_on_visible_rows():
    """N_q > N_k: the first N_q - N_k rows see no key. The oracle's reading: O = 0,
    lse = -inf, no gradient; the remaining rows match torch's lower-right bias."""
    hq, hkv, nq, nk = 2, 2, 10, 6
    q, do = _rand((1, hq, nq, 4), 5), _rand((1, hq, nq, 4), 6)
    k, v = _rand((1, hkv, nk, 4), 7), _rand((1, hkv, nk, 4), 8)
    o, lse = attention_forward(q, k, v, 0.5, "bottom_right")
    empty = nq - nk
    assert np.all(o[:, :, :empty] == 0.0) and np.all(np.isneginf(lse[:, :, :empty]))
    dq, dk, dv = attention_backward(q, k, v, do, 0.5, "bottom_right")
    assert np.all(dq[:, :, :empty] == 0.0)
    # torch on the visible rows only: drop the empty rows (they contribute nothing)
    ref = _torch_ref(q[:, :, empty:], k, v, do[:, :, empty:], 0.5, "bottom_right")
    _close(o[:, :, empty:], ref[0], 1e-11, "O")
    _close(dq[:, :, empty:], ref[1], 1e-11, "dQ")
    _close(dk, ref[2], 1e-11, "dK")
    _close(dv, ref[3], 1e-11, "dV")


def test_reductions_of_bottom_right():
    """N_q = N_k: bottom-right is top-left. N_q = 1: the single row sees every key."""
    q, k, v = _rand((1, 2, 12, 5), 9), _rand((1, 2, 12, 5), 10), _rand((1, 2, 12, 5), 11)
    for a, b in zip(attention_forward(q, k, v, 0.4, "bottom_right"),
                    attention_forward(q, k, v, 0.4, "top_left")):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(attention_forward(q[:, :, :1], k, v, 0.4, "bottom_right"),
                    attention_forward(q[:, :, :1], k, v, 0.4, "none")):
        np.testing.assert_array_equal(a, b)


def test_grouped_heads_equal_repeated_heads():
    """A key/value head shared by g query heads gives the same O as g copies of it, and its
    gradient is the sum of the copies' gradients."""
    q, do = _rand((2, 6, 7, 3), 12), _rand((2, 6, 7, 3), 13)
    k, v = _rand((2, 2, 9, 3), 14), _rand((2, 2, 9, 3), 15)
    kr, vr = np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1)
    for mode in ("none", "bottom_right"):
        o1, l1 = attention_forward(q, k, v, 0.7, mode)
        o2, l2 = attention_forward(q, kr, vr, 0.7, mode)
        _close(o1, o2, 1e-14, "O")
        _close(l1, l2, 1e-14, "lse")
        g1 = attention_backward(q, k, v, do, 0.7, mode)
        g2 = attention_backward(q, kr, vr, do, 0.7, mode)
        _close(g1[0], g2[0], 1e-13, "dQ")
        _close(g1[1], g2[1].reshape(2, 2, 3, 9, 3).sum(2), 1e-13, "dK")
        _close(g1[2], g2[2].reshape(2, 2, 3, 9, 3).sum(2), 1e-13, "dV")


def test_brute_force_offsets_and_groups():
    rng = np.random.default_rng(16)
    for nq, nk in ((1, 3), (2, 4), (4, 2), (3, 3)):
        q = rng.standard_normal((1, 2, nq, 2))
        k, v = rng.standard_normal((1, 1, nk, 2)), rng.standard_normal((1, 1, nk, 2))
        o, lse = attention_forward(q, k, v, 0.9, "bottom_right")
        for h in range(2):
            for i in range(nq):
                w = [math.exp(0.9 * float(q[0, h, i] @ k[0, 0, j])) if j <= i + nk - nq else 0.0
                     for j in range(nk)]
                tot = sum(w)
                if tot == 0:
                    assert np.all(o[0, h, i] == 0) and lse[0, h, i] == -np.inf
                    continue
                ref = [sum(w[j] * float(v[0, 0, j, c]) for j in range(nk)) / tot for c in range(2)]
                _close(o[0, h, i], ref, 1e-14, "brute O")
                _close(lse[0, h, i], math.log(tot), 1e-14, "brute lse")


def test_finite_differences_offsets_and_groups():
    h = 1e-6
    q, do = _rand((1, 4, 5, 3), 17), _rand((1, 4, 5, 3), 18)
    k, v = _rand((1, 2, 7, 3), 19), _rand((1, 2, 7, 3), 20)
    grads = attention_backward(q, k, v, do, 0.6, "bottom_right")
    for which, g in enumerate(grads):
        x = [q, k, v][which]
        fd = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            lp = np.sum(do * attention_forward(*args_p, 0.6, "bottom_right")[0])
            lm = np.sum(do * attention_forward(*args_m, 0.6, "bottom_right")[0])
            fd[idx] = (lp - lm) / (2 * h)
        assert np.max(np.abs(g - fd)) / np.max(np.abs(fd)) <= 1e-6


def test_golden_bottom_right():
    with open(os.path.join(GOLDEN, "bottom_right_mask.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v = (np.array(c[t], np.float64) for t in ("q", "k", "v"))
        o, lse = attention_forward(q, k, v, 1.0, c["mask"])
        _close(o, c["O"], 1e-14, c["name"])
        ref = np.array([-np.inf if x is None else x for x in c["lse"]])
        assert np.array_equal(np.isneginf(lse), np.isneginf(ref))
        _close(lse[np.isfinite(ref)], ref[np.isfinite(ref)], 1e-14, c["name"] + " lse")


def test_sampled_rows_and_keys_with_groups_and_offsets():
    q, do = _rand((1, 4, 20, 4), 21), _rand((1, 4, 20, 4), 22)
    k, v = _rand((1, 2, 26, 4), 23), _rand((1, 2, 26, 4), 24)
    dq, dk, dv, o, lse = attention_backward(q, k, v, do, 0.5, "bottom_right", return_forward=True)
    rows = [(0, 0, 0), (0, 3, 19), (0, 2, 7)]
    ro, rl, rdq = attention_rows(q, k, v, 0.5, "bottom_right", rows, do=do)
    for t, (b, hh, i) in enumerate(rows):
        _close(ro[t], o[b, hh, i], 1e-13, "rows O")
        _close(rl[t], lse[b, hh, i], 1e-13, "rows lse")
        _close(rdq[t], dq[b, hh, i], 1e-12, "rows dQ")
    kdk, kdv = attention_keys(q, k, v, do, 0.5, "bottom_right", (0, 1), [0, 5, 25])
    for t, j in enumerate([0, 5, 25]):
        _close(kdk[t], dk[0, 1, j], 1e-12, "keys dK")
        _close(kdv[t], dv[0, 1, j], 1e-12, "keys dV")


def _mutant_forward(kind):
    """Copies of the definition with one planted mistake in the extended cases."""
    def fwd(q, k, v, scale, mode):
        H, Hkv = q.shape[1], k.shape[1]
        g = H // Hkv
        nq, nk = q.shape[2], k.shape[2]
        off = nk - nq if mode == "bottom_right" else 0
        if kind == "offset_sign":
            off = -off
        o = np.zeros(q.shape)
        for b in range(q.shape[0]):
            for h in range(H):
                kv = h % Hkv if kind == "head_modulo" else h // g
                s = scale * q[b, h] @ k[b, kv].T
                if mode != "none":
                    s = np.where(np.arange(nk)[None, :] <= np.arange(nq)[:, None] + off, s, -np.inf)
                m = s.max(1, keepdims=True)
                m = np.where(np.isfinite(m), m, 0)
                e = np.exp(s - m)
                l = e.sum(1, keepdims=True)
                o[b, h] = (e @ v[b, kv]) / np.where(l == 0, 1, l)
        return o
    return fwd


@pytest.mark.parametrize("kind", ["head_modulo", "offset_sign"])
def test_mutants_of_extended_cases_are_caught(kind):
    q, do = _rand((1, 4, 5, 3), 25), _rand((1, 4, 5, 3), 26)
    k, v = _rand((1, 2, 9, 3), 27), _rand((1, 2, 9, 3), 28)
    ref = _torch_ref(q, k, v, do, 0.5, "bottom_right")[0]
    assert np.max(np.abs(_mutant_forward("none")(q, k, v, 0.5, "bottom_right") - ref)) < 1e-12
    assert np.max(np.abs(_mutant_forward(kind)(q, k, v, 0.5, "bottom_right") - ref)) > 1e-3


def test_attention_keys_with_given_row_stats():
    """attention_keys with the rows' (O, lse) given reproduces the version that computes the
    forward itself; rows that do not see the selected keys are not read (NaN there is fine)."""
    rng = np.random.default_rng(11)
    B, H, N, d = 1, 2, 40, 8
    q, k, v, do = (rng.standard_normal((B, H, N, d)) for _ in range(4))
    scale = 0.3
    keys = [25, 31, 39]
    for h in range(H):
        ref = attention_keys(q, k, v, do, scale, True, (0, h), keys)
        o, lse = attention_forward(q[0, h], k[0, h], v[0, h], scale, True)
        o_s, lse_s = o.copy(), lse.copy()
        o_s[:25], lse_s[:25] = np.nan, np.nan  # causal: key 25 is seen by rows 25 .. N-1 only
        got = attention_keys(q, k, v, do, scale, True, (0, h), keys, stats=(o_s, lse_s))
        for a, b in zip(got, ref):
            assert np.abs(a - b).max() <= 1e-12 * np.abs(b).max()
