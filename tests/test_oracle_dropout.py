"""Pins for the oracle's dropout (CPU only).

The generator is pinned to the published Philox4x32-10 known-answer vectors; the mapping from
an attention entry to its keep decision to a per-element restatement in plain Python integers;
the keep rate and the keep scale to statistics (a dropped entry's expectation is the undropped
entry); and the dropout gradients to torch fp64 autograd through an explicit keep mask and to
finite differences. Planted mistakes in copies must fail one of these pins.
"""

from __future__ import annotations

import json
import os
from dataclasses import dataclass
from typing import Callable

import numpy as np
import pytest

import oracle
from oracle import dropout_keep, dropout_p8, keep_scale, philox4x32_10

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ------------------------------------------------------------------------------------------
# Per-element restatement of the keep rule in plain Python integers (for the layout pin)
# ------------------------------------------------------------------------------------------
def _philox_scalar(ctr, key, rounds=10, mults=(0xD2511F53, 0xCD9E8D57), bump=True):
    c, k = list(ctr), list(key)
    for _ in range(rounds):
        a, b = mults[0] * c[0], mults[1] * c[2]
        c = [(b >> 32) ^ c[1] ^ k[0], b & 0xFFFFFFFF, (a >> 32) ^ c[3] ^ k[1], a & 0xFFFFFFFF]
        if bump:
            k = [(k[0] + 0x9E3779B9) & 0xFFFFFFFF, (k[1] + 0xBB67AE85) & 0xFFFFFFFF]
    return c


def _keep_scalar(bh, i, j, p8, seed, offset):
    w = _philox_scalar((j // 4, i // 4, bh, offset), (seed & 0xFFFFFFFF, seed >> 32))
    return ((w[i % 4] >> (8 * (j % 4))) & 0xFF) >= p8


# ------------------------------------------------------------------------------------------
# Implementations under test: the oracle, and plain materialised copies with planted mistakes
# ------------------------------------------------------------------------------------------
@dataclass
class Impl:
    name: str
    philox: Callable
    keep: Callable
    fwd: Callable  # (q, k, v, scale, causal, dropout) -> (o, lse), single head [N, d]
    bwd: Callable  # (q, k, v, do, scale, causal, dropout) -> (dq, dk, dv)


ORACLE = Impl(
    "oracle",
    philox4x32_10,
    dropout_keep,
    lambda q, k, v, s, c, dr: oracle.attention_forward(q, k, v, s, c, dropout=dr),
    lambda q, k, v, do, s, c, dr: oracle.attention_backward(q, k, v, do, s, c, dropout=dr),
)


def _mutant(kind: str) -> Impl:
    def philox(c0, c1, c2, c3, k0, k1):
        mults = (0xCD9E8D57, 0xD2511F53) if kind == "swapped_multipliers" else (0xD2511F53,
                                                                                 0xCD9E8D57)
        c0, c1, c2, c3 = (np.broadcast_to(np.asarray(x, np.uint64), np.broadcast(
            np.asarray(c0), np.asarray(c1), np.asarray(c2), np.asarray(c3)).shape)
            for x in (c0, c1, c2, c3))
        out = [np.zeros(c0.shape, np.uint32) for _ in range(4)]
        for pos in np.ndindex(*c0.shape):
            w = _philox_scalar((int(c0[pos]), int(c1[pos]), int(c2[pos]), int(c3[pos])),
                               (int(k0), int(k1)), mults=mults, bump=kind != "no_key_bump")
            for t in range(4):
                out[t][pos] = w[t]
        return tuple(out)

    def keep(bh, rows, keys, p8, seed, offset):
        rows = list(rows)
        keys = list(range(keys)) if np.isscalar(keys) else list(keys)
        z = np.zeros((len(rows), len(keys)), bool)
        for a, i in enumerate(rows):
            for b, j in enumerate(keys):
                ci, cj = (j, i) if kind == "counter_rows_cols_swapped" else (i, j)
                w = _philox_scalar((cj // 4, ci // 4, bh, offset), (seed & 0xFFFFFFFF, seed >> 32))
                word, byte = (j % 4, i % 4) if kind == "word_byte_swapped" else (i % 4, j % 4)
                x = (w[word] >> (8 * byte)) & 0xFF
                z[a, b] = x > p8 if kind == "keep_gt" else x >= p8
        return z

    def probs(q, k, scale, causal):
        s = scale * (q @ k.T)
        n, m = s.shape
        vis = np.ones((n, m), bool) if not causal else (np.arange(m)[None, :] <= np.arange(n)[:, None])
        mx = np.where(vis, s, -np.inf).max(axis=1, keepdims=True)
        e = np.where(vis, np.exp(np.where(vis, s, 0) - mx), 0.0)
        l = e.sum(axis=1, keepdims=True)
        return e / l, (mx + np.log(l))[:, 0]

    def fwd(q, k, v, scale, causal, dropout):
        q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
        p, lse = probs(q, k, scale, causal)
        if dropout is None:
            return p @ v, lse
        p8 = dropout_p8(dropout[0])
        z = keep(0, range(q.shape[0]), k.shape[0], p8, dropout[1], dropout[2])
        r = 1.0 if kind == "no_keep_scale" else keep_scale(p8)
        return (r * z * p) @ v, lse

    def bwd(q, k, v, do, scale, causal, dropout):
        q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
        p, _ = probs(q, k, scale, causal)
        p8 = dropout_p8(dropout[0])
        z = keep(0, range(q.shape[0]), k.shape[0], p8, dropout[1], dropout[2]).astype(float)
        r = keep_scale(p8)
        o = (r * z * p) @ v
        o_for_d = p @ v if kind == "D_from_undropped_O" else o
        dd = np.sum(do * o_for_d, axis=1, keepdims=True)
        dv = (r * (p if kind == "dv_without_mask" else z * p)).T @ do
        dp = do @ v.T
        ds = p * ((dp if kind == "ds_without_mask" else r * z * dp) - dd)
        return scale * ds @ k, scale * ds.T @ q, dv

    return Impl(kind, philox, keep, fwd, bwd)


# ------------------------------------------------------------------------------------------
# Pins
# ------------------------------------------------------------------------------------------
def pin_kat(impl):
    vec = json.load(open(os.path.join(GOLDEN, "philox4x32_10_kat.json")))["vectors"]
    for case in vec:
        c = [int(x, 16) for x in case["ctr"]]
        k = [int(x, 16) for x in case["key"]]
        out = impl.philox(*c, *k)
        assert [int(np.asarray(w).reshape(-1)[0]) for w in out] == [int(x, 16) for x in case["out"]]


def pin_layout_scalar(impl):
    """Each keep decision equals the per-element rule, for several heads, offsets, seeds with
    high bits, and rows/keys that cross 4 x 4 block boundaries."""
    rows, keys = [0, 1, 2, 3, 4, 5, 7, 9, 30], [0, 1, 3, 4, 6, 11, 17, 33]
    for bh, p, seed, offset in ((0, 0.5, 1, 0), (5, 0.25, (7 << 32) + 3, 9), (2, 0.9, 2 ** 40, 1)):
        p8 = dropout_p8(p)
        z = impl.keep(bh, rows, keys, p8, seed, offset)
        ref = np.array([[_keep_scalar(bh, i, j, p8, seed, offset) for j in keys] for i in rows])
        assert np.array_equal(z, ref)


def pin_keep_rate(impl):
    """The fraction kept over 64 x 64 entries is (256 - p8)/256 within 5 binomial sigmas."""
    for p in (0.1, 0.5):
        p8 = dropout_p8(p)
        z = impl.keep(3, range(64), 64, p8, 1234, 5)
        q = (256 - p8) / 256
        assert abs(z.mean() - q) <= 5 * np.sqrt(q * (1 - q) / z.size)


def pin_expectation(impl):
    """The mean of the dropped O over many seeds approaches the undropped O: the keep scale is
    1 / keep probability."""
    q, k, v = _rand((6, 4), 1), _rand((6, 4), 2), _rand((6, 4), 3)
    o_ref, _ = oracle.attention_forward(q, k, v, 0.5, False)
    n = 600
    samples = np.stack([impl.fwd(q, k, v, 0.5, False, (0.5, s, 0))[0] for s in range(n)])
    mean, sd = samples.mean(axis=0), samples.std(axis=0) + 1e-12
    assert np.all(np.abs(mean - o_ref) <= 5 * sd / np.sqrt(n))


def pin_lse_undropped(impl):
    q, k, v = _rand((9, 5), 4), _rand((9, 5), 5), _rand((9, 5), 6)
    _, lse_ref = oracle.attention_forward(q, k, v, 0.4, True)
    _, lse = impl.fwd(q, k, v, 0.4, True, (0.3, 77, 1))
    assert np.allclose(lse, lse_ref, rtol=0, atol=1e-12)


def pin_torch_autograd(impl):
    """Gradients against torch fp64 autograd of O = r (Z o softmax(S)) V with the keep mask Z
    given explicitly (from the per-element rule), causal and not."""
    import torch

    n, d = 10, 6
    q, k, v, do = (_rand((n, d), 10 + t) for t in range(4))
    p8 = dropout_p8(0.35)
    z = np.array([[_keep_scalar(0, i, j, p8, 99, 2) for j in range(n)] for i in range(n)], float)
    r = keep_scale(p8)
    for causal in (False, True):
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        s = 0.45 * tq @ tk.T
        if causal:
            s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
        o = (r * torch.tensor(z) * torch.softmax(s, dim=-1)) @ tv
        o.backward(torch.tensor(do))
        got = impl.bwd(q, k, v, do, 0.45, causal, (0.35, 99, 2))
        for g, t in zip(got, (tq, tk, tv)):
            assert np.allclose(g, t.grad.numpy(), rtol=1e-10, atol=1e-12)


def pin_finite_differences(impl):
    """dQ, dK, dV of L = sum(dO o O) by central differences (the keep mask does not depend on
    the values, so L is smooth in them)."""
    n, d = 7, 3
    q, k, v, do = (_rand((n, d), 20 + t) for t in range(4))
    dr = (0.4, 5, 3)
    dq, dk, dv = impl.bwd(q, k, v, do, 0.6, True, dr)
    h = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        for idx in [(0, 0), (3, 1), (6, 2)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if y is x else y for y in (q, k, v)]
            args_m = [xm if y is x else y for y in (q, k, v)]
            lp = np.sum(do * impl.fwd(*args_p, 0.6, True, dr)[0])
            lm = np.sum(do * impl.fwd(*args_m, 0.6, True, dr)[0])
            assert abs((lp - lm) / (2 * h) - g[idx]) <= 1e-6 * (1 + abs(g[idx]))


PINS = [pin_kat, pin_layout_scalar, pin_keep_rate, pin_expectation, pin_lse_undropped,
        pin_torch_autograd, pin_finite_differences]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_dropout_pin(pin):
    pin(ORACLE)


MUTANTS = ["swapped_multipliers", "no_key_bump", "keep_gt", "word_byte_swapped",
           "counter_rows_cols_swapped", "no_keep_scale", "dv_without_mask", "ds_without_mask",
           "D_from_undropped_O"]


def _fails_some(impl, pins):
    failed = []
    for pin in pins:
        try:
            with np.errstate(all="ignore"):
                pin(impl)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


def test_unmutated_copy_passes():
    cheap = [p for p in PINS if p is not pin_expectation]
    assert _fails_some(_mutant("none"), cheap) == []


@pytest.mark.parametrize("kind", MUTANTS)
def test_dropout_mutant_is_caught(kind):
    pins = [pin_kat] if kind in ("swapped_multipliers", "no_key_bump") else \
        [p for p in PINS if p is not pin_kat]
    assert _fails_some(_mutant(kind), pins), f"mutant {kind} passed every pin"


# ------------------------------------------------------------------------------------------
# Consistency of the oracle's own entry points with dropout
# ------------------------------------------------------------------------------------------
def test_p_zero_is_no_dropout():
    q, k, v, do = (_rand((2, 3, 40, 8), 30 + t) for t in range(4))
    a = oracle.attention_backward(q, k, v, do, 0.3, True, return_forward=True)
    b = oracle.attention_backward(q, k, v, do, 0.3, True, return_forward=True,
                                  dropout=(0.0, 11, 0))
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_rows_and_keys_match_full_with_dropout():
    B, H, Hk, n, nk, d = 2, 4, 2, 37, 45, 8
    q, do = _rand((B, H, n, d), 40), _rand((B, H, n, d), 41)
    k, v = _rand((B, Hk, nk, d), 42), _rand((B, Hk, nk, d), 43)
    dr = (0.2, 2024, 7)
    for mode in ("none", "top_left", "bottom_right"):
        dq, dk, dv, o, lse = oracle.attention_backward(q, k, v, do, 0.35, mode,
                                                       return_forward=True, dropout=dr)
        rows = [(1, 2, 0), (0, 3, 36), (1, 0, 17), (0, 1, 9)]
        o_r, lse_r, dq_r = oracle.attention_rows(q, k, v, 0.35, mode, rows, do=do, dropout=dr)
        idx = tuple(np.array(rows).T)
        assert np.allclose(o_r, o[idx], atol=1e-12) and np.allclose(dq_r, dq[idx], atol=1e-12)
        keys = [0, 5, 44, 21]
        dk_r, dv_r = oracle.attention_keys(q, k, v, do, 0.35, mode, (1, 1), keys, dropout=dr)
        assert np.allclose(dk_r, dk[1, 1, keys], atol=1e-12)
        assert np.allclose(dv_r, dv[1, 1, keys], atol=1e-12)


def test_heads_draw_different_masks():
    p8 = dropout_p8(0.5)
    z = [dropout_keep(bh, range(16), 16, p8, 1, 0) for bh in range(3)]
    z.append(dropout_keep(0, range(16), 16, p8, 1, 1))
    z.append(dropout_keep(0, range(16), 16, p8, 2, 0))
    for a in range(len(z)):
        for b in range(a + 1, len(z)):
            assert not np.array_equal(z[a], z[b])
    assert np.array_equal(z[0], dropout_keep(0, range(16), 16, p8, 1, 0))


def test_p8_quantisation():
    assert dropout_p8(0.0) == 0 and dropout_p8(0.1) == 26 and dropout_p8(0.5) == 128
    assert dropout_p8(0.999) == 255
    with pytest.raises(ValueError):
        dropout_p8(1.0)
