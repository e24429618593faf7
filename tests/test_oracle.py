"""Pins for the fp64 oracle (CPU only).

The oracle is checked against facts the pages and the mathematics fix, none of which is a
retyping of its own formulas:
  * hand-worked closed forms (tests/golden/*.json, each with its derivation and source),
  * special cases with closed forms (N = 1, Q = 0, a dominant one-hot logit, V = ones),
  * the pages' online-softmax recurrence and tiled loop (for every block size),
  * brute force in pure Python on tiny inputs (exp(s) / sum exp(s), no max subtraction),
  * central finite differences of the scalar loss sum(dO o O) for the gradients,
  * invariants (shift invariance, column sums of dV and dK, causal row 0),
  * torch's fp64 scaled_dot_product_attention + autograd as a library special case.
Every pin is a function of an implementation (forward, backward). A mutation test plants
plausible mistakes in copies of the definition and requires each copy to fail some pin.
"""

from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass
from typing import Callable

import numpy as np
import pytest

import oracle
from oracle import (attention_backward, attention_forward, attention_keys, attention_probabilities,
                    attention_rows, online_softmax_stats, tiled_attention_forward)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@dataclass
class Impl:
    name: str
    fwd: Callable  # (q, k, v, scale, causal) -> (O, lse)
    bwd: Callable  # (q, k, v, dO, scale, causal) -> (dQ, dK, dV)


ORACLE = Impl("oracle",
              lambda q, k, v, s, c: attention_forward(q, k, v, s, c),
              lambda q, k, v, do, s, c: attention_backward(q, k, v, do, s, c))


def _rand(shape, seed, mult=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * mult


def _close(a, b, tol, what=""):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    if a.shape != b.shape or not np.all(np.isfinite(a)):
        raise AssertionError(f"{what}: shape {a.shape} vs {b.shape} or non-finite")
    err = np.max(np.abs(a - b) / (1.0 + np.abs(b))) if a.size else 0.0
    if not err <= tol:
        raise AssertionError(f"{what}: error {err:.3e} > {tol:.1e}")


# ------------------------------------------------------------------------------------------
# Forward pins
# ------------------------------------------------------------------------------------------
def pin_golden_closed_form(impl: Impl):
    """Hand-worked examples of the definition (tests/golden/attention_closed_form.json)."""
    with open(os.path.join(GOLDEN, "attention_closed_form.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v = (np.array(c[t], np.float64) for t in ("q", "k", "v"))
        o, lse = impl.fwd(q, k, v, c["scale"], c["causal"])
        _close(o, c["O"], 1e-13, c["name"] + " O")
        _close(lse, c["lse"], 1e-13, c["name"] + " lse")
        if "dQ" in c:
            dq, dk, dv = impl.bwd(q, k, v, np.array(c["do"], np.float64), c["scale"], c["causal"])
            _close(dq, c["dQ"], 1e-13, c["name"] + " dQ")
            _close(dk, c["dK"], 1e-13, c["name"] + " dK")
            _close(dv, c["dV"], 1e-13, c["name"] + " dV")


def pin_rows_sum_to_one(impl: Impl):
    """softmax rows sum to 1  <=>  with V = ones every output entry is exactly 1."""
    for causal in (False, True):
        q, k = _rand((2, 24, 5), 1), _rand((2, 24, 5), 2)
        v = np.ones((2, 24, 3))
        o, _ = impl.fwd(q, k, v, 0.7, causal)
        _close(o, np.ones_like(o), 1e-12, f"V=ones causal={causal}")


def pin_single_key(impl: Impl):
    """N = 1: the only weight is 1, so O = V and lse = scale * q . k."""
    for causal in (False, True):
        q, k, v = _rand((3, 1, 4), 3), _rand((3, 1, 4), 4), _rand((3, 1, 4), 5)
        o, lse = impl.fwd(q, k, v, 0.37, causal)
        _close(o, v, 1e-14, "N=1 O")
        _close(lse, 0.37 * np.sum(q * k, axis=-1), 1e-14, "N=1 lse")


def pin_zero_query(impl: Impl):
    """Q = 0: all visible logits are 0, so O_i is the mean of the visible V rows and
    lse_i = ln(number of visible keys)."""
    n, d = 17, 3
    k, v = _rand((n, d), 6), _rand((n, d), 7)
    q = np.zeros((n, d))
    o, lse = impl.fwd(q, k, v, 1.0, False)
    _close(o, np.broadcast_to(v.mean(axis=0), o.shape), 1e-13, "Q=0 O")
    _close(lse, np.full(n, math.log(n)), 1e-13, "Q=0 lse")
    o, lse = impl.fwd(q, k, v, 1.0, True)
    prefix = np.cumsum(v, axis=0) / np.arange(1, n + 1)[:, None]
    _close(o, prefix, 1e-13, "Q=0 causal O")
    _close(lse, np.log(np.arange(1, n + 1)), 1e-13, "Q=0 causal lse")


def pin_one_hot(impl: Impl):
    """A logit exceeding every other by >= 40 selects its V row within e^-40 N |V|."""
    n, d = 12, 4
    rng = np.random.default_rng(8)
    q = rng.standard_normal((n, d))
    k = rng.standard_normal((n, d)) * 0.1
    v = rng.standard_normal((n, d))
    targets = [(i, (3 * i + 1) % n) for i in range(n)]
    for i, j in targets:
        k2 = k.copy()
        k2[j] = q[i] * (60.0 / np.dot(q[i], q[i]))  # s_ij = 60, others |s| < ~5
        o, lse = impl.fwd(q[i:i + 1], k2, v, 1.0, False)
        s = k2 @ q[i]
        assert s[j] - np.max(np.delete(s, j)) >= 40
        bound = math.exp(-40) * n * np.max(np.abs(v)) * 4
        assert np.max(np.abs(o[0] - v[j])) <= bound, "one-hot O"
        assert abs(lse[0] - s[j]) <= 1e-12 + bound, "one-hot lse"


def pin_brute_force(impl: Impl):
    """Pure-Python loops, softmax taken directly as e^s / sum e^s (no max subtraction)."""
    rng = np.random.default_rng(9)
    for n in (1, 2, 3, 4):
        for d in (1, 2, 3):
            for causal in (False, True):
                q, k, v = (rng.standard_normal((n, d)) for _ in range(3))
                scale = 0.8
                o_ref = np.zeros((n, d))
                lse_ref = np.zeros(n)
                for i in range(n):
                    w = []
                    for j in range(n):
                        if causal and j > i:
                            w.append(0.0)
                            continue
                        s = scale * sum(float(q[i, c]) * float(k[j, c]) for c in range(d))
                        w.append(math.exp(s))
                    tot = sum(w)
                    lse_ref[i] = math.log(tot)
                    for c in range(d):
                        o_ref[i, c] = sum(w[j] * float(v[j, c]) for j in range(n)) / tot
                o, lse = impl.fwd(q, k, v, scale, causal)
                _close(o, o_ref, 1e-14, f"brute O n={n} d={d}")
                _close(lse, lse_ref, 1e-14, f"brute lse n={n} d={d}")


def pin_tiled_online_softmax(impl: Impl):
    """The pages' tiled loop with the online-softmax update reaches the same O and lse for
    every block size 1..N, divisors or not."""
    n, d = 23, 4
    q, k, v = _rand((n, d), 10), _rand((n, d), 11), _rand((n, d), 12)
    for causal in (False, True):
        o_ref, lse_ref = impl.fwd(q, k, v, 0.6, causal)
        for block in range(1, n + 1):
            o, lse = tiled_attention_forward(q, k, v, 0.6, causal, block)
            _close(o_ref, o, 1e-12, f"tiled O block={block}")
            _close(lse_ref, lse, 1e-12, f"tiled lse block={block}")


def pin_shift_invariance(impl: Impl):
    """Adding one vector c to every key shifts row i of S by scale * q_i . c: O unchanged and
    lse shifted by that amount."""
    for causal in (False, True):
        q, k, v = _rand((2, 19, 5), 13), _rand((2, 19, 5), 14), _rand((2, 19, 5), 15)
        c = _rand((5,), 16)
        o1, lse1 = impl.fwd(q, k, v, 0.45, causal)
        o2, lse2 = impl.fwd(q, k + c, v, 0.45, causal)
        _close(o2, o1, 1e-12, "shift O")
        _close(lse2, lse1 + 0.45 * (q @ c), 1e-12, "shift lse")


def pin_causal_first_row(impl: Impl):
    """Under the causal mask row 0 sees only key 0: O_0 = v_0, lse_0 = scale q_0 . k_0."""
    q, k, v = _rand((3, 9, 4), 17), _rand((3, 9, 4), 18), _rand((3, 9, 4), 19)
    o, lse = impl.fwd(q, k, v, 0.9, True)
    _close(o[:, 0], v[:, 0], 1e-15, "causal O_0")
    _close(lse[:, 0], 0.9 * np.sum(q[:, 0] * k[:, 0], axis=-1), 1e-15, "causal lse_0")


def pin_torch_sdpa(impl: Impl):
    """Library special case: torch's fp64 CPU scaled_dot_product_attention and autograd, on
    the size of the pages' own check (B = 2, N = 512, D = 64)."""
    import torch
    import torch.nn.functional as F

    for causal in (False, True):
        q, k, v, do = (_rand((2, 1, 512, 64), 20 + t) for t in range(4))
        tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
        scale = 1.0 / 8.0
        to = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        to.backward(torch.tensor(do))
        o, _ = impl.fwd(q, k, v, scale, causal)
        _close(o, to.detach().numpy(), 1e-12, "sdpa O")
        dq, dk, dv = impl.bwd(q, k, v, do, scale, causal)
        _close(dq, tq.grad.numpy(), 1e-11, "sdpa dQ")
        _close(dk, tk.grad.numpy(), 1e-11, "sdpa dK")
        _close(dv, tv.grad.numpy(), 1e-11, "sdpa dV")


# ------------------------------------------------------------------------------------------
# Backward pins
# ------------------------------------------------------------------------------------------
def pin_finite_differences(impl: Impl):
    """Central differences (h = 1e-6) of L = sum(dO o O) w.r.t. Q, K, V; relative error 1e-6."""
    h = 1e-6
    for causal in (False, True):
        n, d = 7, 3
        q, k, v, do = (_rand((n, d), 30 + t) for t in range(4))
        scale = 0.75
        grads = impl.bwd(q, k, v, do, scale, causal)
        for which, g in zip(range(3), grads):
            fd = np.zeros((n, d))
            for i in range(n):
                for c in range(d):
                    args_p = [q.copy(), k.copy(), v.copy()]
                    args_m = [q.copy(), k.copy(), v.copy()]
                    args_p[which][i, c] += h
                    args_m[which][i, c] -= h
                    lp = np.sum(do * impl.fwd(*args_p, scale, causal)[0])
                    lm = np.sum(do * impl.fwd(*args_m, scale, causal)[0])
                    fd[i, c] = (lp - lm) / (2 * h)
            err = np.max(np.abs(np.asarray(g) - fd)) / max(1e-300, np.max(np.abs(fd)))
            if not err <= 1e-6:
                raise AssertionError(f"finite differences tensor {which} causal={causal}: {err:.2e}")


def pin_gradient_invariants(impl: Impl):
    """sum_j dV_j = sum_i dO_i (rows of P sum to 1) and sum_j dK_j = 0 (rows of dS sum to 0,
    since sum_j P_ij dP_ij = dO_i . O_i = D_i)."""
    for causal in (False, True):
        q, k, v, do = (_rand((2, 21, 6), 40 + t) for t in range(4))
        dq, dk, dv = impl.bwd(q, k, v, do, 0.55, causal)
        _close(dv.sum(axis=-2), do.sum(axis=-2), 1e-12, "sum dV")
        _close(dk.sum(axis=-2), np.zeros((2, 6)), 1e-12, "sum dK")


FORWARD_PINS = [pin_golden_closed_form, pin_rows_sum_to_one, pin_single_key, pin_zero_query,
                pin_one_hot, pin_brute_force, pin_tiled_online_softmax, pin_shift_invariance,
                pin_causal_first_row, pin_torch_sdpa]
BACKWARD_PINS = [pin_golden_closed_form, pin_finite_differences, pin_gradient_invariants,
                 pin_torch_sdpa]
ALL_PINS = list(dict.fromkeys(FORWARD_PINS + BACKWARD_PINS))


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(ORACLE)


# ------------------------------------------------------------------------------------------
# Mutation test: plausible mistakes planted in copies of the definition must fail a pin.
# ------------------------------------------------------------------------------------------
def _mutant(kind: str) -> Impl:
    def fwd(q, k, v, scale, causal):
        q, k, v = (np.asarray(x, np.float64) for x in (q, k, v))
        s = np.einsum("...id,...jd->...ij", q, k)
        if kind == "transposed_scores" and s.shape[-1] == s.shape[-2]:
            s = np.swapaxes(s, -1, -2)
        if kind != "dropped_scale":
            s = s * scale
        n, m = s.shape[-2], s.shape[-1]
        if causal:
            i, j = np.arange(n)[:, None], np.arange(m)[None, :]
            mask = {"mask_off_by_one": j < i, "mask_wrong_triangle": j >= i}.get(kind, j <= i)
            mask = np.broadcast_to(mask, s.shape)
        else:
            mask = np.ones(s.shape, bool)
        mx = np.where(mask, s, -np.inf).max(axis=-1, keepdims=True)
        if kind == "exp_against_zero_not_max":
            mx = np.zeros_like(mx)
        e = np.where(mask, np.exp(np.where(mask, s, 0) - mx), 0.0)
        l = e.sum(axis=-1, keepdims=True)
        o = e @ v if kind == "no_normalisation" else (e @ v) / l
        lse = (np.log(l) if kind == "lse_without_max" else
               mx + np.log2(l) if kind == "lse_log2" else mx + np.log(l))[..., 0]
        if kind == "exp_against_zero_not_max":
            lse = np.log(l)[..., 0] + 1e-3  # keep lse off by a visible amount
        return o, lse

    def bwd(q, k, v, do, scale, causal):
        q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
        o, lse = ORACLE.fwd(q, k, v, scale, causal)
        s = scale * np.einsum("...id,...jd->...ij", q, k)
        p = np.exp(s - lse[..., None])
        if causal:
            n = s.shape[-1]
            p = np.where(np.arange(n)[None, :] <= np.arange(n)[:, None], p, 0.0)
        dv = p @ do if kind == "dv_not_transposed" else np.swapaxes(p, -1, -2) @ do
        dp = do @ np.swapaxes(v, -1, -2)
        dd = np.sum(do * (v if kind == "D_from_v" else o), axis=-1, keepdims=True)
        ds = p * (dp + dd) if kind == "ds_sign" else p * (dp - dd)
        dq = scale * (ds @ (q if kind == "dq_uses_q" else k))
        dk_core = ds @ q if kind == "dk_not_transposed" else np.swapaxes(ds, -1, -2) @ q
        dk = dk_core if kind == "dk_dropped_scale" else scale * dk_core
        return dq, dk, dv

    return Impl(kind, fwd, bwd)


FORWARD_MUTANTS = ["dropped_scale", "transposed_scores", "mask_off_by_one", "mask_wrong_triangle",
                   "no_normalisation", "lse_without_max", "lse_log2"]
BACKWARD_MUTANTS = ["dv_not_transposed", "D_from_v", "ds_sign", "dq_uses_q", "dk_not_transposed",
                    "dk_dropped_scale"]


def _fails_some(impl, pins):
    import warnings

    failed = []
    for pin in pins:
        try:
            with warnings.catch_warnings():
                warnings.simplefilter("ignore")
                with np.errstate(all="ignore"):
                    pin(impl)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    return failed


def test_reference_mutant_copy_passes_all_pins():
    """The mutation harness itself: the un-mutated copy passes every pin."""
    assert _fails_some(_mutant("none"), ALL_PINS) == []


@pytest.mark.parametrize("kind", FORWARD_MUTANTS)
def test_forward_mutant_is_caught(kind):
    cheap = [p for p in FORWARD_PINS if p is not pin_torch_sdpa]
    assert _fails_some(_mutant(kind), cheap), f"mutant {kind} passed every forward pin"


@pytest.mark.parametrize("kind", BACKWARD_MUTANTS)
def test_backward_mutant_is_caught(kind):
    cheap = [p for p in BACKWARD_PINS if p is not pin_torch_sdpa]
    assert _fails_some(_mutant(kind), cheap), f"mutant {kind} passed every backward pin"


# ------------------------------------------------------------------------------------------
# The online-softmax recurrence itself, and the pages' flawed listing as a negative pin.
# ------------------------------------------------------------------------------------------
def test_online_softmax_worked_example():
    """Hand-worked example of the update equation (tests/golden/online_softmax_worked_example)."""
    with open(os.path.join(GOLDEN, "online_softmax_worked_example.json")) as f:
        g = json.load(f)
    c1, c2 = g["chunks"]
    m1, d1 = online_softmax_stats(c1, block=2)
    assert abs(m1 - g["after_chunk_1"]["m"]) < 1e-15 and abs(d1 - g["after_chunk_1"]["d"]) < 1e-15
    m2, d2 = online_softmax_stats(c1 + c2, block=2)
    assert abs(m2 - g["after_chunk_2"]["m"]) < 1e-15 and abs(d2 - g["after_chunk_2"]["d"]) < 1e-15
    mc, dc = online_softmax_stats(c2, block=2)
    assert abs(mc - g["chunk_2_alone"]["m"]) < 1e-15 and abs(dc - g["chunk_2_alone"]["d"]) < 1e-15


def test_online_softmax_every_chunking():
    """Chunked statistics equal the unchunked (max, sum e^(x - max)) for every chunk size."""
    rng = np.random.default_rng(50)
    for n in (1, 2, 5, 31, 64):
        x = rng.standard_normal(n) * 4
        m_ref = max(float(t) for t in x)
        d_ref = math.fsum(math.exp(float(t) - m_ref) for t in x)
        for block in range(1, n + 1):
            m, d = online_softmax_stats(x, block)
            assert m == m_ref
            assert abs(d - d_ref) <= 1e-12 * d_ref


def _listing_as_printed(q, k, v, block):
    """The page-3 simulation's per-block update, restated with its flaw kept: the block's
    exponentials are taken against the block's own maximum, while the running sum and partial
    output are rescaled by e^(m_old - m_new) only (codethepapers.com, "Implementation:
    Simulating FlashAttention in PyTorch"). Used only as a negative pin."""
    n = q.shape[-2]
    scale = 1.0 / math.sqrt(q.shape[-1])
    o = np.zeros_like(v)
    m = np.full(q.shape[:-1], -np.inf)
    l = np.zeros(q.shape[:-1])
    for j0 in range(0, n, block):
        for i0 in range(0, n, block):
            s = scale * np.einsum("...id,...jd->...ij", q[..., i0:i0 + block, :],
                                  k[..., j0:j0 + block, :])
            bmax = s.max(axis=-1)
            m_new = np.maximum(m[..., i0:i0 + block], bmax)
            e = np.exp(s - bmax[..., None])          # flaw: against the block max
            alpha = np.exp(m[..., i0:i0 + block] - m_new)
            l[..., i0:i0 + block] = alpha * l[..., i0:i0 + block] + e.sum(axis=-1)
            o[..., i0:i0 + block, :] = alpha[..., None] * o[..., i0:i0 + block, :] + e @ v[..., j0:j0 + block, :]
            m[..., i0:i0 + block] = m_new
    return o / l[..., None]


def test_printed_listing_is_not_the_definition():
    """Negative pin: the flawed per-block rescaling differs from the oracle by far more than
    the listing's own 1e-5 check whenever there is more than one block (B=2, N=512, D=64,
    block 128, the page's verification shape), and agrees when one block covers the row."""
    q, k, v = (_rand((2, 512, 64), 60 + t) for t in range(3))
    o_ref, _ = attention_forward(q, k, v, 1 / 8, False)
    for block in (64, 128):
        diff = np.max(np.abs(_listing_as_printed(q, k, v, block) - o_ref))
        assert diff > 1e-2, f"block {block}: listing unexpectedly matches ({diff:.2e})"
    diff = np.max(np.abs(_listing_as_printed(q, k, v, 512) - o_ref))
    assert diff < 1e-12


# ------------------------------------------------------------------------------------------
# Internal consistency of the oracle's entry points.
# ------------------------------------------------------------------------------------------
def test_probabilities_match_forward():
    for causal in (False, True):
        q, k, v = (_rand((2, 3, 33, 5), 70 + t) for t in range(3))
        p = attention_probabilities(q, k, 0.3, causal)
        _close(p.sum(axis=-1), np.ones(p.shape[:-1]), 1e-13, "P rows")
        o, _ = attention_forward(q, k, v, 0.3, causal)
        _close(p @ v, o, 1e-13, "P V")
        if causal:
            assert np.all(p[..., np.triu_indices(33, 1)[0], np.triu_indices(33, 1)[1]] == 0.0)


def test_row_blocking_does_not_change_results():
    for causal in (False, True):
        q, k, v, do = (_rand((2, 45, 6), 80 + t) for t in range(4))
        a = attention_backward(q, k, v, do, 0.4, causal, block_rows=7, return_forward=True)
        b = attention_backward(q, k, v, do, 0.4, causal, block_rows=1000, return_forward=True)
        for x, y in zip(a, b):
            _close(x, y, 1e-13, "blocking")


def test_sampled_rows_and_keys_match_full():
    for causal in (False, True):
        q, k, v, do = (_rand((2, 2, 40, 6), 90 + t) for t in range(4))
        dq, dk, dv, o, lse = attention_backward(q, k, v, do, 0.5, causal, return_forward=True)
        rows = [(0, 0, 0), (0, 1, 39), (1, 0, 17), (1, 1, 5)]
        ro, rl, rdq = attention_rows(q, k, v, 0.5, causal, rows, do=do)
        for t, (b, h, i) in enumerate(rows):
            _close(ro[t], o[b, h, i], 1e-13, "rows O")
            _close(rl[t], lse[b, h, i], 1e-13, "rows lse")
            _close(rdq[t], dq[b, h, i], 1e-12, "rows dQ")
        keys = [0, 3, 39]
        kdk, kdv = attention_keys(q, k, v, do, 0.5, causal, (1, 0), keys, block_rows=16)
        for t, j in enumerate(keys):
            _close(kdk[t], dk[1, 0, j], 1e-12, "keys dK")
            _close(kdv[t], dv[1, 0, j], 1e-12, "keys dV")


def test_nonsquare_noncausal():
    """N_q != N_k (non-causal): each query row still sees every key."""
    q, k, v = _rand((5, 4), 100), _rand((9, 4), 101), _rand((9, 4), 102)
    o, lse = attention_forward(q, k, v, 0.5, False)
    p = attention_probabilities(q, k, 0.5, False)
    _close(o, p @ v, 1e-13, "nonsquare")


def test_oracle_package_is_independent_of_the_product():
    """The oracle imports nothing from the CUDA path (they share no code)."""
    import ast

    src_dir = os.path.dirname(oracle.__file__)
    for fn in os.listdir(src_dir):
        if fn.endswith(".py"):
            tree = ast.parse(open(os.path.join(src_dir, fn)).read())
            for node in ast.walk(tree):
                if isinstance(node, (ast.Import, ast.ImportFrom)):
                    names = [a.name for a in node.names] + [getattr(node, "module", "") or ""]
                    assert not any("exact_io_aware_66_b200" in n for n in names), fn
