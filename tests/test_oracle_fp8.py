"""Pins for the oracle's FP8 (E4M3) path and for the FP8 forward's error bounds (CPU only).

The decoder is pinned to hand-worked codes of the OCP E4M3 definition and to torch's
float8_e4m3fn conversion over all 256 codes; the FP8 forward to the plain forward on decoded
values; and the bounds in tests/parity.py (fp8_bounds) to an emulation of the kernel's
arithmetic — weights against a running max up to 8 log2-units stale, rounded to E4M3 by torch,
normalised by their rounded sum — which must stay inside them."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle.fp8 import E4M3_MAX, attention_forward_fp8, e4m3_decode
from parity import fp8_bounds


def test_e4m3_hand_worked_codes():
    # sign | exponent (bias 7) | mantissa
    cases = {0x00: 0.0, 0x38: 1.0, 0x40: 2.0, 0x3C: 1.5, 0xB8: -1.0, 0x7E: 448.0, 0xFE: -448.0,
             0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5, 0x80: -0.0}
    for code, val in cases.items():
        assert e4m3_decode(np.uint8(code)) == val, hex(code)
    assert np.isnan(e4m3_decode(np.uint8(0x7F))) and np.isnan(e4m3_decode(np.uint8(0xFF)))
    assert np.nanmax(np.abs(e4m3_decode(np.arange(256, dtype=np.uint8)))) == E4M3_MAX


def test_e4m3_decode_matches_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = e4m3_decode(codes.numpy())
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))


def _fp8_inputs(shape_q, shape_kv, seed):
    g = torch.Generator().manual_seed(seed)
    out = []
    for shp in (shape_q, shape_kv, shape_kv):
        x = torch.randn(*shp, generator=g, dtype=torch.float64)
        f = float(np.float32(x.abs().max().item() / 448.0))
        out.append(((x / f).to(torch.float8_e4m3fn).view(torch.uint8).numpy(), f))
    return out


def test_fp8_forward_is_forward_of_decoded_values():
    (q8, qd), (k8, kd), (v8, vd) = _fp8_inputs((2, 3, 40, 16), (2, 3, 40, 16), 1)
    for causal in (False, True, "bottom_right"):
        o, lse = attention_forward_fp8(q8, k8, v8, qd, kd, vd, 0.25, causal)
        o2, lse2 = oracle.attention_forward(e4m3_decode(q8) * qd, e4m3_decode(k8) * kd,
                                            e4m3_decode(v8) * vd, 0.25, causal)
        assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def _emulate(s, v, delta_log2):
    """Kernel-like FP8 PV: weights exp(s - m) with m = max s - delta (natural-log units from
    log2 units), rounded to E4M3, normalised by their rounded sum."""
    m = s.max(axis=1, keepdims=True) - delta_log2 * np.log(2.0)
    e = np.exp(s - m)
    e8 = torch.from_numpy(e).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    return (e8 @ v) / e8.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("n", [64, 600, 2048])
@pytest.mark.parametrize("delta", [0.0, 3.7, 8.0])
def test_fp8_bounds_hold_for_emulated_kernel_arithmetic(n, delta):
    rng = np.random.default_rng(n + int(10 * delta))
    r, d = 48, 32
    s = rng.standard_normal((r, n)) * rng.uniform(0.5, 3.0, size=(r, 1))  # flat to peaked rows
    v = rng.standard_normal((n, d))
    p = np.exp(s - s.max(axis=1, keepdims=True))
    o_ref = (p @ v) / p.sum(axis=1, keepdims=True)
    o = _emulate(s, v, delta)
    maxb, meanb, ok = fp8_bounds(s, v, o_ref)
    assert ok.all()
    err = np.abs(o - o_ref)
    assert np.all(err <= maxb), f"max bound violated by {np.max(err - maxb):.3e}"
    assert err.mean() <= 2 * meanb.mean(), f"mean {err.mean():.3e} vs {2 * meanb.mean():.3e}"
    # the bounds are not vacuous: pairing each weight with the next key's value breaks them
    o_shift = _emulate(s, np.roll(v, 1, axis=0), delta)
    assert np.any(np.abs(o_shift - o_ref) > maxb)
