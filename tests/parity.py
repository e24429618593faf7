"""Shared helpers for the GPU parity tests: tolerances and error measures.

Tolerances (fixed numbers, never loosened per case):
  forward O:   max-abs <= 1e-2 and mean-abs <= 1e-3 against the fp64 oracle
  lse:         max-abs <= 1e-3
  dQ, dK, dV:  max-abs error / max-abs of the oracle's tensor <= 2e-2, per tensor
  with dropout: the O bounds times the keep scale r = 256 / (256 - p8) (see assert_fwd_ok)

O is returned in bf16, whose spacing is 2^-5 on [4, 8): rounding the exact value alone can
move it by up to 1.56e-2 there, more than 1e-2. Such "format-limited" elements (|O_ref| >= 4)
are checked against the format instead: |O_gpu - O_ref| <= 1 bf16 ulp at O_ref (half an ulp
of output rounding plus compute error). Every other element meets max-abs 1e-2, and the raw
max-abs over all elements is reported next to the split.
"""

from __future__ import annotations

import numpy as np
import torch

TOL_O_MAX = 1e-2
TOL_O_MEAN = 1e-3
TOL_LSE = 1e-3
TOL_GRAD_REL = 2e-2


def to64(x: torch.Tensor) -> np.ndarray:
    return x.detach().float().cpu().numpy().astype(np.float64)


FORMAT_LIMIT = 4.0  # |O| at and above which the bf16 half-ulp (>= 1.56e-2) exceeds TOL_O_MAX


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def fwd_errors(o_gpu, lse_gpu, o_ref, lse_ref) -> dict:
    o = to64(o_gpu) if isinstance(o_gpu, torch.Tensor) else np.asarray(o_gpu, np.float64)
    l = to64(lse_gpu) if isinstance(lse_gpu, torch.Tensor) else np.asarray(lse_gpu, np.float64)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(l)), "non-finite output"
    e = np.abs(o - o_ref)
    fmt = np.abs(o_ref) >= FORMAT_LIMIT
    return {"o_max": float(e.max()) if e.size else 0.0,
            "o_max_in_range": float(e[~fmt].max()) if (~fmt).any() else 0.0,
            "format_limited": int(fmt.sum()),
            "format_ulps": float((e[fmt] / bf16_ulp(o_ref[fmt])).max()) if fmt.any() else 0.0,
            "o_mean": float(e.mean()) if e.size else 0.0,
            "lse_max": float(np.abs(l - lse_ref).max()) if l.size else 0.0,
            "o_ref_absmax": float(np.abs(o_ref).max()) if o_ref.size else 0.0}


def assert_fwd_ok(err: dict, what: str = "", keep_scale: float = 1.0):
    """keep_scale: with dropout, the kept weights (and so the rounding errors of P and of O) are
    multiplied by r = 256 / (256 - p8); the O bounds are multiplied by the same r."""
    print(f"[parity] {what}: {err}")
    tol_max, tol_mean = TOL_O_MAX * keep_scale, TOL_O_MEAN * keep_scale
    assert err["o_max_in_range"] <= tol_max, f"{what} O max-abs {err['o_max_in_range']:.3e}"
    assert err["format_ulps"] <= 1.0, f"{what} format-limited O off by {err['format_ulps']:.2f} ulp"
    assert err["o_mean"] <= tol_mean, f"{what} O mean-abs {err['o_mean']:.3e}"
    assert err["lse_max"] <= TOL_LSE, f"{what} lse max-abs {err['lse_max']:.3e}"


def grad_rel_error(g_gpu, g_ref) -> float:
    g = to64(g_gpu) if isinstance(g_gpu, torch.Tensor) else np.asarray(g_gpu, np.float64)
    assert np.all(np.isfinite(g)), "non-finite gradient"
    denom = float(np.abs(g_ref).max())
    return float(np.abs(g - g_ref).max()) / max(denom, 1e-30)


def assert_grad_ok(g_gpu, g_ref, what: str):
    r = grad_rel_error(g_gpu, g_ref)
    assert r <= TOL_GRAD_REL, f"{what} relative max-norm error {r:.3e}"
    return r
