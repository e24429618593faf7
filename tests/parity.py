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


# ------------------------------------------------------------------------------------------
# FP8 forward bounds
# ------------------------------------------------------------------------------------------
def fp8_bounds(s_rows: np.ndarray, v: np.ndarray, o_ref: np.ndarray):
    """Error bounds of an FP8 forward output row block against the exact O of the decoded inputs.

    s_rows: [r, n] fp64 scores (masked entries -inf), v: [n, d] decoded V, o_ref: [r, d].
    The kernel rounds each weight e_j = exp(s_j - m) to E4M3, with m its running max, at most 8
    log2-units below the row max, and normalises by the sum of the rounded weights, so exactly
        O - O* = sum_j (e~_j - e_j)(v_j - O*) / sum_j e~_j.
    E4M3 rounding moves a weight by at most half a unit in the last place: 2^-4 e_j in the
    normal range (e_j >= 2^-6), and min(e_j, 2^-10) in the subnormal range (spacing 2^-9).
    With e^_j = exp(s_j - max s) (e_j = 2^delta e^_j, delta in [0, 8], so e^_j >= 2^-6 implies
    the normal range) and L^ = sum_j e^_j, dividing through by 2^delta:
        err_j      = 2^-4 e^_j + [e^_j < 2^-6] min(e^_j, 2^-10)
        max bound  = sum_j err_j |v_j - O*| / (L^ - sum_j err_j)
                     + 2^-8 |O*| (bf16 output rounding) + 1e-5 max|v| (fp32 arithmetic)
        mean bound = sqrt(2/pi) 2^-4 / sqrt(3) sqrt(sum_j (e^_j / L^)^2 (v_j - O*)^2)
    the second being the mean absolute value of the sum when the relative rounding errors are
    independent and uniform (standard deviation 2^-4 / sqrt 3). Returns (max_bound [r, d],
    mean_bound [r, d], ok) with ok False where the max bound's denominator is not positive."""
    mx = np.max(s_rows, axis=1, keepdims=True)
    mx = np.where(np.isfinite(mx), mx, 0.0)
    eh = np.exp(s_rows - mx)  # masked entries: exp(-inf) = 0
    L = eh.sum(axis=1, keepdims=True)
    err = 2.0 ** -4 * eh + np.where(eh < 2.0 ** -6, np.minimum(eh, 2.0 ** -10), 0.0)
    dev = np.abs(v[None, :, :] - o_ref[:, None, :])  # [r, n, d]
    num = np.einsum("rn,rnd->rd", err, dev)
    den = L - err.sum(axis=1, keepdims=True)
    ok = den[:, 0] > 0
    maxb = num / np.where(den > 0, den, np.inf) + 2.0 ** -8 * np.abs(o_ref) + 1e-5 * np.abs(v).max()
    w2 = (eh / np.where(L > 0, L, 1.0)) ** 2
    meanb = np.sqrt(2 / np.pi) * 2.0 ** -4 / np.sqrt(3) * np.sqrt(np.einsum("rn,rnd->rd", w2, dev ** 2))
    return maxb, meanb, ok
