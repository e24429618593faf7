"""FP8 (E4M3) forward on the GPU against the oracle's exact attention of the decoded inputs.

Exact cases first: with Q = 0 every weight is 1 (exact in E4M3), so O is the plain mean of the
visible V rows; with one key dominating each row by a wide margin, O is that key's V row. Then
random inputs on ragged, grouped-head and bottom-right shapes, and the causal B=4 H=16 N=4096
d=128 workload on sampled rows, held to the bounds derived in tests/parity.py (fp8_bounds): the
rounding of each probability to E4M3 bounds every element (max bound), the mean absolute error
must stay within twice the independent-rounding estimate (mean bound), lse within 1e-3."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle.fp8 import attention_forward_fp8, e4m3_decode
from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import WORKLOADS, make_inputs_fp8, sampled_rows
from parity import TOL_LSE, fp8_bounds, to64

pytestmark = pytest.mark.gpu


def _codes(t):
    return t.view(torch.uint8).numpy()


def _run(x, mask, d):
    q8, k8, v8 = (x[n].cuda() for n in ("q8", "k8", "v8"))
    o, lse = fa.attention_forward_fp8(q8, k8, v8, x["descale"], causal=mask)
    fa.fa_check_status()
    return to64(o), to64(lse)


def _visible(n_q, n_kv, mode):
    i, j = np.arange(n_q)[:, None], np.arange(n_kv)[None, :]
    if mode in (False, "none"):
        return np.ones((n_q, n_kv), bool)
    return j <= i + (n_kv - n_q if mode == "bottom_right" else 0)


def _check_head(qh, kh, vh, scale, mode, o, lse, o_ref, lse_ref, what):
    """Bounds for one head: qh [n_q, d], kh/vh [n_kv, d] decoded (descales applied)."""
    vis = _visible(qh.shape[0], kh.shape[0], mode)
    s = np.where(vis, scale * (qh @ kh.T), -np.inf)
    live = vis.any(axis=1)
    maxb, meanb, ok = fp8_bounds(s[live], vh, o_ref[live])
    assert ok.all(), f"{what}: bound undefined"
    err = np.abs(o[live] - o_ref[live])
    assert np.all(err <= maxb), f"{what}: max bound exceeded by {np.max(err - maxb):.3e}"
    mean_lim = 2 * meanb.mean() + 2.0 ** -9 * np.abs(o_ref[live]).mean()
    assert err.mean() <= mean_lim, f"{what}: mean error {err.mean():.3e} > {mean_lim:.3e}"
    assert np.abs(lse[live] - lse_ref[live]).max() <= TOL_LSE, f"{what}: lse"
    assert np.all(o[~live] == 0) and np.all(np.isneginf(lse[~live]))
    return float(err.max()), float(err.mean())


@pytest.mark.parametrize("mask", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_fp8_zero_query_gives_plain_means(mask, d):
    x = make_inputs_fp8(1, 2, 2, 300, 300, d, seed=70 + d)
    x["q8"] = torch.zeros_like(x["q8"])
    o, lse = _run(x, mask, d)
    o_ref, lse_ref = attention_forward_fp8(_codes(x["q8"]), _codes(x["k8"]), _codes(x["v8"]),
                                           *x["descale"], fa.default_scale(d), mask)
    vmax = np.abs(e4m3_decode(_codes(x["v8"]))).max() * x["descale"][2]
    assert np.all(np.abs(o - o_ref) <= 2.0 ** -8 * np.abs(o_ref) + 1e-5 * vmax)
    assert np.abs(lse - lse_ref).max() <= 1e-5


@pytest.mark.parametrize("mask", [False, True, "bottom_right"])
def test_fp8_dominant_key_selects_its_value_row(mask):
    """Row i's query is key pi(i)'s code with a large descale: that key's weight is 1 and every
    other weight underflows E4M3, so O_i is V_pi(i) exactly (then rounded to bf16)."""
    n_q, n_kv, d = 200, 333 if mask == "bottom_right" else 200, 128
    x = make_inputs_fp8(1, 1, 1, n_q, n_kv, d, seed=81)
    rng = np.random.default_rng(5)
    off = n_kv - n_q if mask == "bottom_right" else 0
    hi = np.arange(n_q) + off + 1 if mask else np.full(n_q, n_kv)
    pi = (rng.random(n_q) * hi).astype(int)
    x["q8"] = x["k8"][:, :, pi, :].clone().contiguous()
    x["descale"] = (4.0, x["descale"][1], x["descale"][2])
    o, _ = _run(x, mask, d)
    # the kernel forms fp32(V code value * v_descale), then rounds to bf16
    v = e4m3_decode(_codes(x["v8"]))[0, 0].astype(np.float32) * np.float32(x["descale"][2])
    want = torch.from_numpy(v[pi]).to(torch.bfloat16).double().numpy()
    assert np.array_equal(o[0, 0], want)


CASES = [  # (B, H, H_kv, N_q, N_kv, d, mask)
    (1, 2, 2, 256, 256, 128, False),
    (1, 4, 1, 300, 300, 128, True),
    (2, 4, 2, 513, 513, 64, True),
    (1, 2, 2, 100, 700, 128, "bottom_right"),
    (1, 2, 2, 700, 300, 64, "bottom_right"),
    (1, 2, 1, 1000, 1000, 64, False),
    (1, 2, 2, 333, 333, 96, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%dh%dkv%dq%dk%dd%d-%s" % c)
def test_fp8_against_oracle(case):
    B, H, H_kv, N_q, N_kv, d, mask = case
    x = make_inputs_fp8(B, H, H_kv, N_q, N_kv, d, seed=2000 + N_q + N_kv + d)
    o, lse = _run(x, mask, d)
    scale = fa.default_scale(d)
    qd, kd, vd = (float(np.float32(f)) for f in x["descale"])
    q, k, v = (e4m3_decode(_codes(x[n])) * f for n, f in (("q8", qd), ("k8", kd), ("v8", vd)))
    o_ref, lse_ref = oracle.attention_forward(q, k, v, scale, mask)
    g = H // H_kv
    for b in range(B):
        for h in range(H):
            e = _check_head(q[b, h], k[b, h // g], v[b, h // g], scale, mask, o[b, h], lse[b, h],
                            o_ref[b, h], lse_ref[b, h], f"{case} head ({b},{h})")
            print(f"[fp8 parity] {case} head ({b},{h}): max {e[0]:.3e} mean {e[1]:.3e}")


def test_fp8_full_size_sampled_rows():
    w = WORKLOADS["causal_train_b4h16n4096d128"]
    x = make_inputs_fp8(w.B, w.H, w.H, w.N, w.N, w.d, seed=w.seed)
    o, lse = _run(x, True, w.d)
    qd, kd, vd = (float(np.float32(f)) for f in x["descale"])
    q = e4m3_decode(_codes(x["q8"])).astype(np.float32) * np.float32(qd)
    k = e4m3_decode(_codes(x["k8"])).astype(np.float32) * np.float32(kd)
    v = e4m3_decode(_codes(x["v8"])).astype(np.float32) * np.float32(vd)
    rows = sampled_rows(w, 128)
    o_r, lse_r = oracle.attention_rows(q, k, v, w.scale, True, rows)
    for t, (b, h, i) in enumerate(rows):
        kh, vh = k[b, h, :i + 1].astype(np.float64), v[b, h, :i + 1].astype(np.float64)
        s = w.scale * (kh @ q[b, h, i].astype(np.float64))
        maxb, meanb, ok = fp8_bounds(s[None], vh, o_r[t][None])
        assert ok.all()
        assert np.all(np.abs(o[b, h, i] - o_r[t]) <= maxb[0]), f"row {(b, h, i)}"
        assert abs(lse[b, h, i] - lse_r[t]) <= TOL_LSE
    err = np.abs(np.stack([o[r] for r in rows]) - o_r)
    print(f"[fp8 parity] N4096 sampled rows: max {err.max():.3e} mean {err.mean():.3e}")


def test_fp8_rejects_bad_arguments():
    x = make_inputs_fp8(1, 1, 1, 64, 64, 128, seed=3)
    q8, k8, v8 = (x[n].cuda() for n in ("q8", "k8", "v8"))
    o = torch.empty(1, 1, 64, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 1, 64, dtype=torch.float32, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fa_fwd_fp8(q8, k8, v8, (1.0, 0.0, 1.0), o, lse)
    with pytest.raises(fa.FaError):
        fa.fa_fwd_fp8(q8, k8, v8, (1.0, 1.0, 1.0), o, lse,
                      workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
