"""Forward parity: the CUDA path (through the C ABI) against the fp64 oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import WORKLOADS, make_inputs, sampled_rows, workload_inputs
from parity import assert_fwd_ok, fwd_errors, to64

pytestmark = pytest.mark.gpu

SMALL = [  # (B, H, N, d): several tiles, ragged tails, N = 1, N < one tile
    (1, 2, 1, 64), (1, 1, 5, 128), (2, 1, 128, 64), (1, 2, 200, 128), (1, 1, 256, 64),
    (2, 2, 300, 128), (1, 1, 640, 64), (1, 3, 1000, 128), (2, 1, 1152, 64),
]


def _run(x, causal, scale=None):
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=scale)
    fa.fa_check_status()
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "b%dh%dn%dd%d" % s)
def test_fwd_small_full_compare(shape, causal):
    B, H, N, d = shape
    x = make_inputs(B, H, N, d, seed=100 + N + d, with_do=False)
    o, lse = _run(x, causal)
    scale = fa.default_scale(d)
    o_ref, lse_ref = oracle.attention_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]), scale,
                                              causal)
    assert_fwd_ok(fwd_errors(o, lse, o_ref, lse_ref), f"{shape} causal={causal}")


def test_fwd_first_config_full():
    """B=2, H=1, N=512, d=64 non-causal: every O and lse entry against the oracle."""
    w = WORKLOADS["fwd_b2h1n512d64"]
    x = workload_inputs(w)
    o, lse = _run(x, w.causal)
    o_ref, lse_ref = oracle.attention_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]), w.scale,
                                              w.causal)
    err = fwd_errors(o, lse, o_ref, lse_ref)
    assert err["format_limited"] == 0
    assert_fwd_ok(err, w.name)


@pytest.mark.parametrize("name", ["causal_train_b1h16n16384d128", "causal_fwd_b1h8n131072d128",
                                  "causal_train_b4h16n4096d96"])
def test_fwd_full_size_sampled_rows(name):
    """The two long-sequence workloads and the d = 96 one (its products run over 96 columns of
    the d = 128 layout), same launch configuration as the bench: sampled query rows (512, or 256)
    against the oracle, and every output finite. (The d = 64 N = 2048 and d = 128 N = 4096
    workloads are compared element by element in test_bwd_gpu.py.)"""
    w = WORKLOADS[name]
    x = workload_inputs(w, with_do=False)
    o, lse = _run(x, w.causal)
    assert torch.isfinite(o).all() and torch.isfinite(lse).all()
    rows = sampled_rows(w, w.row_samples or 512)
    q, k, v = (x[n] for n in ("q", "k", "v"))
    o_ref, lse_ref = oracle.attention_rows(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                           w.scale, w.causal, rows)
    idx = tuple(np.array(rows).T)
    o_s = to64(o)[idx]
    l_s = to64(lse)[idx]
    err = fwd_errors(o_s, l_s, o_ref, lse_ref)
    assert err["format_limited"] == 0, f"{name}: {err['format_limited']} elements with |O| >= 4"
    assert_fwd_ok(err, name)


@pytest.mark.parametrize("d", [64, 128])
def test_causal_masked_keys_have_no_effect(d):
    """Rows masked out by causality match exactly: changing K and V rows j > i0 leaves O and
    lse of rows <= i0 bit-identical."""
    B, H, N, i0 = 1, 2, 640, 300
    x = make_inputs(B, H, N, d, seed=7, with_do=False)
    o1, l1 = _run(x, True)
    y = dict(x)
    g = torch.Generator().manual_seed(99)
    for n in ("k", "v"):
        t = x[n].clone()
        t[:, :, i0 + 1:] = (torch.randn(t[:, :, i0 + 1:].shape, generator=g) * 3).to(t.dtype)
        y[n] = t
    o2, l2 = _run(y, True)
    assert torch.equal(o1[:, :, :i0 + 1], o2[:, :, :i0 + 1])
    assert torch.equal(l1[:, :, :i0 + 1], l2[:, :, :i0 + 1])
    assert not torch.equal(o1[:, :, i0 + 1:], o2[:, :, i0 + 1:])


@pytest.mark.parametrize("d", [64, 128])
def test_causal_first_row_is_v0(d):
    """Row 0 sees only key 0: O_0 equals V_0 bit for bit; lse_0 = scale q_0 . k_0."""
    x = make_inputs(2, 2, 384, d, seed=8, with_do=False)
    o, lse = _run(x, True)
    assert torch.equal(o[:, :, 0].cpu(), x["v"][:, :, 0])
    s00 = (to64(x["q"][:, :, 0]) * to64(x["k"][:, :, 0])).sum(-1) * fa.default_scale(d)
    assert np.abs(to64(lse[:, :, 0]) - s00).max() <= 1e-5


def test_fwd_deterministic():
    x = make_inputs(1, 4, 1024, 128, seed=9, with_do=False)
    o1, l1 = _run(x, True)
    o2, l2 = _run(x, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_nondefault_scale():
    x = make_inputs(1, 2, 333, 64, seed=10, with_do=False)
    o, lse = _run(x, False, scale=0.05)
    o_ref, lse_ref = oracle.attention_forward(to64(x["q"]), to64(x["k"]), to64(x["v"]),
                                              float(np.float32(0.05)), False)
    assert_fwd_ok(fwd_errors(o, lse, o_ref, lse_ref), "scale=0.05")


def test_fwd_rejects_bad_args_on_gpu():
    x = make_inputs(1, 1, 128, 64, seed=11, with_do=False)
    q = x["q"].cuda()
    with pytest.raises(ValueError):
        fa.attention_forward(q, q.float(), q)
    o = torch.empty_like(q)
    lse = torch.empty(1, 1, 128, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fa_fwd(q, q, q, o, lse, scale=-1.0)
