"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory (for example a
plugin inside a framework that keeps all GPU memory in its own pool and offers no workspace,
or a service that must not allocate after start-up). It uses scratch built into the library
instead of a caller-provided workspace. These tests call it through the C ABI and check that
it gives the same gradients as fa_bwd (the allocating entry point), on two calls in a row, so
that the second call also sees the scratch left behind by the first.

This file is collected last on purpose: it must pass both in a fresh process and after every
other test.
"""

from __future__ import annotations

import pytest
import torch

from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import make_inputs
from parity import TOL_GRAD_REL, grad_rel_error, to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,causal", [((2, 4, 1000, 128), True), ((1, 3, 640, 64), False)])
def test_noalloc_backward_matches_fa_bwd_twice(shape, causal):
    B, H, N, d = shape
    x = make_inputs(B, H, N, d, seed=31 + d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=causal)
    ref = fa.attention_backward(q, k, v, o, do, lse, causal=causal)  # allocating entry point
    fa.fa_check_status()
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        # garbage in the outputs: the call must overwrite every element
        for t in (dq, dk, dv):
            t.fill_(float("nan"))
        fa.fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal=causal)
        torch.cuda.synchronize()
        for g, r, n in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
            assert torch.isfinite(g).all(), f"call {call}: {n} not fully written"
            err = grad_rel_error(g, to64(r))
            assert err <= TOL_GRAD_REL, f"call {call}: {n} differs from fa_bwd by {err:.3e}"
        # dK and dV come from one CTA each in a fixed order: identical to fa_bwd's
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])


def test_noalloc_rejects_sizes_beyond_builtin_scratch():
    """Sizes whose scratch exceeds the built-in 64 MiB fail with FA_ERR_UNSUPPORTED before any
    launch (the pointers are never touched)."""
    B, H, N, d = 1, 64, 4096, 128
    assert fa.fa_bwd_workspace_size(B, H, N, d) > 64 << 20
    fake = 1 << 24  # 16-byte aligned, never dereferenced: validation rejects the call first
    st = fa.lib().fa_bwd_noalloc(fake, fake * 2, fake * 3, fake * 4, fake * 5, fake * 6,
                                 fake * 7, fake * 8, fake * 9, B, H, N, d, 0.088, 1, None)
    assert st == 2
    assert "built into the library" in fa.fa_last_error_string()


def test_noalloc_d256_matches_fa_bwd():
    """d = 256 (the two-pass backward) through the built-in scratch: same gradients as fa_bwd."""
    B, H, N, d = 1, 2, 700, 256
    x = make_inputs(B, H, N, d, seed=39)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    ref = fa.attention_backward(q, k, v, o, do, lse, causal=True)
    fa.fa_check_status()
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        for t in (dq, dk, dv):
            t.fill_(float("nan"))
        fa.fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, causal=True)
        fa.fa_check_status()
        for g, r, n in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
            assert torch.isfinite(g).all(), f"call {call}: {n} not fully written"
            assert grad_rel_error(g, to64(r)) <= TOL_GRAD_REL, f"call {call}: {n}"
        assert torch.equal(dk, ref[1]) and torch.equal(dv, ref[2])
