"""Out-of-bounds writes (a stand-in for a memory checker, which this environment does not
offer): every output and workspace of the library is placed inside a larger buffer whose
margins (8 KiB on each side) hold a sentinel byte pattern, and after the call every margin byte
must be unchanged. The cases are the ones where the kernels clip: ragged row counts (TMA stores
drop rows past N), d = 96 (stores drop columns 96..127), grouped heads, unequal lengths, rows
that see no key, keys that no query sees, the d = 256 forward and backward and the FP8 forward."""

from __future__ import annotations

import pytest
import torch

from exact_io_aware_66_b200 import fa
from exact_io_aware_66_b200.workloads import make_inputs_ex, make_inputs_fp8

pytestmark = pytest.mark.gpu

MARGIN = 8192
SENTINEL = 0xA5


class Guarded:
    """A tensor of `shape` and `dtype` placed MARGIN bytes into a sentinel-filled buffer."""

    def __init__(self, shape, dtype, nbytes=None):
        if nbytes is None:
            n = 1
            for s in shape:
                n *= s
            nbytes = n * torch.empty((), dtype=dtype).element_size()
            self.nbytes, raw = nbytes, False
        else:
            self.nbytes, raw = nbytes, True
        self.buf = torch.full((2 * MARGIN + self.nbytes,), SENTINEL, dtype=torch.uint8,
                              device="cuda")
        inner = self.buf[MARGIN:MARGIN + self.nbytes]
        self.t = inner if raw else inner.view(dtype).view(*shape)

    def check(self, what):
        lo = self.buf[:MARGIN]
        hi = self.buf[MARGIN + self.nbytes:]
        bad_lo = int((lo != SENTINEL).sum())
        bad_hi = int((hi != SENTINEL).sum())
        assert bad_lo == 0 and bad_hi == 0, (
            f"{what}: {bad_lo} bytes changed before and {bad_hi} after the buffer")


CASES = [  # (B, H, H_kv, N_q, N_kv, d, mask)
    (1, 1, 1, 1, 1, 64, False),
    (1, 2, 2, 5, 5, 128, True),
    (2, 1, 1, 200, 200, 64, True),
    (1, 2, 2, 300, 300, 128, False),
    (1, 3, 3, 1000, 1000, 128, True),
    (2, 1, 1, 1152, 1152, 64, False),
    (1, 4, 1, 300, 300, 64, True),
    (2, 8, 2, 513, 513, 128, True),
    (1, 2, 2, 100, 700, 128, "bottom_right"),
    (1, 2, 1, 1, 1000, 64, "bottom_right"),
    (1, 2, 2, 700, 300, 64, "bottom_right"),
    (1, 1, 1, 300, 1, 128, "bottom_right"),
    (1, 2, 2, 200, 600, 64, True),
    (1, 2, 2, 200, 600, 128, True),
    (1, 2, 2, 300, 300, 96, False),
    (2, 4, 2, 513, 513, 96, True),
    (1, 2, 1, 100, 700, 96, "bottom_right"),
]


def _ids(c):
    return "b%dh%dkv%dq%dk%dd%d-%s" % c


@pytest.mark.parametrize("case", CASES, ids=_ids)
@pytest.mark.parametrize("dropout", [None, (0.2, 77, 3)], ids=["plain", "dropout"])
def test_forward_backward_write_only_their_outputs(case, dropout):
    B, H, H_kv, N_q, N_kv, d, mask = case
    x = make_inputs_ex(B, H, H_kv, N_q, N_kv, d, seed=900 + N_q + N_kv + d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o = Guarded((B, H, N_q, d), torch.bfloat16)
    lse = Guarded((B, H, N_q), torch.float32)
    fa.fa_fwd_ex(q, k, v, o.t, lse.t, causal=mask, dropout=dropout)
    fa.fa_check_status()
    o.check("o")
    lse.check("lse")
    dq = Guarded((B, H, N_q, d), torch.bfloat16)
    dk = Guarded((B, H_kv, N_kv, d), torch.bfloat16)
    dv = Guarded((B, H_kv, N_kv, d), torch.bfloat16)
    ws = Guarded(None, torch.uint8,
                 nbytes=fa.fa_bwd_ex_workspace_size(B, H, H_kv, N_q, N_kv, d, mask))
    fa.fa_bwd_ex(q, k, v, o.t, do, lse.t, dq.t, dk.t, dv.t, ws.t, causal=mask, dropout=dropout)
    fa.fa_check_status()
    for g, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (ws, "workspace")):
        g.check(n)
    for t in (o.t, dq.t, dk.t, dv.t):
        assert torch.isfinite(t).all()


@pytest.mark.parametrize("case", [(1, 1, 1, 1, 1, False), (1, 2, 2, 300, 300, True),
                                  (2, 4, 2, 513, 513, True), (1, 2, 1, 100, 700, "bottom_right"),
                                  (1, 2, 2, 700, 300, "bottom_right")],
                         ids=lambda c: "b%dh%dkv%dq%dk%d-%s" % c)
def test_d256_forward_backward_write_only_their_outputs(case):
    B, H, H_kv, N_q, N_kv, mask = case
    x = make_inputs_ex(B, H, H_kv, N_q, N_kv, 256, seed=950 + N_q + N_kv)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o = Guarded((B, H, N_q, 256), torch.bfloat16)
    lse = Guarded((B, H, N_q), torch.float32)
    fa.fa_fwd_ex(q, k, v, o.t, lse.t, causal=mask)
    fa.fa_check_status()
    o.check("o")
    lse.check("lse")
    dq = Guarded((B, H, N_q, 256), torch.bfloat16)
    dk = Guarded((B, H_kv, N_kv, 256), torch.bfloat16)
    dv = Guarded((B, H_kv, N_kv, 256), torch.bfloat16)
    ws = Guarded(None, torch.uint8,
                 nbytes=fa.fa_bwd_ex_workspace_size(B, H, H_kv, N_q, N_kv, 256, mask))
    fa.fa_bwd_ex(q, k, v, o.t, do, lse.t, dq.t, dk.t, dv.t, ws.t, causal=mask)
    fa.fa_check_status()
    for g, n in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (ws, "workspace")):
        g.check(n)
    for t in (dq.t, dk.t, dv.t):
        assert torch.isfinite(t).all()


@pytest.mark.parametrize("case", [(1, 1, 1, 1, 1, 64, False), (1, 2, 2, 300, 300, 128, True),
                                  (2, 4, 2, 513, 513, 96, True),
                                  (1, 2, 1, 100, 700, 64, "bottom_right"),
                                  (1, 2, 2, 700, 300, 128, "bottom_right")], ids=_ids)
def test_fp8_forward_writes_only_its_outputs(case):
    B, H, H_kv, N_q, N_kv, d, mask = case
    x = make_inputs_fp8(B, H, H_kv, N_q, N_kv, d, seed=970 + N_q + N_kv + d)
    q8, k8, v8 = (x[n].cuda() for n in ("q8", "k8", "v8"))
    o = Guarded((B, H, N_q, d), torch.bfloat16)
    lse = Guarded((B, H, N_q), torch.float32)
    ws = Guarded(None, torch.uint8,
                 nbytes=fa.fa_fwd_fp8_workspace_size(B, H, H_kv, N_q, N_kv, d, mask))
    fa.fa_fwd_fp8(q8, k8, v8, x["descale"], o.t, lse.t, causal=mask, workspace=ws.t)
    fa.fa_check_status()
    for g, n in ((o, "o"), (lse, "lse"), (ws, "workspace")):
        g.check(n)
