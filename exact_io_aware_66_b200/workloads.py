"""Seeded synthetic inputs for the attention workloads.

This module is shared by the CUDA path's tests and bench and by the CPU oracle's callers. It
holds no attention arithmetic: it only draws N(0, 1) samples, applies the workload's fixed
multipliers, and rounds to bf16.

Recipe (every workload):
  * generator ``torch.Generator('cpu').manual_seed(seed)``;
  * draw q, k, v and then dO, in that order, each ``torch.randn(B, H, N, d, dtype=float32)``;
  * multiply by the workload's factor (0.5 for the causal N=4096 workload); for the N=131072
    workload, multiply key rows j with j % 97 == 0 by 8 (sharp softmax peaks);
  * round to bf16 (round-to-nearest-even, ``.to(torch.bfloat16)``).
Both multipliers are powers of two, so applying them before or after the bf16 rounding gives
identical bits. The same bf16 bits go to the GPU and, widened to float64, to the oracle.

The workloads mirror the five configurations the method is measured on: a small non-causal
forward (B2 H1 N512 d64), a non-causal training step (B8 H16 N2048 d64), and causal training
steps / forwards at N = 4096, 16384 and 131072 with d = 128.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    backward: bool          # does the workload include the backward pass
    mult: float = 1.0       # factor applied to q, k, v and dO
    spike_every: int = 0    # key rows j with j % spike_every == 0 are multiplied by spike
    spike: float = 1.0
    row_samples: int = 0    # 0 = compare every output; else number of sampled query rows
    key_samples: int = 0    # number of sampled keys for dK/dV (0 = all or none)

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(d) as the fp32 value both sides use."""
        return float(torch.tensor(1.0 / math.sqrt(self.d), dtype=torch.float32).item())

    def fwd_flops(self) -> float:
        """Algorithmic forward FLOPs: 4 B H N^2 d (two N x N x d GEMMs), halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Algorithmic backward FLOPs: 2.5 x forward (five N x N x d GEMMs vs two)."""
        return 2.5 * self.fwd_flops()


WORKLOADS = {
    "fwd_b2h1n512d64": Workload("fwd_b2h1n512d64", 2, 1, 512, 64, False, 1, False),
    "train_b8h16n2048d64": Workload("train_b8h16n2048d64", 8, 16, 2048, 64, False, 2, True),
    "causal_train_b4h16n4096d128": Workload("causal_train_b4h16n4096d128", 4, 16, 4096, 128, True,
                                            3, True, mult=0.5),
    "causal_train_b1h16n16384d128": Workload("causal_train_b1h16n16384d128", 1, 16, 16384, 128,
                                             True, 4, True, row_samples=512, key_samples=64),
    "causal_fwd_b1h8n131072d128": Workload("causal_fwd_b1h8n131072d128", 1, 8, 131072, 128, True,
                                           5, False, spike_every=97, spike=8.0, row_samples=256),
    # head dimension 96 (run by the d = 128 kernels on zero-filled columns), for measurement
    "causal_train_b4h16n4096d96": Workload("causal_train_b4h16n4096d96", 4, 16, 4096, 96, True, 7,
                                           True, mult=0.5, row_samples=256, key_samples=64),
    # head dimension 256, for measurement
    "causal_fwd_b2h16n8192d256": Workload("causal_fwd_b2h16n8192d256", 2, 16, 8192, 256, True, 6,
                                          False, row_samples=256),
    "causal_train_b2h16n8192d256": Workload("causal_train_b2h16n8192d256", 2, 16, 8192, 256, True,
                                            6, True, row_samples=256, key_samples=64),
}


def make_inputs(B: int, H: int, N: int, d: int, seed: int, mult: float = 1.0,
                spike_every: int = 0, spike: float = 1.0, with_do: bool = True) -> dict:
    """Returns {'q','k','v'[, 'do']} as contiguous bf16 CPU tensors of shape [B, H, N, d]."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    names = ["q", "k", "v"] + (["do"] if with_do else [])
    out = {}
    for name in names:
        x = torch.randn(B, H, N, d, dtype=torch.float32, generator=g)
        if mult != 1.0:
            x.mul_(mult)
        if name == "k" and spike_every:
            x[:, :, ::spike_every, :].mul_(spike)
        out[name] = x.to(torch.bfloat16).contiguous()
    return out


def make_inputs_ex(B: int, H: int, H_kv: int, N_q: int, N_kv: int, d: int, seed: int) -> dict:
    """{'q','do'} of shape [B, H, N_q, d] and {'k','v'} of shape [B, H_kv, N_kv, d], contiguous
    bf16 CPU tensors of standard normal draws (for grouped heads and unequal lengths)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    out = {}
    for name, (h, n) in (("q", (H, N_q)), ("k", (H_kv, N_kv)), ("v", (H_kv, N_kv)),
                         ("do", (H, N_q))):
        out[name] = torch.randn(B, h, n, d, dtype=torch.float32, generator=g).to(
            torch.bfloat16).contiguous()
    return out


def make_inputs_fp8(B: int, H: int, H_kv: int, N_q: int, N_kv: int, d: int, seed: int) -> dict:
    """E4M3 inputs: {'q8','k8','v8'} as contiguous torch.float8_e4m3fn CPU tensors (q8 of shape
    [B, H, N_q, d], k8 and v8 of shape [B, H_kv, N_kv, d]) and {'descale': (q, k, v)}, fp32
    factors. Standard normal draws, each tensor divided by amax / 448 and rounded to E4M3 by
    torch, so the codes span E4M3's range; the value of a code is its E4M3 value times its
    factor."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    out, descale = {}, []
    for name, (h, n) in (("q8", (H, N_q)), ("k8", (H_kv, N_kv)), ("v8", (H_kv, N_kv))):
        x = torch.randn(B, h, n, d, dtype=torch.float32, generator=g)
        f = float(torch.tensor(float(x.abs().max()) / 448.0, dtype=torch.float32))
        out[name] = (x / f).to(torch.float8_e4m3fn).contiguous()
        descale.append(f)
    out["descale"] = tuple(descale)
    return out


def workload_inputs(w: Workload, with_do: bool | None = None) -> dict:
    if with_do is None:
        with_do = w.backward
    return make_inputs(w.B, w.H, w.N, w.d, w.seed, w.mult, w.spike_every, w.spike, with_do)


def sampled_rows(w: Workload, n: int, seed_offset: int = 1000):
    """n distinct (b, h, i) query rows drawn uniformly without replacement from
    numpy PCG64(seed + 1000), plus row 0 and row N-1 of head (0, 0) always."""
    import numpy as np

    rng = np.random.Generator(np.random.PCG64(w.seed + seed_offset))
    total = w.B * w.H * w.N
    flat = rng.choice(total, size=min(n, total), replace=False)
    rows = {(0, 0, 0), (0, 0, w.N - 1)}
    for f in flat.tolist():
        b, rem = divmod(int(f), w.H * w.N)
        h, i = divmod(rem, w.N)
        rows.add((b, h, i))
    return sorted(rows)


def sampled_keys(w: Workload, n: int, max_heads: int = 4, seed_offset: int = 2000):
    """n (b, h, j) keys drawn from at most `max_heads` seeded heads (PCG64(seed + 2000)),
    always including key 0 and key N-1 of the first chosen head."""
    import numpy as np

    rng = np.random.Generator(np.random.PCG64(w.seed + seed_offset))
    nheads = min(max_heads, w.B * w.H)
    heads = rng.choice(w.B * w.H, size=nheads, replace=False).tolist()
    per = max(1, n // nheads)
    keys = []
    for t, hh in enumerate(heads):
        b, h = divmod(int(hh), w.H)
        js = set(rng.choice(w.N, size=min(per, w.N), replace=False).tolist())
        if t == 0:
            js |= {0, w.N - 1}
        keys.extend((b, h, int(j)) for j in sorted(js))
    return keys
