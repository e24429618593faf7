"""Exact scaled-dot-product attention and its gradient in plain fp64 NumPy (the oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the product path.

What is computed, and where it is defined:

* Forward. "Breaking the Memory Wall: A Deep Dive into FlashAttention" (codethepapers.com),
  section "The Problem: The Memory Wall": P = softmax(Q K^T / sqrt(d)) and the output is the
  P-weighted sum of V rows; section "The Incremental Softmax Trick" gives
  softmax(x_i) = e^{x_i} / sum_j e^{x_j}. The three pages agree that the method is exact
  ("How FlashAttention Actually Works", section "Practical Takeaways": mathematically identical
  to standard attention), so the oracle is the unchunked definition, not the tiled algorithm.
  Per row i, with s_ij = scale * q_i . k_j:
      m_i   = max_j s_ij                       (running maximum m, "The Secret Weapon: Online
      l_i   = sum_j exp(s_ij - m_i)             Softmax", same page, names m and l)
      O_i   = sum_j exp(s_ij - m_i) v_j / l_i
      lse_i = m_i + ln l_i                      (natural log; the stored "normalization
                                                 factors" of "Backward Pass Recomputation")
  The max subtraction changes nothing mathematically; it keeps exp() in range.
* Causal masking: masked entries are left out of every sum, i.e. they contribute exactly zero.
  The pages name masking only as one of standard attention's HBM passes ("The GPU Memory Wall:
  HBM vs. SRAM"). Modes: "none"; "top_left" (key j visible to query i iff j <= i; also
  `causal=True`); "bottom_right" (iff j <= i + N_k - N_q, the alignment where the last query
  sees every key, as in decoding). A query row that sees no key at all (bottom-right with
  N_q > N_k) has O = 0 and lse = -inf, and contributes nothing to any gradient.
* Grouped heads: when K and V have H_kv < H heads ([B, H_kv, N_k, d] against [B, H, N_q, d],
  H a multiple of H_kv), query head h uses key/value head h // (H / H_kv); the gradients of a
  key/value head sum over the query heads that share it.
* Backward. The pages say only that the scores are recomputed on chip and the gradients
  calculated ("The Backward Pass: Recomputation"). The formulas are the calculus of the
  definition above, with P_ij = exp(s_ij - lse_i) and L a scalar loss with dO = dL/dO:
      dV = P^T dO
      dP = dO V^T
      D_i = sum_c dO_ic O_ic          (= sum_j P_ij dP_ij, the softmax-Jacobian row term)
      dS = P o (dP - D)               (o = elementwise product; masked entries are exactly 0)
      dQ = scale * dS K,   dK = scale * dS^T Q
* Dropout (optional, ``dropout=(p, seed, offset)``): inverted dropout on P, applied where
  "How FlashAttention Actually Works", section "The GPU Memory Wall: HBM vs. SRAM", places it
  (on the softmax matrix, before the product with V). With Z the keep decisions of
  ``oracle.dropout`` and r = 256 / (256 - p8) the keep scale:
      O_i = r sum_j Z_ij P_ij v_j,   lse_i unchanged (the undropped softmax)
      dV = r (Z o P)^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P o (r Z o dP - D)
  (D is still rowsum(dO o O) with the dropped O: sum_j P_ij r Z_ij dP_ij = dO_i . O_i).
* Tiled forward with online softmax. "How does FlashAttention optimize memory and speed via
  tiling?" (iloveeagents.com), section "Core Technical Innovations", item 2 gives the update
      m^(2) = max(m^(1), m~),  d^(2) = e^{m^(1) - m^(2)} d^(1) + e^{m~ - m^(2)} d~
  and "How FlashAttention Actually Works", section "How Tiling Works", gives the loop order
  (blocks of K/V outside, blocks of Q inside). ``tiled_attention_forward`` follows those steps,
  with the partial output rescaled by the same factor as the running sum; it is used only to
  pin that the tiled algorithm reaches the definition for every block size.

Inputs are the exact bf16 values sent to the GPU, widened to float64; ``scale`` is the fp32
value passed to the kernels, widened to float64.

Rows are processed in blocks of ``block_rows`` only to bound memory to O(block_rows * N); each
row's arithmetic is the definition above and does not depend on the blocking (a test checks
this).
"""

from __future__ import annotations

import numpy as np

from .dropout import dropout_keep, dropout_p8, keep_scale

__all__ = [
    "attention_probabilities",
    "attention_forward",
    "attention_backward",
    "attention_rows",
    "attention_keys",
    "online_softmax_stats",
    "tiled_attention_forward",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def _mode(causal) -> str:
    """Normalises the mask argument: False/None/"none", True/"top_left", "bottom_right"."""
    if causal is True:
        return "top_left"
    if causal is False or causal is None:
        return "none"
    if causal in ("none", "top_left", "bottom_right"):
        return causal
    raise ValueError(f"unknown mask mode {causal!r}")


def _visible(i: int, n_q: int, n_keys: int, mode: str) -> int:
    """Number of keys visible to query row i (keys 0 .. result-1); may be 0."""
    if mode == "none":
        return n_keys
    off = (n_keys - n_q) if mode == "bottom_right" else 0
    return int(min(max(i + 1 + off, 0), n_keys))


def _head_iter(shape):
    """Iterate over every leading index of a [..., N, d] array."""
    lead = shape[:-2]
    return np.ndindex(*lead) if lead else iter([()])


def _kv_index(idx, q_shape, k_shape):
    """Leading index of the key/value head used by the query head at leading index `idx`."""
    if len(q_shape) >= 4 and k_shape[-3] != q_shape[-3]:
        group = q_shape[-3] // k_shape[-3]
        return tuple(idx[:-1]) + (idx[-1] // group,)
    return idx


def _softmax_block(s: np.ndarray, mask: np.ndarray | None):
    """Row statistics of a block of scores s [r, n] with optional visibility mask.

    Returns (m, e, l): row max over visible entries, e = exp(s - m) with masked entries set to
    exactly 0, and l = row sum of e.
    """
    if mask is None:
        m = s.max(axis=1)
        e = np.exp(s - m[:, None])
    else:
        m = np.where(mask, s, -np.inf).max(axis=1)
        m_safe = np.where(np.isfinite(m), m, 0.0)  # rows without any visible key
        e = np.where(mask, np.exp(np.where(mask, s, 0.0) - m_safe[:, None]), 0.0)
    return m, e, e.sum(axis=1)


def _dropout(dropout):
    """(p8, keep scale, seed, offset) for ``dropout=(p, seed, offset)``, or None."""
    if dropout is None:
        return None
    p, seed, offset = dropout
    p8 = dropout_p8(p)
    return p8, keep_scale(p8), int(seed), int(offset)


def _flat_head(idx, q_shape) -> int:
    """Flattened query-head index (b * H + h for [B, H, N, d]) of leading index `idx`."""
    lead = q_shape[:-2]
    return int(np.ravel_multi_index(idx, lead)) if lead else 0


def _finish(e, l, m, v, z=None, r=1.0):
    """O = e V / l and lse = m + ln l, with O = 0 and lse = -inf for rows that see no key.
    With dropout keep decisions z and keep scale r: O = r (z o e) V / l."""
    empty = l == 0.0
    num = (e @ v) if z is None else r * ((e * z) @ v)
    o = num / np.where(empty, 1.0, l)[:, None]
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m + np.log(np.where(empty, 1.0, l)))
    return o, lse


def _mask(r0: int, r1: int, n_q: int, n_keys: int, mode: str):
    """Visibility of keys [0, n_keys) to query rows [r0, r1), or None when all are visible."""
    if mode == "none":
        return None
    off = (n_keys - n_q) if mode == "bottom_right" else 0
    rows = np.arange(r0, r1)[:, None]
    cols = np.arange(n_keys)[None, :]
    return cols <= rows + off


def attention_probabilities(q, k, scale: float, causal=False) -> np.ndarray:
    """P = softmax(scale * Q K^T) per the definition (codethepapers.com, "The Problem: The
    Memory Wall"), masked entries exactly 0 (rows that see no key are all 0). Shapes:
    q [..., N, d], k [..., M, d] -> [..., N, M]. Small inputs only (materialises N x M)."""
    q, k = _f64(q), _f64(k)
    mode = _mode(causal)
    scale = float(np.float64(scale))
    out = np.zeros(q.shape[:-1] + (k.shape[-2],), dtype=np.float64)
    for idx in _head_iter(q.shape):
        kh = k[_kv_index(idx, q.shape, k.shape)]
        s = scale * (q[idx] @ kh.T)
        _, e, l = _softmax_block(s, _mask(0, q.shape[-2], q.shape[-2], k.shape[-2], mode))
        out[idx] = e / np.where(l == 0.0, 1.0, l)[:, None]
    return out


def attention_forward(q, k, v, scale: float, causal=False, block_rows: int = 512,
                      dropout=None):
    """Exact attention forward: returns (O [..., N_q, d], lse [..., N_q]) in float64.

    Definition: codethepapers.com, "The Problem: The Memory Wall" (P = softmax(QK^T/sqrt d),
    output P V) with the running max m and sum l of hot.atechcom.net, "The Secret Weapon:
    Online Softmax"; lse = m + ln l. Masked entries contribute exactly 0; `causal` is a mask
    mode (see the module docstring); K/V may have fewer heads than Q (grouped heads);
    `dropout` = (p, seed, offset) applies inverted dropout to P (module docstring).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    mode = _mode(causal)
    drop = _dropout(dropout)
    scale = float(np.float64(scale))
    n, nk = q.shape[-2], k.shape[-2]
    o = np.zeros(q.shape[:-1] + (v.shape[-1],), dtype=np.float64)
    lse = np.zeros(q.shape[:-1], dtype=np.float64)
    for idx in _head_iter(q.shape):
        kvi = _kv_index(idx, q.shape, k.shape)
        qh, kh, vh = q[idx], k[kvi], v[kvi]
        for r0 in range(0, n, block_rows):
            r1 = min(n, r0 + block_rows)
            # keys beyond the last visible one of this block are masked for every row in it
            kv_end = _visible(r1 - 1, n, nk, mode)
            s = scale * (qh[r0:r1] @ kh[:kv_end].T)
            m, e, l = _softmax_block(s, _mask(r0, r1, n, nk, mode)[:, :kv_end]
                                     if mode != "none" else None)
            z, r = None, 1.0
            if drop is not None:
                p8, r, seed, offset = drop
                z = dropout_keep(_flat_head(idx, q.shape), range(r0, r1), kv_end, p8, seed, offset)
            o[idx][r0:r1], lse[idx][r0:r1] = _finish(e, l, m, vh[:kv_end], z, r)
    return o, lse


def attention_backward(q, k, v, do, scale: float, causal: bool = False, block_rows: int = 512,
                       return_forward: bool = False, dropout=None):
    """Gradient of exact attention: returns (dQ, dK, dV) in float64 (and (O, lse) if asked).

    Recomputes O and lse from the definition (attention_forward), then
    P = exp(S - lse), dV = P^T dO, dP = dO V^T, D = rowsum(dO o O), dS = P o (dP - D),
    dQ = scale dS K, dK = scale dS^T Q. These are the calculus of the forward definition; the
    pages only state that scores are recomputed on chip in the backward ("How FlashAttention
    Actually Works", "The Backward Pass: Recomputation"). D uses the oracle's own fp64 O.
    With `dropout`, the module docstring's dropout formulas apply (same keep decisions as the
    forward).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    mode = _mode(causal)
    scale = float(np.float64(scale))
    drop = _dropout(dropout)
    o, lse = attention_forward(q, k, v, scale, mode, block_rows, dropout)
    n, nk = q.shape[-2], k.shape[-2]
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for idx in _head_iter(q.shape):
        kvi = _kv_index(idx, q.shape, k.shape)
        qh, kh, vh, doh = q[idx], k[kvi], v[kvi], do[idx]
        dd = np.sum(doh * o[idx], axis=1)  # D_i
        for r0 in range(0, n, block_rows):
            r1 = min(n, r0 + block_rows)
            kv_end = _visible(r1 - 1, n, nk, mode)
            if kv_end == 0:
                continue  # no row of this block sees a key: no gradient flows
            s = scale * (qh[r0:r1] @ kh[:kv_end].T)
            mask = _mask(r0, r1, n, nk, mode)
            with np.errstate(over="ignore"):
                p = np.exp(s - lse[idx][r0:r1, None])
            if mask is not None:
                p = np.where(mask[:, :kv_end], p, 0.0)
            dp = doh[r0:r1] @ vh[:kv_end].T
            if drop is None:
                dv[kvi][:kv_end] += p.T @ doh[r0:r1]
                ds = p * (dp - dd[r0:r1, None])
            else:
                p8, r, seed, offset = drop
                z = dropout_keep(_flat_head(idx, q.shape), range(r0, r1), kv_end, p8, seed, offset)
                dv[kvi][:kv_end] += r * ((z * p).T @ doh[r0:r1])
                ds = p * (r * z * dp - dd[r0:r1, None])
            dq[idx][r0:r1] = scale * (ds @ kh[:kv_end])
            dk[kvi][:kv_end] += scale * (ds.T @ qh[r0:r1])
    if return_forward:
        return dq, dk, dv, o, lse
    return dq, dk, dv


def attention_rows(q, k, v, scale: float, causal: bool, rows, do=None, dropout=None):
    """Forward (and dQ) for selected query rows only; cost O(N d) per row.

    rows: iterable of index tuples (leading indices..., i), e.g. (b, h, i) for [B, H, N, d].
    Returns (O_rows [n, d], lse_rows [n]) or, with dO given, (O_rows, lse_rows, dQ_rows).
    Each row follows the same definition as attention_forward / attention_backward.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    do = None if do is None else _f64(do)
    mode = _mode(causal)
    drop = _dropout(dropout)
    scale = float(np.float64(scale))
    rows = [tuple(int(t) for t in r) for r in rows]
    n, nk = q.shape[-2], k.shape[-2]
    o_out = np.zeros((len(rows), v.shape[-1]))
    lse_out = np.zeros(len(rows))
    dq_out = np.zeros((len(rows), q.shape[-1])) if do is not None else None
    for t, r in enumerate(rows):
        head, i = r[:-1], r[-1]
        vis = _visible(i, n, nk, mode)
        if vis == 0:
            lse_out[t] = -np.inf  # O and dQ stay 0
            continue
        kvi = _kv_index(head, q.shape, k.shape)
        kh, vh = k[kvi][:vis], v[kvi][:vis]
        s = scale * (kh @ q[head][i])
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        zr = 1.0  # keep decision times keep scale, per key
        if drop is not None:
            p8, r, seed, offset = drop
            zr = r * dropout_keep(_flat_head(head, q.shape), [i], vis, p8, seed, offset)[0]
        o_i = ((e * zr) @ vh) / l
        o_out[t] = o_i
        lse_out[t] = m + np.log(l)
        if do is not None:
            p = e / l
            do_i = do[head][i]
            dp = vh @ do_i
            ds = p * (zr * dp - do_i @ o_i)
            dq_out[t] = scale * (ds @ kh)
    if do is not None:
        return o_out, lse_out, dq_out
    return o_out, lse_out


def attention_keys(q, k, v, do, scale: float, causal, head, keys, block_rows: int = 512,
                   dropout=None, stats=None):
    """dK and dV rows for selected keys j of one key/value head (leading index tuple `head`,
    e.g. (b, h_kv)).

    dV_j = sum_i P_ij dO_i and dK_j = scale sum_i dS_ij q_i over the query rows that see key j,
    in every query head that uses this key/value head. Needs lse_i and D_i of those rows, so
    their full forward is computed first, unless `stats` = (O [n, d], lse [n]) of the query
    head's rows is given (one query head per key/value head only; only the rows that see the
    selected keys are read, so the others may hold anything, e.g. NaN). This lets a caller take
    those rows from ``attention_rows`` when the full forward is too long to run.
    Returns (dK_rows [n, d], dV_rows [n, d]).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    mode = _mode(causal)
    scale = float(np.float64(scale))
    drop = _dropout(dropout)
    head = tuple(int(t) for t in head)
    kh, vh = k[head], v[head]
    n, nk = q.shape[-2], k.shape[-2]
    if q.ndim >= 4 and k.shape[-3] != q.shape[-3]:
        group = q.shape[-3] // k.shape[-3]
        q_heads = [head[:-1] + (head[-1] * group + g,) for g in range(group)]
    else:
        q_heads = [head]
    off = (nk - n) if mode == "bottom_right" else 0
    dk_out = np.zeros((len(keys), kh.shape[1]))
    dv_out = np.zeros((len(keys), vh.shape[1]))
    if stats is not None and len(q_heads) != 1:
        raise ValueError("stats is supported with one query head per key/value head")
    for qh_idx in q_heads:
        qh, doh = q[qh_idx], do[qh_idx]
        bh = _flat_head(qh_idx, q.shape)
        if stats is None:
            o, lse = _forward_one_head(qh, kh, vh, scale, mode, block_rows, bh, drop)
        else:
            o, lse = _f64(stats[0]), _f64(stats[1])
        with np.errstate(invalid="ignore"):  # rows outside i0 .. n may hold NaN
            dd = np.sum(doh * o, axis=1)
        for t, j in enumerate(int(x) for x in keys):
            i0 = 0 if mode == "none" else max(0, j - off)  # rows i with j <= i + off see key j
            if i0 >= n:
                continue
            s = scale * (qh[i0:n] @ kh[j])
            p = np.exp(s - lse[i0:n])
            zr = 1.0
            if drop is not None:
                p8, r, seed, offset = drop
                zr = r * dropout_keep(bh, range(i0, n), [j], p8, seed, offset)[:, 0]
            dv_out[t] += (zr * p) @ doh[i0:n]
            dp = doh[i0:n] @ vh[j]
            ds = p * (zr * dp - dd[i0:n])
            dk_out[t] += scale * (ds @ qh[i0:n])
    return dk_out, dv_out


def _forward_one_head(qh, kh, vh, scale, mode, block_rows, bh, drop):
    """attention_forward of one [N, d] head whose flattened query-head index is bh (the index
    that selects its dropout draws)."""
    n, nk = qh.shape[0], kh.shape[0]
    o = np.zeros((n, vh.shape[1]))
    lse = np.zeros(n)
    for r0 in range(0, n, block_rows):
        r1 = min(n, r0 + block_rows)
        kv_end = _visible(r1 - 1, n, nk, mode)
        s = scale * (qh[r0:r1] @ kh[:kv_end].T)
        m, e, l = _softmax_block(s, _mask(r0, r1, n, nk, mode)[:, :kv_end]
                                 if mode != "none" else None)
        z, r = None, 1.0
        if drop is not None:
            p8, r, seed, offset = drop
            z = dropout_keep(bh, range(r0, r1), kv_end, p8, seed, offset)
        o[r0:r1], lse[r0:r1] = _finish(e, l, m, vh[:kv_end], z, r)
    return o, lse


def online_softmax_stats(logits, block: int):
    """Running (max, sum) of one row of logits processed in chunks of `block` entries.

    The update is the one of iloveeagents.com, "Core Technical Innovations", item 2:
    m^(2) = max(m^(1), m~) and d^(2) = e^{m^(1) - m^(2)} d^(1) + e^{m~ - m^(2)} d~, where m~ and
    d~ are the chunk's own max and sum of e^{x - m~}. Returns (m, d) with d = sum_j e^{x_j - m}.
    """
    x = _f64(logits).reshape(-1)
    m = -np.inf
    d = 0.0
    for c0 in range(0, x.size, block):
        chunk = x[c0:c0 + block]
        m_chunk = chunk.max()
        d_chunk = np.exp(chunk - m_chunk).sum()
        m_new = max(m, m_chunk)
        d = (np.exp(m - m_new) * d if d != 0.0 else 0.0) + np.exp(m_chunk - m_new) * d_chunk
        m = m_new
    return m, d


def tiled_attention_forward(q, k, v, scale: float, causal: bool = False, block: int = 128):
    """The tiled algorithm with online softmax, written as the pages describe it.

    Loop order of hot.atechcom.net, "How Tiling Works": blocks of K and V outside, blocks of Q
    inside, with per-row running max m, running sum l and partial output O kept between
    blocks. Each visit applies the update of iloveeagents.com, "Core Technical Innovations"
    item 2: m_new = max(m_old, block max); the old l and the old partial O are rescaled by
    e^{m_old - m_new}; the block's exponentials are taken against m_new. Final O = O / l and
    lse = m + ln l. Used to pin that the tiled algorithm reaches the definition.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    scale = float(np.float64(scale))
    n, nk = q.shape[-2], k.shape[-2]
    o_all = np.zeros(q.shape[:-1] + (v.shape[-1],))
    lse_all = np.zeros(q.shape[:-1])
    for idx in _head_iter(q.shape):
        qh, kh, vh = q[idx], k[idx], v[idx]
        o = np.zeros((n, vh.shape[1]))
        m = np.full(n, -np.inf)
        l = np.zeros(n)
        for j0 in range(0, nk, block):  # outer: K, V blocks
            j1 = min(nk, j0 + block)
            for i0 in range(0, n, block):  # inner: Q blocks
                i1 = min(n, i0 + block)
                s = scale * (qh[i0:i1] @ kh[j0:j1].T)
                if causal:
                    mask = np.arange(j0, j1)[None, :] <= np.arange(i0, i1)[:, None]
                    s = np.where(mask, s, -np.inf)
                else:
                    mask = np.ones(s.shape, dtype=bool)
                m_old = m[i0:i1]
                m_new = np.maximum(m_old, s.max(axis=1))
                live = np.isfinite(m_new)  # rows with at least one visible key so far
                m_ref = np.where(live, m_new, 0.0)
                alpha = np.where(np.isfinite(m_old), np.exp(np.where(np.isfinite(m_old), m_old, 0.0)
                                                             - m_ref), 0.0)
                p = np.where(mask, np.exp(np.where(mask, s, 0.0) - m_ref[:, None]), 0.0)
                l[i0:i1] = alpha * l[i0:i1] + p.sum(axis=1)
                o[i0:i1] = alpha[:, None] * o[i0:i1] + p @ vh[j0:j1]
                m[i0:i1] = m_new
        o_all[idx] = o / l[:, None]
        lse_all[idx] = m + np.log(l)
    return o_all, lse_all
