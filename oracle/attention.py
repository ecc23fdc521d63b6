"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may call it. It shares no code with the CUDA library.

What it computes is the plain definition, written out with numpy in float64:

    S = scale * Q K^T          (masked to -inf where a key is not visible)
    m = rowmax(S)              (pass 1)
    P = exp(S - m) / rowsum(exp(S - m))   (pass 2)
    O = P V,   LSE = m + ln(rowsum(exp(S - m)))

The pages fix that the tiled method reaches exactly this result: the aikaboom
page "11.4d FlashAttention" lists its accuracy as exact, the same mathematical
result as standard attention (comparison table under "How FlashAttention Fixes
This"), and the zimaspace page says the tiled algorithm still produces exact
attention (section "Flash Attention Tiles the Problem Into On-Chip Working
Sets"). So the oracle is the definition, materialising the full score matrix
(the "standard attention" the aikaboom page's "The Core Problem" describes),
with no tiling, fusion or reordering.

Readings where the pages are silent (each is listed with its reason in the
design notes):
  * layout BHSD; GQA query head h reads KV head h // (Hq // Hkv), the grouping
    the sicorps page describes for GQA (last paragraph);
  * causal masking is bottom-right aligned: query i sees keys j <= i + Nk - Nq;
  * a row with no visible key has O = 0 and LSE = -inf;
  * the decode cache is packed per sequence as [Hkv][L_b][d] starting at token
    offset sum(L_0..L_{b-1}); decode attends to all L_b cached tokens;
  * a sliding window of W keys (the "windowing" scheme the zimaspace page names
    in "Reduced IO Is Not the Same as Eliminating KV Cache") keeps, for causal
    query i, only keys j with i + Nk - Nq - W < j <= i + Nk - Nq, the W most
    recent positions including its own; decode with a window reads the last W
    cached tokens. W = 0 means no window.

``online_softmax_attention`` and ``combine_partials`` are the method's own
steps (the running-statistics softmax of "Online Softmax" on the aikaboom page
and "Online Softmax Avoids Storing the Full Score Matrix" on the zimaspace
page; the merge of two running states follows from the same recurrence). They
are pinned against the two-pass definition in the tests and are not used to
produce expected values for the GPU.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "scores",
    "probabilities",
    "attention_ref",
    "decode_ref",
    "unpack_decode_cache",
    "online_softmax_attention",
    "combine_partials",
]


def _f64(x) -> np.ndarray:
    """Exact conversion of a tensor/array (bf16, fp16, fp32, ...) to float64."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def _visible(nq: int, nk: int, causal: bool, rows: np.ndarray, window: int = 0) -> np.ndarray:
    """Boolean [len(rows), nk]: key j visible to query row i (bottom-right causal,
    optionally limited to the `window` most recent keys)."""
    cols = np.arange(nk)[None, :]
    if not causal:
        if window:
            raise ValueError("a sliding window needs the causal mask")
        return np.ones((rows.size, nk), dtype=bool)
    last = rows[:, None] + (nk - nq)
    vis = cols <= last
    if window:
        vis &= cols > last - window
    return vis


def scores(q_rows: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """S = scale * Q K^T for one head: q_rows [R, d], k [Nk, d] -> [R, Nk]."""
    return scale * (q_rows @ k.T)


def probabilities(q, k, scale: float, causal: bool, window: int = 0) -> np.ndarray:
    """Softmax matrix P for single-head inputs q [Nq, d], k [Nk, d] (two-pass)."""
    q = _f64(q)
    k = _f64(k)
    nq, nk = q.shape[0], k.shape[0]
    s = scores(q, k, scale)
    s = np.where(_visible(nq, nk, causal, np.arange(nq), window), s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe)
    l = e.sum(axis=1, keepdims=True)
    with np.errstate(invalid="ignore", divide="ignore"):
        p = np.where(l > 0, e / np.where(l > 0, l, 1.0), 0.0)
    return p


def _head_ref(qh: np.ndarray, kh: np.ndarray, vh: np.ndarray, scale: float,
              causal: bool, nq: int, rows: np.ndarray, window: int = 0):
    """Two-pass attention for one (batch, head) on the given query rows."""
    nk = kh.shape[0]
    s = scores(qh, kh, scale)                       # [R, Nk]
    s = np.where(_visible(nq, nk, causal, rows, window), s, -np.inf)
    m = s.max(axis=1)                               # pass 1: row max
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m_safe[:, None])                 # pass 2: exponentials
    l = e.sum(axis=1)
    empty = l == 0.0
    p = e / np.where(empty, 1.0, l)[:, None]
    o = p @ vh
    o[empty] = 0.0
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, l)))
    return o, lse


def attention_ref(q, k, v, scale: float, causal: bool, rows=None, nq=None, window: int = 0):
    """Exact attention in fp64.

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d] (any float dtype; converted exactly).
    rows: None (every query row), a 1-D array of row indices used for every
    head, or an integer array [B, Hq, R] of per-head rows.
    nq: when given, q holds only the query rows listed in the 1-D ``rows`` (in
    that order) and nq is the full query length the causal mask refers to.
    window: 0, or the number of most recent keys a causal row sees.
    Returns (O [B, Hq, R, d], LSE [B, Hq, R]) in float64; R = Nq when rows is None.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, Hq, Nq, d = q.shape
    Bk, Hkv, Nk, dk = k.shape
    if Bk != B or dk != d or v.shape != k.shape:
        raise ValueError("shape mismatch")
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    if nq is not None:
        rows_arr = np.asarray(rows, dtype=np.int64)
        if rows_arr.ndim != 1 or rows_arr.size != Nq:
            raise ValueError("with nq, rows must list the rows q holds")
        out = np.zeros((B, Hq, Nq, d))
        lse = np.zeros((B, Hq, Nq))
        for b in range(B):
            for h in range(Hq):
                g = h // group
                out[b, h], lse[b, h] = _head_ref(q[b, h], k[b, g], v[b, g], scale, causal,
                                                 nq, rows_arr, window)
        return out, lse
    if rows is None:
        rows_arr = np.broadcast_to(np.arange(Nq), (B, Hq, Nq))
    else:
        rows_arr = np.asarray(rows, dtype=np.int64)
        if rows_arr.ndim == 1:
            rows_arr = np.broadcast_to(rows_arr, (B, Hq, rows_arr.size))
    R = rows_arr.shape[-1]
    out = np.zeros((B, Hq, R, d))
    lse = np.zeros((B, Hq, R))
    for b in range(B):
        for h in range(Hq):
            g = h // group
            r = rows_arr[b, h]
            out[b, h], lse[b, h] = _head_ref(q[b, h, r], k[b, g], v[b, g], scale,
                                             causal, Nq, r, window)
    return out, lse


def _sequence_ranges(seqlens, Hkv: int, d: int):
    """(start, L) element ranges of each sequence's block in a packed cache."""
    lens = [max(0, int(x)) for x in _f64(seqlens).reshape(-1)]
    out = []
    off = 0
    for L in lens:
        out.append((off, L))
        off += L * Hkv * d
    return out


def _flat(cache):
    try:
        import torch

        if isinstance(cache, torch.Tensor):
            return cache.detach().reshape(-1)
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(cache).reshape(-1)


def unpack_decode_cache(cache, seqlens, Hkv: int, d: int):
    """Split a packed decode cache into per-sequence [Hkv, L_b, d] fp64 arrays."""
    flat = _flat(cache)
    return [_f64(flat[o:o + L * Hkv * d]).reshape(Hkv, L, d)
            for o, L in _sequence_ranges(seqlens, Hkv, d)]


def decode_ref(q, kcache, vcache, seqlens, scale: float, Hkv: int, window: int = 0):
    """One-token decode over a ragged packed cache, in fp64.

    q: [B, Hq, d]; caches packed as described in the module docstring;
    seqlens: [B] ints. Returns (O [B, Hq, d], LSE [B, Hq]).
    Each new token reads the whole cache of its sequence (the "token generation"
    case on the first page: linear in the number of cached entries).
    Sequences are converted to fp64 one at a time, so large caches fit in memory.
    window: 0, or the number of most recent cached tokens the new token reads.
    """
    q = _f64(q)
    B, Hq, d = q.shape
    kf = _flat(kcache)
    vf = _flat(vcache)
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    for b, (o0, L) in enumerate(_sequence_ranges(seqlens, Hkv, d)):
        if L == 0:
            lse[b] = -np.inf
            continue
        kb = _f64(kf[o0:o0 + L * Hkv * d]).reshape(1, Hkv, L, d)
        vb = _f64(vf[o0:o0 + L * Hkv * d]).reshape(1, Hkv, L, d)
        if window:
            kb, vb = kb[:, :, max(0, L - window):], vb[:, :, max(0, L - window):]
        o, l = attention_ref(q[b][None, :, None, :], kb, vb, scale, causal=False)
        out[b] = o[0, :, 0]
        lse[b] = l[0, :, 0]
    return out, lse


def online_softmax_attention(q, k, v, scale: float, causal: bool, tile: int, window: int = 0):
    """The tiled running-softmax recurrence, for single-head q [Nq,d], k/v [Nk,d].

    Key tiles of width ``tile`` are consumed left to right; per query row a
    running max m, running sum l and unnormalised output acc are kept. When a
    tile raises the max, the old l and acc are rescaled by exp(m_old - m_new)
    before the tile's contribution is added. O = acc / l and LSE = m + ln l at
    the end.
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    nq, nk = q.shape[0], k.shape[0]
    rows = np.arange(nq)
    m = np.full(nq, -np.inf)
    l = np.zeros(nq)
    acc = np.zeros((nq, v.shape[1]))
    for j0 in range(0, nk, tile):
        j1 = min(nk, j0 + tile)
        s = scale * (q @ k[j0:j1].T)
        vis = _visible(nq, nk, causal, rows, window)[:, j0:j1]
        s = np.where(vis, s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        m_safe = np.where(np.isfinite(m_new), m_new, 0.0)
        alpha = np.where(np.isfinite(m), np.exp(m - m_safe), 0.0)
        p = np.exp(s - m_safe[:, None])
        l = alpha * l + p.sum(axis=1)
        acc = alpha[:, None] * acc + p @ v[j0:j1]
        m = m_new
    empty = l == 0.0
    o = acc / np.where(empty, 1.0, l)[:, None]
    o[empty] = 0.0
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, np.where(np.isfinite(m), m, 0.0)
                       + np.log(np.where(empty, 1.0, l)))
    return o, lse


def combine_partials(o_parts, lse_parts):
    """Merge normalised partial results computed over disjoint key subsets.

    o_parts: [S, ..., d], lse_parts: [S, ...]. A part over no keys has
    LSE = -inf and contributes nothing. Returns (O, LSE) over the union.
    """
    o_parts = _f64(o_parts)
    lse_parts = _f64(lse_parts)
    mx = lse_parts.max(axis=0)
    mx_safe = np.where(np.isfinite(mx), mx, 0.0)
    w = np.exp(lse_parts - mx_safe[None])
    tot = w.sum(axis=0)
    empty = tot == 0.0
    with np.errstate(invalid="ignore", divide="ignore"):
        o = (w[..., None] * o_parts).sum(axis=0) / np.where(empty, 1.0, tot)[..., None]
        lse = np.where(empty, -np.inf, mx_safe + np.log(np.where(empty, 1.0, tot)))
    o[empty] = 0.0
    return o, lse
