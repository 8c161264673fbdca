"""fp64 CPU oracle for the fused attention forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU
baseline and ``--impl reference`` arm) may import this module. The library
never calls it; the two share no code.

What it computes is the plain definition, two passes per query row, no
tiling, no online recurrence:

  S      = scale * Q K^T                       (CANN "flash_attn", 计算公式;
                                                MindSpore "sparse_flash_attention",
                                                formula; ``scale_value``)
  M      = max_{j visible} S_j
  m      = max(sink, M)     if a sink is given (CANN "flash_attn", 计算公式,
                                                the sink variant)
  O      = sum_j e^{S_j - m} V_j / (sum_j e^{S_j - m} + e^{sink - m})
  LSE    = M + ln sum_j e^{S_j - M}            (CANN "flash_attn", 计算公式,
                                                the softmax_lse definition, and
                                                the ``softmax_lse`` output note)

Readings taken where the pages are silent or ambiguous:

* LSE excludes the sink: the softmax_lse formula is written over S alone.
* The causal mask is bottom-right aligned (MindSpore "sparse_flash_attention",
  ``sparse_mode=3`` "rightDownCausal"): with delta = L_k - L_q, key j is
  visible to query i iff j <= i + delta.
* A sliding window (left, right) keeps i+delta-left <= j <= i+delta+right,
  bounds inclusive, -1 = unbounded (MindSpore Lite "flash_attention",
  ``window_size=(-1, -1)``; MindSpore "sparse_flash_attention",
  ``pre_tokens`` / ``next_tokens``). causal is the same as right = 0.
* GQA: query head h reads KV head floor(h / (H_q / H_kv)) (contiguous groups).
* A row that sees no key gives O = 0 and LSE = -inf, with or without a sink.
* FP8 inputs are decoded exactly and multiplied by their fp32 descale of
  shape (B, H_kv) (MATE "Attention", FMHA dtype notes).
* MLA: the 576-wide row is [512 latent | 64 rope] and V is its first 512
  entries (MindSpore "sparse_flash_attention", ``attention_mode=2``; MATE
  "Attention", MLA example with ``head_dim_v=512``).
* Sparse: the visible set is the listed logical positions that are
  >= 0 and < cache_seqlens[b]; others are skipped.
* Combine (MATE "Attention", FMHA notes on ``flash_attn_combine``; no formula
  is printed): LSE = ln sum_s e^{LSE_s}, O = sum_s e^{LSE_s - LSE} O_s for
  sink-free partials; the sink is applied once afterwards as
  O <- O / (1 + e^{sink - LSE}).

Every function here is pinned by ``tests/test_oracle_pins.py`` against
library routines (torch's fp64 scaled_dot_product_attention, logsumexp,
tril/triu, float8 conversions), closed forms and invariants.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

NEG_INF = -math.inf


# ---------------------------------------------------------------------------
# Number formats, decoded from their definitions
# ---------------------------------------------------------------------------

def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 is the upper half of an IEEE-754 binary32: widen the 16 bits
    into the high half of a 32-bit word and read it as binary32."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):  # NaN codes widen to NaN
        return b.view(np.float32).astype(np.float64)


def decode_fp16(bits: np.ndarray) -> np.ndarray:
    """IEEE-754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits."""
    b = np.asarray(bits).astype(np.uint16).astype(np.int64)
    sign = np.where(b >> 15, -1.0, 1.0)
    e = (b >> 10) & 0x1F
    f = (b & 0x3FF).astype(np.float64)
    normal = sign * np.ldexp(1.0 + f / 1024.0, (e - 15).astype(np.int64))
    sub = sign * np.ldexp(f / 1024.0, -14)
    special = np.where(f == 0, sign * np.inf, np.nan)
    return np.where(e == 0, sub, np.where(e == 31, special, normal))


def decode_e4m3(bits: np.ndarray) -> np.ndarray:
    """OCP 8-bit E4M3 ("fn"): 1 sign, 4 exponent bits (bias 7), 3 mantissa
    bits; no infinities; S.1111.111 is NaN; largest finite value 448;
    exponent field 0 encodes subnormals m/8 * 2^-6."""
    b = np.asarray(bits).astype(np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, -6)
    val = np.where(e == 0, sub, normal)
    return np.where((e == 15) & ((b & 0x7) == 7), np.nan, val)


def decode_e5m2(bits: np.ndarray) -> np.ndarray:
    """OCP 8-bit E5M2: 1 sign, 5 exponent bits (bias 15), 2 mantissa bits,
    IEEE-style infinities and NaNs at exponent 31."""
    b = np.asarray(bits).astype(np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 2) & 0x1F
    m = (b & 0x3).astype(np.float64)
    normal = sign * np.ldexp(1.0 + m / 4.0, (e - 15).astype(np.int64))
    sub = sign * np.ldexp(m / 4.0, -14)
    special = np.where(m == 0, sign * np.inf, np.nan)
    return np.where(e == 0, sub, np.where(e == 31, special, normal))


_DECODERS = {"bf16": decode_bf16, "fp16": decode_fp16, "e4m3": decode_e4m3, "e5m2": decode_e5m2}


def decode(bits: np.ndarray, fmt: str) -> np.ndarray:
    """Raw storage bits (uint16 for bf16/fp16, uint8 for FP8) -> float64."""
    return _DECODERS[fmt](bits)


# ---------------------------------------------------------------------------
# Visibility (masks)
# ---------------------------------------------------------------------------

def visible_range(i: int, len_q: int, len_k: int, causal: bool, window_left: int,
                  window_right: int) -> Tuple[int, int]:
    """Inclusive [lo, hi] of keys visible to query row i (empty if lo > hi).

    delta = len_k - len_q aligns the last query with the last key (bottom
    right). causal caps the right edge at i + delta; a window bound of -1 is
    unbounded."""
    delta = len_k - len_q
    lo = 0
    hi = len_k - 1
    if causal:
        hi = min(hi, i + delta)
    if window_right >= 0:
        hi = min(hi, i + delta + window_right)
    if window_left >= 0:
        lo = max(lo, i + delta - window_left)
    return lo, hi


def visible_mask(len_q: int, len_k: int, causal: bool = False, window_left: int = -1,
                 window_right: int = -1) -> np.ndarray:
    """Boolean (len_q, len_k) matrix of visible (query, key) pairs."""
    mask = np.zeros((len_q, len_k), dtype=bool)
    for i in range(len_q):
        lo, hi = visible_range(i, len_q, len_k, causal, window_left, window_right)
        if lo <= hi:
            mask[i, lo:hi + 1] = True
    return mask


# ---------------------------------------------------------------------------
# The definition, per query row
# ---------------------------------------------------------------------------

def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                   vis: np.ndarray, sink=None, bias=None) -> Tuple[np.ndarray, np.ndarray]:
    """Attention for a block of query rows against one key/value set.

    q (R, D_qk), k (L, D_qk), v (L, D_v), vis (R, L) bool; sink is None, a
    scalar, or an array (R,) of per-row sink logits; bias is None or an
    additive score mask (R, L) added after the scale (Mojo
    "flash_attention_split_kv": input_mask_fn loads additive mask values), a
    key with bias -inf being left out like an invisible one. Returns O (R, D_v)
    and the keys-only LSE (R,), all float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    R = q.shape[0]
    out = np.zeros((R, v.shape[1]), dtype=np.float64)
    lse = np.full((R,), NEG_INF, dtype=np.float64)
    if R == 0 or k.shape[0] == 0:
        return out, lse
    s = scale * (q @ k.T)
    if bias is not None:
        s = s + np.asarray(bias, dtype=np.float64)
        vis = np.logical_and(vis, s > NEG_INF)
    sinks = None
    if sink is not None:
        sinks = np.broadcast_to(np.asarray(sink, dtype=np.float64), (R,))
    for r in range(R):
        J = np.nonzero(vis[r])[0]
        if J.size == 0:
            continue
        sj = s[r, J]
        M = sj.max()
        m = M if sinks is None else max(M, sinks[r])
        e = np.exp(sj - m)
        Z = e.sum()
        if sinks is not None:
            Z += math.exp(sinks[r] - m)
        out[r] = (e @ v[J]) / Z
        lse[r] = M + math.log(np.exp(sj - M).sum())
    return out, lse


def _kv_head(h: int, num_heads_q: int, num_heads_kv: int) -> int:
    return h // (num_heads_q // num_heads_kv)


# ---------------------------------------------------------------------------
# Dense / varlen prefill
# ---------------------------------------------------------------------------

def attention_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale, causal=False,
                     window=(-1, -1), sink=None, q_descale=None, k_descale=None,
                     v_descale=None, rows: Optional[Iterable[Tuple[int, int, int]]] = None,
                     mask=None):
    """Packed (TND) layout: q (T_q, H_q, D), k/v (T_k, H_kv, D) as float64,
    cu_seqlens int arrays (B+1). Returns out (T_q, H_q, D_v) and lse (H_q, T_q).

    ``rows`` optionally restricts the work to (b, i, h) triples; the other
    entries of out/lse are left at 0 / -inf. ``mask`` is None or an additive
    score mask indexed [b, h, i, j] by sequence, query head, and the row and
    key positions within the sequence (broadcastable numpy array)."""
    cu_q = [int(x) for x in cu_seqlens_q]
    cu_k = [int(x) for x in cu_seqlens_k]
    B = len(cu_q) - 1
    return _attention_segments(q, k, v, cu_q[:B], [cu_q[b + 1] - cu_q[b] for b in range(B)],
                               cu_k[:B], [cu_k[b + 1] - cu_k[b] for b in range(B)], scale,
                               causal, window, sink, q_descale, k_descale, v_descale, rows,
                               mask)


def _attention_segments(q, k, v, start_q, len_q, start_k, len_k, scale, causal, window, sink,
                        q_descale, k_descale, v_descale, rows, mask):
    """Sequence b: query rows start_q[b] .. + len_q[b] of q (T_q, H_q, D), keys
    start_k[b] .. + len_k[b] of k/v (T_k, H_kv, D)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B = len(start_q)
    Hq, Hkv = q.shape[1], k.shape[1]
    if mask is not None:
        mask = np.asarray(mask, np.float64)
    out = np.zeros((q.shape[0], Hq, v.shape[2]), np.float64)
    lse = np.full((Hq, q.shape[0]), NEG_INF, np.float64)
    want = None
    if rows is not None:
        want = {}
        for (b, i, h) in rows:
            want.setdefault((b, h), []).append(i)
    for b in range(B):
        Lq, Lk = int(len_q[b]), int(len_k[b])
        q0, k0 = int(start_q[b]), int(start_k[b])
        for h in range(Hq):
            if want is not None and (b, h) not in want:
                continue
            g = _kv_head(h, Hq, Hkv)
            ii = np.arange(Lq) if want is None else np.array(sorted(set(want[(b, h)])))
            qs = q[q0 + ii, h, :]
            ks = k[k0:k0 + Lk, g, :]
            vs = v[k0:k0 + Lk, g, :]
            if q_descale is not None:
                qs = qs * float(q_descale[b][g])
                ks = ks * float(k_descale[b][g])
                vs = vs * float(v_descale[b][g])
            vis = np.zeros((len(ii), Lk), dtype=bool)
            for r, i in enumerate(ii):
                lo, hi = visible_range(int(i), Lq, Lk, causal, window[0], window[1])
                if lo <= hi:
                    vis[r, lo:hi + 1] = True
            bias = None
            if mask is not None:
                mb = mask[b if mask.shape[0] > 1 else 0, h if mask.shape[1] > 1 else 0]
                rows_b = mb[ii] if mb.shape[0] > 1 else np.repeat(mb[:1], len(ii), 0)
                bias = rows_b[:, :Lk] if rows_b.shape[1] > 1 else np.repeat(rows_b, Lk, 1)
            o, l = attention_rows(qs, ks, vs, scale, vis,
                                  None if sink is None else float(sink[h]), bias)
            out[q0 + ii, h, :] = o
            lse[h, q0 + ii] = l
    return out, lse


def attention_padded(q, k, v, scale, causal=False, window=(-1, -1), sink=None,
                     q_descale=None, k_descale=None, v_descale=None, rows=None, mask=None,
                     seqused_q=None, seqused_k=None):
    """Padded (BSHD) layout: q (B, S_q, H_q, D), k/v (B, S_k, H_kv, D).
    Returns out (B, S_q, H_q, D_v) and lse (B, H_q, S_q).

    seqused_q / seqused_k (CANN "flash_attn": seqused_q, seqused_kv) are None
    or per-sequence counts of the rows / keys in use (<= S_q / S_k): sequence b
    is then its first seqused_q[b] rows against its first seqused_k[b] keys
    (bottom-right causal alignment uses those lengths); rows past it stay
    0 / -inf. ``mask`` as in attention_varlen."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Sq, Hq, _ = q.shape
    Sk = k.shape[1]
    len_q = [Sq] * B if seqused_q is None else [int(x) for x in seqused_q]
    len_k = [Sk] * B if seqused_k is None else [int(x) for x in seqused_k]
    o, l = _attention_segments(q.reshape(B * Sq, Hq, -1), k.reshape(B * Sk, k.shape[2], -1),
                               v.reshape(B * Sk, v.shape[2], -1), [b * Sq for b in range(B)],
                               len_q, [b * Sk for b in range(B)], len_k, scale, causal, window,
                               sink, q_descale, k_descale, v_descale, rows, mask)
    return o.reshape(B, Sq, Hq, -1), l.reshape(Hq, B, Sq).transpose(1, 0, 2)


# ---------------------------------------------------------------------------
# Paged KV cache decode
# ---------------------------------------------------------------------------

def gather_pages(cache: np.ndarray, block_table_row: Sequence[int], length: int) -> np.ndarray:
    """Logical rows 0..length-1 of one sequence: row t lives in physical page
    block_table_row[t // page_size] at offset t % page_size."""
    page = cache.shape[1]
    idx = np.arange(length)
    blocks = np.asarray(block_table_row, dtype=np.int64)[idx // page]
    return cache[blocks, idx % page]


def attention_paged(q, k_cache, v_cache, block_table, cache_seqlens, scale, causal=False,
                    window=(-1, -1), sink=None, rows=None, q_descale=None, k_descale=None,
                    v_descale=None, k_new=None, v_new=None):
    """q (B, s_q, H_q, D); caches (num_blocks, page_size, H_kv, D) float64;
    block_table (B, max_pages); cache_seqlens (B,). The s_q query rows are the
    last s_q positions of the sequence (bottom-right alignment).
    FP8 (MATE "Attention", FMHA FP8 paragraph, which covers the KV-cache call
    too): q, k and v of sequence b and KV head g are multiplied by their
    descale [b, g] (all three given or none).
    Appended keys (Mojo "flash_attention_split_kv": the previous keys come
    from the cache and the current ones from separate k and v tensors, read
    as one concatenated sequence): k_new, v_new (B, s_new, H_kv, D) follow
    the cache_seqlens[b] cached rows of sequence b, so the sequence has
    cache_seqlens[b] + s_new keys; the cache itself is not changed.
    Returns out (B, s_q, H_q, D_v) and lse (B, H_q, s_q)."""
    q = np.asarray(q, np.float64)
    B, Sq, Hq, _ = q.shape
    Hkv = k_cache.shape[2]
    out = np.zeros((B, Sq, Hq, v_cache.shape[3]), np.float64)
    lse = np.full((B, Hq, Sq), NEG_INF, np.float64)
    want = None
    if rows is not None:
        want = {}
        for (b, i, h) in rows:
            want.setdefault(b, set()).add((i, h))
    for b in range(B):
        if want is not None and b not in want:
            continue
        L = int(cache_seqlens[b])
        ks = gather_pages(k_cache, block_table[b], L)
        vs = gather_pages(v_cache, block_table[b], L)
        if k_new is not None:
            ks = np.concatenate([ks, np.asarray(k_new[b], np.float64)])
            vs = np.concatenate([vs, np.asarray(v_new[b], np.float64)])
            L = ks.shape[0]
        for h in range(Hq):
            ii = [i for i in range(Sq) if want is None or (i, h) in want[b]]
            if not ii:
                continue
            g = _kv_head(h, Hq, Hkv)
            vis = np.zeros((len(ii), L), dtype=bool)
            for r, i in enumerate(ii):
                lo, hi = visible_range(i, Sq, L, causal, window[0], window[1])
                if lo <= hi:
                    vis[r, lo:hi + 1] = True
            qh, kh, vh = q[b, ii, h, :], ks[:, g, :], vs[:, g, :]
            if q_descale is not None:
                qh = qh * float(q_descale[b][g])
                kh = kh * float(k_descale[b][g])
                vh = vh * float(v_descale[b][g])
            o, l = attention_rows(qh, kh, vh, scale, vis,
                                  None if sink is None else float(sink[h]))
            out[b, ii, h, :] = o
            lse[b, h, ii] = l
    return out, lse


# ---------------------------------------------------------------------------
# Split-KV combine
# ---------------------------------------------------------------------------

def combine(out_partial: np.ndarray, lse_partial: np.ndarray, sink=None):
    """Merge sink-free partial results over disjoint key splits.

    out_partial (n_splits, ..., D_v), lse_partial (n_splits, ...). A split with
    LSE = -inf carries weight 0; if every split is -inf the result is O = 0,
    LSE = -inf. ``sink`` (broadcastable to lse_partial[0]) is applied once
    after the merge. Returns (out, lse)."""
    O = np.asarray(out_partial, np.float64)
    Ls = np.asarray(lse_partial, np.float64)
    Mx = Ls.max(axis=0)
    finite = np.isfinite(Mx)
    Msafe = np.where(finite, Mx, 0.0)
    w = np.where(np.isfinite(Ls), np.exp(Ls - Msafe[None]), 0.0)
    tot = w.sum(axis=0)
    lse = np.where(finite, Msafe + np.log(np.where(finite, tot, 1.0)), NEG_INF)
    wn = np.where(finite[None], w / np.where(finite, tot, 1.0)[None], 0.0)
    out = (wn[..., None] * O).sum(axis=0)
    if sink is not None:
        sk = np.broadcast_to(np.asarray(sink, np.float64), lse.shape)
        factor = np.where(finite, 1.0 / (1.0 + np.exp(sk - np.where(finite, lse, 0.0))), 0.0)
        out = out * factor[..., None]
    return out, lse


# ---------------------------------------------------------------------------
# MLA-absorbed decode (dense and top-k sparse)
# ---------------------------------------------------------------------------

def mla_paged(q, kv_cache, block_table, cache_seqlens, head_dim_v, scale, causal=False,
              rows=None, q_descale=None, k_descale=None, v_descale=None):
    """q (B, s_q, H_q, 576); kv_cache (num_blocks, page_size, H_kv, 576). K is
    the whole row, V its first head_dim_v entries. With H_kv > 1 (MATE
    "Attention", MLA example: a cache of 2 KV heads) query head h reads KV
    head floor(h / (H_q / H_kv)), as in GQA.
    FP8 (MATE "Attention", FMHA FP8 paragraph, applied to the MLA cache): q,
    K and V of sequence b and KV head g are multiplied by q_descale[b, g],
    k_descale[b, g] and v_descale[b, g] (all three given or none); K and V are
    the same cached row, each with its own descale."""
    kv = np.asarray(kv_cache, np.float64)
    return attention_paged(q, kv, kv[..., :head_dim_v], block_table, cache_seqlens, scale,
                           causal, (-1, -1), None, rows, q_descale, k_descale, v_descale)


def mla_sparse(q, kv_cache, block_table, cache_seqlens, indices, head_dim_v, scale,
               rows=None, block_size=1, causal=False, q_descale=None, k_descale=None,
               v_descale=None):
    """q (B, s_q, H_q, 576); kv_cache (num_blocks, page_size, H_kv, 576);
    indices (B, s_q, H_kv, topk) logical positions. Query token (b, i) of
    head h attends, in KV head g = floor(h / (H_q / H_kv)), to the positions
    listed in indices[b, i, g] with 0 <= p < L_b (each listed occurrence
    counts once); the others are skipped.
    block_size > 1 (MindSpore "sparse_flash_attention": sparse_block_size, a
    power of two up to 128): each index k >= 0 lists the block of positions
    k * block_size .. k * block_size + block_size - 1 (reading: the index
    counts blocks); negative indices are skipped.
    causal (sparse_mode=3, "rightDownCausal"): a listed position p is also
    required to satisfy p <= i + L_b - s_q (bottom-right alignment).
    q_descale, k_descale, v_descale (B, H_kv): FP8 descales as in mla_paged.
    Returns out (B, s_q, H_q, D_v) and lse (B, H_q, s_q)."""
    q = np.asarray(q, np.float64)
    kv = np.asarray(kv_cache, np.float64)
    B, Sq, Hq, _ = q.shape
    page, Hkv = kv.shape[1], kv.shape[2]
    out = np.zeros((B, Sq, Hq, head_dim_v), np.float64)
    lse = np.full((B, Hq, Sq), NEG_INF, np.float64)
    want = None
    if rows is not None:
        want = {}
        for (b, i, h) in rows:
            want.setdefault((b, i), []).append(h)
    for b in range(B):
        L = int(cache_seqlens[b])
        for i in range(Sq):
            if want is not None and (b, i) not in want:
                continue
            hs_all = list(range(Hq)) if want is None else sorted(set(want[(b, i)]))
            for g in range(Hkv):
                hs = [h for h in hs_all if _kv_head(h, Hq, Hkv) == g]
                if not hs:
                    continue
                idx = np.asarray(indices[b, i, g], dtype=np.int64)
                if block_size > 1:
                    idx = idx[idx >= 0]
                    idx = (idx[:, None] * block_size + np.arange(block_size)[None, :]).reshape(-1)
                idx = idx[(idx >= 0) & (idx < L)]
                if causal:
                    idx = idx[idx <= i + L - Sq]
                rows_kv = kv[np.asarray(block_table[b], np.int64)[idx // page], idx % page, g, :]
                qs, ks, vs = q[b, i, hs, :], rows_kv, rows_kv[:, :head_dim_v]
                if q_descale is not None:
                    dq, dk, dv = (float(d[b][g]) for d in (q_descale, k_descale, v_descale))
                    qs, ks, vs = qs * dq, ks * dk, vs * dv
                vis = np.ones((len(hs), idx.size), dtype=bool)
                o, l = attention_rows(qs, ks, vs, scale, vis)
                out[b, i, hs, :] = o
                lse[b, hs, i] = l
    return out, lse


def mla_sparse_tnd(q, kv_cache, block_table, cache_seqlens, cu_seqlens_q, indices, head_dim_v,
                   scale, block_size=1, causal=False, q_descale=None, k_descale=None,
                   v_descale=None):
    """The sparse MLA attention with packed (TND) queries (MindSpore
    "sparse_flash_attention", layout_query="TND" with a paged cache): q
    (T, H_q, 576) holds the query tokens of the B sequences back to back,
    sequence b owning tokens cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 (the
    prefix-sum form of actual_seq_lengths_query); indices (T, H_kv, topk).
    Each sequence is the BSND problem of its own tokens (token i of sequence
    b is its i-th query row; causal aligns its last token with the cache's
    last key). q/k/v_descale (B, H_kv): FP8 descales of each sequence, as in
    mla_paged. Returns out (T, H_q, D_v) and lse (H_q, T)."""
    q = np.asarray(q, np.float64)
    T, Hq, _ = q.shape
    out = np.zeros((T, Hq, head_dim_v), np.float64)
    lse = np.full((Hq, T), NEG_INF, np.float64)
    cu = [int(x) for x in cu_seqlens_q]
    for b in range(len(cu) - 1):
        t0, t1 = cu[b], cu[b + 1]
        if t1 <= t0:
            continue
        desc = {}
        if q_descale is not None:
            desc = dict(q_descale=np.asarray(q_descale)[b:b + 1],
                        k_descale=np.asarray(k_descale)[b:b + 1],
                        v_descale=np.asarray(v_descale)[b:b + 1])
        o, l = mla_sparse(q[None, t0:t1], kv_cache, np.asarray(block_table)[b:b + 1],
                          [int(cache_seqlens[b])], np.asarray(indices)[None, t0:t1],
                          head_dim_v, scale, block_size=block_size, causal=causal, **desc)
        out[t0:t1] = o[0]
        lse[:, t0:t1] = l[0]
    return out, lse
