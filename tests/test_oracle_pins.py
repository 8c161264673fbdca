"""Pins for the fp64 oracle, checked on the CPU.

The oracle is compared with things other than itself: torch's own fp64
routines (scaled_dot_product_attention, logsumexp, tril/triu, the float8 /
bfloat16 / float16 conversions), closed forms and invariants that follow from
the pages' formulas, and brute force on tiny inputs. Each test names what it
guards against.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import attention as orc

RNG = np.random.default_rng(1234)


def _sdpa(q, k, v, scale, mask=None):
    """torch fp64 SDPA on (H, L, D) arrays; mask (Lq, Lk) bool, True = visible."""
    tq = torch.as_tensor(q, dtype=torch.float64)[None]
    tk = torch.as_tensor(k, dtype=torch.float64)[None]
    tv = torch.as_tensor(v, dtype=torch.float64)[None]
    m = None if mask is None else torch.as_tensor(mask)[None, None]
    gqa = tq.shape[1] != tk.shape[1]
    return F.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=scale,
                                          enable_gqa=gqa)[0].numpy()


# --------------------------------------------------------------------------
# number formats: every code against torch's conversion
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fmt,tdt,nbits", [
    ("bf16", torch.bfloat16, 16), ("fp16", torch.float16, 16),
    ("e4m3", torch.float8_e4m3fn, 8), ("e5m2", torch.float8_e5m2, 8)])
def test_decode_all_codes_match_torch(fmt, tdt, nbits):
    if nbits == 16:
        codes = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
        ref = torch.from_numpy(codes.view(np.int16).copy()).view(tdt).to(torch.float64).numpy()
    else:
        codes = np.arange(256, dtype=np.uint8)
        ref = torch.from_numpy(codes.copy()).view(tdt).to(torch.float64).numpy()
    got = oracle.decode(codes, fmt)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_e4m3_format_landmarks():
    d = orc.decode_e4m3(np.array([0x7E, 0x08, 0x01, 0x38, 0xB8, 0x7F, 0xFF], np.uint8))
    assert d[0] == 448.0                      # largest finite
    assert d[1] == 2.0 ** -6                  # smallest normal
    assert d[2] == 2.0 ** -9                  # smallest subnormal
    assert d[3] == 1.0 and d[4] == -1.0
    assert np.isnan(d[5]) and np.isnan(d[6])  # S.1111.111


# --------------------------------------------------------------------------
# masks
# --------------------------------------------------------------------------

@pytest.mark.parametrize("lq,lk", [(5, 5), (3, 7), (7, 3), (1, 9), (6, 1)])
def test_causal_mask_is_bottom_right_tril(lq, lk):
    ref = torch.ones(lq, lk, dtype=torch.bool).tril(diagonal=lk - lq).numpy()
    assert np.array_equal(oracle.visible_mask(lq, lk, causal=True), ref)


@pytest.mark.parametrize("lq,lk,left,right", [(9, 9, 2, 0), (9, 9, 3, 1), (4, 10, 2, -1),
                                              (10, 4, -1, 2), (6, 6, 0, 0)])
def test_window_mask_is_band(lq, lk, left, right):
    d = lk - lq
    band = torch.ones(lq, lk, dtype=torch.bool)
    if right >= 0:
        band = band.tril(diagonal=d + right)
    if left >= 0:
        band = band.triu(diagonal=d - left)
    assert np.array_equal(oracle.visible_mask(lq, lk, False, left, right), band.numpy())
    # inclusive bounds: a square window (left, 0) keeps min(i, left) + 1 keys
    if lq == lk and right == 0:
        counts = oracle.visible_mask(lq, lk, False, left, right).sum(1)
        assert list(counts) == [min(i, left) + 1 for i in range(lq)]


def test_mask_special_cases():
    assert oracle.visible_mask(5, 8).all()                                     # (-1,-1): full
    assert oracle.visible_mask(1, 8, causal=True).all()                        # decode row
    assert np.array_equal(oracle.visible_mask(6, 6, True, 100, -1),
                          oracle.visible_mask(6, 6, True))                     # huge window
    assert np.array_equal(oracle.visible_mask(6, 6, False, -1, 0),
                          oracle.visible_mask(6, 6, True))                     # causal == right 0


# --------------------------------------------------------------------------
# the per-row definition
# --------------------------------------------------------------------------

def test_rows_match_torch_sdpa_and_logsumexp():
    R, L, D, Dv = 6, 11, 8, 5
    q, k, v = RNG.normal(size=(R, D)), RNG.normal(size=(L, D)), RNG.normal(size=(L, Dv))
    vis = RNG.random((R, L)) < 0.6
    vis[:, 0] = True
    scale = 0.37
    o, lse = oracle.attention_rows(q, k, v, scale, vis)
    ref = _sdpa(q[None], k[None], v[None], scale, vis)[0]
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)
    s = torch.as_tensor(scale * q @ k.T).masked_fill(~torch.as_tensor(vis), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=1).numpy(), rtol=1e-12, atol=1e-12)


def test_rows_single_key_and_identical_values():
    q, k = RNG.normal(size=(3, 4)), RNG.normal(size=(5, 4))
    v = RNG.normal(size=(5, 3))
    vis = np.zeros((3, 5), bool)
    vis[0, 2] = vis[1, 4] = vis[2, 0] = True
    o, lse = oracle.attention_rows(q, k, v, 0.5, vis)
    for r, j in enumerate([2, 4, 0]):
        np.testing.assert_allclose(o[r], v[j], rtol=0, atol=1e-15)
        assert abs(lse[r] - 0.5 * q[r] @ k[j]) < 1e-14
    vv = np.tile(RNG.normal(size=(1, 3)), (5, 1))
    o2, _ = oracle.attention_rows(q, k, vv, 0.5, np.ones((3, 5), bool))
    np.testing.assert_allclose(o2, np.tile(vv[:1], (3, 1)), rtol=1e-13)


def test_rows_shift_invariance_and_lse_identity():
    q, k, v = RNG.normal(size=(4, 6)), RNG.normal(size=(9, 6)), RNG.normal(size=(9, 2))
    vis = np.ones((4, 9), bool)
    o, lse = oracle.attention_rows(q, k, v, 1.0, vis)
    # adding c to every score (append a constant feature) moves LSE by c only
    c = 3.25
    q2 = np.hstack([q, np.ones((4, 1))])
    k2 = np.hstack([k, np.full((9, 1), c)])
    o2, lse2 = oracle.attention_rows(q2, k2, v, 1.0, vis)
    np.testing.assert_allclose(o2, o, rtol=1e-12)
    np.testing.assert_allclose(lse2, lse + c, rtol=1e-12)
    # sum_j e^{s_j - LSE} = 1 and O = sum_j e^{s_j - LSE} v_j
    w = np.exp(q @ k.T - lse[:, None])
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=1e-12)
    np.testing.assert_allclose(w @ v, o, rtol=1e-12)


def test_sink_closed_forms():
    q, k, v = RNG.normal(size=(5, 4)), RNG.normal(size=(7, 4)), RNG.normal(size=(7, 3))
    vis = np.ones((5, 7), bool)
    vis[1, 3:] = False
    sink = RNG.normal(size=5) * 2
    o0, lse0 = oracle.attention_rows(q, k, v, 0.8, vis)
    o1, lse1 = oracle.attention_rows(q, k, v, 0.8, vis, sink)
    sig = 1.0 / (1.0 + np.exp(sink - lse0))          # O_sink = O * sigma(LSE - sink)
    np.testing.assert_allclose(o1, o0 * sig[:, None], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(lse1, lse0, rtol=0, atol=0)  # keys-only LSE
    o2, _ = oracle.attention_rows(q, k, v, 0.8, vis, np.full(5, -1e4))
    np.testing.assert_allclose(o2, o0, rtol=1e-14)    # sink -> -inf: no sink
    # one key whose score equals the sink: half the weight goes to the sink
    s = 0.8 * q[0] @ k[0]
    o3, _ = oracle.attention_rows(q[:1], k[:1], v[:1], 0.8, np.ones((1, 1), bool), s)
    np.testing.assert_allclose(o3[0], v[0] / 2, rtol=1e-14)


def test_rows_without_visible_keys():
    o, lse = oracle.attention_rows(np.ones((2, 3)), np.ones((4, 3)), np.ones((4, 2)), 1.0,
                                   np.zeros((2, 4), bool), 0.5)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


# --------------------------------------------------------------------------
# layouts: varlen, padded, GQA, FP8 descale
# --------------------------------------------------------------------------

def _varlen_case(lens_q, lens_k, Hq, Hkv, D):
    tq, tk = sum(lens_q), sum(lens_k)
    q = RNG.normal(size=(tq, Hq, D))
    k = RNG.normal(size=(tk, Hkv, D))
    v = RNG.normal(size=(tk, Hkv, D))
    cu_q = np.concatenate([[0], np.cumsum(lens_q)])
    cu_k = np.concatenate([[0], np.cumsum(lens_k)])
    return q, k, v, cu_q, cu_k


@pytest.mark.parametrize("causal,window", [(False, (-1, -1)), (True, (-1, -1)), (True, (3, 0)),
                                           (False, (2, 1))])
def test_varlen_gqa_matches_sdpa(causal, window):
    lens_q, lens_k = [5, 1, 9], [7, 4, 9]
    Hq, Hkv, D = 6, 2, 4
    q, k, v, cu_q, cu_k = _varlen_case(lens_q, lens_k, Hq, Hkv, D)
    out, lse = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.6, causal, window)
    for b in range(3):
        sq = slice(cu_q[b], cu_q[b + 1])
        sk = slice(cu_k[b], cu_k[b + 1])
        mask = torch.ones(lens_q[b], lens_k[b], dtype=torch.bool)
        d = lens_k[b] - lens_q[b]
        if causal or window[1] >= 0:
            mask = mask.tril(diagonal=d + (0 if causal else window[1]))
        if window[0] >= 0:
            mask = mask.triu(diagonal=d - window[0])
        ref = _sdpa(q[sq].transpose(1, 0, 2), k[sk].transpose(1, 0, 2), v[sk].transpose(1, 0, 2),
                    0.6, mask.numpy()).transpose(1, 0, 2)
        rows = mask.any(1).numpy()
        np.testing.assert_allclose(out[sq][rows], ref[rows], rtol=1e-11, atol=1e-12)
        assert np.all(out[sq][~rows] == 0) and np.all(np.isneginf(lse[:, sq][:, ~rows]))


def test_gqa_equals_repeated_heads_and_padded_equals_varlen():
    B, S, Hq, Hkv, D = 2, 6, 4, 2, 3
    q, k, v = (RNG.normal(size=(B, S, Hq, D)), RNG.normal(size=(B, S, Hkv, D)),
               RNG.normal(size=(B, S, Hkv, D)))
    o, l = oracle.attention_padded(q, k, v, 0.7, causal=True)
    kr, vr = np.repeat(k, Hq // Hkv, axis=2), np.repeat(v, Hq // Hkv, axis=2)
    o2, l2 = oracle.attention_padded(q, kr, vr, 0.7, causal=True)
    np.testing.assert_allclose(o, o2, rtol=1e-14)
    np.testing.assert_allclose(l, l2, rtol=1e-14)
    cu = np.arange(B + 1) * S
    o3, l3 = oracle.attention_varlen(q.reshape(B * S, Hq, D), k.reshape(B * S, Hkv, D),
                                     v.reshape(B * S, Hkv, D), cu, cu, 0.7, True)
    np.testing.assert_allclose(o, o3.reshape(B, S, Hq, D), rtol=1e-14)
    np.testing.assert_allclose(l, l3.reshape(Hq, B, S).transpose(1, 0, 2), rtol=1e-14)


def test_row_subset_equals_full():
    q, k, v, cu_q, cu_k = _varlen_case([4, 6], [4, 8], 4, 2, 3)
    out, lse = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.5, True, (2, 0), np.ones(4))
    rows = [(1, 5, 3), (0, 0, 0), (1, 2, 1)]
    o2, l2 = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.5, True, (2, 0), np.ones(4), rows=rows)
    for b, i, h in rows:
        t = cu_q[b] + i
        np.testing.assert_array_equal(o2[t, h], out[t, h])
        assert l2[h, t] == lse[h, t]


def test_fp8_descale_equals_prescaled_inputs():
    q, k, v, cu_q, cu_k = _varlen_case([3, 5], [3, 5], 4, 2, 4)
    qd, kd, vd = (RNG.uniform(0.5, 2, size=(2, 2)) for _ in range(3))
    out, lse = oracle.attention_varlen(q, k, v, cu_q, cu_k, 0.5, True, q_descale=qd,
                                       k_descale=kd, v_descale=vd)
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    for b in range(2):
        for g in range(2):
            q2[cu_q[b]:cu_q[b + 1], 2 * g:2 * g + 2] *= qd[b, g]
            k2[cu_k[b]:cu_k[b + 1], g] *= kd[b, g]
            v2[cu_k[b]:cu_k[b + 1], g] *= vd[b, g]
    o2, l2 = oracle.attention_varlen(q2, k2, v2, cu_q, cu_k, 0.5, True)
    np.testing.assert_allclose(out, o2, rtol=1e-13)
    np.testing.assert_allclose(lse, l2, rtol=1e-13)


# --------------------------------------------------------------------------
# paged cache
# --------------------------------------------------------------------------

def _paged_case(lens, page, Hkv, D, table):
    pages = [max(1, -(-L // page)) for L in lens]
    total = sum(pages)
    cache_k = RNG.normal(size=(total, page, Hkv, D))
    cache_v = RNG.normal(size=(total, page, Hkv, D))
    perm = np.arange(total) if table == "identity" else RNG.permutation(total)
    bt = np.zeros((len(lens), max(pages)), np.int64)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    return cache_k, cache_v, bt


def test_gather_pages_brute_force():
    cache = RNG.normal(size=(5, 4, 1, 2))
    bt = [3, 0, 4]
    got = oracle.gather_pages(cache, bt, 10)
    want = np.stack([cache[bt[t // 4], t % 4] for t in range(10)])
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("table", ["identity", "permuted"])
def test_paged_equals_contiguous(table):
    lens, page, Hq, Hkv, D, sq = [9, 16, 3], 4, 4, 2, 5, 2
    ck, cv, bt = _paged_case(lens, page, Hkv, D, table)
    q = RNG.normal(size=(3, sq, Hq, D))
    sink = RNG.normal(size=Hq)
    out, lse = oracle.attention_paged(q, ck, cv, bt, lens, 0.4, causal=True, sink=sink)
    for b, L in enumerate(lens):
        kk = oracle.gather_pages(ck, bt[b], L)
        vv = oracle.gather_pages(cv, bt[b], L)
        cu_q, cu_k = np.array([0, sq]), np.array([0, L])
        o2, l2 = oracle.attention_varlen(q[b], kk, vv, cu_q, cu_k, 0.4, True, sink=sink)
        np.testing.assert_allclose(out[b], o2, rtol=1e-13)
        np.testing.assert_allclose(lse[b], l2, rtol=1e-13)


def test_paged_descale_equals_varlen_descale_on_gathered_rows():
    # the paged FP8 path scales per (sequence, KV head) exactly as the
    # contiguous one does
    lens, page, Hq, Hkv, D, sq = [7, 12], 4, 4, 2, 3, 2
    ck, cv, bt = _paged_case(lens, page, Hkv, D, "permuted")
    q = RNG.normal(size=(2, sq, Hq, D))
    qd, kd, vd = (RNG.uniform(0.5, 2, size=(2, Hkv)) for _ in range(3))
    out, lse = oracle.attention_paged(q, ck, cv, bt, lens, 0.6, causal=True, q_descale=qd,
                                      k_descale=kd, v_descale=vd)
    plain, _ = oracle.attention_paged(q, ck, cv, bt, lens, 0.6, causal=True)
    assert np.abs(out - plain).max() > 1e-3  # the descales matter
    for b, L in enumerate(lens):
        kk = oracle.gather_pages(ck, bt[b], L)
        vv = oracle.gather_pages(cv, bt[b], L)
        cu_q, cu_k = np.array([0, sq]), np.array([0, L])
        o2, l2 = oracle.attention_varlen(q[b], kk, vv, cu_q, cu_k, 0.6, True,
                                         q_descale=qd[b:b + 1], k_descale=kd[b:b + 1],
                                         v_descale=vd[b:b + 1])
        np.testing.assert_allclose(out[b], o2, rtol=1e-13)
        np.testing.assert_allclose(lse[b], l2, rtol=1e-13)


@pytest.mark.parametrize("lens", [[0, 5], [8, 13]])
def test_paged_append_equals_contiguous_concat_and_cache_written_in_place(lens):
    # appended keys read as one sequence: equal to (a) the varlen oracle on
    # [gathered cache | new rows] and (b) the paged oracle on a cache that
    # holds the new rows at positions L .. L + s_new - 1 with lengths L + s_new
    page, Hq, Hkv, D, sq, sn = 4, 4, 2, 3, 3, 3
    ck, cv, bt = _paged_case([L + sn for L in lens], page, Hkv, D, "permuted")
    q = RNG.normal(size=(2, sq, Hq, D))
    kn, vn = RNG.normal(size=(2, sn, Hkv, D)), RNG.normal(size=(2, sn, Hkv, D))
    out, lse = oracle.attention_paged(q, ck, cv, bt, lens, 0.7, causal=True, window=(4, 0),
                                      k_new=kn, v_new=vn)
    ck2, cv2 = ck.copy(), cv.copy()
    for b, L in enumerate(lens):
        for t in range(sn):
            ck2[bt[b][(L + t) // page], (L + t) % page] = kn[b, t]
            cv2[bt[b][(L + t) // page], (L + t) % page] = vn[b, t]
        kk = np.concatenate([oracle.gather_pages(ck, bt[b], L), kn[b]])
        vv = np.concatenate([oracle.gather_pages(cv, bt[b], L), vn[b]])
        cu_q, cu_k = np.array([0, sq]), np.array([0, L + sn])
        o2, l2 = oracle.attention_varlen(q[b], kk, vv, cu_q, cu_k, 0.7, True, (4, 0))
        np.testing.assert_allclose(out[b], o2, rtol=1e-13)
        np.testing.assert_allclose(lse[b], l2, rtol=1e-13)
    o3, l3 = oracle.attention_paged(q, ck2, cv2, bt, [L + sn for L in lens], 0.7, causal=True,
                                    window=(4, 0))
    np.testing.assert_allclose(out, o3, rtol=1e-13)
    np.testing.assert_allclose(lse, l3, rtol=1e-13)


def test_paged_aliased_table_repeats_one_page():
    page, L = 4, 10
    ck = RNG.normal(size=(1, page, 1, 3))
    cv = RNG.normal(size=(1, page, 1, 3))
    q = RNG.normal(size=(1, 1, 2, 3))
    out, lse = oracle.attention_paged(q, ck, cv, np.zeros((1, 3), np.int64), [L], 1.0)
    kk = np.concatenate([ck[0]] * 3)[:L]
    vv = np.concatenate([cv[0]] * 3)[:L]
    ref = _sdpa(q[0].transpose(1, 0, 2), np.repeat(kk.transpose(1, 0, 2), 2, 0),
                np.repeat(vv.transpose(1, 0, 2), 2, 0), 1.0)
    np.testing.assert_allclose(out[0], ref.transpose(1, 0, 2), rtol=1e-12)


# --------------------------------------------------------------------------
# combine
# --------------------------------------------------------------------------

def test_split_then_combine_equals_unsplit():
    L, D = 23, 4
    q, k, v = RNG.normal(size=(3, D)), RNG.normal(size=(L, D)), RNG.normal(size=(L, D))
    vis = np.ones((3, L), bool)
    vis[2, 10:] = False
    o, lse = oracle.attention_rows(q, k, v, 0.5, vis)
    cuts = [0, 5, 5, 12, 23]            # includes an empty split
    parts = [oracle.attention_rows(q, k[a:b], v[a:b], 0.5, vis[:, a:b]) for a, b in
             zip(cuts[:-1], cuts[1:])]
    oc, lc = oracle.combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(oc, o, rtol=1e-12)
    np.testing.assert_allclose(lc, lse, rtol=1e-12)
    sink = np.array([0.3, -1.0, 2.0])
    o_s, _ = oracle.attention_rows(q, k, v, 0.5, vis, sink)
    oc2, lc2 = oracle.combine(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]),
                              sink)
    np.testing.assert_allclose(oc2, o_s, rtol=1e-12)      # sink applied once
    np.testing.assert_allclose(lc2, lse, rtol=1e-12)


def test_combine_all_empty():
    oc, lc = oracle.combine(np.ones((3, 2, 4)), np.full((3, 2), -np.inf), np.zeros(2))
    assert np.all(oc == 0) and np.all(np.isneginf(lc))


# --------------------------------------------------------------------------
# MLA
# --------------------------------------------------------------------------

def test_mla_dense_equals_sdpa_with_latent_values():
    lens, page, Hq, D, Dv = [7, 12], 4, 3, 10, 6
    ck, _, bt = _paged_case(lens, page, 1, D, "permuted")
    q = RNG.normal(size=(2, 2, Hq, D))
    out, lse = oracle.mla_paged(q, ck, bt, lens, Dv, 0.3)
    for b, L in enumerate(lens):
        kk = oracle.gather_pages(ck, bt[b], L)[:, 0, :]
        for i in range(2):
            ref = _sdpa(q[b, i][:, None, :], np.repeat(kk[None], Hq, 0),
                        np.repeat(kk[None, :, :Dv], Hq, 0), 0.3)[:, 0, :]
            np.testing.assert_allclose(out[b, i], ref, rtol=1e-12)


def _e4m3_values(shape):
    """Random e4m3 codes (NaN codes excluded) decoded to float64."""
    codes = RNG.integers(0, 256, size=shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38
    return oracle.decode(codes, "e4m3")


def test_mla_fp8_descales_match_sdpa_on_scaled_rows():
    # K = row * k_descale and V = row[:Dv] * v_descale of the same cached row:
    # a transposed descale (K's on V) or a dropped one fails here.
    lens, page, Hq, Hkv, D, Dv = [7, 12], 4, 4, 2, 10, 6
    _, _, bt = _paged_case(lens, page, Hkv, D, "permuted")
    ck = _e4m3_values((int(bt.max()) + 1, page, Hkv, D))
    q = _e4m3_values((2, 2, Hq, D))
    qd, kd, vd = (RNG.uniform(0.5, 2, size=(2, Hkv)) for _ in range(3))
    out, lse = oracle.mla_paged(q, ck, bt, lens, Dv, 0.3, q_descale=qd, k_descale=kd,
                                v_descale=vd)
    for b, L in enumerate(lens):
        rows = oracle.gather_pages(ck, bt[b], L)
        for h in range(Hq):
            g = h // (Hq // Hkv)
            kk, vv = rows[:, g, :] * kd[b, g], rows[:, g, :Dv] * vd[b, g]
            qq = q[b, :, h, :] * qd[b, g]
            ref = _sdpa(qq[None], kk[None], vv[None], 0.3)[0]
            np.testing.assert_allclose(out[b, :, h], ref, rtol=1e-12, atol=1e-14)
            s = 0.3 * qq @ kk.T
            np.testing.assert_allclose(lse[b, h], torch.logsumexp(torch.as_tensor(s), -1).numpy(),
                                       rtol=1e-12)


def test_mla_sparse_fp8_descales_match_sdpa_on_gathered_rows():
    lens, page, Hq, D, Dv = [20], 4, 2, 8, 5
    pages = -(-20 // page)
    ck = _e4m3_values((pages, page, 1, D))
    bt = RNG.permutation(pages)[None]
    q = _e4m3_values((1, 1, Hq, D))
    sel = np.array([1, 4, 5, 11, 17, 19])
    qd, kd, vd = (RNG.uniform(0.5, 2, size=(1, 1)) for _ in range(3))
    out, _ = oracle.mla_sparse(q, ck, bt, lens, sel.reshape(1, 1, 1, -1), Dv, 0.5,
                               q_descale=qd, k_descale=kd, v_descale=vd)
    rows = oracle.gather_pages(ck, bt[0], 20)[sel, 0, :]
    ref = _sdpa(q[0, 0][:, None, :] * qd[0, 0], np.repeat(rows[None] * kd[0, 0], Hq, 0),
                np.repeat(rows[None, :, :Dv] * vd[0, 0], Hq, 0), 0.5)[:, 0, :]
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12)


def test_mla_sparse_all_positions_equals_dense_and_skips_invalid():
    lens, page, Hq, D, Dv, topk = [7, 12], 4, 3, 10, 6, 16
    ck, _, bt = _paged_case(lens, page, 1, D, "permuted")
    q = RNG.normal(size=(2, 2, Hq, D))
    idx = np.full((2, 2, 1, topk), -1, np.int64)
    for b, L in enumerate(lens):
        idx[b, :, 0, :L] = np.arange(L)
    idx[0, 1, 0, 10] = 99                       # beyond the cache length: skipped
    o_s, l_s = oracle.mla_sparse(q, ck, bt, lens, idx, Dv, 0.3)
    o_d, l_d = oracle.mla_paged(q, ck, bt, lens, Dv, 0.3)
    np.testing.assert_allclose(o_s, o_d, rtol=1e-12)
    np.testing.assert_allclose(l_s, l_d, rtol=1e-12)


def test_mla_sparse_subset_matches_sdpa_on_gathered_rows():
    lens, page, Hq, D, Dv, topk = [20], 4, 2, 8, 5, 6
    ck, _, bt = _paged_case(lens, page, 1, D, "permuted")
    q = RNG.normal(size=(1, 1, Hq, D))
    sel = np.array([1, 4, 5, 11, 17, 19])
    idx = sel.reshape(1, 1, 1, topk)
    out, _ = oracle.mla_sparse(q, ck, bt, lens, idx, Dv, 0.5)
    kk = oracle.gather_pages(ck, bt[0], 20)[sel, 0, :]
    ref = _sdpa(q[0, 0][:, None, :], np.repeat(kk[None], Hq, 0),
                np.repeat(kk[None, :, :Dv], Hq, 0), 0.5)[:, 0, :]
    np.testing.assert_allclose(out[0, 0], ref, rtol=1e-12)


# ---------------------------------------------------------------------------
# Additive score mask and seqused (padded layout)
# ---------------------------------------------------------------------------

def test_mla_two_kv_heads_equal_each_group_alone():
    # H_kv = 2: heads 0..G-1 read KV head 0 (and its index list), heads
    # G..2G-1 KV head 1; each half equals the one-KV-head problem on its slice
    lens, page, D, Dv, G, sq, topk = [9, 20], 4, 6, 4, 3, 2, 5
    ck, _, bt = _paged_case(lens, page, 2, D, "permuted")
    q = RNG.normal(size=(2, sq, 2 * G, D))
    idx = np.stack([[[RNG.choice(max(L, 1) + 3, topk, replace=False) - 1 for _ in range(2)]
                     for _ in range(sq)] for L in lens])
    do, dl = oracle.mla_paged(q, ck, bt, lens, Dv, 0.5)
    so, sl = oracle.mla_sparse(q, ck, bt, lens, idx, Dv, 0.5)
    for g in range(2):
        hs = slice(g * G, (g + 1) * G)
        o1, l1 = oracle.mla_paged(q[:, :, hs], ck[:, :, g:g + 1], bt, lens, Dv, 0.5)
        np.testing.assert_allclose(do[:, :, hs], o1, rtol=1e-13)
        np.testing.assert_allclose(dl[:, hs], l1, rtol=1e-13)
        o2, l2 = oracle.mla_sparse(q[:, :, hs], ck[:, :, g:g + 1], bt, lens,
                                   idx[:, :, g:g + 1], Dv, 0.5)
        np.testing.assert_allclose(so[:, :, hs], o2, rtol=1e-13)
        np.testing.assert_allclose(sl[:, hs], l2, rtol=1e-13)
    assert np.abs(so[:, :, :G] - so[:, :, G:]).max() > 1e-3


@pytest.mark.parametrize("causal", [False, True])
def test_mla_sparse_tnd_equal_lengths_is_bsnd_reshaped(causal):
    # packed (TND) queries of equal-length sequences are the BSND problem
    # with its batch and token axes merged
    lens, page, D, Dv, Hq, S, topk = [9, 20, 14], 4, 6, 4, 2, 3, 6
    ck, _, bt = _paged_case(lens, page, 1, D, "permuted")
    q = RNG.normal(size=(3, S, Hq, D))
    idx = np.stack([[[RNG.choice(L + 2, topk, replace=False) - 1] for _ in range(S)]
                    for L in lens])
    ro, rl = oracle.mla_sparse(q, ck, bt, lens, idx, Dv, 0.5, causal=causal)
    cu = np.arange(4) * S
    to, tl = oracle.mla_sparse_tnd(q.reshape(3 * S, Hq, D), ck, bt, lens, cu,
                                   idx.reshape(3 * S, 1, topk), Dv, 0.5, causal=causal)
    np.testing.assert_array_equal(to, ro.reshape(3 * S, Hq, Dv))
    np.testing.assert_array_equal(tl, rl.transpose(1, 0, 2).reshape(Hq, 3 * S))


def test_mla_sparse_tnd_unequal_lengths_follow_each_sequence():
    # sequence b's tokens see only sequence b's cache; an empty sequence
    # contributes no tokens
    lens, page, D, Dv, Hq, topk = [9, 30, 14], 4, 6, 4, 2, 5
    ck, _, bt = _paged_case(lens, page, 1, D, "permuted")
    nq = [2, 0, 3]
    cu = np.concatenate([[0], np.cumsum(nq)])
    q = RNG.normal(size=(5, Hq, D))
    idx = np.stack([[RNG.choice(lens[b] + 1, topk, replace=False) - 1]
                    for b in range(3) for _ in range(nq[b])])
    to, tl = oracle.mla_sparse_tnd(q, ck, bt, lens, cu, idx, Dv, 0.5, causal=True)
    for b in (0, 2):
        t0, t1 = cu[b], cu[b + 1]
        o, l = oracle.mla_sparse(q[None, t0:t1], ck, bt[b:b + 1], [lens[b]], idx[None, t0:t1], Dv,
                                 0.5, causal=True)
        np.testing.assert_array_equal(to[t0:t1], o[0])
        np.testing.assert_array_equal(tl[:, t0:t1], l[0])
    # the other sequences' caches are not read: changing them changes nothing
    ck2 = ck.copy()
    ck2[bt[1][:8]] += 1.0
    to2, _ = oracle.mla_sparse_tnd(q, ck2, bt, lens, cu, idx, Dv, 0.5, causal=True)
    np.testing.assert_array_equal(to2, to)


def test_additive_mask_zero_and_constant_shift():
    """A zero mask changes nothing; a mask constant over a row's keys leaves O
    unchanged (softmax is shift-invariant) and adds the constant to the LSE."""
    B, S, Hq, Hkv, D = 2, 9, 4, 2, 8
    q = RNG.normal(size=(B, S, Hq, D))
    k = RNG.normal(size=(B, S, Hkv, D))
    v = RNG.normal(size=(B, S, Hkv, D))
    o0, l0 = oracle.attention_padded(q, k, v, 0.3, causal=True)
    oz, lz = oracle.attention_padded(q, k, v, 0.3, causal=True, mask=np.zeros((1, 1, S, S)))
    np.testing.assert_array_equal(oz, o0)
    np.testing.assert_array_equal(lz, l0)
    c = RNG.normal(size=(B, Hq, S, 1))
    oc, lc = oracle.attention_padded(q, k, v, 0.3, causal=True, mask=np.repeat(c, S, 3))
    np.testing.assert_allclose(oc, o0, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lc, l0 + c[..., 0], rtol=1e-12)


def test_additive_mask_minus_inf_removes_keys_and_bias_matches_sdpa():
    """-inf entries drop those keys (compared with the attention over the
    remaining keys only); a finite bias matches torch SDPA with an additive
    float mask on the same rows."""
    S, Hq, D = 11, 3, 6
    q = RNG.normal(size=(1, S, Hq, D))
    k = RNG.normal(size=(1, S, Hq, D))
    v = RNG.normal(size=(1, S, Hq, D))
    drop = np.zeros((1, 1, S, S))
    keep = np.array([0, 2, 3, 7, 10])
    drop[..., np.setdiff1d(np.arange(S), keep)] = -np.inf
    o, l = oracle.attention_padded(q, k, v, 0.4, mask=drop)
    ref_o, ref_l = oracle.attention_padded(q, k[:, keep], v[:, keep], 0.4)
    np.testing.assert_allclose(o, ref_o, rtol=1e-12)
    np.testing.assert_allclose(l, ref_l, rtol=1e-12)
    bias = RNG.normal(size=(1, Hq, S, S))
    ob, _ = oracle.attention_padded(q, k, v, 0.4, mask=bias)
    qt = torch.tensor(q[0].transpose(1, 0, 2))
    kt = torch.tensor(k[0].transpose(1, 0, 2))
    vt = torch.tensor(v[0].transpose(1, 0, 2))
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.tensor(bias[0]),
                                         scale=0.4).numpy().transpose(1, 0, 2)
    np.testing.assert_allclose(ob[0], ref, rtol=1e-10, atol=1e-12)


def test_seqused_equals_varlen_of_the_used_rows():
    """Padded q/k/v with seqused_q/k = the packed (varlen) attention of each
    sequence's first seqused rows and keys; rows past seqused stay 0 / -inf."""
    B, Sq, Sk, Hq, Hkv, D = 3, 10, 13, 4, 2, 8
    q = RNG.normal(size=(B, Sq, Hq, D))
    k = RNG.normal(size=(B, Sk, Hkv, D))
    v = RNG.normal(size=(B, Sk, Hkv, D))
    uq, uk = [10, 4, 7], [13, 9, 1]
    o, l = oracle.attention_padded(q, k, v, 0.35, causal=True, window=(5, 0),
                                   seqused_q=uq, seqused_k=uk)
    qp = np.concatenate([q[b, :uq[b]] for b in range(B)])
    kp = np.concatenate([k[b, :uk[b]] for b in range(B)])
    vp = np.concatenate([v[b, :uk[b]] for b in range(B)])
    cq, ck = np.concatenate([[0], np.cumsum(uq)]), np.concatenate([[0], np.cumsum(uk)])
    ov, lv = oracle.attention_varlen(qp, kp, vp, cq, ck, 0.35, True, (5, 0))
    for b in range(B):
        np.testing.assert_array_equal(o[b, :uq[b]], ov[cq[b]:cq[b + 1]])
        np.testing.assert_array_equal(l[b, :, :uq[b]], lv[:, cq[b]:cq[b + 1]])
        assert np.all(o[b, uq[b]:] == 0) and np.all(np.isneginf(l[b, :, uq[b]:]))


def test_mla_sparse_blocks_covering_the_cache_equal_dense():
    """Block indices 0 .. L/bs - 1 with block size bs list every position once:
    the result is the dense MLA attention; a -1 entry and a block reaching past
    the cache end only drop positions."""
    lens, page, Hq, D, Dv, bs = [16, 11], 4, 2, 10, 6, 4
    ck, _, bt = _paged_case(lens, page, 1, D, "permuted")
    q = RNG.normal(size=(2, 2, Hq, D))
    idx = np.full((2, 2, 1, 5), -1, np.int64)
    for b, L in enumerate(lens):
        nb = (L + bs - 1) // bs                 # the last block of sequence 1 runs past L
        idx[b, :, 0, :nb] = np.arange(nb)
    o_s, l_s = oracle.mla_sparse(q, ck, bt, lens, idx, Dv, 0.3, block_size=bs)
    o_d, l_d = oracle.mla_paged(q, ck, bt, lens, Dv, 0.3)
    np.testing.assert_allclose(o_s, o_d, rtol=1e-12)
    np.testing.assert_allclose(l_s, l_d, rtol=1e-12)
    # one block of 4: the same as listing its 4 positions with block size 1
    sel = np.array([[[[2, -1]]]])
    o_b, _ = oracle.mla_sparse(q[:1, :1], ck, bt[:1], lens[:1], sel, Dv, 0.3, block_size=4)
    o_1, _ = oracle.mla_sparse(q[:1, :1], ck, bt[:1], lens[:1],
                               np.array([[[[8, 9, 10, 11]]]]), Dv, 0.3)
    np.testing.assert_allclose(o_b, o_1, rtol=1e-12)


def test_mla_sparse_causal_all_positions_equals_dense_causal():
    """sparse_mode=3 (rightDownCausal) over the list of all positions is the
    dense MLA attention with the bottom-right causal mask."""
    lens, page, Hq, D, Dv = [9, 14], 4, 2, 10, 6
    ck, _, bt = _paged_case(lens, page, 1, D, "permuted")
    q = RNG.normal(size=(2, 3, Hq, D))
    idx = np.full((2, 3, 1, 16), -1, np.int64)
    for b, L in enumerate(lens):
        idx[b, :, 0, :L] = np.arange(L)
    o_s, l_s = oracle.mla_sparse(q, ck, bt, lens, idx, Dv, 0.3, causal=True)
    o_d, l_d = oracle.mla_paged(q, ck, bt, lens, Dv, 0.3, causal=True)
    np.testing.assert_allclose(o_s, o_d, rtol=1e-12)
    np.testing.assert_allclose(l_s, l_d, rtol=1e-12)
