"""Randomised pins for the fp64 oracle (hypothesis, CPU): on random small
shapes, lengths, masks and sinks, the oracle agrees with torch's fp64
scaled_dot_product_attention and with the invariants the definition implies
(split + combine = unsplit; GQA = repeated heads; paged = contiguous)."""
import numpy as np
import torch
import torch.nn.functional as F
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

SETTINGS = settings(max_examples=40, deadline=None, derandomize=True)


@st.composite
def problems(draw):
    lq = draw(st.integers(1, 9))
    lk = draw(st.integers(1, 12))
    hkv = draw(st.sampled_from([1, 2]))
    hq = hkv * draw(st.sampled_from([1, 2, 3]))
    d = draw(st.integers(1, 6))
    causal = draw(st.booleans())
    wl = draw(st.sampled_from([-1, 0, 1, 3, 20]))
    wr = draw(st.sampled_from([-1, 0, 2]))
    seed = draw(st.integers(0, 2**31 - 1))
    return lq, lk, hq, hkv, d, causal, wl, wr, seed


@SETTINGS
@given(problems())
def test_varlen_matches_torch_sdpa_on_random_problems(pb):
    lq, lk, hq, hkv, d, causal, wl, wr, seed = pb
    rng = np.random.default_rng(seed)
    q, k, v = (rng.normal(size=(n, h, d)) for n, h in ((lq, hq), (lk, hkv), (lk, hkv)))
    out, lse = oracle.attention_varlen(q, k, v, np.array([0, lq]), np.array([0, lk]), 0.7,
                                       causal, (wl, wr))
    vis = oracle.visible_mask(lq, lk, causal, wl, wr)
    # rows that see nothing: O = 0 and LSE = -inf by the reading; elsewhere SDPA
    rows = vis.any(axis=1)
    assert np.all(out[~rows] == 0) and np.all(np.isneginf(lse[:, ~rows]))
    if rows.any():
        g = hq // hkv
        kk = np.repeat(k.transpose(1, 0, 2), g, 0)
        vv = np.repeat(v.transpose(1, 0, 2), g, 0)
        tq = torch.as_tensor(q.transpose(1, 0, 2))[None]
        m = torch.as_tensor(vis)[None, None]
        ref = F.scaled_dot_product_attention(tq, torch.as_tensor(kk)[None],
                                             torch.as_tensor(vv)[None], attn_mask=m,
                                             scale=0.7)[0].numpy().transpose(1, 0, 2)
        np.testing.assert_allclose(out[rows], ref[rows], rtol=1e-10, atol=1e-12)
        s = np.einsum("qhd,khd->hqk", q, np.repeat(k, g, 1)) * 0.7
        s = np.where(vis[None], s, -np.inf)
        ref_lse = torch.logsumexp(torch.as_tensor(s), dim=-1).numpy()
        np.testing.assert_allclose(lse[:, rows], ref_lse[:, rows], rtol=1e-12)


@SETTINGS
@given(problems(), st.integers(1, 4), st.booleans())
def test_any_key_split_then_combine_equals_unsplit(pb, nsplit, with_sink):
    lq, lk, hq, hkv, d, causal, wl, wr, seed = pb
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(lq, d))
    k, v = rng.normal(size=(lk, d)), rng.normal(size=(lk, d))
    sink = float(rng.normal()) if with_sink else None
    vis = oracle.visible_mask(lq, lk, causal, wl, wr)
    o, l = oracle.attention_rows(q, k, v, 0.5, vis, sink)
    # cut the keys at random points into nsplit disjoint (possibly empty) parts
    cuts = np.sort(rng.integers(0, lk + 1, size=nsplit - 1))
    edges = np.concatenate([[0], cuts, [lk]])
    parts_o, parts_l = [], []
    for a, b in zip(edges[:-1], edges[1:]):
        sub = np.zeros_like(vis)
        sub[:, a:b] = vis[:, a:b]
        po, pl = oracle.attention_rows(q, k, v, 0.5, sub, None)
        parts_o.append(po)
        parts_l.append(pl)
    co, cl = oracle.combine(np.stack(parts_o), np.stack(parts_l),
                            None if sink is None else np.full(lq, sink))
    np.testing.assert_allclose(co, o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(cl, l, rtol=1e-12)


@SETTINGS
@given(st.lists(st.integers(0, 40), min_size=1, max_size=4), st.sampled_from([2, 4, 8]),
       st.integers(0, 2**31 - 1))
def test_paged_equals_contiguous_on_random_tables(lens, page, seed):
    rng = np.random.default_rng(seed)
    hkv, hq, d, sq = 2, 4, 3, 2
    pages = [max(1, -(-L // page)) for L in lens]
    total = sum(pages)
    ck = rng.normal(size=(total, page, hkv, d))
    cv = rng.normal(size=(total, page, hkv, d))
    perm = rng.permutation(total)
    bt = np.zeros((len(lens), max(pages)), np.int64)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    q = rng.normal(size=(len(lens), sq, hq, d))
    out, lse = oracle.attention_paged(q, ck, cv, bt, lens, 0.6, causal=True)
    for b, L in enumerate(lens):
        kk = np.concatenate([ck[bt[b, t // page], t % page][None] for t in range(L)]) \
            if L else np.zeros((0, hkv, d))
        vv = np.concatenate([cv[bt[b, t // page], t % page][None] for t in range(L)]) \
            if L else np.zeros((0, hkv, d))
        o2, l2 = oracle.attention_varlen(q[b], kk, vv, np.array([0, sq]), np.array([0, L]), 0.6,
                                         True)
        np.testing.assert_allclose(out[b], o2, rtol=1e-13)
        np.testing.assert_allclose(lse[b], l2, rtol=1e-13)
