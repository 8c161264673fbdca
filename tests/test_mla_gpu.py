"""MLA-absorbed decode (mla_fwd_paged) and its top-k sparse variant
(mla_sparse_fwd) on the GPU against the fp64 oracle: bf16 outputs within
1e-2 max-abs (5e-2 for e4m3 q and cache with descales), LSE within 1e-3."""
import numpy as np
import pytest
import torch

import oracle
from attention_online_softmax_fmha_b200 import binding as B
from attention_online_softmax_fmha_b200 import build as BUILD
from attention_online_softmax_fmha_b200 import workloads as W
from tests._util import assert_close_lse, assert_close_out, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    BUILD.build()
    B.lib()


def run(inp, use_meta=True, num_ctas=0):
    meta = None
    topk = inp.topk if inp.indices is not None else 0
    if use_meta:
        meta = B.mla_metadata(inp.cache_seqlens, batch=inp.batch, seqlen_q=inp.q.shape[1],
                              num_heads_q=inp.num_heads_q, page_size=inp.page_size, topk=topk,
                              num_ctas=num_ctas, num_heads_kv=inp.num_heads_kv)
    kw = dict(scale=inp.scale, causal=inp.causal, meta=meta, num_ctas=num_ctas,
              q_descale=inp.q_descale, k_descale=inp.k_descale, v_descale=inp.v_descale)
    if inp.indices is None:
        out, lse = B.mla_fwd_paged(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, **kw)
    else:
        out, lse = B.mla_sparse_fwd(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens,
                                    inp.indices, **kw)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    return out, lse


def _desc(inp):
    if inp.q_descale is None:
        return {}
    return dict(q_descale=inp.q_descale.cpu().numpy(), k_descale=inp.k_descale.cpu().numpy(),
                v_descale=inp.v_descale.cpu().numpy())


def _atol(inp):
    return 5e-2 if inp.dtype == "e4m3" else 1e-2


def check(inp, **kw):
    out, lse = run(inp, **kw)
    q, kv = to_f64(inp.q), to_f64(inp.kv_cache)
    bt = inp.block_table.cpu().numpy()
    if inp.indices is None:
        ro, rl = oracle.mla_paged(q, kv, bt, inp.seqlens, 512, inp.scale, inp.causal, **_desc(inp))
    else:
        ro, rl = oracle.mla_sparse(q, kv, bt, inp.seqlens, inp.indices.cpu().numpy(), 512,
                                   inp.scale, **_desc(inp))
    assert_close_out(to_f64(out), ro, _atol(inp))
    assert_close_lse(lse.cpu().numpy(), rl)


LENS = [1, 31, 32, 33, 200, 1000]


@pytest.mark.parametrize("num_ctas", [1, 5, 0])
def test_dense_split_counts(num_ctas):
    inp = W.make_mla(seqlens=LENS, seqlen_q=2, num_heads_q=128, page_size=64, seed=0,
                     device="cuda")
    check(inp, num_ctas=num_ctas)


def test_dense_without_metadata_causal_and_page16():
    inp = W.make_mla(seqlens=[5, 77, 300], seqlen_q=2, num_heads_q=128, page_size=16,
                     causal=True, seed=1, device="cuda")
    check(inp, use_meta=False)
    check(inp, num_ctas=4)


def test_mate_example_shapes():
    # The MATE MLA example: q (1, 32, 8, 576), a 4-page cache of 16-token
    # pages with 2 KV heads, block_table all zeros (page 0 repeats),
    # cache_seqlens [32], head_dim_v 512; with and without metadata.
    g = torch.Generator(device="cuda").manual_seed(0)
    q = torch.randn(1, 32, 8, 576, generator=g, device="cuda").to(torch.bfloat16)
    bt = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    cs = torch.tensor([32], dtype=torch.int32, device="cuda")
    kv2 = torch.randn(4, 16, 2, 576, generator=g, device="cuda").to(torch.bfloat16)
    ro, rl = oracle.mla_paged(to_f64(q), to_f64(kv2), bt.cpu().numpy(), [32], 512, 1 / 24.0)
    meta = B.mla_metadata(cs, batch=1, seqlen_q=32, num_heads_q=8, page_size=16, num_ctas=3,
                          num_heads_kv=2)
    for kw in (dict(), dict(meta=meta, num_ctas=3)):
        out, lse = B.mla_fwd_paged(q, kv2, bt, cs, head_dim_v=512, **kw)
        torch.cuda.synchronize()
        assert B.device_error() == 0
        assert_close_out(to_f64(out), ro, 1e-2)
        assert_close_lse(lse.cpu().numpy(), rl)


@pytest.mark.parametrize("Hq,Hkv,sq", [(256, 2, 1), (64, 4, 3)])
def test_dense_several_kv_heads(Hq, Hkv, sq):
    # 128 query heads per KV head (one row tile per token), and 16 (eight
    # tokens per row tile); split and unsplit
    inp = W.make_mla(seqlens=[7, 100, 700], seqlen_q=sq, num_heads_q=Hq, num_heads_kv=Hkv,
                     page_size=32, causal=sq > 1, seed=40, device="cuda")
    check(inp, num_ctas=5)
    check(inp, use_meta=False)


def test_sparse_several_kv_heads():
    inp = W.make_mla(seqlens=[20, 300, 3000], seqlen_q=2, num_heads_q=128, num_heads_kv=2,
                     page_size=64, topk=128, seed=41, device="cuda")
    assert not torch.equal(inp.indices[:, :, 0], inp.indices[:, :, 1])
    check(inp, num_ctas=3)
    check(inp, use_meta=False)


@pytest.mark.parametrize("num_ctas", [3, 0])
def test_sparse_against_oracle(num_ctas):
    inp = W.make_mla(seqlens=[20, 300, 3000], seqlen_q=2, num_heads_q=128, page_size=64,
                     topk=256, seed=2, device="cuda")
    inp.indices[0, 1, 0, 5] = 19999       # beyond the cache: skipped
    inp.indices[2, 0, 0, 7] = -5          # negative: skipped
    check(inp, num_ctas=num_ctas)
    check(inp, use_meta=False)


def test_sparse_all_positions_equals_dense():
    inp = W.make_mla(seqlens=[64, 100], seqlen_q=1, num_heads_q=128, page_size=32, topk=128,
                     index_kind="all", seed=3, device="cuda")
    out_s, lse_s = run(inp, num_ctas=2)
    dense = W.MlaInputs(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, inp.seqlens,
                        inp.page_size, inp.num_heads_q, 512, False, inp.scale, None, 0)
    out_d, lse_d = run(dense, num_ctas=2)
    assert (to_f64(out_s) - to_f64(out_d)).__abs__().max() <= 2e-2
    assert np.abs(lse_s.cpu().numpy() - lse_d.cpu().numpy()).max() <= 1e-3
    check(inp, num_ctas=2)


def _sampled(name, topk):
    inp = W.build_config(name, seed=0, device="cuda")
    out, lse = run(inp)
    o, l = to_f64(out), lse.cpu().numpy()
    order = np.argsort(inp.seqlens)
    for b in [int(order[0]), int(order[-1]), 9]:
        L = inp.seqlens[b]
        npg = -(-L // inp.page_size)
        pages = inp.block_table[b, :npg].long()
        kv = to_f64(inp.kv_cache[pages])
        q = to_f64(inp.q[b:b + 1])
        desc = {k: v[b:b + 1] for k, v in _desc(inp).items()}
        if topk:
            ro, rl = oracle.mla_sparse(q, kv, np.arange(npg)[None], [L],
                                       inp.indices[b:b + 1].cpu().numpy(), 512, inp.scale, **desc)
        else:
            ro, rl = oracle.mla_paged(q, kv, np.arange(npg)[None], [L], 512, inp.scale, **desc)
        assert_close_out(o[b:b + 1], ro, _atol(inp))
        assert_close_lse(l[b:b + 1], rl)


def test_full_size_dense_sampled():
    """MLA dense decode at full size (64 sequences, L ~ U[4096, 65536], 2
    tokens x 128 heads, pages of 64, permuted table); 3 sequences checked."""
    _sampled("mla_dense", 0)


def test_full_size_sparse_sampled():
    """The top-2048 sparse variant at full size; 3 sequences checked."""
    _sampled("mla_sparse", 2048)


# ---------------------------------------------------------------------------
# e4m3 q and latent cache with (B, H_kv) descales: S on the FP8 codes, P V in
# fp16 on an exact fp16 copy of V. Tolerance 5e-2.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("num_ctas", [1, 5, 0])
def test_fp8_dense_split_counts(num_ctas):
    inp = W.make_mla(seqlens=LENS, seqlen_q=2, num_heads_q=128, page_size=64, dtype="e4m3",
                     seed=50, device="cuda")
    check(inp, num_ctas=num_ctas)


def test_fp8_dense_without_metadata_causal_page16_several_kv_heads():
    inp = W.make_mla(seqlens=[5, 77, 300], seqlen_q=3, num_heads_q=64, num_heads_kv=4,
                     page_size=16, causal=True, dtype="e4m3", seed=51, device="cuda")
    check(inp, use_meta=False)
    check(inp, num_ctas=4)


def test_fp8_without_descales_equals_unit_descales():
    inp = W.make_mla(seqlens=[33, 200], seqlen_q=2, num_heads_q=128, dtype="e4m3", seed=52,
                     device="cuda")
    out1, lse1 = run(inp, num_ctas=3)
    ones = torch.ones_like(inp.q_descale)
    inp.q_descale, inp.k_descale, inp.v_descale = ones, ones, ones.clone()
    out2, lse2 = run(inp, num_ctas=3)
    plain = dict(scale=inp.scale, meta=B.mla_metadata(inp.cache_seqlens, batch=2, seqlen_q=2,
                                                      num_heads_q=128, page_size=64, num_ctas=3),
                 num_ctas=3)
    out3, lse3 = B.mla_fwd_paged(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens, **plain)
    torch.cuda.synchronize()
    assert torch.equal(out2, out3) and torch.equal(lse2, lse3)
    assert not torch.equal(out1, out2)
    check(inp, num_ctas=3)


@pytest.mark.parametrize("num_ctas", [3, 0])
def test_fp8_sparse_against_oracle(num_ctas):
    inp = W.make_mla(seqlens=[20, 300, 3000], seqlen_q=2, num_heads_q=128, page_size=64,
                     topk=256, dtype="e4m3", seed=53, device="cuda")
    inp.indices[0, 1, 0, 5] = 19999
    inp.indices[2, 0, 0, 7] = -5
    check(inp, num_ctas=num_ctas)
    check(inp, use_meta=False)


def test_fp8_sparse_several_kv_heads():
    inp = W.make_mla(seqlens=[20, 300, 3000], seqlen_q=2, num_heads_q=128, num_heads_kv=2,
                     page_size=64, topk=128, dtype="e4m3", seed=54, device="cuda")
    check(inp, num_ctas=3)


def test_fp8_full_size_dense_sampled():
    """The e4m3 MLA dense workload at full size; 3 sequences checked."""
    _sampled("mla_dense_fp8", 0)


def test_fp8_full_size_sparse_sampled():
    _sampled("mla_sparse_fp8", 2048)


@pytest.mark.parametrize("bs,num_ctas", [(4, 3), (64, 0)])
def test_sparse_block_indices(bs, num_ctas):
    """sparse_block_size > 1 (MindSpore sparse_flash_attention): index k lists
    positions k*bs .. k*bs + bs - 1; -1 entries and positions past the cache
    end are skipped."""
    lens, topk = [20, 300, 3000], 64
    inp = W.make_mla(seqlens=lens, seqlen_q=2, num_heads_q=128, page_size=64, topk=topk,
                     seed=5, device="cuda")
    g = torch.Generator().manual_seed(bs)
    idx = torch.full((3, 2, 1, topk), -1, dtype=torch.int32)
    for b, L in enumerate(lens):
        nb = -(-L // bs)
        for i in range(2):
            n = min(nb, topk - 3)
            idx[b, i, 0, :n] = torch.randperm(nb, generator=g)[:n].sort().values.int()
    inp.indices = idx.cuda()
    meta = B.mla_metadata(inp.cache_seqlens, batch=3, seqlen_q=2, num_heads_q=128, page_size=64,
                          topk=topk, num_ctas=num_ctas, sparse_block_size=bs)
    out, lse = B.mla_sparse_fwd(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens,
                                inp.indices, scale=inp.scale, meta=meta, num_ctas=num_ctas,
                                sparse_block_size=bs)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    ro, rl = oracle.mla_sparse(to_f64(inp.q), to_f64(inp.kv_cache), inp.block_table.cpu().numpy(),
                               lens, idx.numpy(), 512, inp.scale, block_size=bs)
    assert_close_out(to_f64(out), ro, 1e-2)
    assert_close_lse(lse.cpu().numpy(), rl)


def test_sparse_causal_right_down():
    """sparse_mode=3 ("rightDownCausal"): listed positions past i + L - s_q are
    skipped as well."""
    lens = [40, 300, 3000]
    inp = W.make_mla(seqlens=lens, seqlen_q=3, num_heads_q=128, page_size=64, topk=128,
                     seed=6, device="cuda")
    # make sure the last positions are listed, so the causal cut removes some
    for b, L in enumerate(lens):
        inp.indices[b, :, 0, -3:] = torch.tensor([L - 3, L - 2, L - 1], dtype=torch.int32)
    meta = B.mla_metadata(inp.cache_seqlens, batch=3, seqlen_q=3, num_heads_q=128, page_size=64,
                          topk=128)
    out, lse = B.mla_sparse_fwd(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens,
                                inp.indices, scale=inp.scale, meta=meta, causal=True)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    ro, rl = oracle.mla_sparse(to_f64(inp.q), to_f64(inp.kv_cache), inp.block_table.cpu().numpy(),
                               lens, inp.indices.cpu().numpy(), 512, inp.scale, causal=True)
    assert_close_out(to_f64(out), ro, 1e-2)
    assert_close_lse(lse.cpu().numpy(), rl)


def _run_tnd(inp, use_meta, num_ctas=0):
    T = inp.q.shape[0]
    meta = None
    if use_meta:
        meta = B.mla_metadata(inp.cache_seqlens, batch=1, seqlen_q=T, num_heads_q=inp.num_heads_q,
                              page_size=inp.page_size, topk=inp.topk, num_ctas=num_ctas)
    out, lse = B.mla_sparse_fwd(inp.q, inp.kv_cache, inp.block_table, inp.cache_seqlens,
                                inp.indices, scale=inp.scale, causal=inp.causal, meta=meta,
                                num_ctas=num_ctas, cu_seqlens_q=inp.cu_seqlens_q)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    return out, lse


@pytest.mark.parametrize("causal", [False, True])
def test_sparse_packed_tnd_queries(causal):
    """Packed (TND) queries (MindSpore sparse_flash_attention,
    layout_query="TND"): sequence b's tokens read only sequence b's cache;
    two sequences (one in the middle) have no query token."""
    inp = W.make_mla_tnd(seqlens=[20, 300, 3000, 50, 90], seqlens_q=[3, 0, 5, 2, 0],
                         num_heads_q=128, topk=128, page_size=64, causal=causal, seed=42,
                         device="cuda")
    ro, rl = oracle.mla_sparse_tnd(to_f64(inp.q), to_f64(inp.kv_cache),
                                   inp.block_table.cpu().numpy(), inp.seqlens,
                                   inp.cu_seqlens_q.cpu().numpy(), inp.indices.cpu().numpy(), 512,
                                   inp.scale, causal=causal)
    for kw in (dict(use_meta=True, num_ctas=3), dict(use_meta=False)):
        out, lse = _run_tnd(inp, **kw)
        assert_close_out(to_f64(out), ro, 1e-2)
        assert_close_lse(lse.cpu().numpy(), rl)



def test_sparse_gathers_from_an_unevenly_strided_cache():
    """A cache with NaN padding after every block (block stride above
    page_size x 576) gives bit for bit the packed cache's result: the sparse
    gathers follow the block stride and never read the padding."""
    inp = W.make_mla(seqlens=[20, 300, 3000], seqlen_q=2, num_heads_q=128, page_size=64,
                     topk=256, seed=55, device="cuda")
    inp.indices[1, 0, 0, 3] = 5000        # beyond the cache: skipped
    nb, P = inp.kv_cache.shape[0], inp.kv_cache.shape[1]
    blk = P * 576 + 64                    # 64 elements of padding after each block
    store = torch.full((nb * blk,), float("nan"), dtype=torch.bfloat16, device="cuda")
    view = store.as_strided((nb, P, 1, 576), (blk, 576, 576, 1))
    view.copy_(inp.kv_cache)
    padded = W.MlaInputs(inp.q, view, inp.block_table, inp.cache_seqlens, inp.seqlens,
                         inp.page_size, inp.num_heads_q, 512, False, inp.scale, inp.indices,
                         inp.topk)
    out_p, lse_p = run(padded, num_ctas=3)
    out_c, lse_c = run(inp, num_ctas=3)
    assert torch.equal(out_p, out_c) and torch.equal(lse_p, lse_c)
    check(inp, num_ctas=3)


@pytest.mark.parametrize("dtype,topk", [("e4m3", 256), ("bf16", 256), ("e4m3", 0), ("bf16", 0)])
def test_repeated_runs_are_bitwise_identical(dtype, topk):
    """The kernels are deterministic (fixed split, fixed order of every sum),
    so repeated runs must agree bit for bit; a race between the roles (a
    stage, an exchange buffer or the O accumulator read too early) shows up as
    a difference. 24 runs each without metadata and with 3 clusters; the first
    run is checked against the oracle."""
    inp = W.make_mla(seqlens=[20, 300, 3000], seqlen_q=2, num_heads_q=128, page_size=64,
                     topk=topk, dtype=dtype, seed=56, device="cuda")
    if topk:
        inp.indices[0, 1, 0, 5] = 19999
        inp.indices[2, 0, 0, 7] = -5
    for kw in (dict(use_meta=False), dict(num_ctas=3)):
        ref_o, ref_l = run(inp, **kw)
        for _ in range(23):
            o, l = run(inp, **kw)
            assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
    check(inp, num_ctas=3)
