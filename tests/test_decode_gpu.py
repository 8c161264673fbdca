"""Paged-KV decode (attn_sched_metadata + attn_fwd_paged_kvcache, which runs
the split kernel and the combine) and attn_combine on the GPU, against the
fp64 oracle. bf16 outputs within 1e-2 max-abs, LSE within 1e-3; the
scheduler metadata is integer work and is checked exactly."""
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


def _np(t):
    return None if t is None else t.cpu().double().numpy()


def oracle_paged(inp, rows=None):
    kn = None if inp.k_new is None else to_f64(inp.k_new)
    vn = None if inp.v_new is None else to_f64(inp.v_new)
    return oracle.attention_paged(to_f64(inp.q), to_f64(inp.k_cache), to_f64(inp.v_cache),
                                  inp.block_table.cpu().numpy(), inp.seqlens, inp.scale,
                                  inp.causal, inp.window, _np(inp.sink), rows,
                                  _np(inp.q_descale), _np(inp.k_descale), _np(inp.v_descale),
                                  kn, vn)


def run_paged(inp, use_meta=True, num_ctas=0):
    meta = None
    if use_meta:
        meta = B.sched_metadata(inp.cache_seqlens, batch=inp.batch, seqlen_q=inp.q.shape[1],
                                num_heads_q=inp.num_heads_q, num_heads_kv=inp.num_heads_kv,
                                head_dim_qk=inp.head_dim, head_dim_v=inp.head_dim,
                                page_size=inp.page_size, num_ctas=num_ctas,
                                seqlen_new=0 if inp.k_new is None else inp.k_new.shape[1])
    out, lse = B.fwd_paged_kvcache(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                   inp.cache_seqlens, scale=inp.scale, causal=inp.causal,
                                   window=inp.window, sink=inp.sink, meta=meta,
                                   num_ctas=num_ctas, q_descale=inp.q_descale,
                                   k_descale=inp.k_descale, v_descale=inp.v_descale,
                                   k_new=inp.k_new, v_new=inp.v_new)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    return out, lse, meta


def check(inp, atol=1e-2, **kw):
    out, lse, _ = run_paged(inp, **kw)
    ro, rl = oracle_paged(inp)
    assert_close_out(to_f64(out), ro, atol)
    assert_close_lse(lse.cpu().numpy(), rl)


LENS = [1, 63, 64, 65, 700, 2000]


@pytest.mark.parametrize("num_ctas", [1, 3, 7, 0])
def test_split_counts(num_ctas):
    inp = W.make_paged(seqlens=LENS, seqlen_q=1, num_heads_q=8, num_heads_kv=2, head_dim=128,
                       page_size=64, seed=0, device="cuda")
    check(inp, num_ctas=num_ctas)


def test_no_metadata_one_cta_per_segment():
    inp = W.make_paged(seqlens=LENS, seqlen_q=1, num_heads_q=8, num_heads_kv=2, head_dim=128,
                       page_size=64, seed=1, device="cuda")
    check(inp, use_meta=False)


@pytest.mark.parametrize("page", [16, 32, 128, 256])
def test_page_sizes(page):
    inp = W.make_paged(seqlens=[5, 129, 300, 1000], seqlen_q=1, num_heads_q=4, num_heads_kv=4,
                       head_dim=64, page_size=page, seed=2, device="cuda")
    check(inp, num_ctas=5)


def test_multi_token_causal_window_sink_and_many_rows():
    # s_q = 4 with H_q / H_kv = 8: 32 rows per KV head -> two row blocks
    inp = W.make_paged(seqlens=[4, 90, 513], seqlen_q=4, num_heads_q=16, num_heads_kv=2,
                       head_dim=128, page_size=32, causal=True, window=(200, 0), sink=True,
                       seed=3, device="cuda")
    check(inp, num_ctas=6)


def test_aliased_block_table_and_empty_sequence():
    # every block_table entry 0 (the MATE MLA example's table), one empty cache
    inp = W.make_paged(seqlens=[32, 0, 100], seqlen_q=1, num_heads_q=4, num_heads_kv=1,
                       head_dim=128, page_size=16, table="aliased", seed=4, device="cuda")
    check(inp, num_ctas=4)
    check(inp, use_meta=False)


# FP8 caches (e4m3 / e5m2, D = 128) with fp32 descales (B, H_kv), bf16 out:
# max-abs 5e-2 (the FP8 bound), LSE 1e-3.
@pytest.mark.parametrize("dtype", ["e4m3", "e5m2"])
@pytest.mark.parametrize("page", [32, 64, 128])
def test_fp8_cache_split(dtype, page):
    inp = W.make_paged(seqlens=LENS, seqlen_q=1, num_heads_q=8, num_heads_kv=2, head_dim=128,
                       page_size=page, dtype=dtype, seed=20, device="cuda")
    assert inp.k_cache.dtype != torch.bfloat16 and inp.q_descale is not None
    check(inp, atol=5e-2, num_ctas=7)


def test_fp8_cache_multi_token_causal_window_sink_no_metadata():
    inp = W.make_paged(seqlens=[4, 90, 513, 0], seqlen_q=4, num_heads_q=16, num_heads_kv=2,
                       head_dim=128, page_size=16, causal=True, window=(200, 0), sink=True,
                       dtype="e4m3", seed=21, device="cuda")
    check(inp, atol=5e-2, num_ctas=6)
    check(inp, atol=5e-2, use_meta=False)


# Appended keys (k_new / v_new read after the cached keys, the cache left
# untouched), against the oracle on the concatenated sequence.
def test_append_new_tokens_causal_split_and_unsplit():
    inp = W.make_paged(seqlens=[0, 1, 63, 64, 65, 700], seqlen_q=3, num_heads_q=8,
                       num_heads_kv=2, head_dim=128, page_size=32, causal=True, seqlen_new=3,
                       seed=30, device="cuda")
    before = inp.k_cache.clone()
    check(inp, num_ctas=7)
    check(inp, use_meta=False)
    assert torch.equal(inp.k_cache, before)


def test_append_two_tiles_of_new_keys_window_d64():
    inp = W.make_paged(seqlens=[5, 129, 300], seqlen_q=1, num_heads_q=4, num_heads_kv=4,
                       head_dim=64, page_size=64, window=(100, 0), causal=True, seqlen_new=70,
                       seed=31, device="cuda")
    check(inp, num_ctas=5)


def test_append_fp8_with_sink():
    inp = W.make_paged(seqlens=[17, 400], seqlen_q=2, num_heads_q=8, num_heads_kv=2,
                       head_dim=128, page_size=64, causal=True, sink=True, seqlen_new=2,
                       dtype="e4m3", seed=32, device="cuda")
    check(inp, atol=5e-2, num_ctas=3)


def test_append_metadata_without_new_keys_is_reported():
    inp = W.make_paged(seqlens=[40, 90], seqlen_q=1, num_heads_q=4, num_heads_kv=1,
                       head_dim=128, page_size=32, seqlen_new=1, seed=33, device="cuda")
    meta = B.sched_metadata(inp.cache_seqlens, batch=2, seqlen_q=1, num_heads_q=4,
                            num_heads_kv=1, head_dim_qk=128, head_dim_v=128, page_size=32,
                            num_ctas=3)  # made for seqlen_new = 0
    B.fwd_paged_kvcache(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens,
                        scale=inp.scale, meta=meta, num_ctas=3, k_new=inp.k_new,
                        v_new=inp.v_new)
    torch.cuda.synchronize()
    assert B.device_error() & 0xff == B.DEVERR_META_MISMATCH
    assert B.device_error() == 0


@pytest.mark.parametrize("lens,G", [([0, 1, 64, 65, 4000, 12, 9000], 9),
                                    ([0, 1, 64, 65, 700, 12, 90], 148)])
def test_metadata_is_a_balanced_partition(lens, G):
    cs = torch.tensor(lens, dtype=torch.int32, device="cuda")
    H_kv = 2
    meta = B.sched_metadata(cs, batch=len(lens), seqlen_q=1, num_heads_q=8, num_heads_kv=H_kv,
                            head_dim_qk=128, head_dim_v=128, page_size=64, num_ctas=G)
    m = meta.cpu().numpy()
    S = len(lens) * H_kv
    assert m[0] == 0x4154544d and m[7] == G and m[8] == S
    off = 16
    cta_begin = m[off:off + G + 1]; off += G + 1
    cta_seg = m[off:off + G]; off += G
    seg_begin = m[off:off + S + 1]; off += S + 1
    first = m[off:off + S]; off += S
    nsplit = m[off:off + S]; off += S
    slot = m[off:off + S]
    units = [(-(-L // 64)) for L in lens for _ in range(H_kv)]
    assert list(np.diff(seg_begin)) == units and seg_begin[0] == 0
    total = sum(units)
    assert cta_begin[0] == 0 and cta_begin[-1] == total
    sizes = np.diff(cta_begin)
    assert sizes.min() >= 0 and sizes.max() - sizes.min() <= 1          # balanced
    busy = int((sizes > 0).sum())
    assert np.all(sizes[:busy] > 0) and np.all(sizes[busy:] == 0)       # idle CTAs last
    used = 0
    for s in range(S):
        touching = [c for c in range(G) if cta_begin[c] < seg_begin[s + 1] and
                    cta_begin[c + 1] > seg_begin[s]]
        assert nsplit[s] == len(touching)
        if touching:
            assert first[s] == touching[0]
        if nsplit[s] >= 2:
            assert slot[s] == used
            used += nsplit[s]
    assert m[13] == used
    for c in range(G):
        if cta_begin[c] < cta_begin[c + 1]:
            s = cta_seg[c]
            assert seg_begin[s] <= cta_begin[c] < seg_begin[s + 1]


def test_metadata_mismatch_is_reported():
    inp = W.make_paged(seqlens=[100, 200], seqlen_q=1, num_heads_q=4, num_heads_kv=2,
                       head_dim=128, page_size=64, seed=5, device="cuda")
    meta = B.sched_metadata(inp.cache_seqlens, batch=2, seqlen_q=1, num_heads_q=4,
                            num_heads_kv=2, head_dim_qk=128, head_dim_v=128, page_size=32,
                            num_ctas=3)   # page size differs from the main call
    B.fwd_paged_kvcache(inp.q, inp.k_cache, inp.v_cache, inp.block_table, inp.cache_seqlens,
                        scale=inp.scale, meta=meta, num_ctas=3)
    torch.cuda.synchronize()
    assert B.device_error() & 0xff == B.DEVERR_META_MISMATCH
    assert B.device_error() == 0


def test_full_size_paged_decode_sampled():
    """The paged decode workload at full size (64 sequences, lengths
    U[1024, 32768], H_q=32, H_kv=8, D=128, pages of 64, permuted table), in the
    launch configuration the benchmark times; rows of 6 sequences are checked
    against the oracle."""
    inp = W.build_config("paged_decode", seed=0, device="cuda")
    out, lse, _ = run_paged(inp)
    o = to_f64(out)
    l = lse.cpu().numpy()
    order = np.argsort(inp.seqlens)
    for b in [int(order[0]), int(order[-1]), 3, 17, 40, 63]:
        L = inp.seqlens[b]
        npg = -(-L // inp.page_size)
        pages = inp.block_table[b, :npg].long()
        kc = to_f64(inp.k_cache[pages])
        vc = to_f64(inp.v_cache[pages])
        q = to_f64(inp.q[b:b + 1])
        ro, rl = oracle.attention_paged(q, kc, vc, np.arange(npg)[None], [L], inp.scale)
        assert_close_out(o[b:b + 1], ro, 1e-2)
        assert_close_lse(l[b:b + 1], rl)


@pytest.mark.parametrize("with_counts", [False, True])
def test_combine_against_oracle(with_counts):
    g = torch.Generator().manual_seed(7)
    n, Bt, S, H, Dv = 5, 3, 2, 4, 128
    op = torch.randn(n, Bt, S, H, Dv, generator=g)
    lp = torch.randn(n, Bt, H, S, generator=g) * 3
    lp[1, 0] = -float("inf")          # an empty split
    lp[:, 2, 1] = -float("inf")       # a row with no key at all
    sink = torch.randn(H, generator=g)
    counts = torch.tensor([5, 2, 4], dtype=torch.int32) if with_counts else None
    out, lse = B.combine(op.cuda(), lp.cuda(), sink=sink.cuda(),
                         num_splits_per_seq=None if counts is None else counts.cuda())
    torch.cuda.synchronize()
    o = to_f64(out)
    l = lse.cpu().numpy()
    for b in range(Bt):
        k = n if counts is None else int(counts[b])
        ro, rl = oracle.combine(op[:k, b].double().numpy(),
                                lp[:k, b].double().numpy().transpose(0, 2, 1),
                                sink.double().numpy()[None, :])
        assert_close_out(o[b], ro, 1e-2)
        assert_close_lse(l[b], rl.T)


def test_unit_count_overflow_is_reported():
    """Sixteen sequences of 2^31 - 1 cached keys and eight KV heads: 128
    segments of 2^25 tiles each, 2^32 units in all, past the int32 prefix
    sums. Only the scheduler runs (it reads cache_seqlens alone); it leaves
    the header invalid and raises the overflow code."""
    lens = torch.full((16,), 2**31 - 1, dtype=torch.int32, device="cuda")
    meta = B.sched_metadata(lens, batch=16, seqlen_q=1, num_heads_q=8, num_heads_kv=8,
                            head_dim_qk=128, head_dim_v=128, page_size=64, num_ctas=5)
    torch.cuda.synchronize()
    word = B.device_error()
    assert word & 0xff == B.DEVERR_UNITS_OVERFLOW and word >> 8 == 50, hex(word)
    assert int(meta[0]) == 0  # no valid magic: a main call would refuse it
    # below the limit: seven sequences, 56 segments, 56 * 2^25 < 2^31
    meta = B.sched_metadata(lens[:7], batch=7, seqlen_q=1, num_heads_q=8, num_heads_kv=8,
                            head_dim_qk=128, head_dim_v=128, page_size=64, num_ctas=5)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    assert int(meta[0]) != 0


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_repeated_runs_are_bitwise_identical(dtype):
    """The split and every sum's order are fixed by the metadata, so repeated
    runs agree bit for bit; a race between the producer and the two consumer
    warpgroups shows up as a difference."""
    inp = W.make_paged(seqlens=[1, 63, 64, 65, 700, 3000, 9000], seqlen_q=1, num_heads_q=32,
                       num_heads_kv=8, head_dim=128, page_size=64, sink=True, dtype=dtype,
                       seed=93, device="cuda")
    ref_o, ref_l, _ = run_paged(inp, num_ctas=11)
    for _ in range(15):
        o, l, _ = run_paged(inp, num_ctas=11)
        assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
