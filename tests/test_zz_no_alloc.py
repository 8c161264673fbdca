"""attn_fwd_paged_kvcache_static: the paged split-KV decode for callers that
cannot allocate device memory (it keeps the scheduler metadata and the split
partials in a buffer inside the library). Its output must match the regular
entry point's, within the tolerances the other tests use, on two calls in a
row (the shared buffer keeps the previous call's contents)."""
import ctypes

import pytest
import torch

from attention_online_softmax_fmha_b200 import binding as B
from attention_online_softmax_fmha_b200 import build as BUILD
from attention_online_softmax_fmha_b200 import workloads as W
from tests._util import assert_close_lse, assert_close_out, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.lib()


def _kw(inp):
    return dict(scale=inp.scale, causal=inp.causal, sink=inp.sink, q_descale=inp.q_descale,
                k_descale=inp.k_descale, v_descale=inp.v_descale, k_new=inp.k_new,
                v_new=inp.v_new)


def _regular(inp, num_ctas, stream=None):
    meta = B.sched_metadata(inp.cache_seqlens, batch=inp.batch, seqlen_q=inp.q.shape[1],
                            num_heads_q=inp.num_heads_q, num_heads_kv=inp.num_heads_kv,
                            head_dim_qk=inp.head_dim, head_dim_v=inp.head_dim,
                            page_size=inp.page_size, num_ctas=num_ctas,
                            seqlen_new=0 if inp.k_new is None else inp.k_new.shape[1],
                            stream=stream)
    return B.fwd_paged_kvcache(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                               inp.cache_seqlens, meta=meta, num_ctas=num_ctas, stream=stream,
                               **_kw(inp))


def _static(lib, inp, num_ctas, stream=None):
    a, out, lse, _ = B.paged_args(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                  inp.cache_seqlens, num_ctas=num_ctas, **_kw(inp))
    st = lib.attn_fwd_paged_kvcache_static(ctypes.byref(a), B._stream(stream))
    assert st == B.OK, B.status_str(st)
    return out, lse


def test_static_scratch_matches_regular_on_two_calls(lib):
    lens = [1, 0, 63, 64, 65, 700, 2000, 5000]
    first = W.make_paged(seqlens=lens, seqlen_q=1, num_heads_q=32, num_heads_kv=8, head_dim=128,
                         page_size=64, sink=True, seed=21, device="cuda")
    second = W.make_paged(seqlens=lens[::-1], seqlen_q=2, num_heads_q=16, num_heads_kv=4,
                          head_dim=128, page_size=32, causal=True, seed=22, device="cuda")
    for inp, num_ctas in ((first, 0), (second, 37)):
        ro, rl = _regular(inp, num_ctas)
        so, sl = _static(lib, inp, num_ctas)
        torch.cuda.synchronize()
        assert B.device_error() == 0
        assert_close_out(to_f64(so), to_f64(ro), 1e-2)
        assert_close_lse(sl.cpu().numpy(), rl.cpu().numpy(), 1e-3)


def test_static_scratch_rejects_caller_buffers_and_oversized_problems(lib):
    inp = W.make_paged(seqlens=[100, 200], seqlen_q=1, num_heads_q=8, num_heads_kv=2,
                       head_dim=128, page_size=64, seed=23, device="cuda")
    a, _, _, _ = B.paged_args(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                              inp.cache_seqlens, scale=inp.scale)
    a.workspace = inp.q.data_ptr()  # a caller buffer is a usage error here
    assert lib.attn_fwd_paged_kvcache_static(ctypes.byref(a), B._stream(None)) == B.INVALID_ARG
    a.workspace = None
    a.batch = 1 << 20               # partials far beyond the built-in 16 MiB
    assert (lib.attn_fwd_paged_kvcache_static(ctypes.byref(a), B._stream(None))
            == B.WORKSPACE_TOO_SMALL)


@pytest.mark.parametrize("case", ["e4m3_descales", "appended_keys", "side_stream"])
def test_static_scratch_matches_regular_variants(lib, case):
    """The paths the static entry point forwards to the metadata and decode
    kernels: an FP8 cache with descales, three appended keys per sequence
    (the metadata counts their tile), and a call on a non-default stream."""
    lens = [0, 5, 64, 300, 3000]
    kw = dict(seqlen_q=2, num_heads_q=16, num_heads_kv=4, head_dim=128, page_size=64,
              causal=True, device="cuda")
    if case == "e4m3_descales":
        inp = W.make_paged(seqlens=lens, dtype="e4m3", sink=True, seed=24, **kw)
        atol = 5e-2
    elif case == "appended_keys":
        inp = W.make_paged(seqlens=lens, seqlen_new=3, seed=25, **kw)
        atol = 1e-2
    else:
        inp = W.make_paged(seqlens=lens, seed=26, **kw)
        atol = 1e-2
    stream = torch.cuda.Stream() if case == "side_stream" else None
    torch.cuda.synchronize()  # the inputs were written on the default stream
    for num_ctas in (0, 9):  # two calls in a row
        ro, rl = _regular(inp, num_ctas, stream)
        # the regular call's metadata and workspace are freed on return: let
        # its kernels finish before anything else is allocated
        torch.cuda.synchronize()
        so, sl = _static(lib, inp, num_ctas, stream)
        torch.cuda.synchronize()
        assert B.device_error() == 0
        assert_close_out(to_f64(so), to_f64(ro), atol)
        assert_close_lse(sl.cpu().numpy(), rl.cpu().numpy(), 1e-3)
