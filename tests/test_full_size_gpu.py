"""The benchmarked workloads at full size, launched exactly as bench.py times
them (its workload builders and its step function on a side stream), with
sampled output rows checked against the fp64 oracle element by element.

Also a varlen causal GQA case with far more work units than SMs, so that
every CTA runs several varlen units back to back, checked on every row.

Tolerances as elsewhere: max-abs 1e-2 on bf16 O (5e-2 for FP8 inputs), 1e-3
on the fp32 LSE, and an identical -inf pattern."""
import numpy as np
import pytest
import torch

import bench
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


def run_benched(name):
    wl = bench.WORKLOADS[name](name, 0, torch.device("cuda", torch.cuda.current_device()))
    stream = torch.cuda.Stream()
    wl["step"](stream)
    stream.synchronize()
    assert B.device_error(stream) == 0
    return wl


def _check_rows(out, lse, ro, rl, rows, atol, varlen, cu=None):
    """Compare the sampled (b, i, h) rows; out/lse in the library's layout."""
    o = out
    for b, i, h in rows:
        if varlen:
            t = int(cu[b]) + i
            got_o, want_o = o[t, h], ro[t, h]
            got_l, want_l = lse[h, t], rl[h, t]
        else:
            got_o, want_o = o[b, i, h], ro[b, i, h]
            got_l, want_l = lse[b, h, i], rl[b, h, i]
        assert_close_out(got_o, want_o, atol, what=f"out[b={b}, i={i}, h={h}]")
        assert_close_lse(np.array([got_l]), np.array([want_l]), what=f"lse[b={b}, i={i}, h={h}]")


def test_varlen_causal_gqa_as_benched():
    """8 sequences with lengths U[512, 4096], H_q=32, H_kv=8, D=128, causal:
    rows 0, 127, 128, 255, 256 and the last row of the longest and shortest
    sequence, every KV-head group, plus middle and last rows of every
    sequence."""
    wl = run_benched("varlen_causal_gqa")
    inp = wl["inp"]
    out, lse = wl["outputs"]
    lens = inp.seqlens_q
    order = np.argsort(lens)
    heads = [g * 4 + (g % 4) for g in range(8)] + [1, 30]
    rows = set()
    for b in (int(order[0]), int(order[-1])):
        for i in (0, 127, 128, 255, 256, lens[b] - 1):
            for h in heads:
                rows.add((b, i, h))
    for b in range(len(lens)):
        for i in (lens[b] // 2, lens[b] - 1, lens[b] - 129):
            rows.add((b, i, 5))
    rows = sorted(rows)
    cu = inp.cu_seqlens_q.cpu().numpy()
    ro, rl = oracle.attention_varlen(to_f64(inp.q), to_f64(inp.k), to_f64(inp.v), cu,
                                     inp.cu_seqlens_k.cpu().numpy(), inp.scale, True, rows=rows)
    _check_rows(to_f64(out), lse.cpu().numpy(), ro, rl, rows, 1e-2, True, cu)


def _window_rows():
    # rows before, at and across the 1024-key window edge, tile edges, the end
    return (0, 1, 127, 128, 255, 256, 1000, 1023, 1024, 1025, 1100, 1151, 1152, 1153, 2047,
            2048, 4095, 6000, 8191)


def test_window_sink_bf16_as_benched():
    """B=4, S=8192, H=32, D=128, causal with window (1024, 0) and a per-head
    sink: rows across the window edge in two sequences, all 32 heads of the
    last row."""
    wl = run_benched("window_sink")
    inp = wl["inp"]
    out, lse = wl["outputs"]
    rows = {(b, i, h) for b in (0, 3) for i in _window_rows() for h in (0, 13, 31)}
    rows |= {(1, 8191, h) for h in range(32)}
    rows |= {(2, 5000, h) for h in range(0, 32, 3)}
    rows = sorted(rows)
    bsel = sorted({b for b, _, _ in rows})
    # decode only the sequences sampled (the full f64 copy would be 3 GB)
    sub = {b: n for n, b in enumerate(bsel)}
    q, k, v = (to_f64(t[bsel]) for t in (inp.q, inp.k, inp.v))
    srows = [(sub[b], i, h) for b, i, h in rows]
    ro, rl = oracle.attention_padded(q, k, v, inp.scale, True, inp.window, inp.sink.cpu().numpy(),
                                     rows=srows)
    o = to_f64(out[bsel])
    l = lse[bsel].cpu().numpy()
    _check_rows(o, l, ro, rl, srows, 1e-2, False)


def test_window_sink_fp8_as_benched():
    """The FP8 e4m3 run of the same shapes with (B, H_kv) descales."""
    wl = run_benched("window_sink_fp8")
    inp = wl["inp"]
    out, lse = wl["outputs"]
    rows = sorted({(b, i, h) for b in (0, 2) for i in _window_rows() for h in (0, 21)})
    bsel = sorted({b for b, _, _ in rows})
    sub = {b: n for n, b in enumerate(bsel)}
    q, k, v = (to_f64(t[bsel]) for t in (inp.q, inp.k, inp.v))
    dq, dk, dv = (t[bsel].cpu().numpy() for t in (inp.q_descale, inp.k_descale, inp.v_descale))
    srows = [(sub[b], i, h) for b, i, h in rows]
    ro, rl = oracle.attention_padded(q, k, v, inp.scale, True, inp.window, inp.sink.cpu().numpy(),
                                     dq, dk, dv, rows=srows)
    _check_rows(to_f64(out[bsel]), lse[bsel].cpu().numpy(), ro, rl, srows, 5e-2, False)


def test_paged_decode_fp8_as_benched():
    """The FP8 e4m3 paged decode (64 sequences, lengths U[1024, 32768], pages
    of 64, (B, H_kv) descales), metadata from the scheduler kernel; six
    sequences checked on every head."""
    wl = run_benched("paged_decode_fp8")
    inp = wl["inp"]
    out, lse = wl["outputs"]
    o = to_f64(out)
    l = lse.cpu().numpy()
    order = np.argsort(inp.seqlens)
    for b in [int(order[0]), int(order[-1]), 3, 17, 40, 63]:
        L = inp.seqlens[b]
        npg = -(-L // inp.page_size)
        pages = inp.block_table[b, :npg].long()
        kc = to_f64(inp.k_cache[pages])
        vc = to_f64(inp.v_cache[pages])
        ro, rl = oracle.attention_paged(to_f64(inp.q[b:b + 1]), kc, vc, np.arange(npg)[None], [L],
                                        inp.scale, q_descale=inp.q_descale[b:b + 1].cpu().numpy(),
                                        k_descale=inp.k_descale[b:b + 1].cpu().numpy(),
                                        v_descale=inp.v_descale[b:b + 1].cpu().numpy())
        assert_close_out(o[b:b + 1], ro, 5e-2)
        assert_close_lse(l[b:b + 1], rl)


def test_varlen_many_units_per_cta_every_row():
    """12 sequences of 600..2000 tokens, H_q=32, H_kv=8, D=128, causal: about
    1,900 work units on 148 SMs, so the K/V ring and the output hand-off carry
    on across varlen units inside each CTA. Every row of 16 heads (two per
    KV group) is checked."""
    lens = W.uniform_lengths(12, 600, 2000, seed=77)
    inp = W.make_prefill(seqlens_q=lens, num_heads_q=32, num_heads_kv=8, head_dim=128,
                         varlen=True, causal=True, seed=78, device="cuda")
    out, lse = B.fwd_varlen(inp.q, inp.k, inp.v, scale=inp.scale, causal=True,
                            cu_seqlens_q=inp.cu_seqlens_q, cu_seqlens_k=inp.cu_seqlens_k,
                            max_seqlen_q=max(lens), max_seqlen_k=max(lens))
    torch.cuda.synchronize()
    assert B.device_error() == 0
    heads = [h for g in range(8) for h in (4 * g + (g % 4), 4 * g + ((g + 2) % 4))]
    rows = [(b, i, h) for b in range(len(lens)) for i in range(lens[b]) for h in heads]
    cu = inp.cu_seqlens_q.cpu().numpy()
    ro, rl = oracle.attention_varlen(to_f64(inp.q), to_f64(inp.k), to_f64(inp.v), cu,
                                     inp.cu_seqlens_k.cpu().numpy(), inp.scale, True, rows=rows)
    o = to_f64(out)[:, heads]
    l = lse.cpu().numpy()[heads]
    assert_close_out(o, ro[:, heads], 1e-2)
    assert_close_lse(l, rl[heads])
