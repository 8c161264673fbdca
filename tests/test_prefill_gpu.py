"""attn_fwd_varlen on the GPU against the fp64 oracle, element by element.

Tolerances: max-abs 1e-2 on bf16/fp16 outputs (N(0,1) inputs), 1e-3 on the
fp32 LSE, and the -inf pattern of the LSE must match exactly."""
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


def run_and_check(inp, atol=1e-2, with_lse=True):
    kw = dict(scale=inp.scale, causal=inp.causal, window=inp.window, sink=inp.sink,
              q_descale=inp.q_descale, k_descale=inp.k_descale, v_descale=inp.v_descale)
    if inp.varlen:
        kw.update(cu_seqlens_q=inp.cu_seqlens_q, cu_seqlens_k=inp.cu_seqlens_k,
                  max_seqlen_q=max(inp.seqlens_q), max_seqlen_k=max(inp.seqlens_k))
    out, lse = B.fwd_varlen(inp.q, inp.k, inp.v, **kw)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    q, k, v = to_f64(inp.q), to_f64(inp.k), to_f64(inp.v)
    sink = None if inp.sink is None else inp.sink.cpu().numpy()
    desc = {}
    if inp.q_descale is not None:
        desc = dict(q_descale=inp.q_descale.cpu().numpy(), k_descale=inp.k_descale.cpu().numpy(),
                    v_descale=inp.v_descale.cpu().numpy())
    if inp.varlen:
        ro, rl = oracle.attention_varlen(q, k, v, inp.cu_seqlens_q.cpu().numpy(),
                                         inp.cu_seqlens_k.cpu().numpy(), inp.scale, inp.causal,
                                         inp.window, sink, **desc)
    else:
        ro, rl = oracle.attention_padded(q, k, v, inp.scale, inp.causal, inp.window, sink, **desc)
    e_o = assert_close_out(to_f64(out), ro, atol)
    e_l = assert_close_lse(lse.cpu().numpy(), rl) if with_lse else 0.0
    return e_o, e_l


def test_tiny_dense_mha_full_config():
    # B=1, H=2, S=128, D=64, non-causal, scale 1/8: the whole workload.
    inp = W.build_config("tiny_dense_mha", seed=0, device="cuda")
    run_and_check(inp)


@pytest.mark.parametrize("D", [64, 128])
def test_varlen_causal_gqa_edge_lengths(D):
    lens = [1, 63, 64, 65, 127, 128, 129, 300]
    inp = W.make_prefill(seqlens_q=lens, num_heads_q=4, num_heads_kv=2, head_dim=D, varlen=True,
                         causal=True, seed=1, device="cuda")
    run_and_check(inp)


def test_padded_window_sink():
    inp = W.make_prefill(seqlens_q=[700] * 2, num_heads_q=4, num_heads_kv=4, head_dim=128,
                         varlen=False, causal=True, window=(100, 0), sink=True, seed=2,
                         device="cuda")
    run_and_check(inp)


@pytest.mark.parametrize("lq,lk", [([5, 130, 200], [300, 140, 200]), ([200, 33], [50, 1])])
def test_varlen_causal_unequal_lengths(lq, lk):
    # bottom-right alignment: L_k > L_q shifts the diagonal right; L_k < L_q
    # leaves the first L_q - L_k rows with no visible key (O = 0, LSE = -inf).
    inp = W.make_prefill(seqlens_q=lq, seqlens_k=lk, num_heads_q=2, num_heads_kv=1,
                         head_dim=128, varlen=True, causal=True, sink=False, seed=3,
                         device="cuda")
    run_and_check(inp)


def test_two_sided_window_and_window_wider_than_sequence():
    inp = W.make_prefill(seqlens_q=[333, 90], num_heads_q=2, num_heads_kv=2, head_dim=64,
                         varlen=True, causal=False, window=(64, 32), seed=4, device="cuda")
    run_and_check(inp)
    inp = W.make_prefill(seqlens_q=[200] * 2, num_heads_q=2, num_heads_kv=2, head_dim=128,
                         varlen=False, causal=True, window=(5000, 0), sink=True, seed=5,
                         device="cuda")
    run_and_check(inp)


def test_fp16_and_no_lse():
    inp = W.make_prefill(seqlens_q=[257] * 2, num_heads_q=4, num_heads_kv=1, head_dim=64,
                         varlen=False, causal=False, dtype="fp16", seed=6, device="cuda")
    run_and_check(inp)
    out, lse = B.fwd_varlen(inp.q, inp.k, inp.v, scale=inp.scale, lse=None)
    a, out2, _ = B.varlen_args(inp.q, inp.k, inp.v, scale=inp.scale)
    a.lse = None
    import ctypes
    assert B.lib().attn_fwd_varlen(ctypes.byref(a), B._stream(None)) == B.OK
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


def test_many_tiles_per_cta():
    # more work tiles than SMs: every CTA runs several tiles back to back
    inp = W.make_prefill(seqlens_q=[1024] * 2, num_heads_q=64, num_heads_kv=8, head_dim=128,
                         varlen=False, causal=True, seed=7, device="cuda")
    kw = dict(scale=inp.scale, causal=True)
    out, lse = B.fwd_varlen(inp.q, inp.k, inp.v, **kw)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    # check a sample of rows with the oracle
    rows = [(b, i, h) for b in range(2) for i in (0, 127, 128, 511, 1023) for h in (0, 9, 63)]
    ro, rl = oracle.attention_padded(to_f64(inp.q), to_f64(inp.k), to_f64(inp.v), inp.scale, True,
                                     rows=rows)
    o = to_f64(out)
    l = lse.cpu().numpy()
    for b, i, h in rows:
        assert_close_out(o[b, i, h], ro[b, i, h], 1e-2)
        assert abs(l[b, h, i] - rl[b, h, i]) <= 1e-3


# ---------------------------------------------------------------------------
# FP8 E4M3 inputs with fp32 descales (B, H_kv), bf16 output: max-abs 5e-2.
# ---------------------------------------------------------------------------

def test_fp8_padded_window_sink():
    inp = W.make_prefill(seqlens_q=[700] * 2, num_heads_q=4, num_heads_kv=2, head_dim=128,
                         varlen=False, causal=True, window=(100, 0), sink=True, dtype="e4m3",
                         seed=11, device="cuda")
    run_and_check(inp, atol=5e-2)


def test_fp8_varlen_causal_gqa_edge_lengths():
    lens = [1, 2, 63, 64, 65, 129, 300, 513]
    inp = W.make_prefill(seqlens_q=lens, num_heads_q=8, num_heads_kv=2, head_dim=128,
                         varlen=True, causal=True, dtype="e4m3", seed=12, device="cuda")
    run_and_check(inp, atol=5e-2)


@pytest.mark.parametrize("fmt", ["e5m2"])
def test_fp8_e5m2_padded_window_sink(fmt):
    # e5m2 inputs (MATE FMHA dtype list): S as an e5m2 MMA, V exactly to fp16.
    inp = W.make_prefill(seqlens_q=[700] * 2, num_heads_q=4, num_heads_kv=2, head_dim=128,
                         varlen=False, causal=True, window=(100, 0), sink=True, dtype=fmt,
                         seed=13, device="cuda")
    run_and_check(inp, atol=5e-2)


def test_fp8_e5m2_varlen_causal_gqa_edge_lengths():
    lens = [1, 2, 63, 64, 65, 129, 300, 513]
    inp = W.make_prefill(seqlens_q=lens, num_heads_q=8, num_heads_kv=2, head_dim=128,
                         varlen=True, causal=True, dtype="e5m2", seed=14, device="cuda")
    run_and_check(inp, atol=5e-2)


def test_fp8_full_size_window_sink_sampled():
    """The FP8 window + sink workload at full size (B=4, S=8192, H=32, D=128,
    window (1024, 0), sink, descales U[0.5, 2]); rows sampled for the oracle."""
    inp = W.build_config("window_sink_fp8", seed=0, device="cuda")
    out, lse = B.fwd_varlen(inp.q, inp.k, inp.v, scale=inp.scale, causal=True,
                            window=inp.window, sink=inp.sink, q_descale=inp.q_descale,
                            k_descale=inp.k_descale, v_descale=inp.v_descale)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    rows = [(b, i, h) for b in (0, 3) for i in (0, 1, 2, 700, 1024, 1025, 4095, 8191)
            for h in (0, 17, 31)]
    q, k, v = to_f64(inp.q), to_f64(inp.k), to_f64(inp.v)
    ro, rl = oracle.attention_padded(q, k, v, inp.scale, True, inp.window,
                                     inp.sink.cpu().numpy(), inp.q_descale.cpu().numpy(),
                                     inp.k_descale.cpu().numpy(), inp.v_descale.cpu().numpy(),
                                     rows=rows)
    o = to_f64(out)
    l = lse.cpu().numpy()
    for b, i, h in rows:
        assert_close_out(o[b, i, h], ro[b, i, h], 5e-2)
        assert abs(l[b, h, i] - rl[b, h, i]) <= 1e-3


# ---------------------------------------------------------------------------
# seqused (padded layout) and the additive score mask
# ---------------------------------------------------------------------------

def _padded_case(B, Sq, Sk, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Sq, Hq, D, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(B, Sk, Hkv, D, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, Sk, Hkv, D, generator=g).to(torch.bfloat16).cuda()
    return q, k, v


def test_padded_seqused_causal_window_gqa():
    """Padded q/k/v with seqused_q/k (CANN flash_attn seqused_q, seqused_kv):
    each sequence is its first seqused rows against its first seqused keys."""
    B, Sq, Sk, Hq, Hkv, D = 3, 300, 400, 4, 2, 128
    q, k, v = _padded_case(B, Sq, Sk, Hq, Hkv, D, 21)
    uq, uk = [300, 17, 129], [400, 5, 250]
    out = torch.zeros(B, Sq, Hq, D, dtype=torch.bfloat16, device="cuda")
    out, lse = B_fwd(q, k, v, scale=D ** -0.5, causal=True, window=(100, 0), out=out,
                     seqused_q=torch.tensor(uq, dtype=torch.int32, device="cuda"),
                     seqused_k=torch.tensor(uk, dtype=torch.int32, device="cuda"))
    ro, rl = oracle.attention_padded(to_f64(q), to_f64(k), to_f64(v), D ** -0.5, True, (100, 0),
                                     seqused_q=uq, seqused_k=uk)
    o = to_f64(out)
    for b in range(B):
        assert_close_out(o[b, :uq[b]], ro[b, :uq[b]], 1e-2)
        assert_close_lse(lse.cpu().numpy()[b, :, :uq[b]], rl[b, :, :uq[b]])
        assert np.all(o[b, uq[b]:] == 0), "rows past seqused_q are not written"


@pytest.mark.parametrize("D", [64, 128])
def test_additive_mask_padded(D):
    """Additive fp32 score mask (Mojo flash_attention_split_kv input_mask_fn)
    per (b, h, i, j), with -inf entries, on top of a causal mask; mask rows
    padded to a multiple of 4 floats."""
    B, S, Hq, Hkv = 2, 333, 4, 2
    q, k, v = _padded_case(B, S, S, Hq, Hkv, D, 22 + D)
    g = torch.Generator().manual_seed(7)
    store = torch.randn(B, Hq, S, 336, generator=g, dtype=torch.float32)
    store[torch.rand(B, Hq, S, 336, generator=g) < 0.1] = -float("inf")
    mask = store.cuda()[..., :S]
    out, lse = B_fwd(q, k, v, scale=D ** -0.5, causal=True, mask=mask)
    ro, rl = oracle.attention_padded(to_f64(q), to_f64(k), to_f64(v), D ** -0.5, True,
                                     mask=store[..., :S].double().numpy())
    assert_close_out(to_f64(out), ro, 1e-2)
    assert_close_lse(lse.cpu().numpy(), rl)


def test_additive_mask_varlen_broadcast_over_heads():
    """Varlen rows index the mask by position within the sequence; a size-1
    head axis broadcasts (stride 0)."""
    lens = [1, 70, 200, 129]
    inp = W.make_prefill(seqlens_q=lens, num_heads_q=4, num_heads_kv=1, head_dim=128, varlen=True,
                         causal=False, seed=23, device="cuda")
    L = max(lens)
    g = torch.Generator().manual_seed(8)
    store = torch.randn(len(lens), 1, L, 200, generator=g, dtype=torch.float32) * 2
    mask = store.cuda()
    out, lse = B.fwd_varlen(inp.q, inp.k, inp.v, scale=inp.scale, cu_seqlens_q=inp.cu_seqlens_q,
                            cu_seqlens_k=inp.cu_seqlens_k, max_seqlen_q=L, max_seqlen_k=L,
                            mask=mask)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    ro, rl = oracle.attention_varlen(to_f64(inp.q), to_f64(inp.k), to_f64(inp.v),
                                     inp.cu_seqlens_q.cpu().numpy(), inp.cu_seqlens_k.cpu().numpy(),
                                     inp.scale, mask=store.double().numpy())
    assert_close_out(to_f64(out), ro, 1e-2)
    assert_close_lse(lse.cpu().numpy(), rl)


def B_fwd(q, k, v, **kw):
    out, lse = B.fwd_varlen(q, k, v, **kw)
    torch.cuda.synchronize()
    assert B.device_error() == 0
    return out, lse


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_repeated_runs_are_bitwise_identical(dtype):
    """Each work unit is computed by one CTA in a fixed order, whichever CTA
    takes it from the counter, so repeated runs agree bit for bit; a race
    between the roles shows up as a difference. 16 runs of a varlen causal
    GQA batch with more units than SMs."""
    lens = W.uniform_lengths(10, 300, 1500, seed=91)
    inp = W.make_prefill(seqlens_q=lens, num_heads_q=16, num_heads_kv=4, head_dim=128,
                         varlen=True, causal=True, dtype=dtype, seed=92, device="cuda")
    kw = dict(scale=inp.scale, causal=True, cu_seqlens_q=inp.cu_seqlens_q,
              cu_seqlens_k=inp.cu_seqlens_k, max_seqlen_q=max(lens), max_seqlen_k=max(lens),
              q_descale=inp.q_descale, k_descale=inp.k_descale, v_descale=inp.v_descale)
    ref_o, ref_l = B_fwd(inp.q, inp.k, inp.v, **kw)
    for _ in range(15):
        o, l = B_fwd(inp.q, inp.k, inp.v, **kw)
        assert torch.equal(o, ref_o) and torch.equal(l, ref_l)


def test_strided_output_view():
    """Output written through a strided view (padding after every head's D
    values and a padding head after every row): equal bit for bit to the
    packed output, and the padding is untouched. Whole 128-row tiles go out
    by TMA store through a tensor map of the view's strides, ragged tiles by
    direct stores; both must follow the strides."""
    lens = [300, 128, 513]
    inp = W.make_prefill(seqlens_q=lens, num_heads_q=8, num_heads_kv=2, head_dim=128,
                         varlen=True, causal=True, seed=97, device="cuda")
    kw = dict(scale=inp.scale, causal=True, cu_seqlens_q=inp.cu_seqlens_q,
              cu_seqlens_k=inp.cu_seqlens_k, max_seqlen_q=max(lens), max_seqlen_k=max(lens))
    ref_o, ref_l = B_fwd(inp.q, inp.k, inp.v, **kw)
    T = inp.q.shape[0]
    big = torch.full((T, 9, 192), float("nan"), dtype=torch.bfloat16, device="cuda")
    view = big[:, :8, :128]
    o, l = B_fwd(inp.q, inp.k, inp.v, out=view, **kw)
    torch.cuda.synchronize()
    assert torch.equal(view, ref_o) and torch.equal(l, ref_l)
    assert torch.isnan(big[:, :8, 128:]).all() and torch.isnan(big[:, 8:, :]).all()
