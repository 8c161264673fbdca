"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies runs out, the kernel returns, the host reads the timeout from the
device error word, and the context stays usable (a prefill right after
still matches the oracle)."""
import time

import pytest
import torch

import oracle
from attention_online_softmax_fmha_b200 import binding as B
from attention_online_softmax_fmha_b200 import build as BUILD
from attention_online_softmax_fmha_b200 import workloads as W
from tests._util import assert_close_lse, assert_close_out, to_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_reports_the_timeout():
    BUILD.build()
    assert B.device_error() == 0
    t0 = time.perf_counter()
    B.selftest_wait_timeout()
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    word = B.device_error()
    assert word & 0xff == B.DEVERR_TIMEOUT and word >> 8 == B.SELFTEST_SITE, hex(word)
    assert B.device_error() == 0          # read and cleared
    assert 1.5 < elapsed < 30.0, elapsed  # the 2 s limit, then the kernel returned
    # the context is still usable
    inp = W.make_prefill(seqlens_q=[200], num_heads_q=2, num_heads_kv=2, head_dim=64,
                         varlen=False, causal=True, seed=50, device="cuda")
    out, lse = B.fwd_varlen(inp.q, inp.k, inp.v, scale=inp.scale, causal=True)
    torch.cuda.synchronize()
    ro, rl = oracle.attention_padded(to_f64(inp.q), to_f64(inp.k), to_f64(inp.v), inp.scale,
                                     causal=True)
    assert_close_out(to_f64(out), ro, 1e-2)
    assert_close_lse(lse.cpu().numpy(), rl)
