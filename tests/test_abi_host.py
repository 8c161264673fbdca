"""The C ABI on the host: the library builds and loads, exports every symbol
the header declares, the ctypes mirrors match the C structs, and bad
host-visible arguments are rejected before anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest

from attention_online_softmax_fmha_b200 import binding as B
from attention_online_softmax_fmha_b200 import build as BUILD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "libattn.h")


@pytest.fixture(scope="module")
def L():
    BUILD.build()
    return B.lib()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(\w+)\s*\(", src, flags=re.M)))


def test_every_declared_function_is_exported(L):
    names = header_functions()
    assert "attn_fwd_varlen" in names and "mla_sparse_fwd" in names
    assert set(B.EXPORTS) <= set(names)
    nm = subprocess.run(["nm", "-D", "--defined-only", BUILD.LIB], capture_output=True, text=True)
    exported = set(re.findall(r" T (\w+)$", nm.stdout, flags=re.M))
    for n in names:
        assert n in exported, n
        assert hasattr(L, n)


def test_enum_values_match_the_header():
    """The binding's status, device-error and scheduler-mode constants are the
    header's enum values."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    vals = {k: int(v) for k, v in re.findall(r"\b(ATTN_\w+)\s*=\s*(\d+)", src)}
    pairs = {"ATTN_OK": B.OK, "ATTN_ERR_DEVICE": B.DEVICE_ERROR,
             "ATTN_DEVERR_TIMEOUT": B.DEVERR_TIMEOUT,
             "ATTN_DEVERR_META_MISMATCH": B.DEVERR_META_MISMATCH,
             "ATTN_DEVERR_SMEM_ALIGN": B.DEVERR_SMEM_ALIGN,
             "ATTN_DEVERR_UNITS_OVERFLOW": B.DEVERR_UNITS_OVERFLOW,
             "ATTN_SCHED_MHA": B.SCHED_MHA, "ATTN_SELFTEST_SITE": B.SELFTEST_SITE}
    for name, value in pairs.items():
        assert vals[name] == value, name


def test_struct_mirrors_match(L):
    for which, cls in B.ARG_STRUCTS.items():
        assert L.attn_args_sizeof(which) == ctypes.sizeof(cls), cls.__name__


def test_status_strings(L):
    assert B.status_str(B.OK) == "ok"
    assert "invalid" in B.status_str(B.INVALID_ARG)


def _varlen(**over):
    a = B.VarlenArgs()
    base = dict(q=0x1000, k=0x2000, v=0x3000, out=0x4000, batch=2, max_seqlen_q=128,
                max_seqlen_k=128, num_heads_q=8, num_heads_kv=2, head_dim_qk=128,
                head_dim_v=128, q_stride_b=128 * 8 * 128, q_stride_s=8 * 128, q_stride_h=128,
                k_stride_b=128 * 2 * 128, k_stride_s=2 * 128, k_stride_h=128,
                v_stride_b=128 * 2 * 128, v_stride_s=2 * 128, v_stride_h=128,
                o_stride_b=128 * 8 * 128, o_stride_s=8 * 128, o_stride_h=128,
                lse_stride_b=8 * 128, lse_stride_h=128, dtype=B.DTYPE_BF16, scale=0.08,
                window_left=-1, window_right=-1)
    base.update(over)
    for k, v in base.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,want", [
    (dict(q=None), B.INVALID_ARG),
    (dict(batch=0), B.INVALID_ARG),                 # empty tensor (zero-size axis)
    (dict(max_seqlen_q=0), B.INVALID_ARG),
    (dict(num_heads_kv=3), B.INVALID_ARG),          # H_q % H_kv != 0
    (dict(scale=-1.0), B.INVALID_ARG),
    (dict(scale=float("nan")), B.INVALID_ARG),
    (dict(window_left=-2), B.INVALID_ARG),
    (dict(q=0x1008), B.INVALID_ARG),                # not 16-byte aligned
    (dict(q_stride_s=8 * 128 + 1), B.INVALID_ARG),  # row start not 16-byte aligned
    (dict(dtype=9), B.INVALID_ARG),
    (dict(dtype=B.DTYPE_E4M3), B.INVALID_ARG),      # FP8 without descales
    (dict(dtype=B.DTYPE_E5M2, q_descale=8, k_descale=8, v_descale=8, head_dim_qk=64,
          head_dim_v=64), B.UNSUPPORTED),            # FP8 is built for D = 128
    (dict(head_dim_qk=96, head_dim_v=96), B.UNSUPPORTED),
    (dict(head_dim_v=64), B.UNSUPPORTED),
    (dict(cu_seqlens_q=0x5000), B.INVALID_ARG),     # cu_seqlens_k missing
    (dict(cu_seqlens_q=0x5000, cu_seqlens_k=0x6000, total_q=0, total_k=5), B.INVALID_ARG),
])
def test_varlen_rejects_bad_arguments(L, over, want):
    a = _varlen(**over)
    assert L.attn_fwd_varlen(ctypes.byref(a), None) == want


def _paged(**over):
    a = B.PagedArgs()
    base = dict(q=0x1000, k_cache=0x2000, v_cache=0x3000, block_table=0x4000,
                cache_seqlens=0x5000, out=0x6000, batch=2, seqlen_q=1, num_heads_q=8,
                num_heads_kv=2, head_dim=128, page_size=64, num_blocks=16, max_pages_per_seq=8,
                block_table_stride=8, q_stride_b=8 * 128, q_stride_s=8 * 128, q_stride_h=128,
                kc_stride_blk=64 * 2 * 128, kc_stride_tok=2 * 128, kc_stride_h=128,
                vc_stride_blk=64 * 2 * 128, vc_stride_tok=2 * 128, vc_stride_h=128,
                o_stride_b=8 * 128, o_stride_s=8 * 128, o_stride_h=128, dtype=B.DTYPE_BF16,
                scale=0.1, window_left=-1, window_right=-1)
    base.update(over)
    for k, v in base.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("over,want", [
    (dict(k_cache=None), B.INVALID_ARG),
    (dict(num_heads_kv=3), B.INVALID_ARG),
    (dict(block_table_stride=4), B.INVALID_ARG),    # shorter than a table row
    (dict(dtype=B.DTYPE_E4M3), B.INVALID_ARG),      # FP8 without descales
    (dict(dtype=B.DTYPE_E5M2, q_descale=8, k_descale=8), B.INVALID_ARG),
    (dict(dtype=B.DTYPE_E4M3, q_descale=8, k_descale=8, v_descale=8, head_dim=64),
     B.UNSUPPORTED),                                # FP8 is built for D = 128
    (dict(head_dim=96), B.UNSUPPORTED),
    (dict(page_size=8), B.UNSUPPORTED),
    (dict(k_new=0x7000, seqlen_new=2, kn_stride_b=2 * 256, kn_stride_s=256, kn_stride_h=128),
     B.INVALID_ARG),                                # v_new missing
    (dict(seqlen_new=2), B.INVALID_ARG),            # seqlen_new without k_new / v_new
    (dict(k_new=0x7000, v_new=0x8000, seqlen_new=0, kn_stride_b=256, kn_stride_s=256,
          kn_stride_h=128, vn_stride_b=256, vn_stride_s=256, vn_stride_h=128), B.INVALID_ARG),
])
def test_paged_rejects_bad_arguments(L, over, want):
    a = _paged(**over)
    assert L.attn_fwd_paged_kvcache(ctypes.byref(a), None) == want


def test_sched_rejects_appended_keys_outside_gqa_decode(L):
    a = B.SchedArgs(0x1000, 2, 1, 128, 1, 576, 512, 64, B.SCHED_MLA, 0, 0, 0x2000, 1 << 20, 0, 4)
    assert L.attn_sched_metadata(ctypes.byref(a), None) == B.INVALID_ARG
    a.mode, a.num_heads_kv, a.num_heads_q, a.head_dim_qk, a.head_dim_v = B.SCHED_MHA, 2, 8, 128, 128
    a.seqlen_new = -1
    assert L.attn_sched_metadata(ctypes.byref(a), None) == B.INVALID_ARG


def test_mla_packed_queries_are_sparse_only(L):
    a = B.MlaArgs()
    base = dict(q=0x1000, kv_cache=0x2000, block_table=0x3000, cache_seqlens=0x4000,
                out=0x5000, batch=2, seqlen_q=9, num_heads_q=128, num_heads_kv=1,
                head_dim_qk=576, head_dim_v=512, page_size=64, num_blocks=8,
                max_pages_per_seq=4, block_table_stride=4, q_stride_s=128 * 576,
                q_stride_h=576, kv_stride_blk=64 * 576, kv_stride_tok=576,
                o_stride_s=128 * 512, o_stride_h=512, scale=0.04, cu_seqlens_q=0x6000)
    for k, v in base.items():
        setattr(a, k, v)
    assert L.mla_fwd_paged(ctypes.byref(a), None) == B.UNSUPPORTED  # dense: BSND only


def test_null_struct_is_invalid(L):
    for fn in ["attn_fwd_varlen", "attn_sched_metadata", "attn_fwd_paged_kvcache",
               "attn_combine", "mla_fwd_paged", "mla_sparse_fwd"]:
        assert getattr(L, fn)(None, None) == B.INVALID_ARG, fn
