"""Thin Python binding of libattn (ctypes).

Argument marshalling only: torch tensors supply device pointers, shapes and
strides; every step of the computation runs in libattn's CUDA kernels. There
is no fallback: if libattn.so is missing or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")

c_i32, c_i64, c_f32, c_vp, c_sz = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                   ctypes.c_void_p, ctypes.c_size_t)

# status codes and enums (include/libattn.h)
OK, INVALID_ARG, UNSUPPORTED, WORKSPACE_TOO_SMALL, CUDA_ERROR, DEVICE_ERROR = range(6)
DTYPE_BF16, DTYPE_FP16, DTYPE_E4M3, DTYPE_E5M2, DTYPE_FP32 = range(5)
SCHED_MHA, SCHED_MLA, SCHED_MLA_SPARSE = range(3)
DEVERR_TIMEOUT, DEVERR_META_MISMATCH, DEVERR_SMEM_ALIGN, DEVERR_UNITS_OVERFLOW = 1, 2, 3, 4
SELFTEST_SITE = 200

_TORCH_DTYPE = {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_FP16,
                torch.float8_e4m3fn: DTYPE_E4M3, torch.float8_e5m2: DTYPE_E5M2}


class VarlenArgs(ctypes.Structure):
    _fields_ = [("q", c_vp), ("k", c_vp), ("v", c_vp), ("out", c_vp), ("lse", c_vp),
                ("cu_seqlens_q", c_vp), ("cu_seqlens_k", c_vp),
                ("batch", c_i32), ("max_seqlen_q", c_i32), ("max_seqlen_k", c_i32),
                ("total_q", c_i32), ("total_k", c_i32), ("num_heads_q", c_i32),
                ("num_heads_kv", c_i32), ("head_dim_qk", c_i32), ("head_dim_v", c_i32),
                ("q_stride_b", c_i64), ("q_stride_s", c_i64), ("q_stride_h", c_i64),
                ("k_stride_b", c_i64), ("k_stride_s", c_i64), ("k_stride_h", c_i64),
                ("v_stride_b", c_i64), ("v_stride_s", c_i64), ("v_stride_h", c_i64),
                ("o_stride_b", c_i64), ("o_stride_s", c_i64), ("o_stride_h", c_i64),
                ("lse_stride_b", c_i64), ("lse_stride_h", c_i64),
                ("dtype", c_i32), ("scale", c_f32), ("causal", c_i32),
                ("window_left", c_i32), ("window_right", c_i32),
                ("sink", c_vp), ("q_descale", c_vp), ("k_descale", c_vp), ("v_descale", c_vp),
                ("seqused_q", c_vp), ("seqused_k", c_vp), ("mask", c_vp),
                ("mask_stride_b", c_i64), ("mask_stride_h", c_i64), ("mask_stride_s", c_i64),
                ("work_counter", c_vp)]


class SchedArgs(ctypes.Structure):
    _fields_ = [("cache_seqlens", c_vp), ("batch", c_i32), ("seqlen_q", c_i32),
                ("num_heads_q", c_i32), ("num_heads_kv", c_i32), ("head_dim_qk", c_i32),
                ("head_dim_v", c_i32), ("page_size", c_i32), ("mode", c_i32), ("topk", c_i32),
                ("num_ctas", c_i32), ("meta", c_vp), ("meta_bytes", c_sz),
                ("sparse_block_size", c_i32), ("seqlen_new", c_i32)]


class PagedArgs(ctypes.Structure):
    _fields_ = [("q", c_vp), ("k_cache", c_vp), ("v_cache", c_vp), ("block_table", c_vp),
                ("cache_seqlens", c_vp), ("out", c_vp), ("lse", c_vp),
                ("batch", c_i32), ("seqlen_q", c_i32), ("num_heads_q", c_i32),
                ("num_heads_kv", c_i32), ("head_dim", c_i32), ("page_size", c_i32),
                ("num_blocks", c_i32), ("max_pages_per_seq", c_i32),
                ("block_table_stride", c_i64),
                ("q_stride_b", c_i64), ("q_stride_s", c_i64), ("q_stride_h", c_i64),
                ("kc_stride_blk", c_i64), ("kc_stride_tok", c_i64), ("kc_stride_h", c_i64),
                ("vc_stride_blk", c_i64), ("vc_stride_tok", c_i64), ("vc_stride_h", c_i64),
                ("o_stride_b", c_i64), ("o_stride_s", c_i64), ("o_stride_h", c_i64),
                ("dtype", c_i32), ("scale", c_f32), ("causal", c_i32),
                ("window_left", c_i32), ("window_right", c_i32), ("sink", c_vp),
                ("meta", c_vp), ("meta_bytes", c_sz), ("num_ctas", c_i32), ("workspace", c_vp),
                ("workspace_bytes", c_sz), ("q_descale", c_vp), ("k_descale", c_vp),
                ("v_descale", c_vp), ("k_new", c_vp), ("v_new", c_vp), ("seqlen_new", c_i32),
                ("kn_stride_b", c_i64), ("kn_stride_s", c_i64), ("kn_stride_h", c_i64),
                ("vn_stride_b", c_i64), ("vn_stride_s", c_i64), ("vn_stride_h", c_i64)]


class CombineArgs(ctypes.Structure):
    _fields_ = [("out_partial", c_vp), ("lse_partial", c_vp), ("out", c_vp), ("lse", c_vp),
                ("num_splits_per_seq", c_vp), ("sink", c_vp), ("num_splits", c_i32),
                ("batch", c_i32), ("seqlen_q", c_i32), ("num_heads", c_i32),
                ("head_dim_v", c_i32), ("o_stride_b", c_i64), ("o_stride_s", c_i64),
                ("o_stride_h", c_i64), ("out_dtype", c_i32)]


class MlaArgs(ctypes.Structure):
    _fields_ = [("q", c_vp), ("kv_cache", c_vp), ("block_table", c_vp), ("cache_seqlens", c_vp),
                ("indices", c_vp), ("out", c_vp), ("lse", c_vp),
                ("batch", c_i32), ("seqlen_q", c_i32), ("num_heads_q", c_i32),
                ("num_heads_kv", c_i32), ("head_dim_qk", c_i32), ("head_dim_v", c_i32),
                ("page_size", c_i32), ("num_blocks", c_i32), ("max_pages_per_seq", c_i32),
                ("topk", c_i32), ("block_table_stride", c_i64),
                ("q_stride_b", c_i64), ("q_stride_s", c_i64), ("q_stride_h", c_i64),
                ("kv_stride_blk", c_i64), ("kv_stride_tok", c_i64),
                ("o_stride_b", c_i64), ("o_stride_s", c_i64), ("o_stride_h", c_i64),
                ("idx_stride_b", c_i64), ("idx_stride_s", c_i64),
                ("scale", c_f32), ("causal", c_i32), ("meta", c_vp), ("meta_bytes", c_sz),
                ("num_ctas", c_i32), ("workspace", c_vp), ("workspace_bytes", c_sz),
                ("sparse_block_size", c_i32), ("kv_stride_h", c_i64), ("idx_stride_h", c_i64),
                ("cu_seqlens_q", c_vp), ("dtype", c_i32), ("q_descale", c_vp),
                ("k_descale", c_vp), ("v_descale", c_vp)]


ARG_STRUCTS = {0: VarlenArgs, 1: SchedArgs, 2: PagedArgs, 3: CombineArgs, 4: MlaArgs}

EXPORTS = ["attn_fwd_varlen", "attn_sched_metadata_size", "attn_sched_metadata",
           "attn_paged_workspace_size", "attn_fwd_paged_kvcache", "attn_combine",
           "mla_workspace_size", "mla_fwd_paged", "mla_sparse_fwd", "attn_get_device_error",
           "attn_status_str", "attn_args_sizeof", "attn_fwd_paged_kvcache_static",
           "attn_selftest_wait_timeout"]

_lib = None


class AttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_str(status)} (status {status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libattn.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"libattn.so not built at {LIB_PATH}; run "
                          "`python -m attention_online_softmax_fmha_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name in ["attn_fwd_varlen", "attn_sched_metadata", "attn_fwd_paged_kvcache",
                     "attn_combine", "mla_fwd_paged", "mla_sparse_fwd",
                     "attn_fwd_paged_kvcache_static"]:
            getattr(L, name).argtypes = [c_vp, c_vp]
            getattr(L, name).restype = c_i32
        for name in ["attn_sched_metadata_size"]:
            getattr(L, name).argtypes = [c_vp]
            getattr(L, name).restype = c_sz
        for name in ["attn_paged_workspace_size", "mla_workspace_size"]:
            getattr(L, name).argtypes = [c_vp]
            getattr(L, name).restype = c_sz
        L.attn_get_device_error.argtypes = [c_vp, c_vp]
        L.attn_get_device_error.restype = c_i32
        L.attn_status_str.argtypes = [c_i32]
        L.attn_status_str.restype = ctypes.c_char_p
        L.attn_args_sizeof.argtypes = [c_i32]
        L.attn_args_sizeof.restype = c_sz
        L.attn_selftest_wait_timeout.argtypes = [c_vp]
        L.attn_selftest_wait_timeout.restype = c_i32
        _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().attn_status_str(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _rows(**tensors):
    """The C structs carry element strides of the outer axes only: the last
    axis of every tensor must be contiguous."""
    for name, t in tensors.items():
        if t is not None and t.numel() > 1 and t.stride(-1) != 1:
            raise ValueError(f"{name}: the last axis must be contiguous (stride 1)")


def _dense(**tensors):
    """Tensors the C side indexes as plain contiguous arrays."""
    for name, t in tensors.items():
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def _same_dtype(q, **tensors):
    """The C structs carry one input dtype for q and every K/V operand."""
    for name, t in tensors.items():
        if t is not None and t.dtype != q.dtype:
            raise ValueError(f"{name}: dtype {t.dtype} differs from q's {q.dtype}")


def _int32(**tensors):
    for name, t in tensors.items():
        if t is not None and t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, status: int):
    if status != OK:
        raise AttnError(fn, status)


def _keep_for(stream, *tensors):
    """Buffers allocated here and used by work queued on another stream than
    torch's current one are released only after that work (record_stream)."""
    if stream is None or not hasattr(stream, "cuda_stream"):
        return
    for t in tensors:
        if t is not None and t is not False:
            t.record_stream(stream)


def device_error(stream=None) -> int:
    """Read and clear the device error word (synchronises the stream)."""
    code = c_i32(0)
    st = lib().attn_get_device_error(ctypes.byref(code), _stream(stream))
    if st not in (OK, DEVICE_ERROR):
        raise AttnError("attn_get_device_error", st)
    return code.value


def selftest_wait_timeout(stream=None):
    """Run the failure-detection self-test (attn_selftest_wait_timeout): a
    bounded wait that nothing satisfies runs out and reports
    DEVERR_TIMEOUT at SELFTEST_SITE. Read it with device_error()."""
    _check("attn_selftest_wait_timeout", lib().attn_selftest_wait_timeout(_stream(stream)))


def out_dtype_for(dtype: torch.dtype) -> torch.dtype:
    """FP8 and bf16 inputs give bf16 outputs; fp16 gives fp16."""
    return torch.float16 if dtype == torch.float16 else torch.bfloat16


# ---------------------------------------------------------------------------
# attn_fwd_varlen
# ---------------------------------------------------------------------------

def varlen_args(q, k, v, *, cu_seqlens_q=None, cu_seqlens_k=None, max_seqlen_q=None,
                max_seqlen_k=None, scale=None, causal=False, window=(-1, -1), sink=None,
                q_descale=None, k_descale=None, v_descale=None, out=None, lse=None,
                seqused_q=None, seqused_k=None, mask=None, work_counter=None):
    """Build the argument struct (and allocate out/lse if not given).

    mask: fp32 tensor indexed [b, h, i, j] (a 4-D view; size-1 axes broadcast
    with stride 0); seqused_q/k: int32 (B,) for the padded layout.
    work_counter: an int32 tensor of one element for the dynamic unit
    schedule (allocated here if not given; kept alive by the struct); False:
    the static schedule."""
    varlen = cu_seqlens_q is not None
    _rows(q=q, k=k, v=v, out=out, lse=lse)
    _same_dtype(q, k=k, v=v)
    _dense(cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k, seqused_q=seqused_q,
           seqused_k=seqused_k, sink=sink, q_descale=q_descale, k_descale=k_descale,
           v_descale=v_descale)
    _int32(cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k, seqused_q=seqused_q,
           seqused_k=seqused_k)
    Hq, D = q.shape[-2], q.shape[-1]
    Hkv, Dv = k.shape[-2], v.shape[-1]
    if varlen:
        B = cu_seqlens_q.numel() - 1
        assert max_seqlen_q is not None and max_seqlen_k is not None, "varlen needs max lengths"
        if out is None:
            out = torch.empty(q.shape[0], Hq, Dv, device=q.device, dtype=out_dtype_for(q.dtype))
        if lse is None:
            lse = torch.empty(Hq, q.shape[0], device=q.device, dtype=torch.float32)
        qsb = ksb = vsb = osb = 0
        qss, qsh = q.stride(0), q.stride(1)
        kss, ksh = k.stride(0), k.stride(1)
        vss, vsh = v.stride(0), v.stride(1)
        oss, osh = out.stride(0), out.stride(1)
        lsb, lsh = 0, lse.stride(0)
        sq, sk = int(max_seqlen_q), int(max_seqlen_k)
    else:
        B, sq, sk = q.shape[0], q.shape[1], k.shape[1]
        if out is None:
            out = torch.empty(B, sq, Hq, Dv, device=q.device, dtype=out_dtype_for(q.dtype))
        if lse is None:
            lse = torch.empty(B, Hq, sq, device=q.device, dtype=torch.float32)
        qsb, qss, qsh = q.stride(0), q.stride(1), q.stride(2)
        ksb, kss, ksh = k.stride(0), k.stride(1), k.stride(2)
        vsb, vss, vsh = v.stride(0), v.stride(1), v.stride(2)
        osb, oss, osh = out.stride(0), out.stride(1), out.stride(2)
        lsb, lsh = lse.stride(0), lse.stride(1)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    msb = msh = mss = 0
    if mask is not None:
        assert mask.dim() == 4 and mask.dtype == torch.float32, "mask: fp32 [b, h, i, j]"
        assert mask.stride(3) == 1, "mask rows must be contiguous"
        msb, msh, mss = (mask.stride(d) if mask.shape[d] > 1 else 0 for d in range(3))
    a = VarlenArgs(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
        B, sq, sk, q.shape[0] if varlen else 0, k.shape[0] if varlen else 0, Hq, Hkv, D, Dv,
        qsb, qss, qsh, ksb, kss, ksh, vsb, vss, vsh, osb, oss, osh, lsb, lsh,
        _TORCH_DTYPE.get(q.dtype, -1), float(scale), int(bool(causal)), int(window[0]),
        int(window[1]), _ptr(sink), _ptr(q_descale), _ptr(k_descale), _ptr(v_descale),
        _ptr(seqused_q), _ptr(seqused_k), _ptr(mask), msb, msh, mss)
    if work_counter is None:
        work_counter = torch.empty(1, dtype=torch.int32, device=q.device)
    if work_counter is not False:
        _int32(work_counter=work_counter)
        a.work_counter = work_counter.data_ptr()
        a._keep = work_counter  # the struct holds its address
    return a, out, lse


def fwd_varlen(q, k, v, *, stream=None, **kw):
    """Attention forward (attn_fwd_varlen). Returns (out, lse)."""
    a, out, lse = varlen_args(q, k, v, **kw)
    _check("attn_fwd_varlen", lib().attn_fwd_varlen(ctypes.byref(a), _stream(stream)))
    _keep_for(stream, getattr(a, "_keep", None))
    return out, lse


# ---------------------------------------------------------------------------
# attn_sched_metadata
# ---------------------------------------------------------------------------

def sched_args(cache_seqlens, *, batch, seqlen_q, num_heads_q, num_heads_kv, head_dim_qk,
               head_dim_v, page_size, mode=SCHED_MHA, topk=0, num_ctas=0, sparse_block_size=0,
               seqlen_new=0):
    return SchedArgs(_ptr(cache_seqlens), batch, seqlen_q, num_heads_q, num_heads_kv, head_dim_qk,
                     head_dim_v, page_size, mode, topk, num_ctas, None, 0, sparse_block_size,
                     seqlen_new)


def sched_metadata_size(a: SchedArgs) -> int:
    return int(lib().attn_sched_metadata_size(ctypes.byref(a)))


def sched_metadata(cache_seqlens, *, stream=None, meta=None, **kw) -> torch.Tensor:
    """Scheduler metadata (attn_sched_metadata); returns the int32 buffer."""
    a = sched_args(cache_seqlens, **kw)
    nbytes = sched_metadata_size(a)
    if nbytes == 0:
        raise AttnError("attn_sched_metadata_size", INVALID_ARG)
    if meta is None:
        meta = torch.empty(nbytes // 4, dtype=torch.int32, device=cache_seqlens.device)
    a.meta = meta.data_ptr()
    a.meta_bytes = meta.numel() * 4
    _check("attn_sched_metadata", lib().attn_sched_metadata(ctypes.byref(a), _stream(stream)))
    return meta


# ---------------------------------------------------------------------------
# attn_fwd_paged_kvcache
# ---------------------------------------------------------------------------

def paged_args(q, k_cache, v_cache, block_table, cache_seqlens, *, scale=None, causal=False,
               window=(-1, -1), sink=None, meta=None, num_ctas=0, workspace=None, out=None,
               lse=None, q_descale=None, k_descale=None, v_descale=None, k_new=None,
               v_new=None):
    """FP8 (float8_e4m3fn / float8_e5m2 q and caches, D = 128) takes
    q/k/v_descale as contiguous fp32 (B, H_kv) device tensors. k_new, v_new
    (B, s_new, H_kv, D) are keys read after each sequence's cached ones (the
    metadata must then be made with seqlen_new=s_new)."""
    _rows(q=q, k_cache=k_cache, v_cache=v_cache, out=out, block_table=block_table, k_new=k_new,
          v_new=v_new)
    _same_dtype(q, k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new)
    _dense(cache_seqlens=cache_seqlens, lse=lse, sink=sink, q_descale=q_descale,
           k_descale=k_descale, v_descale=v_descale)
    _int32(block_table=block_table, cache_seqlens=cache_seqlens)
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    B, sq, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    if out is None:
        out = torch.empty(B, sq, Hq, D, device=q.device, dtype=out_dtype_for(q.dtype))
    if lse is None:
        lse = torch.empty(B, Hq, sq, device=q.device, dtype=torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    a = PagedArgs(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(cache_seqlens), _ptr(out),
        _ptr(lse), B, sq, Hq, Hkv, D, k_cache.shape[1], k_cache.shape[0], block_table.shape[1],
        block_table.stride(0), q.stride(0), q.stride(1), q.stride(2), k_cache.stride(0),
        k_cache.stride(1), k_cache.stride(2), v_cache.stride(0), v_cache.stride(1),
        v_cache.stride(2), out.stride(0), out.stride(1), out.stride(2),
        _TORCH_DTYPE.get(q.dtype, -1), float(scale), int(bool(causal)), int(window[0]),
        int(window[1]), _ptr(sink), _ptr(meta), 0 if meta is None else meta.numel() * 4,
        int(num_ctas), None, 0, _ptr(q_descale), _ptr(k_descale), _ptr(v_descale),
        _ptr(k_new), _ptr(v_new), 0 if k_new is None else k_new.shape[1],
        *((0, 0, 0) if k_new is None else k_new.stride()[:3]),
        *((0, 0, 0) if v_new is None else v_new.stride()[:3]))
    if meta is not None:
        nbytes = int(lib().attn_paged_workspace_size(ctypes.byref(a)))
        if workspace is None:
            workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel()
    return a, out, lse, workspace


def fwd_paged_kvcache(q, k_cache, v_cache, block_table, cache_seqlens, *, stream=None, **kw):
    """Paged-KV decode (attn_fwd_paged_kvcache, combine included). Returns (out, lse)."""
    a, out, lse, ws = paged_args(q, k_cache, v_cache, block_table, cache_seqlens, **kw)
    _check("attn_fwd_paged_kvcache", lib().attn_fwd_paged_kvcache(ctypes.byref(a),
                                                                 _stream(stream)))
    _keep_for(stream, ws)
    return out, lse


def fwd_paged_kvcache_static(q, k_cache, v_cache, block_table, cache_seqlens, *, stream=None,
                             num_ctas=0, **kw):
    """Paged-KV decode with the library's built-in scratch
    (attn_fwd_paged_kvcache_static): for callers that cannot allocate the
    metadata and workspace buffers. Returns (out, lse)."""
    a, out, lse, _ = paged_args(q, k_cache, v_cache, block_table, cache_seqlens,
                                num_ctas=num_ctas, **kw)
    _check("attn_fwd_paged_kvcache_static",
           lib().attn_fwd_paged_kvcache_static(ctypes.byref(a), _stream(stream)))
    return out, lse


# ---------------------------------------------------------------------------
# attn_combine
# ---------------------------------------------------------------------------

def combine(out_partial, lse_partial, *, num_splits_per_seq=None, sink=None, out=None, lse=None,
            out_dtype=torch.bfloat16, stream=None):
    """Merge split partials: out_partial fp32 (n, B, S, H, Dv), lse_partial fp32
    (n, B, H, S). Returns (out (B, S, H, Dv), lse (B, H, S))."""
    n, B, S, H, Dv = out_partial.shape
    if out is None:
        out = torch.empty(B, S, H, Dv, device=out_partial.device, dtype=out_dtype)
    if lse is None:
        lse = torch.empty(B, H, S, device=out_partial.device, dtype=torch.float32)
    a = CombineArgs(_ptr(out_partial), _ptr(lse_partial), _ptr(out), _ptr(lse),
                    _ptr(num_splits_per_seq), _ptr(sink), n, B, S, H, Dv, out.stride(0),
                    out.stride(1), out.stride(2), _TORCH_DTYPE[out.dtype])
    _check("attn_combine", lib().attn_combine(ctypes.byref(a), _stream(stream)))
    return out, lse


# ---------------------------------------------------------------------------
# mla_fwd_paged / mla_sparse_fwd
# ---------------------------------------------------------------------------

def mla_args(q, kv_cache, block_table, cache_seqlens, *, head_dim_v=512, scale=None,
             causal=False, indices=None, meta=None, num_ctas=0, workspace=None, out=None,
             lse=None, sparse_block_size=0, cu_seqlens_q=None, q_descale=None, k_descale=None,
             v_descale=None):
    """BSND: q (B, s_q, H_q, 576), indices (B, s_q, H_kv, topk); out
    (B, s_q, H_q, 512), lse (B, H_q, s_q). Packed (TND, sparse only, with
    cu_seqlens_q int32 (B+1)): q (T, H_q, 576), indices (T, H_kv, topk); out
    (T, H_q, 512), lse (H_q, T). q and kv_cache are both bf16 or both
    float8_e4m3fn; e4m3 takes fp32 (B, H_kv) descales (all three or none)."""
    _rows(q=q, kv_cache=kv_cache, out=out, block_table=block_table, indices=indices)
    _same_dtype(q, kv_cache=kv_cache)
    _dense(cache_seqlens=cache_seqlens, lse=lse, cu_seqlens_q=cu_seqlens_q,
           q_descale=q_descale, k_descale=k_descale, v_descale=v_descale)
    _int32(block_table=block_table, cache_seqlens=cache_seqlens, indices=indices,
           cu_seqlens_q=cu_seqlens_q)
    tnd = cu_seqlens_q is not None
    if tnd:
        if q.dim() != 3 or indices is None:
            raise ValueError("packed queries: q (T, H_q, 576) and sparse indices")
        B = cache_seqlens.numel()
        sq, Hq, Dqk = q.shape
        if out is None:
            out = torch.empty(sq, Hq, head_dim_v, device=q.device, dtype=torch.bfloat16)
        if lse is None:
            lse = torch.empty(Hq, sq, device=q.device, dtype=torch.float32)
        qs = (0, q.stride(0), q.stride(1))
        os_ = (0, out.stride(0), out.stride(1))
        ist = (0, indices.stride(0), indices.stride(1))
    else:
        B, sq, Hq, Dqk = q.shape
        if out is None:
            out = torch.empty(B, sq, Hq, head_dim_v, device=q.device, dtype=torch.bfloat16)
        if lse is None:
            lse = torch.empty(B, Hq, sq, device=q.device, dtype=torch.float32)
        qs = (q.stride(0), q.stride(1), q.stride(2))
        os_ = (out.stride(0), out.stride(1), out.stride(2))
        ist = (0, 0, 0) if indices is None else (indices.stride(0), indices.stride(1),
                                                 indices.stride(2))
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    topk = 0 if indices is None else indices.shape[-1]
    a = MlaArgs(
        _ptr(q), _ptr(kv_cache), _ptr(block_table), _ptr(cache_seqlens), _ptr(indices),
        _ptr(out), _ptr(lse), B, sq, Hq, kv_cache.shape[2], Dqk, head_dim_v, kv_cache.shape[1],
        kv_cache.shape[0], block_table.shape[1], topk, block_table.stride(0), *qs,
        kv_cache.stride(0), kv_cache.stride(1), *os_, ist[0], ist[1], float(scale),
        int(bool(causal)), _ptr(meta), 0 if meta is None else meta.numel() * 4, int(num_ctas),
        None, 0, int(sparse_block_size), kv_cache.stride(2), ist[2], _ptr(cu_seqlens_q),
        _TORCH_DTYPE.get(q.dtype, -1), _ptr(q_descale), _ptr(k_descale), _ptr(v_descale))
    if meta is not None:
        nbytes = int(lib().mla_workspace_size(ctypes.byref(a)))
        if workspace is None:
            workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
        a.workspace = workspace.data_ptr()
        a.workspace_bytes = workspace.numel()
    return a, out, lse, workspace


def mla_fwd_paged(q, kv_cache, block_table, cache_seqlens, *, stream=None, **kw):
    """MLA-absorbed decode over a paged latent cache. Returns (out, lse)."""
    a, out, lse, ws = mla_args(q, kv_cache, block_table, cache_seqlens, **kw)
    _check("mla_fwd_paged", lib().mla_fwd_paged(ctypes.byref(a), _stream(stream)))
    _keep_for(stream, ws)
    return out, lse


def mla_sparse_fwd(q, kv_cache, block_table, cache_seqlens, indices, *, stream=None, **kw):
    """MLA decode over top-k index sets. Returns (out, lse)."""
    a, out, lse, ws = mla_args(q, kv_cache, block_table, cache_seqlens, indices=indices, **kw)
    _check("mla_sparse_fwd", lib().mla_sparse_fwd(ctypes.byref(a), _stream(stream)))
    _keep_for(stream, ws)
    return out, lse


def mla_metadata(inp_cache_seqlens, *, batch, seqlen_q, num_heads_q, page_size, topk=0,
                 num_ctas=0, stream=None, sparse_block_size=0, num_heads_kv=1):
    """Scheduler metadata for mla_fwd_paged (topk = 0) or mla_sparse_fwd. For
    packed (TND) queries pass batch=1 and seqlen_q=T."""
    return sched_metadata(inp_cache_seqlens, batch=batch, seqlen_q=seqlen_q,
                          num_heads_q=num_heads_q, num_heads_kv=num_heads_kv, head_dim_qk=576,
                          head_dim_v=512, page_size=page_size,
                          mode=SCHED_MLA_SPARSE if topk else SCHED_MLA, topk=topk,
                          num_ctas=num_ctas, stream=stream, sparse_block_size=sparse_block_size)
