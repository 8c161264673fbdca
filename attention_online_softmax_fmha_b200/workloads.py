"""Seeded synthetic inputs for the attention forward workloads.

This module is shared by the tests, the benchmark and the oracle checks. It
holds no attention arithmetic: it only draws random tensors, sequence lengths,
page permutations and sparse index sets, and packs them into the layouts the
library's C ABI takes. Every draw is seeded; the same (name, seed, device)
always gives the same bytes.

Workload shapes follow the problem statement of the pages:

* dense / varlen prefill: q (T, H_q, D) packed with int32 cu_seqlens, or
  padded (B, S, H, D) -- MindSpore "sparse_flash_attention" (TND / BSND
  layouts) and MATE "Attention" / FMHA (``flash_attn_varlen_func``);
* paged KV cache (num_blocks, page_size, H_kv, D) with an int32 block_table
  (B, max_pages) and int32 cache_seqlens (B,) -- MATE "Attention" / MLA
  example;
* MLA-absorbed rows of 576 = 512 latent + 64 rope, V = the first 512 --
  MindSpore "sparse_flash_attention", ``attention_mode=2``;
* top-k sparse indices (B, S_q, 1, 2048) of logical token positions --
  MindSpore "sparse_flash_attention", ``sparse_indices``.

Values are N(0, 1) rounded to bf16 (round to nearest even, done by torch's
dtype conversion); FP8 E4M3 inputs are N(0, 1) converted by torch to
``float8_e4m3fn``; descales are U[0.5, 2].
"""
from __future__ import annotations

import dataclasses
import itertools
import math
from typing import List, Optional, Sequence

import torch

__all__ = [
    "PrefillInputs", "PagedInputs", "MlaInputs",
    "uniform_lengths", "make_prefill", "make_paged", "make_mla",
    "CONFIGS",
]

_FP8 = {"e4m3": torch.float8_e4m3fn, "e5m2": torch.float8_e5m2}
_F16 = {"bf16": torch.bfloat16, "fp16": torch.float16}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def uniform_lengths(n: int, lo: int, hi: int, seed: int) -> List[int]:
    """n integers uniform in [lo, hi] (inclusive), drawn on the CPU so the
    lengths do not depend on the device the tensors live on."""
    g = _gen(seed, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def _values(shape, dtype: str, g: torch.Generator, device) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if dtype in _F16:
        return x.to(_F16[dtype])
    if dtype in _FP8:
        return x.to(_FP8[dtype])
    raise ValueError(f"unknown dtype {dtype!r}")


@dataclasses.dataclass
class PrefillInputs:
    """Dense (padded BSHD) or varlen (packed THD) prefill inputs."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    cu_seqlens_q: Optional[torch.Tensor]   # int32 (B+1) or None for padded
    cu_seqlens_k: Optional[torch.Tensor]
    seqlens_q: List[int]
    seqlens_k: List[int]
    num_heads_q: int
    num_heads_kv: int
    head_dim: int
    causal: bool
    window: tuple
    scale: float
    sink: Optional[torch.Tensor]           # fp32 (H_q,)
    q_descale: Optional[torch.Tensor]      # fp32 (B, H_kv)
    k_descale: Optional[torch.Tensor]
    v_descale: Optional[torch.Tensor]
    dtype: str
    # additive score mask fp32 [b, 1, i, j] (broadcast over heads), rows padded
    # to a multiple of 4 floats in storage; None = no mask
    mask: Optional[torch.Tensor] = None

    @property
    def batch(self) -> int:
        return len(self.seqlens_q)

    @property
    def varlen(self) -> bool:
        return self.cu_seqlens_q is not None


def make_prefill(*, seqlens_q: Sequence[int], seqlens_k: Optional[Sequence[int]] = None,
                 num_heads_q: int, num_heads_kv: int, head_dim: int, varlen: bool,
                 causal: bool = False, window=(-1, -1), sink: bool = False,
                 dtype: str = "bf16", scale: Optional[float] = None, seed: int = 0,
                 mask: bool = False, device="cpu") -> PrefillInputs:
    """Prefill inputs. ``varlen`` packs the sequences back to back (TND with
    cu_seqlens); otherwise all sequences must share one length and the tensors
    are padded BSHD. ``mask``: an additive fp32 score mask N(0, 1) per
    (sequence, row, key), shared by the heads."""
    seqlens_q = [int(x) for x in seqlens_q]
    seqlens_k = [int(x) for x in (seqlens_k if seqlens_k is not None else seqlens_q)]
    B = len(seqlens_q)
    assert len(seqlens_k) == B
    g = _gen(seed, device)
    if varlen:
        tq, tk = sum(seqlens_q), sum(seqlens_k)
        q = _values((tq, num_heads_q, head_dim), dtype, g, device)
        k = _values((tk, num_heads_kv, head_dim), dtype, g, device)
        v = _values((tk, num_heads_kv, head_dim), dtype, g, device)
        cq = [0]
        ck = [0]
        for a, b in zip(seqlens_q, seqlens_k):
            cq.append(cq[-1] + a)
            ck.append(ck[-1] + b)
        cu_q = torch.tensor(cq, dtype=torch.int32, device=device)
        cu_k = torch.tensor(ck, dtype=torch.int32, device=device)
    else:
        assert len(set(seqlens_q)) == 1 and len(set(seqlens_k)) == 1, "padded layout needs equal lengths"
        q = _values((B, seqlens_q[0], num_heads_q, head_dim), dtype, g, device)
        k = _values((B, seqlens_k[0], num_heads_kv, head_dim), dtype, g, device)
        v = _values((B, seqlens_k[0], num_heads_kv, head_dim), dtype, g, device)
        cu_q = cu_k = None
    sink_t = (torch.randn(num_heads_q, generator=g, device=device, dtype=torch.float32)
              if sink else None)
    qd = kd = vd = None
    if dtype in _FP8:
        qd = torch.rand(B, num_heads_kv, generator=g, device=device) * 1.5 + 0.5
        kd = torch.rand(B, num_heads_kv, generator=g, device=device) * 1.5 + 0.5
        vd = torch.rand(B, num_heads_kv, generator=g, device=device) * 1.5 + 0.5
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    mask_t = None
    if mask:
        lq, lk = max(seqlens_q), max(seqlens_k)
        store = torch.randn(B, 1, lq, (lk + 3) // 4 * 4, generator=g, device=device,
                            dtype=torch.float32)
        mask_t = store[..., :lk]
    return PrefillInputs(q, k, v, cu_q, cu_k, seqlens_q, seqlens_k, num_heads_q, num_heads_kv,
                         head_dim, bool(causal), tuple(window), float(scale), sink_t, qd, kd, vd,
                         dtype, mask_t)


@dataclasses.dataclass
class PagedInputs:
    """Decode against a paged KV cache."""
    q: torch.Tensor                # (B, s_q, H_q, D)
    k_cache: torch.Tensor          # (num_blocks, page_size, H_kv, D)
    v_cache: torch.Tensor
    block_table: torch.Tensor      # int32 (B, max_pages)
    cache_seqlens: torch.Tensor    # int32 (B,)
    seqlens: List[int]
    page_size: int
    num_heads_q: int
    num_heads_kv: int
    head_dim: int
    causal: bool
    window: tuple
    scale: float
    sink: Optional[torch.Tensor]
    dtype: str
    q_descale: Optional[torch.Tensor] = None   # FP8: fp32 (B, H_kv) in [0.5, 2]
    k_descale: Optional[torch.Tensor] = None
    v_descale: Optional[torch.Tensor] = None
    k_new: Optional[torch.Tensor] = None       # appended keys (B, s_new, H_kv, D)
    v_new: Optional[torch.Tensor] = None

    @property
    def batch(self) -> int:
        return len(self.seqlens)


def _block_table(seqlens: Sequence[int], page_size: int, layout: str, g_cpu: torch.Generator,
                 extra_blocks: int = 0):
    """Physical page assignment. ``permuted``: a seeded random permutation of
    all pages; ``identity``: pages in order; ``aliased``: every entry 0 (the
    MATE MLA example's all-zeros table)."""
    pages = [max(1, -(-L // page_size)) for L in seqlens]
    total = sum(pages)
    max_pages = max(pages)
    if layout == "permuted":
        perm = torch.randperm(total, generator=g_cpu).to(torch.int32)
    elif layout == "identity":
        perm = torch.arange(total, dtype=torch.int32)
    elif layout == "aliased":
        perm = torch.zeros(total, dtype=torch.int32)
    else:
        raise ValueError(layout)
    bt = torch.zeros(len(seqlens), max_pages, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages):
        bt[b, :n] = perm[off:off + n]
        off += n
    num_blocks = (1 if layout == "aliased" else total) + extra_blocks
    return bt, num_blocks


def make_paged(*, seqlens: Sequence[int], seqlen_q: int, num_heads_q: int, num_heads_kv: int,
               head_dim: int, page_size: int = 64, table: str = "permuted", causal: bool = False,
               window=(-1, -1), sink: bool = False, dtype: str = "bf16",
               scale: Optional[float] = None, seqlen_new: int = 0, seed: int = 0,
               device="cpu") -> PagedInputs:
    seqlens = [int(x) for x in seqlens]
    g_cpu = _gen(seed + 7919, "cpu")
    bt, nblocks = _block_table(seqlens, page_size, table, g_cpu)
    g = _gen(seed, device)
    B = len(seqlens)
    q = _values((B, seqlen_q, num_heads_q, head_dim), dtype, g, device)
    kc = _values((nblocks, page_size, num_heads_kv, head_dim), dtype, g, device)
    vc = _values((nblocks, page_size, num_heads_kv, head_dim), dtype, g, device)
    sink_t = (torch.randn(num_heads_q, generator=g, device=device, dtype=torch.float32)
              if sink else None)
    desc = [None, None, None]
    if dtype in _FP8:
        desc = [torch.rand(B, num_heads_kv, generator=g, device=device) * 1.5 + 0.5
                for _ in range(3)]
    new = [None, None]
    if seqlen_new > 0:
        new = [_values((B, seqlen_new, num_heads_kv, head_dim), dtype, g, device)
               for _ in range(2)]
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return PagedInputs(q, kc, vc, bt.to(device), torch.tensor(seqlens, dtype=torch.int32,
                       device=device), seqlens, page_size, num_heads_q, num_heads_kv, head_dim,
                       bool(causal), tuple(window), float(scale), sink_t, dtype, *desc, *new)


@dataclasses.dataclass
class MlaInputs:
    """MLA-absorbed decode: H_kv latent KV heads (usually 1) whose 576-wide
    rows are [512 latent | 64 rope]; V is the first 512 of the row."""
    q: torch.Tensor                # (B, s_q, H_q, 576)
    kv_cache: torch.Tensor         # (num_blocks, page_size, H_kv, 576)
    block_table: torch.Tensor
    cache_seqlens: torch.Tensor
    seqlens: List[int]
    page_size: int
    num_heads_q: int
    head_dim_v: int
    causal: bool
    scale: float
    indices: Optional[torch.Tensor]  # int32 (B, s_q, H_kv, topk) or None
    topk: int
    num_heads_kv: int = 1
    dtype: str = "bf16"              # "bf16", or "e4m3" for q and the cache
    q_descale: Optional[torch.Tensor] = None   # e4m3: fp32 (B, H_kv) in [0.5, 2]
    k_descale: Optional[torch.Tensor] = None
    v_descale: Optional[torch.Tensor] = None

    @property
    def batch(self) -> int:
        return len(self.seqlens)


def sparse_indices(seqlens: Sequence[int], seqlen_q: int, topk: int, seed: int,
                   kind: str = "uniform") -> torch.Tensor:
    """int32 (B, s_q, 1, topk). ``uniform``: topk distinct positions drawn
    uniformly below the sequence's cache length, sorted ascending (fewer than
    topk positions: all of them, padded with -1). ``all``: positions 0..L-1
    then -1 padding."""
    g = _gen(seed + 104729, "cpu")
    B = len(seqlens)
    out = torch.full((B, seqlen_q, 1, topk), -1, dtype=torch.int32)
    for b, L in enumerate(seqlens):
        for i in range(seqlen_q):
            if kind == "all" or L <= topk:
                n = min(L, topk)
                out[b, i, 0, :n] = torch.arange(n, dtype=torch.int32)
            else:
                idx = torch.randperm(L, generator=g)[:topk].sort().values
                out[b, i, 0, :] = idx.to(torch.int32)
    return out


def make_mla(*, seqlens: Sequence[int], seqlen_q: int, num_heads_q: int, page_size: int = 64,
             head_dim: int = 576, head_dim_v: int = 512, table: str = "permuted",
             causal: bool = False, topk: int = 0, index_kind: str = "uniform",
             scale: Optional[float] = None, num_heads_kv: int = 1, dtype: str = "bf16",
             seed: int = 0, device="cpu") -> MlaInputs:
    """MLA inputs; dtype "e4m3" draws q and the cache as N(0, 1) converted to
    e4m3 and descales U[0.5, 2] per (sequence, KV head)."""
    seqlens = [int(x) for x in seqlens]
    g_cpu = _gen(seed + 7919, "cpu")
    bt, nblocks = _block_table(seqlens, page_size, table, g_cpu)
    g = _gen(seed, device)
    B = len(seqlens)
    q = _values((B, seqlen_q, num_heads_q, head_dim), dtype, g, device)
    kv = _values((nblocks, page_size, num_heads_kv, head_dim), dtype, g, device)
    desc = [None] * 3
    if dtype in _FP8:
        desc = [torch.rand(B, num_heads_kv, generator=g, device=device) * 1.5 + 0.5
                for _ in range(3)]
    idx = None
    if topk:
        # one index list per KV head (the first with the given seed)
        idx = torch.cat([sparse_indices(seqlens, seqlen_q, topk, seed + 7 * h, index_kind)
                         for h in range(num_heads_kv)], dim=2).to(device)
    if scale is None:
        scale = 1.0 / math.sqrt(head_dim)
    return MlaInputs(q, kv, bt.to(device), torch.tensor(seqlens, dtype=torch.int32, device=device),
                     seqlens, page_size, num_heads_q, head_dim_v, bool(causal), float(scale), idx,
                     int(topk), int(num_heads_kv), dtype, *desc)


@dataclasses.dataclass
class MlaTndInputs:
    """Sparse MLA with packed (TND) queries: sequence b owns query tokens
    cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and reads its own cache."""
    q: torch.Tensor                # (T, H_q, 576)
    kv_cache: torch.Tensor         # (num_blocks, page_size, 1, 576)
    block_table: torch.Tensor
    cache_seqlens: torch.Tensor
    cu_seqlens_q: torch.Tensor     # int32 (B + 1)
    seqlens: List[int]
    seqlens_q: List[int]
    page_size: int
    num_heads_q: int
    causal: bool
    scale: float
    indices: torch.Tensor          # int32 (T, 1, topk)
    topk: int


def make_mla_tnd(*, seqlens: Sequence[int], seqlens_q: Sequence[int], num_heads_q: int,
                 topk: int, page_size: int = 64, causal: bool = False, seed: int = 0,
                 device="cpu") -> MlaTndInputs:
    seqlens = [int(x) for x in seqlens]
    seqlens_q = [int(x) for x in seqlens_q]
    g_cpu = _gen(seed + 7919, "cpu")
    bt, nblocks = _block_table(seqlens, page_size, "permuted", g_cpu)
    g = _gen(seed, device)
    T = sum(seqlens_q)
    q = _values((T, num_heads_q, 576), "bf16", g, device)
    kv = _values((nblocks, page_size, 1, 576), "bf16", g, device)
    idx = torch.cat([sparse_indices([L], n, topk, seed + b)[0, :, 0]
                     for b, (L, n) in enumerate(zip(seqlens, seqlens_q)) if n > 0])
    cu = torch.tensor([0] + list(itertools.accumulate(seqlens_q)), dtype=torch.int32)
    return MlaTndInputs(q, kv, bt.to(device),
                        torch.tensor(seqlens, dtype=torch.int32, device=device), cu.to(device),
                        seqlens, seqlens_q, page_size, num_heads_q, bool(causal),
                        1.0 / math.sqrt(576), idx[:, None, :].contiguous().to(device), int(topk))


# The five workloads the benchmark and the full-size parity tests use.
CONFIGS = {
    "tiny_dense_mha": dict(kind="prefill", seqlens_q=[128], num_heads_q=2, num_heads_kv=2,
                           head_dim=64, varlen=False, causal=False, scale=1.0 / 8.0),
    "varlen_causal_gqa": dict(kind="prefill", lengths=(8, 512, 4096), num_heads_q=32,
                              num_heads_kv=8, head_dim=128, varlen=True, causal=True),
    "window_sink": dict(kind="prefill", seqlens_q=[8192] * 4, num_heads_q=32, num_heads_kv=32,
                        head_dim=128, varlen=False, causal=True, window=(1024, 0), sink=True),
    "window_sink_fp8": dict(kind="prefill", seqlens_q=[8192] * 4, num_heads_q=32,
                            num_heads_kv=32, head_dim=128, varlen=False, causal=True,
                            window=(1024, 0), sink=True, dtype="e4m3"),
    # the same with e5m2 inputs (MATE FMHA dtype list)
    "window_sink_e5m2": dict(kind="prefill", seqlens_q=[8192] * 4, num_heads_q=32,
                             num_heads_kv=32, head_dim=128, varlen=False, causal=True,
                             window=(1024, 0), sink=True, dtype="e5m2"),
    # an additive score mask on a causal padded prefill (B4 S4096 H32/8 D128;
    # the mask is 4 x 4096 x 4096 fp32, shared by the heads)
    "dense_mask": dict(kind="prefill", seqlens_q=[4096] * 4, num_heads_q=32, num_heads_kv=8,
                       head_dim=128, varlen=False, causal=True, mask=True),
    "paged_decode": dict(kind="paged", lengths=(64, 1024, 32768), seqlen_q=1, num_heads_q=32,
                         num_heads_kv=8, head_dim=128, page_size=64),
    # the same decode against an e4m3 cache with per-(sequence, KV head) descales
    "paged_decode_fp8": dict(kind="paged", lengths=(64, 1024, 32768), seqlen_q=1,
                             num_heads_q=32, num_heads_kv=8, head_dim=128, page_size=64,
                             dtype="e4m3"),
    # the same decode with 16 sequences (about 1.1 GB of cache), for profiler
    # captures that must stay small
    "paged_decode_small": dict(kind="paged", lengths=(16, 1024, 32768), seqlen_q=1,
                               num_heads_q=32, num_heads_kv=8, head_dim=128, page_size=64),
    "mla_dense": dict(kind="mla", lengths=(64, 4096, 65536), seqlen_q=2, num_heads_q=128,
                      page_size=64),
    "mla_sparse": dict(kind="mla", lengths=(64, 4096, 65536), seqlen_q=2, num_heads_q=128,
                       page_size=64, topk=2048),
    # the MLA workloads against an e4m3 latent cache (and e4m3 q) with
    # per-(sequence, KV head) descales
    "mla_dense_fp8": dict(kind="mla", lengths=(64, 4096, 65536), seqlen_q=2, num_heads_q=128,
                          page_size=64, dtype="e4m3"),
    "mla_sparse_fp8": dict(kind="mla", lengths=(64, 4096, 65536), seqlen_q=2, num_heads_q=128,
                           page_size=64, topk=2048, dtype="e4m3"),
    # 8-sequence versions of the MLA workloads, for profiler captures
    "mla_dense_small": dict(kind="mla", lengths=(8, 4096, 65536), seqlen_q=2, num_heads_q=128,
                            page_size=64),
    "mla_sparse_small": dict(kind="mla", lengths=(8, 4096, 65536), seqlen_q=2,
                             num_heads_q=128, page_size=64, topk=2048),
    # reduced-batch FP8 versions, for profiler captures
    "paged_decode_fp8_small": dict(kind="paged", lengths=(16, 1024, 32768), seqlen_q=1,
                                   num_heads_q=32, num_heads_kv=8, head_dim=128, page_size=64,
                                   dtype="e4m3"),
    "mla_dense_fp8_small": dict(kind="mla", lengths=(8, 4096, 65536), seqlen_q=2,
                                num_heads_q=128, page_size=64, dtype="e4m3"),
    "mla_sparse_fp8_small": dict(kind="mla", lengths=(8, 4096, 65536), seqlen_q=2,
                                 num_heads_q=128, page_size=64, topk=2048, dtype="e4m3"),
}


def build_config(name: str, seed: int = 0, device="cpu"):
    """Materialise one of CONFIGS at full size."""
    c = dict(CONFIGS[name])
    kind = c.pop("kind")
    if "lengths" in c:
        n, lo, hi = c.pop("lengths")
        lens = uniform_lengths(n, lo, hi, seed)
    else:
        lens = None
    if kind == "prefill":
        if lens is not None:
            c["seqlens_q"] = lens
        return make_prefill(seed=seed, device=device, **c)
    if kind == "paged":
        return make_paged(seqlens=lens, seed=seed, device=device, **c)
    if kind == "mla":
        return make_mla(seqlens=lens, seed=seed, device=device, **c)
    raise ValueError(kind)
