"""The seeded input generator: determinism, shapes, value distribution and
page/index structure."""
import torch

from attention_online_softmax_fmha_b200 import workloads as W


def test_prefill_is_deterministic_and_shaped():
    a = W.make_prefill(seqlens_q=[5, 9], num_heads_q=4, num_heads_kv=2, head_dim=8, varlen=True,
                       causal=True, sink=True, seed=3)
    b = W.make_prefill(seqlens_q=[5, 9], num_heads_q=4, num_heads_kv=2, head_dim=8, varlen=True,
                       causal=True, sink=True, seed=3)
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.sink, b.sink)
    assert a.q.shape == (14, 4, 8) and a.k.shape == (14, 2, 8)
    assert a.cu_seqlens_q.tolist() == [0, 5, 14] and a.q.dtype == torch.bfloat16
    c = W.make_prefill(seqlens_q=[5, 9], num_heads_q=4, num_heads_kv=2, head_dim=8, varlen=True,
                       seed=4)
    assert not torch.equal(a.q, c.q)


def test_values_are_standard_normal():
    x = W.make_prefill(seqlens_q=[4096], num_heads_q=4, num_heads_kv=4, head_dim=64,
                       varlen=False, seed=0).q.float()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1) < 0.01


def test_fp8_inputs_and_descales():
    a = W.make_prefill(seqlens_q=[64] * 2, num_heads_q=4, num_heads_kv=2, head_dim=16,
                       varlen=False, dtype="e4m3", seed=1)
    assert a.q.dtype == torch.float8_e4m3fn and a.q_descale.shape == (2, 2)
    assert float(a.q_descale.min()) >= 0.5 and float(a.q_descale.max()) <= 2.0


def test_lengths_uniform_in_range():
    L = W.uniform_lengths(1000, 512, 4096, 0)
    assert min(L) >= 512 and max(L) <= 4096 and max(L) - min(L) > 3000


def test_paged_table_is_permutation():
    p = W.make_paged(seqlens=[100, 1, 64, 65], seqlen_q=1, num_heads_q=4, num_heads_kv=2,
                     head_dim=8, page_size=16, seed=2)
    pages = [7, 1, 4, 5]
    used = torch.cat([p.block_table[b, :n] for b, n in enumerate(pages)])
    assert sorted(used.tolist()) == list(range(sum(pages)))
    assert p.k_cache.shape == (sum(pages), 16, 2, 8)
    assert p.cache_seqlens.tolist() == [100, 1, 64, 65]


def test_sparse_indices_distinct_sorted_below_length():
    idx = W.sparse_indices([5000, 300], 2, 256, seed=0)
    for b, L in enumerate([5000, 300]):
        for i in range(2):
            row = idx[b, i, 0]
            valid = row[row >= 0]
            assert valid.numel() == min(L, 256)
            assert torch.all(valid[1:] > valid[:-1]) and int(valid.max()) < L


def test_paged_fp8_descales_and_appended_keys():
    p = W.make_paged(seqlens=[30, 70], seqlen_q=2, num_heads_q=4, num_heads_kv=2, head_dim=16,
                     page_size=16, dtype="e5m2", seqlen_new=3, seed=5)
    assert p.k_cache.dtype == torch.float8_e5m2 and p.q.dtype == torch.float8_e5m2
    for t in (p.q_descale, p.k_descale, p.v_descale):
        assert t.shape == (2, 2) and float(t.min()) >= 0.5 and float(t.max()) <= 2.0
    assert p.k_new.shape == (2, 3, 2, 16) and p.k_new.dtype == torch.float8_e5m2
    assert not torch.equal(p.k_new.float(), p.v_new.float())
    plain = W.make_paged(seqlens=[30, 70], seqlen_q=2, num_heads_q=4, num_heads_kv=2,
                         head_dim=16, page_size=16, seed=5)
    assert plain.k_new is None and plain.q_descale is None
