"""bench.py's host-side arithmetic on the CPU: the algorithmic work that the
roofline divides by, and the source hashes that key the committed DRAM
traffic figures."""
import json
import os

import numpy as np
import pytest

import bench
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("lq,lk,causal,wl,wr", [
    (7, 7, False, -1, -1), (7, 7, True, -1, -1), (5, 12, True, -1, -1), (12, 5, True, -1, -1),
    (9, 9, True, 3, 0), (9, 9, False, 2, 4), (1, 40, True, 10, 0), (6, 6, False, 0, 0),
    (30, 64, True, 16, 0)])
def test_visible_pairs_closed_form_counts_the_mask(lq, lk, causal, wl, wr):
    # the prefill FLOP count uses this per (sequence, head); it must equal
    # the number of visible (query, key) pairs of the oracle's mask
    want = int(oracle.visible_mask(lq, lk, causal, wl, wr).sum())
    assert bench._visible_pairs(lq, lk, causal, wl, wr) == want


def test_source_hashes_are_per_kernel_family():
    pre = bench.source_hash("prefill_kernel<128,0>")
    assert pre == bench.source_hash("prefill_kernel<128,2>")
    assert len({pre, bench.source_hash("decode_kernel<128,0>"),
                bench.source_hash("mla_kernel<0>"), bench.source_hash()}) == 4
    assert bench.source_hash("unknown_kernel") == bench.source_hash()


def test_committed_traffic_entries_are_well_formed():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    assert t, "no traffic entries"
    for k, v in t.items():
        assert k.split("<")[0] in ("prefill_kernel", "decode_kernel", "mla_kernel"), k
        assert v["bytes_per_launch"] > 0 and len(v["source_hash"]) == 16
        assert v["captured_on"] in bench.WORKLOADS, v["captured_on"]
