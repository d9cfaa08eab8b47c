"""Host-side pieces of the measurement: the seeded input generators (shapes,
determinism, the structural promises the kernels and the oracle rely on) and
the work counts bench.py divides by.  No GPU."""

import numpy as np
import pytest
import torch

import bench
from learned_token_indexer_b200 import workloads as W


def test_generators_are_seeded_and_shaped():
    w = W.scaled(W.TINY, n=64)
    a = W.make_prefill_inputs(w, "cpu")
    b = W.make_prefill_inputs(w, "cpu")
    for key in ("qI", "kI", "w", "q", "latent"):
        assert torch.equal(a[key], b[key]), key
    assert a["qI"].shape == (w.B, 64, w.HI, w.dI) and a["qI"].dtype == torch.bfloat16
    assert a["kI"].shape == (w.B, 64, w.dI)
    assert a["q"].shape == (w.B, 64, w.H, w.Dqk) and a["latent"].shape == (w.B, 64, w.Dqk)
    # integer workloads: integer-valued q^I, k^I in range; w on the 1/w_den grid
    assert torch.all(a["qI"].float().abs() <= w.qk_int_max) and torch.equal(a["qI"].float(), a["qI"].float().round())
    assert torch.equal((a["w"] * w.w_den).round(), a["w"] * w.w_den)


def test_fp8_preparation_is_per_token_amax_over_448():
    w = W.scaled(W.PREFILL_FP8, B=1, n=16, seed=3)
    d = W.make_prefill_inputs(w, "cpu", with_attention=False, keep_bf16=True)
    codes = d["kI"].float()
    assert codes.abs().amax(dim=-1).max() <= W.FP8_MAX
    # the largest code of every token is +-448 (its amax maps to the top of the range)
    assert torch.allclose(codes.abs().amax(dim=-1), torch.full((1, 16), W.FP8_MAX))
    assert d["k_scale"].shape == (1, 16) and torch.all(d["k_scale"] > 0)
    assert d["q_scale"].shape == (1, 16)


@pytest.mark.parametrize("q_offset,k", [(0, 4), (3, 6), (0, 64)])
def test_make_selection_is_a_valid_causal_selection(q_offset, k):
    B, nq, kv_len = 2, 20, q_offset + 20
    sel = W.make_selection(B, nq, kv_len, k, q_offset=q_offset, seed=5)
    assert sel.shape == (B, nq, k) and sel.dtype == torch.int32
    assert torch.equal(sel, W.make_selection(B, nq, kv_len, k, q_offset=q_offset, seed=5))
    for b in range(B):
        for i in range(nq):
            t = q_offset + i
            row = sel[b, i].tolist()
            m = min(k, t + 1)
            assert all(0 <= p <= t for p in row[:m])          # valid slots first, causal
            assert all(p == -1 for p in row[m:])              # then -1
            assert len(set(row[:m])) == m                     # distinct


def test_make_teacher_is_nonnegative_with_exact_zeros():
    t = W.make_teacher((3, 50, 40), seed=2)
    assert torch.all(t >= 0) and t.dtype == torch.float32
    frac0 = float((t == 0).float().mean())
    assert 0.05 < frac0 < 0.15
    assert torch.equal(t, W.make_teacher((3, 50, 40), seed=2))


@pytest.mark.parametrize("t0,n,k", [(0, 100, 16), (0, 10, 16), (5000, 300, 2048), (0, 8192, 2048)])
def test_work_counts_match_brute_force(t0, n, k):
    # (t, s) pairs that need a score: rows with t + 1 > k score all t + 1 keys
    pairs = sum(t + 1 for t in range(t0, t0 + n) if t + 1 > k)
    assert bench.count_pairs_needed(t0, n, k) == pairs
    assert bench.selected_entries(t0, n, k) == sum(min(k, t + 1) for t in range(t0, t0 + n))


def test_decode_lengths_are_in_range_and_seeded():
    L = W.decode_lengths(W.DECODE)
    assert L.shape == (W.DECODE.B,)
    assert int(L.min()) >= W.DECODE.L_min and int(L.max()) <= W.DECODE.L_max
    assert torch.equal(L, W.decode_lengths(W.DECODE))


def test_sample_rows_cover_the_edges():
    rows = W.sample_rows(W.LONG, 256)
    rs = set(rows)
    for i in (0, 1, W.LONG.k - 2, W.LONG.k - 1, W.LONG.k, W.LONG.n - 1):
        assert (0, i) in rs
    for c0 in range(0, W.LONG.n, W.LONG.chunk):
        assert (0, c0) in rs and (0, c0 + W.LONG.chunk - 1) in rs
    assert len(rows) == len(rs) >= 256


def test_traffic_records_name_their_summaries_and_cases():
    """Every DRAM-traffic record the bench may attach to a roofline names a
    committed ncu summary; a record taken on another launch than the timed
    one says which (the long prefill's long-history chunk), and a record is
    dropped for a workload it was not taken on."""
    import json
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "traffic.json")) as f:
        records = json.load(f)
    for key, rec in records.items():
        kernel, _, workload = key.partition(":")
        assert kernel in bench.KERNEL_SOURCES and workload, key
        assert os.path.exists(os.path.join(root, rec["summary"])), rec["summary"]
        assert rec["bytes_per_launch"] > 0
    rec = records["indexer_topk_prefill:long_prefill"]
    assert "captured launch" in rec["case"]
    bytes_, case = bench.measured_traffic("indexer_topk_prefill", "long_prefill")
    if rec["source_hash"] == bench.kernel_source_hash(bench.KERNEL_SOURCES["indexer_topk_prefill"]):
        assert bytes_ == rec["bytes_per_launch"] and case == rec["case"]
    else:   # the kernel changed since the capture: no traffic figure
        assert bytes_ is None and case is None
    assert bench.measured_traffic("indexer_topk_prefill", "no_such_workload") == (None, None)
