"""The decode-step selection entry point that allocates nothing.

dsa_indexer_topk_decode_noalloc serves callers that cannot allocate device
memory (a component inside a runtime that owns every device allocation, or
code called where no allocator is reachable), so it cannot take a workspace
and uses a scratch buffer built into the library instead.  These tests call
it through the C ABI and check that it returns what dsa_indexer_topk_decode
(the entry point with a caller workspace) returns on the same inputs, over
two calls in a row that share the built-in buffer, and that a step larger
than the buffer is refused.

The file is named so that pytest collects it last; it also passes alone in a
fresh process (the first call on a device does the buffer's set-up).
"""

import ctypes as C

import numpy as np
import pytest
import torch

import learned_token_indexer_b200 as dsa
from learned_token_indexer_b200 import _lib
from learned_token_indexer_b200 import workloads as W
from tests import checks

pytestmark = pytest.mark.gpu

MAX_KEYS = 1 << 22          # the built-in buffer's limit, in cached keys per call


@pytest.fixture(scope="module", autouse=True)
def built():
    from learned_token_indexer_b200.build import build
    build()
    torch.cuda.init()
    yield


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _call_noalloc(d, k, total, maxlen, fp8=False):
    """One call through the C ABI; the outputs are allocated here, by the test."""
    B, HI, dI = d["qI"].shape
    dev = d["qI"].device
    idx = torch.full((B, k), -7, dtype=torch.int32, device=dev)
    val = torch.full((B, k), float("nan"), dtype=torch.float32, device=dev)
    status = torch.full((2,), -1, dtype=torch.int32, device=dev)
    st = _lib.load().dsa_indexer_topk_decode_noalloc(
        B, HI, dI, k, dsa.FP8_E4M3 if fp8 else dsa.BF16, _p(d["qI"]), _p(d.get("q_scale")), _p(d["w"]),
        _p(d["kI_cache"]), _p(d.get("k_scale")), _p(d["cu_seqlens"]), total, maxlen, _p(idx), _p(val), _p(status),
        C.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    assert st == 0, _lib.load().dsa_last_error().decode()
    return idx, val, status


def _sorted_rows(idx, val):
    """Rows as (positions, scores) sorted by position: the order of the k
    selected entries within a row is not part of the result."""
    i = idx.cpu().numpy()
    v = val.cpu().double().numpy()
    order = np.argsort(i, axis=1, kind="stable")
    return np.take_along_axis(i, order, 1), np.take_along_axis(v, order, 1)


def _inputs(seed, lengths, fp8=False):
    w = W.scaled(W.DECODE, B=len(lengths), k=300, seed=seed)
    d = W.make_decode_inputs(w, "cuda", lengths=torch.tensor(lengths))
    if fp8:     # per-token scales: q_scale [B] over all heads, k_scale [total_len]
        d["qI"], d["q_scale"] = W.quantize_fp8_per_token(d["qI"], 2)
        d["kI_cache"], d["k_scale"] = W.quantize_fp8_per_token(d["kI_cache"], 1)
    return w, d


@pytest.mark.parametrize("fp8", [False, True])
def test_noalloc_matches_workspace_entry_two_calls(fp8):
    # the second call is smaller than the first, so the built-in buffer still
    # holds the first call's scores beyond the second call's keys
    cases = [(11, [1, 129, 300, 1000, 4097, 2500]), (12, [700, 5, 301, 64])]
    for seed, lengths in cases:
        w, d = _inputs(seed, lengths, fp8)
        total, maxlen = sum(lengths), max(lengths)
        idx, val, status = _call_noalloc(d, w.k, total, maxlen, fp8)
        ws = dsa.Workspace("cuda")
        ref_idx, ref_val = dsa.indexer_topk_decode(d["qI"], d["w"], d["kI_cache"], d["cu_seqlens"], w.k, total,
                                                   maxlen, q_scale=d.get("q_scale"), k_scale=d.get("k_scale"),
                                                   return_scores=True, workspace=ws)
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        ws.check()
        gi, gv = _sorted_rows(idx, val)
        ri, rv = _sorted_rows(ref_idx, ref_val)
        assert np.array_equal(gi, ri), f"seed {seed}: selected positions differ"
        bad = checks.close_errors(np.where(gi >= 0, gv, 0.0), np.where(ri >= 0, rv, 0.0), 1e-5, 1e-5,
                                  "selected scores")
        assert not bad, bad[:5]
        for b, L in enumerate(lengths):         # -1 padding for rows shorter than k
            assert (gi[b] >= 0).sum() == min(w.k, L)


def test_noalloc_refuses_steps_beyond_its_buffer():
    w, d = _inputs(13, [64, 64])
    idx = torch.empty((2, w.k), dtype=torch.int32, device="cuda")
    st = _lib.load().dsa_indexer_topk_decode_noalloc(
        2, w.HI, w.dI, w.k, dsa.BF16, _p(d["qI"]), None, _p(d["w"]), _p(d["kI_cache"]), None, _p(d["cu_seqlens"]),
        MAX_KEYS + 1, MAX_KEYS, _p(idx), None, None, C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert dsa.STATUS[st] == "DSA_ERR_UNSUPPORTED"
    msg = _lib.load().dsa_last_error().decode()
    assert str(MAX_KEYS) in msg and "dsa_indexer_topk_decode" in msg
