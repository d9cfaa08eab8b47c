"""GPU parity of the dense masked attention (the short-prefill path of the
DSA page §2) and of the teacher mass coverage M_k (§3.1 eq. (15)), through
the C ABI, against the CPU oracle on the same seeded inputs.

Attention tolerance: |gpu - oracle| <= 2e-2 + 1e-2 |oracle| elementwise
(bf16 inputs, fp32 accumulation, bf16 probabilities and outputs), lse within
1e-3.  M_k is exp(lse_sparse - lse_dense), so its error is bounded by the two
lse errors: |dM| <= M (e^{2e-3} - 1) < 3e-3 for M <= 1.
"""

import numpy as np
import pytest
import torch

import learned_token_indexer_b200 as dsa
import oracle as O
from learned_token_indexer_b200 import workloads as W
from tests import checks
from tests.gpu_util import host_f64

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 1e-2


@pytest.fixture(scope="module", autouse=True)
def built():
    from learned_token_indexer_b200.build import build
    build()
    torch.cuda.init()
    yield


def _no_device_errors(ws):
    st, detail = ws.status()
    assert st == 0, f"device status {dsa.STATUS.get(st)} detail 0x{detail:x}"


def _inputs(B, n, kv_len, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, n, 16, 576), generator=g, device="cuda").bfloat16()
    lat = torch.randn((B, kv_len, 576), generator=g, device="cuda").bfloat16()
    return q, lat


def _check_rows(q, lat, idx, out, lse, q_offset, rows, scale=1 / 24):
    """Oracle eq. (3) per row: over idx's selection when given (rows with
    t + 1 <= k select every position), else over every causal key."""
    bi = torch.tensor([b for b, _ in rows], device=q.device)
    ii = torch.tensor([i for _, i in rows], device=q.device)
    qh, oh, lh = host_f64(q[bi, ii]), host_f64(out[bi, ii]), lse[bi, ii].cpu().double().numpy()
    ih = idx[bi, ii].cpu().numpy() if idx is not None else None
    lat_h = {b: host_f64(lat[b]) for b in sorted({b for b, _ in rows})}
    bad = []
    for r, (b, i) in enumerate(rows):
        t = q_offset + i
        sel = np.arange(t + 1) if ih is None else ih[r]
        ro, rl = O.sparse_attention_row(qh[r], lat_h[b][: t + 1], sel, scale, 512)
        bad += checks.close_errors(oh[r], ro, ATOL, RTOL, f"out[{b},{i}]")
        bad += checks.close_errors(lh[r], rl, 1e-3, 1e-3, f"lse[{b},{i}]")
    assert not bad, bad[:5]


def test_dense_causal_all_rows():
    """Plain causal attention over every key (no selection); 150 rows = 18
    full 8-token blocks and a ragged block of 6."""
    B, n = 2, 150
    q, lat = _inputs(B, n, n, 1)
    ws = dsa.Workspace("cuda")
    out, lse = dsa.attn_dense_prefill(q, lat, 512, scale=1 / 24, return_lse=True, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    _check_rows(q, lat, None, out, lse, 0, [(b, i) for b in range(B) for i in range(n)])


def test_dense_causal_chunk_with_offset():
    """A chunk of queries [100, 170) against keys [0, 300): keys past each
    row's position are never seen (the rest of the history is present)."""
    B, kv, q0, nq = 1, 300, 100, 70
    qall, lat = _inputs(B, kv, kv, 2)
    q = qall[:, q0:q0 + nq].contiguous()
    ws = dsa.Workspace("cuda")
    out, lse = dsa.attn_dense_prefill(q, lat, 512, q_offset=q0, scale=1 / 24, return_lse=True, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    _check_rows(q, lat, None, out, lse, q0, [(0, i) for i in range(nq)])


def test_dense_masked_equals_the_sparse_selection():
    """The indexer's own selection (integer workload, k = 64): rows with
    t + 1 <= k see every position, the others only their selection; the
    result is eq. (3) on that selection, as the gathering kernel computes."""
    w = W.scaled(W.PREFILL, B=2, n=700, HI=8, dI=64, k=64, seed=7)
    d = W.make_prefill_inputs(w, "cuda")
    ws = dsa.Workspace("cuda")
    idx = dsa.indexer_topk_prefill(d["qI"], d["kI"], d["w"], w.k, workspace=ws)
    out, lse = dsa.attn_dense_prefill(d["q"], d["latent"], 512, idx=idx, scale=w.scale, return_lse=True,
                                      workspace=ws)
    sp, sp_lse = dsa.sparse_attn_prefill(d["q"], d["latent"], idx, 512, scale=w.scale, return_lse=True,
                                         workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    rows = [(b, i) for b in range(2) for i in list(range(0, 70)) + list(range(330, 700, 7))]
    _check_rows(d["q"], d["latent"], idx, out, lse, 0, rows, w.scale)
    # the two engines agree with each other within the same bound
    diff = (out.float() - sp.float()).abs() - (ATOL + RTOL * sp.float().abs())
    assert float(diff.max()) <= 0.0
    assert float((lse - sp_lse).abs().max()) <= 2e-3


def test_dense_masked_random_selection_and_bad_index():
    """Seeded selections in random slot order (valid first, then -1), chunked
    with an offset, and one index past the history: it is reported and
    skipped."""
    B, kv, q0, nq, k = 2, 520, 200, 160, 96
    qall, lat = _inputs(B, kv, kv, 3)
    q = qall[:, q0:q0 + nq].contiguous()
    idx = W.make_selection(B, nq, kv, k, q_offset=q0, seed=5, device="cuda")
    bad = idx.clone()
    bad[1, 40, 3] = kv + 9
    ws = dsa.Workspace("cuda")
    out, lse = dsa.attn_dense_prefill(q, lat, 512, idx=bad, q_offset=q0, scale=1 / 24, return_lse=True,
                                      workspace=ws)
    st, detail = ws.status()
    assert st == 6 and detail == 0xA77E
    fixed = bad.clone()
    fixed[1, 40, 3] = -1
    _check_rows(q, lat, fixed, out, lse, q0, [(b, i) for b in range(B) for i in range(0, nq, 3)] + [(1, 40)])


def test_mass_coverage_matches_oracle():
    """M_k (eq. (15)) of the indexer's selection, per head and aggregated
    (eq. (16): heads summed, L1-normalised), from the lse of the sparse
    attention over the selection and of the dense causal attention."""
    w = W.scaled(W.PREFILL, B=1, n=600, HI=8, dI=64, k=48, seed=8)
    d = W.make_prefill_inputs(w, "cuda")
    ws = dsa.Workspace("cuda")
    idx = dsa.indexer_topk_prefill(d["qI"], d["kI"], d["w"], w.k, workspace=ws)
    _, lse_s = dsa.sparse_attn_prefill(d["q"], d["latent"], idx, 512, scale=w.scale, return_lse=True, workspace=ws)
    _, lse_d = dsa.attn_dense_prefill(d["q"], d["latent"], 512, scale=w.scale, return_lse=True, workspace=ws)
    m, mn, ph = dsa.mass_coverage(lse_s, lse_d, per_head=True)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    qh, lat, ih = host_f64(d["q"][0]), host_f64(d["latent"][0]), idx[0].cpu().numpy()
    m, mn, ph = m[0].cpu().double().numpy(), mn[0].cpu().double().numpy(), ph[0].cpu().double().numpy()
    for i in list(range(0, 60)) + list(range(60, 600, 11)):
        r = O.mass_coverage_row(qh[i], lat[: i + 1], ih[i], w.scale)
        assert abs(m[i] - r["M"]) <= 3e-3, (i, m[i], r["M"])
        assert np.all(np.abs(ph[i] - r["per_head"]) <= 3e-3), i
        assert abs(mn[i] - r["min"]) <= 3e-3
        if i + 1 <= w.k:
            assert abs(m[i] - 1.0) <= 3e-3          # every position selected


@pytest.mark.slow
def test_dense_masked_full_prefill_sampled():
    """n = 8192 prefill workload (k = 2048): the masked dense path on the
    fused indexer's selection, 256 sampled rows against the oracle."""
    w = W.PREFILL
    d = W.make_prefill_inputs(w, "cuda")
    ws = dsa.Workspace("cuda")
    idx = dsa.indexer_topk_prefill(d["qI"], d["kI"], d["w"], w.k, workspace=ws)
    out, lse = dsa.attn_dense_prefill(d["q"], d["latent"], 512, idx=idx, scale=w.scale, return_lse=True,
                                      workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    _check_rows(d["q"], d["latent"], idx, out, lse, 0, W.sample_rows(w, 256), w.scale)


def test_attn_prefill_length_dispatch_gives_the_same_result():
    """dsa_attn_prefill picks the dense masked path for a short history and
    the gathering path for a long one; on the same selection both equal the
    gathering kernel's output within the attention tolerance."""
    ws = dsa.Workspace("cuda")
    for kv, q0, nq, k in ((1000, 0, 1000, 128), (6300, 6150, 150, 96)):
        qall, lat = _inputs(1, kv, kv, 11 + kv)
        q = qall[:, q0:q0 + nq].contiguous()
        idx = W.make_selection(1, nq, kv, k, q_offset=q0, seed=kv, device="cuda")
        path = dsa.prefill_attention_path(1, nq, q0, kv, 16, 576, 512, k)
        assert path == (dsa.PATH_DENSE_MASKED if kv <= 6144 else dsa.PATH_GATHER)
        out, lse = dsa.attn_prefill(q, lat, idx, 512, q_offset=q0, scale=1 / 24, return_lse=True, workspace=ws)
        ref, ref_lse = dsa.sparse_attn_prefill(q, lat, idx, 512, scale=1 / 24, return_lse=True, workspace=ws)
        torch.cuda.synchronize()
        _no_device_errors(ws)
        diff = (out.float() - ref.float()).abs() - (ATOL + RTOL * ref.float().abs())
        assert float(diff.max()) <= 0.0
        assert float((lse - ref_lse).abs().max()) <= 2e-3
        _check_rows(q, lat, idx, out, lse, q0, [(0, i) for i in range(0, nq, 13)])
