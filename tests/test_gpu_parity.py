"""GPU parity: the CUDA path (called through the C ABI) against the CPU oracle
on the same seeded inputs.

Integer-valued indexer inputs give exact fp32 scores, so there indices must
match the oracle bit for bit (ties to the lower position on both sides).
Float inputs use the tolerance-aware selection check (tests/checks.py) and
attention uses |gpu - oracle| <= 2e-2 + 1e-2 |oracle| (bf16), 5e-2 for the
FP8 workload, with the oracle's eq. (3) run on the GPU's own indices.
"""

import math

import numpy as np
import pytest
import torch

import learned_token_indexer_b200 as dsa
import oracle as O
from learned_token_indexer_b200 import workloads as W
from tests import checks
from tests.gpu_util import host_dequant, host_f64, indexer_host_inputs

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 1e-2


@pytest.fixture(scope="module", autouse=True)
def built():
    from learned_token_indexer_b200.build import build
    build()
    torch.cuda.init()
    yield


def _ws():
    return dsa.Workspace("cuda")


def _no_device_errors(ws):
    st, detail = ws.status()
    assert st == 0, f"device status {dsa.STATUS.get(st)} detail 0x{detail:x}"


# --------------------------------------------------------------------------
# bounded waits and device checks
# --------------------------------------------------------------------------

def test_bounded_wait_times_out_with_status():
    ws = _ws()
    dsa.selftest_bounded_wait(2_000_000, ws)          # 2 ms
    st, detail = ws.status()
    assert st == 5 and detail == 0x7E57
    _no_device_errors(ws)                             # status was cleared
    x = torch.ones(4, device="cuda")                  # the context still works
    assert float(x.sum()) == 4.0


# --------------------------------------------------------------------------
# eq. (1): dense scores through the tcgen05 scan kernel
# --------------------------------------------------------------------------

@pytest.mark.parametrize("HI,dI", [(4, 32), (8, 64), (16, 128), (32, 96), (64, 128), (64, 64)])
def test_indexer_scores_integer_exact(HI, dI):
    w = W.scaled(W.TINY, B=2, n=300, HI=HI, dI=dI, qk_int_max=3, w_den=8, seed=11 + HI)
    d = W.make_prefill_inputs(w, "cuda", with_attention=False)
    ws = _ws()
    got = dsa.indexer_scores(d["qI"], d["kI"], d["w"], workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    q, k, wt = indexer_host_inputs(d)
    ref = O.indexer_scores(q, k, wt)
    assert np.array_equal(got.cpu().double().numpy(), ref)


def test_indexer_scores_with_offset_and_fp8():
    w = W.scaled(W.PREFILL_FP8, B=2, n=384, seed=5)
    d = W.make_prefill_inputs(w, "cuda", with_attention=False)
    ws = _ws()
    got = dsa.indexer_scores(d["qI"][:, 128:].contiguous(), d["kI"], d["w"][:, 128:].contiguous(), q_offset=128,
                             q_scale=d["q_scale"][:, 128:].contiguous(), k_scale=d["k_scale"], workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    q, k, wt = indexer_host_inputs(d)
    ref = O.indexer_scores(q[:, 128:], k, wt[:, 128:], q_offset=128)
    g = got.cpu().double().numpy()
    assert np.array_equal(np.isneginf(g), np.isneginf(ref))
    fin = np.isfinite(ref)
    scale = np.abs(ref[fin]).max()
    assert np.max(np.abs(g[fin] - ref[fin])) <= 1e-5 * scale


# --------------------------------------------------------------------------
# eq. (2): standalone row top-k
# --------------------------------------------------------------------------

@pytest.mark.parametrize("k", [1, 7, 64, 2048])
def test_topk_rows_exact_with_ties(k):
    g = torch.Generator().manual_seed(k)
    rows, ncols = 33, 5000
    s = torch.randint(-40, 40, (rows, ncols), generator=g).float() / 4     # many ties
    s[3] = 0.0
    s[4, ::2] = -0.0                                                       # -0 == +0
    s[5] = torch.randn(ncols, generator=g)
    lens = torch.randint(0, ncols + 1, (rows,), generator=g).int()
    lens[0], lens[1], lens[2] = 0, 1, ncols
    ws = _ws()
    idx, val = dsa.topk_rows(s.cuda(), k, row_len=lens.cuda(), return_values=True, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    idx, val = idx.cpu().numpy(), val.cpu().numpy()
    for r in range(rows):
        L = int(lens[r])
        if L == 0:
            assert np.all(idx[r] == -1)
            continue
        ref = O.causal_topk_row(s[r, :L].double().numpy(), L - 1, k)
        errs = checks.topk_exact_errors(idx[r], ref, L - 1, k)
        assert not errs, errs
        m = min(k, L)
        assert np.array_equal(val[r, :m], s[r, idx[r, :m]].numpy() + 0.0)


def _topk_rows_check(s, lens, k):
    ws = _ws()
    idx, val = dsa.topk_rows(s.cuda(), k, row_len=lens.cuda(), return_values=True, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    idx, val = idx.cpu().numpy(), val.cpu().numpy()
    for r in range(s.shape[0]):
        L = int(lens[r])
        ref = O.causal_topk_row(s[r, :L].double().numpy(), L - 1, k)
        errs = checks.topk_exact_errors(idx[r], ref, L - 1, k)
        assert not errs, (r, errs[:3])
        m = min(k, L)
        assert np.array_equal(val[r, :m], s[r, idx[r, :m]].numpy() + 0.0)


@pytest.mark.parametrize("k", [512, 2048])
def test_topk_rows_long_rows_sample_prefilter(k):
    """Rows of 8192..65536 entries take the sampled cut-off and the gather into
    shared memory; rows of an odd width start off the 16-byte grid (head and
    tail entries).  The result is the exact top-k."""
    g = torch.Generator().manual_seed(100 + k)
    rows, ncols = 8, 65543
    s = torch.randn((rows, ncols), generator=g)
    s[1] += torch.linspace(-3, 3, ncols)                   # a positional trend
    s[2] = torch.randn(ncols, generator=g).exp()           # skewed
    s[3, -3:] = 50.0                                       # the largest in the tail
    s[4, :3] = 50.0                                        # ... and in the head
    lens = torch.tensor([ncols, 65536, 40001, ncols, 20000, 8192, 8191, 4 * k + 1], dtype=torch.int32)
    _topk_rows_check(s, lens, k)


@pytest.mark.parametrize("k", [512, 2048])
def test_topk_rows_long_rows_prefilter_fallbacks(k):
    """Rows on which the sampled cut-off cannot work and the two-pass path
    takes over: the sampled entries (every 16th group of four in a 16-byte
    aligned row of 65536) hold the largest values, so fewer than k entries
    reach the cut-off; all entries equal; four distinct values (the gathered
    candidates overflow shared memory); a 0/1 row whose 1s are fewer than k."""
    g = torch.Generator().manual_seed(200 + k)
    rows, ncols = 5, 65536
    s = torch.randn((rows, ncols), generator=g)
    samp = (torch.arange(ncols) // 4) % 16 == 0
    s[0, samp] += 100.0
    s[1] = 0.25
    s[2] = torch.randint(0, 4, (ncols,), generator=g).float()
    s[3] = 0.0
    s[3, torch.randperm(ncols, generator=g)[: k // 2]] = 1.0
    s[4, samp] = 7.0
    lens = torch.full((rows,), ncols, dtype=torch.int32)
    _topk_rows_check(s, lens, k)


# --------------------------------------------------------------------------
# eqs. (1)+(2) fused, prefill
# --------------------------------------------------------------------------

def _prefill_exact(w, q_offset=0, nq=None, chunk=None, rows=None):
    d = W.make_prefill_inputs(w, "cuda", with_attention=False)
    n = w.n
    ws = _ws()
    if chunk is None:
        idx = dsa.indexer_topk_prefill(d["qI"], d["kI"], d["w"], w.k, workspace=ws)
    else:
        idx = torch.empty((w.B, n, w.k), dtype=torch.int32, device="cuda")
        for c0 in range(0, n, chunk):
            c1 = min(n, c0 + chunk)
            dsa.indexer_topk_prefill(d["qI"][:, c0:c1], d["kI"], d["w"][:, c0:c1], w.k, q_offset=c0,
                                     idx_out=idx[:, c0:c1], workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    q, k, wt = indexer_host_inputs(d)
    todo = rows if rows is not None else [(b, i) for b in range(w.B) for i in range(n)]
    ref = O.indexer_topk(q, k, wt, w.k, rows=todo)
    idx = idx.cpu().numpy()
    bad = []
    for b, i in todo:
        bad += checks.topk_exact_errors(idx[b, i], ref[b, i], i, w.k)
    assert not bad, bad[:5]


def test_prefill_wide_plan_integer_exact():
    """A chunk whose causal history reaches 16384 keys takes the wide
    accumulator plan of the fused indexer (bf16, H^I = 64: MMA N = 256, two
    accumulators of four tokens); the chunk before it, 16381 keys, keeps
    N = 128.  Integer values, so both are bit-exact against the oracle: every
    row of the wide chunk (67 rows, a ragged 8-token block at its end) and
    rows of the other around k and at its end."""
    w = W.scaled(W.PREFILL, B=1, n=16448, seed=5)
    rows = [(0, i) for i in range(16381, w.n)] + [(0, i) for i in (0, 2047, 2048, 2049, 8191, 16380)]
    _prefill_exact(w, chunk=16381, rows=rows)


def test_prefill_tiny_exact():
    _prefill_exact(W.TINY)


@pytest.mark.parametrize("HI,dI,n,k", [(64, 128, 1000, 100), (16, 64, 777, 33), (8, 32, 530, 300),
                                       (64, 128, 1100, 1)])
def test_prefill_integer_exact_ragged(HI, dI, n, k):
    w = W.scaled(W.PREFILL, B=2, n=n, HI=HI, dI=dI, k=k, seed=HI + n)
    _prefill_exact(w)


def test_prefill_bounded_workspace_second_pass():
    """History past 16384 keys with the bounded workspace: keys with equal
    scores everywhere but at 300 raised positions, so every token accepts its
    whole history and overflows its candidate buffer; 256 rows (four batches
    of the second pass) are recomputed and selected exactly: the raised keys
    up to t, then the lowest positions (eq. (2), ties to the lower position).
    The full-history workspace (no second pass) gives the same indices."""
    g = torch.Generator().manual_seed(31)
    B, kv, nq, HI, dI, k = 1, 20480, 256, 8, 64, 2048
    q0 = kv - nq
    base = torch.randint(-2, 3, (dI,), generator=g).float()
    kI = base.repeat(B, kv, 1)
    raised = torch.randperm(kv, generator=g)[:300]
    kI[0, raised] = 2 * base
    qI = base.repeat(B, nq, HI, 1) + torch.randint(0, 2, (B, nq, HI, dI), generator=g).float()
    w = torch.randint(1, 16, (B, nq, HI), generator=g).float() / 16
    qd, kd, wd = qI.bfloat16().cuda(), kI.bfloat16().cuda(), w.cuda()
    ws = _ws()
    idx = dsa.indexer_topk_prefill(qd, kd, wd, k, q_offset=q0, workspace=ws)
    full = dsa.indexer_topk_prefill(qd, kd, wd, k, q_offset=q0, workspace=ws, full_workspace=True)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    assert torch.equal(idx.sort(-1).values, full.sort(-1).values)     # slot order is unspecified
    rows = [(0, i) for i in range(0, nq, 5)] + [(0, nq - 1)]
    ref = O.indexer_topk(qI.double().numpy(), kI.double().numpy(), w.double().numpy(), k, q_offset=q0, rows=rows)
    idx = idx.cpu().numpy()
    bad = []
    for b, i in rows:
        bad += checks.topk_exact_errors(idx[b, i], ref[b, i], q0 + i, k)
    assert not bad, bad[:5]


def test_prefill_bounded_workspace_second_pass_fp8():
    """The bounded workspace's second pass with an e4m3 indexer: identical
    key rows get identical codes and scales (per-token quantisation), so the
    scores tie exactly and the selection is exact; every row of the chunk
    overflows and is recomputed by the e4m3 scan."""
    g = torch.Generator().manual_seed(32)
    B, kv, nq, HI, dI, k = 1, 18432, 160, 8, 64, 2048
    q0 = kv - nq
    base = torch.randn((dI,), generator=g)
    kI = base.repeat(B, kv, 1)
    raised = torch.randperm(kv, generator=g)[:200]
    kI[0, raised] = 2 * base
    qI = base.repeat(B, nq, HI, 1) + 0.25 * torch.randn((B, nq, HI, dI), generator=g)
    w = torch.rand((B, nq, HI), generator=g) + 0.1
    q8, qs = W.quantize_fp8_per_token(qI, 2)
    k8, ks = W.quantize_fp8_per_token(kI, 1)
    ws = _ws()
    args = (q8.cuda(), k8.cuda(), w.cuda(), k)
    idx = dsa.indexer_topk_prefill(*args, q_offset=q0, q_scale=qs.cuda(), k_scale=ks.cuda(), workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    qh, kh = host_dequant(q8, qs, 2), host_dequant(k8, ks, 1)
    rows = [(0, i) for i in range(0, nq, 7)] + [(0, nq - 1)]
    idx = idx.cpu().numpy()
    bad = []
    for b, i in rows:
        sc = O.indexer_scores_row(qh[b, i], kh[b, : q0 + i + 1], w[b, i].double().numpy())
        errs, _ = checks.topk_tolerant_errors(idx[b, i], sc, q0 + i, k)
        bad += errs
    assert not bad, bad[:5]


def test_prefill_chunked_equals_whole():
    w = W.scaled(W.PREFILL, B=1, n=1536, k=200, seed=77)
    _prefill_exact(w, chunk=512)


def test_prefill_scores_output_matches_oracle():
    w = W.scaled(W.PREFILL, B=1, n=640, k=64, seed=9)
    d = W.make_prefill_inputs(w, "cuda", with_attention=False)
    ws = _ws()
    idx, sc = dsa.indexer_topk_prefill(d["qI"], d["kI"], d["w"], w.k, return_scores=True, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    q, k, wt = indexer_host_inputs(d)
    full = O.indexer_scores(q, k, wt)
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    for i in range(w.n):
        m = min(w.k, i + 1)
        assert np.array_equal(sc[0, i, :m], full[0, i, idx[0, i, :m]])
        assert np.all(np.isneginf(sc[0, i, m:]))


def _prefill_tolerant(w, rows, chunk=None):
    d = W.make_prefill_inputs(w, "cuda", with_attention=False)
    ws = _ws()
    kw = {}
    if "q_scale" in d:
        kw = dict(q_scale=d["q_scale"], k_scale=d["k_scale"])
    if chunk is None:
        idx = dsa.indexer_topk_prefill(d["qI"], d["kI"], d["w"], w.k, workspace=ws, **kw)
    else:
        idx = torch.empty((w.B, w.n, w.k), dtype=torch.int32, device="cuda")
        for c0 in range(0, w.n, chunk):
            c1 = min(w.n, c0 + chunk)
            ckw = {}
            if kw:
                ckw = dict(q_scale=kw["q_scale"][:, c0:c1].contiguous(), k_scale=kw["k_scale"])
            dsa.indexer_topk_prefill(d["qI"][:, c0:c1], d["kI"], d["w"][:, c0:c1], w.k, q_offset=c0,
                                     idx_out=idx[:, c0:c1], workspace=ws, **ckw)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    idx = idx.cpu().numpy()
    q, k, wt = indexer_host_inputs(d)
    bad, overlaps = [], []
    for b, i in rows:
        s = O.indexer_scores_row(q[b, i], k[b, : i + 1], wt[b, i])
        errs, st = checks.topk_tolerant_errors(idx[b, i], s, i, w.k)
        bad += errs
        overlaps.append(st["overlap"])
    assert not bad, bad[:5]
    return float(np.mean(overlaps))


def test_prefill_fp8_small():
    w = W.scaled(W.PREFILL_FP8, B=2, n=2304, k=256, seed=21)
    ov = _prefill_tolerant(w, W.sample_rows(w, 96))
    assert ov > 0.99


def test_prefill_float_bf16_chunked():
    w = W.scaled(W.LONG, n=4096, k=512, chunk=1024, seed=31)
    ov = _prefill_tolerant(w, W.sample_rows(w, 96), chunk=1024)
    assert ov > 0.99


# --------------------------------------------------------------------------
# eq. (3): sparse attention
# --------------------------------------------------------------------------

def _attn_check(q, latent, idx, out, lse, scale, dv, rows, atol=ATOL, rtol=RTOL):
    qh, lh, ih = host_f64(q), host_f64(latent), idx.cpu().numpy()
    oh, lseh = host_f64(out), lse.cpu().double().numpy()
    bad = []
    for b, i in rows:
        ro, rl = O.sparse_attention_row(qh[b, i], lh[b], ih[b, i], scale, dv)
        bad += checks.close_errors(oh[b, i], ro, atol, rtol, f"out[{b},{i}]")
        bad += checks.close_errors(lseh[b, i], rl, 1e-3, 1e-3, f"lse[{b},{i}]")
    assert not bad, bad[:5]


def test_attention_tiny_full():
    w = W.TINY
    d = W.make_prefill_inputs(w, "cuda")
    ws = _ws()
    idx = dsa.indexer_topk_prefill(d["qI"], d["kI"], d["w"], w.k, workspace=ws)
    out, lse = dsa.sparse_attn_prefill(d["q"], d["latent"], idx, w.Dv, scale=w.scale, return_lse=True, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    _attn_check(d["q"], d["latent"], idx, out, lse, w.scale, w.Dv, [(0, i) for i in range(w.n)])


def test_attention_mla_shapes_random_indices():
    # 576/512 latent rows, 16 heads, random valid / -1 slots, ragged k
    g = torch.Generator(device="cuda").manual_seed(3)
    B, nq, kv, H, k = 2, 40, 3000, 16, 300
    q = torch.randn((B, nq, H, 576), generator=g, device="cuda").bfloat16()
    lat = torch.randn((B, kv, 576), generator=g, device="cuda").bfloat16()
    idx = torch.randint(0, kv, (B, nq, k), generator=g, device="cuda", dtype=torch.int32)
    idx[:, :, 250:] = -1
    idx[0, 0, :] = -1                       # a row with nothing selected
    idx[1, 3, 5:] = -1
    ws = _ws()
    out, lse = dsa.sparse_attn_prefill(q, lat, idx, 512, scale=1 / 24, return_lse=True, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    assert torch.all(out[0, 0] == 0) and torch.all(torch.isneginf(lse[0, 0]))
    _attn_check(q, lat, idx, out, lse, 1 / 24, 512, [(b, i) for b in range(B) for i in range(nq)])


def test_attention_bad_index_is_reported_and_skipped():
    B, nq, kv, H, k = 1, 4, 100, 16, 32
    q = torch.randn((B, nq, H, 64), device="cuda").bfloat16()
    lat = torch.randn((B, kv, 64), device="cuda").bfloat16()
    idx = torch.randint(0, kv, (B, nq, k), device="cuda", dtype=torch.int32)
    idx[0, 2, 7] = kv + 5
    ws = _ws()
    out, lse = dsa.sparse_attn_prefill(q, lat, idx, 64, scale=0.125, return_lse=True, workspace=ws)
    st, detail = ws.status()
    assert st == 6 and detail == 0xA77E
    fixed = idx.clone()
    fixed[0, 2, 7] = -1
    _attn_check(q, lat, fixed, out, lse, 0.125, 64, [(0, i) for i in range(nq)])


def test_worked_example_through_the_library():
    """The page's three-token example (§1.1, eqs. (4)-(6)) embedded in padded
    shapes: H_I 2 -> 4 and d_I 2 -> 32 with zero rows / weights (exact)."""
    n, HI, dI = 3, 4, 32
    qI = torch.zeros((1, n, HI, dI))
    qI[0, 2, 0, 0] = 1.0
    qI[0, 2, 1, 1] = 1.0
    kI = torch.zeros((1, n, dI))
    kI[0, :, :2] = torch.tensor([[2.0, -1.0], [1.0, 3.0], [-1.0, 4.0]])
    w = torch.zeros((1, n, HI))
    w[0, 2, :2] = torch.tensor([0.75, 0.25])
    ws = _ws()
    args = (qI.bfloat16().cuda(), kI.bfloat16().cuda(), w.cuda())
    sc = dsa.indexer_scores(*args, workspace=ws)
    assert sc[0, 2].tolist() == [1.5, 1.5, 1.0]
    idx, val = dsa.indexer_topk_prefill(*args, 2, return_scores=True, workspace=ws)
    assert sorted(idx[0, 2].tolist()) == [0, 1]
    assert sorted(val[0, 2].tolist()) == [1.5, 1.5]
    idx1 = dsa.indexer_topk_prefill(*args, 1, workspace=ws)
    assert idx1[0, 2].tolist() == [0]
    # attention half: logits 0.2 / 1.2 on values (2,0) / (0,3), through a
    # constructed latent row c_s = (v_s, 0.., a_s) and q = (0.., 1), scale 1
    lat = torch.zeros((1, n, 64))
    lat[0, 0, :2] = torch.tensor([2.0, 0.0])
    lat[0, 1, :2] = torch.tensor([0.0, 3.0])
    lat[0, :, 63] = torch.tensor([0.2, 1.2, 2.0])
    q = torch.zeros((1, n, 1, 64))
    q[0, :, 0, 63] = 1.0
    out = dsa.sparse_attn_prefill(q.bfloat16().cuda(), lat.bfloat16().cuda(), idx, 64, scale=1.0, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    o = out[0, 2, 0, :2].float().cpu().numpy()
    assert np.allclose(o, [0.538, 2.193], atol=1e-2)          # bf16 logits 0.2002 / 1.2031


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------

def _decode_case(w, lengths, attention=True):
    d = W.make_decode_inputs(w, "cuda", lengths=lengths)
    total, maxlen = int(lengths.sum()), int(lengths.max())
    ws = _ws()
    idx = dsa.indexer_topk_decode(d["qI"], d["w"], d["kI_cache"], d["cu_seqlens"], w.k, total, maxlen,
                                  q_scale=d.get("q_scale"), k_scale=d.get("k_scale"), workspace=ws)
    out, lse = dsa.sparse_attn_decode(d["q"], d["latent_cache"], d["cu_seqlens"], idx, w.Dv, total, scale=w.scale,
                                      return_lse=True, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    cu = d["cu_seqlens"].cpu().numpy()
    if w.fp8:   # the oracle scores the dequantised codes (the quantisation is an input)
        qh, kh = host_dequant(d["qI"], d["q_scale"], 2), host_dequant(d["kI_cache"], d["k_scale"], 1)
    else:
        qh, kh = host_f64(d["qI"]), host_f64(d["kI_cache"])
    wh = host_f64(d["w"])
    idx_h = idx.cpu().numpy()
    bad = []
    for b in range(len(lengths)):
        s = O.indexer_scores_row(qh[b], kh[cu[b]:cu[b + 1]], wh[b])
        errs, _ = checks.topk_tolerant_errors(idx_h[b], s, int(lengths[b]) - 1, w.k)
        bad += errs
    assert not bad, bad[:5]
    if not attention:
        return
    ro, rl = O.decode_sparse_attention(host_f64(d["q"]), host_f64(d["latent_cache"]), cu, idx_h, w.scale, w.Dv)
    bad = checks.close_errors(host_f64(out), ro, ATOL, RTOL, "decode out")
    bad += checks.close_errors(lse.cpu().double().numpy(), rl, 1e-3, 1e-3, "decode lse")
    assert not bad, bad


def test_decode_small_ragged():
    w = W.scaled(W.DECODE, B=5, k=300)
    _decode_case(w, torch.tensor([1, 129, 300, 1000, 4097]))


def test_decode_fp8_cache_small_ragged():
    # e4m3 K^I cache with one scale per key, e4m3 queries with one scale per token
    w = W.scaled(W.DECODE_FP8, B=5, k=300)
    _decode_case(w, torch.tensor([1, 129, 300, 1000, 4097]))


def test_decode_lengths_around_the_selection_thresholds():
    """Sequences at the row top-k's boundaries with k = 2048: t + 1 = k - 1,
    k, k + 1 (everything / all but one selected), just below, at and above
    the sampled cut-off's 8192-entry minimum, and around the 16384 entries
    where the sample switches to 1024 entries."""
    w = W.scaled(W.DECODE, k=2048)
    _decode_case(w, torch.tensor([2047, 2048, 2049, 8191, 8192, 8193, 16383, 16384, 16389]), attention=False)


def test_decode_selection_with_equal_scores():
    """Decode selection on caches whose keys mostly repeat one vector, so the
    scan's histogram puts whole sequences into one cut-off bin: more entries
    than shared memory holds for the longest (the refinement then runs over
    the row), a sequence whose raised keys all fit, and short ones.  Integer
    values: the selection is exact (equal scores go to the lower position)."""
    g = torch.Generator().manual_seed(41)
    lengths = torch.tensor([40000, 20000, 2100, 5])
    B, HI, dI, k = lengths.numel(), 16, 64, 2048
    cu = torch.zeros(B + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    total = int(cu[-1])
    base = torch.randint(-2, 3, (dI,), generator=g).float()
    kc = base.repeat(total, 1)
    raised = torch.randperm(total, generator=g)[:700]
    kc[raised] = 2 * base
    q = base.repeat(B, HI, 1) + torch.randint(0, 2, (B, HI, dI), generator=g).float()
    w = torch.randint(1, 16, (B, HI), generator=g).float() / 16
    ws = _ws()
    idx = dsa.indexer_topk_decode(q.bfloat16().cuda(), w.cuda(), kc.bfloat16().cuda(), cu.cuda(), k, total,
                                  int(lengths.max()), workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    ref = O.decode_indexer_topk(q.double().numpy(), w.double().numpy(), kc.double().numpy(), cu, k)
    idx = idx.cpu().numpy()
    bad = []
    for b in range(B):
        bad += checks.topk_exact_errors(idx[b], ref[b], int(lengths[b]) - 1, k)
    assert not bad, bad[:5]


def test_decode_selection_long_rows_exact():
    """Long ragged sequences (65536, 50001, 32771, 40000, 16385 and 9000
    cached keys, which take the sampled cut-off of the row top-k) beside a
    3-key one, and a sequence whose highest scores are 3000 equal keys at its
    end, so the cut-off falls inside a tie.  Integer values, so the selection
    is exact (ties to the lower position)."""
    g = torch.Generator().manual_seed(43)
    lengths = torch.tensor([65536, 50001, 32771, 40000, 16385, 9000, 3])
    B, HI, dI, k = lengths.numel(), 16, 64, 2048
    cu = torch.zeros(B + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    total = int(cu[-1])
    kc = torch.randint(-3, 4, (total, dI), generator=g).float()
    # sequence 3: positive queries, and its last 3000 keys all equal to 3, so
    # they score far above the rest (and tie among themselves)
    q = torch.randint(-3, 4, (B, HI, dI), generator=g).float()
    q[3] = q[3].abs() + 1
    s3 = int(cu[3])
    kc[s3 + 37000:s3 + 40000] = 3.0
    w = torch.randint(1, 16, (B, HI), generator=g).float() / 16
    ws = _ws()
    idx = dsa.indexer_topk_decode(q.bfloat16().cuda(), w.cuda(), kc.bfloat16().cuda(), cu.cuda(), k, total,
                                  int(lengths.max()), workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    ref = O.decode_indexer_topk(q.double().numpy(), w.double().numpy(), kc.double().numpy(), cu, k)
    idx = idx.cpu().numpy()
    bad = []
    for b in range(B):
        bad += checks.topk_exact_errors(idx[b], ref[b], int(lengths[b]) - 1, k)
    assert not bad, bad[:5]
    # sequence 3's selection is its raised block's first 2048 keys (ties to the lower position)
    assert sorted(idx[3]) == list(range(37000, 37000 + k))


def test_decode_attention_scattered_and_bad_slots():
    """The decode step's attention (128 heads, 576/512 latent rows: the
    tensor-core kernel whose two CTAs split the latent columns) on ragged
    sequences whose index rows hold -1 anywhere, a row with one usable slot,
    an empty row and an index past the sequence end, which is reported and
    skipped."""
    g = torch.Generator().manual_seed(12)
    lengths = torch.tensor([3000, 1, 700, 2500, 64, 129])
    B, H, k, Dqk, Dv = lengths.numel(), 128, 640, 576, 512
    cu = torch.zeros(B + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    total = int(cu[-1])
    q = torch.randn((B, H, Dqk), generator=g).bfloat16().cuda()
    lat = torch.randn((total, Dqk), generator=g).bfloat16().cuda()
    idx = torch.full((B, k), -1, dtype=torch.int32)
    for b in range(B):
        L = int(lengths[b])
        m = min(k, L)
        idx[b, :m] = torch.randperm(L, generator=g)[:m].int()
        drop = torch.rand(k, generator=g) < 0.3
        idx[b, drop] = -1                       # unused slots anywhere in the row
    idx[1] = -1
    idx[1, 5] = 0                               # one usable slot, not the first
    idx[4] = -1                                 # nothing selected
    bad = idx.clone()
    bad[2, 77] = int(lengths[2]) + 3            # past the end of sequence 2
    ws = _ws()
    out, lse = dsa.sparse_attn_decode(q, lat, cu.cuda(), bad.cuda(), Dv, total, scale=1 / 24, return_lse=True,
                                      workspace=ws)
    st, detail = ws.status()
    assert st == 6 and detail == 0xA77E
    fixed = bad.clone()
    fixed[2, 77] = -1
    ro, rl = O.decode_sparse_attention(host_f64(q), host_f64(lat), cu.numpy(), fixed.numpy(), 1 / 24, Dv)
    o, l_ = host_f64(out), lse.cpu().double().numpy()
    assert np.all(o[4] == 0) and np.all(np.isneginf(l_[4]))
    errs = checks.close_errors(o, ro, ATOL, RTOL, "decode out") + checks.close_errors(l_, rl, 1e-3, 1e-3, "lse")
    assert not errs, errs
    # the same call twice gives the same bits (no state kept between launches)
    out2 = dsa.sparse_attn_decode(q, lat, cu.cuda(), fixed.cuda(), Dv, total, scale=1 / 24, workspace=ws)
    out3 = dsa.sparse_attn_decode(q, lat, cu.cuda(), fixed.cuda(), Dv, total, scale=1 / 24, workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    assert torch.equal(out2, out3)


@pytest.mark.slow
def test_decode_full_workload():
    _decode_case(W.DECODE, W.decode_lengths(W.DECODE))


@pytest.mark.slow
def test_decode_fp8_full_workload():
    _decode_case(W.DECODE_FP8, W.decode_lengths(W.DECODE_FP8))


# --------------------------------------------------------------------------
# full-size workloads, sampled rows
# --------------------------------------------------------------------------

def _attn_check_rows(q, latent, idx, out, lse, scale, dv, rows, atol=ATOL, rtol=RTOL):
    """The oracle's eq. (3) on the GPU's own indices for a sample of rows;
    only the sampled rows (and each sampled sequence's latent rows) are
    copied to the host."""
    bs = sorted({b for b, _ in rows})
    lat = {b: host_f64(latent[b]) for b in bs}
    bi = torch.tensor([b for b, _ in rows], device=q.device)
    ii = torch.tensor([i for _, i in rows], device=q.device)
    qh, ih = host_f64(q[bi, ii]), idx[bi, ii].cpu().numpy()
    oh, lseh = host_f64(out[bi, ii]), lse[bi, ii].cpu().double().numpy()
    bad = []
    for r, (b, i) in enumerate(rows):
        ro, rl = O.sparse_attention_row(qh[r], lat[b], ih[r], scale, dv)
        bad += checks.close_errors(oh[r], ro, atol, rtol, f"out[{b},{i}]")
        bad += checks.close_errors(lseh[r], rl, 1e-3, 1e-3, f"lse[{b},{i}]")
    assert not bad, bad[:5]


def _full_prefill_case(w, nrows=256, atol=ATOL, rtol=RTOL):
    """A full-size prefill workload through the library in the launch
    configuration the benchmark times (whole sequence, or chunks of w.chunk
    queries against the full causal history): fused indexer + top-k, then
    sparse attention with lse.  Checked on a seeded sample of nrows query rows
    (rows 0, 1, k-2, k-1, k, the last row and every chunk's first and last
    row always included): integer workloads bit-exact on the index sets,
    float workloads with the tolerance-aware selection check, and the
    attention output against the oracle's eq. (3) on the GPU's indices."""
    d = W.make_prefill_inputs(w, "cuda")
    ws = _ws()
    chunk = w.chunk or w.n
    idx = torch.empty((w.B, w.n, w.k), dtype=torch.int32, device="cuda")
    out = torch.empty((w.B, w.n, w.H, w.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((w.B, w.n, w.H), dtype=torch.float32, device="cuda")
    for c0 in range(0, w.n, chunk):
        c1 = min(w.n, c0 + chunk)
        sl = (slice(None), slice(c0, c1))
        kw = {}
        if "q_scale" in d:
            kw = dict(q_scale=d["q_scale"][sl].contiguous(), k_scale=d["k_scale"])
        dsa.indexer_topk_prefill(d["qI"][sl], d["kI"], d["w"][sl], w.k, q_offset=c0, idx_out=idx[sl],
                                 workspace=ws, **kw)
        dsa.sparse_attn_prefill(d["q"][sl], d["latent"], idx[sl], w.Dv, scale=w.scale, out=out[sl], lse=lse[sl],
                                workspace=ws)
    torch.cuda.synchronize()
    _no_device_errors(ws)
    rows = W.sample_rows(w, nrows)
    assert len(rows) >= nrows
    # host copies of the sampled query rows only (a full float64 copy of q^I
    # would be several GB); every sequence's keys in full
    bi = torch.tensor([b for b, _ in rows], device="cuda")
    ii = torch.tensor([i for _, i in rows], device="cuda")
    if "q_scale" in d:
        q = host_dequant(d["qI"][bi, ii], d["q_scale"][bi, ii], 2)
        k = host_dequant(d["kI"], d["k_scale"], 1)
    else:
        q, k = host_f64(d["qI"][bi, ii]), host_f64(d["kI"])
    wt = host_f64(d["w"][bi, ii])
    ih = idx[bi, ii].cpu().numpy()
    bad, overlaps = [], []
    for r, (b, i) in enumerate(rows):
        s = O.indexer_scores_row(q[r], k[b, : i + 1], wt[r])
        if w.integer_valued:
            bad += checks.topk_exact_errors(ih[r], O.causal_topk_row(s, i, w.k), i, w.k)
        else:
            errs, st = checks.topk_tolerant_errors(ih[r], s, i, w.k)
            bad += errs
            overlaps.append(st["overlap"])
    assert not bad, bad[:5]
    del q, k, wt
    _attn_check_rows(d["q"], d["latent"], idx, out, lse, w.scale, w.Dv, rows, atol, rtol)
    return float(np.mean(overlaps)) if overlaps else 1.0


@pytest.mark.slow
def test_prefill_full_integer_workload_sampled():
    """n = 8192 integer-valued prefill: indices bit-exact, attention within
    2e-2 + 1e-2 |ref| on 256 sampled rows."""
    _full_prefill_case(W.PREFILL)


@pytest.mark.slow
def test_prefill_full_fp8_workload_sampled():
    """B = 2, n = 32768 FP8-e4m3 indexer: tolerance-aware selection on the
    dequantised oracle scores, attention within 5e-2 (abs and rel) on 256
    sampled rows."""
    ov = _full_prefill_case(W.PREFILL_FP8, atol=5e-2, rtol=5e-2)
    assert ov > 0.98


@pytest.mark.slow
def test_long_prefill_chunked_sampled():
    """n = 131072 bf16 prefill in 8192-query chunks against the full causal
    history: selection and attention on 256 sampled rows including every
    chunk boundary."""
    ov = _full_prefill_case(W.LONG)
    assert ov > 0.98


# --------------------------------------------------------------------------
# selection diagnostic (eq. (14))
# --------------------------------------------------------------------------

def test_selection_overlap_matches_oracle_recall():
    g = torch.Generator().manual_seed(14)
    rows, k, max_pos = 40, 64, 300
    a = torch.stack([torch.randperm(max_pos, generator=g)[:k] for _ in range(rows)]).int()
    b = torch.stack([torch.randperm(max_pos, generator=g)[:k] for _ in range(rows)]).int()
    b[:5] = a[:5].flip(-1)                      # identical sets in another order
    for r in range(5, 10):                      # half shared, positions distinct within the row
        keep = a[r, : k // 2]
        rest = [int(x) for x in torch.randperm(max_pos, generator=g) if int(x) not in set(keep.tolist())]
        b[r] = torch.cat([keep, torch.tensor(rest[: k - k // 2], dtype=torch.int32)])
    a[10:15, 40:] = -1                          # short rows padded with -1
    b[15:20] = -1                               # empty student
    a[20:25] = -1                               # empty teacher
    inter, cnt = dsa.selection_overlap(a.cuda(), b.cuda(), max_pos, return_counts=True)
    torch.cuda.synchronize()
    inter, cnt = inter.cpu().numpy(), cnt.cpu().numpy()
    for r in range(rows):
        assert cnt[r] == int((a[r] >= 0).sum())
        rec = inter[r] / cnt[r] if cnt[r] else 1.0
        assert rec == O.selection_recall_row(a[r].numpy(), b[r].numpy()), r
