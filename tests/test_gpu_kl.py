"""GPU parity of the sparse-stage indexer KL (eq. (8), §1.2 of the DSA page):
loss and gradients from the CUDA path (through the C ABI) against the CPU
oracle on the same seeded inputs.

The indexer inputs are integer-valued, so every q.k and every score is exact
in fp32 and the ReLU masks agree on both sides.  The remaining error comes
from fp32 softmax / log arithmetic and from the bf16 rounding of
G = g * w * [q.k > 0] before the two backward products.  The tolerances are
bounds derived from that arithmetic, evaluated per element with the oracle's
own quantities (unit roundoff of bf16 u = 2^-8; fp32 sums of <= 2048 terms):
  kl      : 1e-5 + 2e-6 * sum_s p_s (|log p_s| + |log softmax_s|)
  g_s     : 1e-5 * (softmax_s + p_s) * |grad_scale|
  dw_j    : sum_s |dg_s| ReLU(d_sj) + 1e-5 * sum_s |g_s| ReLU(d_sj)
  dq, dk  : (u + 1e-5) * (|G| |K|)  +  |dG| |K|   (resp. |Q|), |dG| from g's bound
"""

import numpy as np
import pytest
import torch

import learned_token_indexer_b200 as dsa
import oracle as O
from learned_token_indexer_b200 import workloads as W
from tests.gpu_util import host_f64

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def built():
    from learned_token_indexer_b200.build import build
    build()
    torch.cuda.init()
    yield


def _int_inputs(B, n, HI, dI, seed, qk_max=3, w_den=16):
    w = W.scaled(W.PREFILL, B=B, n=n, HI=HI, dI=dI, qk_int_max=qk_max, w_den=w_den, seed=seed)
    return W.make_prefill_inputs(w, device="cuda", with_attention=False)


def _row_bounds(q_t, k_all, w_t, sel, teacher, gs):
    """Per-element error bounds of one row (see the module docstring)."""
    v = sel >= 0
    HI, dI = q_t.shape
    K = sel.shape[0]
    zero = {"kl": 1e-5, "g": np.zeros(K), "dw": np.full(HI, 1e-7), "dq": np.full((HI, dI), 1e-7),
            "dk": np.zeros((K, dI))}
    if not v.any() or not teacher[v].sum() > 0:
        return zero
    kS = k_all[sel[v]]
    dots = kS @ q_t.T
    sc = np.maximum(dots, 0) @ w_t
    lq = sc - sc.max() - np.log(np.exp(sc - sc.max()).sum())
    qs = np.exp(lq)
    p = teacher[v] / teacher[v].sum()
    g = gs * (qs - p)
    dg = 1e-5 * (qs + p) * abs(gs)
    mask = dots > 0
    relu = np.maximum(dots, 0)
    with np.errstate(divide="ignore"):
        lp = np.where(p > 0, np.log(np.where(p > 0, p, 1.0)), 0.0)
    out = {"kl": 1e-5 + 2e-6 * float(np.sum(p * (np.abs(lp) + np.abs(lq))))}
    out["g"] = np.zeros(K)
    out["g"][v] = dg + 1e-12
    out["dw"] = dg @ relu + 1e-5 * (np.abs(g) @ relu) + 1e-7
    Gabs = np.abs(g)[:, None] * np.abs(w_t)[None, :] * mask          # [m, HI]
    dGabs = dg[:, None] * np.abs(w_t)[None, :] * mask
    out["dq"] = (U_BF16 + 1e-5) * (Gabs.T @ np.abs(kS)) + dGabs.T @ np.abs(kS) + 1e-7
    out["dk"] = np.zeros((K, dI))
    out["dk"][v] = (U_BF16 + 1e-5) * (Gabs @ np.abs(q_t)) + dGabs @ np.abs(q_t) + 1e-7
    return out


def _check_kl(d, idx, teacher, gs, res, rows, dk_rows_only=False):
    """Compare the GPU result with the oracle on the given (b, i) rows.

    dk is checked against the oracle's sum over exactly these rows (the GPU
    run must then have been made on these rows only when dk_rows_only)."""
    q, kk, w = host_f64(d["qI"]), host_f64(d["kI"]), host_f64(d["w"])
    idx_h = idx.cpu().numpy().astype(np.int64)
    t_h = teacher.cpu().double().numpy()
    kl = res["kl"].cpu().double().numpy()
    dq = res["dq"].cpu().double().numpy() if "dq" in res else None
    dw = res["dw"].cpu().double().numpy() if "dw" in res else None
    gl = res["grad_logits"].cpu().double().numpy() if "grad_logits" in res else None
    B, kv_len, dI = kk.shape
    dk_ref = np.zeros((B, kv_len, dI))
    dk_tol = np.zeros((B, kv_len, dI))
    for b, i in rows:
        r = O.indexer_kl_sparse_row(q[b, i], kk[b], w[b, i], idx_h[b, i], t_h[b, i], gs)
        bd = _row_bounds(q[b, i], kk[b], w[b, i], idx_h[b, i], t_h[b, i], gs)
        assert abs(kl[b, i] - r["kl"]) <= bd["kl"], (b, i, kl[b, i], r["kl"])
        if gl is not None:
            err = np.abs(gl[b, i] - r["grad_logits"])
            assert np.all(err <= bd["g"]), (b, i, err.max())
        if dw is not None:
            assert np.all(np.abs(dw[b, i] - r["dw"]) <= bd["dw"]), (b, i)
        if dq is not None:
            err = np.abs(dq[b, i] - r["dq"])
            assert np.all(err <= bd["dq"]), (b, i, err.max(), (err / bd["dq"]).max())
        v = idx_h[b, i] >= 0
        np.add.at(dk_ref[b], idx_h[b, i][v], r["dk"][v])
        np.add.at(dk_tol[b], idx_h[b, i][v], bd["dk"][v])
    if "dk" in res and dk_rows_only:
        dk = res["dk"].cpu().double().numpy()
        err = np.abs(dk - dk_ref)
        assert np.all(err <= dk_tol + 1e-6 * np.abs(dk_ref) + 1e-7), (err.max(), (err / (dk_tol + 1e-7)).max())


@pytest.mark.parametrize("B,n,HI,dI,k", [(2, 150, 64, 128, 80), (1, 200, 4, 32, 16), (2, 97, 16, 64, 64),
                                          (1, 130, 37, 128, 130), (1, 300, 64, 64, 4096)])
def test_kl_small_ragged_matches_oracle(B, n, HI, dI, k):
    d = _int_inputs(B, n, HI, dI, seed=11 + n)
    idx = W.make_selection(B, n, n, k, seed=n, device="cuda")
    teacher = W.make_teacher((B, n, k), seed=n, device="cuda")
    ws = dsa.Workspace("cuda")
    gs = 0.37
    res = dsa.indexer_kl_sparse(d["qI"], d["kI"], d["w"], idx, teacher, grad_scale=gs, grad_logits=True,
                                workspace=ws)
    torch.cuda.synchronize()
    st, detail = ws.status()
    assert st == 0, hex(detail)
    _check_kl(d, idx, teacher, gs, res, [(b, i) for b in range(B) for i in range(n)], dk_rows_only=True)


def test_kl_forward_only_and_partial_gradients():
    B, n, HI, dI, k = 1, 120, 64, 128, 64
    d = _int_inputs(B, n, HI, dI, seed=5)
    idx = W.make_selection(B, n, n, k, seed=5, device="cuda")
    teacher = W.make_teacher((B, n, k), seed=5, device="cuda")
    full = dsa.indexer_kl_sparse(d["qI"], d["kI"], d["w"], idx, teacher)
    fwd = dsa.indexer_kl_sparse(d["qI"], d["kI"], d["w"], idx, teacher, grads=())
    only_dw = dsa.indexer_kl_sparse(d["qI"], d["kI"], d["w"], idx, teacher, grads=("dw",))
    torch.cuda.synchronize()
    assert torch.equal(fwd["kl"], full["kl"]) and torch.equal(only_dw["kl"], full["kl"])
    assert torch.equal(only_dw["dw"], full["dw"])
    _check_kl(d, idx, teacher, 1.0, full, [(0, i) for i in range(n)], dk_rows_only=True)


def test_kl_degenerate_rows_and_bad_indices():
    B, n, HI, dI, k = 1, 64, 16, 64, 32
    d = _int_inputs(B, n, HI, dI, seed=6)
    idx = W.make_selection(B, n, n, k, seed=6, device="cuda")
    teacher = W.make_teacher((B, n, k), seed=6, device="cuda")
    idx[0, 40] = -1                                   # no valid slot
    teacher[0, 41] = 0.0                              # no teacher mass
    idx[0, 42, 3] = n + 5                             # out of range: skipped and reported
    ws = dsa.Workspace("cuda")
    res = dsa.indexer_kl_sparse(d["qI"], d["kI"], d["w"], idx, teacher, grad_logits=True, workspace=ws)
    torch.cuda.synchronize()
    st, detail = ws.status()
    assert st == 6 and detail == 0xA77E            # DSA_ERR_DEVICE_CHECK
    for i in (40, 41):
        assert res["kl"][0, i].item() == 0.0
        assert not res["dq"][0, i].any() and not res["dw"][0, i].any() and not res["grad_logits"][0, i].any()
    idx_clean = idx.clone()
    idx_clean[0, 42, 3] = -1                          # what the kernel did with the bad slot
    _check_kl(d, idx_clean, teacher, 1.0, res, [(0, i) for i in range(n)], dk_rows_only=True)


@pytest.mark.slow
def test_kl_full_prefill_workload_sampled():
    """n = 8192, H^I = 64, d^I = 128, k = 2048 in the launch the bench times:
    kl, grad_logits, dq, dw on 256 sampled rows of the full run; dk on a
    second run over exactly those rows (dk sums over rows)."""
    w = W.PREFILL
    d = W.make_prefill_inputs(w, device="cuda", with_attention=False)
    idx = W.make_selection(1, w.n, w.n, w.k, seed=w.seed, device="cuda")
    teacher = W.make_teacher((1, w.n, w.k), seed=w.seed, device="cuda")
    gs = 1.0 / w.n
    ws = dsa.Workspace("cuda")
    res = dsa.indexer_kl_sparse(d["qI"], d["kI"], d["w"], idx, teacher, grad_scale=gs, grad_logits=True,
                                workspace=ws)
    torch.cuda.synchronize()
    assert ws.status()[0] == 0
    rows = W.sample_rows(w, 256, salt=5)
    _check_kl(d, idx, teacher, gs, res, rows)
    sel = torch.tensor([i for _, i in rows], device="cuda")
    sub = {"qI": d["qI"][:, sel].contiguous(), "kI": d["kI"], "w": d["w"][:, sel].contiguous()}
    res2 = dsa.indexer_kl_sparse(sub["qI"], sub["kI"], sub["w"], idx[:, sel].contiguous(),
                                 teacher[:, sel].contiguous(), grad_scale=gs, workspace=ws)
    torch.cuda.synchronize()
    assert torch.allclose(res2["kl"], res["kl"][:, sel], rtol=0, atol=0)
    _check_kl(sub, idx[:, sel], teacher[:, sel], gs, res2, [(0, j) for j in range(len(rows))], dk_rows_only=True)
