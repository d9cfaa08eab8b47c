"""Pins of the CPU oracle against facts fixed by the DSA page and by mathematics.

None of these tests re-run the oracle's own formula: each compares it with a
printed value (the page's worked example), an exact brute force written with
different arithmetic (Python integers / fractions), a library routine for a
special case (torch's scaled_dot_product_attention, torch's FP8 cast), or an
invariant the page states (order invariance §3.1, renormalisation eq. (19)
and bound eq. (20) §3.2).
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _worked():
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# FP8 decoding
# --------------------------------------------------------------------------

def test_e4m3_decode_known_codes():
    v = O.e4m3_to_float64(np.array([0x38, 0x7E, 0x01, 0x08, 0xB8, 0x00, 0x80, 0x7F], dtype=np.uint8))
    assert v[0] == 1.0
    assert v[1] == 448.0            # largest finite e4m3
    assert v[2] == 2.0 ** -9        # smallest subnormal
    assert v[3] == 2.0 ** -6        # smallest normal
    assert v[4] == -1.0
    assert v[5] == 0.0 and v[6] == 0.0
    assert math.isnan(v[7])


def test_e4m3_decode_matches_torch_cast():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_to_float64(codes.numpy())
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[finite], ref[finite])


def test_dequantize_scales_each_token_group():
    """Dequantised value = code value x the scale of its token (§2: quantised
    indexer key cache with its scales).  Keys carry one scale per key over
    d^I (one trailing axis); queries one scale per token over H^I x d^I (two
    trailing axes).  Scales are distinct and neither 1 nor self-reciprocal,
    so a scale divided instead of multiplied, or broadcast over the head axis
    instead of the token axis, changes the values checked here."""
    # codes 0x38 = 1.0, 0x40 = 2.0, 0xB0 = -0.5, 0x00 = 0.0, 0x44 = 3.0
    one, two, mhalf, zero, three = 0x38, 0x40, 0xB0, 0x00, 0x44
    keys = np.array([[one, two, mhalf], [three, zero, one]], dtype=np.uint8)      # [2 keys, 3 dims]
    kscale = np.array([0.25, 3.0])
    got = O.dequantize(keys, kscale, 1)
    assert got.shape == (2, 3)
    assert got.tolist() == [[0.25, 0.5, -0.125], [9.0, 0.0, 3.0]]

    # queries [3 tokens, 2 heads, 2 dims]; the head count (2) differs from the
    # token count (3), and token 1's scale differs from head 1's position
    q = np.array([[[one, two], [three, mhalf]],
                  [[one, one], [two, zero]],
                  [[mhalf, three], [one, two]]], dtype=np.uint8)
    qscale = np.array([2.0, 0.125, 5.0])
    got = O.dequantize(q, qscale, 2)
    assert got.shape == (3, 2, 2)
    want = [[[2.0, 4.0], [6.0, -1.0]],
            [[0.125, 0.125], [0.25, 0.0]],
            [[-2.5, 15.0], [5.0, 10.0]]]
    assert got.tolist() == want
    # leading batch axis: [B=2, tokens=3] scales over [B, tokens, H, d] codes
    got_b = O.dequantize(np.stack([q, q]), np.stack([qscale, qscale[::-1]]), 2)
    assert got_b[0].tolist() == want
    assert got_b[1, 0].tolist() == (np.array(want[0]) / 2.0 * 5.0).tolist()
    assert got_b[1, 2].tolist() == (np.array(want[2]) / 5.0 * 2.0).tolist()


# --------------------------------------------------------------------------
# Worked example of §1.1 (eqs. (4)-(6) and the text after them)
# --------------------------------------------------------------------------

def test_worked_example_scores():
    g = _worked()
    s = O.indexer_scores_row(np.array(g["q"], float), np.array(g["keys"], float), np.array(g["w"]))
    assert s.tolist() == g["scores"]
    # the per-head ReLU table printed on the page
    dots = np.array(g["keys"], float) @ np.array(g["q"], float).T
    assert np.maximum(dots, 0).tolist() == g["per_head_relu"]


def test_worked_example_selection():
    g = _worked()
    s = np.array(g["scores"])
    t = len(s) - 1                       # the query is the third token (0-based t = 2)
    idx = O.causal_topk_row(s, t, g["k"])
    assert sorted(idx.tolist()) == g["selected_positions_0based"]
    assert [p + 1 for p in sorted(idx.tolist())] == g["selected_positions_1based"]
    # derived from the tie rule (lower position wins) and eq. (2)
    assert O.causal_topk_row(s, t, 1).tolist() == [0]
    assert O.causal_topk_row(s, t, 3).tolist() == [0, 1, 2]
    assert O.causal_topk_row(s, t, 5).tolist() == [0, 1, 2, -1, -1]


def _example_attention_inputs(g):
    # Embedding of the printed logits: c_s = (v_s | a_s), q = (0, 0 | 1), scale 1,
    # so scale * q . c_s = a_s exactly and the value is the first 2 columns.
    a = g["attention_logits"] + [g["miss_case_logit_position3"]]
    v = g["attention_values"] + [[7.0, -5.0]]      # any value for position 3
    latent = np.array([vi + [ai] for vi, ai in zip(v, a)], float)
    q = np.array([[0.0, 0.0, 1.0]])
    return q, latent


def test_worked_example_attention():
    g = _worked()
    q, latent = _example_attention_inputs(g)
    out, lse = O.sparse_attention_row(q, latent, np.array(g["selected_positions_0based"]), 1.0, 2)
    tol = 0.5 * 10 ** -g["printed_decimals"]
    e = np.exp(np.array(g["attention_logits"]))
    weights = e / e.sum()
    assert np.allclose(weights, g["attention_weights_printed"], atol=tol, rtol=0)
    assert np.allclose(out[0], g["attention_output_printed"], atol=tol, rtol=0)
    assert abs(out[0, 0] - 0.537883) < 1e-6 and abs(out[0, 1] - 2.193176) < 1e-6
    assert abs(lse[0] - math.log(math.exp(0.2) + math.exp(1.2))) < 1e-12


def test_worked_example_miss_case_renormalises():
    """If position 3 had the largest full logit, the sparse softmax still only
    renormalises over {1, 2} (1-based): the output is unchanged by position 3."""
    g = _worked()
    q, latent = _example_attention_inputs(g)
    sparse, _ = O.sparse_attention_row(q, latent, np.array([0, 1, -1]), 1.0, 2)
    dense, _ = O.sparse_attention_row(q, latent, np.array([0, 1, 2]), 1.0, 2)
    assert np.allclose(sparse[0], g["attention_output_printed"], atol=5e-4)
    assert not np.allclose(dense, sparse, atol=1e-2)


# --------------------------------------------------------------------------
# Eq. (1) special cases and invariants
# --------------------------------------------------------------------------

def test_single_head_unit_weight_is_relu_of_dot():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 16))
    k = rng.standard_normal((40, 16))
    s_pos = O.indexer_scores_row(q, k, np.array([1.0]))
    s_neg = O.indexer_scores_row(q, k, np.array([-1.0]))
    for j in range(40):
        d = float(np.dot(q[0], k[j]))
        assert s_pos[j] == pytest.approx(max(d, 0.0), rel=1e-12, abs=1e-12)
        assert s_neg[j] == pytest.approx(-max(d, 0.0), rel=1e-12, abs=1e-12)


def test_scores_are_linear_in_head_weights():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((8, 32))
    k = rng.standard_normal((50, 32))
    w1, w2 = rng.standard_normal(8), rng.standard_normal(8)
    s1 = O.indexer_scores_row(q, k, w1)
    s2 = O.indexer_scores_row(q, k, w2)
    assert np.allclose(O.indexer_scores_row(q, k, w1 + w2), s1 + s2, atol=1e-12)
    assert np.allclose(O.indexer_scores_row(q, k, -3.0 * w1), -3.0 * s1, atol=1e-12)


def test_relu_drops_negative_dots_and_negative_weights_subtract():
    # every key has a negative dot product with head 0 and positive with head 1
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    k = np.array([[-1.0, 2.0], [-3.0, 0.5]])
    s = O.indexer_scores_row(q, k, np.array([5.0, -1.0]))
    assert s.tolist() == [-2.0, -0.5]
    s0 = O.indexer_scores_row(q, k, np.array([5.0, 0.0]))
    assert s0.tolist() == [0.0, 0.0] and not np.signbit(s0).any()


def test_positive_head_scaling_and_query_scaling_commute_with_relu():
    # ReLU(c x) = c ReLU(x) for c > 0: scaling a head's query by c equals
    # scaling its weight by c (this is what lets FP8 query scales fold into w).
    rng = np.random.default_rng(2)
    q = rng.standard_normal((4, 16))
    k = rng.standard_normal((30, 16))
    w = rng.standard_normal(4)
    c = np.array([0.5, 2.0, 3.0, 0.25])
    a = O.indexer_scores_row(q * c[:, None], k, w)
    b = O.indexer_scores_row(q, k, w * c)
    assert np.allclose(a, b, atol=1e-12)


def test_prefill_scores_causal_mask_and_offset():
    rng = np.random.default_rng(3)
    B, n, HI, dI = 2, 12, 3, 8
    q = rng.integers(-3, 4, (B, n, HI, dI)).astype(float)
    k = rng.integers(-3, 4, (B, n, dI)).astype(float)
    w = rng.integers(-4, 5, (B, n, HI)) / 4.0
    full = O.indexer_scores(q, k, w)
    for b in range(B):
        for t in range(n):
            assert np.all(np.isneginf(full[b, t, t + 1:]))
            assert np.all(np.isfinite(full[b, t, : t + 1]))
    # a chunk of queries starting at position 5 sees the same rows
    part = O.indexer_scores(q[:, 5:9], k, w[:, 5:9], q_offset=5)
    assert np.array_equal(part, full[:, 5:9])


# --------------------------------------------------------------------------
# Eq. (2): selection
# --------------------------------------------------------------------------

def _brute_scores_fraction(q, k, w_num, w_den):
    """Exact eq. (1) with Python integers and Fractions, explicit loops."""
    HI, dI = len(q), len(q[0])
    out = []
    for ks in k:
        total = Fraction(0)
        for j in range(HI):
            d = 0
            for x in range(dI):
                d += int(q[j][x]) * int(ks[x])
            if d > 0:
                total += Fraction(int(w_num[j]), w_den) * d
        out.append(total)
    return out


def _brute_select(scores, k):
    """Repeatedly take the best remaining position: larger score first, and
    among equal scores the lower position (explicit loops, no sorting)."""
    remaining = list(range(len(scores)))
    chosen = []
    while remaining and len(chosen) < k:
        best = remaining[0]
        for p in remaining[1:]:
            if scores[p] > scores[best]:
                best = p
        chosen.append(best)
        remaining.remove(best)
    return chosen + [-1] * (k - len(chosen))


@pytest.mark.parametrize("seed", range(12))
def test_selection_matches_brute_force_with_ties(seed):
    rng = np.random.default_rng(100 + seed)
    n, HI, dI, w_den = 24, 3, 4, 4
    q = rng.integers(-2, 3, (n, HI, dI))
    k = rng.integers(-2, 3, (n, dI))
    w_num = rng.integers(-4, 5, (n, HI))
    for topk in (1, 3, 8, 30):
        got = O.indexer_topk(q[None].astype(float), k[None].astype(float),
                             (w_num / w_den)[None], topk)[0]
        for t in range(n):
            exact = _brute_scores_fraction(q[t], k[: t + 1], w_num[t], w_den)
            assert got[t].tolist() == _brute_select(exact, topk), (seed, topk, t)


def test_short_history_rule():
    rng = np.random.default_rng(5)
    n, topk = 20, 8
    q = rng.standard_normal((1, n, 2, 4))
    k = rng.standard_normal((1, n, 4))
    w = rng.standard_normal((1, n, 2))
    idx = O.indexer_topk(q, k, w, topk)[0]
    for t in range(n):
        m = min(topk, t + 1)
        assert sorted(idx[t, :m].tolist()) == sorted(set(idx[t, :m].tolist()))
        assert all(0 <= p <= t for p in idx[t, :m])
        assert np.all(idx[t, m:] == -1)
        if t + 1 <= topk:
            assert sorted(idx[t, :m].tolist()) == list(range(t + 1))


def test_selection_invariant_under_shift_and_positive_scale():
    rng = np.random.default_rng(6)
    s = rng.integers(-5, 6, 60).astype(float)      # many ties
    base = O.causal_topk_row(s, 59, 17)
    assert np.array_equal(O.causal_topk_row(2.5 * s + 11.0, 59, 17), base)
    # -0.0 and +0.0 are the same score
    z = np.array([0.0, -0.0, 0.0, -0.0])
    assert O.causal_topk_row(z, 3, 2).tolist() == [0, 1]


def test_selection_stats_margin():
    s = np.array([3.0, 1.0, 5.0, 1.0, 2.0])
    st = O.selection_stats_row(s, 4, 3)
    assert st["tau"] == 2.0 and st["n_above"] == 2 and st["margin"] == 1.0
    st = O.selection_stats_row(s, 4, 4)
    assert st["tau"] == 1.0 and st["n_above"] == 3 and st["margin"] == 0.0
    st = O.selection_stats_row(s, 4, 5)
    assert st["margin"] == math.inf


# --------------------------------------------------------------------------
# Eq. (3): attention
# --------------------------------------------------------------------------

def test_full_budget_equals_causal_dense_attention():
    """With k >= t+1 every position is selected and eq. (3) is ordinary causal
    attention with one shared key/value row per position (MQA form)."""
    rng = np.random.default_rng(7)
    n, H, Dqk, Dv = 10, 3, 16, 12
    q = rng.standard_normal((1, n, H, Dqk))
    lat = rng.standard_normal((1, n, Dqk))
    scale = 0.3
    idx = np.stack([np.concatenate([np.arange(t + 1)[::-1], -np.ones(n - t - 1, int)]) for t in range(n)])
    out, lse = O.sparse_attention(q, lat, idx[None], scale, Dv)
    qt = torch.from_numpy(q[0]).permute(1, 0, 2)               # [H, n, Dqk]
    kt = torch.from_numpy(lat[0])[None].expand(H, n, Dqk)
    vt = torch.from_numpy(lat[0, :, :Dv])[None].expand(H, n, Dv)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    assert np.allclose(out[0], ref.permute(1, 0, 2).numpy(), atol=1e-12)
    logits = scale * torch.einsum("hqd,hkd->hqk", qt, kt)
    mask = torch.ones(n, n, dtype=torch.bool).tril()
    ref_lse = torch.logsumexp(logits.masked_fill(~mask, -math.inf), dim=-1)
    assert np.allclose(lse[0], ref_lse.permute(1, 0).numpy(), atol=1e-12)


def test_sparse_renormalisation_identity_and_bound():
    """Eq. (19): the sparse output equals sum_{j in S} (a_j / M_k) v_j with a the
    dense softmax; eq. (20): |o - o~| <= 2 (1 - M_k) V with V = max |v_j|."""
    rng = np.random.default_rng(8)
    m, Dqk, Dv = 40, 8, 6
    lat = rng.standard_normal((m, Dqk)) * 1.5
    q = rng.standard_normal((1, Dqk))
    sel = rng.choice(m, 15, replace=False)
    dense, _ = O.sparse_attention_row(q, lat, np.arange(m), 1.0, Dv)
    sparse, _ = O.sparse_attention_row(q, lat, sel, 1.0, Dv)
    z = lat @ q[0]
    a = np.exp(z - z.max())
    a /= a.sum()
    M = a[sel].sum()
    v = lat[:, :Dv]
    renorm = (a[sel, None] / M * v[sel]).sum(axis=0)
    assert np.allclose(sparse[0], renorm, atol=1e-12)
    V = np.linalg.norm(v, axis=1).max()
    assert np.linalg.norm(dense[0] - sparse[0]) <= 2 * (1 - M) * V + 1e-12


# --------------------------------------------------------------------------
# Eq. (15): teacher probability mass covered by a selection
# --------------------------------------------------------------------------

def _single_head_latents(logits):
    """Latent rows whose logits against q = e_0 (scale 1) are `logits`."""
    lat = np.zeros((len(logits), 4))
    lat[:, 0] = logits
    lat[:, 1:] = np.arange(1, len(logits) + 1)[:, None] * np.array([0.5, -1.0, 2.0])
    return np.array([[1.0, 0.0, 0.0, 0.0]]), lat


def test_mass_coverage_worked_example_miss_case():
    """§1.1 miss case: full logits 0.2, 1.2, 2.0 at positions 1, 2, 3 and the
    selector returned {1, 2}: the covered mass is the closed form
    (e^0.2 + e^1.2) / (e^0.2 + e^1.2 + e^2.0); selecting all three covers 1."""
    g = _worked()
    logits = g["attention_logits"] + [g["miss_case_logit_position3"]]
    q, lat = _single_head_latents(logits)
    r = O.mass_coverage_row(q, lat, np.array(g["selected_positions_0based"]), 1.0)
    want = (math.exp(0.2) + math.exp(1.2)) / (math.exp(0.2) + math.exp(1.2) + math.exp(2.0))
    assert abs(r["M"] - want) < 1e-15 and abs(r["per_head"][0] - want) < 1e-15
    assert abs(r["M"] - 0.3807) < 1e-4           # the missed top position held ~62% of the mass
    full = O.mass_coverage_row(q, lat, np.array([2, 0, 1, -1]), 1.0)
    assert abs(full["M"] - 1.0) < 1e-15


def test_mass_coverage_renormalisation_factor_from_the_page():
    """§3.2 after eq. (19): with M_k = 0.6 the retained positions are scaled by
    1/M_k ~ 1.67, with M_k = 0.98 by ~1.02.  Build dense probabilities with
    exactly that retained mass and check both M_k and eq. (19)'s rescaling of
    the sparse output."""
    for kept, factor in ((0.6, 1.67), (0.98, 1.02)):
        a = np.array([kept / 2, kept / 2, (1 - kept) / 3, (1 - kept) / 3, (1 - kept) / 3])
        q, lat = _single_head_latents(np.log(a))
        r = O.mass_coverage_row(q, lat, np.array([0, 1]), 1.0)
        assert abs(r["M"] - kept) < 1e-12
        assert abs(1.0 / r["M"] - factor) < 5e-3
        sparse, _ = O.sparse_attention_row(q, lat, np.array([0, 1]), 1.0, 4)
        renorm = (a[:2, None] / r["M"] * lat[:2, :4]).sum(axis=0)
        assert np.allclose(sparse[0], renorm, atol=1e-12)


def test_mass_coverage_per_head_and_eq19_identity():
    """Per head, the sparse output equals sum_{j in S} a_j^(h) v_j / m_h with m_h
    the head's covered mass (eq. (19)); the aggregate M is the mean over heads
    of m_h (sum over heads, then L1 along the sequence, eq. (16))."""
    rng = np.random.default_rng(15)
    H, t1, Dqk, Dv = 3, 23, 10, 6
    q = rng.standard_normal((H, Dqk))
    lat = rng.standard_normal((t1, Dqk)) * 1.3
    sel = rng.choice(t1, 9, replace=False)
    r = O.mass_coverage_row(q, lat, sel, 0.7)
    sparse, _ = O.sparse_attention_row(q, lat, sel, 0.7, Dv)
    for h in range(H):
        z = 0.7 * (lat @ q[h])
        a = np.exp(z - z.max())
        a /= a.sum()
        assert abs(r["per_head"][h] - a[sel].sum()) < 1e-13
        assert np.allclose(sparse[h], (a[sel, None] * lat[sel, :Dv]).sum(axis=0) / r["per_head"][h], atol=1e-12)
    assert abs(r["M"] - r["per_head"].mean()) < 1e-13
    assert abs(r["min"] - r["per_head"].min()) < 1e-15
    # slot order, -1 padding and a repeated position do not change the set
    r2 = O.mass_coverage_row(q, lat, np.concatenate([sel[::-1], [-1, sel[0]]]), 0.7)
    assert abs(r2["M"] - r["M"]) < 1e-14


def test_mass_coverage_three_heads_cannot_share_two_slots():
    """§3.1 three-head example: heads put 0.9 of their mass on positions 10,
    20 and 30, budget k = 2.  Every shared pair leaves one head with at most
    the remaining 0.1 of its mass, while the mean coverage stays ~0.63."""
    n = 40
    peaks = (10, 20, 30)
    a = np.full((3, n), 0.1 / (n - 1))
    for h, pos in enumerate(peaks):
        a[h, pos] = 0.9
    # logits realising these probabilities (q_h = e_h, latent column h = log a_h)
    lat = np.zeros((n, 3))
    lat[:, :] = np.log(a).T
    q = np.eye(3)
    for pair in ((10, 20), (10, 30), (20, 30)):
        r = O.mass_coverage_row(q, lat, np.array(pair), 1.0)
        assert r["min"] < 0.1 + 1e-12
        assert abs(r["M"] - (2 * 0.9 + 3 * 0.1 / (n - 1) * 2 - 0.1 / (n - 1) * 2) / 3) < 1e-12
        assert np.sum(r["per_head"] > 0.9 - 1e-12) == 2


def test_mass_coverage_brute_force_small():
    """Explicit loops with Python floats on a tiny two-head case."""
    rng = np.random.default_rng(16)
    H, t1, Dqk = 2, 6, 3
    q = rng.integers(-2, 3, (H, Dqk)).astype(float)
    lat = rng.integers(-2, 3, (t1, Dqk)).astype(float)
    sel = [4, 1, 5]
    scale = 0.5
    per = []
    for h in range(H):
        ez = [math.exp(scale * sum(q[h, d] * lat[j, d] for d in range(Dqk))) for j in range(t1)]
        per.append(sum(ez[j] for j in sel) / sum(ez))
    r = O.mass_coverage_row(q, lat, np.array(sel), scale)
    assert np.allclose(r["per_head"], per, atol=1e-14)
    assert abs(r["M"] - sum(per) / H) < 1e-14


def test_attention_ignores_padding_and_slot_order():
    rng = np.random.default_rng(9)
    lat = rng.standard_normal((30, 8))
    q = rng.standard_normal((2, 8))
    sel = np.array([4, 17, 2, 9])
    a, la = O.sparse_attention_row(q, lat, sel, 0.5, 5)
    b, lb = O.sparse_attention_row(q, lat, np.array([9, -1, 2, 17, -1, 4]), 0.5, 5)
    assert np.allclose(a, b, atol=1e-13) and np.allclose(la, lb, atol=1e-13)
    e, le = O.sparse_attention_row(q, lat, np.array([-1, -1]), 0.5, 5)
    assert np.all(e == 0) and np.all(np.isneginf(le))


# --------------------------------------------------------------------------
# Decode = last row of prefill
# --------------------------------------------------------------------------

def test_decode_equals_last_prefill_row():
    rng = np.random.default_rng(10)
    lens = [7, 13, 5]
    HI, dI, H, Dqk, Dv, topk = 2, 4, 3, 8, 6, 4
    cu = np.concatenate([[0], np.cumsum(lens)])
    kc = rng.integers(-3, 4, (cu[-1], dI)).astype(float)
    lat = rng.standard_normal((cu[-1], Dqk))
    qI = rng.integers(-3, 4, (3, HI, dI)).astype(float)
    w = rng.integers(-4, 5, (3, HI)) / 4.0
    q = rng.standard_normal((3, H, Dqk))
    idx = O.decode_indexer_topk(qI, w, kc, cu, topk)
    out, lse = O.decode_sparse_attention(q, lat, cu, idx, 0.4, Dv)
    for b, L in enumerate(lens):
        lo = cu[b]
        qpre = np.zeros((1, L, HI, dI))
        qpre[0, -1] = qI[b]
        wpre = np.zeros((1, L, HI))
        wpre[0, -1] = w[b]
        pre = O.indexer_topk(qpre, kc[None, lo:lo + L], wpre, topk, rows=[(0, L - 1)])
        assert pre[0, L - 1].tolist() == idx[b].tolist()
        o2, l2 = O.sparse_attention_row(q[b], lat[lo:lo + L], idx[b], 0.4, Dv)
        assert np.allclose(out[b], o2) and np.allclose(lse[b], l2)


def test_selection_recall_pins():
    # eq. (14): R = |T ∩ S| / |T|, order-free, unused slots ignored
    assert O.selection_recall_row([0, 1, 2, 3], [3, 2, 1, 0]) == 1.0
    assert O.selection_recall_row([0, 1, 2, 3], [4, 5, 6, 7]) == 0.0
    assert O.selection_recall_row([0, 1, 2, 3], [1, 3, 8, 9]) == 0.5
    assert O.selection_recall_row([5, 2, -1, -1], [2, 7, -1, -1]) == 0.5
    assert O.selection_recall_row([-1, -1], [3, -1]) == 1.0
    # the worked example's top-2 {0, 1} against a selector that swapped in position 2
    ex = _worked()
    s = np.array(ex["scores"], dtype=float)
    teacher = O.causal_topk_row(s, 2, 2)
    assert O.selection_recall_row(teacher, [0, 2]) == 0.5
    # brute force on random sets: the definition written out with loops
    rng = np.random.default_rng(5)
    for _ in range(50):
        a = rng.choice(40, size=10, replace=False)
        b = rng.choice(40, size=10, replace=False)
        hits = sum(1 for x in a for y in b if x == y)
        assert O.selection_recall_row(a, b) == hits / 10


# --------------------------------------------------------------------------
# Eq. (8): sparse-stage indexer KL and the sparse-attention teacher (§1.2)
# --------------------------------------------------------------------------

def _example_kl_inputs(g):
    q = np.array(g["q"], float)
    keys = np.array(g["keys"], float)
    w = np.array(g["w"], float)
    sel = np.array(g["selected_positions_0based"] + [-1])      # width 3, one unused slot
    return q, keys, w, sel


def test_kl_worked_example_teacher_and_loss():
    """The printed example: the selector keeps 1-based positions 1 and 2 with
    indexer scores 1.5 and 1.5 (eqs. (5)-(6)), while the main attention puts
    weights of about 0.269 / 0.731 on them.  With one attention head the
    sparse-attention teacher is exactly those weights, and the student is
    uniform, so KL = ln 2 - H(p) (a closed form, not the oracle's sum)."""
    g = _worked()
    qa, latent = _example_attention_inputs(g)
    sel = np.array(g["selected_positions_0based"] + [-1])
    p = O.attention_teacher_row(qa, latent, sel, 1.0)
    tol = 0.5 * 10 ** -g["printed_decimals"]
    assert np.allclose(p[:2], g["attention_weights_printed"], atol=tol, rtol=0)
    assert p[2] == 0.0
    q, keys, w, sel = _example_kl_inputs(g)
    r = O.indexer_kl_sparse_row(q, keys, w, sel, p)
    a = np.array(g["attention_logits"])
    pa = np.exp(a) / np.exp(a).sum()
    entropy = -(pa * np.log(pa)).sum()
    assert abs(r["kl"] - (math.log(2.0) - entropy)) < 1e-12
    # the gradient with respect to the scores is student - teacher = 0.5 - p
    assert np.allclose(r["grad_logits"], [0.5 - pa[0], 0.5 - pa[1], 0.0], atol=1e-12, rtol=0)
    # with the printed (rounded) weights the loss agrees to the rounding
    r2 = O.indexer_kl_sparse_row(q, keys, w, sel, np.array(g["attention_weights_printed"] + [0.0]))
    assert abs(r2["kl"] - r["kl"]) < 2e-3


def test_kl_dense_subvector_is_renormalised_by_retained_mass():
    """Remark after eq. (8): a teacher cut out of a dense distribution is divided
    by its retained mass.  The page's miss case gives position 3 a full logit
    of 2.0; the dense softmax's sub-vector on {1, 2} must give the same loss
    as the sparse-attention teacher on that set."""
    g = _worked()
    q, keys, w, sel = _example_kl_inputs(g)
    a = np.array(g["attention_logits"] + [g["miss_case_logit_position3"]])
    dense = np.exp(a) / np.exp(a).sum()
    sub = np.array([dense[0], dense[1], 0.0])
    assert sub.sum() < 0.5                         # most mass is outside the set
    qa, latent = _example_attention_inputs(g)
    p = O.attention_teacher_row(qa, latent, sel, 1.0)
    r_sub = O.indexer_kl_sparse_row(q, keys, w, sel, sub)
    r_p = O.indexer_kl_sparse_row(q, keys, w, sel, p)
    assert abs(r_sub["kl"] - r_p["kl"]) < 1e-12
    for key in ("grad_logits", "dq", "dw", "dk"):
        assert np.allclose(r_sub[key], r_p[key], atol=1e-12, rtol=0)


def _kl_case(rng, HI=3, dI=5, kv_len=11, k=8, n_valid=6):
    q = rng.standard_normal((HI, dI))
    keys = rng.standard_normal((kv_len, dI))
    w = rng.standard_normal(HI)
    sel = np.full(k, -1)
    sel[:n_valid] = rng.choice(kv_len, n_valid, replace=False)
    perm = rng.permutation(k)                      # unused slots anywhere
    sel = sel[perm]
    teacher = np.where(sel >= 0, rng.random(k) + 0.05, 0.0)
    return q, keys, w, sel, teacher


@pytest.mark.parametrize("seed", range(4))
def test_kl_matches_torch_kl_div(seed):
    rng = np.random.default_rng(100 + seed)
    q, keys, w, sel, teacher = _kl_case(rng)
    r = O.indexer_kl_sparse_row(q, keys, w, sel, teacher)
    v = sel >= 0
    scores = torch.from_numpy(O.indexer_scores_row(q, keys[sel[v]], w))     # eq. (1), pinned above
    target = torch.from_numpy(teacher[v] / teacher[v].sum())
    ref = torch.nn.functional.kl_div(torch.log_softmax(scores, 0), target, reduction="sum")
    assert abs(r["kl"] - float(ref)) < 1e-12
    assert r["kl"] >= 0.0


def test_kl_is_zero_when_teacher_equals_student():
    rng = np.random.default_rng(7)
    q, keys, w, sel, _ = _kl_case(rng)
    v = sel >= 0
    teacher = np.zeros(sel.shape[0])
    teacher[v] = 3.0 * np.exp(O.indexer_scores_row(q, keys[sel[v]], w))   # unnormalised on purpose
    r = O.indexer_kl_sparse_row(q, keys, w, sel, teacher)
    assert abs(r["kl"]) < 1e-14
    for key in ("grad_logits", "dq", "dw", "dk"):
        assert np.abs(r[key]).max() < 1e-14


def test_kl_invariances_and_degenerate_rows():
    rng = np.random.default_rng(8)
    q, keys, w, sel, teacher = _kl_case(rng)
    r = O.indexer_kl_sparse_row(q, keys, w, sel, teacher)
    # the teacher's scale does not matter (it is renormalised over S_t)
    r2 = O.indexer_kl_sparse_row(q, keys, w, sel, 4.25 * teacher)
    assert abs(r2["kl"] - r["kl"]) < 1e-12
    # the slot order does not matter
    perm = rng.permutation(sel.shape[0])
    r3 = O.indexer_kl_sparse_row(q, keys, w, sel[perm], teacher[perm])
    assert abs(r3["kl"] - r["kl"]) < 1e-12
    assert np.allclose(r3["dq"], r["dq"], atol=1e-12) and np.allclose(r3["dw"], r["dw"], atol=1e-12)
    assert np.allclose(r3["dk"], r["dk"][perm], atol=1e-12)
    assert np.allclose(r3["grad_logits"], r["grad_logits"][perm], atol=1e-12)
    # the score gradient is a difference of two distributions: it sums to 0
    assert abs(r["grad_logits"].sum()) < 1e-12
    # grad_scale multiplies every gradient, not the loss
    r4 = O.indexer_kl_sparse_row(q, keys, w, sel, teacher, grad_scale=0.5)
    assert r4["kl"] == r["kl"] and np.allclose(r4["dq"], 0.5 * r["dq"], atol=1e-15)
    # no valid slot, or a teacher with no mass on S_t: loss and gradients are 0
    for s, t in ((np.full(8, -1), teacher), (sel, np.zeros(8))):
        e = O.indexer_kl_sparse_row(q, keys, w, s, t)
        assert e["kl"] == 0.0 and not np.any(e["dq"]) and not np.any(e["dk"]) and not np.any(e["dw"])
    # a single valid slot: the student and the teacher are both a point mass
    one = np.full(8, -1)
    one[3] = 5
    e = O.indexer_kl_sparse_row(q, keys, w, one, teacher + 1.0)
    assert e["kl"] == 0.0 and np.abs(e["dq"]).max() == 0.0


def _central_difference(f, x, h=1e-6):
    grad = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + h
        fp = f()
        x[i] = old - h
        fm = f()
        x[i] = old
        grad[i] = (fp - fm) / (2 * h)
    return grad


@pytest.mark.parametrize("seed", range(3))
def test_kl_gradients_match_finite_differences(seed):
    """Every analytic gradient of eq. (8) against a central difference of the
    summed loss, on a 2-sequence chunk whose rows share keys (so dk sums
    over rows).  Inputs keep every q.k at least 1e-3 away from the ReLU kink."""
    rng = np.random.default_rng(200 + seed)
    B, nq, kv_len, HI, dI, k, gs = 2, 3, 9, 3, 4, 6, 0.7
    while True:
        q = rng.standard_normal((B, nq, HI, dI))
        kk = rng.standard_normal((B, kv_len, dI))
        if np.abs(np.einsum("bnhd,bsd->bnhs", q, kk)).min() > 1e-3:
            break
    w = rng.standard_normal((B, nq, HI))
    idx = np.full((B, nq, k), -1)
    for b in range(B):
        for i in range(nq):
            m = [6, 4, 1][i]
            idx[b, i, :m] = rng.choice(kv_len, m, replace=False)
    teacher = np.where(idx >= 0, rng.random((B, nq, k)) + 0.1, 0.0)
    res = O.indexer_kl_sparse(q, kk, w, idx, teacher, grad_scale=gs)

    def loss():
        return gs * O.indexer_kl_sparse(q, kk, w, idx, teacher)["kl"].sum()

    for name, x in (("dq", q), ("dw", w), ("dk", kk)):
        num = _central_difference(loss, x)
        assert np.allclose(res[name], num, atol=1e-7, rtol=1e-6), name
    # keys nobody selected get no gradient
    used = np.zeros((B, kv_len), bool)
    for b in range(B):
        used[b, idx[b][idx[b] >= 0]] = True
    assert not np.any(res["dk"][~used])


def test_attention_teacher_reproduces_the_mean_head_output():
    """Sum over heads then L1 normalisation (eq. (16) with the DSA report's
    aggregation): with every head normalised, p @ C must equal the mean over
    heads of the eq. (3) output (pinned above against scaled_dot_product_attention)
    when the value is the whole latent row; the latent rows are linearly
    independent, so this fixes p."""
    rng = np.random.default_rng(9)
    H, Dqk, kv_len, k = 4, 16, 12, 8
    q = rng.standard_normal((H, Dqk))
    latent = rng.standard_normal((kv_len, Dqk))
    sel = np.array([3, -1, 7, 0, 11, -1, 5, 9])
    p = O.attention_teacher_row(q, latent, sel, 0.3)
    v = sel >= 0
    assert np.all(p[~v] == 0.0) and abs(p.sum() - 1.0) < 1e-12 and np.all(p[v] > 0)
    out, _ = O.sparse_attention_row(q, latent, sel, 0.3, Dqk)
    assert np.allclose(p[v] @ latent[sel[v]], out.mean(axis=0), atol=1e-12, rtol=0)
    assert not np.any(O.attention_teacher_row(q, latent, np.full(5, -1), 0.3))
