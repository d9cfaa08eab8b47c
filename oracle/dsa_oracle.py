"""Plain CPU oracle for the DeepSeek Sparse Attention (DSA) hot path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The CUDA library never calls it, and it shares no code, constant or
helper with the CUDA library.

Source: the page "2.2.1 · DSA 与索引器: 先召回 token, 再计算 Sparse MLA"
(called "the DSA page" below), §1.1 eqs. (1)-(6), §1.2 eqs. (8) and (16)
(sparse-stage indexer KL and its teacher), §2 (decode, quantised indexer key
cache) and §3.1 eqs. (14), (15), (18), §3.2 eqs. (19)-(20).

Everything is float64 numpy.  Inputs are converted exactly to float64 first:
bf16 values are exact in float64, and FP8-e4m3 codes are decoded by
``e4m3_to_float64`` and multiplied by their fp32 scale (both exact in float64),
so the quantisation is part of the input, not of the arithmetic.

Readings of points the page leaves open (each is repeated where it is used):
  * positions are 0-based and the current token is a candidate (eq. (2));
  * ties in the score are broken toward the lower position;
  * -0.0 is the same score as +0.0;
  * unused slots of the fixed-width index tensor hold -1, after the valid ones;
  * the attention of eq. (3) uses an explicit softmax scale; the key is the
    whole latent row and the value is its first ``Dv`` columns; the rotary
    part of query and latent arrives already rotated;
  * a decode step's query is the last token of its sequence (position L-1)
    and it scans all L cached keys, itself included;
  * eq. (8): teacher weights arrive per slot of the index tensor and are
    divided by their sum over the valid slots (the retained mass); a row with
    no valid slot or zero retained mass has loss 0 and zero gradient;
    0 * log 0 = 0; the ReLU of eq. (1) has derivative 0 at 0;
  * the sparse-stage teacher sums the heads' attention probabilities over the
    selected set and L1-normalises the sum (eq. (16) with the aggregation
    the DSA report uses: sum over heads, then L1 along the sequence).

Parity status: every function here is pinned by ``tests/test_oracle.py``
(worked example of §1.1, the min(k, t+1) rule, brute force on tiny inputs,
library special cases, the invariants of §3.1/§3.2, and for eq. (8) the
worked example's KL, torch's kl_div and central finite differences of the
loss for every gradient).
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "e4m3_to_float64",
    "dequantize",
    "indexer_scores_row",
    "indexer_scores",
    "causal_topk_row",
    "indexer_topk",
    "selection_stats_row",
    "selection_recall_row",
    "mass_coverage_row",
    "mass_coverage",
    "sparse_attention_row",
    "sparse_attention",
    "decode_indexer_topk",
    "decode_sparse_attention",
    "attention_teacher_row",
    "attention_teacher",
    "indexer_kl_sparse_row",
    "indexer_kl_sparse",
]


# ---------------------------------------------------------------------------
# Inputs: exact conversion to float64
# ---------------------------------------------------------------------------

def e4m3_to_float64(codes) -> np.ndarray:
    """Decode FP8 E4M3 ("fn" variant) byte codes to float64, exactly.

    The DSA page (§2, quantised indexer key cache) says the indexer may run in
    FP8 with a quantised key cache plus scales.  The format: 1 sign bit, 4
    exponent bits with bias 7, 3 mantissa bits; exponent field 0 is subnormal
    (value = m/8 * 2^-6); there is no infinity and only S.1111.111 is NaN.
    """
    c = np.asarray(codes).astype(np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = sign * (1.0 + m / 8.0) * np.power(2.0, (e - 7).astype(np.float64))
    subnormal = sign * (m / 8.0) * 2.0 ** -6
    out = np.where(e == 0, subnormal, normal)
    out = np.where((e == 0xF) & ((c & 0x7) == 0x7), np.nan, out)
    return out


def dequantize(codes, scale, axis_shape) -> np.ndarray:
    """Dequantised value = e4m3 value x its per-token fp32 scale (float64).

    ``scale`` has the leading shape of ``codes`` minus ``axis_shape`` trailing
    dimensions (one scale per token, shared by the quantised group).
    """
    v = e4m3_to_float64(codes)
    s = np.asarray(scale, dtype=np.float64)
    return v * s.reshape(s.shape + (1,) * axis_shape)


def _f64(x) -> np.ndarray:
    """Exact conversion of a float array (numpy or torch, any float dtype)."""
    if hasattr(x, "detach"):  # a torch tensor: go through float64 on the CPU
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# Eq. (1): Lightning Indexer score
# ---------------------------------------------------------------------------

def indexer_scores_row(q_t, k_hist, w_t) -> np.ndarray:
    """Scores of one query against a list of keys, eq. (1) of the DSA page:

        I[t, s] = sum_j  w[t, j] * ReLU( q[t, j] . k[s] )

    q_t: [H_I, d_I] indexer queries of token t; k_hist: [m, d_I] keys;
    w_t: [H_I] real-valued (possibly negative) head weights.
    Returns [m] float64 with -0.0 replaced by +0.0.
    """
    q_t = _f64(q_t)
    k_hist = _f64(k_hist)
    w_t = _f64(w_t)
    dots = k_hist @ q_t.T                     # [m, H_I]: q[t,j] . k[s]
    relu = np.maximum(dots, 0.0)              # per-head ReLU
    scores = relu @ w_t                       # weighted sum over heads
    return scores + 0.0                       # -0.0 -> +0.0


def indexer_scores(q, k, w, q_offset: int = 0) -> np.ndarray:
    """Dense causal score matrix for a prefill chunk (DSA page §1.1 shapes).

    q: [B, nq, H_I, d_I], k: [B, kv_len, d_I], w: [B, nq, H_I].
    Query row i of the chunk sits at absolute position t = q_offset + i and
    sees keys 0 <= s <= t.  Returns [B, nq, kv_len] float64, -inf where s > t.
    """
    q = _f64(q)
    k = _f64(k)
    w = _f64(w)
    B, nq = q.shape[0], q.shape[1]
    kv_len = k.shape[1]
    out = np.full((B, nq, kv_len), -np.inf)
    for b in range(B):
        for i in range(nq):
            t = q_offset + i
            out[b, i, : t + 1] = indexer_scores_row(q[b, i], k[b, : t + 1], w[b, i])
    return out


# ---------------------------------------------------------------------------
# Eq. (2): causal top-k with a fixed-width, -1 padded index tensor
# ---------------------------------------------------------------------------

def causal_topk_row(scores_row, t: int, k: int) -> np.ndarray:
    """S_t = TopK({I[t, s] : 0 <= s <= t}, min(k, t + 1)), eq. (2).

    Positions are 0-based and include the current token.  Ties go to the
    lower position.  The result has width k: the min(k, t+1) selected
    positions in rank order (score descending, then position ascending),
    followed by -1 in every unused slot.
    """
    s = np.asarray(scores_row, dtype=np.float64)[: t + 1] + 0.0
    m = min(k, t + 1)
    # A stable sort of -score keeps equal scores in ascending position order.
    order = np.argsort(-s, kind="stable")[:m]
    out = np.full(k, -1, dtype=np.int64)
    out[:m] = order
    return out


def selection_stats_row(scores_row, t: int, k: int) -> dict:
    """Cut-off quantities of one row for tolerance-aware comparison.

    tau       -- the score at rank m = min(k, t+1) (the last one kept);
    n_above   -- how many scores are strictly above tau (all must be kept);
    margin    -- Delta_k = s_(k) - s_(k+1), eq. (18) of the DSA page §3.1
                 (+inf when nothing is left out);
    max_abs   -- the largest |score| in the row.
    """
    s = np.asarray(scores_row, dtype=np.float64)[: t + 1] + 0.0
    m = min(k, t + 1)
    srt = np.sort(s)[::-1]
    tau = srt[m - 1]
    nxt = srt[m] if m < s.size else -np.inf
    return {
        "tau": float(tau),
        "n_above": int(np.count_nonzero(s > tau)),
        "margin": float(tau - nxt),
        "max_abs": float(np.max(np.abs(s))),
    }


def selection_recall_row(teacher_row, student_row) -> float:
    """Set recall R = |T ∩ S| / |T| of a student selection S against a teacher
    selection T, eq. (14) of the DSA page §3.1 (there |T| = k; for a row with
    t + 1 <= k both sets hold its t + 1 positions, so |T| is the count of
    valid teacher entries).  Entries < 0 are unused slots; slot order is
    irrelevant.  A row with an empty teacher set has recall 1.
    """
    t = {int(x) for x in np.asarray(teacher_row).ravel() if x >= 0}
    s = {int(x) for x in np.asarray(student_row).ravel() if x >= 0}
    if not t:
        return 1.0
    return len(t & s) / len(t)


def mass_coverage_row(q_t, latent_hist, sel, scale: float) -> dict:
    """Teacher probability mass covered by a selection, eq. (15) of the DSA
    page §3.1:  M_k = sum_{j in S_k} a_{tj}.

    a_{tj} is the dense attention probability of the main attention over the
    whole causal history 0..t (the teacher); with several query heads each
    head h has its own a^(h) and the teacher the DSA report uses is their sum
    over heads, L1-normalised along the sequence (eq. (16) with equal
    weights), i.e. the mean over heads.  The page also asks for the lowest
    per-head coverage, so both are returned.

    q_t: [H, Dqk] query heads of token t; latent_hist: [t+1, Dqk] latent rows
    0..t (the key is the whole row, as in eq. (3)); sel: selected positions,
    -1 entries ignored.  Returns {"M": float, "per_head": [H], "min": float}.
    """
    q_t = _f64(q_t)
    latent_hist = _f64(latent_hist)
    sel = np.asarray(sel, dtype=np.int64)
    sel = np.unique(sel[sel >= 0])
    z = scale * (q_t @ latent_hist.T)               # [H, t+1] dense logits
    e = np.exp(z - z.max(axis=1, keepdims=True))
    a = e / e.sum(axis=1, keepdims=True)            # a^(h)_{tj}, each row sums to 1
    per_head = a[:, sel].sum(axis=1)                # coverage of each head
    p = a.sum(axis=0)                               # sum over heads ...
    p = p / p.sum()                                 # ... L1-normalised along the sequence
    return {"M": float(p[sel].sum()), "per_head": per_head, "min": float(per_head.min())}


def mass_coverage(q, latent, idx, scale: float, q_offset: int = 0, rows=None) -> dict:
    """``mass_coverage_row`` for a prefill chunk: q [B, nq, H, Dqk], latent
    [B, kv_len, Dqk], idx [B, nq, k]; row i sits at t = q_offset + i.
    Returns M [B, nq], per_head [B, nq, H] and min [B, nq] (NaN in rows left
    out by ``rows``)."""
    q = _f64(q)
    latent = _f64(latent)
    idx = np.asarray(idx.cpu() if hasattr(idx, "cpu") else idx, dtype=np.int64)
    B, nq, H = q.shape[0], q.shape[1], q.shape[2]
    out = {"M": np.full((B, nq), np.nan), "per_head": np.full((B, nq, H), np.nan), "min": np.full((B, nq), np.nan)}
    todo = rows if rows is not None else [(b, i) for b in range(B) for i in range(nq)]
    for b, i in todo:
        t = q_offset + i
        r = mass_coverage_row(q[b, i], latent[b, : t + 1], idx[b, i], scale)
        out["M"][b, i], out["per_head"][b, i], out["min"][b, i] = r["M"], r["per_head"], r["min"]
    return out


def indexer_topk(q, k, w, topk: int, q_offset: int = 0, rows=None) -> np.ndarray:
    """Eq. (1) then eq. (2) for a prefill chunk.  Returns [B, nq, topk] int64.

    ``rows`` optionally restricts the work to a list of (b, i) query rows;
    the other rows of the result are left at -2 (not computed).
    """
    q = _f64(q)
    k = _f64(k)
    w = _f64(w)
    B, nq = q.shape[0], q.shape[1]
    out = np.full((B, nq, topk), -2, dtype=np.int64)
    todo = rows if rows is not None else [(b, i) for b in range(B) for i in range(nq)]
    for b, i in todo:
        t = q_offset + i
        sc = indexer_scores_row(q[b, i], k[b, : t + 1], w[b, i])
        out[b, i] = causal_topk_row(sc, t, topk)
    return out


# ---------------------------------------------------------------------------
# Eq. (3): sparse attention over the selected latent rows
# ---------------------------------------------------------------------------

def sparse_attention_row(q_t, latent, sel, scale: float, dv: int):
    """u_t = Attn(h_t, {c_s : s in S_t}), eq. (3) of the DSA page, one token.

    The selector only chooses rows; the attention computes its own logits
    (the indexer scores are not reused, §1.1).  Every query head attends the
    same selected set (the key is shared by all heads, §1.1).

    q_t: [H, Dqk] query heads; latent: [kv_len, Dqk] latent cache rows c_s;
    sel: selected positions, -1 entries are ignored.
    logits z[h, s] = scale * q_t[h] . c_s;  p = softmax over the selected s;
    out[h] = sum_s p[h, s] * c_s[:dv];  lse[h] = log sum_s exp z[h, s].
    With no valid entry the output is 0 and lse is -inf.
    """
    q_t = _f64(q_t)
    latent = _f64(latent)
    sel = np.asarray(sel, dtype=np.int64)
    sel = sel[sel >= 0]
    H = q_t.shape[0]
    if sel.size == 0:
        return np.zeros((H, dv)), np.full(H, -np.inf)
    c = latent[sel]                                  # [m, Dqk]
    z = scale * (q_t @ c.T)                          # [H, m]
    zmax = z.max(axis=1, keepdims=True)
    e = np.exp(z - zmax)
    denom = e.sum(axis=1, keepdims=True)
    p = e / denom
    out = p @ c[:, :dv]                              # [H, dv]
    lse = (zmax + np.log(denom))[:, 0]
    return out, lse


def sparse_attention(q, latent, idx, scale: float, dv: int, rows=None):
    """Eq. (3) for a prefill chunk.

    q: [B, nq, H, Dqk], latent: [B, kv_len, Dqk], idx: [B, nq, k] (-1 padded).
    Returns out [B, nq, H, dv] and lse [B, nq, H] (float64).  ``rows``
    optionally restricts the work to a list of (b, i) rows (others are NaN).
    """
    q = _f64(q)
    latent = _f64(latent)
    idx = np.asarray(idx.cpu() if hasattr(idx, "cpu") else idx, dtype=np.int64)
    B, nq, H = q.shape[0], q.shape[1], q.shape[2]
    out = np.full((B, nq, H, dv), np.nan)
    lse = np.full((B, nq, H), np.nan)
    todo = rows if rows is not None else [(b, i) for b in range(B) for i in range(nq)]
    for b, i in todo:
        out[b, i], lse[b, i] = sparse_attention_row(q[b, i], latent[b], idx[b, i], scale, dv)
    return out, lse


# ---------------------------------------------------------------------------
# Decode step (DSA page §2: one new query scans every cached indexer key)
# ---------------------------------------------------------------------------

def decode_indexer_topk(q, w, k_cache, cu_seqlens, topk: int, with_scores: bool = False):
    """One decode step of the indexer and selector for a batch of sequences.

    q: [B, H_I, d_I] the new token's indexer queries; w: [B, H_I];
    k_cache: [sum L, d_I] ragged indexer key cache, sequence b in rows
    cu_seqlens[b] .. cu_seqlens[b+1]-1; L_b includes the new token, whose
    position is t = L_b - 1.  Returns idx [B, topk] of positions local to
    each sequence (and the per-sequence score rows if asked).
    """
    q = _f64(q)
    w = _f64(w)
    k_cache = _f64(k_cache)
    cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64)
    B = q.shape[0]
    out = np.full((B, topk), -1, dtype=np.int64)
    rows = []
    for b in range(B):
        lo, hi = int(cu[b]), int(cu[b + 1])
        sc = indexer_scores_row(q[b], k_cache[lo:hi], w[b])
        out[b] = causal_topk_row(sc, hi - lo - 1, topk)
        rows.append(sc)
    return (out, rows) if with_scores else out


def decode_sparse_attention(q, latent_cache, cu_seqlens, idx, scale: float, dv: int):
    """Eq. (3) for a decode step: every query head of a sequence attends the
    same selected rows of that sequence's latent cache (the MQA form of §2).

    q: [B, H, Dqk]; latent_cache: [sum L, Dqk]; idx: [B, k] local positions.
    Returns out [B, H, dv], lse [B, H].
    """
    q = _f64(q)
    latent_cache = _f64(latent_cache)
    cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64)
    idx = np.asarray(idx.cpu() if hasattr(idx, "cpu") else idx, dtype=np.int64)
    B, H = q.shape[0], q.shape[1]
    out = np.zeros((B, H, dv))
    lse = np.zeros((B, H))
    for b in range(B):
        lo, hi = int(cu[b]), int(cu[b + 1])
        out[b], lse[b] = sparse_attention_row(q[b], latent_cache[lo:hi], idx[b], scale, dv)
    return out, lse


# ---------------------------------------------------------------------------
# Eq. (8): sparse-stage indexer KL on the selected set, and its teacher
# ---------------------------------------------------------------------------

def attention_teacher_row(q_t, latent, sel, scale: float) -> np.ndarray:
    """Teacher distribution of token t over its selected set, taken from the
    sparse main attention (DSA page §1.2, the remark after eq. (8), and
    eq. (16) with the DSA report's aggregation).

    For every query head h the attention probabilities over the selected set,
    a_h[s] = softmax_s(scale * q_t[h] . c_s), are recomputed from scratch;
    they are summed over the heads and the sum is L1-normalised along the
    selected positions.  Returns one weight per slot of ``sel`` (0 in the
    unused slots, which hold -1); all zeros if no slot is valid.
    """
    q_t = _f64(q_t)
    latent = _f64(latent)
    sel = np.asarray(sel, dtype=np.int64)
    out = np.zeros(sel.shape[0])
    valid = sel >= 0
    if not valid.any():
        return out
    c = latent[sel[valid]]                           # [m, Dqk]
    z = scale * (q_t @ c.T)                          # [H, m]
    e = np.exp(z - z.max(axis=1, keepdims=True))
    a = e / e.sum(axis=1, keepdims=True)             # per-head softmax over S_t
    p = a.sum(axis=0)                                # sum over heads
    out[valid] = p / p.sum()                         # L1 normalisation
    return out


def attention_teacher(q, latent, idx, scale: float, rows=None) -> np.ndarray:
    """``attention_teacher_row`` for a prefill chunk.

    q: [B, nq, H, Dqk], latent: [B, kv_len, Dqk], idx: [B, nq, k].
    Returns [B, nq, k] float64 (NaN in rows left out by ``rows``).
    """
    q = _f64(q)
    latent = _f64(latent)
    idx = np.asarray(idx.cpu() if hasattr(idx, "cpu") else idx, dtype=np.int64)
    B, nq, k = idx.shape
    out = np.full((B, nq, k), np.nan)
    todo = rows if rows is not None else [(b, i) for b in range(B) for i in range(nq)]
    for b, i in todo:
        out[b, i] = attention_teacher_row(q[b, i], latent[b], idx[b, i], scale)
    return out


def indexer_kl_sparse_row(q_t, k_all, w_t, sel, teacher, grad_scale: float = 1.0) -> dict:
    """Eq. (8) of the DSA page for one token t, with its gradient.

        KL_t = D_KL( p_{t,S_t} || Softmax(I_{t,S_t}) )

    Steps, in the page's order:
      1. the teacher's weights on the selected slots are divided by their
         sum (the retained mass), so both sides are distributions over S_t;
      2. the indexer scores I_{t,s} of eq. (1) are recomputed for s in S_t;
      3. the student is the softmax of those scores over S_t;
      4. KL_t = sum_s p_s (log p_s - log softmax(I)_s), with 0 log 0 = 0.
    Backward, for a loss L with dL/dKL_t = grad_scale:
      g_s  = dL/dI_s = grad_scale * (softmax(I)_s - p_s)
      dw_j = sum_s g_s ReLU(d_sj),             d_sj = q_t[j] . k_s
      dq_j = sum_s g_s w_j [d_sj > 0] k_s       (ReLU'(0) = 0)
      dk_s = sum_j g_s w_j [d_sj > 0] q_t[j]

    q_t: [H_I, d_I]; k_all: [kv_len, d_I]; w_t: [H_I]; sel: [k] positions
    (-1 = unused slot; the valid ones are distinct); teacher: [k] weights
    >= 0.  Returns kl (float), grad_logits [k] (0 in unused slots),
    dq [H_I, d_I], dw [H_I] and dk [k, d_I] (row r is the gradient of key
    sel[r]; zero rows for unused slots).
    """
    q_t = _f64(q_t)
    k_all = _f64(k_all)
    w_t = _f64(w_t)
    sel = np.asarray(sel, dtype=np.int64)
    teacher = _f64(teacher)
    K = sel.shape[0]
    HI, dI = q_t.shape
    res = {"kl": 0.0, "grad_logits": np.zeros(K), "dq": np.zeros((HI, dI)),
           "dw": np.zeros(HI), "dk": np.zeros((K, dI))}
    valid = sel >= 0
    if not valid.any():
        return res
    p = teacher[valid]
    mass = p.sum()
    if not mass > 0.0:
        return res
    p_hat = p / mass                                  # step 1
    kS = k_all[sel[valid]]                            # [m, d_I]
    dots = kS @ q_t.T                                 # [m, H_I]
    scores = np.maximum(dots, 0.0) @ w_t              # step 2, eq. (1)
    top = scores.max()
    log_z = top + math.log(np.exp(scores - top).sum())
    log_student = scores - log_z                      # step 3
    pos = p_hat > 0.0
    res["kl"] = float(np.sum(p_hat[pos] * (np.log(p_hat[pos]) - log_student[pos])))   # step 4
    g = grad_scale * (np.exp(log_student) - p_hat)
    G = g[:, None] * w_t[None, :] * (dots > 0.0)      # dL/d d_sj
    res["grad_logits"][valid] = g
    res["dw"] = (np.maximum(dots, 0.0) * g[:, None]).sum(axis=0)
    res["dq"] = G.T @ kS
    res["dk"][valid] = G @ q_t
    return res


def indexer_kl_sparse(q, k, w, idx, teacher, grad_scale: float = 1.0, rows=None) -> dict:
    """Eq. (8) summed over the rows of a prefill chunk, with gradients.

    q: [B, nq, H_I, d_I], k: [B, kv_len, d_I], w: [B, nq, H_I],
    idx: [B, nq, topk], teacher: [B, nq, topk].  Returns kl [B, nq],
    grad_logits [B, nq, topk], dq, dw (shapes of q and w) and dk [B, kv_len,
    d_I], the sum over rows of each selected key's gradient.  ``rows``
    restricts the work to a list of (b, i) rows (the others stay 0).
    """
    q = _f64(q)
    k = _f64(k)
    w = _f64(w)
    teacher = _f64(teacher)
    idx = np.asarray(idx.cpu() if hasattr(idx, "cpu") else idx, dtype=np.int64)
    B, nq, topk = idx.shape
    out = {"kl": np.zeros((B, nq)), "grad_logits": np.zeros((B, nq, topk)),
           "dq": np.zeros(q.shape), "dw": np.zeros(w.shape), "dk": np.zeros(k.shape)}
    todo = rows if rows is not None else [(b, i) for b in range(B) for i in range(nq)]
    for b, i in todo:
        r = indexer_kl_sparse_row(q[b, i], k[b], w[b, i], idx[b, i], teacher[b, i], grad_scale)
        out["kl"][b, i] = r["kl"]
        out["grad_logits"][b, i] = r["grad_logits"]
        out["dq"][b, i] = r["dq"]
        out["dw"][b, i] = r["dw"]
        v = idx[b, i] >= 0
        np.add.at(out["dk"][b], idx[b, i][v], r["dk"][v])
    return out


def softmax_scale_default(dqk: int) -> float:
    """Default attention scale 1/sqrt(Dqk) (the dense-attention scale written
    on the page "2 · 动态路由", §3.1); the page on DSA leaves it implicit."""
    return 1.0 / math.sqrt(dqk)
