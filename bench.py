"""Benchmark of the DSA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl b200|reference]

One step = the whole hot path over one batch of synthetic, HBM-resident input:
the fused Lightning Indexer + causal top-k (eqs. (1)-(2) of the page
"2.2.1 · DSA 与索引器") followed by sparse attention over the selected latent
rows (eq. (3)).  The default workload is the integer-valued prefill
(B=1, n=8192, HI=64, dI=128, k=2048, 16 heads, latent 576/512); the metric is
query tokens per second.  --workload decode|decode_fp8|prefill_fp8|long_prefill|tiny
selects the other workloads; --workload indexer_kl times the sparse training
stage's indexer step instead: selection, the sparse attention forward with
its lse, the teacher recomputed on the selected set, then the eq. (8) KL on
that set, forward and backward.

Timing: W warm-up steps, then exactly K steps, each bracketed by CUDA events
on the launching stream; L2 is flushed (a 256 MiB write) before every timed
step, outside the events.  Per-kernel events give the roofline of the
dominant kernel.  Under torchrun every rank runs its own batch (weak
scaling, no collective on the data path); rank 0 prints the max over ranks.

End to end (`e2e`): every step uploads its inputs from pinned host memory,
runs through the public API and downloads its result; timed both one step
after another on one stream and with consecutive steps overlapped on three
streams (two replicas of the device buffers), reporting the faster.

--impl reference times the CPU oracle (float64 numpy) on a bounded sample of
the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from learned_token_indexer_b200 import workloads as W  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
LONG_STEP_MS = 50.0   # steps at least this long time their kernels at the sustained clock
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = {
    "prefill": ("prefill query-tokens/s (indexer+top-k+sparse attn)", "query-tokens/s"),
    "decode": ("decode tokens/s (indexer scan+top-k+sparse attn)", "tokens/s"),
    "train": ("sparse-stage indexer training query-tokens/s (indexer+top-k, sparse attn, teacher, eq. 8 KL fwd/bwd)",
              "query-tokens/s"),
}


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "learned_token_indexer_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "indexer_topk_prefill": ["indexer_topk_prefill.cu", "indexer_common.cuh", "select.cuh", "sm100.cuh"],
    "sparse_attn": ["sparse_attn.cu", "sm100.cuh"],
    "dense_attn": ["latent_attn_dense.cu", "latent_attn.cuh", "sm100.cuh"],
    "latent_attn_decode": ["latent_attn_decode.cu", "latent_attn.cuh", "sm100.cuh"],
    "indexer_scan": ["indexer_scan.cu", "indexer_common.cuh", "sm100.cuh"],
    "topk_rows": ["topk.cu", "select.cuh"],
    "indexer_kl": ["indexer_kl.cu", "sm100.cuh"],
    "attn_teacher": ["attn_teacher.cu", "sm100.cuh"],
}


def measured_traffic(kernel: str, workload: str):
    """(DRAM bytes per launch, captured case or None) from a committed ncu
    summary; (None, None) when the summary is missing or the kernel source
    changed since it was taken.  The case names the launch that was captured
    when it is not a launch of the timed workload itself (a full-size launch
    too large to capture)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}:{workload}")
    if not e or e.get("source_hash") != kernel_source_hash(KERNEL_SOURCES[kernel]):
        return None, None
    return e.get("bytes_per_launch"), e.get("case")


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"dsa_clocks_{os.getpid()}_{gpu_index}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(parts)
                except ValueError:
                    pass
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def count_pairs_needed(n_rows_first: int, n_rows: int, k: int) -> int:
    """(t, s) score pairs eq. (2) needs: rows with t + 1 > k score all t + 1
    keys; rows with t + 1 <= k select every key without a score."""
    tot = 0
    lo = max(n_rows_first, k)
    hi = n_rows_first + n_rows       # rows t in [n_rows_first, hi)
    if hi > lo:
        tot = (hi * (hi + 1) - lo * (lo + 1)) // 2
    return tot


def selected_entries(t0: int, n_rows: int, k: int) -> int:
    return sum(min(k, t + 1) for t in range(t0, t0 + n_rows))


# ----------------------------------------------------------------------------
# the B200 arm
# ----------------------------------------------------------------------------

class PrefillRun:
    def __init__(self, w: W.Workload, device):
        import learned_token_indexer_b200 as dsa
        self.dsa, self.w, self.dev = dsa, w, device
        self.d = W.make_prefill_inputs(w, device, keep_bf16=w.fp8)
        self.ws_idx = dsa.Workspace(device)
        self.ws_att = dsa.Workspace(device)
        self.idx = torch.empty((w.B, w.n, w.k), dtype=torch.int32, device=device)
        self.out = torch.empty((w.B, w.n, w.H, w.Dv), dtype=torch.bfloat16, device=device)
        self.chunk = w.chunk or w.n
        self.kw = {}
        if w.fp8:
            self.kw = dict(q_scale=self.d["q_scale"], k_scale=self.d["k_scale"])
        self.launches_per_step = 0
        # the attention path the library's length dispatch takes (§2); every
        # chunk of these workloads takes the same one
        paths = {dsa.prefill_attention_path(w.B, min(w.n, c0 + self.chunk) - c0, c0, w.n, w.H, w.Dqk, w.Dv, w.k)
                 for c0 in range(0, w.n, self.chunk)}
        assert len(paths) == 1, "mixed attention paths within one workload"
        self.attn_name = "dense_attn" if paths.pop() == dsa.PATH_DENSE_MASKED else "sparse_attn"

    def step(self, ev=None):
        dsa, w, d = self.dsa, self.w, self.d
        launches = 0
        for c0 in range(0, w.n, self.chunk):
            c1 = min(w.n, c0 + self.chunk)
            sl = (slice(None), slice(c0, c1))
            kw = dict(self.kw)
            if w.fp8 and self.chunk != w.n:
                kw["q_scale"] = self.kw["q_scale"][sl].contiguous()
            e0 = self._rec(ev)
            dsa.indexer_topk_prefill(d["qI"][sl], d["kI"], d["w"][sl], w.k, q_offset=c0, idx_out=self.idx[sl],
                                     workspace=self.ws_idx, **kw)
            e1 = self._rec(ev)
            dsa.attn_prefill(d["q"][sl], d["latent"], self.idx[sl], w.Dv, q_offset=c0, scale=w.scale,
                             out=self.out[sl], workspace=self.ws_att)
            e2 = self._rec(ev)
            if ev is not None:
                ev["indexer_topk_prefill"].append((e0, e1))
                ev[self.attn_name].append((e1, e2))
            triv = c0 < w.k
            # this library's kernels: the indexer when some row of the chunk has
            # t + 1 > k, the trivial-row fill, the attention, and on the dense
            # path the selection bits (its buffer is cleared by a memset)
            scored = c1 > w.k
            bits = self.attn_name == "dense_attn" and scored
            launches += (1 if scored else 0) + (1 if triv else 0) + 1 + (1 if bits else 0)
        self.launches_per_step = launches

    @staticmethod
    def _rec(ev=True):
        """A recorded timing event (None when the step is not being timed)."""
        if ev is None:
            return None
        e = torch.cuda.Event(enable_timing=True)
        e.record()
        return e

    def rows(self):
        return self.w.B * self.w.n

    def selection_diagnostics(self):
        """FP8 indexer only (outside the timed region): the set recall
        R = |T ∩ S| / |T| (eq. (14)) of this step's e4m3 selection S against
        the bf16 selection T of the same draws, over rows with t + 1 > k."""
        w, d, dsa = self.w, self.d, self.dsa
        if not w.fp8 or "qI_bf16" not in d:
            return None
        ref = torch.empty_like(self.idx)
        ws = dsa.Workspace(self.dev)
        for c0 in range(0, w.n, self.chunk):
            c1 = min(w.n, c0 + self.chunk)
            sl = (slice(None), slice(c0, c1))
            dsa.indexer_topk_prefill(d["qI_bf16"][sl], d["kI_bf16"], d["w"][sl], w.k, q_offset=c0, idx_out=ref[sl],
                                     workspace=ws)
        inter, cnt = dsa.selection_overlap(ref, self.idx, w.n, return_counts=True)
        torch.cuda.synchronize()
        ws.check()
        rec_all = inter.float() / cnt.clamp(min=1).float()
        rec = rec_all[:, w.k:].flatten()
        q = torch.quantile(rec, torch.tensor([0.01, 0.5], device=rec.device))
        out = {"fp8_vs_bf16_recall": {"mean": round(float(rec.mean()), 5), "p01": round(float(q[0]), 5),
                                      "median": round(float(q[1]), 5), "min": round(float(rec.min()), 5),
                                      "rows": int(rec.numel()),
                                      "definition": "|T ∩ S| / |T|, T = bf16 selection of the same draws, "
                                                    "S = e4m3 selection; rows with t + 1 > k"}}
        mass = self._mass_coverage(ref, ws)
        out["mass_coverage"] = mass["summary"]
        out["recall_by_margin"] = self._recall_by_margin(rec_all, ws, mass_loss=mass["loss"])
        return out

    def _mass_coverage(self, ref, ws):
        """Teacher mass coverage M_k (eq. (15)) of both selections: the dense
        causal attention's probabilities (heads summed, L1-normalised, eq.
        (16)) on the selected positions, from the lse of the dense attention
        and of the sparse attention over each selection (dsa_mass_coverage).
        §2 asks FP8 validation to compare set overlap and this coverage."""
        w, d, dsa = self.w, self.d, self.dsa
        scratch = torch.empty_like(self.out)
        _, lse_d = dsa.attn_dense_prefill(d["q"], d["latent"], w.Dv, scale=w.scale, out=scratch, return_lse=True,
                                          workspace=ws)
        res = {}
        for name, sel in (("e4m3", self.idx), ("bf16", ref)):
            _, lse_s = dsa.sparse_attn_prefill(d["q"], d["latent"], sel, w.Dv, scale=w.scale, out=scratch,
                                               return_lse=True, workspace=ws)
            res[name] = dsa.mass_coverage(lse_s, lse_d)
        torch.cuda.synchronize()
        ws.check()
        summary = {}
        for name, (m, mn) in res.items():
            mm, mh = m[:, w.k:].flatten().double(), mn[:, w.k:].flatten().double()
            qs = torch.quantile(mm, torch.tensor([0.01, 0.5], dtype=torch.float64, device=mm.device))
            summary[name] = {"mean": round(float(mm.mean()), 5), "p01": round(float(qs[0]), 5),
                             "median": round(float(qs[1]), 5), "min": round(float(mm.min()), 5),
                             "lowest_head_mean": round(float(mh.mean()), 5), "lowest_head_min": round(float(mh.min()), 5)}
        loss_all = (res["bf16"][0] - res["e4m3"][0]).double()
        loss = loss_all[:, w.k:].flatten()
        summary["loss_bf16_minus_e4m3"] = {"mean": float(loss.mean()), "max": float(loss.max()),
                                           "min": float(loss.min())}
        summary["definition"] = ("M_k = sum over the selection of the dense attention probability (eq. (15)), "
                                 "teacher = heads summed then L1-normalised (eq. (16)); lowest_head = the "
                                 "smallest per-head coverage; rows with t + 1 > k; bf16 = the selection of "
                                 "the same draws rounded to bf16, e4m3 = the timed FP8 selection")
        return {"summary": summary, "loss": loss_all}

    def _recall_by_margin(self, rec_all, ws, strip: int = 512, buckets: int = 4, mass_loss=None):
        """Recall of the e4m3 selection grouped by the bf16 cut-off margin
        Delta_k = s_(k) - s_(k+1) (eq. (18), §3.1: small margins are where a
        perturbation swaps boundary tokens).  On the last `strip` rows of the
        first sequence: dense bf16 scores (dsa_indexer_scores), their top
        k + 1 (dsa_topk_rows), then quartiles of the margin."""
        w, d, dsa = self.w, self.d, self.dsa
        t0 = w.n - strip
        sl = (slice(0, 1), slice(t0, w.n))
        sc = dsa.indexer_scores(d["qI_bf16"][sl].contiguous(), d["kI_bf16"][:1].contiguous(),
                                d["w"][sl].contiguous(), q_offset=t0, workspace=ws)[0]
        row_len = torch.arange(t0 + 1, w.n + 1, dtype=torch.int32, device=sc.device)
        _, val = dsa.topk_rows(sc, w.k + 1, row_len=row_len, return_values=True, workspace=ws)
        torch.cuda.synchronize()
        ws.check()
        top = torch.sort(val, dim=1, descending=True).values
        margin = (top[:, w.k - 1] - top[:, w.k]).double()
        rec = rec_all[0, t0:].double()
        edges = torch.quantile(margin, torch.linspace(0, 1, buckets + 1, dtype=torch.float64, device=margin.device))
        rows = []
        for i in range(buckets):
            lo, hi = float(edges[i]), float(edges[i + 1])
            m = (margin >= lo) & ((margin <= hi) if i == buckets - 1 else (margin < hi))
            if int(m.sum()) == 0:
                continue
            row = {"margin": [round(lo, 6), round(hi, 6)], "rows": int(m.sum()),
                   "mean_recall": round(float(rec[m].mean()), 5)}
            if mass_loss is not None:
                row["mean_mass_loss"] = float(mass_loss[0, t0:][m].mean())
            rows.append(row)
        return {"strip": f"rows {t0}..{w.n - 1} of sequence 0", "buckets": rows,
                "definition": "Delta_k = s_(k) - s_(k+1) of the bf16 scores (eq. (18)); quartile buckets; "
                              "mass loss = M_k(bf16 selection) - M_k(e4m3 selection)"}

    def kernel_work(self):
        w = self.w
        pairs = 0
        ent = 0
        for c0 in range(0, w.n, self.chunk):
            c1 = min(w.n, c0 + self.chunk)
            pairs += count_pairs_needed(c0, c1 - c0, w.k)
        ent = selected_entries(0, w.n, w.k)
        return {
            "indexer_topk_prefill": {"flops": 2 * w.HI * w.dI * w.B * pairs, "unit": "TFLOP/s",
                                     "per_unit": f"2*HI*dI = {2 * w.HI * w.dI} FLOP per scored (t,s) pair",
                                     "units": w.B * pairs},
            self.attn_name: self._attn_work(ent),
        }

    def _attn_work(self, ent):
        w = self.w
        r = {"flops": 2 * w.H * w.B * ent * (w.Dqk + w.Dv), "unit": "TFLOP/s",
             "per_unit": f"2*H*(Dqk+Dv) = {2 * w.H * (w.Dqk + w.Dv)} FLOP per selected entry",
             "units": w.B * ent}
        if self.attn_name == "sparse_attn":
            r["gather_bytes"] = w.B * ent * w.Dqk * 2
        else:
            pairs = sum(t + 1 for t in range(w.n))
            r["path"] = ("dense masked (short prefill, §2): every causal key tile is multiplied, "
                         f"{2 * w.H * w.B * pairs * (w.Dqk + w.Dv) / 1e12:.3f} TFLOP per step executed")
        return r

    def host_inputs(self):
        return {k: v.cpu().pin_memory() for k, v in self.d.items()
                if isinstance(v, torch.Tensor) and not k.endswith("_bf16")}

    def load_inputs(self, host):
        for k, v in host.items():
            self.d[k].copy_(v, non_blocking=True)

    def result(self):
        return self.out


class DecodeRun:
    def __init__(self, w: W.Workload, device):
        import learned_token_indexer_b200 as dsa
        self.dsa, self.w, self.dev = dsa, w, device
        self.d = W.make_decode_inputs(w, device)
        self.lengths = self.d["lengths"]
        self.total = int(self.lengths.sum())
        self.maxlen = int(self.lengths.max())
        self.ws_idx = dsa.Workspace(device)
        self.ws_att = dsa.Workspace(device)
        self.idx = torch.empty((w.B, w.k), dtype=torch.int32, device=device)
        self.out = torch.empty((w.B, w.H, w.Dv), dtype=torch.bfloat16, device=device)
        self.launches_per_step = 3

    def step(self, ev=None):
        dsa, w, d = self.dsa, self.w, self.d
        e0 = PrefillRun._rec(ev)
        dsa.indexer_topk_decode(d["qI"], d["w"], d["kI_cache"], d["cu_seqlens"], w.k, self.total, self.maxlen,
                                q_scale=d.get("q_scale"), k_scale=d.get("k_scale"), idx_out=self.idx,
                                workspace=self.ws_idx)
        e1 = PrefillRun._rec(ev)
        dsa.sparse_attn_decode(d["q"], d["latent_cache"], d["cu_seqlens"], self.idx, w.Dv, self.total,
                               scale=w.scale, out=self.out, workspace=self.ws_att)
        e2 = PrefillRun._rec(ev)
        if ev is not None:
            ev["indexer_topk_decode"].append((e0, e1))
            ev["sparse_attn_decode"].append((e1, e2))

    def rows(self):
        return self.w.B

    def kernel_work(self):
        w = self.w
        eb = 1 if w.fp8 else 2   # K^I bytes per element (FP8 adds one fp32 scale per key)
        scan_bytes = self.total * (w.dI * eb + (4 if w.fp8 else 0)) + w.B * w.HI * (w.dI * eb + 4) + self.total * 4 * 2
        gather = w.B * w.k * w.Dqk * 2
        return {
            "indexer_topk_decode": {"bytes": scan_bytes, "unit": "GB/s",
                                    "per_unit": (f"dI*{eb} = {w.dI * eb} B of K^I per cached key"
                                                 f"{' + 4 B scale' if w.fp8 else ''} (+ q, w, fp32 scores)"),
                                    "units": self.total},
            "sparse_attn_decode": {"bytes": gather + w.B * w.H * (w.Dqk + w.Dv) * 2, "unit": "GB/s",
                                   "per_unit": f"Dqk*2 = {w.Dqk * 2} B per selected latent row (+ q, out)",
                                   "units": w.B * w.k},
        }

    def host_inputs(self):
        """A decode step's host inputs: the new tokens' queries (q^I, w, q)
        and the sequence offsets.  The K^I and latent caches are device state
        that persists across steps, so they are not re-sent."""
        keys = ("qI", "w", "q", "cu_seqlens") + (("q_scale",) if "q_scale" in self.d else ())
        return {k: self.d[k].cpu().pin_memory() for k in keys}

    def load_inputs(self, host):
        for k, v in host.items():
            self.d[k].copy_(v, non_blocking=True)

    def result(self):
        return self.out


class TrainRun(PrefillRun):
    """Sparse training stage, indexer side (§1.2): the fused indexer + top-k
    selects S_t; the sparse attention forward (eq. (3)) returns its lse; the
    teacher is recomputed on S_t from it (heads summed, L1-normalised); then
    the eq. (8) KL on S_t with dq, dw and dk (dk is zeroed inside the step:
    it accumulates)."""

    def __init__(self, w: W.Workload, device):
        import learned_token_indexer_b200 as dsa
        self.dsa, self.w, self.dev = dsa, w, device
        self.d = W.make_prefill_inputs(w, device)
        self.ws_idx = dsa.Workspace(device)
        self.ws_att = dsa.Workspace(device)
        self.idx = torch.empty((w.B, w.n, w.k), dtype=torch.int32, device=device)
        self.out = torch.empty((w.B, w.n, w.H, w.Dv), dtype=torch.bfloat16, device=device)
        self.lse = torch.empty((w.B, w.n, w.H), dtype=torch.float32, device=device)
        self.teacher = torch.empty((w.B, w.n, w.k), dtype=torch.float32, device=device)
        self.dk = torch.zeros((w.B, w.n, w.dI), dtype=torch.float32, device=device)
        self.kl = torch.zeros((w.B, w.n), dtype=torch.float32, device=device)   # the step's result
        self.res = None
        self.launches_per_step = 0

    def step(self, ev=None):
        dsa, w, d = self.dsa, self.w, self.d
        e0 = self._rec(ev)
        dsa.indexer_topk_prefill(d["qI"], d["kI"], d["w"], w.k, idx_out=self.idx, workspace=self.ws_idx)
        e1 = self._rec(ev)
        dsa.sparse_attn_prefill(d["q"], d["latent"], self.idx, w.Dv, scale=w.scale, out=self.out, lse=self.lse,
                                workspace=self.ws_att)
        e2 = self._rec(ev)
        dsa.attn_teacher_prefill(d["q"], d["latent"], self.idx, self.lse, scale=w.scale, out=self.teacher,
                                 workspace=self.ws_att)
        e3 = self._rec(ev)
        self.dk.zero_()
        self.res = dsa.indexer_kl_sparse(d["qI"], d["kI"], d["w"], self.idx, self.teacher, grad_scale=1.0 / w.n,
                                         dk_out=self.dk, workspace=self.ws_att)
        e4 = self._rec(ev)
        self.kl.copy_(self.res["kl"])
        if ev is not None:
            for name, a, b in (("indexer_topk_prefill", e0, e1), ("sparse_attn", e1, e2), ("attn_teacher", e2, e3),
                               ("indexer_kl", e3, e4)):
                ev[name].append((a, b))
        # fill_trivial_rows, indexer_topk_prefill, sparse_attn, attn_teacher, indexer_kl
        self.launches_per_step = 5

    def selection_diagnostics(self):
        return None

    def kernel_work(self):
        w = self.w
        pairs = count_pairs_needed(0, w.n, w.k)
        ent = selected_entries(0, w.n, w.k)
        return {
            "indexer_topk_prefill": {"flops": 2 * w.HI * w.dI * w.B * pairs, "unit": "TFLOP/s",
                                     "per_unit": f"2*HI*dI = {2 * w.HI * w.dI} FLOP per scored (t,s) pair",
                                     "units": w.B * pairs},
            "sparse_attn": {"flops": 2 * w.H * w.B * ent * (w.Dqk + w.Dv), "unit": "TFLOP/s",
                            "per_unit": f"2*H*(Dqk+Dv) = {2 * w.H * (w.Dqk + w.Dv)} FLOP per selected entry",
                            "units": w.B * ent, "gather_bytes": w.B * ent * w.Dqk * 2},
            "attn_teacher": {"flops": 2 * w.H * w.B * ent * w.Dqk, "unit": "TFLOP/s",
                             "gather_bytes": w.B * ent * w.Dqk * 2,
                             "per_unit": f"2*H*Dqk = {2 * w.H * w.Dqk} FLOP per selected entry (logits recompute)",
                             "units": w.B * ent},
            "indexer_kl": {"flops": 6 * w.HI * w.dI * w.B * ent, "unit": "TFLOP/s",
                           "per_unit": (f"6*HI*dI = {6 * w.HI * w.dI} FLOP per selected entry (scores, dq, dk: "
                                        "three HI x dI products; the kernel's recompute is not counted)"),
                           "units": w.B * ent},
        }

    def host_inputs(self):
        return {k: self.d[k].cpu().pin_memory() for k in ("qI", "kI", "w", "q", "latent")}

    def result(self):
        return self.kl


def time_steps(run, steps, flush):
    """Per-step device times (ms) and, per kernel, the duration of each
    launch (ms) over `steps` timed steps."""
    ev = {name: [] for name in run.kernel_work()}
    starts, ends = [], []
    for _ in range(steps):
        flush.fill_(1)
        s = PrefillRun._rec()
        run.step(ev)
        e = PrefillRun._rec()
        starts.append(s)
        ends.append(e)
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    seg_ms = {name: [a.elapsed_time(b) for a, b in pairs] for name, pairs in ev.items()}
    return step_ms, seg_ms


def time_e2e(run, steps):
    """End to end through the public API, one step after another on one
    stream: H2D of the step's inputs from pinned memory, the step, D2H of its
    result.  Returns (ms per step, H2D bytes, D2H bytes)."""
    host = run.host_inputs()
    res = run.result()
    res_host = torch.empty(res.shape, dtype=res.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = res.numel() * res.element_size()
    run.load_inputs(host)
    run.step()
    res_host.copy_(run.result(), non_blocking=True)
    torch.cuda.synchronize()
    s = PrefillRun._rec()
    for _ in range(steps):
        run.load_inputs(host)
        run.step()
        res_host.copy_(run.result(), non_blocking=True)
    e = PrefillRun._rec()
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps, h2d, d2h


def time_e2e_pipelined(runs, steps):
    """The same per-step work as time_e2e, with consecutive steps overlapped
    the way a serving loop does it: inputs go in on one stream, steps run on a
    second, results come out on a third, and two replicas of the step's
    device buffers alternate (step i + 1's upload and step i - 1's download
    overlap step i).  Every step still uploads its inputs from pinned host
    memory and downloads its result.  Returns ms per step (device events from
    the first upload to the last download)."""
    assert len(runs) >= 2, "the next step's upload goes to the other replica"
    host = runs[0].host_inputs()
    shape, dtype = runs[0].result().shape, runs[0].result().dtype
    res_host = [torch.empty(shape, dtype=dtype, pin_memory=True) for _ in runs]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def go(n, start=None):
        done_run = [None] * len(runs)   # the replica's last step has consumed its inputs
        done_out = [None] * len(runs)   # the replica's last result has been read out
        loaded = [None] * len(runs)     # the replica's inputs for its next step are in

        def upload(i):
            j = i % len(runs)
            with torch.cuda.stream(s_in):
                if done_run[j] is not None:
                    s_in.wait_event(done_run[j])
                runs[j].load_inputs(host)
                loaded[j] = torch.cuda.Event()
                loaded[j].record(s_in)

        if start is not None:
            start.record(s_in)
        upload(0)
        for i in range(n):
            j = i % len(runs)
            r = runs[j]
            # the next step's upload is queued before this step, so it overlaps
            # the step even when a call inside the step waits on the host
            if i + 1 < n:
                upload(i + 1)
            with torch.cuda.stream(s_run):
                s_run.wait_event(loaded[j])
                if done_out[j] is not None:
                    s_run.wait_event(done_out[j])
                r.step()
                done_run[j] = torch.cuda.Event()
                done_run[j].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_run[j])
                res_host[j].copy_(r.result(), non_blocking=True)
                done_out[j] = torch.cuda.Event()
                done_out[j].record(s_out)
        end = torch.cuda.Event(enable_timing=True)
        end.record(s_out)
        return end

    go(2 * len(runs))
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = go(steps, start)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps


def cpu_baseline(w: W.Workload, budget_s: float = 15.0, run_inputs=None):
    """The oracle, as it stands, on a seeded sample of the workload's rows."""
    import oracle as O
    threads = _blas_threads()
    if w.kind == "decode":
        d = run_inputs if run_inputs is not None else W.make_decode_inputs(w, "cpu")
        cu = d["cu_seqlens"].cpu().numpy()
        ww = d["w"].cpu().double().numpy()
        t0 = time.perf_counter()
        done = 0
        for b in range(w.B):
            lo, hi = int(cu[b]), int(cu[b + 1])
            qb, kc = _decode_indexer_host(O, w, d, b, lo, hi)
            s = O.indexer_scores_row(qb, kc, ww[b])
            sel = O.causal_topk_row(s, hi - lo - 1, w.k)
            lat = d["latent_cache"][lo:hi].cpu().double().numpy()
            O.sparse_attention_row(d["q"][b].cpu().double().numpy(), lat, sel, w.scale, w.Dv)
            done += 1
            if time.perf_counter() - t0 > budget_s:
                break
        dt = time.perf_counter() - t0
        return {"value": done / dt, "unit": METRIC["decode"][1], "cores": threads, "kind": "oracle",
                "sample": f"{done} of {w.B} sequences of one decode step (float64 numpy)"}
    d = run_inputs if run_inputs is not None else _host_prefill_inputs(w)
    rows = W.sample_rows(w, 4096)
    rng = np.random.default_rng(7)
    rng.shuffle(rows)
    one = _oracle_train_row if w.kind == "train" else _oracle_row
    t0 = time.perf_counter()
    done = 0
    for b, i in rows:
        one(O, w, d, b, i)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    what = ("indexer + top-k + attention + teacher + eq. (8) KL with gradients" if w.kind == "train"
            else "indexer + top-k + attention")
    return {"value": done / dt, "unit": METRIC[w.kind][1], "cores": threads, "kind": "oracle",
            "sample": f"{done} seeded query rows of B*n={w.B * w.n} (uniform over positions), {what} per row, "
                      f"float64 numpy"}


def _host_prefill_inputs(w):
    return W.make_prefill_inputs(w, "cpu")


def _oracle_train_row(O, w, d, b, i):
    """One row of the sparse-stage indexer step: selection, attention forward,
    teacher on S_t, eq. (8) KL with gradients."""
    q = d["qI"][b, i].double().numpy()
    kk = d["kI"][b].double().numpy()
    ww = d["w"][b, i].double().numpy()
    s = O.indexer_scores_row(q, kk[: i + 1], ww)
    sel = O.causal_topk_row(s, i, w.k)
    qa = d["q"][b, i].double().numpy()
    lat = d["latent"][b].double().numpy()
    O.sparse_attention_row(qa, lat, sel, w.scale, w.Dv)
    p = O.attention_teacher_row(qa, lat, sel, w.scale)
    O.indexer_kl_sparse_row(q, kk, ww, sel, p, 1.0 / w.n)


def _oracle_row(O, w, d, b, i):
    if w.fp8:
        q = O.dequantize(d["qI"][b, i].view(torch.uint8).numpy(), d["q_scale"][b, i].numpy(), 2)
        k = O.dequantize(d["kI"][b, : i + 1].view(torch.uint8).numpy(), d["k_scale"][b, : i + 1].numpy(), 1)
    else:
        q = d["qI"][b, i].double().numpy()
        k = d["kI"][b, : i + 1].double().numpy()
    s = O.indexer_scores_row(q, k, d["w"][b, i].double().numpy())
    sel = O.causal_topk_row(s, i, w.k)
    lat = d["latent"][b].double().numpy()
    O.sparse_attention_row(d["q"][b, i].double().numpy(), lat, sel, w.scale, w.Dv)


def _decode_indexer_host(O, w, d, b, lo, hi):
    """Float64 q^I of sequence b and its K^I cache rows (dequantised for FP8)."""
    if w.fp8:
        q = O.dequantize(d["qI"][b].view(torch.uint8).cpu().numpy(), d["q_scale"][b].cpu().numpy(), 2)
        k = O.dequantize(d["kI_cache"][lo:hi].view(torch.uint8).cpu().numpy(), d["k_scale"][lo:hi].cpu().numpy(), 1)
        return q, k
    return d["qI"][b].cpu().double().numpy(), d["kI_cache"][lo:hi].cpu().double().numpy()


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def workload_label(w: W.Workload):
    if w.kind == "decode":
        return (f"decode B={w.B} L~U[{w.L_min},{w.L_max}] HI={w.HI} dI={w.dI} k={w.k} "
                f"{'fp8-e4m3' if w.fp8 else 'bf16'} K^I cache; "
                f"attn H={w.H} latent {w.Dqk}/{w.Dv}")
    dt = "fp8-e4m3 indexer" if w.fp8 else ("bf16 integer-valued indexer" if w.integer_valued else "bf16 indexer")
    if w.kind == "train":
        return (f"sparse-stage indexer step: prefill B={w.B} n={w.n} HI={w.HI} dI={w.dI} k={w.k} {dt}; "
                f"attn H={w.H} latent {w.Dqk}/{w.Dv} with lse; teacher on S_t from it; KL fwd + dq, dw, dk")
    ch = f" in {w.chunk}-query chunks" if w.chunk else ""
    return (f"prefill B={w.B} n={w.n} HI={w.HI} dI={w.dI} k={w.k} {dt}{ch}; attn H={w.H} latent {w.Dqk}/{w.Dv}")


def workload_config(w: W.Workload, world: int) -> dict:
    """The JSON line's `config`: the workload and how it is laid out (the same
    dict for the B200 arm and the reference arm)."""
    return {"workload": workload_label(w), "global_batch": world * w.B,
            "seq_len": w.n if w.kind != "decode" else w.L_max,
            "parallelism": f"replicas x{world} (independent batches per GPU)",
            "l2": "flushed (256 MiB write) before every timed step, outside the timed events"}


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank number over all ranks (identity without a process
    group): every multi-rank duration in the JSON line is the slowest rank's."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    if torch.distributed.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w, rank: int):
    """Each rank draws its own batch of the same workload (weak scaling)."""
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 7919 * rank)


def job_throughput(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Units every rank processed in one step, over the slowest rank's step time."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def make_run(w, dev):
    return {"decode": DecodeRun, "train": TrainRun}.get(w.kind, PrefillRun)(w, dev)


def measure_fp8_peak(dev, n: int = 8192, reps: int = 10):
    """Dense e4m3 tensor throughput on this GPU: torch._scaled_mm (a library
    GEMM, unit scales, bf16 output) on n x n x n, best of `reps` launches,
    2 n^3 FLOP each.  None when the call is unavailable."""
    try:
        g = torch.Generator(device=dev).manual_seed(5)
        a = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), generator=g, device=dev).to(torch.float8_e4m3fn).t()   # column-major operand
        one = torch.ones((), device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        best = float("inf")
        for _ in range(reps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e.record()
            torch.cuda.synchronize()
            best = min(best, s.elapsed_time(e))
        del a, b
        return {"tflops": round(2.0 * n ** 3 / (best * 1e-3) / 1e12, 1),
                "how": f"torch._scaled_mm e4m3 x e4m3 -> bf16, {n}^3, best of {reps} (CUDA events), in this run"}
    except Exception as exc:   # pragma: no cover - depends on the torch build
        return {"tflops": None, "how": f"unavailable: {type(exc).__name__}"}


def measure_workload(w, args, dev, world, rank, local, steps, warmup, cpu_budget, fp8_peak=None):
    """Time one workload: `warmup` untimed steps, then exactly `steps` timed
    steps (CUDA events on the launching stream, L2 flushed before each, a
    barrier on both sides), per-kernel roofline, end-to-end loops and, on
    rank 0 at N = 1, the oracle on a bounded sample.  Returns the record on
    rank 0 (None elsewhere); every rank takes the same collective steps."""
    w = rank_workload(w, rank)
    run = make_run(w, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        run.step()
    torch.cuda.synchronize()
    run.ws_idx.check()
    run.ws_att.check()
    sampler = ClockSampler(local)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    step_ms, seg_ms = time_steps(run, steps, flush)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    run.ws_idx.check()
    run.ws_att.check()
    ms = max_over_ranks(float(np.mean(step_ms)), dev)
    e2e = None
    if not args.no_e2e:
        n_e2e = max(4, min(20, steps))
        serial_ms, h2d, d2h = time_e2e(run, n_e2e)
        replica = make_run(w, dev)
        pipe_ms = time_e2e_pipelined([run, replica], n_e2e)
        del replica
        serial_ms = max_over_ranks(serial_ms, dev)
        pipe_ms = max_over_ranks(pipe_ms, dev)
        # the loop a serving system would run: whichever of the two is faster
        # (overlap pays once transfers are long; tiny steps are launch-bound)
        modes = {"pipelined": (pipe_ms, "upload, step and download of consecutive steps overlap on three streams, "
                                        "two replicas of the device buffers alternate"),
                 "serial": (serial_ms, "upload, step and download one after another on one stream")}
        best = min(modes, key=lambda m: modes[m][0])
        e2e = {"value": job_throughput(world, run.rows(), modes[best][0]), "unit": METRIC[w.kind][1],
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": modes[best][0],
               "mode": f"{best}: {modes[best][1]}",
               "modes_ms_per_step": {m: round(v[0], 4) for m, v in modes.items()}}
    diag = run.selection_diagnostics() if (rank == 0 and hasattr(run, "selection_diagnostics")) else None
    launches = run.launches_per_step * steps
    work = run.kernel_work()
    rows = run.rows()
    del run, flush
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    # a kernel timed inside a long step runs at the power-capped clock: its
    # tensor peak is the sustained figure, the burst one for a short step
    long_step = ms >= LONG_STEP_MS and "bf16_tflops_sustained" in peaks
    tensor_peak = peaks["bf16_tflops_sustained"] if long_step else peaks["bf16_tflops"]
    names = list(work.keys())
    kernels = {}
    for name, wk in work.items():
        # per launch: each step launches each kernel once per chunk
        per_step_launches = max(1, len(seg_ms[name]) // max(1, steps))
        t_launch = float(np.mean(seg_ms[name]))
        fp8_mma = w.fp8 and name == names[0] and "flops" in wk
        if "flops" in wk:
            per_launch = wk["flops"] / per_step_launches
            # a contraction takes the peak of its own dtype: e4m3 = the
            # measured bf16 figure x the nominal fp8 / bf16 ratio (2)
            peak = tensor_peak * (2.0 if fp8_mma else 1.0)
            ach = per_launch / (t_launch * 1e-3) / 1e12
            bound = "tensor"
        else:
            per_launch = wk["bytes"] / per_step_launches
            peak = peaks["hbm_gbs"]
            ach = per_launch / (t_launch * 1e-3) / 1e9
            bound = "hbm"
        tkey = {"indexer_topk_decode": "indexer_scan", "sparse_attn_decode": "latent_attn_decode"}.get(name, name)
        # the training step's selection and attention are the prefill workload's launches
        twl = "prefill" if (w.kind == "train" and name in ("indexer_topk_prefill", "sparse_attn")) else w.name
        t_bytes, t_case = measured_traffic(tkey, twl)
        kernels[name] = {"bound": bound, "achieved": round(ach, 2), "peak": peak, "unit": wk["unit"],
                         "frac": round(ach / peak, 4), "ms_per_launch": round(t_launch, 4),
                         "traffic": t_bytes,
                         "algorithmic_per_launch": per_launch, "per_unit": wk["per_unit"]}
        if t_case:
            kernels[name]["traffic_case"] = t_case
        if bound == "tensor":
            kernels[name]["peak_source"] = (
                f"sustained bf16 ({peaks['bf16_tflops_sustained']} TFLOP/s: timed inside a {ms:.0f} ms step)"
                if long_step else "burst bf16")
            kernels[name]["frac_of_burst"] = round(ach / (peaks["bf16_tflops"] * (2.0 if fp8_mma else 1.0)), 4)
        if fp8_mma:
            kernels[name]["peak_source"] += "; fp8 = 2 x that bf16 figure (nominal ratio)"
            if fp8_peak and fp8_peak.get("tflops"):
                kernels[name]["fp8_peak_measured"] = dict(fp8_peak)
                kernels[name]["frac_of_measured_fp8"] = round(ach / fp8_peak["tflops"], 4)
        if "gather_bytes" in wk:
            # the selected latent rows come from L2, not HBM: their rate is the
            # secondary bound of the gathering kernels
            kernels[name]["l2_gather_TBps"] = round(wk["gather_bytes"] / per_step_launches / (t_launch * 1e-3) / 1e12,
                                                    3)
    dom = max(kernels, key=lambda n: kernels[n]["ms_per_launch"] * max(1, len(seg_ms[n]) // max(1, steps)))
    roof = {k: kernels[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roof["kernel"] = dom
    if "traffic_case" in kernels[dom]:
        roof["traffic_case"] = kernels[dom]["traffic_case"]
    roof["peak_source"] = (f"{peak_src} "
                           f"({kernels[dom].get('peak_source', 'copy bandwidth')}; of {peak_src})")
    if "frac_of_burst" in kernels[dom]:
        roof["frac_of_burst"] = kernels[dom]["frac_of_burst"]
    if w.kind == "decode" and all(k["bound"] == "hbm" for k in kernels.values()):
        # the decode step's scan (+ top-k) and gather together: the step's
        # algorithmic bytes over the summed event-timed launch durations
        tot_b = sum(k["algorithmic_per_launch"] for k in kernels.values())
        tot_ms = sum(k["ms_per_launch"] for k in kernels.values())
        ach = tot_b / (tot_ms * 1e-3) / 1e9
        roof["scan_plus_gather"] = {"achieved": round(ach, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                    "frac": round(ach / peaks["hbm_gbs"], 4), "kernels": list(kernels)}
    metric, unit = METRIC[w.kind]
    rec = {
        "metric": metric, "value": job_throughput(world, rows, ms), "unit": unit,
        "steps": steps, "warmup": warmup, "ms_per_step": ms,
        "dtype": "fp8-e4m3 indexer / bf16 attention, fp32 accumulate" if w.fp8 else "bf16 in, fp32 accumulate",
        "config": workload_config(w, world),
        "roofline": roof,
        "kernels": kernels,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if e2e is not None:
        rec["e2e"] = e2e
    if diag:
        rec["diagnostics"] = diag
    if world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_baseline(w, cpu_budget)
    return rec


# The default run: the largest single-GPU prefill configuration is the line's
# value; the other configurations of the metric are sub-records.
DEFAULT_WORKLOAD = "long_prefill"
DEFAULT_SUBS = ("prefill", "prefill_fp8", "decode", "short_prefill")
HEADLINE_METRIC = "prefill query-tokens/s (indexer+top-k+sparse attn) & decode tokens/s; % roofline"


def run_b200(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)
    from learned_token_indexer_b200.build import build
    if rank == 0:
        build()
    if world > 1:
        torch.distributed.barrier()
    main_w = W.ALL[args.workload]
    subs = [] if args.no_subs else [s for s in (args.subs.split(",") if args.subs else DEFAULT_SUBS)
                                    if s and s != args.workload]
    need_fp8 = any(W.ALL[x].fp8 for x in [args.workload] + subs)
    fp8_peak = measure_fp8_peak(dev) if (need_fp8 and rank == 0) else None
    rec = measure_workload(main_w, args, dev, world, rank, local, args.steps, args.warmup, args.cpu_budget,
                           fp8_peak)
    sub_recs = {}
    for name in subs:
        r = measure_workload(W.ALL[name], args, dev, world, rank, local, args.sub_steps, args.warmup,
                             args.sub_cpu_budget, fp8_peak)
        if rank == 0:
            sub_recs[name] = r
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": HEADLINE_METRIC if main_w.kind == "prefill" and args.workload == DEFAULT_WORKLOAD
            else rec["metric"],
            "value": rec["value"], "unit": rec["unit"], "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": rec["dtype"],
            "data": "synthetic (seeded, HBM-resident)", "config": rec["config"]}
    if line["metric"] == HEADLINE_METRIC:
        line["value_is"] = (f"{rec['metric']} on the largest single-GPU configuration ({args.workload}); "
                            "decode tokens/s and the other prefill configurations are in sub_records")
    for key in ("roofline", "kernels", "gpu_launches", "clocks", "e2e", "cpu_baseline", "diagnostics"):
        if key in rec:
            line[key] = rec[key]
    if fp8_peak:
        line["fp8_peak_measured"] = fp8_peak
    if sub_recs:
        line["sub_records"] = sub_recs
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# reference arm: the oracle on host cores
# ----------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle as O
    w = W.ALL[args.workload]
    metric, unit = METRIC[w.kind]
    if args.workload == DEFAULT_WORKLOAD:
        metric = HEADLINE_METRIC
    world = int(os.environ.get("WORLD_SIZE", "1"))
    total_budget = args.ref_budget
    nsteps = args.steps + args.warmup
    if w.kind == "decode":
        d = W.make_decode_inputs(w, "cpu")
        cu = d["cu_seqlens"].numpy()
        def one(b):
            lo, hi = int(cu[b]), int(cu[b + 1])
            qb, kc = _decode_indexer_host(O, w, d, b, lo, hi)
            s = O.indexer_scores_row(qb, kc, d["w"][b].double().numpy())
            sel = O.causal_topk_row(s, hi - lo - 1, w.k)
            O.sparse_attention_row(d["q"][b].double().numpy(), d["latent_cache"][lo:hi].double().numpy(), sel,
                                   w.scale, w.Dv)
        units = list(range(w.B))
        unit_name = "sequences"
    else:
        d = _host_prefill_inputs(w)
        units = W.sample_rows(w, 4096)
        np.random.default_rng(7).shuffle(units)
        row_fn = _oracle_train_row if w.kind == "train" else _oracle_row
        def one(u):
            row_fn(O, w, d, *u)
        unit_name = "query rows"
    t0 = time.perf_counter()
    one(units[0])
    per_unit = max(1e-4, time.perf_counter() - t0)
    per_step = max(1, int(total_budget / nsteps / per_unit))
    pos = 1
    def step():
        nonlocal pos
        for _ in range(per_step):
            one(units[pos % len(units)])
            pos += 1
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = args.steps * per_step / dt
    threads = _blas_threads()
    sample = (f"{per_step} seeded {unit_name} per step of B*n={w.B * max(w.n, 1)} "
              f"({'uniform over positions' if w.kind != 'decode' else 'of one decode step'}), float64 numpy oracle")
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": workload_config(w, world),
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.ALL))
    ap.add_argument("--subs", default="", help="comma-separated workloads measured after the main one "
                                                "(default: " + ",".join(DEFAULT_SUBS) + ")")
    ap.add_argument("--no-subs", action="store_true")
    ap.add_argument("--sub-steps", type=int, default=50)
    ap.add_argument("--sub-cpu-budget", type=float, default=10.0)
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override a field of the main workload (e.g. B=8, L_max=8192) for a smaller case, "
                         "such as a profiler capture")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=90.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.set:
        base = W.ALL[args.workload]
        changes = {}
        for kv in args.set:
            key, _, val = kv.partition("=")
            if not hasattr(base, key):
                ap.error(f"--set: workload has no field {key!r}")
            changes[key] = type(getattr(base, key))(val)
        W.ALL[args.workload] = dataclasses.replace(base, **changes)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_b200(args)


if __name__ == "__main__":
    main()
