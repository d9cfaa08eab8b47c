"""Seeded synthetic workloads for the DSA hot path.

This module only draws random inputs; it holds none of the method's
arithmetic.  Both the CUDA path and the CPU oracle consume exactly the tensors
it returns (the oracle gets host copies).  The one transformation it applies
is input preparation for the FP8 workload: each token's values are divided by
a per-token scale (amax / 448) and rounded to FP8-e4m3 by torch's cast; the
codes and the fp32 scales then *are* the inputs of both sides.

Shapes and value distributions follow the workloads the DSA path is
measured on (tiny integer prefill, integer prefill n=8192, FP8 prefill
2x32768, decode batch 64 with ragged contexts 4096..65536 (bf16 or FP8 key
cache), long prefill n=131072 in 8192-query chunks, and the sparse training
stage's indexer KL on the n=8192 prefill).  No dataset is involved.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

FP8_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill", "decode" or "train" (indexer KL, eq. (8))
    B: int
    n: int                    # tokens per sequence (prefill)
    HI: int                   # indexer heads
    dI: int                   # indexer head dim
    k: int                    # top-k budget
    H: int                    # attention query heads
    Dqk: int                  # latent row width (key)
    Dv: int                   # value width (first Dv columns of the latent row)
    qk_dist: str              # "int" (uniform integers) or "normal"
    qk_int_max: int = 0       # integers in [-qk_int_max, qk_int_max]
    w_den: int = 0            # w = randint(-w_den, w_den) / w_den (int configs)
    w_std: float = 0.1        # w ~ N(0, w_std^2) (float configs)
    fp8: bool = False
    chunk: int = 0            # prefill query chunk (0 = whole sequence)
    seed: int = 0
    L_min: int = 0            # decode context lengths uniform in [L_min, L_max]
    L_max: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.Dqk)

    @property
    def integer_valued(self) -> bool:
        return self.qk_dist == "int"


TINY = Workload("tiny", "prefill", B=1, n=512, HI=4, dI=32, k=16, H=4, Dqk=64, Dv=64,
                qk_dist="int", qk_int_max=4, w_den=4, seed=0)
PREFILL = Workload("prefill", "prefill", B=1, n=8192, HI=64, dI=128, k=2048, H=16, Dqk=576,
                   Dv=512, qk_dist="int", qk_int_max=3, w_den=16, seed=1)
PREFILL_FP8 = Workload("prefill_fp8", "prefill", B=2, n=32768, HI=64, dI=128, k=2048, H=16,
                       Dqk=576, Dv=512, qk_dist="normal", w_std=0.1, fp8=True, seed=2)
DECODE = Workload("decode", "decode", B=64, n=0, HI=64, dI=128, k=2048, H=128, Dqk=576, Dv=512,
                  qk_dist="normal", w_std=0.1, seed=3, L_min=4096, L_max=65536)
DECODE_FP8 = Workload("decode_fp8", "decode", B=64, n=0, HI=64, dI=128, k=2048, H=128, Dqk=576, Dv=512,
                      qk_dist="normal", w_std=0.1, fp8=True, seed=3, L_min=4096, L_max=65536)
LONG = Workload("long_prefill", "prefill", B=1, n=131072, HI=64, dI=128, k=2048, H=16, Dqk=576,
                Dv=512, qk_dist="normal", w_std=0.1, chunk=8192, seed=4)
# Short prefill (every row has t + 1 <= k): the case §2 says DSA runs as
# masked dense attention; the prefill workload's distributions, 8 sequences.
SHORT_PREFILL = Workload("short_prefill", "prefill", B=8, n=2048, HI=64, dI=128, k=2048, H=16, Dqk=576, Dv=512,
                         qk_dist="int", qk_int_max=3, w_den=16, seed=5)
# Sparse training stage (eq. (8)): the prefill workload's inputs; the teacher
# comes from the sparse attention on each row's selected set.
INDEXER_KL = Workload("indexer_kl", "train", B=1, n=8192, HI=64, dI=128, k=2048, H=16, Dqk=576, Dv=512,
                      qk_dist="int", qk_int_max=3, w_den=16, seed=1)

ALL = {w.name: w for w in (TINY, PREFILL, PREFILL_FP8, DECODE, DECODE_FP8, LONG, SHORT_PREFILL, INDEXER_KL)}


def scaled(w: Workload, **changes) -> Workload:
    """A copy of a workload with some sizes changed (for small parity cases)."""
    return dataclasses.replace(w, **changes)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _ints(shape, lim, g, device):
    return torch.randint(-lim, lim + 1, shape, generator=g, device=device)


def quantize_fp8_per_token(x: torch.Tensor, group_dims: int):
    """Per-token FP8-e4m3 input preparation: scale = amax / 448 over the last
    ``group_dims`` dimensions, codes = round-to-nearest-even(x / scale)."""
    red = tuple(range(x.dim() - group_dims, x.dim()))
    amax = x.float().abs().amax(dim=red)
    scale = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
    y = x.float() / scale.reshape(scale.shape + (1,) * group_dims)
    codes = y.clamp(-FP8_MAX, FP8_MAX).to(torch.float8_e4m3fn)
    return codes, scale.float().contiguous()


def make_prefill_inputs(w: Workload, device="cpu", n: Optional[int] = None,
                        with_attention: bool = True, keep_bf16: bool = False) -> dict:
    """All inputs of one prefill workload (whole sequence; chunks are views).

    Returns a dict of tensors on ``device``:
      qI [B,n,HI,dI] bf16 (or e4m3 codes + q_scale [B,n]),
      kI [B,n,dI]    bf16 (or e4m3 codes + k_scale [B,n]),
      w  [B,n,HI]    fp32,
      q  [B,n,H,Dqk] bf16, latent [B,n,Dqk] bf16  (if with_attention).
    FP8 workloads with keep_bf16 also return qI_bf16 / kI_bf16: the same
    draws rounded to bf16 instead of quantised (a reference selection).
    """
    n = w.n if n is None else n
    g = _gen(device, w.seed)
    out = {}
    if w.qk_dist == "int":
        out["qI"] = _ints((w.B, n, w.HI, w.dI), w.qk_int_max, g, device).to(torch.bfloat16)
        out["kI"] = _ints((w.B, n, w.dI), w.qk_int_max, g, device).to(torch.bfloat16)
        out["w"] = (_ints((w.B, n, w.HI), w.w_den, g, device).float() / w.w_den).contiguous()
    else:
        qI = torch.randn((w.B, n, w.HI, w.dI), generator=g, device=device)
        kI = torch.randn((w.B, n, w.dI), generator=g, device=device)
        if w.fp8:
            out["qI"], out["q_scale"] = quantize_fp8_per_token(qI, 2)
            out["kI"], out["k_scale"] = quantize_fp8_per_token(kI, 1)
            if keep_bf16:
                out["qI_bf16"] = qI.to(torch.bfloat16)
                out["kI_bf16"] = kI.to(torch.bfloat16)
        else:
            out["qI"] = qI.to(torch.bfloat16)
            out["kI"] = kI.to(torch.bfloat16)
        del qI, kI
        out["w"] = (torch.randn((w.B, n, w.HI), generator=g, device=device) * w.w_std).float()
    if with_attention:
        out["q"] = torch.randn((w.B, n, w.H, w.Dqk), generator=g, device=device).to(torch.bfloat16)
        out["latent"] = torch.randn((w.B, n, w.Dqk), generator=g, device=device).to(torch.bfloat16)
    return out


def decode_lengths(w: Workload, B: Optional[int] = None) -> torch.Tensor:
    """Seeded context lengths L_b uniform in [L_min, L_max] (CPU generator)."""
    B = w.B if B is None else B
    g = _gen("cpu", w.seed)
    return torch.randint(w.L_min, w.L_max + 1, (B,), generator=g)


def make_decode_inputs(w: Workload, device="cpu", lengths: Optional[torch.Tensor] = None) -> dict:
    """Inputs of one decode step: ragged caches plus the new token's queries.

    Returns cu_seqlens int64 [B+1] (device), lengths (CPU),
      qI [B,HI,dI] bf16, w [B,HI] fp32, kI_cache [sum L, dI] bf16,
      q [B,H,Dqk] bf16, latent_cache [sum L, Dqk] bf16.
    FP8 workloads draw the same bf16 values, then quantise q^I per query
    token (q_scale [B]) and the K^I cache per key (k_scale [sum L]) to e4m3.
    """
    lengths = decode_lengths(w) if lengths is None else lengths
    B = lengths.numel()
    cu = torch.zeros(B + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(lengths, 0)
    total = int(cu[-1])
    g = _gen(device, w.seed + 1000)
    out = {"lengths": lengths, "cu_seqlens": cu.to(device)}
    out["qI"] = torch.randn((B, w.HI, w.dI), generator=g, device=device).to(torch.bfloat16)
    out["w"] = (torch.randn((B, w.HI), generator=g, device=device) * w.w_std).float()
    out["kI_cache"] = torch.randn((total, w.dI), generator=g, device=device).to(torch.bfloat16)
    out["q"] = torch.randn((B, w.H, w.Dqk), generator=g, device=device).to(torch.bfloat16)
    out["latent_cache"] = torch.randn((total, w.Dqk), generator=g, device=device).to(torch.bfloat16)
    if w.fp8:
        out["qI"], out["q_scale"] = quantize_fp8_per_token(out["qI"], 2)
        out["kI_cache"], out["k_scale"] = quantize_fp8_per_token(out["kI_cache"], 1)
    return out


def sample_rows(w: Workload, nrows: int = 256, n: Optional[int] = None, salt: int = 0):
    """Seeded sample of query rows (b, i) for parity checks on large workloads.

    Always includes rows 0, 1, k-2, k-1, k and the last row of batch 0 (and,
    for chunked workloads, the first and last row of every chunk); the rest
    are drawn uniformly.
    """
    n = w.n if n is None else n
    g = torch.Generator().manual_seed(1234 + w.seed + salt)
    must = {0, 1, w.k - 2, w.k - 1, w.k, n - 1}
    if w.chunk:
        for c0 in range(0, n, w.chunk):
            must.add(c0)
            must.add(min(n, c0 + w.chunk) - 1)
    rows = {(0, i) for i in must if 0 <= i < n}
    while len(rows) < min(nrows, w.B * n):
        b = int(torch.randint(0, w.B, (1,), generator=g))
        i = int(torch.randint(0, n, (1,), generator=g))
        rows.add((b, i))
    return sorted(rows)


def make_selection(B: int, nq: int, kv_len: int, k: int, q_offset: int = 0, seed: int = 0,
                   device="cpu", rows_per_draw: int = 2048) -> torch.Tensor:
    """Seeded synthetic selections (input of the sparse-stage KL, not a top-k).

    Row i of each sequence sits at t = q_offset + i and holds min(k, t + 1)
    distinct positions drawn uniformly from [0, t] in random slot order,
    then -1 in the unused slots.  Returns int32 [B, nq, k] on ``device``.
    """
    g = _gen(device, seed + 77)
    out = torch.empty((B, nq, k), dtype=torch.int32, device=device)
    pos = torch.arange(kv_len, device=device)
    for b in range(B):
        for r0 in range(0, nq, rows_per_draw):
            r1 = min(nq, r0 + rows_per_draw)
            t = (q_offset + torch.arange(r0, r1, device=device))[:, None]
            u = torch.rand((r1 - r0, kv_len), generator=g, device=device)
            u = torch.where(pos[None, :] <= t, u, torch.full_like(u, 2.0))      # keys after t never drawn
            kk = min(k, kv_len)
            sel = torch.topk(u, kk, dim=1, largest=False).indices
            sel = torch.where(sel <= t, sel, torch.full_like(sel, -1))
            # valid first, then -1 (the index semantics of the prefill selector)
            key = torch.where(sel >= 0, torch.zeros_like(sel), torch.ones_like(sel))
            sel = torch.gather(sel, 1, torch.sort(key, dim=1, stable=True).indices)
            row = torch.full((r1 - r0, k), -1, dtype=torch.int32, device=device)
            row[:, :kk] = sel.to(torch.int32)
            out[b, r0:r1] = row
    return out


def make_teacher(shape, seed: int = 0, device="cpu", zero_frac: float = 0.1) -> torch.Tensor:
    """Seeded synthetic teacher weights >= 0 (fp32) with a fraction of exact
    zeros; entries in unused slots are drawn too (the KL ignores them)."""
    g = _gen(device, seed + 91)
    t = torch.rand(shape, generator=g, device=device) ** 3
    z = torch.rand(shape, generator=g, device=device) < zero_frac
    return torch.where(z, torch.zeros_like(t), t).float().contiguous()
