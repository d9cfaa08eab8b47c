"""B200 (sm_100a) DeepSeek Sparse Attention hot path: Python binding.

Every function here marshals torch tensors (device pointers, sizes, the
current CUDA stream) into one call of libdsa.so (include/dsa.h); all
arithmetic runs in the library's CUDA kernels.  Torch is used only to
allocate outputs and workspaces and to provide the stream.

Entry points (page "2.2.1 · DSA 与索引器", §1.1 eqs. (1)-(3), §2 decode):
    indexer_topk_prefill  fused indexer + causal top-k of a prefill chunk
    sparse_attn_prefill   sparse attention over the selected latent rows
    indexer_topk_decode   one decode step of the indexer + top-k (ragged caches)
    sparse_attn_decode    the decode step's sparse attention (MQA form)
    indexer_scores, topk_rows, selftest_bounded_wait   debug / test
"""

from __future__ import annotations

import ctypes as C
import math
from typing import Optional

import torch

from . import _lib

BF16, FP8_E4M3 = 0, 1
STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_WORKSPACE",
          4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT", 6: "DSA_ERR_DEVICE_CHECK"}


class DSAError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def lib():
    return _lib.load()


def _check(st: int):
    if st != 0:
        raise DSAError(st, lib().dsa_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(device) -> C.c_void_p:
    return C.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype in (torch.float8_e4m3fn, torch.uint8):
        return FP8_E4M3
    raise TypeError(f"indexer operands must be bfloat16 or float8_e4m3fn, got {t.dtype}")


class Workspace:
    """A device scratch buffer (256-byte status header + kernel scratch).

    Grows on demand; the header is zeroed once when the buffer is made."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            _check(lib().dsa_workspace_init(_ptr(self.buf), self.buf.numel(), _stream(self.device)))
        return self.buf

    def status(self):
        """Synchronise and return (status_code, detail); clears the status."""
        if self.buf is None:
            return 0, 0
        d = C.c_uint32(0)
        st = lib().dsa_read_device_status(_ptr(self.buf), _stream(self.device), C.byref(d))
        return st, d.value

    def check(self):
        st, d = self.status()
        if st != 0:
            raise DSAError(st, lib().dsa_last_error().decode())


_default_ws: dict = {}


def _ws(ws: Optional[Workspace], device) -> Workspace:
    if ws is not None:
        return ws
    key = torch.device(device).index if torch.device(device).index is not None else torch.cuda.current_device()
    if key not in _default_ws:
        _default_ws[key] = Workspace(torch.device("cuda", key))
    return _default_ws[key]


def version() -> str:
    return lib().dsa_version().decode()


def set_wait_timeout_ns(ns: int):
    lib().dsa_set_wait_timeout_ns(int(ns))


def get_wait_timeout_ns() -> int:
    return int(lib().dsa_get_wait_timeout_ns())


# --------------------------------------------------------------------------
# Prefill
# --------------------------------------------------------------------------

def indexer_topk_prefill(qI, kI, w, k: int, q_offset: int = 0, q_scale=None, k_scale=None,
                         idx_out=None, score_out=None, return_scores: bool = False,
                         workspace: Optional[Workspace] = None, full_workspace: bool = False):
    """Fused eq. (1) + eq. (2) for a prefill chunk.

    qI [B, nq, HI, dI], kI [B, kv_len, dI] (bf16, or e4m3 with q_scale [B, nq]
    and k_scale [B, kv_len]), w [B, nq, HI] fp32.  Returns idx [B, nq, k]
    int32 (and scores [B, nq, k] fp32 if asked).

    The default workspace is bounded past 16384 keys (rows whose candidates
    outgrow it take a second pass, and the call synchronises once);
    full_workspace=True sizes the candidate buffers for the whole history
    (no second pass, no synchronisation, memory grows with kv_len)."""
    B, nq, HI, dI = qI.shape
    kv_len = kI.shape[1]
    dt = _dtype_code(qI)
    dev = qI.device
    if idx_out is None:
        idx_out = torch.empty((B, nq, k), dtype=torch.int32, device=dev)
    if return_scores and score_out is None:
        score_out = torch.empty((B, nq, k), dtype=torch.float32, device=dev)
    L = lib()
    size = L.dsa_indexer_topk_prefill_workspace_full if full_workspace else L.dsa_indexer_topk_prefill_workspace
    need = size(B, nq, kv_len, HI, dI, k, dt)
    wsb = _ws(workspace, dev).get(need)
    # exactly `need` bytes: the library picks the capped or the full-history
    # mode from the size it is given
    _check(L.dsa_indexer_topk_prefill(B, nq, q_offset, kv_len, HI, dI, k, dt, _ptr(qI), _ptr(q_scale), _ptr(kI),
                                      _ptr(k_scale), _ptr(w), _ptr(idx_out), _ptr(score_out), _ptr(wsb),
                                      need, _stream(dev)))
    return (idx_out, score_out) if score_out is not None else idx_out


def sparse_attn_prefill(q, latent, idx, dv: int, scale: Optional[float] = None, out=None, lse=None,
                        return_lse: bool = False, workspace: Optional[Workspace] = None):
    """Eq. (3): q [B, nq, H, Dqk] bf16, latent [B, kv_len, Dqk] bf16,
    idx [B, nq, k] int32 -> out [B, nq, H, dv] bf16 (and lse [B, nq, H])."""
    B, nq, H, Dqk = q.shape
    kv_len = latent.shape[1]
    k = idx.shape[-1]
    scale = Dqk ** -0.5 if scale is None else scale
    dev = q.device
    if out is None:
        out = torch.empty((B, nq, H, dv), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, nq, H), dtype=torch.float32, device=dev)
    L = lib()
    wsb = _ws(workspace, dev).get(L.dsa_sparse_attn_workspace())
    _check(L.dsa_sparse_attn_prefill(B, nq, kv_len, H, Dqk, dv, k, float(scale), _ptr(q), _ptr(latent), _ptr(idx),
                                     _ptr(out), _ptr(lse), _ptr(wsb), wsb.numel(), _stream(dev)))
    return (out, lse) if lse is not None else out


def attn_dense_prefill(q, latent, dv: int, idx=None, k: Optional[int] = None, q_offset: int = 0,
                       scale: Optional[float] = None, out=None, lse=None, return_lse: bool = False,
                       workspace: Optional[Workspace] = None):
    """Eq. (3) over dense causal key tiles (§2, short prefill as masked MHA):
    q [B, nq, 16, 576], latent [B, kv_len, 576]; with idx [B, nq, k] the rows
    with t + 1 > k see only their selection (the same result as
    sparse_attn_prefill), without it every causal key (the dense attention
    whose lse normalises eq. (15))."""
    B, nq, H, Dqk = q.shape
    kv_len = latent.shape[1]
    if idx is not None:
        k = idx.shape[-1] if k is None else k
    scale = Dqk ** -0.5 if scale is None else scale
    dev = q.device
    if out is None:
        out = torch.empty((B, nq, H, dv), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, nq, H), dtype=torch.float32, device=dev)
    L = lib()
    wsb = _ws(workspace, dev).get(L.dsa_attn_dense_prefill_workspace(B, nq, kv_len, 1 if idx is not None else 0))
    _check(L.dsa_attn_dense_prefill(B, nq, q_offset, kv_len, H, Dqk, dv, int(k or 0), float(scale), _ptr(q),
                                    _ptr(latent), _ptr(idx), _ptr(out), _ptr(lse), _ptr(wsb), wsb.numel(),
                                    _stream(dev)))
    return (out, lse) if lse is not None else out


PATH_GATHER, PATH_DENSE_MASKED = 0, 1


def prefill_attention_path(B: int, nq: int, q_offset: int, kv_len: int, H: int, Dqk: int, Dv: int, k: int) -> int:
    """The prefill attention path the library picks for a chunk (§2 length
    dispatch): PATH_DENSE_MASKED for short histories, else PATH_GATHER."""
    return int(lib().dsa_prefill_attention_path(B, nq, q_offset, kv_len, H, Dqk, Dv, k))


def attn_prefill(q, latent, idx, dv: int, q_offset: int = 0, scale: Optional[float] = None, out=None, lse=None,
                 return_lse: bool = False, workspace: Optional[Workspace] = None):
    """Eq. (3) for a prefill chunk on the path the length dispatch picks (the
    dense masked path for short histories, the gathering path otherwise);
    arguments as attn_dense_prefill with a required index tensor."""
    B, nq, H, Dqk = q.shape
    kv_len = latent.shape[1]
    k = idx.shape[-1]
    scale = Dqk ** -0.5 if scale is None else scale
    dev = q.device
    if out is None:
        out = torch.empty((B, nq, H, dv), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, nq, H), dtype=torch.float32, device=dev)
    L = lib()
    wsb = _ws(workspace, dev).get(L.dsa_attn_prefill_workspace(B, nq, q_offset, kv_len, H, Dqk, dv, k))
    _check(L.dsa_attn_prefill(B, nq, q_offset, kv_len, H, Dqk, dv, k, float(scale), _ptr(q), _ptr(latent),
                              _ptr(idx), _ptr(out), _ptr(lse), _ptr(wsb), wsb.numel(), _stream(dev)))
    return (out, lse) if lse is not None else out


def mass_coverage(lse_sparse, lse_dense, per_head: bool = False):
    """Teacher mass coverage M_k of eq. (15) per query row from the two lse
    tensors [..., H]: returns (M, min over heads) [...] (and the per-head
    coverage [..., H] with per_head=True)."""
    H = lse_sparse.shape[-1]
    rows = lse_sparse.numel() // H
    dev = lse_sparse.device
    m = torch.empty(lse_sparse.shape[:-1], dtype=torch.float32, device=dev)
    mn = torch.empty_like(m)
    ph = torch.empty_like(lse_sparse) if per_head else None
    _check(lib().dsa_mass_coverage(rows, H, _ptr(lse_sparse), _ptr(lse_dense), _ptr(m), _ptr(ph), _ptr(mn),
                                   _stream(dev)))
    return (m, mn, ph) if per_head else (m, mn)


# --------------------------------------------------------------------------
# Decode
# --------------------------------------------------------------------------

def indexer_topk_decode(qI, w, kI_cache, cu_seqlens, k: int, total_len: int, max_len: int, q_scale=None,
                        k_scale=None, idx_out=None, score_out=None, return_scores: bool = False,
                        workspace: Optional[Workspace] = None):
    """One decode step of eqs. (1)-(2): qI [B, HI, dI], w [B, HI],
    kI_cache [total_len, dI], cu_seqlens int64 [B+1] on the device.
    Returns idx [B, k] of local positions (and scores)."""
    B, HI, dI = qI.shape
    dt = _dtype_code(qI)
    dev = qI.device
    if idx_out is None:
        idx_out = torch.empty((B, k), dtype=torch.int32, device=dev)
    if return_scores and score_out is None:
        score_out = torch.empty((B, k), dtype=torch.float32, device=dev)
    L = lib()
    need = L.dsa_indexer_topk_decode_workspace(B, HI, dI, k, dt, int(total_len), int(max_len))
    wsb = _ws(workspace, dev).get(need)
    _check(L.dsa_indexer_topk_decode(B, HI, dI, k, dt, _ptr(qI), _ptr(q_scale), _ptr(w), _ptr(kI_cache),
                                     _ptr(k_scale), _ptr(cu_seqlens), int(total_len), int(max_len), _ptr(idx_out),
                                     _ptr(score_out), _ptr(wsb), wsb.numel(), _stream(dev)))
    return (idx_out, score_out) if score_out is not None else idx_out


def indexer_topk_decode_noalloc(qI, w, kI_cache, cu_seqlens, k: int, total_len: int, max_len: int, idx_out,
                                score_out=None, status_out=None, q_scale=None, k_scale=None):
    """indexer_topk_decode for callers that cannot allocate device memory:
    the library's built-in scratch (at most 2^22 cached keys per call) takes
    the place of the workspace, and every output buffer is the caller's.
    status_out, if given, is a device uint32 [2] that receives the call's
    device status word. Calls that overlap on the GPU share that scratch and
    race; order them on one stream."""
    B, HI, dI = qI.shape
    _check(lib().dsa_indexer_topk_decode_noalloc(B, HI, dI, k, _dtype_code(qI), _ptr(qI), _ptr(q_scale), _ptr(w),
                                                 _ptr(kI_cache), _ptr(k_scale), _ptr(cu_seqlens), int(total_len),
                                                 int(max_len), _ptr(idx_out), _ptr(score_out), _ptr(status_out),
                                                 _stream(qI.device)))
    return (idx_out, score_out) if score_out is not None else idx_out


def sparse_attn_decode(q, latent_cache, cu_seqlens, idx, dv: int, total_len: int, scale: Optional[float] = None,
                       out=None, lse=None, return_lse: bool = False, workspace: Optional[Workspace] = None):
    """Eq. (3) for a decode step: q [B, H, Dqk], latent_cache [total_len, Dqk],
    idx [B, k] local positions -> out [B, H, dv] (and lse [B, H])."""
    B, H, Dqk = q.shape
    k = idx.shape[-1]
    scale = Dqk ** -0.5 if scale is None else scale
    dev = q.device
    if out is None:
        out = torch.empty((B, H, dv), dtype=torch.bfloat16, device=dev)
    if return_lse and lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=dev)
    L = lib()
    wsb = _ws(workspace, dev).get(L.dsa_sparse_attn_workspace())
    _check(L.dsa_sparse_attn_decode(B, H, Dqk, dv, k, float(scale), _ptr(q), _ptr(latent_cache), _ptr(cu_seqlens),
                                    int(total_len), _ptr(idx), _ptr(out), _ptr(lse), _ptr(wsb), wsb.numel(),
                                    _stream(dev)))
    return (out, lse) if lse is not None else out


def selection_overlap(idx_teacher, idx_student, max_pos: int, return_counts: bool = False):
    """Per-row |T ∩ S| of two [rows, k] int32 selections on the device (the
    numerator of the set recall R_k, eq. (14)); with return_counts also
    |T| per row.  Recall = inter / count."""
    k = idx_teacher.shape[-1]
    rows = idx_teacher.numel() // k
    dev = idx_teacher.device
    inter = torch.empty(idx_teacher.shape[:-1], dtype=torch.int32, device=dev)
    count = torch.empty_like(inter) if return_counts else None
    _check(lib().dsa_selection_overlap(rows, k, int(max_pos), _ptr(idx_teacher), _ptr(idx_student), _ptr(inter),
                                       _ptr(count), _stream(dev)))
    return (inter, count) if return_counts else inter


# --------------------------------------------------------------------------
# Training: sparse-stage indexer KL (eq. (8))
# --------------------------------------------------------------------------

def indexer_kl_sparse(qI, kI, w, idx, teacher, grad_scale: float = 1.0, grads=("dq", "dw", "dk"),
                      grad_logits: bool = False, dk_out=None, workspace: Optional[Workspace] = None):
    """KL_t of eq. (8) on each row's selected set, with the gradients of a
    loss L (dL/dKL_t = grad_scale) with respect to qI, w and kI.

    qI [B, nq, HI, dI] bf16, kI [B, kv_len, dI] bf16, w [B, nq, HI] fp32,
    idx [B, nq, k] int32, teacher [B, nq, k] fp32 (renormalised per row over
    the valid slots).  Returns a dict with "kl" [B, nq] and the requested
    gradients (fp32): "dq", "dw", "dk" [B, kv_len, dI] (added to dk_out when
    given, else to a fresh zero buffer) and "grad_logits" [B, nq, k]."""
    B, nq, HI, dI = qI.shape
    kv_len = kI.shape[1]
    k = idx.shape[-1]
    dev = qI.device
    if qI.dtype != torch.bfloat16 or kI.dtype != torch.bfloat16:
        raise TypeError("the KL path takes bfloat16 indexer operands")
    out = {"kl": torch.empty((B, nq), dtype=torch.float32, device=dev)}
    if "dq" in grads:
        out["dq"] = torch.empty((B, nq, HI, dI), dtype=torch.float32, device=dev)
    if "dw" in grads:
        out["dw"] = torch.empty((B, nq, HI), dtype=torch.float32, device=dev)
    if "dk" in grads:
        out["dk"] = dk_out if dk_out is not None else torch.zeros((B, kv_len, dI), dtype=torch.float32, device=dev)
    if grad_logits:
        out["grad_logits"] = torch.empty((B, nq, k), dtype=torch.float32, device=dev)
    L = lib()
    wsb = _ws(workspace, dev).get(L.dsa_indexer_kl_workspace())
    _check(L.dsa_indexer_kl_sparse(B, nq, kv_len, HI, dI, k, _ptr(qI), _ptr(kI), _ptr(w), _ptr(idx), _ptr(teacher),
                                   float(grad_scale), _ptr(out["kl"]), _ptr(out.get("grad_logits")),
                                   _ptr(out.get("dq")), _ptr(out.get("dw")), _ptr(out.get("dk")), _ptr(wsb),
                                   wsb.numel(), _stream(dev)))
    return out


def attn_teacher_prefill(q, latent, idx, lse, scale: Optional[float] = None, out=None,
                         workspace: Optional[Workspace] = None):
    """Teacher of eq. (8) from the sparse attention: per slot of idx, the
    heads' attention probabilities (recomputed with the forward's lse)
    summed over heads and L1-normalised over the row's selected positions.
    q [B, nq, H, Dqk] bf16, latent [B, kv_len, Dqk] bf16, idx [B, nq, k],
    lse [B, nq, H] fp32 (from sparse_attn_prefill).  Returns [B, nq, k] fp32."""
    B, nq, H, Dqk = q.shape
    kv_len = latent.shape[1]
    k = idx.shape[-1]
    dev = q.device
    if scale is None:
        scale = 1.0 / math.sqrt(Dqk)
    if out is None:
        out = torch.empty((B, nq, k), dtype=torch.float32, device=dev)
    L = lib()
    wsb = _ws(workspace, dev).get(L.dsa_small_workspace())
    _check(L.dsa_attn_teacher_prefill(B, nq, kv_len, H, Dqk, k, float(scale), _ptr(q), _ptr(latent), _ptr(idx),
                                      _ptr(lse), _ptr(out), _ptr(wsb), wsb.numel(), _stream(dev)))
    return out


# --------------------------------------------------------------------------
# Debug / test
# --------------------------------------------------------------------------

def indexer_scores(qI, kI, w, q_offset: int = 0, q_scale=None, k_scale=None, out=None,
                   workspace: Optional[Workspace] = None):
    """Dense causal scores [B, nq, kv_len] fp32 (-inf beyond the diagonal)."""
    B, nq, HI, dI = qI.shape
    kv_len = kI.shape[1]
    dt = _dtype_code(qI)
    dev = qI.device
    if out is None:
        out = torch.empty((B, nq, kv_len), dtype=torch.float32, device=dev)
    L = lib()
    wsb = _ws(workspace, dev).get(L.dsa_small_workspace())
    _check(L.dsa_indexer_scores(B, nq, q_offset, kv_len, HI, dI, dt, _ptr(qI), _ptr(q_scale), _ptr(kI), _ptr(k_scale),
                                _ptr(w), _ptr(out), _ptr(wsb), wsb.numel(), _stream(dev)))
    return out


def topk_rows(scores, k: int, row_len=None, idx_out=None, val_out=None, return_values: bool = False,
              workspace: Optional[Workspace] = None):
    """Top-k of each row of a [rows, ncols] fp32 matrix (row_len: int32 [rows])."""
    rows, ncols = scores.shape
    dev = scores.device
    if idx_out is None:
        idx_out = torch.empty((rows, k), dtype=torch.int32, device=dev)
    if return_values and val_out is None:
        val_out = torch.empty((rows, k), dtype=torch.float32, device=dev)
    L = lib()
    wsb = _ws(workspace, dev).get(L.dsa_small_workspace())
    _check(L.dsa_topk_rows(rows, ncols, scores.stride(0), _ptr(scores), _ptr(row_len), k, _ptr(idx_out),
                           _ptr(val_out), _ptr(wsb), wsb.numel(), _stream(dev)))
    return (idx_out, val_out) if val_out is not None else idx_out


def selftest_bounded_wait(timeout_ns: int, workspace: Workspace):
    L = lib()
    wsb = workspace.get(L.dsa_small_workspace())
    _check(L.dsa_selftest_bounded_wait(int(timeout_ns), _ptr(wsb), wsb.numel(), _stream(wsb.device)))
