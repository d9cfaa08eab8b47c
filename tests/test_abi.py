"""The C-ABI library: it loads, exports every function include/dsa.h declares,
and its host-side argument checks reject bad calls before touching a GPU."""

import ctypes as C
import os
import re

import pytest

import learned_token_indexer_b200 as dsa
from learned_token_indexer_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from learned_token_indexer_b200.build import build
    build()
    return _lib.load()


def test_header_declares_the_hot_path():
    names = _declared_functions()
    for required in ("dsa_indexer_topk_prefill", "dsa_sparse_attn_prefill", "dsa_indexer_topk_decode",
                     "dsa_sparse_attn_decode", "dsa_topk_rows", "dsa_indexer_scores"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding has no signature for {name}"


def test_no_torch_in_the_boundary():
    text = open(HEADER).read()
    assert "torch" not in text.lower().replace("no torch", "")
    assert "at::" not in text


def test_version_and_status_strings(lib):
    assert b"sm_100a" in lib.dsa_version()
    assert lib.dsa_status_string(5) == b"DSA_ERR_TIMEOUT"
    assert lib.dsa_status_string(99) == b"unknown dsa_status"


def test_timeout_setting_roundtrip(lib):
    old = lib.dsa_get_wait_timeout_ns()
    lib.dsa_set_wait_timeout_ns(12345)
    assert lib.dsa_get_wait_timeout_ns() == 12345
    lib.dsa_set_wait_timeout_ns(old)


def _prefill(lib, **kw):
    a = dict(B=1, nq=16, q_offset=0, kv_len=16, HI=64, dI=128, k=8, dtype=0, q=16, qs=None, kI=16, ks=None, w=16,
             idx=16, sc=None, ws=256, wsb=1 << 30)
    a.update(kw)
    p = lambda v: None if v is None else C.c_void_p(v)
    return lib.dsa_indexer_topk_prefill(a["B"], a["nq"], a["q_offset"], a["kv_len"], a["HI"], a["dI"], a["k"],
                                        a["dtype"], p(a["q"]), p(a["qs"]), p(a["kI"]), p(a["ks"]), p(a["w"]),
                                        p(a["idx"]), p(a["sc"]), p(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(HI=3), 2),                 # unsupported head count
    (dict(HI=128), 2),
    (dict(dI=100), 2),               # not a multiple of 8
    (dict(dI=136), 2),
    (dict(dtype=1, dI=120), 2),      # FP8 needs a multiple of 16
    (dict(dtype=7), 1),
    (dict(k=0), 1),
    (dict(q_offset=4, nq=16, kv_len=16), 1),   # rows past the keys
    (dict(q=None), 1),
    (dict(q=24), 1),                 # misaligned TMA operand
    (dict(dtype=1, qs=None, ks=None), 1),      # FP8 without scales
    (dict(ws=None), 3),
    (dict(ws=512 + 16), 3),          # misaligned workspace
    (dict(wsb=64), 3),               # too small
])
def test_prefill_argument_checks(lib, kw, status):
    assert _prefill(lib, **kw) == status
    assert lib.dsa_last_error()


def test_attention_argument_checks(lib):
    f = lib.dsa_sparse_attn_prefill
    v = C.c_void_p(256)
    assert f(1, 4, 16, 16, 576, 500, 8, 0.1, v, v, v, v, None, v, 256, None) == 2     # Dv
    assert f(1, 4, 16, 16, 72, 64, 8, 0.1, v, v, v, v, None, v, 256, None) == 2      # Dqk % 16
    assert f(1, 4, 16, 16, 576, 512, 0, 0.1, v, v, v, v, None, v, 256, None) == 1    # k
    assert f(1, 4, 16, 16, 576, 512, 8, float("nan"), v, v, v, v, None, v, 256, None) == 1
    assert f(1, 4, 16, 16, 576, 512, 8, 0.1, v, v, v, v, None, v, 8, None) == 3     # workspace


def test_workspace_sizes(lib):
    small = lib.dsa_small_workspace()
    assert small == 256
    pf = lib.dsa_indexer_topk_prefill_workspace(1, 8192, 8192, 64, 128, 2048, 0)
    assert pf > 256 and (pf - 256) % (8 * 8192 * 8) == 0
    assert pf == lib.dsa_indexer_topk_prefill_workspace_full(1, 8192, 8192, 64, 128, 2048, 0)


def test_prefill_workspace_is_bounded_past_16384_keys(lib):
    """Candidate buffers stop growing at 16384 entries per token; only the
    second pass's 64 score rows (and the B * nq overflow list) follow kv_len."""
    ws = lambda nq, kv: lib.dsa_indexer_topk_prefill_workspace(1, nq, kv, 64, 128, 2048, 0)
    full = lambda nq, kv: lib.dsa_indexer_topk_prefill_workspace_full(1, nq, kv, 64, 128, 2048, 0)
    sms = (full(8, 16384) - 256) // (12 * 16384 * 8)
    assert full(8, 16384) == 256 + sms * 12 * 16384 * 8 == ws(8, 16384)
    cand = 256 + sms * 12 * 16384 * 8
    assert ws(8192, 131072) == cand + 256 + 8192 * 4 + 64 * 131072 * 4
    assert ws(8192, 262144) - ws(8192, 131072) == 64 * 131072 * 4
    assert full(8192, 131072) == 256 + sms * 12 * 131072 * 8
    if sms == 148:
        assert ws(8192, 131072) < 0.3e9 < 1.8e9 < full(8192, 131072)
    dec = lib.dsa_indexer_topk_decode_workspace(64, 64, 128, 2048, 0, 1000, 100)
    assert dec >= 256 + 4000


def _decode(lib, **kw):
    a = dict(B=2, HI=64, dI=128, k=8, dtype=0, q=16, qs=None, w=16, kc=16, ks=None, cu=16, total=100, maxlen=60,
             idx=16, sc=None, ws=256, wsb=1 << 30)
    a.update(kw)
    p = lambda v: None if v is None else C.c_void_p(v)
    return lib.dsa_indexer_topk_decode(a["B"], a["HI"], a["dI"], a["k"], a["dtype"], p(a["q"]), p(a["qs"]),
                                       p(a["w"]), p(a["kc"]), p(a["ks"]), p(a["cu"]), a["total"], a["maxlen"],
                                       p(a["idx"]), p(a["sc"]), p(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), 0),                  # an empty batch launches nothing
    (dict(B=-1), 1),
    (dict(k=0), 1),
    (dict(HI=3), 2),
    (dict(w=24), 1),                 # head weights are staged by a 16-byte bulk copy
    (dict(q=8), 1),                  # misaligned TMA operand
    (dict(kc=None), 1),
    (dict(dtype=1, qs=None, ks=None), 1),
    (dict(total=1 << 31), 2),        # cache rows past 2^31
    (dict(wsb=64), 3),               # too small for the step's scores
])
def test_decode_argument_checks(lib, kw, status):
    """Host checks of the decode step run before any launch (no GPU needed)."""
    assert _decode(lib, **kw) == status


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.load()


def test_indexer_kl_argument_checks(lib):
    f = lib.dsa_indexer_kl_sparse
    v = C.c_void_p(256)

    def call(B=1, nq=4, kv_len=16, HI=64, dI=128, k=8, q=v, grad_scale=1.0, ws=v, wsb=256):
        return f(B, nq, kv_len, HI, dI, k, q, v, v, v, v, grad_scale, v, None, None, None, None, ws, wsb, None)

    assert call(HI=65) == 2                      # more heads than the kernel pads to
    assert call(dI=48) == 2
    assert call(k=4097) == 2                     # the row's scores live in shared memory
    assert call(k=0) == 1
    assert call(q=None) == 1
    assert call(q=C.c_void_p(264)) == 1          # misaligned operand
    assert call(grad_scale=float("inf")) == 1
    assert call(wsb=8) == 3
    assert call(nq=0) == 0                       # nothing to do
    assert lib.dsa_indexer_kl_workspace() == 256


def test_attn_teacher_argument_checks(lib):
    f = lib.dsa_attn_teacher_prefill
    v = C.c_void_p(256)

    def call(B=1, nq=4, kv_len=16, H=16, Dqk=576, k=8, scale=0.1, q=v, ws=v, wsb=256):
        return f(B, nq, kv_len, H, Dqk, k, scale, q, v, v, v, v, ws, wsb, None)

    assert call(Dqk=600) == 2                    # past the fixed 576-column row
    assert call(Dqk=72) == 2                     # not a multiple of 16
    assert call(k=4097) == 2
    assert call(k=0) == 1
    assert call(q=None) == 1
    assert call(scale=float("nan")) == 1
    assert call(wsb=8) == 3
    assert call(nq=0) == 0


def test_prefill_attention_length_dispatch(lib):
    """§2: short histories take the masked dense path, long ones gather; only
    the dense kernel's shape (16 heads, 576/512 latent rows) can go dense."""
    path = lib.dsa_prefill_attention_path
    assert path(1, 2048, 0, 2048, 16, 576, 512, 2048) == dsa.PATH_DENSE_MASKED
    assert path(4, 4096, 0, 4096, 16, 576, 512, 2048) == dsa.PATH_DENSE_MASKED
    assert path(1, 8192, 0, 8192, 16, 576, 512, 2048) == dsa.PATH_GATHER
    assert path(1, 6144, 0, 6144, 16, 576, 512, 2048) == dsa.PATH_DENSE_MASKED
    assert path(1, 1024, 5376, 8192, 16, 576, 512, 2048) == dsa.PATH_GATHER    # chunk ends past 6144
    assert path(1, 512, 0, 512, 4, 64, 64, 16) == dsa.PATH_GATHER              # other head / width
    assert path(1, 0, 0, 16, 16, 576, 512, 16) == dsa.PATH_GATHER
    assert lib.dsa_attn_prefill_workspace(1, 2048, 0, 2048, 16, 576, 512, 2048) >= 256 + 2048 * 32 * 8
    assert lib.dsa_attn_prefill_workspace(1, 8192, 0, 8192, 16, 576, 512, 2048) == lib.dsa_sparse_attn_workspace()


def test_dense_attention_host_checks(lib):
    ws = (C.c_uint8 * 512)()
    wsp = C.cast(ws, C.c_void_p)
    fake = C.c_void_p(4096)          # never dereferenced: the checks fail first
    st = lib.dsa_attn_dense_prefill(1, 16, 0, 16, 8, 576, 512, 16, 0.1, fake, fake, None, fake, None, wsp, 512, None)
    assert st == 2                   # DSA_ERR_UNSUPPORTED (8 heads)
    st = lib.dsa_attn_dense_prefill(1, 16, 8, 16, 16, 576, 512, 16, 0.1, fake, fake, None, fake, None, wsp, 512, None)
    assert st == 1                   # q_offset + nq > kv_len
    st = lib.dsa_attn_dense_prefill(1, 16, 0, 16, 16, 576, 512, 16, 0.1, fake, fake, fake, fake, None, wsp, 16, None)
    assert st == 3                   # workspace too small for the selection bits
    st = lib.dsa_mass_coverage(4, 0, fake, fake, None, None, None, None)
    assert st == 1
