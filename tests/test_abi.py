"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host before any CUDA work (no GPU needed)."""
import ctypes
import os
import re

import pytest

import attention_gqa_b200 as gqa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gptoss_attn.h")


def _header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(gptoss_attn_\w+)\s*\(", text)))


def _header_codes():
    text = open(HEADER).read()
    return {m.group(1): int(m.group(2))
            for m in re.finditer(r"(GPTOSS_ATTN_(?:OK|ERR_\w+))\s*=\s*(-?\d+)", text)}


@pytest.fixture(scope="module")
def lib():
    from attention_gqa_b200 import build
    build.build()
    return gqa._load()


def test_exports_every_declared_symbol(lib):
    syms = _header_symbols()
    assert len(syms) >= 8
    for s in syms:
        assert hasattr(lib, s), s


def test_abi_version_and_status_strings(lib):
    assert lib.gptoss_attn_abi_version() == 1
    codes = _header_codes()
    assert codes["GPTOSS_ATTN_OK"] == 0
    strings = set()
    for name, code in codes.items():
        s = lib.gptoss_attn_status_string(code).decode()
        assert s and s != "unknown status", name
        strings.add(s)
    assert len(strings) == len(codes)
    assert lib.gptoss_attn_status_string(12345).decode() == "unknown status"


def _prefill(lib, q=16, k=32, v=48, sinks=64, pos=80, window=0, out=96, batch=1, seqlen=8,
             ws=112, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = max(1, lib.gptoss_attn_prefill_workspace_bytes(batch, seqlen))
    return lib.gptoss_attn_prefill(q, k, v, sinks, pos, window, out, batch, seqlen, ws, ws_bytes,
                                   None)


def test_prefill_argument_errors(lib):
    c = _header_codes()
    assert _prefill(lib, q=None) == c["GPTOSS_ATTN_ERR_NULL_PTR"]
    assert _prefill(lib, out=None) == c["GPTOSS_ATTN_ERR_NULL_PTR"]
    assert _prefill(lib, batch=0) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert _prefill(lib, seqlen=0) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert _prefill(lib, seqlen=131073) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert _prefill(lib, k=40) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    assert _prefill(lib, pos=82) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    assert _prefill(lib, ws=None) == c["GPTOSS_ATTN_ERR_NULL_PTR"]
    assert _prefill(lib, ws=120) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    need = lib.gptoss_attn_prefill_workspace_bytes(2, 100)
    assert need == 2 * 100 * 8 * 64 * 2
    assert _prefill(lib, batch=2, seqlen=100, ws_bytes=need - 1) == \
        c["GPTOSS_ATTN_ERR_SMALL_WORKSPACE"]
    assert lib.gptoss_attn_prefill_workspace_bytes(0, 5) == 0


def _decode(lib, q=16, kc=32, vc=48, sinks=64, ln=80, window=0, out=96, batch=2, max_len=100,
            ws=128, ws_bytes=None):
    if ws_bytes is None:
        ws_bytes = lib.gptoss_attn_decode_workspace_bytes(batch, max_len, window)
    return lib.gptoss_attn_decode(q, kc, vc, sinks, ln, window, out, batch, max_len, ws, ws_bytes,
                                  None)


def test_decode_argument_errors(lib):
    c = _header_codes()
    assert _decode(lib, kc=None) == c["GPTOSS_ATTN_ERR_NULL_PTR"]
    assert _decode(lib, ws=None) == c["GPTOSS_ATTN_ERR_NULL_PTR"]
    assert _decode(lib, batch=0, ws_bytes=1 << 20) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert _decode(lib, max_len=0, ws_bytes=1 << 20) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert _decode(lib, out=100) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    assert _decode(lib, ws=136) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    need = lib.gptoss_attn_decode_workspace_bytes(2, 100, 0)
    assert need > 0
    assert _decode(lib, ws_bytes=need - 1) == c["GPTOSS_ATTN_ERR_SMALL_WORKSPACE"]


def test_workspace_query(lib):
    assert lib.gptoss_attn_decode_workspace_bytes(0, 10, 0) == 0
    assert lib.gptoss_attn_decode_workspace_bytes(1, 0, 0) == 0
    full = lib.gptoss_attn_decode_workspace_bytes(64, 8192, 0)
    slid = lib.gptoss_attn_decode_workspace_bytes(64, 8192, 128)
    assert full >= slid > 0
    # per (batch, head, split): 64 fp32 partial outputs + (max, sum)
    assert full % (64 * 64 * (64 * 4 + 8)) == 0
    # full-length layers split the keys over several CTAs (here 3 splits for 512
    # (sequence, kv head) pairs); short visible ranges (<= 256 keys) take one split
    assert full == 64 * 64 * 3 * (64 * 4 + 8)
    assert slid == 64 * 64 * 1 * (64 * 4 + 8)
    assert lib.gptoss_attn_decode_workspace_bytes(2, 256, 0) == 2 * 64 * (64 * 4 + 8)
    assert lib.gptoss_attn_decode_workspace_bytes(2, 257, 0) > 2 * 64 * (64 * 4 + 8)


def test_python_binding_refuses_without_device():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    q = torch.zeros(1, 4, 64, 64, dtype=torch.bfloat16)
    kv = torch.zeros(1, 4, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        gqa.prefill(q, kv, kv, torch.zeros(64), torch.zeros(1, 4, dtype=torch.int32), 0)


def test_debug_wait_timeout_argument_errors(lib):
    c = _header_codes()
    assert lib.gptoss_attn_debug_wait_timeout(0, None) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert lib.gptoss_attn_debug_wait_timeout(2000001, None) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]


def test_prefill_chunk_argument_errors(lib):
    c = _header_codes()
    f = lib.gptoss_attn_prefill_chunk
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] + [ctypes.c_void_p] * 3 + \
        [ctypes.c_int] * 4 + [ctypes.c_void_p]
    ok = dict(q=16, k=32, v=48, s=64, p=80, w=0, o=96, kc=112, vc=128, b=1, st=0, n=8, L=64)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["q"], a["k"], a["v"], a["s"], a["p"], a["w"], a["o"], a["kc"], a["vc"], a["b"],
                 a["st"], a["n"], a["L"], None)
    assert call(kc=None) == c["GPTOSS_ATTN_ERR_NULL_PTR"]
    assert call(n=0) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert call(st=-1) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert call(st=60) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]          # start + n > max_len
    assert call(L=131073, n=8) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert call(b=0) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert call(vc=136) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    assert call(p=82) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]


def test_decode_noalloc_binding_checks_shapes_before_the_library(monkeypatch):
    """Each mis-shaped argument of decode_noalloc() raises before any library
    call: the kernels take their bounds from q and kcache, so a wrong shape
    that reached them would read or write out of bounds."""
    import torch

    def no_library():
        raise AssertionError("the library was called")
    monkeypatch.setattr(gqa, "_load", no_library)
    B, L = 3, 40
    good = dict(q=torch.zeros(B, 64, 64, dtype=torch.bfloat16),
                kcache=torch.zeros(B, L, 8, 64, dtype=torch.bfloat16),
                vcache=torch.zeros(B, L, 8, 64, dtype=torch.bfloat16),
                sinks=torch.zeros(64, dtype=torch.float32),
                lengths=torch.zeros(B, dtype=torch.int32))
    bad = [
        ("q", torch.zeros(B, 64, 32, dtype=torch.bfloat16)),
        ("q", torch.zeros(B, 8, 64, 64, dtype=torch.bfloat16)),
        ("kcache", torch.zeros(B + 1, L, 8, 64, dtype=torch.bfloat16)),
        ("kcache", torch.zeros(B, L, 64, 64, dtype=torch.bfloat16)),
        ("vcache", torch.zeros(B, L + 1, 8, 64, dtype=torch.bfloat16)),
        ("vcache", torch.zeros(B - 1, L, 8, 64, dtype=torch.bfloat16)),
        ("sinks", torch.zeros(8, dtype=torch.float32)),
        ("lengths", torch.zeros(B + 2, dtype=torch.int32)),
        ("kcache", torch.zeros(B, 8, L, 64, dtype=torch.bfloat16).transpose(1, 2)),
    ]
    for name, t in bad:
        args = dict(good, **{name: t})
        with pytest.raises(ValueError):
            gqa.decode_noalloc(args["q"], args["kcache"], args["vcache"], args["sinks"],
                               args["lengths"], 0)
    with pytest.raises(ValueError):
        gqa.decode_noalloc(*good.values(), 0, out=torch.zeros(B, 64, 63, dtype=torch.bfloat16))
    with pytest.raises(TypeError):
        gqa.decode_noalloc(*list(good.values())[:4], torch.zeros(B, dtype=torch.int64), 0)
    # well-formed host tensors pass the shape checks and are refused as not on a device
    with pytest.raises(ValueError, match="device tensors"):
        gqa.decode_noalloc(*good.values(), 0)


def test_yarn_entry_points_argument_errors(lib):
    """The _yarn entry points validate exactly like the plain ones, and the YaRN
    decode refuses caches longer than the table's 131072 positions. Every call
    here has one bad argument, so none reaches a device."""
    c = _header_codes()
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    fp = lib.gptoss_attn_prefill_yarn
    fp.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, vp, sz, vp]
    need = lib.gptoss_attn_prefill_workspace_bytes(1, 8)
    assert fp(None, 32, 48, 64, 80, 0, 96, 1, 8, 112, need, None) == c["GPTOSS_ATTN_ERR_NULL_PTR"]
    assert fp(16, 32, 48, 64, 80, 0, 96, 1, 131073, 112, need, None) == \
        c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert fp(16, 40, 48, 64, 80, 0, 96, 1, 8, 112, need, None) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    assert fp(16, 32, 48, 64, 80, 0, 96, 1, 8, 112, need - 1, None) == \
        c["GPTOSS_ATTN_ERR_SMALL_WORKSPACE"]
    fd = lib.gptoss_attn_decode_yarn
    fd.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, vp, sz, vp]
    big = 131073
    wsb = lib.gptoss_attn_decode_workspace_bytes(1, big, 0)
    assert fd(16, 32, 48, 64, 80, 0, 96, 1, big, 128, wsb, None) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert fd(16, 32, None, 64, 80, 0, 96, 1, 64, 128, 1 << 20, None) == \
        c["GPTOSS_ATTN_ERR_NULL_PTR"]


def test_training_entry_points_argument_errors(lib):
    """gptoss_attn_prefill_lse and gptoss_attn_prefill_backward reject bad
    arguments on the host, and the backward workspace is sized as declared."""
    c = _header_codes()
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    fl = lib.gptoss_attn_prefill_lse
    fl.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, vp, sz, vp]
    need = lib.gptoss_attn_prefill_workspace_bytes(1, 8)
    assert fl(16, 32, 48, 64, 80, 0, 96, None, 1, 8, 112, need, None) == \
        c["GPTOSS_ATTN_ERR_NULL_PTR"]
    assert fl(16, 32, 48, 64, 80, 0, 96, 130, 1, 8, 112, need, None) == \
        c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    wb = lib.gptoss_attn_prefill_backward_workspace_bytes
    wb.argtypes = [i32, i32]
    wb.restype = sz
    assert wb(0, 8) == 0 and wb(1, 0) == 0 and wb(1, 131073) == 0

    def r256(x):
        return (x + 255) // 256 * 256
    B, S = 2, 100
    rows = B * S * 64
    assert wb(B, S) == (r256(rows * 64 * 2) + r256(B * S * 8 * 64 * 2) + 2 * r256((rows + 128) * 4)
                        + 2 * r256(B * S * 8 * 64 * 4))
    fb = lib.gptoss_attn_prefill_backward
    fb.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, i32, i32, vp, sz, vp]
    ok = dict(q=16, k=32, v=48, s=64, p=80, w=0, o=96, lse=112, do=128, dq=144, dk=160,
              dv=176, ds=192, b=B, S=S, ws=208, n=wb(B, S))

    def call(**kw):
        a = dict(ok, **kw)
        return fb(a["q"], a["k"], a["v"], a["s"], a["p"], a["w"], a["o"], a["lse"], a["do"],
                  a["dq"], a["dk"], a["dv"], a["ds"], a["b"], a["S"], a["ws"], a["n"], None)
    for name in ("q", "lse", "do", "dq", "dk", "dv", "ds", "ws"):
        assert call(**{name: None}) == c["GPTOSS_ATTN_ERR_NULL_PTR"], name
    assert call(b=0) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert call(S=0) == c["GPTOSS_ATTN_ERR_BAD_SHAPE"]
    assert call(dk=168) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    assert call(ds=194) == c["GPTOSS_ATTN_ERR_BAD_ALIGN"]
    assert call(n=wb(B, S) - 1) == c["GPTOSS_ATTN_ERR_SMALL_WORKSPACE"]
