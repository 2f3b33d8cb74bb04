"""gpt-oss-style grouped-query attention with sinks on B200 (sm_100a).

Thin ctypes binding over ``libgptoss_attn.so`` (C ABI in
``include/gptoss_attn.h``). This module only marshals arguments: every step
of the attention runs in the library's CUDA kernels. PyTorch supplies device
memory and streams. There is no CPU fallback: if the library or a CUDA
device is missing, calls raise.

Shapes (bf16 unless noted):
    prefill: q [B, S, 64, 64], k/v [B, S, 8, 64], sinks fp32 [64],
             pos int32 [B, S]  ->  out [B, S, 64, 64]
    prefill_chunk: q [B, n, 64, 64], k/v [B, n, 8, 64], pos int32 [B, n],
             kcache/vcache [B, L, 8, 64] holding `start` cached tokens
             -> out [B, n, 64, 64]; the chunk's rotated keys and values are
             written to rows [start, start+n) of the caches
    decode:  q [B, 64, 64] (un-rotated), kcache/vcache [B, L, 8, 64]
             (keys rotated), sinks fp32 [64], lengths int32 [B] -> out [B, 64, 64]
``window <= 0`` is full causal; ``window = W > 0`` the W-key sliding window.
``rope="yarn"`` selects the library's YaRN rotation (factor 32 over a
4096-token original context) in place of plain RoPE; a cache filled with one
rotation must be read with the same one.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["prefill", "prefill_lse", "prefill_backward", "decode", "decode_noalloc",
           "prefill_workspace_bytes",
           "decode_workspace_bytes", "prefill_chunk", "check", "debug_wait_timeout", "init", "rope_table",
           "library_path", "GptossAttnError", "NUM_HEADS", "NUM_KV_HEADS", "HEAD_DIM",
           "MAX_POSITION"]

NUM_HEADS = 64
NUM_KV_HEADS = 8
HEAD_DIM = 64
MAX_POSITION = 131072
ABI_VERSION = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libgptoss_attn.so"
_lib = None


class GptossAttnError(RuntimeError):
    """A non-zero status returned by the C library."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, _status_string(status), status))


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise ImportError("%s is not built; run `python -m attention_gqa_b200.build`" % path)
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gptoss_attn_abi_version.restype = i32
    lib.gptoss_attn_status_string.argtypes = [i32]
    lib.gptoss_attn_status_string.restype = ctypes.c_char_p
    lib.gptoss_attn_init.restype = i32
    lib.gptoss_attn_rope_table.argtypes = [ctypes.POINTER(vp)]
    lib.gptoss_attn_rope_table.restype = i32
    lib.gptoss_attn_prefill_workspace_bytes.argtypes = [i32, i32]
    lib.gptoss_attn_prefill_workspace_bytes.restype = sz
    lib.gptoss_attn_prefill.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, vp, sz, vp]
    lib.gptoss_attn_prefill.restype = i32
    lib.gptoss_attn_prefill_chunk.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, vp, i32, i32, i32,
                                              i32, vp]
    lib.gptoss_attn_prefill_chunk.restype = i32
    lib.gptoss_attn_decode_workspace_bytes.argtypes = [i32, i32, i32]
    lib.gptoss_attn_decode_workspace_bytes.restype = sz
    lib.gptoss_attn_decode.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, vp, sz, vp]
    lib.gptoss_attn_decode.restype = i32
    lib.gptoss_attn_check.argtypes = [vp]
    lib.gptoss_attn_check.restype = i32
    lib.gptoss_attn_debug_wait_timeout.argtypes = [ctypes.c_uint, vp]
    lib.gptoss_attn_debug_wait_timeout.restype = i32
    lib.gptoss_attn_init_yarn.restype = i32
    lib.gptoss_attn_rope_table_yarn.argtypes = [ctypes.POINTER(vp)]
    lib.gptoss_attn_rope_table_yarn.restype = i32
    lib.gptoss_attn_prefill_yarn.argtypes = lib.gptoss_attn_prefill.argtypes
    lib.gptoss_attn_prefill_yarn.restype = i32
    lib.gptoss_attn_prefill_chunk_yarn.argtypes = lib.gptoss_attn_prefill_chunk.argtypes
    lib.gptoss_attn_prefill_chunk_yarn.restype = i32
    lib.gptoss_attn_decode_yarn.argtypes = lib.gptoss_attn_decode.argtypes
    lib.gptoss_attn_decode_yarn.restype = i32
    lib.gptoss_attn_prefill_lse.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, i32, i32, vp, sz, vp]
    lib.gptoss_attn_prefill_lse.restype = i32
    lib.gptoss_attn_prefill_backward_workspace_bytes.argtypes = [i32, i32]
    lib.gptoss_attn_prefill_backward_workspace_bytes.restype = sz
    lib.gptoss_attn_prefill_backward.argtypes = [vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp,
                                                 vp, i32, i32, vp, sz, vp]
    lib.gptoss_attn_prefill_backward.restype = i32
    if lib.gptoss_attn_abi_version() != ABI_VERSION:
        raise ImportError("%s has ABI %d, expected %d" % (path, lib.gptoss_attn_abi_version(),
                                                          ABI_VERSION))
    _lib = lib
    return lib


def _status_string(status: int) -> str:
    try:
        return _load().gptoss_attn_status_string(status).decode()
    except Exception:
        return "unknown"


def _raise(status: int, what: str):
    if status != 0:
        raise GptossAttnError(status, what)


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dev(t: torch.Tensor, dtype, name: str, device) -> torch.Tensor:
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def _target_device(*ts):
    for t in ts:
        if t.device.type == "cuda":
            return t.device
    if not torch.cuda.is_available():
        raise RuntimeError("gptoss attention needs a CUDA device (sm_100a); none is available")
    return torch.device("cuda", torch.cuda.current_device())


ROPES = ("plain", "yarn")


def _rope(rope: str) -> bool:
    if rope not in ROPES:
        raise ValueError("rope must be one of %s, got %r" % (ROPES, rope))
    return rope == "yarn"


def init(rope: str = "plain") -> None:
    """Build the current device's rotary table (allocates; call before graph capture)."""
    if _rope(rope):
        _raise(_load().gptoss_attn_init_yarn(), "gptoss_attn_init_yarn")
    else:
        _raise(_load().gptoss_attn_init(), "gptoss_attn_init")


class _DevicePtr:
    """Exposes a library-owned device buffer to torch through __cuda_array_interface__."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3}


def rope_table(rope: str = "plain") -> torch.Tensor:
    """A copy of the device rotary table, fp32 [131072, 32, 2] of (cos, sin)."""
    p = ctypes.c_void_p()
    lib = _load()
    fn = lib.gptoss_attn_rope_table_yarn if _rope(rope) else lib.gptoss_attn_rope_table
    _raise(fn(ctypes.byref(p)), "gptoss_attn_rope_table")
    view = torch.as_tensor(_DevicePtr(p.value, (MAX_POSITION, HEAD_DIM // 2, 2), "<f4"),
                           device="cuda")
    return view.clone()


def prefill_workspace_bytes(batch: int, seqlen: int) -> int:
    return int(_load().gptoss_attn_prefill_workspace_bytes(batch, seqlen))


def prefill(q, k, v, sinks, pos, window: int = 0, out=None, workspace=None,
            stream=None, rope: str = "plain") -> torch.Tensor:
    """Causal grouped-query attention with sinks over whole sequences.

    Host (CPU) tensors are copied to the current CUDA device first and the
    result is copied back, so the call works end to end from host memory.
    """
    lib = _load()
    host = q.device.type != "cuda"
    device = _target_device(q, k, v)
    if host:
        with torch.cuda.device(device):
            s = stream if stream is not None else torch.cuda.current_stream()
            with torch.cuda.stream(s):
                res = prefill(q.to(device, non_blocking=True), k.to(device, non_blocking=True),
                              v.to(device, non_blocking=True),
                              sinks.to(device, non_blocking=True),
                              pos.to(device, non_blocking=True), window, None, workspace, s,
                              rope)
                if out is None:
                    out = torch.empty(res.shape, dtype=res.dtype, pin_memory=True)
                out.copy_(res, non_blocking=True)
            s.synchronize()
        return out
    q = _dev(q, torch.bfloat16, "q", device)
    k = _dev(k, torch.bfloat16, "k", device)
    v = _dev(v, torch.bfloat16, "v", device)
    sinks = _dev(sinks, torch.float32, "sinks", device)
    pos = _dev(pos, torch.int32, "pos", device)
    if q.dim() != 4 or q.shape[2:] != (NUM_HEADS, HEAD_DIM):
        raise ValueError("q must be [B, S, 64, 64], got %s" % (tuple(q.shape),))
    B, S = q.shape[0], q.shape[1]
    for name, t in (("k", k), ("v", v)):
        if tuple(t.shape) != (B, S, NUM_KV_HEADS, HEAD_DIM):
            raise ValueError("%s must be [B, S, 8, 64], got %s" % (name, tuple(t.shape)))
    if tuple(sinks.shape) != (NUM_HEADS,):
        raise ValueError("sinks must be [64]")
    if tuple(pos.shape) != (B, S):
        raise ValueError("pos must be [B, S]")
    dev_out = out if (out is not None and out.device.type == "cuda") else torch.empty(
        (B, S, NUM_HEADS, HEAD_DIM), dtype=torch.bfloat16, device=device)
    if workspace is None:
        workspace = torch.empty(prefill_workspace_bytes(B, S), dtype=torch.uint8, device=device)
    fn = lib.gptoss_attn_prefill_yarn if _rope(rope) else lib.gptoss_attn_prefill
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), sinks.data_ptr(), pos.data_ptr(),
            int(window), dev_out.data_ptr(), B, S, workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gptoss_attn_prefill")
    return dev_out


def _prefill_shapes(q, k, v, sinks, pos, device):
    q = _dev(q, torch.bfloat16, "q", device)
    k = _dev(k, torch.bfloat16, "k", device)
    v = _dev(v, torch.bfloat16, "v", device)
    sinks = _dev(sinks, torch.float32, "sinks", device)
    pos = _dev(pos, torch.int32, "pos", device)
    if q.dim() != 4 or q.shape[2:] != (NUM_HEADS, HEAD_DIM):
        raise ValueError("q must be [B, S, 64, 64], got %s" % (tuple(q.shape),))
    B, S = q.shape[0], q.shape[1]
    for name, t in (("k", k), ("v", v)):
        if tuple(t.shape) != (B, S, NUM_KV_HEADS, HEAD_DIM):
            raise ValueError("%s must be [B, S, 8, 64], got %s" % (name, tuple(t.shape)))
    if tuple(sinks.shape) != (NUM_HEADS,) or tuple(pos.shape) != (B, S):
        raise ValueError("sinks must be [64] and pos [B, S]")
    return B, S


def prefill_lse(q, k, v, sinks, pos, window: int = 0, out=None, lse=None, workspace=None,
                stream=None):
    """prefill() that also returns the natural-log softmax normaliser of every
    query row (sink included), fp32 [B, S, 64], for prefill_backward(). Device
    tensors only."""
    lib = _load()
    device = _target_device(q, k, v)
    B, S = _prefill_shapes(q, k, v, sinks, pos, device)
    if out is None:
        out = torch.empty((B, S, NUM_HEADS, HEAD_DIM), dtype=torch.bfloat16, device=device)
    _dev(out, torch.bfloat16, "out", device)
    if lse is None:
        lse = torch.empty((B, S, NUM_HEADS), dtype=torch.float32, device=device)
    _dev(lse, torch.float32, "lse", device)
    if tuple(out.shape) != (B, S, NUM_HEADS, HEAD_DIM) or tuple(lse.shape) != (B, S, NUM_HEADS):
        raise ValueError("out must be [B, S, 64, 64] and lse [B, S, 64]")
    if workspace is None:
        workspace = torch.empty(prefill_workspace_bytes(B, S), dtype=torch.uint8, device=device)
    st = lib.gptoss_attn_prefill_lse(q.data_ptr(), k.data_ptr(), v.data_ptr(), sinks.data_ptr(),
                                     pos.data_ptr(), int(window), out.data_ptr(), lse.data_ptr(),
                                     B, S, workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(),
                                     _stream_handle(stream))
    _raise(st, "gptoss_attn_prefill_lse")
    return out, lse


def prefill_backward_workspace_bytes(batch: int, seqlen: int) -> int:
    return int(_load().gptoss_attn_prefill_backward_workspace_bytes(batch, seqlen))


def prefill_backward(q, k, v, sinks, pos, window, out, lse, dout, workspace=None, stream=None):
    """Gradients (dq, dk, dv bf16; dsinks fp32 [64]) of sum(dout * out) for the
    prefill with these inputs; out and lse come from prefill_lse(). Device
    tensors only."""
    lib = _load()
    device = _target_device(q, k, v)
    B, S = _prefill_shapes(q, k, v, sinks, pos, device)
    for name, t, dt, shape in (("out", out, torch.bfloat16, (B, S, NUM_HEADS, HEAD_DIM)),
                               ("lse", lse, torch.float32, (B, S, NUM_HEADS)),
                               ("dout", dout, torch.bfloat16, (B, S, NUM_HEADS, HEAD_DIM))):
        _dev(t, dt, name, device)
        if tuple(t.shape) != shape:
            raise ValueError("%s must be %s, got %s" % (name, shape, tuple(t.shape)))
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    dsinks = torch.empty(NUM_HEADS, dtype=torch.float32, device=device)
    if workspace is None:
        workspace = torch.empty(prefill_backward_workspace_bytes(B, S), dtype=torch.uint8,
                                device=device)
    st = lib.gptoss_attn_prefill_backward(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), sinks.data_ptr(), pos.data_ptr(), int(window),
        out.data_ptr(), lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
        dv.data_ptr(), dsinks.data_ptr(), B, S, workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gptoss_attn_prefill_backward")
    return dq, dk, dv, dsinks


def prefill_chunk(q, k, v, sinks, pos, kcache, vcache, start: int, window: int = 0, out=None,
                  stream=None, rope: str = "plain") -> torch.Tensor:
    """Prefill of the next n = q.shape[1] tokens after `start` cached ones: writes
    their rotated keys and values into rows [start, start+n) of kcache / vcache
    ([B, max_len, 8, 64], device) and returns the chunk's attention output."""
    lib = _load()
    device = _target_device(q, k, v)
    q = _dev(q, torch.bfloat16, "q", device)
    k = _dev(k, torch.bfloat16, "k", device)
    v = _dev(v, torch.bfloat16, "v", device)
    sinks = _dev(sinks, torch.float32, "sinks", device)
    pos = _dev(pos, torch.int32, "pos", device)
    for name, t in (("kcache", kcache), ("vcache", vcache)):
        if t.device != device or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous bf16 tensor on %s" % (name, device))
    if q.dim() != 4 or q.shape[2:] != (NUM_HEADS, HEAD_DIM):
        raise ValueError("q must be [B, n, 64, 64], got %s" % (tuple(q.shape),))
    B, n = q.shape[0], q.shape[1]
    for name, t in (("k", k), ("v", v)):
        if tuple(t.shape) != (B, n, NUM_KV_HEADS, HEAD_DIM):
            raise ValueError("%s must be [B, n, 8, 64], got %s" % (name, tuple(t.shape)))
    if kcache.dim() != 4 or kcache.shape[0] != B or kcache.shape[2:] != (NUM_KV_HEADS, HEAD_DIM):
        raise ValueError("kcache must be [B, max_len, 8, 64]")
    if vcache.shape != kcache.shape:
        raise ValueError("vcache must match kcache")
    if tuple(sinks.shape) != (NUM_HEADS,) or tuple(pos.shape) != (B, n):
        raise ValueError("sinks must be [64] and pos [B, n]")
    dev_out = out if out is not None else torch.empty((B, n, NUM_HEADS, HEAD_DIM),
                                                      dtype=torch.bfloat16, device=device)
    fn = lib.gptoss_attn_prefill_chunk_yarn if _rope(rope) else lib.gptoss_attn_prefill_chunk
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), sinks.data_ptr(), pos.data_ptr(),
            int(window), dev_out.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), B, int(start), n,
            kcache.shape[1], _stream_handle(stream))
    _raise(st, "gptoss_attn_prefill_chunk")
    return dev_out


def decode_workspace_bytes(batch: int, max_len: int, window: int = 0) -> int:
    return int(_load().gptoss_attn_decode_workspace_bytes(batch, max_len, int(window)))


def decode(q, kcache, vcache, sinks, lengths, window: int = 0, out=None, workspace=None,
           stream=None, rope: str = "plain") -> torch.Tensor:
    """One decode step against a rotated key cache; see the module docstring."""
    lib = _load()
    host = q.device.type != "cuda"
    device = _target_device(q, kcache, vcache)
    if host:
        with torch.cuda.device(device):
            s = stream if stream is not None else torch.cuda.current_stream()
            with torch.cuda.stream(s):
                res = decode(q.to(device, non_blocking=True),
                             kcache.to(device, non_blocking=True),
                             vcache.to(device, non_blocking=True),
                             sinks.to(device, non_blocking=True),
                             lengths.to(device, non_blocking=True), window, None, workspace, s,
                             rope)
                if out is None:
                    out = torch.empty(res.shape, dtype=res.dtype, pin_memory=True)
                out.copy_(res, non_blocking=True)
            s.synchronize()
        return out
    q = _dev(q, torch.bfloat16, "q", device)
    kcache = _dev(kcache, torch.bfloat16, "kcache", device)
    vcache = _dev(vcache, torch.bfloat16, "vcache", device)
    sinks = _dev(sinks, torch.float32, "sinks", device)
    lengths = _dev(lengths, torch.int32, "lengths", device)
    if q.dim() != 3 or q.shape[1:] != (NUM_HEADS, HEAD_DIM):
        raise ValueError("q must be [B, 64, 64]")
    B = q.shape[0]
    if kcache.dim() != 4 or kcache.shape[0] != B or kcache.shape[2:] != (NUM_KV_HEADS, HEAD_DIM):
        raise ValueError("kcache must be [B, L, 8, 64]")
    if vcache.shape != kcache.shape:
        raise ValueError("vcache must match kcache")
    L = kcache.shape[1]
    need = decode_workspace_bytes(B, L, window)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    dev_out = out if (out is not None and out.device.type == "cuda") else torch.empty(
        (B, NUM_HEADS, HEAD_DIM), dtype=torch.bfloat16, device=device)
    fn = lib.gptoss_attn_decode_yarn if _rope(rope) else lib.gptoss_attn_decode
    st = fn(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), sinks.data_ptr(),
            lengths.data_ptr(), int(window), dev_out.data_ptr(), B, L, workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gptoss_attn_decode")
    return dev_out


def decode_noalloc(q, kcache, vcache, sinks, lengths, window: int = 0, out=None,
                   stream=None) -> torch.Tensor:
    """decode() for callers that cannot allocate device memory: the split
    partials live in the library's fixed device array (GPTOSS_ATTN_NOALLOC_
    SCRATCH_BYTES) instead of a workspace. Device tensors only; pass `out` to
    allocate nothing here either. Calls whose kernels overlap in time race.

    Every argument's dtype, shape and contiguity is checked before the library
    is touched, since the kernels derive their bounds from q and kcache."""
    for name, t, dt in (("q", q, torch.bfloat16), ("kcache", kcache, torch.bfloat16),
                        ("vcache", vcache, torch.bfloat16), ("sinks", sinks, torch.float32),
                        ("lengths", lengths, torch.int32)):
        if t.dtype != dt:
            raise TypeError("%s must be %s, got %s" % (name, dt, t.dtype))
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)
    if q.dim() != 3 or tuple(q.shape[1:]) != (NUM_HEADS, HEAD_DIM):
        raise ValueError("q must be [B, 64, 64], got %s" % (tuple(q.shape),))
    B = q.shape[0]
    if kcache.dim() != 4 or kcache.shape[0] != B or \
            tuple(kcache.shape[2:]) != (NUM_KV_HEADS, HEAD_DIM):
        raise ValueError("kcache must be [B, L, 8, 64] with B = %d, got %s"
                         % (B, tuple(kcache.shape)))
    if tuple(vcache.shape) != tuple(kcache.shape):
        raise ValueError("vcache must match kcache %s, got %s"
                         % (tuple(kcache.shape), tuple(vcache.shape)))
    if tuple(sinks.shape) != (NUM_HEADS,):
        raise ValueError("sinks must be [64], got %s" % (tuple(sinks.shape),))
    if tuple(lengths.shape) != (B,):
        raise ValueError("lengths must be [B] with B = %d, got %s" % (B, tuple(lengths.shape)))
    if out is not None:
        if out.dtype != torch.bfloat16 or not out.is_contiguous() or \
                tuple(out.shape) != (B, NUM_HEADS, HEAD_DIM):
            raise ValueError("out must be a contiguous bf16 [B, 64, 64] tensor, got %s %s"
                             % (out.dtype, tuple(out.shape)))
    device = q.device
    if device.type != "cuda":
        raise ValueError("decode_noalloc takes device tensors")
    for name, t in (("kcache", kcache), ("vcache", vcache), ("sinks", sinks),
                    ("lengths", lengths)) + ((("out", out),) if out is not None else ()):
        if t.device != device:
            raise ValueError("%s is on %s, expected %s" % (name, t.device, device))
    lib = _load()
    fn = lib.gptoss_attn_decode_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, vp]
    fn.restype = i32
    L = kcache.shape[1]
    if out is None:
        out = torch.empty((B, NUM_HEADS, HEAD_DIM), dtype=torch.bfloat16, device=device)
    st = fn(q.data_ptr(), kcache.data_ptr(), vcache.data_ptr(), sinks.data_ptr(),
            lengths.data_ptr(), int(window), out.data_ptr(), B, L, _stream_handle(stream))
    _raise(st, "gptoss_attn_decode_noalloc")
    return out


def check(stream=None) -> None:
    """Synchronize and raise if a kernel reported a device-side error."""
    _raise(_load().gptoss_attn_check(_stream_handle(stream)), "gptoss_attn_check")


def debug_wait_timeout(timeout_us: int, stream=None) -> None:
    """Diagnostic: run the bounded pipeline wait against a barrier that never
    completes; the next check() raises the device-timeout status."""
    _raise(_load().gptoss_attn_debug_wait_timeout(int(timeout_us), _stream_handle(stream)),
           "gptoss_attn_debug_wait_timeout")
