"""The allocation-free decode entry point.

gptoss_attn_decode_noalloc() serves callers that cannot allocate device
memory while they decode (engines that own all device memory in a pool of
their own, latency-bound loops that cannot pay for an allocation's
synchronization). Its split partials live in a fixed
array in the library's device image instead of a caller workspace. These
tests call it through the C ABI and check it against gptoss_attn_decode()
on the same inputs, twice in a row (the fixed array is reused by every call).
"""
import ctypes

import numpy as np
import pytest
import torch

import attention_gqa_b200 as gqa
import synth
from tests._util import bits_to_dev, compare, dev_to_f64

NQ, NKV, D = 64, 8, 64
SMALL_WORKSPACE = -4


def _noalloc(lib):
    fn = lib.gptoss_attn_decode_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, i32, vp, i32, i32, vp]
    fn.restype = i32
    return fn


def test_rejects_sizes_beyond_the_fixed_scratch():
    """Requests whose partials exceed the fixed array fail before any work."""
    from attention_gqa_b200 import build
    build.build()
    lib = gqa._load()
    fn = _noalloc(lib)
    limit = 8 << 20
    # one split per sequence once batch * 8 fills the GPU; 64 heads * 264 bytes each
    batch = limit // (64 * 264) + 64
    assert lib.gptoss_attn_decode_workspace_bytes(batch, 64, 0) > limit - 256
    assert fn(16, 32, 48, 64, 80, 0, 96, batch, 64, None) == SMALL_WORKSPACE
    assert fn(None, 32, 48, 64, 80, 0, 96, 2, 64, None) == -1


@pytest.mark.gpu
@pytest.mark.parametrize("window", [0, 128])
def test_noalloc_decode_matches_workspace_decode(cuda_device, window):
    lib = gqa._load()
    fn = _noalloc(lib)
    lens = [8192, 8191, 4000, 129, 128, 1, 0, 5000]
    x = synth.make_decode_inputs(47, window, len(lens), 8192, lengths=lens)
    q, kc, vc = bits_to_dev(x["q"]), bits_to_dev(x["kcache"]), bits_to_dev(x["vcache"])
    sinks = torch.from_numpy(x["sinks"]).cuda()
    ln = torch.from_numpy(x["len"]).cuda()
    ref = gqa.decode(q, kc, vc, sinks, ln, window)
    gqa.check()
    ref64 = dev_to_f64(ref)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        out = torch.full((len(lens), NQ, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = fn(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), sinks.data_ptr(), ln.data_ptr(),
                window, out.data_ptr(), len(lens), 8192, stream)
        assert st == 0, st
        torch.cuda.synchronize()
        got = dev_to_f64(out)
        compare(got, ref64, "no-alloc call %d W=%d" % (call, window))
        # same kernels and split plan as the workspace path: identical bits
        assert np.array_equal(got, ref64)
