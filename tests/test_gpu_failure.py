"""The device-side failure path, exercised without faulting the GPU.

Every pipeline wait in the kernels is bounded. gptoss_attn_debug_wait_timeout()
runs that same wait against a barrier nothing arrives at, so the wait runs
out, sets the timeout bit of the device error word and returns. These tests
check that gptoss_attn_check() reports and clears it, and that prefill and
decode kernels launched while it is set skip their work (their outputs stay
untouched) and work again once it is cleared.
"""
import numpy as np
import pytest
import torch

import attention_gqa_b200 as gqa
import oracle
import synth
from tests._util import bits_to_dev, compare, dev_to_f64

DEVICE_TIMEOUT = -9


@pytest.mark.gpu
def test_wait_timeout_is_reported_then_cleared(cuda_device):
    lib = gqa._load()
    gqa.check()
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.gptoss_attn_debug_wait_timeout(2000, stream) == 0  # 2 ms
    assert lib.gptoss_attn_check(stream) == DEVICE_TIMEOUT
    assert lib.gptoss_attn_check(stream) == 0  # cleared by the first check


@pytest.mark.gpu
def test_kernels_skip_work_while_a_timeout_is_pending(cuda_device):
    lib = gqa._load()
    stream = torch.cuda.current_stream().cuda_stream
    x = synth.make_prefill_inputs(1, 0, 1, 96)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks = torch.from_numpy(x["sinks"]).cuda()
    pos = torch.from_numpy(x["pos"]).cuda()
    d = synth.make_decode_inputs(4, 0, 2, 256)
    dq, kc, vc = bits_to_dev(d["q"]), bits_to_dev(d["kcache"]), bits_to_dev(d["vcache"])
    dsinks, ln = torch.from_numpy(d["sinks"]).cuda(), torch.from_numpy(d["len"]).cuda()
    gqa.check()

    for window in (0, 64):
        assert lib.gptoss_attn_debug_wait_timeout(1000, stream) == 0
        out = torch.full((1, 96, 64, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
        gqa.prefill(q, k, v, sinks, pos, window, out=out)
        dout = torch.full((2, 64, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
        gqa.decode(dq, kc, vc, dsinks, ln, window, out=dout)
        assert lib.gptoss_attn_check(stream) == DEVICE_TIMEOUT
        assert torch.isnan(out.float()).all() and torch.isnan(dout.float()).all()

        # cleared: the same calls now run and match the oracle
        gqa.prefill(q, k, v, sinks, pos, window, out=out)
        gqa.decode(dq, kc, vc, dsinks, ln, window, out=dout)
        gqa.check()
        qf, kf, vf = (synth.bf16_bits_to_f64(x[n]) for n in ("q", "k", "v"))
        compare(dev_to_f64(out), oracle.prefill(qf, kf, vf, x["sinks"], x["pos"], window),
                "prefill after clear W=%d" % window)
        ref = oracle.decode(synth.bf16_bits_to_f64(d["q"]), synth.bf16_bits_to_f64(d["kcache"]),
                            synth.bf16_bits_to_f64(d["vcache"]), d["sinks"], d["len"], window)
        compare(dev_to_f64(dout), ref, "decode after clear W=%d" % window)


@pytest.mark.gpu
def test_backward_skips_work_while_a_timeout_is_pending(cuda_device):
    """The dQ and dK/dV kernels check the error word at start-up like the
    forward kernels: launched while a timeout is pending they leave the
    gradients untouched; after the clear the same call gives the gradients."""
    lib = gqa._load()
    stream = torch.cuda.current_stream().cuda_stream
    x = synth.make_prefill_inputs(3, 1, 1, 80)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks, pos = torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["pos"]).cuda()
    out, lse = gqa.prefill_lse(q, k, v, sinks, pos, 0)
    dout = bits_to_dev(synth.bf16_normal(0xD9, (1, 80, 64, 64)))
    ref = gqa.prefill_backward(q, k, v, sinks, pos, 0, out, lse, dout)
    gqa.check()
    ws = torch.empty(gqa.prefill_backward_workspace_bytes(1, 80), dtype=torch.uint8, device="cuda")

    def nan_like(t):
        return torch.full(t.shape, float("nan"), dtype=t.dtype, device="cuda")
    grads = [nan_like(t) for t in ref[:3]] + [torch.zeros(64, device="cuda")]

    def call():
        return lib.gptoss_attn_prefill_backward(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), sinks.data_ptr(), pos.data_ptr(), 0,
            out.data_ptr(), lse.data_ptr(), dout.data_ptr(), grads[0].data_ptr(),
            grads[1].data_ptr(), grads[2].data_ptr(), grads[3].data_ptr(), 1, 80, ws.data_ptr(),
            ws.numel(), stream)
    assert lib.gptoss_attn_debug_wait_timeout(1000, stream) == 0
    assert call() == 0
    assert lib.gptoss_attn_check(stream) == DEVICE_TIMEOUT
    assert all(torch.isnan(g.float()).all() for g in grads[:3])
    assert call() == 0
    gqa.check()
    for g, r in zip(grads[:3], ref[:3]):
        assert torch.equal(g, r)


@pytest.mark.gpu
def test_timeout_stays_on_its_stream(cuda_device):
    """Error words are per stream: a timeout pending on one stream does not
    make kernels on another stream skip their work, and only a check of its
    own stream reports it."""
    lib = gqa._load()
    x = synth.make_prefill_inputs(1, 1, 1, 70)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks, pos = torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["pos"]).cuda()
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    gqa.check(side)
    gqa.check(main)
    assert lib.gptoss_attn_debug_wait_timeout(1000, side.cuda_stream) == 0
    torch.cuda.synchronize()
    out = torch.full((1, 70, 64, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
    gqa.prefill(q, k, v, sinks, pos, 0, out=out, stream=main)
    assert lib.gptoss_attn_check(main.cuda_stream) == 0
    qf, kf, vf = (synth.bf16_bits_to_f64(x[n]) for n in ("q", "k", "v"))
    compare(dev_to_f64(out), oracle.prefill(qf, kf, vf, x["sinks"], x["pos"], 0),
            "prefill on another stream")
    assert lib.gptoss_attn_check(side.cuda_stream) == DEVICE_TIMEOUT
    assert lib.gptoss_attn_check(side.cuda_stream) == 0
