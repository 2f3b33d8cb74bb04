"""GPU parity of the backward pass (gptoss_attn_prefill_backward) and of the
forward's row normaliser (gptoss_attn_prefill_lse) against the fp64 oracle.

The gradients are sums of bf16-rounded products (rotated q and k, the
probabilities, dS, dO, V) accumulated in fp32 and rounded to bf16 once, so
their error scales with the size of the gradient tensor itself: each tensor G
must satisfy max|G - G_ref| <= 2e-2 * max|G_ref| and mean|G - G_ref| <=
1e-2 * mean|G_ref| (bf16 keeps 8 significant bits, 2^-8 = 3.9e-3; a gradient
entry adds up to thousands of such terms whose rounding errors are
independent). The sink gradient is an fp32 sum over every query row of
exp(sigma - lse) * (dO . out) with bf16 out: relative 1e-2 of its largest
entry.
"""
import numpy as np
import pytest
import torch

import attention_gqa_b200 as gqa
import oracle
import synth
from oracle import backward as obwd
from tests._util import bits_to_dev, dev_to_f64

pytestmark = pytest.mark.gpu

NQ, NKV, D = 64, 8, 64


def _lse_ref(q, k, sinks, pos, window):
    """ln(exp(sigma_h) + sum over visible j of exp(s_ij)), fp64, [B, S, 64]."""
    B, S = q.shape[0], q.shape[1]
    qr = oracle.rope(q, pos[:, :, None] * np.ones((1, 1, NQ)))
    kr = oracle.rope(k, pos[:, :, None] * np.ones((1, 1, NKV)))
    i = np.arange(S)[:, None]
    j = np.arange(S)[None, :]
    vis = j <= i
    if 0 < window < S:
        vis &= j > i - window
    out = np.empty((B, S, NQ))
    for b in range(B):
        for h in range(NQ):
            s = qr[b, :, h] @ kr[b, :, h // 8].T / 8.0
            s = np.where(vis, s, -np.inf)
            m = np.maximum(s.max(axis=1), sinks[h])
            out[b, :, h] = m + np.log(np.exp(sinks[h] - m) + np.exp(s - m[:, None]).sum(axis=1))
    return out


def _grad_compare(got, ref, what):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), what
    scale_max, scale_mean = np.abs(ref).max(), np.abs(ref).mean()
    assert err.max() <= 2e-2 * scale_max, "%s: max err %.3e vs max|ref| %.3e" % (
        what, err.max(), scale_max)
    assert err.mean() <= 1e-2 * scale_mean, "%s: mean err %.3e vs mean|ref| %.3e" % (
        what, err.mean(), scale_mean)
    return err.max() / scale_max, err.mean() / scale_mean


def _run(cfg, B, S, window, seed_dout):
    x = synth.make_prefill_inputs(cfg, 0, B, S)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks, pos = torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["pos"]).cuda()
    out, lse = gqa.prefill_lse(q, k, v, sinks, pos, window)
    dout_bits = synth.bf16_normal(seed_dout, (B, S, NQ, D))
    dout = bits_to_dev(dout_bits)
    dq, dk, dv, dsinks = gqa.prefill_backward(q, k, v, sinks, pos, window, out, lse, dout)
    gqa.check()
    f = synth.bf16_bits_to_f64
    ref = obwd.prefill_backward(f(x["q"]), f(x["k"]), f(x["v"]), x["sinks"], x["pos"], window,
                                f(dout_bits))
    return x, lse, (dq, dk, dv, dsinks), ref


@pytest.mark.parametrize("B,S,window", [(1, 1, 0), (2, 17, 0), (1, 17, 5), (1, 129, 0),
                                        (2, 129, 128), (1, 300, 7), (1, 383, 128)])
def test_backward_small(cuda_device, B, S, window):
    x, lse, got, ref = _run(200 + S, B, S, window, 0xD0 + S)
    for name, g, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        _grad_compare(dev_to_f64(g), r, "%s B=%d S=%d W=%d" % (name, B, S, window))
    ds = got[3].double().cpu().numpy()
    assert np.max(np.abs(ds - ref[3])) <= 1e-2 * np.max(np.abs(ref[3])) + 1e-6
    f = synth.bf16_bits_to_f64
    lref = _lse_ref(f(x["q"]), f(x["k"]), x["sinks"], x["pos"], window)
    assert np.max(np.abs(lse.double().cpu().numpy() - lref)) < 3e-2


@pytest.mark.parametrize("window", [0, 128])
def test_backward_4096(cuda_device, window):
    """B=1, S=4096 (the two-layer workload's shapes), full causal and W=128."""
    x, lse, got, ref = _run(2, 1, 4096, window, 0xD1 + window)
    for name, g, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        _grad_compare(dev_to_f64(g), r, "%s S=4096 W=%d" % (name, window))
    ds = got[3].double().cpu().numpy()
    assert np.max(np.abs(ds - ref[3])) <= 1e-2 * np.max(np.abs(ref[3])) + 1e-6


def test_lse_matches_the_forward(cuda_device):
    """prefill_lse() writes the same output as prefill() and the row normaliser."""
    x = synth.make_prefill_inputs(210, 0, 2, 200)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks, pos = torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["pos"]).cuda()
    for window in (0, 128, 3):
        out, lse = gqa.prefill_lse(q, k, v, sinks, pos, window)
        plain = gqa.prefill(q, k, v, sinks, pos, window)
        gqa.check()
        assert torch.equal(out, plain)
        f = synth.bf16_bits_to_f64
        lref = _lse_ref(f(x["q"]), f(x["k"]), x["sinks"], x["pos"], window)
        assert np.max(np.abs(lse.double().cpu().numpy() - lref)) < 3e-2, window


def test_backward_ignores_workspace_contents(cuda_device):
    """The workspace needs no initialisation: a NaN-filled one gives the same
    gradients (the per-row arrays' padding, read by the last dK/dV steps of a
    sequence whose length is not a multiple of 8, is cleared by the call)."""
    B, S, window = 1, 77, 0
    x = synth.make_prefill_inputs(230, 0, B, S)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks, pos = torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["pos"]).cuda()
    out, lse = gqa.prefill_lse(q, k, v, sinks, pos, window)
    dout = bits_to_dev(synth.bf16_normal(0xD7, (B, S, NQ, D)))
    clean = gqa.prefill_backward(q, k, v, sinks, pos, window, out, lse, dout)
    nbytes = gqa.prefill_backward_workspace_bytes(B, S)
    ws = torch.full((nbytes // 4,), float("nan"), dtype=torch.float32, device="cuda")
    dirty = gqa.prefill_backward(q, k, v, sinks, pos, window, out, lse, dout,
                                 workspace=ws.view(torch.uint8))
    gqa.check()
    for a, b in zip(clean[:3], dirty[:3]):
        assert torch.isfinite(b.float()).all()
        assert torch.equal(a, b)
    assert torch.isfinite(dirty[3]).all()
