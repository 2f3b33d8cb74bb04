"""GPU parity of the YaRN rotation path (the _yarn entry points) against the
fp64 oracle's YaRN mode, through the C ABI.

YaRN (techniques map row "YaRN RoPE scaling"; factor 32 over the 4096-token
initial context of the llm-atlas field tables) changes only the rotary table:
blended frequencies and cos/sin scaled by 0.1 ln 32 + 1. The bars are the plain
path's (max-abs 2e-2, mean-abs 2e-3) scaled by the factor the logits grow by,
(0.1 ln 32 + 1)^2 = 1.81: the output error comes from the bf16 rounding of the
rotated q and k, which perturbs each logit in proportion to its size.
"""
import math

import numpy as np
import pytest
import torch

import attention_gqa_b200 as gqa
import oracle
import synth
from tests import _util
from tests._util import bits_to_dev, dev_to_f64

pytestmark = pytest.mark.gpu

NQ, NKV, D = 64, 8, 64
MSCALE = 0.1 * math.log(32.0) + 1.0


def compare(got, ref, what):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), what
    assert err.max() <= _util.MAX_ABS_TOL * MSCALE ** 2, "%s: max abs err %.3e" % (what, err.max())
    assert err.mean() <= _util.MEAN_ABS_TOL * MSCALE ** 2, "%s: mean abs err %.3e" % (
        what, err.mean())


def test_yarn_table_matches_oracle_rotation(cuda_device):
    tab = gqa.rope_table("yarn").cpu().numpy().astype(np.float64)       # [P, 32, 2]
    rng = np.random.default_rng(31)
    ps = np.concatenate([[0, 1, 2, 4095, 4096, 65535, 131071], rng.integers(0, 131072, 57)])
    eye = np.zeros((32, D))
    eye[np.arange(32), np.arange(32)] = 1.0
    for p in ps:
        y = oracle.rope(eye, float(p), rope="yarn")
        cos_ref = y[np.arange(32), np.arange(32)]
        sin_ref = y[np.arange(32), np.arange(32) + 32]
        assert np.max(np.abs(tab[p, :, 0] - cos_ref)) < 1.2e-7 * MSCALE, p
        assert np.max(np.abs(tab[p, :, 1] - sin_ref)) < 1.2e-7 * MSCALE, p
    # the plain table is untouched by building the YaRN one
    plain = gqa.rope_table().cpu().numpy().astype(np.float64)
    assert abs(plain[1000, 0, 0] - math.cos(1000.0)) < 1e-7


def _prefill(x, window, rope="yarn"):
    out = gqa.prefill(bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"]),
                      torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["pos"]).cuda(),
                      window, rope=rope)
    gqa.check()
    return dev_to_f64(out)


def _oracle(x, window):
    return oracle.prefill(synth.bf16_bits_to_f64(x["q"]), synth.bf16_bits_to_f64(x["k"]),
                          synth.bf16_bits_to_f64(x["v"]), x["sinks"], x["pos"], window,
                          rope="yarn")


@pytest.mark.parametrize("B,S,window", [(1, 256, 0), (1, 256, 128), (2, 77, 0), (1, 300, 5),
                                        (3, 129, 128)])
def test_yarn_prefill_small(cuda_device, B, S, window):
    x = synth.make_prefill_inputs(60, window, B, S)
    compare(_prefill(x, window), _oracle(x, window), "yarn B=%d S=%d W=%d" % (B, S, window))


def test_yarn_prefill_large_positions(cuda_device):
    """Positions far beyond the 4096-token original context, where YaRN's
    interpolated pairs matter."""
    x = synth.make_prefill_inputs(61, 0, 1, 300)
    x["pos"] = (x["pos"] + 131072 - 300).astype(np.int32)
    compare(_prefill(x, 0), _oracle(x, 0), "yarn large positions")


@pytest.mark.parametrize("layer,window", [(0, 128), (1, 0)])
def test_yarn_prefill_4096(cuda_device, layer, window):
    x = synth.make_prefill_inputs(2, layer, 1, 4096)
    compare(_prefill(x, window), _oracle(x, window), "yarn S=4096 W=%d" % window)


def test_yarn_prefill_131072_sampled_rows(cuda_device):
    """The 131072-token full-causal layer with the YaRN table, on sampled rows."""
    from synth import device as sdev
    dev = torch.device("cuda")
    B, S, cfg, layer = 1, 131072, 5, 0
    q = sdev.bf16_normal(synth.seed_for(cfg, layer, synth.TENSOR_Q), (B, S, NQ, D), dev)
    k = sdev.bf16_normal(synth.seed_for(cfg, layer, synth.TENSOR_K), (B, S, NKV, D), dev)
    v = sdev.bf16_normal(synth.seed_for(cfg, layer, synth.TENSOR_V), (B, S, NKV, D), dev)
    sinks = sdev.f32_normal(synth.seed_for(cfg, layer, synth.TENSOR_SINKS), (NQ,), dev)
    pos = torch.arange(S, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    out = gqa.prefill(q, k, v, sinks, pos, 0, rope="yarn")
    gqa.check()
    rng = np.random.default_rng(62)
    toks = sorted(set(range(64)) | set(range(S - 64, S)) | set(rng.integers(0, S, 96).tolist()))
    rows = [(0, t) for t in toks]
    it = torch.tensor(toks, device=dev)
    got = dev_to_f64(out[0, it])
    q_rows = dev_to_f64(q[0, it])
    del out, q
    ref = oracle.prefill_rows(q_rows, dev_to_f64(k), dev_to_f64(v), sinks.double().cpu().numpy(),
                              pos.cpu().numpy(), 0, rows, rope="yarn")
    compare(got, ref, "yarn S=131072")


@pytest.mark.parametrize("window", [0, 128])
def test_yarn_decode(cuda_device, window):
    lens = [8192, 8191, 4097, 4096, 129, 1, 0, 6000]
    x = synth.make_decode_inputs(63, window, len(lens), 8192, lengths=lens)
    out = gqa.decode(bits_to_dev(x["q"]), bits_to_dev(x["kcache"]), bits_to_dev(x["vcache"]),
                     torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["len"]).cuda(),
                     window, rope="yarn")
    gqa.check()
    ref = oracle.decode(synth.bf16_bits_to_f64(x["q"]), synth.bf16_bits_to_f64(x["kcache"]),
                        synth.bf16_bits_to_f64(x["vcache"]), x["sinks"], x["len"], window,
                        rope="yarn")
    compare(dev_to_f64(out), ref, "yarn decode W=%d" % window)


def test_yarn_chunks_then_decode(cuda_device):
    """A sequence prefilled in chunks with YaRN matches the whole-sequence
    oracle, and a decode step against the cache it wrote matches too."""
    B, S, L, window = 2, 700, 1024, 128
    x = synth.make_prefill_inputs(64, 0, B, S)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks, pos = torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["pos"]).cuda()
    kc = torch.zeros(B, L, NKV, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs = []
    for a, b in ((0, 300), (300, 301), (301, S - 1)):
        outs.append(gqa.prefill_chunk(q[:, a:b].contiguous(), k[:, a:b].contiguous(),
                                      v[:, a:b].contiguous(), sinks, pos[:, a:b].contiguous(),
                                      kc, vc, a, window, rope="yarn"))
    gqa.check()
    ref = _oracle(x, window)
    compare(dev_to_f64(torch.cat(outs, dim=1)), ref[:, :S - 1], "yarn chunks")
    # decode of the last token against the cache (its key and value appended first)
    gqa.prefill_chunk(q[:, S - 1:].contiguous(), k[:, S - 1:].contiguous(),
                      v[:, S - 1:].contiguous(), sinks, pos[:, S - 1:].contiguous(), kc, vc,
                      S - 1, window, rope="yarn")
    lens = torch.full((B,), S, dtype=torch.int32, device="cuda")
    out = gqa.decode(q[:, S - 1].contiguous(), kc, vc, sinks, lens, window, rope="yarn")
    gqa.check()
    compare(dev_to_f64(out), ref[:, S - 1], "yarn decode after chunks")
