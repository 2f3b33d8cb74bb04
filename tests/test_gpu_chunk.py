"""Chunked prefill against a key/value cache (gptoss_attn_prefill_chunk).

A sequence prefilled in pieces must give the same outputs as one prefill of
the whole sequence (checked against the fp64 oracle), leave in the cache
exactly the rotated keys and the values a one-shot prefill computes, and read
no cache row past its last key (rows there are filled with NaN).
"""
import numpy as np
import pytest
import torch

import attention_gqa_b200 as gqa
import oracle
import synth
from tests._util import bits_to_dev, compare, dev_to_f64

NAN_BF16 = 0x7FC0


def _nan_cache(B, L):
    return torch.full((B, L, 8, 64), NAN_BF16, dtype=torch.int16, device="cuda").view(torch.bfloat16)


@pytest.mark.gpu
@pytest.mark.parametrize("window", [0, 128, 5, 1000])
@pytest.mark.parametrize("cuts", [[0, 300, 700, 1000], [0, 1, 33, 160, 161, 1000]])
def test_chunks_match_whole_sequence(cuda_device, window, cuts):
    B, S, L = 2, cuts[-1], 1100
    x = synth.make_prefill_inputs(1, 3, B, S)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks = torch.from_numpy(x["sinks"]).cuda()
    pos = torch.from_numpy(x["pos"]).cuda()
    kc, vc = _nan_cache(B, L), _nan_cache(B, L)
    outs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        outs.append(gqa.prefill_chunk(q[:, a:b].contiguous(), k[:, a:b].contiguous(),
                                      v[:, a:b].contiguous(), sinks, pos[:, a:b].contiguous(),
                                      kc, vc, a, window))
    gqa.check()
    got = dev_to_f64(torch.cat(outs, dim=1))
    ref = oracle.prefill(synth.bf16_bits_to_f64(x["q"]), synth.bf16_bits_to_f64(x["k"]),
                         synth.bf16_bits_to_f64(x["v"]), x["sinks"], x["pos"], window)
    compare(got, ref, "chunks %s W=%d" % (cuts, window))

    # the cache holds exactly what a one-shot prefill rotates, and the values
    ws = torch.empty(gqa.prefill_workspace_bytes(B, S), dtype=torch.uint8, device="cuda")
    gqa.prefill(q, k, v, sinks, pos, window, workspace=ws)
    gqa.check()
    rot = ws[: B * S * 8 * 64 * 2].view(torch.int16).view(B, S, 8, 64)
    assert torch.equal(kc[:, :S].view(torch.int16), rot)
    assert torch.equal(vc[:, :S].view(torch.int16), v.view(torch.int16))
    assert torch.isnan(kc[:, S:].float()).all() and torch.isnan(vc[:, S:].float()).all()


@pytest.mark.gpu
def test_chunk_then_decode_uses_the_cache(cuda_device):
    """Prefill 500 tokens in two chunks, then decode token 501 from the cache."""
    B, S, L = 3, 501, 640
    x = synth.make_prefill_inputs(1, 4, B, S)
    q, k, v = bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"])
    sinks = torch.from_numpy(x["sinks"]).cuda()
    pos = torch.from_numpy(x["pos"]).cuda()
    kc, vc = _nan_cache(B, L), _nan_cache(B, L)
    for a, b in ((0, 200), (200, S)):  # the last chunk is the single decode token
        out = gqa.prefill_chunk(q[:, a:b].contiguous(), k[:, a:b].contiguous(),
                                v[:, a:b].contiguous(), sinks, pos[:, a:b].contiguous(), kc, vc,
                                a, 128)
    gqa.check()
    # decode the last token against the cache the chunks wrote (rows past S stay NaN)
    dq = q[:, S - 1].contiguous()
    ln = torch.full((B,), S, dtype=torch.int32, device="cuda")
    dec = gqa.decode(dq, kc, vc, sinks, ln, 128)
    gqa.check()
    ref = oracle.prefill(synth.bf16_bits_to_f64(x["q"]), synth.bf16_bits_to_f64(x["k"]),
                         synth.bf16_bits_to_f64(x["v"]), x["sinks"], x["pos"], 128)[:, S - 1]
    compare(dev_to_f64(dec), ref, "decode after chunks")
    compare(dev_to_f64(out[:, -1]), ref, "last chunk row")


@pytest.mark.gpu
def test_chunk_argument_errors(cuda_device):
    lib = gqa._load()
    z = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    p = z.data_ptr()
    # start + n beyond the cache, negative start, empty chunk
    assert lib.gptoss_attn_prefill_chunk(p, p, p, p, p, 0, p, p, p, 1, 60, 8, 64, None) == -2
    assert lib.gptoss_attn_prefill_chunk(p, p, p, p, p, 0, p, p, p, 1, -1, 8, 64, None) == -2
    assert lib.gptoss_attn_prefill_chunk(p, p, p, p, p, 0, p, p, p, 1, 0, 0, 64, None) == -2
    assert lib.gptoss_attn_prefill_chunk(p, p, p, p, p, 0, p, None, p, 1, 0, 8, 64, None) == -1
    assert lib.gptoss_attn_prefill_chunk(p + 8, p, p, p, p, 0, p, p, p, 1, 0, 8, 64, None) == -3
