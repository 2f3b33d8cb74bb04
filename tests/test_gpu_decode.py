"""GPU parity of the split-KV decode path (decode + combine kernels) against the
fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import attention_gqa_b200 as gqa
import oracle
import synth
from tests._util import bits_to_dev, compare, dev_to_f64

pytestmark = pytest.mark.gpu

NQ, NKV, D = 64, 8, 64


def _run(x, window, max_len=None):
    kc, vc = x["kcache"], x["vcache"]
    out = gqa.decode(bits_to_dev(x["q"]), bits_to_dev(kc), bits_to_dev(vc),
                     torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["len"]).cuda(), window)
    gqa.check()
    return dev_to_f64(out)


def _oracle(x, window):
    return oracle.decode(synth.bf16_bits_to_f64(x["q"]), synth.bf16_bits_to_f64(x["kcache"]),
                         synth.bf16_bits_to_f64(x["vcache"]), x["sinks"], x["len"], window)


@pytest.mark.parametrize("layer,window", [(0, 128), (1, 0)])
def test_decode_batch64_len8192(cuda_device, layer, window):
    """B=64 sequences, one query token each, cache length 8192; sliding layers
    read the last 128 entries."""
    x = synth.make_decode_inputs(4, layer, 64, 8192)
    compare(_run(x, window), _oracle(x, window), "decode W=%d" % window)


@pytest.mark.parametrize("window", [0, 1, 7, 128, 5000])
def test_ragged_lengths(cuda_device, window):
    """Per-sequence lengths: empty, single key, tile edges and a full cache."""
    lens = [0, 1, 2, 63, 64, 65, 127, 128, 129, 1000, 3001, 4096]
    x = synth.make_decode_inputs(40, window, len(lens), 4096, lengths=lens)
    got = _run(x, window)
    compare(got, _oracle(x, window), "ragged W=%d" % window)
    assert np.all(got[0] == 0.0)  # len 0: all mass on the sink


def test_sink_minus_inf_and_empty(cuda_device):
    x = synth.make_decode_inputs(41, 0, 3, 300, lengths=[0, 5, 300])
    x["sinks"] = np.full(NQ, -np.inf, dtype=np.float32)
    got = _run(x, 0)
    compare(got, _oracle(x, 0), "sink -inf")
    assert np.all(got[0] == 0.0)


def test_split_count_invariance(cuda_device):
    """The same visible keys in caches of different capacity (hence different
    split counts) give the same result up to fp32 summation order."""
    x = synth.make_decode_inputs(42, 0, 4, 1000, lengths=[1000, 999, 500, 17])
    a = _run(x, 0)
    big = {k: v for k, v in x.items()}
    pad = np.zeros((4, 7000, NKV, D), dtype=np.uint16)
    big["kcache"] = np.concatenate([x["kcache"], pad], axis=1)
    big["vcache"] = np.concatenate([x["vcache"], pad], axis=1)
    assert gqa.decode_workspace_bytes(4, 8000) != gqa.decode_workspace_bytes(4, 1000)
    b = _run(big, 0)
    assert np.max(np.abs(a - b)) < 1e-2
    compare(b, _oracle(x, 0), "padded cache")


def test_decode_matches_last_prefill_row(cuda_device):
    """Decode of token S-1 against the rotated prefix cache equals row S-1 of prefill."""
    S, B = 777, 2
    x = synth.make_prefill_inputs(43, 0, B, S)
    kf = synth.bf16_bits_to_f64(x["k"])
    krot = oracle.rope(kf, x["pos"][:, :, None].astype(np.float64))
    kc = synth.f32_to_bf16_bits(krot.astype(np.float32))
    dec = {"q": np.ascontiguousarray(x["q"][:, S - 1]), "kcache": kc, "vcache": x["v"],
           "sinks": x["sinks"], "len": np.full(B, S, dtype=np.int32)}
    got_dec = _run(dec, 0)
    pre = gqa.prefill(bits_to_dev(x["q"]), bits_to_dev(x["k"]), bits_to_dev(x["v"]),
                      torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["pos"]).cuda(), 0)
    gqa.check()
    got_pre = dev_to_f64(pre[:, S - 1])
    assert np.max(np.abs(got_dec - got_pre)) < 2e-2
    compare(got_dec, _oracle(dec, 0), "decode vs oracle")


def test_bad_length_is_reported(cuda_device):
    x = synth.make_decode_inputs(44, 0, 2, 64, lengths=[10, 65])
    gqa.decode(bits_to_dev(x["q"]), bits_to_dev(x["kcache"]), bits_to_dev(x["vcache"]),
               torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["len"]).cuda(), 0)
    with pytest.raises(gqa.GptossAttnError) as e:
        gqa.check()
    assert e.value.status == -11
    gqa.check()


def test_workspace_canaries(cuda_device):
    x = synth.make_decode_inputs(45, 0, 3, 500, lengths=[500, 250, 3])
    need = gqa.decode_workspace_bytes(3, 500)
    ws = torch.full((need + 8192,), 0x5A, dtype=torch.uint8, device="cuda")
    out_buf = torch.full((3 * NQ * D + 2048,), 2.5, dtype=torch.bfloat16, device="cuda")
    out = out_buf[1024:1024 + 3 * NQ * D].view(3, NQ, D)
    gqa.decode(bits_to_dev(x["q"]), bits_to_dev(x["kcache"]), bits_to_dev(x["vcache"]),
               torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["len"]).cuda(), 0,
               out=out, workspace=ws[4096:4096 + need])
    gqa.check()
    assert torch.all(ws[:4096] == 0x5A) and torch.all(ws[4096 + need:] == 0x5A)
    assert torch.all(out_buf[:1024] == 2.5) and torch.all(out_buf[1024 + 3 * NQ * D:] == 2.5)
    compare(dev_to_f64(out), _oracle(x, 0), "canaries")


@pytest.mark.gpu
@pytest.mark.parametrize("window", [0, 128])
def test_cache_rows_past_length_are_never_used(cuda_device, window):
    """Rows at or past len[b] may hold anything (here NaN): the output must not see them."""
    lens = [8192, 8000, 4001, 129, 77, 1, 0]
    x = synth.make_decode_inputs(4, 7, len(lens), 8192, lengths=lens)
    kb, vb = x["kcache"].copy(), x["vcache"].copy()
    for b, n in enumerate(lens):
        kb[b, n:] = 0x7FC0  # bf16 NaN
        vb[b, n:] = 0x7FC0
    out = gqa.decode(bits_to_dev(x["q"]), bits_to_dev(kb), bits_to_dev(vb),
                     torch.from_numpy(x["sinks"]).cuda(), torch.from_numpy(x["len"]).cuda(), window)
    gqa.check()
    ref = oracle.decode(synth.bf16_bits_to_f64(x["q"]), synth.bf16_bits_to_f64(x["kcache"]),
                        synth.bf16_bits_to_f64(x["vcache"]), x["sinks"], x["len"], window)
    compare(dev_to_f64(out), ref, "decode with NaN past len, W=%d" % window)
