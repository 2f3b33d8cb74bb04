"""Pins of the fp64 oracle against facts fixed outside the oracle itself.

Each test names the passage of the gpt-oss pages (or the piece of mathematics)
that fixes the expected value. None of them retypes the oracle's loops: they
use closed forms, library special cases (torch's fp64 scaled-dot-product
attention), invariants, or the independent brute-force transcription.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NQ, NKV, D = 64, 8, 64


def _rand_inputs(seed, B, S, pos_offset=0):
    q = synth.bf16_bits_to_f64(synth.bf16_normal(seed + 1, (B, S, NQ, D)))
    k = synth.bf16_bits_to_f64(synth.bf16_normal(seed + 2, (B, S, NKV, D)))
    v = synth.bf16_bits_to_f64(synth.bf16_normal(seed + 3, (B, S, NKV, D)))
    sinks = synth.f32_normal(seed + 4, (NQ,)).astype(np.float64)
    pos = np.broadcast_to(np.arange(S, dtype=np.float64) + pos_offset, (B, S)).copy()
    return q, k, v, sinks, pos


def _sdpa(q, k, v, window, sink=None):
    """torch fp64 SDPA with K/V heads repeated as kv = h // 8; no rotation.

    With ``sink`` given, the sink enters as one extra key, visible to every
    query, whose scaled score equals the sink logit and whose value is zero.
    """
    B, S = q.shape[:2]
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)                       # B,H,S,D
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(NQ // NKV, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(NQ // NKV, dim=1)
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    mask = j <= i
    if window > 0:
        mask = mask & (j > i - window)
    mask = mask.expand(B, NQ, S, S)
    if sink is not None:
        ones = torch.ones(B, NQ, S, 1, dtype=torch.float64)
        qt = torch.cat([qt, ones], dim=-1)
        kt = torch.cat([kt, torch.zeros(B, NQ, S, 1, dtype=torch.float64)], dim=-1)
        ks = torch.zeros(B, NQ, 1, D + 1, dtype=torch.float64)
        ks[..., D] = torch.from_numpy(sink)[None, :, None] * math.sqrt(D)
        kt = torch.cat([ks, kt], dim=2)
        vt = torch.cat([torch.zeros(B, NQ, 1, D, dtype=torch.float64), vt], dim=2)
        mask = torch.cat([torch.ones(B, NQ, S, 1, dtype=torch.bool), mask], dim=-1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                         scale=1.0 / math.sqrt(D))
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- constants

def test_golden_constants():
    """The oracle's constants are the ones the pages' config tables print."""
    vals = {}
    with open(os.path.join(GOLDEN, "gptoss_constants.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                name, val = (s.strip() for s in line.split("="))
                vals[name] = int(val)
    assert oracle.NQ == vals["num_attention_heads"]
    assert oracle.NKV == vals["num_key_value_heads"]
    assert oracle.D == vals["head_dim"]
    assert oracle.ROPE_THETA == vals["rope_theta"]
    assert oracle.SCALE == 1.0 / math.sqrt(vals["head_dim"])
    assert vals["num_hidden_layers_20b"] == 2 * vals["sliding_layers_20b"]


# ---------------------------------------------------------------- generator

def test_splitmix64_published_word():
    """First output word of SplitMix64 seeded with 0 (published test value)."""
    assert int(synth.splitmix64(0, 0, 1)[0]) == 0xE220A8397B1DCDAF


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, 1.0 + 2 ** -8 + 2 ** -20, -2.5, 3.0e38],
                 dtype=np.float32)
    bits = synth.f32_to_bf16_bits(x)
    # 1+2^-8 is a tie -> even (1.0); 1+3*2^-8 is a tie -> even (1+2^-6);
    # just above a tie rounds up.
    assert list(bits[:5]) == [0x3F80, 0x3F80, 0x3F82, 0x3F81, 0xC020]
    assert synth.bf16_bits_to_f64(bits[:1])[0] == 1.0


def test_normal_moments():
    x = synth.normal(7, 1 << 20)
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1.0) < 5e-3


# ---------------------------------------------------------------- rotation

def test_rope_identity_at_zero():
    x = np.random.default_rng(0).standard_normal((5, D))
    assert np.array_equal(oracle.rope(x, 0.0), x)


def test_rope_unit_vectors_closed_form():
    """Half-split pairing (k, k+32), frequency theta^(-2k/64), sign of sin.

    Pair 0 turns by exactly p radians; pair 16 by p / sqrt(theta); a unit
    vector in the second half picks up -sin in the first half.
    """
    p = 1234.0
    e0 = np.zeros(D); e0[0] = 1.0
    y = oracle.rope(e0, p)
    assert y[0] == pytest.approx(math.cos(p), abs=1e-12)
    assert y[32] == pytest.approx(math.sin(p), abs=1e-12)
    assert np.count_nonzero(np.abs(y) > 1e-15) == 2
    e16 = np.zeros(D); e16[16] = 1.0
    y = oracle.rope(e16, p)
    a = p / math.sqrt(150000.0)
    assert y[16] == pytest.approx(math.cos(a), abs=1e-12)
    assert y[48] == pytest.approx(math.sin(a), abs=1e-12)
    e40 = np.zeros(D); e40[40] = 1.0          # second half, pair 8
    y = oracle.rope(e40, p)
    a = p * 150000.0 ** (-0.25)
    assert y[8] == pytest.approx(-math.sin(a), abs=1e-12)
    assert y[40] == pytest.approx(math.cos(a), abs=1e-12)


def test_rope_norm_and_composition():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((16, D))
    p = rng.integers(0, 131072, size=16).astype(np.float64)
    y = oracle.rope(x, p)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    a, b = 70000.0, 61071.0
    assert np.allclose(oracle.rope(oracle.rope(x, a), b), oracle.rope(x, a + b), atol=1e-9)


def _yarn_turn_rate(k, p=0.75, **kw):
    """Angle per unit position that YaRN gives pair k (from one small rotation)."""
    e = np.zeros(D); e[k] = 1.0
    y = oracle.rope_yarn(e, p, **kw)
    return math.atan2(y[k + 32], y[k]) / p, math.hypot(y[k], y[k + 32])


def test_yarn_factor_one_is_plain_rope():
    """With scaling factor 1 the interpolated and original frequencies agree and
    the attention factor is 1: YaRN reduces to the plain rotation."""
    rng = np.random.default_rng(21)
    for p in (0.0, 1.0, 4095.0, 131071.0):
        x = rng.standard_normal(D)
        assert np.allclose(oracle.rope_yarn(x, p, factor=1.0), oracle.rope(x, p), atol=1e-12)


def test_yarn_bands_and_attention_factor():
    """NTK-by-parts structure of YaRN with s = 32 over a 4096-token original context:
    pairs whose wavelength fits more than beta_fast = 32 times into the original
    context keep their frequency; pairs fitting less than beta_slow = 1 time are
    interpolated (frequency / 32, the same as the plain rotation at position p / 32);
    every rotated vector is scaled by 0.1 ln 32 + 1."""
    mscale = 0.1 * math.log(32.0) + 1.0
    turns = [4096.0 * 150000.0 ** (-2.0 * k / 64) / (2 * math.pi) for k in range(32)]
    for k in range(32):
        rate, norm = _yarn_turn_rate(k)
        assert norm == pytest.approx(mscale, rel=1e-13)
        plain = 150000.0 ** (-2.0 * k / 64)
        if turns[k] > 32.0:
            assert rate == pytest.approx(plain, rel=1e-12), k
        elif turns[k] < 1.0:
            assert rate == pytest.approx(plain / 32.0, rel=1e-12), k
        else:
            assert plain / 32.0 < rate < plain, k
    assert [k for k in range(32) if 1.0 <= turns[k] <= 32.0] == list(range(9, 18))
    rng = np.random.default_rng(22)
    x = rng.standard_normal(D)
    x[:18] = 0.0
    x[32:50] = 0.0                            # only interpolated pairs 18..31
    p = 77777.0
    assert np.allclose(oracle.rope_yarn(x, p), mscale * oracle.rope(x, p / 32.0), atol=1e-9)
    # the model's mode of the row-rotation entry is this same rotation
    assert np.allclose(oracle.rope(x[None], np.array([p]), rope="yarn")[0], oracle.rope_yarn(x, p),
                       atol=1e-15)


def test_yarn_ramp_is_linear_in_the_pair_index():
    """Between the two correction pairs the blend weight of the interpolated
    frequency rises linearly with the pair index (the transformers yarn ramp),
    not linearly with the number of turns: the weights of pairs 9..17 have zero
    second differences and reach 0 and 1 where the pair index where the
    wavelength fits 32 resp. 1 times into 4096 tokens."""
    w = []
    for k in range(32):
        rate, _ = _yarn_turn_rate(k)
        plain = 150000.0 ** (-2.0 * k / 64)
        w.append((plain - rate) / (plain - plain / 32.0))   # 0: original, 1: interpolated
    w = np.array(w)
    assert np.all(w[:9] == pytest.approx(0.0, abs=1e-12))
    assert np.all(w[18:] == pytest.approx(1.0, abs=1e-12))
    assert np.allclose(np.diff(w[9:18], 2), 0.0, atol=1e-10)
    # the straight line through the ramp hits 0 and 1 at the correction pairs,
    # where 4096 * theta^(-2k/64) / (2 pi) equals 32 and 1
    slope = w[10] - w[9]
    k0 = 9 - w[9] / slope
    k1 = k0 + 1.0 / slope
    assert 4096.0 * 150000.0 ** (-2.0 * k0 / 64) / (2 * math.pi) == pytest.approx(32.0, rel=1e-9)
    assert 4096.0 * 150000.0 ** (-2.0 * k1 / 64) / (2 * math.pi) == pytest.approx(1.0, rel=1e-9)


def test_yarn_attention_scales_logits_by_mscale_squared():
    """With YaRN both q and k carry the attention factor, so at positions 0 the
    output equals plain attention with q scaled by (0.1 ln 32 + 1)^2."""
    B, S = 1, 12
    rng = np.random.default_rng(23)
    q = rng.standard_normal((B, S, NQ, D))
    k = rng.standard_normal((B, S, NKV, D))
    v = rng.standard_normal((B, S, NKV, D))
    sinks = rng.standard_normal(NQ)
    pos = np.zeros((B, S))
    m2 = (0.1 * math.log(32.0) + 1.0) ** 2
    got = oracle.prefill(q, k, v, sinks, pos, 5, rope="yarn")
    assert np.allclose(got, oracle.prefill(q * m2, k, v, sinks, pos, 5), atol=1e-12)
    dec = oracle.decode(q[:, -1], oracle.rope(k, np.zeros((B, S, NKV)), rope="yarn"), v, sinks,
                        [S], 5, rope="yarn")
    pos2 = np.broadcast_to(np.arange(S, dtype=np.float64), (B, S)).copy()
    full = oracle.prefill(q, k, v, sinks, pos2, 5, rope="yarn")
    kr = oracle.rope(k, pos2[:, :, None] * np.ones((1, 1, NKV)), rope="yarn")
    dec = oracle.decode(q[:, -1], kr, v, sinks, [S], 5, rope="yarn")
    assert np.allclose(dec, full[:, -1], atol=1e-12)


def test_relative_position_invariance():
    """Shifting every position by a constant leaves the output unchanged."""
    q, k, v, s, pos = _rand_inputs(100, 1, 40)
    o1 = oracle.prefill(q, k, v, s, pos, 0)
    o2 = oracle.prefill(q, k, v, s, pos + 97531.0, 0)
    assert np.max(np.abs(o1 - o2)) < 1e-10


# ---------------------------------------------------------------- softmax core

@pytest.mark.parametrize("window", [0, 1, 3, 64])
def test_no_sink_no_rotation_equals_sdpa(window):
    """sigma = -inf and pos = 0 reduce to plain grouped-query softmax attention.

    torch's fp64 SDPA on K/V repeated to 64 heads with kv = h // 8 is the
    library special case; this also pins the GQA head mapping.
    """
    q, k, v, _, _ = _rand_inputs(200, 2, 150)
    sinks = np.full(NQ, -np.inf)
    pos = np.zeros((2, 150))
    o = oracle.prefill(q, k, v, sinks, pos, window)
    ref = _sdpa(q, k, v, window)
    assert np.max(np.abs(o - ref)) < 1e-12


@pytest.mark.parametrize("window", [0, 5])
def test_sink_equals_virtual_zero_value_key(window):
    """A sink is one extra always-visible logit sigma_h, unscaled, with no value.

    Written as SDPA over one more key whose scaled score is sigma_h and whose
    value is zero (techniques map, row "Learnable attention sink").
    """
    q, k, v, sinks, _ = _rand_inputs(300, 1, 70)
    sinks = sinks * 3.0
    pos = np.zeros((1, 70))
    o = oracle.prefill(q, k, v, sinks, pos, window)
    ref = _sdpa(q, k, v, window, sink=sinks)
    assert np.max(np.abs(o - ref)) < 1e-12


def test_window_at_least_seqlen_is_full_causal():
    q, k, v, s, pos = _rand_inputs(400, 1, 33)
    full = oracle.prefill(q, k, v, s, pos, 0)
    for w in (33, 34, 1000):
        assert np.array_equal(oracle.prefill(q, k, v, s, pos, w), full)


@pytest.mark.parametrize("window", [0, 1, 4, 128])
def test_zero_query_constant_value_closed_form(window):
    """Q = 0 makes every score 0: out = c * n / (n + e^sigma), n = visible keys.

    Pins the sink in the denominator, the unscaled sink (a scaled sink would
    give e^(sigma/8)) and the window count: n = min(i+1, W) keys, the query
    included (sliding_window = 128 in the config tables).
    """
    B, S = 2, 300
    q = np.zeros((B, S, NQ, D))
    c = np.random.default_rng(5).standard_normal((NKV, D))
    v = np.broadcast_to(c, (B, S, NKV, D)).copy()
    k = synth.bf16_bits_to_f64(synth.bf16_normal(9, (B, S, NKV, D)))
    sinks = synth.f32_normal(10, (NQ,)).astype(np.float64)
    pos = np.broadcast_to(np.arange(S, dtype=np.float64), (B, S))
    o = oracle.prefill(q, k, v, sinks, pos, window)
    i = np.arange(S, dtype=np.float64)
    n = i + 1 if window <= 0 else np.minimum(i + 1, window)
    frac = n[:, None] / (n[:, None] + np.exp(sinks)[None, :])            # S, H
    ref = frac[None, :, :, None] * np.repeat(c, NQ // NKV, axis=0)[None, None, :, :]
    assert np.max(np.abs(o - ref)) < 1e-13


def test_window_one_closed_form():
    """W = 1: each query sees only itself; equal positions cancel the rotation.

    out_i = v_i e^s / (e^s + e^sigma) with s = q_i . k_i / 8 on the un-rotated
    vectors (the rotation is orthogonal and the same for both).
    """
    q, k, v, sinks, pos = _rand_inputs(500, 2, 20, pos_offset=5000)
    o = oracle.prefill(q, k, v, sinks, pos, 1)
    kk = np.repeat(k, NQ // NKV, axis=2)
    vv = np.repeat(v, NQ // NKV, axis=2)
    s = np.einsum("bihd,bihd->bih", q, kk) / 8.0
    p = np.exp(s) / (np.exp(s) + np.exp(sinks)[None, None, :])
    assert np.max(np.abs(o - p[..., None] * vv)) < 1e-13


def test_two_token_closed_form():
    """Query at position 1 against a key at position 0: score = a b cos(1) / 8.

    Only element 0 of q (value a) and of k (value b) is non-zero, so the
    score is a b cos(p_i - p_j) / 8 with pair-0 frequency 1; the self key is
    zero (score 0); sigma = 0; v_0 = e_0, v_1 = e_1.
    """
    a, b = 8.0, 8.0
    q = np.zeros((1, 2, NQ, D)); q[0, 1, :, 0] = a
    k = np.zeros((1, 2, NKV, D)); k[0, 0, :, 0] = b
    v = np.zeros((1, 2, NKV, D)); v[0, 0, :, 0] = 1.0; v[0, 1, :, 1] = 1.0
    sinks = np.zeros(NQ)
    pos = np.array([[0.0, 1.0]])
    o = oracle.prefill(q, k, v, sinks, pos, 0)
    s0 = a * b * math.cos(1.0) / 8.0
    den = math.exp(s0) + 1.0 + 1.0
    assert o[0, 1, 0, 0] == pytest.approx(math.exp(s0) / den, abs=1e-15)
    assert o[0, 1, 0, 1] == pytest.approx(1.0 / den, abs=1e-15)
    assert o[0, 0, 0, 0] == pytest.approx(0.5, abs=1e-15)   # row 0: one zero score + sink 0, v_0 = e_0


def test_sink_limits():
    q, k, v, sinks, pos = _rand_inputs(600, 1, 24)
    o_inf = oracle.prefill(q, k, v, np.full(NQ, -np.inf), pos, 0)
    o_neg = oracle.prefill(q, k, v, np.full(NQ, -800.0), pos, 0)
    assert np.max(np.abs(o_inf - o_neg)) < 1e-15
    o_pos = oracle.prefill(q, k, v, np.full(NQ, 800.0), pos, 0)
    assert np.max(np.abs(o_pos)) < 1e-300


# ---------------------------------------------------------------- brute force

@pytest.mark.parametrize("S,windows", [(1, [0, 1, 2]), (5, [0, 1, 2, 3, 4, 5, 6]),
                                       (16, [0, 1, 2, 7, 15, 16, 17])])
def test_brute_force_small(S, windows):
    """The literal transcription (materialized scores, appended sink column,
    fsum softmax, sink column dropped) agrees with the oracle on tiny inputs
    with large positions."""
    q, k, v, sinks, pos = _rand_inputs(700 + S, 1, S, pos_offset=120000)
    for w in windows:
        o = oracle.prefill(q, k, v, sinks, pos, w)
        ref = np.array(brute.attention(q, k, v, sinks, pos, w))
        assert np.max(np.abs(o - ref)) < 1e-12, w


def test_rows_subset_matches_full():
    q, k, v, sinks, pos = _rand_inputs(800, 2, 50)
    full = oracle.prefill(q, k, v, sinks, pos, 7)
    rows = [(1, 49), (0, 0), (1, 3), (0, 20)]
    q_rows = np.stack([q[b, i] for b, i in rows])
    sub = oracle.prefill_rows(q_rows, k, v, sinks, pos, 7, rows)
    for n, (b, i) in enumerate(rows):
        assert np.array_equal(sub[n], full[b, i])


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("window", [0, 6])
def test_decode_is_last_prefill_row(window):
    """decode(q_last, R(K), V, len) equals row len-1 of prefill on the prefix.

    Ragged lengths per sequence; the cache holds keys rotated at their
    positions; the new query is rotated at position len-1.
    """
    B, S = 3, 30
    q, k, v, sinks, _ = _rand_inputs(900, B, S)
    pos = np.broadcast_to(np.arange(S, dtype=np.float64), (B, S)).copy()
    lens = np.array([30, 17, 1])
    kc = oracle.rope(k, pos[:, :, None])
    qd = np.stack([q[b, lens[b] - 1] for b in range(B)])
    o = oracle.decode(qd, kc, v, sinks, lens, window)
    for b in range(B):
        L = lens[b]
        ref = oracle.prefill(q[b:b + 1, :L], k[b:b + 1, :L], v[b:b + 1, :L], sinks,
                             pos[b:b + 1, :L], window)[0, L - 1]
        assert np.max(np.abs(o[b] - ref)) < 1e-12


def test_decode_empty_cache_is_zero():
    q = np.ones((2, NQ, D)); kc = np.ones((2, 4, NKV, D)); vc = np.ones((2, 4, NKV, D))
    o = oracle.decode(q, kc, vc, np.zeros(NQ), np.array([0, 0]), 0)
    assert np.all(o == 0.0)


def test_torch_evaluation_of_the_input_recipe_matches_numpy():
    """synth.device evaluates the same seeded recipe with torch (used for the
    large bench and full-size test inputs); on the CPU it gives the numpy
    generator's values exactly, including slices drawn on their own."""
    import torch
    from synth import device as sdev
    seed = synth.seed_for(5, 1, synth.TENSOR_V)
    w = sdev.splitmix64(seed, 12345, 1000, "cpu").numpy().view(np.uint64)
    assert np.array_equal(w, synth.splitmix64(seed, 12345, 1000))
    host = synth.bf16_normal(seed, (5, 300, 64))
    got = sdev.bf16_normal(seed, (5, 300, 64), "cpu").view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, host)
    part = sdev.bf16_normal_range(seed, 2 * 4567, 3000, "cpu").view(torch.int16).numpy()
    assert np.array_equal(part.view(np.uint16), host.reshape(-1)[2 * 4567:2 * 4567 + 3000])
    assert np.array_equal(synth.bf16_normal_range(seed, 2 * 4567, 3000),
                          host.reshape(-1)[2 * 4567:2 * 4567 + 3000])
    sinks = synth.seed_for(5, 1, synth.TENSOR_SINKS)
    assert np.array_equal(sdev.f32_normal(sinks, (64,), "cpu").numpy(),
                          synth.f32_normal(sinks, (64,)))
