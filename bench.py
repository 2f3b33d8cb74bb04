"""Throughput of the gpt-oss attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload default|s4096|tiny256|batch16k|layers36|chunk16k]

One step is one pass of the whole path over one batch of synthetic inputs. The
default workload is the largest single-GPU configuration:
  * prefill, B=1, S=131072, 64 query / 8 key-value heads, head_dim 64: one
    full-causal layer and one 128-token sliding-window layer, each with its
    own seeded q/k/v/sinks (key rotation, then the attention kernel: Q
    rotation, QK^T, sink-seeded online softmax, PV, epilogue);
  * decode, B=64 sequences against a bf16 cache of 8192 tokens: one
    full-causal layer and one sliding layer (its last 128 entries)
    (split-KV partials + log-sum-exp combine).
``--workload s4096`` runs the same step with a B=1, S=4096 prefill (a W=128
layer, then a full-causal layer). ``value`` is the prefill attention
throughput in TFLOP/s counting unmasked FLOPs only (4 * 64 * 64 per visible
(query, key) pair per head); the decode half of the metric (HBM GB/s over the
algorithmic bytes) is reported in the ``decode`` object. L2 is flushed (256 MB
write) before every step, outside the timed events. Per-kernel times come from
CUDA events on the launching stream. With N > 1 (torchrun), every rank runs
the same per-GPU workload (weak scaling, no collective on the data path);
times are the max over ranks.

Inputs follow the seeded recipe of ``synth`` (SplitMix64 -> Box-Muller ->
fp32 -> bf16), evaluated on the device by ``synth.device``.

``--impl reference`` times the fp64 CPU oracle on the host cores, rank 0 only:
each step is one bounded sample of the same workload (evenly spaced query rows
of both prefill layers, a few decode sequences of both decode layers).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "attention TFLOP/s (unmasked) & % bf16 peak; decode HBM GB/s & % of peak"
NQ, NKV, D = 64, 8, 64

# A step workload: a prefill of B x S tokens through `pre_layers` [(layer, window)]
# with the seeds of configuration `pre_cfg`, then decode of DB sequences against
# DL cached tokens through `dec_layers` with the seeds of configuration `dec_cfg`.
STEP_WORKLOADS = {
    "default": dict(
        pre_cfg=5, B=1, S=131072, pre_layers=((0, 0), (1, 128)),
        dec_cfg=4, DB=64, DL=8192, dec_layers=((0, 0), (1, 128)), peak="sustained",
        desc="prefill B=1 S=131072 64q/8kv d64 (one full-causal layer + one W=128 layer) + "
             "decode B=64 L=8192 (one full layer + one W=128 layer)"),
    "s4096": dict(
        pre_cfg=2, B=1, S=4096, pre_layers=((0, 128), (1, 0)),
        dec_cfg=4, DB=64, DL=8192, dec_layers=((0, 0), (1, 128)), peak="burst",
        desc="prefill B=1 S=4096 64q/8kv d64 (W=128 layer + full-causal layer) + "
             "decode B=64 L=8192 (full layer + W=128 layer)"),
}


def visible_pairs(S: int, window: int) -> int:
    if window <= 0 or window >= S:
        return S * (S + 1) // 2
    return window * S - window * (window - 1) // 2


def prefill_flops(B: int, S: int, window: int) -> float:
    return 4.0 * D * NQ * B * visible_pairs(S, window)


def prefill_bytes(B: int, S: int) -> float:
    return float(B * S * (2 * NQ * D * 2 + 2 * NKV * D * 2))  # q, out, k, v (bf16)


def decode_bytes(B: int, L: int, window: int) -> float:
    n = L if window <= 0 else min(window, L)
    return float(B * n * NKV * D * 2 * 2 + 2 * B * NQ * D * 2)  # visible K and V, q, out


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def source_digest() -> str:
    """Digest of the full-causal prefill kernel's sources (kernel file and the
    header it shares with the narrow-band kernel)."""
    h = hashlib.sha256()
    for name in ("prefill_sm100.cu", "prefill_common.cuh"):
        with open(os.path.join(ROOT, "attention_gqa_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(path: str):
    """DRAM bytes per launch of the full-causal prefill kernel from a committed
    ncu summary, if it was taken on the current kernel source."""
    try:
        vals = {}
        with open(path) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    vals[k.strip()] = v.strip()
        if vals.get("kernel_source_sha256_16") != source_digest():
            return None
        return float(vals["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """Samples SM clocks and clock-event reasons through NVML while timing runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, index: int, period_s: float = 0.02):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


EXP_PER_CLK_PER_SM = 16   # ex2.approx.ftz.f32 results per clock per SM on B200 (probe)
NUM_SMS = 148


def exp_roofline(flops: float, ms: float, clocks: dict) -> dict:
    """Exponential-unit roofline of a full-causal prefill launch: FLOPs / 256 exps."""
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965
    achieved = flops / 256.0 / (ms * 1e-3) / 1e9
    peak = EXP_PER_CLK_PER_SM * NUM_SMS * mhz * 1e6 / 1e9
    return {"bound": "alu (exponential unit)", "achieved": achieved, "peak": peak,
            "unit": "Gexp/s", "frac": achieved / peak,
            "peak_basis": "16 ex2 results/clk/SM (measured) x 148 SMs x %.0f MHz median SM clock"
                          % mhz}


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def step_config(wl: dict) -> dict:
    """The workload description both arms print (identical, so the lines compare)."""
    return {"workload": wl["desc"], "prefill": {"batch": wl["B"], "seq_len": wl["S"],
                                                "windows": [w for _, w in wl["pre_layers"]]},
            "decode": {"batch": wl["DB"], "cache_len": wl["DL"],
                       "windows": [w for _, w in wl["dec_layers"]]},
            "l2": "flushed before every step (256 MB write)"}


# ------------------------------------------------------------------ CPU oracle leg

def _seed(cfg, layer, tid):
    import synth
    return synth.seed_for(cfg, layer, tid)


class OracleSampler:
    """Bounded samples of a step workload for the fp64 CPU oracle.

    Holds, on the host, the keys and values of every prefill layer and of a few
    decode sequences per decode layer (same seeded recipe as the GPU arm). One
    sample is: `rows` evenly spaced query rows (all 64 heads) of each prefill
    layer, shifted by the sample index, and `seqs` decode sequences of each
    decode layer."""

    def __init__(self, wl: dict, tensors=None, n_seqs: int = 2):
        import torch

        import synth
        from synth import device as sdev
        self.wl = wl
        B, S = wl["B"], wl["S"]
        self.pre = []
        for i, (layer, window) in enumerate(wl["pre_layers"]):
            if tensors is not None:
                t = tensors["pre"][i]
                k, v, sinks = (t["k"].double().cpu().numpy(), t["v"].double().cpu().numpy(),
                               t["sinks"].double().cpu().numpy())
            else:
                k = sdev.bf16_normal(_seed(wl["pre_cfg"], layer, synth.TENSOR_K),
                                     (B, S, NKV, D), "cpu").double().numpy()
                v = sdev.bf16_normal(_seed(wl["pre_cfg"], layer, synth.TENSOR_V),
                                     (B, S, NKV, D), "cpu").double().numpy()
                sinks = sdev.f32_normal(_seed(wl["pre_cfg"], layer, synth.TENSOR_SINKS), (NQ,),
                                        "cpu").double().numpy()
            pos = np.broadcast_to(np.arange(S, dtype=np.int32), (B, S)).copy()
            self.pre.append(dict(layer=layer, window=window, k=k, v=v, sinks=sinks, pos=pos))
        DB, DL = wl["DB"], wl["DL"]
        self.n_seqs = min(n_seqs, DB)
        self.dec = []
        per_seq = DL * NKV * D
        for layer, window in wl["dec_layers"]:
            qseed = _seed(wl["dec_cfg"], layer, synth.TENSOR_Q)
            kseed = _seed(wl["dec_cfg"], layer, synth.TENSOR_K)
            vseed = _seed(wl["dec_cfg"], layer, synth.TENSOR_V)
            def rows(seed, n):
                return torch.stack([sdev.bf16_normal_range(seed, i * n, n, "cpu")
                                    for i in range(self.n_seqs)]).double().numpy()
            q, kc, vc = rows(qseed, NQ * D), rows(kseed, per_seq), rows(vseed, per_seq)
            sinks = sdev.f32_normal(_seed(wl["dec_cfg"], layer, synth.TENSOR_SINKS), (NQ,),
                                    "cpu").double().numpy()
            self.dec.append(dict(
                layer=layer, window=window,
                q=q.reshape(self.n_seqs, NQ, D), kc=kc.reshape(self.n_seqs, DL, NKV, D),
                vc=vc.reshape(self.n_seqs, DL, NKV, D), sinks=sinks))
        self.q_seeds = [_seed(wl["pre_cfg"], layer, synth.TENSOR_Q)
                        for layer, _ in wl["pre_layers"]]

    def sample(self, index: int, rows: int, seqs: int):
        """Runs one sample; returns dict(prefill_flops, prefill_s, decode_bytes, decode_s)."""
        import torch

        import oracle
        from synth import device as sdev
        oracle._load()
        B, S = self.wl["B"], self.wl["S"]
        pf = ps = 0.0
        for p, qseed in zip(self.pre, self.q_seeds):
            stride = S / rows
            toks = ((np.arange(rows) + (index * 0.618034) % 1.0) * stride).astype(np.int64)
            toks = np.clip(toks, 0, S - 1)
            rws = [(int(i % B), int(t)) for i, t in enumerate(toks)]
            q = torch.stack([sdev.bf16_normal_range(qseed, (b * S + t) * NQ * D, NQ * D, "cpu")
                             for b, t in rws]).double().numpy().reshape(rows, NQ, D)
            t0 = time.perf_counter()
            oracle.prefill_rows(q, p["k"], p["v"], p["sinks"], p["pos"], p["window"], rws)
            ps += time.perf_counter() - t0
            pf += sum(4.0 * D * NQ * (min(t + 1, p["window"]) if 0 < p["window"] < S else t + 1)
                      for t in toks)
        db = ds = 0.0
        DL = self.wl["DL"]
        for d in self.dec:
            sel = [(index * seqs + j) % self.n_seqs for j in range(seqs)]
            lens = np.full(seqs, DL, dtype=np.int64)
            t0 = time.perf_counter()
            oracle.decode(d["q"][sel], d["kc"][sel], d["vc"][sel], d["sinks"], lens, d["window"])
            ds += time.perf_counter() - t0
            db += decode_bytes(seqs, DL, d["window"])
        return dict(prefill_flops=pf, prefill_s=ps, decode_bytes=db, decode_s=ds)

    def calibrate(self, target_s: float):
        """Rows per prefill layer and sequences per decode layer for a sample of
        about target_s seconds."""
        rows, seqs = 8, 1
        while True:
            r = self.sample(0, rows, seqs)
            t = r["prefill_s"] + r["decode_s"]
            if t >= target_s / 4 or rows >= 4096:
                break
            rows *= 4
        rows = max(8, min(4096, int(rows * target_s / max(t, 1e-3))))
        return rows, seqs


def run_reference(args, rank: int, wl: dict):
    """The reference arm: the fp64 oracle on the host cores, one bounded sample
    of the workload per step (rank 0 only; other ranks exit without work)."""
    if rank != 0:
        return 0
    sampler = OracleSampler(wl)
    rows, seqs = sampler.calibrate(target_s=2.0)
    for w in range(args.warmup):
        sampler.sample(1000 + w, rows, seqs)
    res = []
    t_wall = time.perf_counter()
    for s in range(args.steps):
        res.append(sampler.sample(s, rows, seqs))
    t_wall = time.perf_counter() - t_wall
    pf = sum(r["prefill_flops"] for r in res)
    ps = sum(r["prefill_s"] for r in res)
    db = sum(r["decode_bytes"] for r in res)
    dsec = sum(r["decode_s"] for r in res)
    value = pf / ps / 1e12
    cores = host_cores()
    sample = ("per step: %d evenly spaced query rows (all 64 heads) of each of the %d prefill "
              "layers and %d sequence(s) of each of the %d decode layers; %.3g unmasked FLOPs and "
              "%.3g decode bytes per step on average" % (
                  rows, len(wl["pre_layers"]), seqs, len(wl["dec_layers"]), pf / args.steps,
                  db / args.steps))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_wall * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic: seeded recipe (synth), same "
        "as the GPU arm", "config": step_config(wl),
        "sample": sample,
        "extrapolated": {"full_step_s": sum(prefill_flops(wl["B"], wl["S"], w)
                                            for _, w in wl["pre_layers"]) * ps / pf +
                         sum(decode_bytes(wl["DB"], wl["DL"], w)
                             for _, w in wl["dec_layers"]) * dsec / db,
                         "how": "one whole step at the sampled rates (prefill by unmasked FLOPs, "
                                "decode by bytes); an extrapolation, not a measurement"},
        "decode": {"value": db / dsec / 1e9, "unit": "GB/s"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU leg

def _prefill_layer(cfg, layer, window, B, S, dev, gqa):
    import torch

    import synth
    from synth import device as sdev
    return dict(
        q=sdev.bf16_normal(_seed(cfg, layer, synth.TENSOR_Q), (B, S, NQ, D), dev),
        k=sdev.bf16_normal(_seed(cfg, layer, synth.TENSOR_K), (B, S, NKV, D), dev),
        v=sdev.bf16_normal(_seed(cfg, layer, synth.TENSOR_V), (B, S, NKV, D), dev),
        sinks=sdev.f32_normal(_seed(cfg, layer, synth.TENSOR_SINKS), (NQ,), dev),
        pos=torch.arange(S, dtype=torch.int32, device=dev).repeat(B, 1).contiguous(),
        window=window, out=torch.empty(B, S, NQ, D, dtype=torch.bfloat16, device=dev),
        ws=torch.empty(gqa.prefill_workspace_bytes(B, S), dtype=torch.uint8, device=dev))


def _decode_layer(cfg, layer, window, B, L, dev, gqa):
    import torch

    import synth
    from synth import device as sdev
    return dict(
        q=sdev.bf16_normal(_seed(cfg, layer, synth.TENSOR_Q), (B, NQ, D), dev),
        kc=sdev.bf16_normal(_seed(cfg, layer, synth.TENSOR_K), (B, L, NKV, D), dev),
        vc=sdev.bf16_normal(_seed(cfg, layer, synth.TENSOR_V), (B, L, NKV, D), dev),
        sinks=sdev.f32_normal(_seed(cfg, layer, synth.TENSOR_SINKS), (NQ,), dev),
        len=torch.full((B,), L, dtype=torch.int32, device=dev), window=window,
        ws=torch.empty(gqa.decode_workspace_bytes(B, L, window), dtype=torch.uint8, device=dev),
        out=torch.empty(B, NQ, D, dtype=torch.bfloat16, device=dev))


def run_ours(args, rank: int, world: int, wl: dict):
    import torch
    import torch.distributed as dist

    import attention_gqa_b200 as gqa
    from attention_gqa_b200 import shard

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    shard.init_from_env("nccl", dev)
    if rank == 0:
        from attention_gqa_b200 import build
        build.build()
    if world > 1:
        dist.barrier()
    gqa.init()
    stream = torch.cuda.current_stream()
    B, S, DB, DL = wl["B"], wl["S"], wl["DB"], wl["DL"]
    pre_layers, dec_layers = wl["pre_layers"], wl["dec_layers"]

    # inputs resident in HBM
    pre = [_prefill_layer(wl["pre_cfg"], layer, w, B, S, dev, gqa) for layer, w in pre_layers]
    dec = [_decode_layer(wl["dec_cfg"], layer, w, DB, DL, dev, gqa) for layer, w in dec_layers]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step(ev=None):
        i = 0
        if ev is not None:
            ev[i].record(stream)
        for p in pre:
            gqa.prefill(p["q"], p["k"], p["v"], p["sinks"], p["pos"], p["window"], out=p["out"],
                        workspace=p["ws"])
            i += 1
            if ev is not None:
                ev[i].record(stream)
        for d in dec:
            gqa.decode(d["q"], d["kc"], d["vc"], d["sinks"], d["len"], d["window"], out=d["out"],
                       workspace=d["ws"])
            i += 1
            if ev is not None:
                ev[i].record(stream)

    n_marks = 1 + len(pre_layers) + len(dec_layers)
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    gqa.check()

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_marks)]
              for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_wall = time.perf_counter()
        for s in range(args.steps):
            flush.fill_(s & 0xFF)
            step(events[s])
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    if world > 1:
        dist.barrier()
    gqa.check()

    seg = np.array([[events[s][i].elapsed_time(events[s][i + 1]) for i in range(n_marks - 1)]
                    for s in range(args.steps)])  # ms, [steps, kernels]
    seg_total = seg.sum(axis=0)                                       # ms per segment over K steps
    seg_total = np.array(shard.max_over_ranks(seg_total, dev))  # the slowest rank sets the time
    npre = len(pre_layers)
    pre_ms = float(seg_total[:npre].sum()) / args.steps
    dec_ms = float(seg_total[npre:].sum()) / args.steps
    step_ms = pre_ms + dec_ms
    pre_flops = sum(prefill_flops(B, S, w) for _, w in pre_layers)
    dec_bytes = sum(decode_bytes(DB, DL, w) for _, w in dec_layers)
    value = world * pre_flops / (pre_ms * 1e-3) / 1e12
    dec_gbs = world * dec_bytes / (dec_ms * 1e-3) / 1e9

    hbm, tf_burst, tf_sus, peak_src = load_peaks()
    peak = tf_sus if wl["peak"] == "sustained" else tf_burst
    # dominant kernel: the full-causal prefill layer
    full_idx = [i for i, (_, w) in enumerate(pre_layers) if w <= 0][0]
    full_ms = float(seg_total[full_idx]) / args.steps
    full_tf = prefill_flops(B, S, 0) / (full_ms * 1e-3) / 1e12
    slid_idx = [i for i, (_, w) in enumerate(pre_layers) if w > 0][0]
    slid_ms = float(seg_total[slid_idx]) / args.steps
    slid_bytes = prefill_bytes(B, S)
    dfull_idx = npre + [i for i, (_, w) in enumerate(dec_layers) if w <= 0][0]
    dfull_ms = float(seg_total[dfull_idx]) / args.steps
    dfull_gbs = decode_bytes(DB, DL, 0) / (dfull_ms * 1e-3) / 1e9

    # end to end through the public API from pinned host buffers (prefill layers):
    # every step copies each layer's inputs in and its output out
    hostin = []
    h2d = d2h = 0
    for p in pre:
        hq, hk, hv = (p[n].cpu().pin_memory() for n in ("q", "k", "v"))
        hs, hp = p["sinks"].cpu().pin_memory(), p["pos"].cpu().pin_memory()
        ho = torch.empty(p["out"].shape, dtype=torch.bfloat16).pin_memory()
        hostin.append((hq, hk, hv, hs, hp, p["window"], ho))
        h2d += sum(t.numel() * t.element_size() for t in (hq, hk, hv, hs, hp))
        d2h += ho.numel() * ho.element_size()
    e2e_steps = max(3, min(args.steps, 20 if S <= 16384 else 3))
    for hq, hk, hv, hs, hp, w, ho in hostin:
        gqa.prefill(hq, hk, hv, hs, hp, w, out=ho)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        for hq, hk, hv, hs, hp, w, ho in hostin:
            gqa.prefill(hq, hk, hv, hs, hp, w, out=ho)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = shard.max_over_ranks([e2e_ms], dev)[0]
    e2e_value = world * pre_flops / (e2e_ms * 1e-3) / 1e12
    del hostin

    if rank == 0:
        cpu = None
        if world == 1:
            sampler = OracleSampler(wl, tensors={"pre": pre})
            rows, seqs = sampler.calibrate(target_s=3.0)
            res = [sampler.sample(i, rows, seqs) for i in range(4)]
            pf = sum(r["prefill_flops"] for r in res)
            ps = sum(r["prefill_s"] for r in res)
            cpu = {"value": pf / ps / 1e12, "unit": "TFLOP/s", "cores": host_cores(),
                   "kind": "oracle",
                   "sample": "4 samples of %d evenly spaced query rows (all 64 heads) of each "
                             "prefill layer: %.3g unmasked FLOPs in %.1f s" % (rows, pf, ps)}
        traffic = profiled_traffic(os.path.join(
            ROOT, "profiles", "prefill_kernel_full_S%d_traffic.txt" % S))
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded N(0,1) bf16 q/k/v and caches, N(0,1) fp32 sinks "
                    "(synth recipe, drawn on the device)",
            "config": step_config(wl),
            "parallelism": "dp%d (independent replicas)" % world,
            "timing": {"prefill_ms_per_step": pre_ms, "decode_ms_per_step": dec_ms,
                       "full_layer_ms": full_ms, "sliding_layer_ms": slid_ms,
                       "wall_s": t_wall},
            "roofline": {"kernel": "prefill (key rotation + prefill_kernel, full-causal layer, "
                                   "B=%d S=%d)" % (B, S), "bound": "tensor",
                         "achieved": full_tf, "peak": peak, "unit": "TFLOP/s",
                         "frac": full_tf / peak,
                         "peak_source": "%s (%s)" % (peak_src, wl["peak"]),
                         "traffic": traffic,
                         "algorithmic_bytes": prefill_bytes(B, S),
                         "flops_per_launch": prefill_flops(B, S, 0),
                         "launch_ms": full_ms},
            # the unit that binds prefill_kernel at head_dim 64: one exp2 per visible
            # (query, key, head), 16 results per clock per SM (measured), 148 SMs, at the
            # median SM clock seen during the timed steps
            "exp_roofline": exp_roofline(prefill_flops(B, S, 0), full_ms, clk.summary()),
            "sliding_roofline": {"kernel": "prefill (key rotation + prefill_band_kernel, W=128)",
                                 "bound": "hbm",
                                 "achieved": slid_bytes / (slid_ms * 1e-3) / 1e9, "peak": hbm,
                                 "unit": "GB/s",
                                 "frac": slid_bytes / (slid_ms * 1e-3) / 1e9 / hbm,
                                 "algorithmic_bytes": slid_bytes, "launch_ms": slid_ms},
            "decode": {"value": dec_gbs, "unit": "GB/s", "frac": dec_gbs / world / hbm,
                       "peak": hbm, "full_layer_gbs": dfull_gbs,
                       "full_layer_frac": dfull_gbs / hbm, "full_layer_ms": dfull_ms},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "what": "prefill layers via host buffers"},
            # per step: key rotation + attention per prefill layer; per decode layer the
            # split kernel, plus the combine kernel unless one split covers the range
            "gpu_launches": args.steps * (2 * len(pre_layers) + sum(
                1 if (min(w, DL) if w > 0 else DL) <= 256 else 2 for _, w in dec_layers)),
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ long prefill workloads

LONG_WORKLOADS = {
    # name: (config id of the seed recipe, B, S, [(layer, window), ...], description)
    "tiny256": (1, 1, 256, [(0, 0), (1, 128)],
                "prefill B=1 S=256 64q/8kv d64, one full-causal layer + one W=128 layer "
                "(launch-latency bound)"),
    "batch16k": (3, 4, 16384, [(i, 128 if i % 2 == 0 else 0) for i in range(24)],
                 "prefill B=4 S=16384 64q/8kv d64, 12 W=128 layers + 12 full-causal layers "
                 "alternating, each with its own inputs"),
    "seq128k": (5, 1, 131072, [(0, 0), (1, 128)],
                "prefill B=1 S=131072 64q/8kv d64, one full-causal layer + one W=128 layer"),
    # the 36-layer stack of the larger model: W=128 and full-causal layers alternating
    "layers36": (7, 1, 4096, [(i, 128 if i % 2 == 0 else 0) for i in range(36)],
                 "prefill B=1 S=4096 64q/8kv d64 through 36 layers, 18 W=128 + 18 full-causal "
                 "alternating, each with its own inputs"),
}


def oracle_rows_sample(layers, budget_s: float = 12.0):
    """Times the fp64 oracle on evenly spaced query rows of the given layers
    ([(q, k, v, sinks, pos, window) device tensors]); returns (TFLOP/s, s, rows, FLOPs)."""
    import oracle
    oracle._load()
    total_flops, total_s, nrows = 0.0, 0.0, 0
    per_layer = budget_s / len(layers)
    for q, k, v, sinks, pos, window in layers:
        B, S = q.shape[0], q.shape[1]
        kh = k.double().cpu().numpy()
        vh = v.double().cpu().numpy()
        sh = sinks.double().cpu().numpy()
        ph = pos.cpu().numpy()
        n = 8
        while True:
            toks = np.linspace(0, S - 1, n).astype(np.int64)
            rows = [(int(i % B), int(t)) for i, t in enumerate(toks)]
            q_rows = np.stack([q[b, t].double().cpu().numpy() for b, t in rows])
            t0 = time.perf_counter()
            oracle.prefill_rows(q_rows, kh, vh, sh, ph, window, rows)
            dt = time.perf_counter() - t0
            if dt >= per_layer / 3 or n >= 4096:
                break
            n *= 4
        total_flops += sum(4.0 * D * NQ * (min(t + 1, window) if 0 < window < S else t + 1)
                           for t in toks)
        total_s += dt
        nrows += n
    return total_flops / total_s / 1e12, total_s, nrows, total_flops


def run_long(args, name: str):
    """One GPU: a step is every layer of the named long workload once (distinct
    buffers per layer, inputs drawn on the device). Prints one JSON line."""
    import torch

    import attention_gqa_b200 as gqa
    from attention_gqa_b200 import build
    build.build()
    cfg, B, S, layers, desc = LONG_WORKLOADS[name]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    gqa.init()
    stream = torch.cuda.current_stream()
    bufs = [_prefill_layer(cfg, layer, window, B, S, dev, gqa) for layer, window in layers]
    steps = max(1, min(args.steps, 20))

    def step(ev=None):
        for i, p in enumerate(bufs):
            if ev is not None:
                ev[i].record(stream)
            gqa.prefill(p["q"], p["k"], p["v"], p["sinks"], p["pos"], p["window"], out=p["out"],
                        workspace=p["ws"])
        if ev is not None:
            ev[len(bufs)].record(stream)

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    gqa.check()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(bufs) + 1)]
              for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        for s_ in range(steps):
            flush.fill_(s_ & 0xFF)
            step(events[s_])
        torch.cuda.synchronize()
    gqa.check()
    seg = np.array([[events[s_][i].elapsed_time(events[s_][i + 1]) for i in range(len(bufs))]
                    for s_ in range(steps)]).sum(axis=0) / steps        # ms per layer
    flops = [prefill_flops(B, S, w) for _, w in layers]
    step_ms = float(seg.sum())
    value = sum(flops) / (step_ms * 1e-3) / 1e12
    full = [i for i, (_, w) in enumerate(layers) if w <= 0]
    slid = [i for i, (_, w) in enumerate(layers) if w > 0]
    full_ms = float(seg[full].sum()) / len(full)
    slid_ms = float(seg[slid].sum()) / len(slid)
    full_tf = prefill_flops(B, S, 0) / (full_ms * 1e-3) / 1e12
    slid_tf = prefill_flops(B, S, 128) / (slid_ms * 1e-3) / 1e12
    # algorithmic bytes of a sliding layer (q, out, k, v once each; the key
    # pre-pass's extra read and write of k is a cost of the implementation)
    slid_bytes = prefill_bytes(B, S)
    hbm, tf_burst, tf_sus, peak_src = load_peaks()

    # end to end through host buffers, one full-causal layer
    p = bufs[full[0]]
    hq, hk, hv = (p[n].cpu().pin_memory() for n in ("q", "k", "v"))
    hs, hp = p["sinks"].cpu().pin_memory(), p["pos"].cpu().pin_memory()
    ho = torch.empty(p["out"].shape, dtype=torch.bfloat16).pin_memory()
    gqa.prefill(hq, hk, hv, hs, hp, 0, out=ho)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    gqa.prefill(hq, hk, hv, hs, hp, 0, out=ho)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_tf = prefill_flops(B, S, 0) / (e0.elapsed_time(e1) * 1e-3) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hs, hp))

    cpu_v, cpu_s, cpu_rows, cpu_flops = oracle_rows_sample(
        [(bufs[i]["q"], bufs[i]["k"], bufs[i]["v"], bufs[i]["sinks"], bufs[i]["pos"], layers[i][1])
         for i in (full[0], slid[0])])
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 q/k/v and fp32 sinks (synth recipe, drawn on "
                "the device), pos = token index",
        "config": {"workload": desc,
                   "l2": "flushed before every step (256 MB write)" +
                         ("; every layer's inputs exceed L2" if prefill_bytes(B, S) > 126e6
                          else "; a layer's inputs fit in L2"),
                   "full_layer_ms": full_ms, "full_layer_tflops": full_tf,
                   "sliding_layer_ms": slid_ms, "sliding_layer_tflops": slid_tf,
                   "sliding_layer_gbs": slid_bytes / (slid_ms * 1e-3) / 1e9},
        "roofline": {"kernel": "prefill (key rotation + prefill_kernel, full-causal layer)",
                     "bound": "tensor", "achieved": full_tf, "peak": tf_sus, "unit": "TFLOP/s",
                     "frac": full_tf / tf_sus, "peak_source": peak_src + " (sustained)",
                     "traffic": None, "algorithmic_bytes": prefill_bytes(B, S),
                     "launch_ms": full_ms},
        "exp_roofline": exp_roofline(prefill_flops(B, S, 0), full_ms, clk.summary()),
        "sliding_roofline": {"bound": "hbm", "achieved": slid_bytes / (slid_ms * 1e-3) / 1e9,
                             "peak": hbm, "unit": "GB/s",
                             "frac": slid_bytes / (slid_ms * 1e-3) / 1e9 / hbm},
        "cpu_baseline": {"value": cpu_v, "unit": "TFLOP/s", "cores": host_cores(),
                         "kind": "oracle",
                         "sample": "%d evenly spaced query rows (all 64 heads) of one full and "
                                   "one sliding layer, %.3g unmasked FLOPs, %.1f s"
                                   % (cpu_rows, cpu_flops, cpu_s)},
        "e2e": {"value": e2e_tf, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": ho.numel() * ho.element_size(),
                "what": "one full-causal layer via host buffers"},
        "gpu_launches": steps * 2 * len(layers),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_chunk(args):
    """One GPU: a step is a 4096-token chunk prefilled against a 12288-token
    cached prefix (gptoss_attn_prefill_chunk), for a full-causal and a W=128
    layer, each with its own cache. Prints one JSON line."""
    import torch

    import attention_gqa_b200 as gqa
    from attention_gqa_b200 import build
    build.build()
    B, L, start, n = 1, 16384, 12288, 4096
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    gqa.init()
    stream = torch.cuda.current_stream()
    layers = []
    for layer, window in ((0, 0), (1, 128)):
        def draw(shape, tid):
            g = torch.Generator(device=dev)
            g.manual_seed(0x6A77 ^ (6 << 24) ^ (layer << 12) ^ tid)
            return torch.randn(shape, generator=g, device=dev, dtype=torch.float32)
        q = draw((B, L, NQ, D), 1).to(torch.bfloat16)
        k = draw((B, L, NKV, D), 2).to(torch.bfloat16)
        v = draw((B, L, NKV, D), 3).to(torch.bfloat16)
        sinks = draw((NQ,), 4)
        pos = torch.arange(L, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
        kc = torch.empty(B, L, NKV, D, dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        # the cached prefix, written once (untimed)
        gqa.prefill_chunk(q[:, :start].contiguous(), k[:, :start].contiguous(),
                          v[:, :start].contiguous(), sinks, pos[:, :start].contiguous(), kc, vc,
                          0, window)
        layers.append(dict(q=q, k=k, v=v, sinks=sinks, pos=pos, window=window, kc=kc, vc=vc,
                           cq=q[:, start:].contiguous(), ck=k[:, start:].contiguous(),
                           cv=v[:, start:].contiguous(), cp=pos[:, start:].contiguous(),
                           out=torch.empty(B, n, NQ, D, dtype=torch.bfloat16, device=dev)))
    gqa.check()
    steps = max(1, min(args.steps, 20))

    def step(ev=None):
        for i, p in enumerate(layers):
            if ev is not None:
                ev[i].record(stream)
            gqa.prefill_chunk(p["cq"], p["ck"], p["cv"], p["sinks"], p["cp"], p["kc"], p["vc"],
                              start, p["window"], out=p["out"])
        if ev is not None:
            ev[len(layers)].record(stream)

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    gqa.check()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(layers) + 1)]
              for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        for s_ in range(steps):
            flush.fill_(s_ & 0xFF)
            step(events[s_])
        torch.cuda.synchronize()
    gqa.check()
    seg = np.array([[events[s_][i].elapsed_time(events[s_][i + 1]) for i in range(len(layers))]
                    for s_ in range(steps)]).sum(axis=0) / steps
    pairs = [n * start + n * (n + 1) // 2, 128 * n]      # visible pairs of the chunk's queries
    flops = [4.0 * D * NQ * B * p for p in pairs]
    step_ms = float(seg.sum())
    value = sum(flops) / (step_ms * 1e-3) / 1e12
    full_tf = flops[0] / (seg[0] * 1e-3) / 1e12
    hbm, tf_burst, tf_sus, peak_src = load_peaks()
    # e2e: the chunk's inputs from pinned host memory, its output back, per layer
    p = layers[0]
    host = [t.cpu().pin_memory() for t in (p["cq"], p["ck"], p["cv"], p["sinks"], p["cp"])]
    dbuf = [torch.empty_like(t, device=dev) for t in host]
    hout = torch.empty(p["out"].shape, dtype=torch.bfloat16).pin_memory()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for d_, h_ in zip(dbuf, host):
        d_.copy_(h_, non_blocking=True)
    gqa.prefill_chunk(dbuf[0], dbuf[1], dbuf[2], dbuf[3], dbuf[4], p["kc"], p["vc"], start, 0,
                      out=p["out"])
    hout.copy_(p["out"], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_tf = flops[0] / (e0.elapsed_time(e1) * 1e-3) / 1e12
    cpu_v, cpu_s, cpu_rows, cpu_flops = oracle_chunk_sample(layers[0], start, n)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: N(0,1) bf16 q/k/v and fp32 sinks drawn on the device (torch "
                "generator seeded per layer), pos = token index",
        "config": {"workload": "chunked prefill B=1: 4096 new tokens after 12288 cached ones "
                               "(cache 16384), one full-causal layer + one W=128 layer",
                   "l2": "flushed before every step (256 MB write)",
                   "full_layer_ms": float(seg[0]), "full_layer_tflops": full_tf,
                   "sliding_layer_ms": float(seg[1])},
        "roofline": {"kernel": "chunked prefill (value copy + key rotation + prefill_kernel, "
                               "full-causal layer)", "bound": "tensor", "achieved": full_tf,
                     "peak": tf_burst, "unit": "TFLOP/s", "frac": full_tf / tf_burst,
                     "peak_source": peak_src + " (burst)", "traffic": None,
                     "launch_ms": float(seg[0])},
        "cpu_baseline": {"value": cpu_v, "unit": "TFLOP/s", "cores": host_cores(),
                         "kind": "oracle",
                         "sample": "%d evenly spaced query rows (all 64 heads) of the full-causal "
                                   "chunk, %.3g unmasked FLOPs, %.1f s"
                                   % (cpu_rows, cpu_flops, cpu_s)},
        "e2e": {"value": e2e_tf, "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host),
                "d2h_bytes_per_step": hout.numel() * hout.element_size(),
                "what": "the full-causal chunk with its inputs from pinned host memory"},
        "gpu_launches": steps * 2 * len(layers),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


BACKWARD_WORKLOADS = {
    # name: (config id of the seed recipe, B, S, [(layer, window), ...], description)
    "bwd4k": (2, 1, 4096, [(0, 128), (1, 0)],
              "backward of the prefill B=1 S=4096 64q/8kv d64, one W=128 layer + one full-causal "
              "layer (dq, dk, dv, dsinks from out, lse and a random dO)"),
    "bwd16k": (3, 4, 16384, [(0, 128), (1, 0)],
               "backward of the prefill B=4 S=16384 64q/8kv d64, one W=128 layer + one "
               "full-causal layer"),
}


def run_backward(args, name: str):
    """One GPU: a step is the backward pass of every layer of the workload once.
    FLOPs follow the usual convention for attention backward: 2.5 times the
    forward's unmasked FLOPs (the five products S, dP, dV, dK, dQ over the
    visible pairs; the kernels recompute S and dP once more). Prints one line."""
    import torch

    import attention_gqa_b200 as gqa
    import synth
    from attention_gqa_b200 import build
    from synth import device as sdev
    build.build()
    cfg, B, S, layers, desc = BACKWARD_WORKLOADS[name]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    gqa.init()
    stream = torch.cuda.current_stream()
    bufs = []
    for layer, window in layers:
        p = _prefill_layer(cfg, layer, window, B, S, dev, gqa)
        p["out"], p["lse"] = gqa.prefill_lse(p["q"], p["k"], p["v"], p["sinks"], p["pos"], window)
        p["dout"] = sdev.bf16_normal(_seed(cfg, layer, 5), (B, S, NQ, D), dev)
        p["bws"] = torch.empty(gqa.prefill_backward_workspace_bytes(B, S), dtype=torch.uint8,
                               device=dev)
        bufs.append(p)
    gqa.check()
    steps = max(1, min(args.steps, 20))

    def step(ev=None):
        for i, p in enumerate(bufs):
            if ev is not None:
                ev[i].record(stream)
            gqa.prefill_backward(p["q"], p["k"], p["v"], p["sinks"], p["pos"], p["window"],
                                 p["out"], p["lse"], p["dout"], workspace=p["bws"])
        if ev is not None:
            ev[len(bufs)].record(stream)

    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    gqa.check()
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(bufs) + 1)]
              for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        for s_ in range(steps):
            flush.fill_(s_ & 0xFF)
            step(events[s_])
        torch.cuda.synchronize()
    gqa.check()
    seg = np.array([[events[s_][i].elapsed_time(events[s_][i + 1]) for i in range(len(bufs))]
                    for s_ in range(steps)]).sum(axis=0) / steps
    flops = [2.5 * prefill_flops(B, S, w) for _, w in layers]
    step_ms = float(seg.sum())
    value = sum(flops) / (step_ms * 1e-3) / 1e12
    full = [i for i, (_, w) in enumerate(layers) if w <= 0][0]
    full_tf = flops[full] / (seg[full] * 1e-3) / 1e12
    hbm, tf_burst, tf_sus, peak_src = load_peaks()
    line = {
        "metric": "attention backward TFLOP/s (2.5x the unmasked forward FLOPs)", "value": value,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) bf16 q/k/v/dO and fp32 sinks (synth recipe, drawn on "
                "the device), pos = token index",
        "config": {"workload": desc, "l2": "flushed before every step (256 MB write)",
                   "layer_ms": [float(x) for x in seg]},
        "roofline": {"kernel": "backward (rotations + prep + bwd_dq_kernel + bwd_dkv_kernel), "
                               "full-causal layer", "bound": "tensor", "achieved": full_tf,
                     "peak": tf_burst, "unit": "TFLOP/s", "frac": full_tf / tf_burst,
                     "peak_source": peak_src + " (burst)", "traffic": None,
                     "launch_ms": float(seg[full])},
        "gpu_launches": steps * 5 * len(layers),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def oracle_chunk_sample(p, start: int, n: int, budget_s: float = 6.0):
    """The fp64 oracle on evenly spaced query rows of a chunk (keys: the whole
    cached prefix plus the chunk); returns (TFLOP/s, s, rows, FLOPs)."""
    import oracle
    oracle._load()
    kh = p["k"].double().cpu().numpy()
    vh = p["v"].double().cpu().numpy()
    sh = p["sinks"].double().cpu().numpy()
    ph = p["pos"].cpu().numpy()
    m = 8
    while True:
        toks = start + np.linspace(0, n - 1, m).astype(np.int64)
        rows = [(0, int(t)) for t in toks]
        q_rows = np.stack([p["q"][0, t].double().cpu().numpy() for _, t in rows])
        t0 = time.perf_counter()
        oracle.prefill_rows(q_rows, kh, vh, sh, ph, p["window"], rows)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 3 or m >= 4096:
            break
        m *= 4
    flops = sum(4.0 * D * NQ * (t + 1) for t in toks)
    return flops / dt / 1e12, dt, m, flops


def run_call(args):
    """One GPU, no timing: one attention operation run --reps times on seeded
    inputs (the command the ncu captures under profiles/ run). --op fwd runs
    the prefill, bwd the backward pass, dec the decode."""
    import torch

    import attention_gqa_b200 as gqa
    from attention_gqa_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    gqa.init()
    B, S, W = args.batch, args.seqlen, args.window
    if args.op == "dec":
        d = _decode_layer(4, 0, W, B, S, dev, gqa)
        for _ in range(args.reps):
            gqa.decode(d["q"], d["kc"], d["vc"], d["sinks"], d["len"], W, out=d["out"],
                       workspace=d["ws"])
    else:
        p = _prefill_layer(9, 0, W, B, S, dev, gqa)
        if args.op == "fwd":
            for _ in range(args.reps):
                gqa.prefill(p["q"], p["k"], p["v"], p["sinks"], p["pos"], W, out=p["out"],
                            workspace=p["ws"])
        else:
            import synth
            from synth import device as sdev
            out, lse = gqa.prefill_lse(p["q"], p["k"], p["v"], p["sinks"], p["pos"], W)
            dout = sdev.bf16_normal(synth.seed_for(9, 0, 5), (B, S, NQ, D), dev)
            ws = torch.empty(gqa.prefill_backward_workspace_bytes(B, S), dtype=torch.uint8,
                             device=dev)
            for _ in range(args.reps):
                gqa.prefill_backward(p["q"], p["k"], p["v"], p["sinks"], p["pos"], W, out, lse,
                                     dout, workspace=ws)
    gqa.check()
    torch.cuda.synchronize()
    print(json.dumps({"call": args.op, "batch": B, "seqlen": S, "window": W, "reps": args.reps}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(STEP_WORKLOADS) + ["chunk16k", "call"] +
                    sorted(LONG_WORKLOADS) + sorted(BACKWARD_WORKLOADS), default="default",
                    help="default: prefill B=1 S=131072 + decode B=64 L=8192; s4096: the same "
                         "step with a B=1 S=4096 prefill; tiny256 / batch16k / seq128k / "
                         "layers36: prefill-only workloads; chunk16k: chunked prefill against a "
                         "cache; bwd4k / bwd16k: the backward pass (one GPU, at most 20 timed "
                         "steps); call: run --op once per --reps, untimed (for profilers)")
    ap.add_argument("--op", choices=["fwd", "bwd", "dec"], default="fwd")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--seqlen", type=int, default=16384)
    ap.add_argument("--window", type=int, default=0)
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        wl = STEP_WORKLOADS.get(args.workload, STEP_WORKLOADS["default"])
        return run_reference(args, rank, wl)
    if args.workload in STEP_WORKLOADS:
        return run_ours(args, rank, world, STEP_WORKLOADS[args.workload])
    if world > 1:
        print("--workload %s runs on one GPU" % args.workload, file=sys.stderr)
        return 2
    if args.workload == "chunk16k":
        return run_chunk(args)
    if args.workload == "call":
        return run_call(args)
    if args.workload in BACKWARD_WORKLOADS:
        return run_backward(args, args.workload)
    return run_long(args, args.workload)


if __name__ == "__main__":
    sys.exit(main())
