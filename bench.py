"""Benchmark of the int4 blockwise-quantised Qwen2 decoder step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

Default workload (N = 1): the full 28-layer decoder_step at 1.5B shapes (hidden 1536, 12/2 heads
x 128, intermediate 8960, vocab 151936 tied), symmetric int4 block-32 weights from N(0, 0.02)
masters, batch 1, past P = 1024, sequences of 64 consecutive steps that each append to the
GPU-resident KV cache (the length is reset to 1024 after every 64 steps).  A bench step is one
decoder_step.  Inputs are seeded synthetic data; weights (1.2 GB) and the lm_head (467 MB) are far
larger than L2, so no flush is needed between steps.

Multi-GPU (torchrun): replicas only -- every rank runs its own decoder on its own GPU, no
collective on the data path; value = tokens of all ranks / max-over-ranks device time.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = ("decode step µs & tok/s at batch 1; achieved HBM GB/s vs B200 peak (1.5B, 7B)")

CONFIGS = {
    # name: (shape, mode, past P, steps per sequence, description)
    "decode-1p5b": (synth.SHAPE_1P5B, "int4", 1024, 64,
                    "28-layer decoder_step, 1.5B shapes, int4 sym block-32, P=1024, batch 1"),
    "decode-7b": (synth.SHAPE_7B, "int4", 4096, 64,
                  "28-layer decoder_step, 7B shapes, int4 sym block-32, P=4096, batch 1"),
    "decode-asr-1p5b": (synth.SHAPE_1P5B, "ternary", 4530, 256,
                        "ASR-shaped long decode, 1.5B ternary, P=4530 -> 4785, batch 1"),
    "decode-0p5b": (synth.SHAPE_0P5B, "int4", 1024, 64,
                    "20-layer decoder_step, Realtime-0.5B shapes (hidden 896, 7 q / 1 kv heads of "
                    "128), int4 sym block-32, P=1024, batch 1"),
    "layer-1p5b": (synth.Shape("layer", 1536, 1, 12, 2, 128, 8960, 151936, tied=True), "ternary",
                   128, 64, "one decoder layer + lm_head, 1.5B shapes, ternary, P=128"),
}


PREFILL_CONFIGS = {
    # name: (shape, mode, S, audio frames N, description)
    "prefill-asr-1p5b": (synth.SHAPE_1P5B, "int4", 4530, 4500,
                         "28-layer decoder_init, 1.5B shapes, int4 sym block-32, S=4530 (20 text "
                         "ids + 4500 spliced audio_features + 10 text ids), batch 1"),
}


def std_for(shape):
    return 0.015 if shape.hidden == 3584 else 0.02


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------------- bytes
def phase_bytes(shape, P):
    """Algorithmic bytes per launch of each decode phase at past length P (per layer, except
    the lm_head which is per step): the bytes the method must move from HBM -- packed weights
    (16 code bytes + 2 scale bytes per 32 weights), fp16 biases and RMSNorm gammas, the KV read
    (P positions) and write (1 position), the fp16 lm_head, the fp32 logits and the fp16 input
    embedding.  Activations between phases stay on chip / in L2 and are not counted."""
    H, D, Hq, Hkv, I, V = shape.hidden, shape.head_dim, shape.n_q, shape.n_kv, shape.inter, shape.vocab

    def packed(N, K):
        return N * (K // 32) * 18

    qkv_rows = (Hq + 2 * Hkv) * D
    return {
        "qkv": packed(qkv_rows, H) + 2 * qkv_rows + 2 * H,
        "attn": 2 * Hkv * (P + 1) * D * 2,
        "o_proj": packed(H, Hq * D),
        "gate_up": 2 * packed(I, H) + 2 * H,
        "down": packed(H, I),
        "lm_head": V * H * 2 + 2 * H + 4 * V + 2 * H,
    }


def prefill_flops(shape, S):
    """Algorithmic FLOPs of one decoder_init over S positions: the GEMM part (q/k/v, o, gate/up,
    down over all S rows) and the causal attention part (QK^T and PV over the S(S+1)/2 visible
    pairs), plus the last row's lm_head."""
    H, D, Hq, Hkv, I, V = shape.hidden, shape.head_dim, shape.n_q, shape.n_kv, shape.inter, shape.vocab
    gemm = 2 * S * (H * (Hq + 2 * Hkv) * D + Hq * D * H + H * 2 * I + I * H) * shape.layers
    attn = 2 * 2 * Hq * D * (S * (S + 1) // 2) * shape.layers
    return {"gemm": gemm, "attention": attn, "lm_head": 2 * V * H}


def variant_step_bytes(shape, Ps, kv_bytes=2):
    """Algorithmic bytes of one step of len(Ps) sequences stepped together: the weights and the
    lm_head once, each sequence's KV read (P_b positions) and write in the cache's element size,
    its logits and its input embedding."""
    b = phase_bytes(shape, 0)
    L, Hkv, D = shape.layers, shape.n_kv, shape.head_dim
    weights = L * sum(v for k, v in b.items() if k not in ("lm_head", "attn"))
    head_w = shape.vocab * shape.hidden * 2 + 2 * shape.hidden
    per_seq = sum(L * 2 * Hkv * (P + 1) * D * kv_bytes + 4 * shape.vocab + 2 * shape.hidden
                  for P in Ps)
    return weights + head_w + per_seq


def step_bytes(shape, P):
    b = phase_bytes(shape, P)
    return shape.layers * sum(v for k, v in b.items() if k != "lm_head") + b["lm_head"]


# ----------------------------------------------------------------------------------- ranks
def max_over_ranks(value, dist, device):
    """The slowest rank's value (every rank gets it); the identity without a process group."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, world, ms):
    """Units of all ranks per second over the max-over-ranks time `ms` (weak scaling)."""
    return world * units_per_rank / (ms / 1e3)


# ----------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.dev = device_index
        import tempfile

        self.path = os.path.join(tempfile.gettempdir(), f"vv_clocks_rank{device_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.dev)], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


# ------------------------------------------------------------------------------ CPU baseline
class OracleSample:
    """The oracle (as it stands) on a bounded sample of one decode step: one decoder layer
    (weights dequantised inside the call, as the oracle always does) plus 1/L of the lm_head
    rows.  L such samples make one step, so step time ~= L x sample time."""

    def __init__(self, shape, mode, P, layers=2):
        from oracle import decoder as odec
        from oracle import pack as opack

        std = std_for(shape)
        self.shape, self.P = shape, P
        self.layers = []
        for li in range(layers):
            lw = dict(synth.layer_vectors(shape, li))
            for m in synth.MATRICES:
                W = synth.master(shape, m, li, std)
                lw[m] = (opack.pack_ternary(W, opack.ternary_scale(W)) if mode == "ternary"
                         else opack.pack_sym_int4(W))
            self.layers.append(lw)
        tables = synth.model_tables(shape)
        rows = -(-shape.vocab // shape.layers)
        self.lm_slice = np.ascontiguousarray(tables["lm_head"][:rows])
        self.final_norm = tables["final_norm"]
        sub = synth.Shape(shape.name, shape.hidden, layers, shape.n_q, shape.n_kv,
                          shape.head_dim, shape.inter, shape.vocab, shape.tied)
        self.kp, self.vp = synth.past_kv(sub, P)
        self.emb = synth.input_embeds(shape)[0]
        self.cfg1 = odec.Config(shape.hidden, 1, shape.n_q, shape.n_kv, shape.head_dim,
                                shape.inter, shape.vocab, shape.eps, shape.theta)
        self.i = 0

    def run(self):
        """One sample; returns the scaled step time in seconds."""
        from oracle import decoder as odec

        li = self.i % len(self.layers)
        self.i += 1
        W1 = {"layers": [self.layers[li]]}
        t0 = time.perf_counter()
        r = odec.decoder_step(self.cfg1, dict(W1, lm_head=self.lm_slice,
                                              final_norm=self.final_norm, embed=None),
                              self.emb, self.P, [self.kp[li]], [self.vp[li]])
        dt = time.perf_counter() - t0
        assert np.isfinite(r["logits"]).all()
        return dt * self.shape.layers

    def describe(self, n):
        return (f"oracle: {n} samples of one decoder layer (dequantised in the call) + 1/"
                f"{self.shape.layers} of the lm_head rows at P={self.P}; step time = "
                f"{self.shape.layers} x median sample")


def oracle_sample_time(shape, mode, P, samples=8):
    o = OracleSample(shape, mode, P)
    ts = [o.run() for _ in range(samples)]
    return statistics.median(ts), o.describe(samples), blas_threads()


def oracle_sample_time_1thread(shape, mode, P, samples=3):
    """The same oracle sample with BLAS limited to one thread."""
    from threadpoolctl import threadpool_limits

    o = OracleSample(shape, mode, P)
    with threadpool_limits(limits=1):
        ts = [o.run() for _ in range(samples)]
    return statistics.median(ts), o.describe(samples)


def decode_cpu_baseline(shape, mode, P, samples=8):
    """The oracle's decode step on the host cores (all BLAS threads) and at one thread."""
    st, sample, thr = oracle_sample_time(shape, mode, P, samples)
    rec = {"value": round(1.0 / st, 4), "unit": "tok/s", "cores": thr, "kind": "oracle",
           "sample": sample, "host_cpus": os.cpu_count()}
    try:
        st1, sample1 = oracle_sample_time_1thread(shape, mode, P, min(samples, 3))
        rec["one_thread"] = {"value": round(1.0 / st1, 4), "unit": "tok/s", "cores": 1,
                             "sample": sample1}
    except Exception as e:  # threadpoolctl missing: report the all-cores figure only
        rec["one_thread"] = {"error": str(e)[:200]}
    return rec


def prefill_cpu_baseline(shape, mode, S, N):
    """The oracle's prefill over S positions (one decoder layer, scaled by L) at all BLAS threads
    and at one thread."""
    o = OraclePrefillSample(shape, mode, S, N)
    st = o.run()
    rec = {"value": round(S / st, 3), "unit": "tok/s", "cores": blas_threads(), "kind": "oracle",
           "sample": o.describe(1), "host_cpus": os.cpu_count()}
    try:
        from threadpoolctl import threadpool_limits

        with threadpool_limits(limits=1):
            st1 = o.run()
        rec["one_thread"] = {"value": round(S / st1, 3), "unit": "tok/s", "cores": 1,
                             "sample": o.describe(1)}
    except Exception as e:
        rec["one_thread"] = {"error": str(e)[:200]}
    return rec


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ------------------------------------------------------------------------------------ ours
def init_dist(world, local_rank):
    import torch

    torch.cuda.set_device(local_rank)
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist_mod

    dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    return dist_mod


def build_model(shape, mode):
    from int4_blockwise_quantised_b200 import _vv
    from int4_blockwise_quantised_b200.model import PackedModel

    std = std_for(shape)
    vmode = _vv.VV_TERNARY if mode == "ternary" else _vv.VV_SYM_INT4
    return PackedModel(shape, vmode, lambda li, m: synth.master(shape, m, li, std),
                       lambda li: synth.layer_vectors(shape, li), synth.model_tables(shape),
                       "cuda")


def measure_variant(config, steps, warmup, local_rank, model, batch=1, kv=None):
    """Device-timed decode steps of a variant of `config` on one GPU: `batch` sequences stepped
    together (pasts P, P - 96, ...) and/or a KV cache of another element type (kv: "bf16" or
    "f32").  Greedy tokens fed back on the device; the metric counts every sequence's token."""
    import torch

    from int4_blockwise_quantised_b200.model import Decoder

    shape, mode, P, seq, desc = CONFIGS[config]
    tdt = {None: torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[kv]
    eb = {None: 2, "bf16": 2, "f32": 4}[kv]
    Ps = [P - 96 * b for b in range(batch)]
    dec = Decoder(model, P + steps + warmup + 16, kv_dtype=tdt, batch=batch)
    for b in range(batch):
        kp, vp = synth.past_kv(shape, Ps[b], base=17 * b)
        dec.k_cache[:, b, :, :Ps[b]] = torch.from_numpy(kp).cuda().to(tdt)
        dec.v_cache[:, b, :, :Ps[b]] = torch.from_numpy(vp).cuda().to(tdt)
        del kp, vp
    stream = torch.cuda.current_stream()
    tok = torch.full((batch,), 151643 % shape.vocab, dtype=torch.int32, device="cuda")
    pos = torch.tensor(Ps, dtype=torch.int32, device="cuda")
    logits = torch.empty((batch, shape.vocab), dtype=torch.float32, device="cuda")
    dec.set_lengths(Ps)
    for i in range(warmup):
        dec.step(pos, token=tok, logits=logits, argmax=tok)
        pos.add_(1)
    dec.sync_status()
    dec.set_lengths(Ps)
    pos.copy_(torch.tensor(Ps, dtype=torch.int32))
    clocks = ClockSampler(local_rank)
    clocks.start()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for i in range(steps):
        dec.step(pos, token=tok, logits=logits, argmax=tok)
        pos.add_(1)
    ev1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    dec.sync_status()
    ms = ev0.elapsed_time(ev1)
    us = ms * 1e3 / steps
    mean_Ps = [p_ + (steps - 1) / 2 for p_ in Ps]
    byts = variant_step_bytes(shape, mean_Ps, eb)
    peak, kind = peaks()
    gbs = byts / (us * 1e-6) / 1e9
    del dec
    torch.cuda.empty_cache()
    return {"workload": config + (f"-batch{batch}" if batch > 1 else "") + (f"-kv-{kv}" if kv else ""),
            "value": round(batch * steps / (ms * 1e-3), 1), "unit": "tok/s",
            "us_per_step": round(us, 2), "batch": batch, "pasts": Ps,
            "kv_dtype": {None: "f16", "bf16": "bf16", "f32": "f32"}[kv],
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(gbs / peak, 4), "peak_kind": kind,
                         "bytes_per_step": int(byts)},
            "clocks": clk}


def measure_decode(config, steps, warmup, dist, world, local_rank, model=None):
    """Device-timed decode steps of one config (inputs resident, greedy token fed back on the
    device), the per-step distribution over one sequence, the end-to-end variant through the
    public API with host buffers, the roofline of the step kernel and its timeline breakdown.
    Returns (record, model)."""
    import torch

    from int4_blockwise_quantised_b200.model import Decoder

    shape, mode, P, seq, desc = CONFIGS[config]
    t0 = time.time()
    if model is None:
        model = build_model(shape, mode)
    setup_s = time.time() - t0
    cap = P + max(seq, 64) + 8
    dec = Decoder(model, cap)
    kp, vp = synth.past_kv(shape, P)
    dec.k_cache[:, 0, :, :P] = torch.from_numpy(kp).cuda()
    dec.v_cache[:, 0, :, :P] = torch.from_numpy(vp).cuda()
    del kp, vp
    dec.set_length(P)
    stream = torch.cuda.current_stream()

    # Device-resident inputs for the device-timed value: token ids fed back greedily.
    tok = torch.tensor([151643 % shape.vocab], dtype=torch.int32, device="cuda")
    pos = torch.tensor([P], dtype=torch.int32, device="cuda")
    logits = torch.empty(shape.vocab, dtype=torch.float32, device="cuda")

    def one_step(i):
        # i = index within the sequence; position = P + i; greedy token fed back on device.
        if i == 0:
            dec.set_length(P)
            pos.fill_(P)
        dec.step(pos, token=tok, logits=logits, argmax=tok)
        pos.add_(1)

    n_launch = dec.step_launches
    # warm-up (also captures the graph)
    for i in range(warmup):
        one_step(i % seq)
    dec.sync_status()

    clocks = ClockSampler(local_rank)
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    seq_starts = 0
    for i in range(steps):
        if i % seq == 0:
            seq_starts += 1  # vv_decoder_set_length: one set_int_kernel
        one_step(i % seq)
    ev1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    dec.sync_status()
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, dist, "cuda")
    ms_per_step = ms / steps
    tok_s = whole_job_rate(steps, world, ms)
    # this library's kernels only: one step launch per step (persistent kernel) plus the length
    # reset at each sequence start; torch's position fill / increment are not counted
    gpu_launches = steps * n_launch + seq_starts

    # -------------------------------------- per-step distribution (one sequence, not timed above)
    step_ev = [torch.cuda.Event(enable_timing=True) for _ in range(seq + 1)]
    torch.cuda.synchronize()
    step_ev[0].record(stream)
    for i in range(seq):
        one_step(i)
        step_ev[i + 1].record(stream)
    torch.cuda.synchronize()
    per_step = sorted(step_ev[i].elapsed_time(step_ev[i + 1]) * 1e3 for i in range(seq))
    pct = {"p50": round(per_step[len(per_step) // 2], 2),
           "p90": round(per_step[min(len(per_step) - 1, (9 * len(per_step)) // 10)], 2),
           "steps": seq, "note": "per-step CUDA events over one sequence of steps from P "
                                 "(includes the position increment), outside the timed region"}

    # ---------------------------------------------------------------- e2e (host buffers)
    emb_host = torch.from_numpy(synth.input_embeds(shape, 1)[0]).pin_memory()
    pos_host = torch.tensor([P], dtype=torch.int32).pin_memory()
    out_host = torch.empty(1, dtype=torch.int32).pin_memory()
    emb_dev = torch.empty(shape.hidden, dtype=torch.float16, device="cuda")
    pos_dev = torch.empty(1, dtype=torch.int32, device="cuda")
    am_dev = torch.empty(1, dtype=torch.int32, device="cuda")
    e2e_steps = min(steps, 256)
    for i in range(3):  # capture the e2e graph (different pointers) outside the timed region
        dec.set_length(P)
        emb_dev.copy_(emb_host, non_blocking=True)
        pos_dev.copy_(pos_host, non_blocking=True)
        dec.step(pos_dev, input_embeds=emb_dev, argmax=am_dev)
        out_host.copy_(am_dev, non_blocking=True)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        if i % seq == 0:
            dec.set_length(P)
        pos_host[0] = P + (i % seq)
        emb_dev.copy_(emb_host, non_blocking=True)
        pos_dev.copy_(pos_host, non_blocking=True)
        dec.step(pos_dev, input_embeds=emb_dev, argmax=am_dev)
        out_host.copy_(am_dev, non_blocking=True)
        stream.synchronize()  # the host reads the greedy token every step
        _ = int(out_host[0])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
    e2e_tok_s = whole_job_rate(e2e_steps, world, e2e_ms)

    # -------------------------------------------------- roofline of the dominant kernel
    # One persistent cooperative kernel per step: its average launch duration is the timed
    # region's ms_per_step (CUDA events on the launching stream, one launch per step).
    sb = step_bytes(shape, P + seq // 2)
    peak, peak_kind = peaks()
    achieved = sb / (ms_per_step * 1e-3) / 1e9
    roofline = {"bound": "hbm", "kernel": "step_kernel (persistent decode step, 1 launch/step)",
                "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "traffic": traffic_for("step_kernel", config),
                "algorithmic_bytes_per_launch": sb, "avg_launch_us": round(ms_per_step * 1e3, 2)}
    # per-phase breakdown from the kernel's timeline tap (one extra step, not timed)
    try:
        dec.set_length(P)
        pos.fill_(P)
        stamps, _ = dec.step_timeline(pos, token=tok)
        roofline["phases_us"] = phase_breakdown(stamps.astype(np.int64), shape.layers)
    except Exception as e:  # the tap is diagnostics only
        roofline["phases_us"] = {"error": str(e)[:200]}
    dec.close()
    rec = {
        "value": round(tok_s, 2), "unit": "tok/s", "ms_per_step": round(ms_per_step, 5),
        "config": {"workload": config, "description": desc, "batch": 1, "past_P": P,
                   "steps_per_sequence": seq, "weights": f"{mode} block-32",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (weights %.0f MB, L2 126 MB); no flush" % (
                       sb / 1e6)},
        "step_us": round(ms_per_step * 1e3, 2),
        "step_us_percentiles": pct,
        "hbm_gbs": round(achieved, 1),
        "hbm_frac_of_measured": round(achieved / peak, 4),
        "hbm_frac_of_8tbs": round(sb / (ms_per_step * 1e-3) / 8e12, 4),
        "algorithmic_bytes_per_step": sb,
        "roofline": roofline,
        "e2e": {"value": round(e2e_tok_s, 2), "unit": "tok/s",
                "h2d_bytes_per_step": shape.hidden * 2 + 4, "d2h_bytes_per_step": 4,
                "steps": e2e_steps,
                "note": "public API: pinned host input_embeds + position -> device copy, graph step, "
                        "argmax device->host read and stream sync every step"},
        "gpu_launches": gpu_launches,
        "clocks": clk,
        "setup_s": round(setup_s, 1),
    }
    return rec, model


def run_ours(args, rank, world, local_rank):
    import torch

    dist = init_dist(world, local_rank)
    rec, model = measure_decode(args.config, args.steps, args.warmup, dist, world, local_rank)
    result = {"metric": METRIC, "value": rec["value"], "unit": "tok/s", "n_gpus": world,
              "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec["ms_per_step"],
              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
              "data": "synthetic"}
    result.update({k: v for k, v in rec.items() if k not in result})
    if args.config == "decode-1p5b" and not args.no_prefill:
        # decoder_init at S = 4530 on the same int4 1.5B weights (the ASR prefill workload)
        pshape, _, pS, pN, _ = PREFILL_CONFIGS["prefill-asr-1p5b"]
        pr = measure_prefill(model, pshape, pS, pN, 10, 3, dist, world)
        result["prefill"] = {"workload": "prefill-asr-1p5b", "value": round(pr["tok_s"], 1),
                             "unit": "tok/s", "ms": round(pr["ms"], 3),
                             "tflops_whole_prefill": round(pr["tflops_whole"], 1),
                             "e2e_tok_s": round(pr["e2e_tok_s"], 1), "roofline": pr["roofline"],
                             "clocks": pr["clocks"]}
        result["gpu_launches_prefill"] = pr["launches"] * 10
    if args.config == "decode-1p5b" and not args.no_extra and world == 1:
        # batch 2 (the CFG pair) and the bf16 / fp32 KV-cache variants of the same workload
        variants = {}
        for batch, kv in ((2, None), (1, "bf16"), (1, "f32")):
            r3 = measure_variant(args.config, min(args.steps, 64), args.warmup, local_rank, model,
                                 batch=batch, kv=kv)
            variants[r3["workload"]] = r3
        result["variants"] = variants
    del model
    torch.cuda.empty_cache()
    if args.config == "decode-1p5b" and not args.no_extra:
        # the metric's other model size and the long-context decode, each a sub-record with its
        # own roofline, e2e and clocks (same timing protocol, fewer steps)
        for sub in ("decode-7b", "decode-asr-1p5b", "decode-0p5b"):
            r2, m2 = measure_decode(sub, min(args.steps, 64), args.warmup, dist, world, local_rank)
            del m2
            torch.cuda.empty_cache()
            r2["steps"] = min(args.steps, 64)
            result[sub.replace("-", "_")] = r2
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        shape, mode, P, _, _ = CONFIGS[args.config]
        result["cpu_baseline"] = decode_cpu_baseline(shape, mode, P)
        if "decode_7b" in result:  # the 7B decode (config 4) at all cores and one thread
            s7, m7, P7, _, _ = CONFIGS["decode-7b"]
            result["decode_7b"]["cpu_baseline"] = decode_cpu_baseline(s7, m7, P7, samples=3)
        if "prefill" in result:  # the S = 4530 prefill (config 5) at one thread as well
            pshape, pmode, pS, pN, _ = PREFILL_CONFIGS["prefill-asr-1p5b"]
            result["prefill"]["cpu_baseline"] = prefill_cpu_baseline(pshape, pmode, pS, pN)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# ----------------------------------------------------------------------------------- prefill
def prefill_inputs(shape, S, N):
    prefix = 20
    ids, pos, feats, off = synth.asr_prompt(shape, N, prefix=prefix, suffix=S - N - prefix)
    assert ids.size == S
    return ids, pos, feats, off


def measure_prefill(model, shape, S, N, steps, warmup, dist=None, world=1):
    """Device-timed decoder_init over S positions (inputs resident), the end-to-end variant
    (pinned host ids / positions / audio_features copied in, argmax read back, every step), and
    the per-kind breakdown from one profiled prefill."""
    import torch

    from int4_blockwise_quantised_b200.model import Decoder

    dec = Decoder(model, S + 8, max_prefill=S)
    ids, pos, feats, off = prefill_inputs(shape, S, N)
    ids_d, pos_d, feats_d = (torch.from_numpy(a).cuda() for a in (ids, pos, feats))
    logits = torch.empty(shape.vocab, dtype=torch.float32, device="cuda")
    am = torch.empty(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        dec.init(ids_d, pos_d, feats_d, off, logits=logits, argmax=am)
    dec.sync_status()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        dec.init(ids_d, pos_d, feats_d, off, logits=logits, argmax=am)
    ev1.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    dec.sync_status()
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, dist, "cuda")
    ms_per = ms / steps
    # end to end: host buffers in, greedy token out
    ids_h, pos_h, feats_h = (torch.from_numpy(a).pin_memory() for a in (ids, pos, feats))
    out_h = torch.empty(1, dtype=torch.int32).pin_memory()
    e2e_steps = max(3, min(steps, 20))
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        ids_d.copy_(ids_h, non_blocking=True)
        pos_d.copy_(pos_h, non_blocking=True)
        feats_d.copy_(feats_h, non_blocking=True)
        dec.init(ids_d, pos_d, feats_d, off, argmax=am)
        out_h.copy_(am, non_blocking=True)
        stream.synchronize()
        _ = int(out_h[0])
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dist, "cuda")
    kind_ms, kind_n = dec.profile_init(ids_d, pos_d, feats_d, off, logits=logits, argmax=am)
    dec.sync_status()
    dec.close()
    fl = prefill_flops(shape, S)
    mp = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    peak = mp.get("bf16_tflops", 1590.0)
    peak_sus = mp.get("bf16_tflops_sustained", 1400.0)
    kind = "measured" if mp else "fallback"
    gemm_ms = kind_ms["gemm"]
    ach = fl["gemm"] / (gemm_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "kernel": "gemm_tc (tcgen05 kind::f16, persistent, 128 x 256, 192 or 128 tiles, 2 TMEM accumulators)",
            "achieved": round(ach, 1), "peak": peak, "peak_kind": f"{kind} bf16 burst (fp16 dense "
            "rate = bf16 on B200, nominal ratio 1)", "unit": "TFLOP/s",
            "frac": round(ach / peak, 4), "frac_of_sustained": round(ach / peak_sus, 4),
            "traffic": traffic_for("gemm_tc"),
            "algorithmic_flops_per_launch": fl["gemm"] // max(kind_n["gemm"], 1),
            "avg_launch_us": round(gemm_ms * 1e3 / max(kind_n["gemm"], 1), 2),
            "launches_per_prefill": kind_n["gemm"],
            "breakdown_ms": {k: round(v, 3) for k, v in kind_ms.items()},
            "breakdown_launches": kind_n,
            "attention_tflops": round(fl["attention"] / (kind_ms["attention"] * 1e-3) / 1e12, 1)
            if kind_ms["attention"] > 0 else None}
    total_fl = fl["gemm"] + fl["attention"] + fl["lm_head"]
    return {
        "tok_s": world * S / (ms_per * 1e-3), "ms": ms_per, "steps": steps,
        "e2e_tok_s": world * S / (e2e_ms * 1e-3), "e2e_ms": e2e_ms,
        "h2d_bytes": ids.nbytes + pos.nbytes + feats.nbytes, "d2h_bytes": 4,
        "tflops_whole": total_fl / (ms_per * 1e-3) / 1e12, "roofline": roof, "clocks": clk,
        # kernels of one prefill: the profiled marks minus the per-layer bias copies
        "launches": sum(kind_n.values()) - shape.layers,
    }


class OraclePrefillSample:
    """The oracle on a bounded sample of one decoder_init: one decoder layer over all S
    positions (weights dequantised inside the call) plus the lm_head row; prefill time =
    L x that sample."""

    def __init__(self, shape, mode, S, N):
        from oracle import decoder as odec
        from oracle import pack as opack

        std = std_for(shape)
        self.shape = shape
        lw = dict(synth.layer_vectors(shape, 0))
        for m in synth.MATRICES:
            W = synth.master(shape, m, 0, std)
            lw[m] = (opack.pack_ternary(W, opack.ternary_scale(W)) if mode == "ternary"
                     else opack.pack_sym_int4(W))
        tables = synth.model_tables(shape)
        self.W = {"layers": [lw], "embed": tables["embed"], "lm_head": tables["lm_head"],
                  "final_norm": tables["final_norm"]}
        self.cfg1 = odec.Config(shape.hidden, 1, shape.n_q, shape.n_kv, shape.head_dim,
                                shape.inter, shape.vocab, shape.eps, shape.theta)
        self.inputs = prefill_inputs(shape, S, N)
        self.S = S

    def run(self):
        from oracle import decoder as odec

        ids, pos, feats, off = self.inputs
        t0 = time.perf_counter()
        r = odec.decoder_init(self.cfg1, self.W, ids, pos, feats, off)
        dt = time.perf_counter() - t0
        assert np.isfinite(r["logits"]).all()
        return dt * self.shape.layers

    def describe(self, n):
        return (f"oracle: {n} sample(s) of decoder_init with one decoder layer over all "
                f"S={self.S} positions (+ the last row's lm_head); prefill time = "
                f"{self.shape.layers} x sample")


def run_prefill(args, rank, world, local_rank):
    import torch

    from int4_blockwise_quantised_b200 import _vv
    from int4_blockwise_quantised_b200.model import PackedModel

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        import datetime

        dist = dist_mod
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    shape, mode, S, N, desc = PREFILL_CONFIGS[args.config]
    vmode = _vv.VV_TERNARY if mode == "ternary" else _vv.VV_SYM_INT4
    t0 = time.time()
    model = PackedModel(shape, vmode, lambda li, m: synth.master(shape, m, li, std_for(shape)),
                        lambda li: synth.layer_vectors(shape, li), synth.model_tables(shape),
                        "cuda")
    setup_s = time.time() - t0
    r = measure_prefill(model, shape, S, N, args.steps, args.warmup, dist, world)
    result = {
        "metric": "prefill tok/s (decoder_init, batch 1); tensor-core GEMM TFLOP/s vs B200 peak",
        "value": round(r["tok_s"], 1), "unit": "tok/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(r["ms"], 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16 (fp32 accumulate)",
        "data": "synthetic",
        "config": {"workload": args.config, "description": desc, "S": S, "audio_frames": N,
                   "weights": f"{mode} block-32",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (weights 1.2 GB read and 120 MB activations "
                         "per layer); no flush"},
        "tflops_whole_prefill": round(r["tflops_whole"], 1),
        "roofline": r["roofline"],
        "e2e": {"value": round(r["e2e_tok_s"], 1), "unit": "tok/s",
                "h2d_bytes_per_step": r["h2d_bytes"], "d2h_bytes_per_step": r["d2h_bytes"],
                "note": "public API: pinned host input_ids + position_ids + audio_features -> "
                        "device, decoder_init, argmax device->host read + sync every step"},
        "gpu_launches": r["launches"] * args.steps,
        "clocks": r["clocks"], "setup_s": round(setup_s, 1),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        o = OraclePrefillSample(shape, mode, S, N)
        st = o.run()
        result["cpu_baseline"] = {"value": round(S / st, 3), "unit": "tok/s",
                                  "cores": blas_threads(), "kind": "oracle",
                                  "sample": o.describe(1)}
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


PHASES = ("qkv", "attn", "o", "gu_down")


def timeline_names(L):
    """Stamp names of one CTA's row, in the step kernel's order: kernel start; per layer the
    barrier before each phase (arrive, exit; none before layer 0's q/k/v), then the point where
    the phase's input is staged (q/k/v, gate/up) or its work is done (attention, o-proj); in the
    gate/up + down phase also the end of gate/up and the staged h; the layer end; then the lm_head
    barrier, its staged input and the end."""
    names = ["start"]
    for l in range(L):
        if l > 0:
            names += [f"L{l}.qkv.arrive", f"L{l}.qkv.exit"]
        names += [f"L{l}.qkv.staged"]
        names += [f"L{l}.attn.arrive", f"L{l}.attn.exit", f"L{l}.attn.done"]
        names += [f"L{l}.o.arrive", f"L{l}.o.exit", f"L{l}.o.done"]
        names += [f"L{l}.gu_down.arrive", f"L{l}.gu_down.exit", f"L{l}.gu_down.staged",
                  f"L{l}.gu_down.gu_done", f"L{l}.gu_down.h_staged", f"L{l}.end"]
    names += ["head.arrive", "head.exit", "head.staged", "end"]
    return names


def phase_breakdown(st, L):
    """Critical-path time per phase summed over layers (us) from the timeline stamps: a phase
    runs from the last CTA's exit of its barrier (kernel start for layer 0's q/k/v) to the last
    CTA's arrival at the next barrier; barrier = release latency after the last arrival."""
    names = timeline_names(L)
    if st.shape[1] != len(names):
        return {"error": f"{st.shape[1]} stamps, expected {len(names)}"}
    ix = {k: i for i, k in enumerate(names)}
    st = st - st[:, 0].min()
    out = {}
    for l in range(L):
        for j, ph in enumerate(PHASES):
            b = ix["start"] if (l == 0 and j == 0) else ix[f"L{l}.{ph}.exit"]
            nxt = f"L{l}.{PHASES[j + 1]}" if j + 1 < len(PHASES) else (
                f"L{l + 1}.qkv" if l + 1 < L else "head")
            e = ix[nxt + ".arrive"]
            out[ph] = out.get(ph, 0) + (st[:, e].max() - st[:, b].max())
            out["barriers"] = out.get("barriers", 0) + (st[:, ix[nxt + ".exit"]].max() - st[:, e].max())
    out["lm_head"] = st[:, ix["end"]].max() - st[:, ix["head.exit"]].max()
    out["total"] = st[:, ix["end"]].max()
    return {k: round(v / 1e3, 1) for k, v in out.items()}


def traffic_for(kernel, workload=None):
    """DRAM bytes per launch from the committed ncu summary (entry "kernel/workload", or "kernel"
    when no workload is named), or None when there is no capture of that workload or the
    kernel's source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    tab = json.load(open(p))
    d = tab.get(f"{kernel}/{workload}") if workload else tab.get(kernel)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] if os.path.exists(src) else None
    return d["dram_bytes_per_launch"] if h == d.get("source_sha") else None


# ------------------------------------------------------------------------------ reference arm
class OracleFullStep:
    """The oracle (as it stands) running whole decode steps: every layer (each packed matrix
    dequantised inside the call, as the oracle always does) and the full lm_head."""

    def __init__(self, shape, mode, P):
        from oracle import decoder as odec
        from oracle import pack as opack

        std = std_for(shape)
        self.shape, self.P = shape, P
        layers = []
        for li in range(shape.layers):
            lw = dict(synth.layer_vectors(shape, li))
            for m in synth.MATRICES:
                W = synth.master(shape, m, li, std)
                lw[m] = (opack.pack_ternary(W, opack.ternary_scale(W)) if mode == "ternary"
                         else opack.pack_sym_int4(W))
            layers.append(lw)
        self.W = dict(synth.model_tables(shape), layers=layers)
        self.kp, self.vp = synth.past_kv(shape, P)
        self.emb = synth.input_embeds(shape)[0]
        self.cfg = odec.Config(shape.hidden, shape.layers, shape.n_q, shape.n_kv,
                               shape.head_dim, shape.inter, shape.vocab, shape.eps, shape.theta)

    def run(self):
        from oracle import decoder as odec

        t0 = time.perf_counter()
        r = odec.decoder_step(self.cfg, self.W, self.emb, self.P, list(self.kp), list(self.vp))
        dt = time.perf_counter() - t0
        assert np.isfinite(r["logits"]).all()
        return dt


def run_reference(args, rank):
    """The oracle as the reference arm: whole decode steps (all layers + lm_head) of this arm's
    config, metric and unit; at most 1 warm-up and 3 timed steps (each is seconds of CPU work).
    Under torchrun only rank 0 runs."""
    if rank != 0:
        return
    if args.config in PREFILL_CONFIGS:
        run_reference_prefill(args)
        return
    shape, mode, P, seq, desc = CONFIGS[args.config]
    t0 = time.perf_counter()
    o = OracleFullStep(shape, mode, P)
    setup_s = time.perf_counter() - t0
    warm, steps = min(args.warmup, 1), min(args.steps, 3)
    for _ in range(warm):
        o.run()
    t0 = time.perf_counter()
    ts = [o.run() for _ in range(steps)]
    wall = time.perf_counter() - t0
    st = statistics.median(ts)
    value = 1.0 / st
    result = {
        "metric": METRIC, "value": round(value, 4), "unit": "tok/s", "n_gpus": 1,
        "steps": steps, "warmup": warm, "ms_per_step": round(st * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": args.config, "description": desc, "batch": 1, "past_P": P},
        "cpu_baseline": {"value": round(value, 4), "unit": "tok/s", "cores": blas_threads(),
                         "kind": "oracle",
                         "sample": f"{steps} whole oracle decode steps ({shape.layers} layers, "
                                   f"dequantised per call, full lm_head) at P={P}; median"},
        "e2e": {"value": round(value, 4), "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 2), "setup_s": round(setup_s, 1),
    }
    print(json.dumps(result), flush=True)


def run_reference_prefill(args):
    """Reference arm for a prefill config: the oracle's decoder_init on one layer over all S
    positions per step (scaled by L); at most 1 warm-up and 3 timed samples (each is tens of
    seconds of CPU work)."""
    shape, mode, S, N, desc = PREFILL_CONFIGS[args.config]
    o = OraclePrefillSample(shape, mode, S, N)
    warm, steps = min(args.warmup, 1), min(args.steps, 3)
    for _ in range(warm):
        o.run()
    t0 = time.perf_counter()
    est = [o.run() for _ in range(steps)]
    wall = time.perf_counter() - t0
    st = statistics.median(est)
    value = S / st
    print(json.dumps({
        "metric": "prefill tok/s (decoder_init, batch 1); tensor-core GEMM TFLOP/s vs B200 peak",
        "value": round(value, 3), "unit": "tok/s", "n_gpus": 1, "steps": steps, "warmup": warm,
        "ms_per_step": round(st * 1e3, 1), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": args.config, "description": desc, "S": S, "audio_frames": N},
        "cpu_baseline": {"value": round(value, 3), "unit": "tok/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": o.describe(steps)},
        "e2e": {"value": round(value, 3), "unit": "tok/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 2),
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--config", default="decode-1p5b",
                    choices=sorted(CONFIGS) + sorted(PREFILL_CONFIGS))
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill measurement added to the default decode line")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the 7B and long-context decode sub-records of the default line")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.config in PREFILL_CONFIGS:
        run_prefill(args, rank, world, local_rank)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
