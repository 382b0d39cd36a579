#!/usr/bin/env python
"""Throughput of block-sparse attention forward + backward on B200 (sm_100a).

One step = one pass of the whole hot path over one batch: metadata (KV lists, transposed
lists) + forward (Out, LSE) + backward (dQ, dK, dV), all in the library's CUDA kernels.  The
default workload is the long-context block-sparse attention: B=1, N=32, S=131072, D=128 with
128x128 blocks, each q block selecting min(64, causal) KV blocks (diagonal, 4 previous, the
first block, the rest uniform), causal (synthetic, seeded).  --config 2 runs the S=8192 workload
(B=2, N=16, causal Bernoulli(0.25) mask).

The metric is effective TFLOP/s: credited FLOPs / time, with forward 4*D*V and backward
10*D*V for V visible (query, key) pairs (the diagonal block counts only its visible half).  Per
kernel the credits are forward 4*D*V (S, O), KV-major pass 8*D*V (S, dP, dV, dK) and Q-major pass
2*D*V (dQ only: its S and dP are recomputations already credited to the KV pass).

The end-to-end number copies each step's inputs in from pinned host memory and every output back,
with the host-to-device and device-to-host copies on their own streams, double-buffered against
the compute stream (the copies of step i+1 and i-1 overlap the compute of step i).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 1|2|3|4|5]

--config 3 runs the NSA selected-attention workload (TND, 4 batches of 4096..32768 tokens, GQA
64/4, 16 blocks of 64 tokens per token) forward + backward under the same metric; --config 4
runs the paged sparse decode workload (gathered-KV bandwidth).

With N > 1 (launched by torchrun, one process per GPU) every rank runs its own copy of the
workload (independent batches: weak scaling, no collective on the data path); time is the max
over ranks.  --impl reference times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import synth  # noqa: E402

METRIC = "effective block-sparse attn fwd+bwd TFLOP/s (bf16)"
METRIC_NSA = "effective NSA selected attn fwd+bwd TFLOP/s (bf16)"
METRIC_DEC = "sparse decode gathered-KV bandwidth (paged, bf16)"
METRIC_DEC_BWD = "sparse decode backward gathered-KV + gradient-row bandwidth (paged, bf16)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# nominal B200 figures, reported beside the measured-peak fractions: dense bf16 and HBM3e
SPEC_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}


def with_spec(roof):
    """Add the nominal peak and the fraction of it to a roofline entry (None passes through)."""
    if roof is None:
        return None
    spec = SPEC_PEAKS["hbm_gbs" if roof["unit"] == "GB/s" else "bf16_tflops"]
    roof["spec_peak"] = spec
    roof["frac_of_spec"] = roof["achieved"] / spec if roof["achieved"] is not None else None
    return roof

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum of one launch) from an ncu
# capture of each kernel, valid only while the kernel's source file is unchanged (sha1 prefix of
# the file recorded at capture time); reported as null once the source has changed.
NCU_TRAFFIC = [
    {"kernel": "bsa_bwd_kv", "bytes": 492699648 + 103334144, "config": 2, "src": "selected_attention_b200/csrc/bsa_bwd.cu",
     "src_sha1": "0143e70727d3"},
    {"kernel": "bsa_bwd_q", "bytes": 270674688 + 52001024, "config": 2, "src": "selected_attention_b200/csrc/bsa_bwd.cu",
     "src_sha1": "0143e70727d3"},
    {"kernel": "bsa_fwd", "bytes": 201507840 + 52752640, "config": 2, "src": "selected_attention_b200/csrc/bsa_fwd.cu",
     "src_sha1": "3b1165691fa4"},
    # full-size launches of the S=131072 workload (one-pass DRAM counters)
    {"kernel": "bsa_bwd_kv", "bytes": 12216385024 + 2114009088, "config": 5,
     "src": "selected_attention_b200/csrc/bsa_bwd.cu", "src_sha1": "0143e70727d3"},
    {"kernel": "bsa_bwd_q", "bytes": 5664402432 + 1057575936, "config": 5, "src": "selected_attention_b200/csrc/bsa_bwd.cu",
     "src_sha1": "0143e70727d3"},
    {"kernel": "bsa_fwd", "bytes": 4296163840 + 1075880960, "config": 5, "src": "selected_attention_b200/csrc/bsa_fwd.cu",
     "src_sha1": "3b1165691fa4"},
    {"kernel": "sfa_decode", "bytes": 147508480 + 4237312, "config": 4, "src": "selected_attention_b200/csrc/sfa_decode.cu",
     "src_sha1": "6c80d26dac90"},
]


def ncu_traffic(kernel, config):
    """DRAM bytes of one launch of `kernel` on workload `config` from an ncu capture, or None when
    there is none or the kernel's source has changed since."""
    for tr in NCU_TRAFFIC:
        if tr["kernel"] == kernel and tr["config"] == config and tr["src_sha1"] == source_sha1(tr["src"]):
            return tr["bytes"]
    return None


def visible_pairs_bsa(mask: np.ndarray, bx: int, by: int, s_q: int, s_kv: int) -> int:
    """Exact number of (query, key) pairs that are selected and causal-visible."""
    nqb, nkb = mask.shape[-2:]
    per_block = np.zeros((nqb, nkb), dtype=np.int64)
    for qb in range(nqb):
        rows = np.arange(qb * bx, min(s_q, (qb + 1) * bx))
        for kb in range(nkb):
            k0, k1 = kb * by, min(s_kv, (kb + 1) * by)
            if k0 > rows[-1]:
                continue
            per_block[qb, kb] = np.clip(np.minimum(rows, k1 - 1) - k0 + 1, 0, None).sum()
    sel = (mask != 0).reshape(-1, nqb, nkb).sum(axis=0)
    return int((sel * per_block).sum())


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clocks / throttle reasons, sampled every 50 ms from just before the timed region to
    just after it.  Entering waits (at most 3 s) for the first sample, so sampling is live when the
    timed steps start; summary() uses the samples taken inside the block, or, when the block was
    shorter than the sampling period, the nearest sample on each side of it."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []  # (host time, csv line)
        self.t_in = self.t_out = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            deadline = time.monotonic() + 3.0
            while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
        except (OSError, ValueError):
            self.proc = None
        self.t_in = time.monotonic()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def __exit__(self, *a):
        self.t_out = time.monotonic()
        if self.proc is not None:
            time.sleep(0.06)  # one more sample after the block
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        inside = [ln for t, ln in self.lines if self.t_in <= t <= self.t_out]
        window = "timed region"
        if not inside:
            before = [ln for t, ln in self.lines if t < self.t_in][-1:]
            after = [ln for t, ln in self.lines if t > self.t_out][:1]
            inside, window = before + after, "nearest samples around a timed region shorter than 50 ms"
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in inside:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "window": window}


def bsa_workload(config: int):
    w = synth.workload(config)
    assert isinstance(w, synth.BsaWorkload), "bench supports the BSA workloads (1, 2, 5)"
    return w


def cpu_oracle_sample(w, mask, budget_s: float, chunk: int = 64):
    """Time the fp64 oracle (forward + backward) on runs of about `chunk` Q blocks spread over each
    (b, h) head slice in turn (every unit's full contribution: its dQ rows and its share of dK /
    dV), until budget_s of oracle time has passed; returns (credited FLOPs, seconds, description)."""
    from oracle import attention as A
    flops, dt, units, t_wall = 0, 0.0, 0, time.perf_counter()
    nqb = mask.shape[2]
    for b in range(w.B):
        for h in range(w.N1):
            q = A.bf16_to_f64(w.tensor("q", b, h))[None]
            k = A.bf16_to_f64(w.tensor("k", b, h))
            v = A.bf16_to_f64(w.tensor("v", b, h))
            do = A.bf16_to_f64(w.tensor("dout", b, h))[None]
            n_runs = -(-nqb // chunk)
            for r0 in range(n_runs):  # run r0 takes q blocks r0, r0 + n_runs, ...: spread over the head
                qbs = list(range(r0, nqb, n_runs))
                t0 = time.perf_counter()
                A.bsa_slice_backward(q, k, v, do, mask[b, h][None], w.block, w.block, w.mask_mode, w.scale,
                                     q_blocks=qbs, out_storage="bf16")
                dt += time.perf_counter() - t0
                sub = np.zeros_like(mask[b, h])
                sub[qbs] = mask[b, h][qbs]
                flops += 14 * w.D * visible_pairs_bsa(sub[None, None], w.block, w.block, w.S, w.S)
                units += len(qbs)
                if dt >= budget_s or time.perf_counter() - t_wall >= 4 * budget_s:
                    return flops, dt, (f"oracle fwd+bwd on {units} of {w.B * w.N1 * nqb} (b, h, q block) units "
                                       f"(head slices in order, {chunk} q blocks spread over the head at a time)")
    return flops, dt, f"oracle fwd+bwd on all {units} (b, h, q block) units"


def cpu_oracle_sample_decode(w, budget_s: float):
    """Time the fp64 oracle decode one batch at a time until budget_s of oracle time has passed;
    returns (gathered bytes done, seconds, description)."""
    from oracle import attention as A
    table, idx = w.selection()
    seqused = np.full(w.B, w.context, np.int32)
    q, qr = w.query("q"), w.query("q_rope")
    per_batch = w.count * w.sparse_block * (w.D + w.Dr + w.D) * 2
    done, dt = [], 0.0
    for b in range(w.B):
        pages = [int(pg) for pg in table[b, idx[b, 0, 0]]]
        kc = {pg: w.pages("k", [pg])[0] for pg in pages}
        krc = {pg: w.pages("k_rope", [pg])[0] for pg in pages}
        vc = {pg: w.pages("v", [pg])[0] for pg in pages}
        t0 = time.perf_counter()
        A.sfa_decode(q, qr, kc, krc, vc, table, idx, seqused, w.page, w.sparse_block, w.scale, batches=[b])
        dt += time.perf_counter() - t0
        done.append(b)
        if dt >= budget_s:
            break
    return len(done) * per_batch, dt, f"oracle decode of {len(done)} of {w.B} batches"


def decode_dout(w):
    """The synthetic dOut of the paged decode workload: bf16 bits [B, 1, N1, D]."""
    return synth.normal_rows_bf16(w.seed, "dout", w.B, w.N1 * w.D, 1).reshape(w.B, 1, w.N1, w.D)


def cpu_oracle_sample_decode_bwd(w, budget_s: float):
    """Time the fp64 oracle backward of the decode one batch at a time (the batch's selected pages
    gathered into small caches) until budget_s of oracle time has passed; returns (bytes credited:
    gathered rows read plus gradient rows written, seconds, description)."""
    from oracle import attention as A
    table, idx = w.selection()
    seqused = np.full(w.B, w.context, np.int32)
    q, qr, do = w.query("q"), w.query("q_rope"), decode_dout(w)
    per_batch = 2 * w.count * w.sparse_block * (w.D + w.Dr + w.D) * 2
    ppb = w.sparse_block // w.page
    done, dt = [], 0.0
    for b in range(w.B):
        logical = sorted({int(j) * ppb + x for j in idx[b, 0, 0] if j >= 0 for x in range(ppb)})
        phys = [int(table[b, lp]) for lp in logical]
        small = {tag: w.pages(tag, phys) for tag in ("k", "k_rope", "v")}
        t2 = np.zeros((1, table.shape[1]), np.int32)
        t2[0, logical] = np.arange(len(logical), dtype=np.int32)
        t0 = time.perf_counter()
        A.sfa_backward(q[b:b + 1], qr[b:b + 1], small["k"], small["k_rope"], small["v"], do[b:b + 1], t2,
                       idx[b:b + 1], seqused[b:b + 1], w.page, w.sparse_block, w.scale)
        dt += time.perf_counter() - t0
        done.append(b)
        if dt >= budget_s:
            break
    return len(done) * per_batch, dt, f"oracle decode backward of {len(done)} of {w.B} batches"


def visible_pairs_nsa(w, topk: np.ndarray) -> int:
    """(token, query head, key) triples the NSA mask keeps: per listed block id j (duplicates
    counted), keys j*bs .. min((j+1)*bs, len) - 1, and under the causal mask only keys <= pos."""
    total = 0
    cu = w.cu_seqlens()
    for b in range(w.B):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        pos = np.arange(t1 - t0)[:, None, None]
        ids = topk[t0:t1].astype(np.int64)
        hi = np.minimum((ids + 1) * w.sel_block, t1 - t0)
        if w.mask_mode == 2:
            hi = np.minimum(hi, pos + 1)
        n = np.clip(hi - ids * w.sel_block, 0, None)
        total += int(np.where(ids >= 0, n, 0).sum())
    return total * (w.N1 // w.N2)


def cpu_oracle_sample_nsa(w, topk, budget_s: float, chunk: int = 32):
    """Time the fp64 oracle (forward + backward) on chunks of `chunk` tokens of each (b, kv head)
    slice, round robin over the slices, until budget_s has passed."""
    from oracle import attention as A
    cu = w.cu_seqlens()
    G = w.N1 // w.N2
    f = A.bf16_to_f64
    flops, done, t_start = 0, [], time.perf_counter()
    slices = {}
    for b in range(w.B):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        q, do = w.tensor("q", t0, t1), w.tensor("dout", t0, t1)
        k, v = w.tensor("k", t0, t1), w.tensor("v", t0, t1)
        for g in range(w.N2):
            hs = slice(g * G, (g + 1) * G)
            slices[(b, g)] = (f(q[:, hs]), f(k[:, g]), f(v[:, g]), topk[t0:t1, g], f(do[:, hs]), t1 - t0)
        if b == 0:  # the first batch's slices are enough for a bounded sample
            break
    t_start = time.perf_counter()
    rnd = 0
    while True:
        for (b, g), (q, k, v, tk, do, S) in slices.items():
            toks = list(range(rnd * chunk, min(S, (rnd + 1) * chunk)))
            A.nsa_slice(q, k, v, tk, w.sel_block, w.mask_mode, w.scale, dout_g=do, tokens=toks, out_storage="bf16")
            sub = tk[toks]
            pos = np.asarray(toks)[:, None]
            hi = np.minimum((sub.astype(np.int64) + 1) * w.sel_block, S)
            if w.mask_mode == 2:
                hi = np.minimum(hi, pos + 1)
            vis = int(np.where(sub >= 0, np.clip(hi - sub.astype(np.int64) * w.sel_block, 0, None), 0).sum())
            flops += (8 * w.D + 6 * w.dv) * vis * G
            done.append((b, g, len(toks)))
            if time.perf_counter() - t_start >= budget_s:
                n = sum(x[2] for x in done)
                return flops, time.perf_counter() - t_start, \
                    f"oracle fwd+bwd on {n} (token, kv head) rows of batch 0 ({chunk}-token chunks)"
        rnd += 1


def cpu_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((x.get("num_threads", 1) for x in info), default=1)
        return int(n)
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def pipelined_e2e(steps, host_in, dev_in, dev_out, host_out, compute, barrier, max_over_ranks):
    """End-to-end steps through the public API with host buffers: every step copies its inputs from
    pinned host memory (host_in) into device buffer set i % 2 on a host-to-device stream, computes
    on the current stream, and copies every output of set i % 2 back to pinned host memory
    (host_out) on a device-to-host stream.  Events order each buffer set's reuse, so the copies of
    neighbouring steps overlap the compute.  Returns the device-timed ms per step (max over ranks)
    measured on the compute stream from before the first copy to after the last."""
    import torch
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, done, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(n):
        for i in range(n):
            j = i % 2
            if i >= 2:
                s_in.wait_event(done[j])          # compute of step i - 2 has read input set j
            with torch.cuda.stream(s_in):
                for t, x in dev_in[j].items():
                    x.copy_(host_in[t], non_blocking=True)
                in_ready[j].record(s_in)
            main.wait_event(in_ready[j])
            if i >= 2:
                main.wait_event(out_read[j])      # outputs of step i - 2 have been copied back
            compute(dev_in[j], dev_out[j])
            done[j].record(main)
            s_out.wait_event(done[j])
            with torch.cuda.stream(s_out):
                for t, x in dev_out[j].items():
                    host_out[t].copy_(x, non_blocking=True)
                out_read[j].record(s_out)
        for j in range(min(n, 2)):
            main.wait_event(out_read[j])

    run(2)  # warm-up of the copy paths
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    run(steps)
    e1.record(main)
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(e0.elapsed_time(e1) / steps)



def tensor_peak(peaks, peak_src, timed_ms):
    """The bf16 tensor denominator: the measured burst figure for a region under a second, the
    sustained (power-capped, seconds-long loop) figure for longer timed regions."""
    if timed_ms >= 1000.0 and "bf16_tflops_sustained" in peaks:
        return peaks["bf16_tflops_sustained"], f"{peak_src} bf16_tflops_sustained (timed region {timed_ms:.0f} ms)"
    return peaks["bf16_tflops"], f"{peak_src} bf16_tflops (burst; timed region {timed_ms:.0f} ms)"


def kernel_table(prof, alg, steps, peak):
    """Per kernel: launches and ms per step, and for the attention kernels their credited TFLOP/s
    and its fraction of the tensor denominator."""
    out = {}
    for n, (c, t) in prof.items():
        e = {"launches": c, "ms_per_step": t / steps}
        if n in alg and t > 0:
            tf = alg[n] * c / (t * 1e-3) / 1e12
            e.update({"credited_tflops": tf, "frac": tf / peak})
        out[n] = e
    return out



def schedule_balance(sa, torch, step, dev, capacity=512):
    """One extra step with the per-CTA start / finish record on: per persistent kernel, the time
    from the first CTA's start to the last CTA's finish (span), the spread of the CTAs' finish
    times, and the idle tail: the fraction of CTA-time (CTAs x span) spent after a CTA finished
    and before the last one did."""
    buf = torch.zeros(3, capacity, 2, dtype=torch.int64, device=dev)
    sa.bsa_profile_cta_clock(buf)
    step()
    torch.cuda.synchronize()
    sa.bsa_profile_cta_clock(None)
    t = buf.cpu().numpy()
    out = {}
    for slot, name in enumerate(("bsa_fwd", "bsa_bwd_kv", "bsa_bwd_q")):
        rows = t[slot][t[slot][:, 1] > 0]
        if len(rows) == 0:
            continue
        start, end = rows[:, 0], rows[:, 1]
        span = float(end.max() - start.min())
        out[name] = {"ctas": int(len(rows)), "span_us": span / 1e3,
                     "finish_spread_us": float(end.max() - end.min()) / 1e3,
                     "start_spread_us": float(start.max() - start.min()) / 1e3,
                     "idle_tail_frac": float((end.max() - end).sum()) / (len(rows) * span) if span > 0 else 0.0}
    return out



def run_reference(args, rank, world):
    """--impl reference: the fp64 oracle on the host cores, rank 0 only."""
    if rank != 0:
        return
    w = nsa_workload(args) if args.config == 3 else synth.workload(args.config)
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; warm-up steps are a no-op
    total_f, total_t, desc = 0, 0.0, ""
    step_budget = min(args.ref_step_seconds, 150.0 / max(1, args.steps))  # whole run ~2.5 min at most
    metric, unit, scale = METRIC, "TFLOP/s", 1e12
    if isinstance(w, synth.NsaWorkload):
        topk = w.topk()
        sample = lambda: cpu_oracle_sample_nsa(w, topk, budget_s=step_budget)  # noqa: E731
        cfg = config_dict_nsa(w, args)
        metric = METRIC_NSA
    elif isinstance(w, synth.BsaWorkload):
        if world > 1:  # the same job as the GPU arm: the workload's batches times the rank count
            import dataclasses
            w = dataclasses.replace(w, name=f"{w.name}_x{world}", B=w.B * world)
        mask = w.block_mask()
        sample = lambda: cpu_oracle_sample(w, mask, budget_s=step_budget)  # noqa: E731
        cfg = config_dict(w, args)
    elif getattr(args, "decode_bwd", False):  # the decode's backward: gathered and gradient bytes per second
        sample = lambda: cpu_oracle_sample_decode_bwd(w, budget_s=step_budget)  # noqa: E731
        cfg = dict(config_dict_decode(w), op="backward")
        metric, unit, scale = METRIC_DEC_BWD, "GB/s", 1e9
    else:  # paged sparse decode: gathered bytes per second
        sample = lambda: cpu_oracle_sample_decode(w, budget_s=step_budget)  # noqa: E731
        cfg = config_dict_decode(w)
        metric, unit, scale = METRIC_DEC, "GB/s", 1e9
    for _ in range(args.steps):
        f, t, desc = sample()
        total_f += f
        total_t += t
    value = total_f / total_t / scale
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": unit, "cores": cpu_threads(), "cpu_model": cpu_model(),
                         "kind": "oracle", "sample": f"each step: {desc}"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


def config_dict_decode(w):
    return {"workload": f"{w.name}: B={w.B}, N1={w.N1}, N2={w.N2}, D={w.D}+{w.Dr}, {w.context}-token "
                        f"cache, page {w.page}, {w.count} sparse blocks of {w.sparse_block} per query",
            "l2": "flushed (256 MiB write) before every timed rep",
            "timing": "mean over the timed reps, each one CUDA-graph replay timed with events"}


def config_dict(w, args):
    """w: the job's workload (B already multiplied by the rank count)."""
    world = args.gpus
    return {
        "workload": f"{w.name}: block-sparse attention fwd+bwd, BNSD B={w.B} N={w.N1} S={w.S} D={w.D}, "
                    f"{w.block}x{w.block} blocks, selection={w.selection} {w.sel_args}, causal",
        "B": w.B, "N": w.N1, "S": w.S, "D": w.D, "block": w.block, "seed": w.seed,
        "l2": "no flush: inputs (Q,K,V,dOut) exceed the 126 MB L2" if 4 * w.B * w.N1 * w.S * w.D * 2 > 126e6
        else "inputs fit in L2 (small parity workload)",
        "parallelism": "single GPU" if world == 1 else
        (f"dp{world}: {w.B} batches, contiguous (batch, kv head) slice ranges per rank balanced by selected "
         f"tiles; no collective on the data path"),
    }


def config_dict_nsa(w, args):
    return {
        "workload": f"{w.name}: NSA selected attention fwd+bwd, TND seqlens={w.seqlens} (T={w.T}), N1={w.N1} "
                    f"N2={w.N2} D={w.D} Dv={w.dv}, {w.sel_count} blocks of {w.sel_block} per (token, kv head), causal",
        "T": w.T, "N1": w.N1, "N2": w.N2, "D": w.D, "Dv": w.dv, "sel_block": w.sel_block, "sel_count": w.sel_count,
        "seed": w.seed, "l2": "no flush: inputs (Q, dOut 1 GiB each) exceed the 126 MB L2",
        "parallelism": f"replicas x{args.gpus} (independent batches)",
    }


def nsa_workload(args):
    """The NSA workload; --nsa-seqlens swaps in other batch lengths (same seed and shapes), a
    smaller problem for profiler captures."""
    import dataclasses
    w = synth.workload(3)
    if args.nsa_seqlens:
        lens = [int(x) for x in args.nsa_seqlens.split(",")]
        w = dataclasses.replace(w, seqlens=lens, name=f"{w.name}_seqlens_{'_'.join(map(str, lens))}")
    if getattr(args, "nsa_dqk", 128) != 128:  # q / k head dim 192 with v's 128 (the page's head-dim pair)
        w = dataclasses.replace(w, D=args.nsa_dqk, Dv=w.D, name=f"{w.name}_dqk{args.nsa_dqk}")
    return w


def sum_over_ranks(world, dev, x):
    """Bookkeeping outside the timed region (the job's credited work): the sum of x over ranks."""
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t)
    return float(t.item())


def _dist_helpers(world, dev):
    import torch

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def max_over_ranks(x):
        if world > 1:
            t = torch.tensor([x], dtype=torch.float64, device=dev)
            torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
            return float(t.item())
        return x
    return barrier, max_over_ranks


def run_nsa(args, rank, world, local_rank):
    """NSA selected attention (TND varlen, GQA) forward + backward: one step = metadata + forward
    + backward over the whole 61440-token batch."""
    import torch

    import selected_attention_b200 as sa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = nsa_workload(args)
    topk = w.topk()
    cu = w.cu_seqlens()
    vpairs = visible_pairs_nsa(w, topk)
    # forward 2 (D + Dv) per visible pair (S, O); backward S, dQ, dK 2 D each and dP, dV 2 Dv each
    flops_step = (8 * w.D + 6 * w.dv) * vpairs
    S = max(w.seqlens)
    host = {t: torch.from_numpy(w.tensor(t)).view(torch.bfloat16) for t in ("q", "k", "v", "dout")}
    host["topk"], host["cu"] = torch.from_numpy(topk), torch.from_numpy(cu)
    d = {t: x.to(dev) for t, x in host.items()}
    out = torch.empty(w.T, w.N1, w.dv, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(w.T, w.N1, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(d["q"]), torch.empty_like(d["k"]), torch.empty_like(d["v"])
    p = sa.nsa_params(d["q"], d["k"], d["topk"], d["cu"], S, w.sel_block, w.mask_mode, w.scale, w.dv)
    ws_f = torch.empty(sa.nsa_selected_fwd_workspace_size(p), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(sa.nsa_selected_bwd_workspace_size(p), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    barrier, max_over_ranks = _dist_helpers(world, dev)

    def step(x=d):
        sa.nsa_selected_fwd(x["q"], x["k"], x["v"], x["topk"], x["cu"], S, w.sel_block, w.mask_mode, w.scale,
                            out=out, lse=lse, workspace=ws_f)
        sa.nsa_selected_bwd(x["q"], x["k"], x["v"], out, x["dout"], lse, x["topk"], x["cu"], S, w.sel_block,
                            w.mask_mode, w.scale, dq=dq, dk=dk, dv=dv, workspace=ws_b)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert sa.bsa_get_status(ws_f) == 0 and sa.bsa_get_status(ws_b) == 0, "device status bits set"
    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize()
        sa.bsa_profile_enable(True)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        prof = sa.bsa_profile_collect()
        sa.bsa_profile_enable(False)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps)
    value = world * flops_step / (ms * 1e-3) / 1e12

    # end to end: pinned host inputs in, all outputs back, every step (copies on their own streams)
    pin = {t: x.pin_memory() for t, x in host.items()}
    outs = {"out": out, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
    h_out = {n_: torch.empty(x.shape, dtype=x.dtype).pin_memory() for n_, x in outs.items()}
    dev_in = [d, {t: torch.empty_like(x) for t, x in d.items()}]
    dev_out = [outs, {n_: torch.empty_like(x) for n_, x in outs.items()}]
    h2d = sum(x.numel() * x.element_size() for x in pin.values())
    d2h = sum(x.numel() * x.element_size() for x in h_out.values())

    def e2e_compute(x, o):
        sa.nsa_selected_fwd(x["q"], x["k"], x["v"], x["topk"], x["cu"], S, w.sel_block, w.mask_mode, w.scale,
                            out=o["out"], lse=o["lse"], workspace=ws_f)
        sa.nsa_selected_bwd(x["q"], x["k"], x["v"], o["out"], x["dout"], o["lse"], x["topk"], x["cu"], S,
                            w.sel_block, w.mask_mode, w.scale, dq=o["dq"], dk=o["dk"], dv=o["dv"], workspace=ws_b)

    e2e_ms = pipelined_e2e(args.steps, pin, dev_in, dev_out, h_out, e2e_compute, barrier, max_over_ranks)

    peaks, peak_src = measured_peaks()
    # forward 4*D per visible pair; dK/dV pass 8*D (S^T, dP^T, dV, dK); dQ pass 2*D (dQ; its S and dP
    # recompute what the dK/dV pass is credited with)
    # forward S, O; dK/dV pass S^T, dP^T, dV, dK; dQ pass dQ (its S and dP are recomputations)
    alg = {"nsa_fwd": 2 * (w.D + w.dv) * vpairs, "nsa_bwd_dkdv": (4 * w.D + 4 * w.dv) * vpairs,
           "nsa_bwd_dq": 2 * w.D * vpairs}
    if w.D != w.dv:  # 192-dim q / k: dK / dV run on the warp-level kernel
        alg["nsa_bwd_dkdv_warp"] = alg["nsa_bwd_dkdv"]
    peak, peak_desc = tensor_peak(peaks, peak_src, ms * args.steps)
    dom = max(prof.items(), key=lambda kv: kv[1][1])[0] if prof else None
    roof = None
    if dom in alg:
        launches, total = prof[dom]
        avg_ms = total / launches
        achieved = alg[dom] / (avg_ms * 1e-3) / 1e12
        traffic = ncu_traffic(dom, args.config)
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "peak_source": peak_desc, "traffic": traffic,
                "avg_launch_ms": avg_ms, "frac_of_burst": achieved / peaks["bf16_tflops"]}
    kernels = kernel_table(prof, alg, args.steps, peak)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, t, desc = cpu_oracle_sample_nsa(w, topk, budget_s=args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "cpu_model": cpu_model(),
               "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps({
            "metric": METRIC_NSA, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_dict_nsa(w, args),
            "e2e": {"value": world * flops_step / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": sum(c for c, _ in prof.values()), "kernels": kernels, "roofline": with_spec(roof),
            "cpu_baseline": cpu, "clocks": clocks.summary(), "visible_pairs": vpairs,
            "credited_flops_per_step": flops_step,
        }))


def run_decode(args, rank, world, local_rank):
    """Paged sparse decode workload (B=32, 128 heads, 65536-token cache, 32 pages of 64 selected):
    gathered-KV bandwidth against the HBM roofline.  Each timed rep is one CUDA-graph replay of the
    whole decode call (metadata, work list, decode, combine) after an L2 flush (256 MiB write)."""
    import torch

    import selected_attention_b200 as sa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.workload(4)
    table, idx = w.selection()
    seqused = np.full(w.B, w.context, np.int32)
    used = np.unique(table[np.arange(w.B)[:, None], idx[:, 0, 0, :]].ravel())
    caches = {}
    for tag, d in (("k", 512), ("k_rope", 64), ("v", 512)):
        t = torch.zeros((w.n_pages, w.page, 1, d), dtype=torch.bfloat16, device=dev)
        t[torch.from_numpy(used).long().to(dev)] = torch.from_numpy(w.pages(tag, used)).view(torch.bfloat16).to(dev)
        caches[tag] = t
    q = torch.from_numpy(w.query("q")).view(torch.bfloat16).to(dev)
    qr = torch.from_numpy(w.query("q_rope")).view(torch.bfloat16).to(dev)
    tb, ti, tu = (torch.from_numpy(x).to(dev) for x in (table, idx, seqused))
    p = sa.sfa_params(q, caches["k"], tb, ti, tu, w.sparse_block, w.scale)
    ws = torch.empty(sa.sfa_sparse_decode_workspace_size(p), dtype=torch.uint8, device=dev)
    out = torch.empty(w.B, 1, w.N1, w.D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(w.B, 1, w.N1, dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def call():
        sa.sfa_sparse_decode(q, qr, caches["k"], caches["k_rope"], caches["v"], tb, ti, tu, w.sparse_block,
                             w.scale, out=out, lse=lse, workspace=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    torch.cuda.synchronize()
    tokens = int(w.B * w.count * w.sparse_block)
    gathered = tokens * (w.D + w.Dr + w.D) * 2
    flops = tokens * w.N1 * 2 * (w.D + w.Dr + w.D)
    barrier, max_over_ranks = _dist_helpers(world, dev)
    times = []
    with ClockSampler(local_rank) as clocks:
        barrier()
        for _ in range(args.steps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        barrier()
    ms = max_over_ranks(float(np.mean(times)))
    assert sa.bsa_get_status(ws) == 0
    sa.bsa_profile_enable(True)
    for _ in range(3):
        flush.fill_(1)
        call()
    prof = sa.bsa_profile_collect()
    sa.bsa_profile_enable(False)
    launches_per_call = sum(c for c, _ in prof.values()) // 3

    # end to end through the API: each step copies the step's inputs (the query and its rope part,
    # the block table, the sparse indices, seqused) from pinned host memory and reads Out and LSE
    # back; the paged cache is resident device state, as in a serving loop
    h_in = {n_: x.cpu().pin_memory() for n_, x in (("q", q), ("qr", qr), ("tb", tb), ("ti", ti), ("tu", tu))}
    d_in = {n_: torch.empty_like(x) for n_, x in (("q", q), ("qr", qr), ("tb", tb), ("ti", ti), ("tu", tu))}
    h_out, h_lse = torch.empty(out.shape, dtype=out.dtype).pin_memory(), torch.empty(lse.shape).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in h_in.values())
    d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()

    def e2e_step():
        for n_ in d_in:
            d_in[n_].copy_(h_in[n_], non_blocking=True)
        sa.sfa_sparse_decode(d_in["q"], d_in["qr"], caches["k"], caches["k_rope"], caches["v"], d_in["tb"],
                             d_in["ti"], d_in["tu"], w.sparse_block, w.scale, out=out, lse=lse, workspace=ws)
        h_out.copy_(out, non_blocking=True)
        h_lse.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e2e_times = []
    barrier()
    for _ in range(args.steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e2e_times.append(e0.elapsed_time(e1))
    barrier()
    e2e_ms = max_over_ranks(float(np.mean(e2e_times)))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f_, t_, desc = cpu_oracle_sample_decode(w, budget_s=args.cpu_seconds)
        cpu = {"value": f_ / t_ / 1e9, "unit": "GB/s", "cores": cpu_threads(), "cpu_model": cpu_model(),
               "kind": "oracle", "sample": desc}
    peaks, src = measured_peaks()
    value = world * gathered / (ms * 1e-3) / 1e9  # every rank decodes its own copy of the batch
    dec_ms = prof["sfa_decode"][1] / prof["sfa_decode"][0] if "sfa_decode" in prof else None
    dec_gbs = gathered / (dec_ms * 1e-3) / 1e9 if dec_ms else None
    dec_traffic = ncu_traffic("sfa_decode", args.config)
    line = {
        "metric": METRIC_DEC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict_decode(w),
        "e2e": {"value": world * gathered / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_call * args.steps,
        "effective_tflops": world * flops / (ms * 1e-3) / 1e12,
        # dominant kernel: the decode kernel alone, its gathered bytes over its mean launch time
        "roofline": with_spec({"bound": "hbm", "kernel": "sfa_decode", "achieved": dec_gbs,
                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": dec_gbs / peaks["hbm_gbs"] if dec_gbs else None,
                               "peak_source": f"{src} hbm_gbs (burst)", "traffic": dec_traffic,
                               "avg_launch_ms": dec_ms}),
        "kernels": {n: {"launches": c, "ms_per_call": t / c} for n, (c, t) in prof.items()},
        "cpu_baseline": cpu, "clocks": clocks.summary(), "gathered_bytes_per_step": gathered,
    }
    if rank == 0:
        print(json.dumps(line))


def run_decode_bwd(args, rank, world, local_rank):
    """Backward of the paged sparse decode workload: each timed rep is one CUDA-graph replay of the
    whole backward call (page lists, readers of each cache row-block, preprocess, the token-major
    products, the dQ sum, the cache-row scatter) after an L2 flush.  Credited bytes: the gathered
    K, K_rope, V rows read and their gradient rows written."""
    import torch

    import selected_attention_b200 as sa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = synth.workload(4)
    if args.decode_batches:  # a smaller batch of the same problem (profiler captures)
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}_B{args.decode_batches}", B=args.decode_batches)
    table, idx = w.selection()
    seqused = np.full(w.B, w.context, np.int32)
    used = np.unique(table[np.arange(w.B)[:, None], idx[:, 0, 0, :]].ravel())
    caches, grads = {}, {}
    for tag, d in (("k", 512), ("k_rope", 64), ("v", 512)):
        t = torch.zeros((w.n_pages, w.page, 1, d), dtype=torch.bfloat16, device=dev)
        t[torch.from_numpy(used).long().to(dev)] = torch.from_numpy(w.pages(tag, used)).view(torch.bfloat16).to(dev)
        caches[tag] = t
        grads[tag] = torch.zeros_like(t)
    q = torch.from_numpy(w.query("q")).view(torch.bfloat16).to(dev)
    qr = torch.from_numpy(w.query("q_rope")).view(torch.bfloat16).to(dev)
    do = torch.from_numpy(decode_dout(w)).view(torch.bfloat16).to(dev)
    tb, ti, tu = (torch.from_numpy(x).to(dev) for x in (table, idx, seqused))
    out, lse = sa.sfa_sparse_decode(q, qr, caches["k"], caches["k_rope"], caches["v"], tb, ti, tu, w.sparse_block,
                                    w.scale)
    p = sa.sfa_params(q, caches["k"], tb, ti, tu, w.sparse_block, w.scale)
    ws = torch.empty(sa.sfa_sparse_decode_bwd_workspace_size(p), dtype=torch.uint8, device=dev)
    dq, dqr = torch.empty_like(q), torch.empty_like(qr)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def call(qq=q, qqr=qr, dd=do, oo=out, ll=lse, t_b=tb, t_i=ti, t_u=tu):
        sa.sfa_sparse_decode_bwd(qq, qqr, caches["k"], caches["k_rope"], caches["v"], oo, dd, ll, t_b, t_i, t_u,
                                 w.sparse_block, w.scale, dq=dq, dq_rope=dqr, dk_cache=grads["k"],
                                 dk_rope_cache=grads["k_rope"], dv_cache=grads["v"], workspace=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    torch.cuda.synchronize()
    tokens = int(w.B * w.count * w.sparse_block)
    moved = 2 * tokens * (w.D + w.Dr + w.D) * 2
    flops = tokens * w.N1 * 2 * (3 * (w.D + w.Dr) + 2 * w.D)
    barrier, max_over_ranks = _dist_helpers(world, dev)
    times = []
    with ClockSampler(local_rank) as clocks:
        barrier()
        for _ in range(args.steps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        barrier()
    ms = max_over_ranks(float(np.mean(times)))
    assert sa.bsa_get_status(ws) == 0
    sa.bsa_profile_enable(True)
    for _ in range(3):
        flush.fill_(1)
        call()
    prof = sa.bsa_profile_collect()
    sa.bsa_profile_enable(False)
    launches_per_call = sum(c for c, _ in prof.values()) // 3

    # end to end through the API: the step's query-side inputs (q, q_rope, dOut, Out, LSE and the
    # selection) come from pinned host memory and dQ, dQ_rope go back; the caches and their
    # gradients are resident device state
    named = (("q", q), ("qr", qr), ("do", do), ("o", out), ("l", lse), ("tb", tb), ("ti", ti), ("tu", tu))
    h_in = {n_: x.cpu().pin_memory() for n_, x in named}
    d_in = {n_: torch.empty_like(x) for n_, x in named}
    h_dq, h_dqr = torch.empty(dq.shape, dtype=dq.dtype).pin_memory(), torch.empty(dqr.shape, dtype=dqr.dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in h_in.values())
    d2h = h_dq.numel() * h_dq.element_size() + h_dqr.numel() * h_dqr.element_size()

    def e2e_step():
        for n_ in d_in:
            d_in[n_].copy_(h_in[n_], non_blocking=True)
        call(d_in["q"], d_in["qr"], d_in["do"], d_in["o"], d_in["l"], d_in["tb"], d_in["ti"], d_in["tu"])
        h_dq.copy_(dq, non_blocking=True)
        h_dqr.copy_(dqr, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    e2e_times = []
    barrier()
    for _ in range(args.steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        e2e_step()
        e1.record()
        torch.cuda.synchronize()
        e2e_times.append(e0.elapsed_time(e1))
    barrier()
    e2e_ms = max_over_ranks(float(np.mean(e2e_times)))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f_, t_, desc = cpu_oracle_sample_decode_bwd(w, budget_s=args.cpu_seconds)
        cpu = {"value": f_ / t_ / 1e9, "unit": "GB/s", "cores": cpu_threads(), "cpu_model": cpu_model(),
               "kind": "oracle", "sample": desc}
    peaks, src = measured_peaks()
    value = world * moved / (ms * 1e-3) / 1e9
    k_ms = prof["sfa_bwd"][1] / prof["sfa_bwd"][0] if "sfa_bwd" in prof else None
    line = {
        "metric": METRIC_DEC_BWD, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_dict_decode(w), op="backward"),
        "e2e": {"value": world * moved / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_call * args.steps,
        "effective_tflops": world * flops / (ms * 1e-3) / 1e12,
        # the token-major kernel reads the gathered rows; the scatter writes the gradient rows: the
        # roofline line credits the kernel with the reads, the step with both
        "roofline": with_spec({"bound": "hbm", "kernel": "sfa_bwd",
                               "achieved": (moved / 2) / (k_ms * 1e-3) / 1e9 if k_ms else None,
                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": (moved / 2) / (k_ms * 1e-3) / 1e9 / peaks["hbm_gbs"] if k_ms else None,
                               "peak_source": f"{src} hbm_gbs (burst)", "traffic": None, "avg_launch_ms": k_ms}),
        "kernels": {n: {"launches": c, "ms_per_call": t / c} for n, (c, t) in prof.items()},
        "cpu_baseline": cpu, "clocks": clocks.summary(), "bytes_per_step": moved,
    }
    if rank == 0:
        print(json.dumps(line))


def bsa_job(w, world, rank):
    """The rank's share of the block-sparse job.  With N ranks the job is N times the workload's
    batches (B * N batches under the workload's seed: weak scaling); bsa_partition cuts its
    (batch, kv head) slices into N contiguous ranges balanced by selected tiles, and each rank runs
    its range as contiguous BNSD pieces (b0, b1, g0, g1).  The slices are independent, so no
    collective runs on the data path.  With one rank the single piece is the whole workload.
    Returns (job workload, job mask, pieces, the cut)."""
    import dataclasses

    from selected_attention_b200 import shard
    wj = w if world == 1 else dataclasses.replace(w, name=f"{w.name}_x{world}", B=w.B * world)
    mask = wj.block_mask()
    starts, pieces = shard.split(mask, wj.N2, world, rank)
    return wj, mask, pieces, starts


def piece_tensor(wj, tag, b0, b1, h0, h1):
    """bf16 bits [b1 - b0, h1 - h0, S, D] of q/k/v/dout: the job's rows for batches b0..b1-1 and
    heads h0..h1-1, generated by row range (the same values as the whole tensor holds there)."""
    heads = wj.N1 if tag in ("q", "dout") else wj.N2
    rows = [synth.normal_rows_bf16(wj.seed, tag, wj.B * heads * wj.S, wj.D, wj.S, (b * heads + h0) * wj.S,
                                   (b * heads + h1) * wj.S) for b in range(b0, b1)]
    return np.concatenate(rows).reshape(b1 - b0, h1 - h0, wj.S, wj.D)


def run_ours(args, rank, world, local_rank):
    import torch

    import selected_attention_b200 as sa

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w0 = bsa_workload(args.config)
    w, mask_job, pieces, starts = bsa_job(w0, world, rank)
    G = w.N1 // w.N2
    bx = by = w.block
    barrier, max_over_ranks = _dist_helpers(world, dev)

    # per piece: host inputs, device inputs and outputs, workspaces
    P = []
    for b0, b1, g0, g1 in pieces:
        host = {t: torch.from_numpy(piece_tensor(w, t, b0, b1, *((g0 * G, g1 * G) if t in ("q", "dout") else
                                                                (g0, g1)))).view(torch.bfloat16)
                for t in ("q", "k", "v", "dout")}
        m = np.ascontiguousarray(mask_job[b0:b1, g0 * G:g1 * G])
        d = {t: host[t].to(dev) for t in host}
        d["mask"] = torch.from_numpy(m).to(dev)
        o = {"out": torch.empty_like(d["q"]), "lse": torch.empty(b1 - b0, (g1 - g0) * G, w.S, dtype=torch.float32,
                                                                  device=dev),
             "dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]), "dv": torch.empty_like(d["v"])}
        prm = sa.bsa_params(d["q"], d["k"], d["mask"], bx, by, w.mask_mode, w.scale)
        P.append({"host": host, "mask": m, "dev": d, "out": o, "vpairs": visible_pairs_bsa(m, bx, by, w.S, w.S),
                  "ws_f": torch.empty(sa.bsa_fwd_workspace_size(prm), dtype=torch.uint8, device=dev),
                  "ws_b": torch.empty(sa.bsa_bwd_workspace_size(prm), dtype=torch.uint8, device=dev)})
    vpairs = sum(x["vpairs"] for x in P)
    flops_rank = 14 * w.D * vpairs
    flops_job = sum_over_ranks(world, dev, flops_rank)
    stream = torch.cuda.current_stream()

    def compute(x, o, pc):
        sa.bsa_fwd(x["q"], x["k"], x["v"], x["mask"], bx, by, w.mask_mode, w.scale, out=o["out"], lse=o["lse"],
                   workspace=pc["ws_f"])
        sa.bsa_bwd(x["q"], x["k"], x["v"], o["out"], x["dout"], o["lse"], x["mask"], bx, by, w.mask_mode, w.scale,
                   dq=o["dq"], dk=o["dk"], dv=o["dv"], workspace=pc["ws_b"])

    def step():
        for pc in P:
            compute(pc["dev"], pc["out"], pc)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for pc in P:
        assert sa.bsa_get_status(pc["ws_f"]) == 0 and sa.bsa_get_status(pc["ws_b"]) == 0, "device status bits set"

    # ---- device-timed region: inputs resident in HBM
    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize()
        sa.bsa_profile_enable(True)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        prof = sa.bsa_profile_collect()
        sa.bsa_profile_enable(False)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps)
    value = flops_job / (ms * 1e-3) / 1e12
    sched = schedule_balance(sa, torch, step, dev)  # an extra, untimed step

    # ---- end to end through the public API with host buffers (pinned), copies timed, each on its
    # own stream and double-buffered against the compute
    pin, d0, outs = {}, {}, {}
    for i, pc in enumerate(P):
        for t, x in pc["host"].items():
            pin[f"{t}{i}"] = x.pin_memory()
        pin[f"mask{i}"] = torch.from_numpy(pc["mask"]).pin_memory()
        d0.update({f"{t}{i}": x for t, x in pc["dev"].items()})
        outs.update({f"{n}{i}": x for n, x in pc["out"].items()})
    h_out = {n: torch.empty(x.shape, dtype=x.dtype).pin_memory() for n, x in outs.items()}
    dev_in = [d0, {t: torch.empty_like(x) for t, x in d0.items()}]
    dev_out = [outs, {n: torch.empty_like(x) for n, x in outs.items()}]
    h2d = sum(x.numel() * x.element_size() for x in pin.values())
    d2h = sum(x.numel() * x.element_size() for x in h_out.values())

    def e2e_compute(x, o):
        for i, pc in enumerate(P):
            compute({t: x[f"{t}{i}"] for t in ("q", "k", "v", "dout", "mask")},
                    {n: o[f"{n}{i}"] for n in ("out", "lse", "dq", "dk", "dv")}, pc)

    e2e_ms = pipelined_e2e(args.steps, pin, dev_in, dev_out, h_out, e2e_compute, barrier, max_over_ranks)

    # ---- roofline of the dominant kernel
    peaks, peak_src = measured_peaks()
    # forward 4*D per visible pair (S, O); KV-major pass 8*D (S^T, dP^T, dV, dK); Q-major pass 2*D (dQ;
    # its S and dP recompute what the KV pass is credited with): 14*D in all
    alg = {"bsa_fwd": 4 * w.D * vpairs, "bsa_bwd_kv": 8 * w.D * vpairs, "bsa_bwd_q": 2 * w.D * vpairs}
    peak, peak_desc = tensor_peak(peaks, peak_src, ms * args.steps)
    dom = max(prof.items(), key=lambda kv: kv[1][1])[0] if prof else None
    roof = None
    if dom in alg:
        launches, total = prof[dom]
        avg_ms = total / launches
        achieved = alg[dom] / len(P) / (avg_ms * 1e-3) / 1e12  # a launch's average share of the work
        traffic = ncu_traffic(dom, args.config) if world == 1 else None
        roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "peak_source": peak_desc, "traffic": traffic, "avg_launch_ms": avg_ms,
                "frac_of_burst": achieved / peaks["bf16_tflops"]}
    kernels = kernel_table(prof, {n: f / len(P) for n, f in alg.items()}, args.steps, peak)
    launches_total = sum(c for c, _ in prof.values())

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, t, desc = cpu_oracle_sample(w, mask_job, budget_s=args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(), "cpu_model": cpu_model(),
               "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(w, args),
            "e2e": {"value": flops_job / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": launches_total, "kernels": kernels, "roofline": with_spec(roof), "cpu_baseline": cpu,
            "clocks": clocks.summary(), "visible_pairs": vpairs, "credited_flops_per_step": flops_job,
            "schedule": sched,
        }
        if world > 1:
            line["shard"] = {"slice_cut": [int(x) for x in starts], "rank0_pieces": [list(x) for x in pieces]}
        print(json.dumps(line))


def source_sha1(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=5, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--nsa-seqlens", default="", help="config 3 only: comma-separated batch lengths")
    ap.add_argument("--decode-bwd", action="store_true", help="config 4 only: time the decode's backward")
    ap.add_argument("--nsa-dqk", type=int, default=128, choices=[128, 192],
                    help="config 3 only: head dim of q / k (v keeps 128)")
    ap.add_argument("--decode-batches", type=int, default=0, help="--decode-bwd only: fewer batches (profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.config == 4 and args.decode_bwd:
            run_decode_bwd(args, rank, world, local_rank)
        elif args.config == 4:
            run_decode(args, rank, world, local_rank)
        elif args.config == 3:
            run_nsa(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
