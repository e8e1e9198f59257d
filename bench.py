#!/usr/bin/env python
"""Benchmark of the MLA decode layer step on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload v2|v2_fp8|lite|lite_fp8|long|prefill] [--no-cpu-baseline] [--no-extra]

--gpus N must match the ranks torch.distributed.run launched (WORLD_SIZE);
started without it and N > 1, bench.py launches the N ranks itself.

A step is one pass of the whole hot path over one batch: compress_append ->
absorb_q -> decode attention (+ LSE combine) -> out_proj, through the C ABI.
Default workload: the DeepSeek-V2-shaped layer, decode batch 64 with cache
lengths uniform in [1, 8192] on a randomly permuted page table.  Its cache
(302 MB) and weights (298 MB) exceed the 126 MB L2, so no flush is needed
between steps.  Under torchrun each rank runs an independent replica (the
decode batch shards by sequence; no collective on the data path).

After the headline workload the same run measures the other shapes of the
scope (V2-Lite decode, 131072-token long-context decode, chunked prefill) and
adds one block per workload to the same JSON line ("workloads"): tokens/s,
ms per step, the attention roofline against its binding roof; the headline
fields are not affected (--no-extra skips them).

--impl reference times the fp64 CPU oracle (the reference arm of this
comparison) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MLA decode tokens/s (1 B200) and achieved % of HBM / bf16 tensor roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOAD_TEXT = {
    "v2": "DeepSeek-V2-shaped MLA layer (d=5120, n_h=128, d_h=128, d_c=512, d_c'=1536, d_h^R=64), bf16, "
          "decode batch 64, prior cache lengths uniform in [1,8192], block 64, permuted page table",
    "lite": "DeepSeek-V2-Lite-shaped MLA layer (d=2048, n_h=16, d_h=128, d_c=512, d_h^R=64), bf16, "
            "decode batch 32, 4096 prior tokens each, block 64",
    "v2_fp8": "the V2 workload over an FP8 latent cache (E4M3 codes of c^KV with a power-of-two scale per row, "
              "bf16 k^R: 656 bytes per token), bf16 compute",
    "lite_fp8": "the V2-Lite workload over an FP8 latent cache (E4M3 codes of c^KV with a power-of-two scale "
                "per row, bf16 k^R: 656 bytes per token), bf16 compute",
    "long": "V2-shaped MLA layer, bf16, decode batch 4 over 131072 prior tokens each, YaRN s=40, split-KV",
    "prefill": "V2-shaped MLA layer, bf16, chunked prefill: 8 sequences x 4096 new tokens over 4096 cached",
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="mla_clocks_", suffix=".csv")
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, n = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                n += 1
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": n}


def physical_gpu_index(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v.strip() for v in vis.split(",") if v.strip()]
    if ids and all(v.isdigit() for v in ids) and local < len(ids):
        return int(ids[local])
    return local


def attention_sources(workload: str):
    """The sources the workload's attention kernel is built from: the CTA-pair
    kernel (128 heads) also takes tc_attn2.cuh."""
    from head_latent_attention_03_b200 import inputs as I
    pair = I.WORKLOADS[workload].dims.n_h == 128
    return ("common.cuh", "tc_attn.cuh") + (("tc_attn2.cuh",) if pair else ())


def kernel_source_hash(workload: str) -> str:
    """Hash of every source the workload's attention kernel is built from."""
    h = hashlib.sha256()
    for name in attention_sources(workload):
        with open(os.path.join(ROOT, "head_latent_attention_03_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def attention_tokens_per_s(world: int, rows: int, attn_ms: float):
    """Decode tokens/s of the attention stage alone (plan + attention + LSE
    combine, one call per step), whole job: every rank's rows per call time."""
    return round(world * rows / (attn_ms * 1e-3), 1) if attn_ms > 0 else None


def committed_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu summary, if it was
    taken on the current source of that kernel; else None."""
    p = os.path.join(ROOT, "profiles", "attn_dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_source_sha256_16") != kernel_source_hash(workload):
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# work accounting (algorithmic, per attention launch)
# ---------------------------------------------------------------------------
def cache_row_bytes(dims) -> int:
    """Bytes of one cached row: [c^KV | k^R] in bf16 (1152 at d_c 512, d_h^R 64),
    or the FP8 row (E4M3 codes, bf16 k^R, fp32 scale, padded to 16 bytes: 656)."""
    if getattr(dims, "cache_dtype", "bf16") == "fp8":
        return (dims.d_c + 2 * dims.d_hr + 4 + 15) // 16 * 16
    return dims.row * 2


def attention_work(dims, kv_len, rows):
    """Bytes that must move and FLOPs of one attention launch (absorbed form)."""
    tok = int(sum(kv_len))
    bytes_ = tok * cache_row_bytes(dims) + rows * dims.n_h * dims.row * 2 + rows * dims.n_h * dims.d_c * 2
    flops = tok * 2 * dims.n_h * (2 * dims.d_c + dims.d_hr)
    return bytes_, flops


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_oracle_baseline(w, seconds: float = 12.0):
    """Time the fp64 oracle (un-absorbed form) on whole sequences of the workload
    until `seconds` have passed; tokens/s = decoded tokens / time."""
    import numpy as np
    from head_latent_attention_03_b200 import inputs as I
    from oracle import mla_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([p.get("num_threads", 1) for p in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        cores = os.cpu_count() or 1
    W = I.gen_weights(w)
    lens = I.prior_lengths(w)
    order = list(range(w.batch))
    done, t_total, toks = 0, 0.0, 0
    for b in order:
        batch = I.gen_batch(w, seqs=[b])
        t0 = time.perf_counter()
        if w.new_tokens == 1:
            O.decode_batch(batch, W, absorbed=False)
            toks += 1
        else:
            D = w.dims
            prior = O.gather_rows(batch.pool, batch.block_table[0], int(batch.prior_len[0]), D.block_size)
            O.prefill_sequence(D, W, batch.h[:1], int(batch.prior_len[0]), prior, [0], absorbed=False)
            toks += 1
        t_total += time.perf_counter() - t0
        done += 1
        if t_total >= seconds:
            break
    sample = (f"{done} whole sequence(s) of the workload (cache lengths {[int(lens[b]) for b in order[:done]]}), "
              f"fp64 un-absorbed oracle (eqs 9-11 then MHA), numpy BLAS")
    return {"value": toks / t_total, "unit": "tokens/s", "cores": int(cores), "kind": "oracle", "sample": sample,
            "cpu_model": cpu_model(), "host_cores": os.cpu_count()}


def roofline_of(attn_bytes, attn_flops, attn_ms, peaks, peak_src):
    """Attention roofline: achieved against the binding roof (the larger of
    bytes / HBM peak and FLOPs / bf16 peak)."""
    hbm = float(peaks["hbm_gbs"])
    tensor = float(peaks["bf16_tflops"])
    achieved_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9
    achieved_tf = attn_flops / (attn_ms * 1e-3) / 1e12
    t_hbm, t_tensor = attn_bytes / (hbm * 1e9), attn_flops / (tensor * 1e12)
    if t_hbm >= t_tensor:
        roof = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved_gbs / hbm, 4)}
    else:
        roof = {"bound": "tensor", "achieved": round(achieved_tf, 1), "peak": tensor, "unit": "TFLOP/s",
                "frac": round(achieved_tf / tensor, 4)}
    roof.update({"peak_source": f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else "fallback",
                 "other_roof": {"hbm_frac": round(achieved_gbs / hbm, 4), "tensor_frac": round(achieved_tf / tensor, 4),
                                "attn_bytes_per_launch": attn_bytes, "attn_flops_per_launch": attn_flops,
                                "attn_us": round(attn_ms * 1e3, 2)}})
    return roof


def workload_work(w, batch):
    """Algorithmic attention bytes and FLOPs of one step of workload w.  Decode
    reads every cached row once per sequence; a prefill chunk reads each of its
    sequences' rows once (all its queries share them) and does the causal
    query x key products of the latent form."""
    rows = batch.h.shape[0]
    if w.new_tokens == 1:
        return attention_work(w.dims, batch.prior_len + 1, rows)
    D = w.dims
    per_q = [int(L) + q + 1 for L in batch.prior_len for q in range(w.new_tokens)]
    _, flops = attention_work(D, per_q, rows)
    cached = int(sum(int(L) + w.new_tokens for L in batch.prior_len))
    bytes_ = cached * D.row * 2 + rows * D.n_h * D.row * 2 + rows * D.n_h * D.d_c * 2
    return bytes_, flops


def unabsorbed_work(w, batch):
    """Algorithmic bytes and FLOPs of the un-absorbed prefill attention: the
    per-head products 2 n_h (2 d_h + d_h^R) per (query, key) pair plus the
    decompression of every cached row (2 x 2 n_h d_h d_c); bytes = the cached
    rows, q^C, q^R and o once."""
    from head_latent_attention_03_b200.layer import prefill_flops
    D = w.dims
    flops = prefill_flops(D, batch.prior_len, w.new_tokens)["unabsorbed"]
    rows = batch.h.shape[0]
    cached = int(sum(int(L) + w.new_tokens for L in batch.prior_len))
    bytes_ = cached * D.row * 2 + rows * D.n_h * (2 * D.d_h + D.d_hr) * 2
    return bytes_, flops


def measure_extra(name, steps, warmup, dev, peaks, peak_src):
    """One more workload of the scope in the same run: whole-step and
    attention-stage device times (CUDA events, max over ranks).  A prefill
    chunk runs in the form with fewer FLOPs (layer.cheaper_prefill_form)."""
    import torch
    from head_latent_attention_03_b200 import inputs as I, mla
    from head_latent_attention_03_b200.layer import MLALayer, cheaper_prefill_form
    w = I.WORKLOADS[name]
    batch = I.gen_batch(w)
    layer = MLALayer(w.dims, I.gen_weights(w), device=str(dev))
    st = layer.upload(batch)
    rows = st.h.shape[0]
    form = cheaper_prefill_form(w.dims, batch.prior_len, w.new_tokens) if w.new_tokens > 1 else "absorbed"
    if form == "unabsorbed":
        attn_bytes, attn_flops = unabsorbed_work(w, batch)
        layer.prefill_buffers(st)
        calls = [lambda: layer.compress_append(st),
                 lambda: mla.queries(layer.desc, layer.cw, st.h, st.pos, st.q_c, st.q_rope, st.ws)]
        attend = lambda: mla.prefill_attn_unabsorbed(layer.desc, layer.cw, st.q_c, st.q_rope, layer.cache(st),
                                                     st.q_start, st.new_per_seq, st.ws_pf, st.o, st.lse)
        after = lambda: mla.out_proj_unabsorbed(layer.desc, layer.cw, st.o, st.u)
    else:
        attn_bytes, attn_flops = workload_work(w, batch)
        calls = [lambda: layer.compress_append_absorb_q(st)]
        attend = lambda: layer.attend(st)
        after = lambda: layer.out_proj(st)
    stream = torch.cuda.current_stream()

    def one(k=None):
        for f in calls:
            f()
        if k is not None:
            ev[k][0].record(stream)
        attend()
        if k is not None:
            ev[k][1].record(stream)
        after()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    code = mla.get_last_error()
    if code != 0:
        raise RuntimeError(f"{name}: device status after warm-up: {mla.status_string(code)}")
    # whole steps back to back (the throughput), then steps with events around
    # the attention stage, then (latent form) around the attention kernel alone
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(steps):
        one()
    e1.record(stream)
    for k in range(steps):
        one(k)
    kern = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if form == "absorbed":
        for a, b in kern:  # create the events
            a.record(stream)
            b.record(stream)
        for k in range(steps):
            mla.debug_attention_events(*kern[k])
            one()
        mla.debug_attention_events(None, None)
    torch.cuda.synchronize()
    code = mla.get_last_error()
    if code != 0:
        raise RuntimeError(f"{name}: device status after timed steps: {mla.status_string(code)}")
    t_ms = e0.elapsed_time(e1)
    attn_ms = sum(a.elapsed_time(b) for a, b in ev) / steps
    kern_ms = sum(a.elapsed_time(b) for a, b in kern) / steps if form == "absorbed" else 0.0
    t_ms, attn_ms, kern_ms = max_over_ranks([t_ms, attn_ms, kern_ms], dev)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    out = {"workload": WORKLOAD_TEXT[name], "value": round(world * rows * steps / (t_ms * 1e-3), 1),
           "unit": "tokens/s", "steps": steps, "warmup": warmup, "ms_per_step": round(t_ms / steps, 4),
           "roofline": roofline_of(attn_bytes, attn_flops, attn_ms, peaks, peak_src)}
    out["roofline"]["traffic"] = committed_traffic(name) if form == "absorbed" else None
    if form == "absorbed" and kern_ms > 0:
        # the attention kernel alone is the roofline; the stage beside it
        kname = "mla_attn_pair_kernel" if w.dims.n_h == 128 else "mla_attn_kernel"
        stage = out["roofline"]
        out["roofline"] = roofline_of(attn_bytes, attn_flops, kern_ms, peaks, peak_src)
        out["roofline"].update({"traffic": stage.pop("traffic"), "kernel": f"{kname} alone (library-recorded events)"})
        out["roofline"]["stage"] = {"us": round(attn_ms * 1e3, 2), "bound": stage["bound"], "achieved": stage["achieved"],
                                    "unit": stage["unit"], "frac": stage["frac"],
                                    "tokens_per_s": attention_tokens_per_s(world, rows, attn_ms)}
    if w.new_tokens > 1:
        out["form"] = form
        if form == "unabsorbed":
            # the latent form of the same chunk, for comparison (attention only)
            lat_bytes, lat_flops = workload_work(w, batch)
            torch.cuda.synchronize()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            layer.absorb_q(st)
            a0.record(stream)
            layer.attend(st)
            a1.record(stream)
            torch.cuda.synchronize()
            (lat_ms,) = max_over_ranks([a0.elapsed_time(a1)], dev)
            out["latent_form_attention"] = {"attn_ms": round(lat_ms, 3),
                                            "roofline": roofline_of(lat_bytes, lat_flops, lat_ms, peaks, peak_src)}
    del layer, st
    torch.cuda.empty_cache()
    return out


# Steps of the extra workloads (their steps are longer than the headline's).
EXTRA_STEPS = {"lite": (100, 5), "lite_fp8": (100, 5), "v2_fp8": (100, 5), "long": (20, 3), "prefill": (2, 1)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def max_over_ranks(values, device):
    """Element-wise max of per-rank timings over the process group (the
    slowest rank times the job); the values themselves without one."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from head_latent_attention_03_b200 import build, inputs as I, mla
    from head_latent_attention_03_b200.layer import MLALayer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    build.build()
    dev = torch.device("cuda", torch.cuda.current_device())

    w = I.WORKLOADS[args.workload]
    W = I.gen_weights(w)
    batch = I.gen_batch(w)
    layer = MLALayer(w.dims, W, device=str(dev))
    st = layer.upload(batch)
    rows = st.h.shape[0]
    attn_bytes, attn_flops = workload_work(w, batch)
    stream = torch.cuda.current_stream()

    def step(ev_pair=None):
        layer.compress_append_absorb_q(st)
        if ev_pair is not None:
            ev_pair[0].record(stream)
        layer.attend(st)
        if ev_pair is not None:
            ev_pair[1].record(stream)
        layer.out_proj(st)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    code = mla.get_last_error()
    if code != 0:
        raise RuntimeError(f"device status after warm-up: {mla.status_string(code)}")

    sampler = ClockSampler(physical_gpu_index(local))
    if not args.profile_run:
        sampler.start()
        # keep the GPU busy while the sampler spins up so its samples fall under load
        t_pre = time.time()
        while time.time() - t_pre < 0.6:
            step()
    def pairs(n):
        return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]

    # (1) the headline: K whole steps back to back, nothing between the kernels
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = mla.launch_count()
    e0.record(stream)
    for k in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    n_launch = mla.launch_count() - n0
    if world > 1:
        dist.barrier()
    # (2) the attention stage (plan + attention kernel + combine) of each step,
    # between events, and (3) the attention kernel alone, between events the
    # library records around it (mla_debug_attention_events)
    attn_ev, kern_ev = pairs(args.steps), pairs(args.steps)
    for a, b in kern_ev:  # create the events
        a.record(stream)
        b.record(stream)
    for k in range(args.steps):
        step(attn_ev[k])
    for k in range(args.steps):
        mla.debug_attention_events(*kern_ev[k])
        step()
    mla.debug_attention_events(None, None)
    torch.cuda.synchronize()
    clocks = sampler.stop() if not args.profile_run else {"sm_mhz": None, "sm_max_mhz": None,
                                                          "reasons": ["not sampled (profile run)"]}
    code = mla.get_last_error()
    if code != 0:
        raise RuntimeError(f"device status after timed steps: {mla.status_string(code)}")
    t_ms = e0.elapsed_time(e1)
    attn_ms = sum(a.elapsed_time(b) for a, b in attn_ev) / args.steps
    kern_ms = sum(a.elapsed_time(b) for a, b in kern_ev) / args.steps
    t_ms, attn_ms, kern_ms = max_over_ranks([t_ms, attn_ms, kern_ms], dev)

    # end to end through the public API: pinned host inputs in, result out, every step
    h_host = st.h.cpu().pin_memory()
    pos_host = st.pos.cpu().pin_memory()
    seq_host = st.seq_idx.cpu().pin_memory()
    kv_host = st.kv_len.cpu().pin_memory()
    u_host = torch.empty(st.u.shape, dtype=st.u.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_host, pos_host, seq_host, kv_host))
    d2h = u_host.numel() * u_host.element_size()

    # Two step states share the cache, the page table and the workspace but
    # have their own input and output buffers, so that while step k runs its
    # kernels the inputs of step k+1 cross to the device and the result of
    # step k-1 comes back (copy engines on their own streams).  Every step
    # still copies its own inputs in and its result out.
    import dataclasses as _dc
    st2 = _dc.replace(st, h=torch.empty_like(st.h), pos=torch.empty_like(st.pos),
                      seq_idx=torch.empty_like(st.seq_idx), kv_len=torch.empty_like(st.kv_len),
                      u=torch.empty_like(st.u))
    states = (st, st2)
    u_hosts = (u_host, torch.empty(st.u.shape, dtype=st.u.dtype).pin_memory())
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    in_free = [torch.cuda.Event() for _ in range(2)]
    out_ready = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n, start=None):
        if start is not None:
            s_in.wait_event(start)
            s_out.wait_event(start)
        for k in range(n):
            b = k & 1
            sk = states[b]
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(in_free[b])  # step k-2 has read these inputs
                sk.h.copy_(h_host, non_blocking=True)
                sk.pos.copy_(pos_host, non_blocking=True)
                sk.seq_idx.copy_(seq_host, non_blocking=True)
                sk.kv_len.copy_(kv_host, non_blocking=True)
                in_ready[b].record(s_in)
            stream.wait_event(in_ready[b])
            if k >= 2:
                stream.wait_event(out_done[b])  # step k-2's result has left this buffer
            layer.step(sk)
            in_free[b].record(stream)
            out_ready[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(out_ready[b])
                u_hosts[b].copy_(sk.u, non_blocking=True)
                out_done[b].record(s_out)
        for b in range(min(n, 2)):
            stream.wait_event(out_done[b])

    e2e_steps = 0 if args.profile_run else args.steps
    if e2e_steps:
        e2e_run(3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    e2e_run(e2e_steps, start=f0)
    f1.record(stream)
    torch.cuda.synchronize()
    (t_e2e,) = max_over_ranks([max(f0.elapsed_time(f1), 1e-9)], dev)
    if world > 1:
        dist.barrier()

    peaks, peak_src = load_peaks()
    extra = {}
    if not args.no_extra and not args.profile_run:
        del layer, st
        torch.cuda.empty_cache()
        for name in ("lite", "lite_fp8", "v2_fp8", "long", "prefill"):
            if name != args.workload:
                k, wu = EXTRA_STEPS[name]
                extra[name] = measure_extra(name, k, wu, dev, peaks, peak_src)

    if rank == 0:
        traffic = committed_traffic(args.workload)
        attn_kernel = "mla_attn_pair_kernel" if w.dims.n_h == 128 else "mla_attn_kernel"
        # the dominant kernel: the attention kernel alone, between CUDA events
        # the library records on its launch stream around every launch
        roof = roofline_of(attn_bytes, attn_flops, kern_ms, peaks, peak_src)
        roof.update({"traffic": traffic,
                     "kernel": f"{attn_kernel}: algorithmic bytes per launch / its average launch duration, CUDA "
                               f"events the library records on the launch stream around it ({args.steps} steps of "
                               f"their own after the timed steps); traffic: ncu DRAM bytes per launch"})
        st_roof = roofline_of(attn_bytes, attn_flops, attn_ms, peaks, peak_src)
        roof["stage"] = {"what": f"mla_attn_plan_kernel + {attn_kernel} + mla_combine_kernel between events around "
                                 f"the attention call", "us": round(attn_ms * 1e3, 2), "bound": st_roof["bound"],
                         "achieved": st_roof["achieved"], "unit": st_roof["unit"], "frac": st_roof["frac"],
                         "tokens_per_s": attention_tokens_per_s(world, rows, attn_ms)}
        value = world * rows * args.steps / (t_ms * 1e-3)
        e2e_value = world * rows * e2e_steps / (t_e2e * 1e-3) if e2e_steps else None
        out = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(t_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1/fan_in) weights, N(0,1) hidden states and prior latents)",
            "config": {"workload": WORKLOAD_TEXT[args.workload], "tokens_per_step_per_gpu": rows,
                       "l2": "inputs exceed L2 (cache + weights > 126 MB), no flush",
                       "parallelism": f"{world} independent replica(s), sequences sharded, no collective"},
            "roofline": roof,
            "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
            "e2e": {"value": round(e2e_value, 1) if e2e_value else None, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "copies": "pinned host buffers; each step's inputs in and u out on their own streams, "
                              "double-buffered, overlapping the neighbouring steps' kernels"},
            "gpu_launches": int(n_launch),
            "impl": "ours",
        }
        if extra:
            out["workloads"] = extra
        if world == 1 and not args.no_cpu_baseline and not args.profile_run:
            out["cpu_baseline"] = cpu_oracle_baseline(w)
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    from head_latent_attention_03_b200 import inputs as I
    from oracle import mla_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([p.get("num_threads", 1) for p in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        cores = os.cpu_count() or 1
    w = I.WORKLOADS[args.workload]
    W = I.gen_weights(w)
    lens = I.prior_lengths(w)
    # each step decodes one whole sequence of the workload (its new token over
    # its full cache), cycling through the batch in order
    order = list(range(w.batch)) if w.new_tokens == 1 else [0]
    batches = {}

    def one(i):
        b = order[i % len(order)]
        if b not in batches:
            batches[b] = I.gen_batch(w, seqs=[b])
        bt = batches[b]
        if w.new_tokens == 1:
            O.decode_batch(bt, W, absorbed=False)
        else:
            D = w.dims
            prior = O.gather_rows(bt.pool, bt.block_table[0], int(bt.prior_len[0]), D.block_size)
            O.prefill_sequence(D, W, bt.h[:1], int(bt.prior_len[0]), prior, [0], absorbed=False)

    for i in range(max(3, args.warmup)):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(max(3, args.warmup) + i)
    t = time.perf_counter() - t0
    value = args.steps / t
    sample = (f"each step = one sequence's decode token over its whole cache (fp64 un-absorbed oracle), cycling "
              f"the {len(order)} sequences of the workload in order")
    out = {"metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": int(os.environ.get(
        "WORLD_SIZE", "1")), "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(t / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT[args.workload]}, "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["v2", "v2_fp8", "lite", "lite_fp8", "long", "prefill"], default="v2")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="only the headline workload")
    ap.add_argument("--profile-run", action="store_true",
                    help="only the timed device steps (for ncu launch lists): no clock sampling, e2e or CPU leg")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world:
        if "RANK" not in os.environ and args.gpus > 1:
            # one process per GPU: start the ranks under torch.distributed.run
            import socket
            with socket.socket() as s:
                s.bind(("127.0.0.1", 0))
                port = s.getsockname()[1]
            cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
                   "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
            sys.exit(subprocess.call(cmd))
        sys.exit(f"bench.py: --gpus {args.gpus} but {world} rank(s) were launched")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
