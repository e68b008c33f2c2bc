#!/usr/bin/env python3
"""Benchmark of the paged-attention hot path on B200.

One step = one pass of the whole hot path over one batch: pa_kv_write of the
step's new K/V rows, then pa_attention_mixed (plan, decode with its split-KV
merge, prefill as the batch needs).  The headline workload is the Llama-3-8B-shaped
decode batch (256 requests, context U[512, 4096], 32 q / 8 kv heads, head_dim
128, 70k-block pool); the metric is KV bytes the attention must read per
second (sum over requests of seq_len * Hkv * D * 2 tensors * 2 bytes, exact
tokens).  The mixed 8192-token step (192 decodes + prefill chunks) is timed
too and reported as tokens/s under "mixed_step".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): replicas only -- every rank runs its own copy of the
workload on its own GPU, no collective on the data path; the step time is the
max over ranks (weak scaling).  --impl reference times the fp64 CPU oracle on
a bounded sample of the same workload (the only reference this method has).
"""
from __future__ import annotations

import argparse
import atexit
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode paged-attn KV GB/s (% of HBM peak); mixed-step tokens/s on 1 B200"
HEADLINE = "llama3_8b_decode"
MIXED = "mixed_step_8192"
PROFILES = os.path.join(ROOT, "profiles")


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _kernel_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "paged_kv_cache_461_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic(name, files):
    """DRAM bytes per launch from a committed ncu summary, if the kernel is unchanged since."""
    p = os.path.join(PROFILES, f"{name}.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        d = json.load(f)
    if d.get("source_hash") != _kernel_hash(files):
        return None, d
    return d.get("dram_bytes_per_launch"), d


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampled every period_ms in the background; stop() keeps the samples that
    arrived inside the timed window (host monotonic clock)."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, period_ms: int = 10):
        self.rows = []
        self.proc = None
        self.first = threading.Event()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            atexit.register(self._kill)  # never leave the sampler running if the bench ends early
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            self.first.wait(timeout=5.0)
        except OSError:
            self.proc = None

    def _kill(self):
        p = self.proc
        if p is not None and p.poll() is None:
            p.terminate()
            try:
                p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                p.kill()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 7:
                self.rows.append((time.monotonic(), parts))
                self.first.set()

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.05)
        self._kill()
        self.t.join(timeout=2)
        inside = [r for ts, r in self.rows if t0 <= ts <= t1 + 0.02]
        note = "samples inside the timed region"
        if not inside:  # region shorter than the sampling period: take the samples bracketing it
            after = [r for ts, r in self.rows if ts >= t0][:2]
            before = [r for ts, r in self.rows if ts < t0][-1:]
            inside = before + after
            note = "timed region shorter than the sampling period; nearest samples"
        num = lambda v: v.replace(".", "", 1).isdigit()
        sm = [float(r[0]) for r in inside if num(r[0])]
        mx = [float(r[1]) for r in inside if num(r[1])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i in range(4) if r[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside), "note": note}


# --------------------------------------------------------------------------- distributed plumbing

def _dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return ws, rank, local


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, ws: int) -> float:
    """Slowest rank's value (NCCL on GPUs, gloo on CPU-only process groups)."""
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(bytes_per_rank: float, ms_per_step_local: float, ws: int) -> tuple:
    """(value, ms_per_step): every rank processes its own replica; the job's step time is the max over ranks."""
    ms = _max_over_ranks(ms_per_step_local, ws)
    return ws * bytes_per_rank / (ms * 1e-3) / 1e9, ms


def job_config(lay, n_gpus: int) -> dict:
    """The `config` object of both arms: the workload and how the job is laid out, nothing arm-specific."""
    return {**lay.describe(), "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single device",
            "step": "KV write of the step's new rows + attention over the whole batch"}


# --------------------------------------------------------------------------- our arm

class Step:
    """Device-resident inputs of one workload and the hot-path call sequence."""

    def __init__(self, name: str, seed=None):
        import torch

        from paged_kv_cache_461_b200 import api
        from paged_kv_cache_461_b200 import workloads as W
        self.api = api
        self.lay = W.workload_layout(name, seed)
        self.vals = W.make_values_torch(self.lay, "cuda")
        lay = self.lay
        d = "cuda"
        self.qsl = torch.from_numpy(lay.query_start_loc).to(d)
        self.seq_lens = torch.from_numpy(lay.seq_lens).to(d)
        self.bt = torch.from_numpy(lay.block_table).to(d)
        self.slots = torch.from_numpy(lay.slot_mapping).to(d)
        self.out = torch.empty_like(self.vals.q)
        self.ws = api.alloc_workspace(lay.num_seqs, lay.num_tokens, lay.num_q_heads, self.vals.k_cache, lay.max_seq_len)
        self.scale = 1.0 / math.sqrt(lay.head_dim)
        G = lay.num_q_heads // lay.num_kv_heads
        NT = 1 if G <= 8 else (2 if G <= 16 else 0)
        cap = 8 * NT
        # the KV write with the plan (one launch), decode (split merge inside), prefill when the batch has
        # prefill work
        self.launches_per_step = 1 + (1 if NT else 0) + (1 if lay.max_query_len * G > cap else 0)
        self.kv_bytes = lay.kv_bytes()
        q = lay.q_lens.astype(np.int64)
        c = lay.ctx_lens.astype(np.int64)
        pf = q * lay.num_q_heads // lay.num_kv_heads > cap
        # causal (query, key) pairs of prefill rows: sum_i (c + i + 1)
        pairs = (q * c + q * (q + 1) // 2)[pf].sum()
        self.prefill_flops = float(pairs) * 4 * lay.num_q_heads * lay.head_dim
        self.prefill_requests = np.nonzero(pf)[0]

    def kv_write(self):
        v = self.vals
        self.api.kv_write(v.k_new, v.v_new, self.slots, v.k_cache, v.v_cache)

    def attention(self):
        lay, v = self.lay, self.vals
        self.api.attention_mixed(v.q, v.k_cache, v.v_cache, self.qsl, self.seq_lens, self.bt, lay.max_query_len,
                                 lay.max_seq_len, softmax_scale=self.scale, out=self.out, workspace=self.ws)

    def step(self):
        """One step of the hot path through the public API: pa_attention_mixed_write writes the step's new K/V
        (in the launch that also plans the step) and attends; the same as kv_write() then attention(), bit
        for bit, one launch fewer."""
        lay, v = self.lay, self.vals
        self.api.attention_mixed_write(v.q, v.k_new, v.v_new, self.slots, v.k_cache, v.v_cache, self.qsl,
                                       self.seq_lens, self.bt, lay.max_query_len, lay.max_seq_len,
                                       softmax_scale=self.scale, out=self.out, workspace=self.ws)


def _time_region(fn, steps, warmup, ws, window=None):
    """W untimed steps, then EXACTLY `steps` steps between barrier+sync on both sides.
    `window` (a list) receives the host monotonic times bracketing the timed region."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    _barrier(ws)
    stream = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    h0 = time.monotonic()
    t0.record(stream)
    for _ in range(steps):
        fn()
    t1.record(stream)
    torch.cuda.synchronize()
    h1 = time.monotonic()
    _barrier(ws)
    if window is not None:
        window[:] = [h0, h1]
    return t0.elapsed_time(t1)


def _attention_only_ms(st: Step, steps: int):
    """Average duration of the attention launches inside a step loop (events on the launching stream)."""
    import torch
    stream = torch.cuda.current_stream()
    evs = []
    for _ in range(steps):
        st.kv_write()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        st.attention()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def _window(fn, seconds: float = 0.3, min_steps: int = 50):
    """Back-to-back steps for about `seconds` (at least min_steps), each bracketed by its own CUDA events on the
    launching stream: (median ms, mean ms, steps, host seconds)."""
    import torch
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(5):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    n = max(min_steps, int(seconds * 1e3 / max(a.elapsed_time(b) / 5, 1e-3)))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    h0 = time.monotonic()
    for e0, e1 in evs:
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize()
    h1 = time.monotonic()
    ms = [e0.elapsed_time(e1) for e0, e1 in evs]
    return statistics.median(ms), statistics.mean(ms), n, h1 - h0


def _kv_write_alone(st: "Step", peaks: dict, launches: int = 100):
    """pa_kv_write of the mixed step's 8192 new tokens on its own, back to back: launches cycle through four
    input sets (the step's own new rows and slots, and three more 8192-token sets whose slots come from the
    same workload drawn with other seeds), so the rows read and the slots written (4 x 64 MB) exceed L2
    (126 MB) and every launch goes to HBM.  CUDA events around the whole loop; per-launch time = total / launches.
    Also the median of single launches, each after a 256 MB read that leaves L2 cold and clean.  The extra sets
    overwrite cache slots of the step's pool, so this runs after everything else that uses that pool.
    Algorithmic bytes: the new K and V rows read once and written once."""
    import torch
    from paged_kv_cache_461_b200 import workloads as W
    lay, v = st.lay, st.vals
    sets = [(v.k_new, v.v_new, st.slots)]
    for seed in (13, 23, 33):
        other = W.workload_layout(lay.name, seed)
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        kn = torch.randn(v.k_new.shape, generator=g, device="cuda").to(torch.bfloat16)
        vn = torch.randn(v.v_new.shape, generator=g, device="cuda").to(torch.bfloat16)
        sets.append((kn, vn, torch.from_numpy(other.slot_mapping).cuda()))
    valid = int((lay.slot_mapping >= 0).sum())
    moved = 2 * 2 * valid * lay.num_kv_heads * lay.head_dim * 2   # (K, V) x (read, write) x bf16
    run = lambda i: st.api.kv_write(sets[i % 4][0], sets[i % 4][1], sets[i % 4][2], v.k_cache, v.v_cache)
    for i in range(8):
        run(i)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(launches):
        run(i)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / launches
    flush = torch.zeros(64 << 20, dtype=torch.float32, device="cuda")
    cold = []
    for i in range(20):
        flush.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run(i)
        e1.record(stream)
        e1.synchronize()
        cold.append(e0.elapsed_time(e1))
    # size-matched reference: a plain device copy (torch's copy kernel) of the same K and V rows into four
    # rotating contiguous destinations, back to back -- what moving these bytes costs without the scatter
    dst = [(torch.empty_like(v.k_new), torch.empty_like(v.v_new)) for _ in range(4)]
    copy = lambda i: (dst[i % 4][0].copy_(sets[i % 4][0]), dst[i % 4][1].copy_(sets[i % 4][1]))
    for i in range(8):
        copy(i)
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for i in range(launches):
        copy(i)
    c1.record(stream)
    torch.cuda.synchronize()
    copy_ms = c0.elapsed_time(c1) / launches
    del flush, sets, dst
    gbs = moved / (ms * 1e-3) / 1e9
    return {"ms_per_launch": ms, "launches": launches, "tokens": valid, "bytes_read_plus_written": moved,
            "value": gbs, "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
            "l2": "back to back over 4 input sets of 64 MB each (more than L2)",
            "ms_single_cold_launch": statistics.median(cold),
            "same_bytes_device_copy": {"ms": copy_ms, "value": moved / (copy_ms * 1e-3) / 1e9, "unit": "GB/s",
                                       "frac_of_it": copy_ms / ms,
                                       "what": "torch copy_ of the same K and V rows into 4 rotating contiguous "
                                               "buffers, back to back (two copy kernels per set)"},
            "workload": lay.name}, launches + 28


def _prefill_only_call(st: Step):
    """pa_attention_mixed on the prefill chunks of the mixed step alone, as a prefill-only batch
    (decode_max_query_len = -1: the prefill kernel alone, no decode grid beside it)."""
    import torch
    from paged_kv_cache_461_b200 import workloads as W
    lay = st.lay
    idx = st.prefill_requests
    qsl = lay.query_start_loc
    rows = np.concatenate([np.arange(qsl[r], qsl[r + 1]) for r in idx])
    sub = W.StepLayout("prefill_only", lay.num_q_heads, lay.num_kv_heads, lay.head_dim, lay.num_blocks,
                       lay.q_lens[idx], lay.ctx_lens[idx], lay.block_table[idx])
    q = st.vals.q[torch.from_numpy(rows).cuda()].contiguous()
    qsl_d = torch.from_numpy(sub.query_start_loc).cuda()
    sl_d = torch.from_numpy(sub.seq_lens).cuda()
    bt_d = torch.from_numpy(sub.block_table).cuda()
    out = torch.empty_like(q)
    ws = st.api.alloc_workspace(sub.num_seqs, sub.num_tokens, sub.num_q_heads, st.vals.k_cache, sub.max_seq_len,
                                decode_max_query_len=-1)

    def call():
        st.api.attention_mixed(q, st.vals.k_cache, st.vals.v_cache, qsl_d, sl_d, bt_d, sub.max_query_len,
                               sub.max_seq_len, softmax_scale=st.scale, out=out, workspace=ws,
                               decode_max_query_len=-1)
    return call


def _prefill_burst(call, launches: int, warmup: int):
    """`launches` prefill-only launches back to back (a few ms), timed with events: the figure that compares
    with the burst GEMM peak.  Taken before the mixed steps are timed: their tensor-heavy run leaves the power
    manager holding the clocks lower for a while."""
    import torch
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(launches):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / launches


def _prefill_sustained(call, ms_hint: float):
    """About 0.3 s of prefill-only launches back to back, timed with events and sampled for SM clocks:
    the run reaches the power cap, so it compares with the sustained GEMM peak."""
    import torch
    n = max(20, int(300.0 / max(ms_hint, 1e-3)))
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(torch.cuda.current_device())
    h0 = time.monotonic()
    a.record(stream)
    for _ in range(n):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    h1 = time.monotonic()
    return a.elapsed_time(b) / n, n, sampler.stop(h0, h1)


def _e2e(st: Step, steps: int, warmup: int):
    """Same metric through the public API with host buffers: every step copies its inputs from pinned
    host memory (q, new K/V, metadata), runs the step's C-ABI call and reads its output back, all inside
    the timed region.  Steps are pipelined the way a serving loop runs them: double-buffered device
    inputs/outputs, step i+1's inputs copied on an H2D stream and step i-1's output on a D2H stream
    while step i computes."""
    import torch
    v = st.vals
    host = {k: t.cpu().pin_memory() for k, t in
            (("q", v.q), ("k_new", v.k_new), ("v_new", v.v_new), ("slots", st.slots), ("qsl", st.qsl),
             ("seq_lens", st.seq_lens), ("bt", st.bt))}
    dev = [{k: torch.empty_like(t, device="cuda") for k, t in host.items()} for _ in range(2)]
    out_d = [torch.empty_like(st.out) for _ in range(2)]
    out_h = [torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory() for _ in range(2)]
    lay = st.lay
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h[0].numel() * out_h[0].element_size()
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    e_in, e_comp, e_out = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def copy_in(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(e_comp[b])          # step i-2 is done with these buffers
            for k in host:
                dev[b][k].copy_(host[k], non_blocking=True)
            e_in[b].record(s_in)

    def run(n):
        copy_in(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                copy_in(i + 1)
            comp.wait_event(e_in[b])
            if i >= 2:
                comp.wait_event(e_out[b])           # step i-2's output has been read back
            d = dev[b]
            st.api.attention_mixed_write(d["q"], d["k_new"], d["v_new"], d["slots"], v.k_cache, v.v_cache,
                                         d["qsl"], d["seq_lens"], d["bt"], lay.max_query_len, lay.max_seq_len,
                                         softmax_scale=st.scale, out=out_d[b], workspace=st.ws)
            e_comp[b].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_comp[b])
                out_h[b].copy_(out_d[b], non_blocking=True)
                e_out[b].record(s_out)
        for b in range(2):
            comp.wait_event(e_out[b])
    run(warmup)
    torch.cuda.synchronize()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    s_in.wait_stream(comp)
    run(steps)
    z.record(comp)
    torch.cuda.synchronize()
    ms = a.elapsed_time(z) / steps
    # the last output read back equals the device result
    assert torch.equal(out_h[(steps - 1) % 2].view(torch.int16), out_d[(steps - 1) % 2].cpu().view(torch.int16))
    return ms, h2d, d2h


def _follow_on(st: Step, steps: int, warmup: int, peaks: dict):
    """The follow-on operations on the headline decode batch: KV write fused into the decode kernel,
    decode over a token-major (NHD) cache, and whole-block pack / unpack of every block the batch's
    requests hold.  Events on the launching stream, as for the headline."""
    import torch
    api, lay, v = st.api, st.lay, st.vals
    hbm = peaks["hbm_gbs"]
    res, launches = {}, 0

    def fused():
        api.attention_decode_fused(v.q, v.k_new, v.v_new, v.k_cache, v.v_cache, st.qsl, st.seq_lens, st.bt,
                                   lay.max_query_len, lay.max_seq_len, softmax_scale=st.scale, out=st.out,
                                   workspace=st.ws)
    ms_sep = _time_region(st.step, steps, warmup, 1) / steps
    ms_fused = _time_region(fused, steps, warmup, 1) / steps
    launches += (2 * st.launches_per_step - 1) * steps
    res["fused_kv_write_decode"] = {
        "value": st.kv_bytes / (ms_fused * 1e-3) / 1e9, "unit": "GB/s", "frac": st.kv_bytes / (ms_fused * 1e-3) / 1e9 / hbm,
        "ms_per_step": ms_fused, "ms_per_step_write_then_attend": ms_sep,
        "launches_per_step": st.launches_per_step - 1, "launches_per_step_write_then_attend": st.launches_per_step}

    kn, vn = v.k_cache.transpose(1, 2).contiguous(), v.v_cache.transpose(1, 2).contiguous()
    ws_n = api.alloc_workspace(lay.num_seqs, lay.num_tokens, lay.num_q_heads, kn, lay.max_seq_len, layout="NHD")

    def nhd():
        api.attention_mixed(v.q, kn, vn, st.qsl, st.seq_lens, st.bt, lay.max_query_len, lay.max_seq_len,
                            softmax_scale=st.scale, out=st.out, workspace=ws_n, layout="NHD")
    ms_n = _time_region(nhd, steps, warmup, 1) / steps
    ms_h = _time_region(st.attention, steps, warmup, 1) / steps
    launches += 2 * (st.launches_per_step - 1) * steps
    res["nhd_decode"] = {"value": st.kv_bytes / (ms_n * 1e-3) / 1e9, "unit": "GB/s",
                         "frac": st.kv_bytes / (ms_n * 1e-3) / 1e9 / hbm, "ms_per_launch": ms_n,
                         "ms_per_launch_hnd": ms_h, "layout": "[num_blocks, 16, num_kv_heads, head_dim]"}
    del kn, vn, ws_n
    torch.cuda.empty_cache()

    nblk = (lay.seq_lens + 15) // 16
    ids = np.concatenate([lay.block_table[r, :n] for r, n in enumerate(nblk)]).astype(np.int32)
    ids_d = torch.from_numpy(ids).cuda()
    elems = lay.num_kv_heads * 16 * lay.head_dim
    staging = torch.empty((len(ids), 2, elems), dtype=torch.bfloat16, device="cuda")
    moved = 2 * staging.numel() * 2            # every staged byte is read once and written once
    ms_pack = _time_region(lambda: api.kv_pack(v.k_cache, v.v_cache, ids_d, staging), steps, warmup, 1) / steps
    # unpack the staged blocks back over the same blocks (same bytes, same traffic as a fresh pool)
    ms_unpack = _time_region(lambda: api.kv_unpack(staging, ids_d, v.k_cache, v.v_cache), steps, warmup, 1) / steps
    launches += 2 * steps
    res["kv_pack"] = {"value": moved / (ms_pack * 1e-3) / 1e9, "unit": "GB/s",
                      "frac": moved / (ms_pack * 1e-3) / 1e9 / hbm, "ms_per_launch": ms_pack, "blocks": len(ids),
                      "bytes_read_plus_written": moved}
    res["kv_unpack"] = {"value": moved / (ms_unpack * 1e-3) / 1e9, "unit": "GB/s",
                        "frac": moved / (ms_unpack * 1e-3) / 1e9 / hbm, "ms_per_launch": ms_unpack,
                        "blocks": len(ids), "bytes_read_plus_written": moved}
    res["peak"] = {"hbm_gbs": hbm, "source": f"{peaks['source']} hbm_gbs (burst copy)"}
    del staging
    torch.cuda.empty_cache()

    # speculative verification: the same requests, each scoring k = 3 drafted tokens plus the last
    # accepted one (q_len 4, 16 packed rows per kv head) in one pass
    from paged_kv_cache_461_b200 import workloads as W
    sl = W.build_layout("spec_verify_k3", lay.ctx_lens, np.full(lay.num_seqs, 4, np.int32),
                        num_q_heads=lay.num_q_heads, num_kv_heads=lay.num_kv_heads, head_dim=lay.head_dim,
                        num_blocks=lay.num_blocks, seed=lay.seed)
    sv = W.make_values_torch(sl, "cuda")
    sq = {k: torch.from_numpy(a).cuda() for k, a in (("qsl", sl.query_start_loc), ("sl", sl.seq_lens),
                                                       ("bt", sl.block_table), ("slots", sl.slot_mapping))}
    api.kv_write(sv.k_new, sv.v_new, sq["slots"], sv.k_cache, sv.v_cache)
    s_out = torch.empty_like(sv.q)
    ws_dec = api.alloc_workspace(sl.num_seqs, sl.num_tokens, sl.num_q_heads, sv.k_cache, sl.max_seq_len,
                                 decode_max_query_len=4)
    ws_pf = api.alloc_workspace(sl.num_seqs, sl.num_tokens, sl.num_q_heads, sv.k_cache, sl.max_seq_len)

    def spec(dq, wsp):
        return lambda: api.attention_mixed(sv.q, sv.k_cache, sv.v_cache, sq["qsl"], sq["sl"], sq["bt"],
                                           sl.max_query_len, sl.max_seq_len, out=s_out, workspace=wsp,
                                           decode_max_query_len=dq)
    ms_dec = _time_region(spec(4, ws_dec), steps, warmup, 1) / steps
    ms_pf = _time_region(spec(0, ws_pf), steps, warmup, 1) / steps
    launches += 5 * steps  # plan + decode; plan + decode (no work) + prefill
    kvb = sl.kv_bytes()
    res["spec_verify_k3"] = {"value": kvb / (ms_dec * 1e-3) / 1e9, "unit": "GB/s",
                             "frac": kvb / (ms_dec * 1e-3) / 1e9 / hbm, "ms_per_launch": ms_dec,
                             "tokens_per_s": sl.num_tokens / (ms_dec * 1e-3),
                             "ms_per_launch_through_prefill_kernel": ms_pf,
                             "workload": {**sl.describe(), "q_len": 4, "decode_max_query_len": 4}}
    del sv, s_out, ws_dec, ws_pf
    torch.cuda.empty_cache()
    return res, launches


def _other_workloads(steps: int, warmup: int, peaks: dict):
    """The long-context decode batch (split-KV with the in-kernel merge) and the prefix-sharing batch
    (128 requests whose first 128 blocks are the same physical blocks): attention call only, CUDA events.
    Prefix sharing reports the logical KV bytes the requests attend over and the unique bytes HBM must
    deliver (the shared blocks are read once from HBM, then from L2)."""
    import torch
    res = {}
    for name in ("long_context_decode", "prefix_sharing"):
        st = Step(name)
        st.kv_write()
        ms = _time_region(st.attention, steps, warmup, 1) / steps
        lay = st.lay
        logical = lay.kv_bytes()
        d = {"ms_per_launch": ms, "value": logical / (ms * 1e-3) / 1e9, "unit": "GB/s",
             "frac": logical / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "workload": lay.describe()}
        if name == "prefix_sharing":
            # unique tokens: the shared 2048-token prefix once plus every private suffix
            shared = 2048
            uniq_tokens = shared + int((lay.seq_lens - shared).sum())
            unique = uniq_tokens * lay.num_kv_heads * lay.head_dim * 2 * 2
            d.update({"value_unique": unique / (ms * 1e-3) / 1e9,
                      "frac_unique": unique / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                      "unique_kv_bytes": unique, "logical_kv_bytes": logical})
        res[name] = d
        del st
        torch.cuda.empty_cache()
    return res, 2 * 2 * steps  # plan + decode per call, two workloads


def _prefix_hash_rate():
    """Host-side prefix caching on the prefix-sharing workload's shape (128 requests, 2048 shared prompt
    tokens plus private suffixes, synthetic token ids): chained block hashing of every request and the
    longest-hit walk of every request after all were inserted.  One host thread."""
    from paged_kv_cache_461_b200 import api
    from paged_kv_cache_461_b200 import workloads as W
    lay = W.workload_layout("prefix_sharing")
    rng = np.random.default_rng(5)
    shared = rng.integers(0, 128256, size=2048).astype(np.int32)
    reqs = [np.concatenate([shared, rng.integers(0, 128256, size=int(L) - 2048).astype(np.int32)])
            for L in lay.seq_lens]
    n_tok = sum(len(t) for t in reqs)
    res = {"requests": len(reqs), "tokens": n_tok, "threads": 1, "where": "host (C++ in libpa_b200.so)"}
    for algo in ("fnv1a64", "sha256"):
        t0 = time.perf_counter()
        hs = [api.prefix_block_hashes(t, algo) for t in reqs]
        dt = time.perf_counter() - t0
        res[f"{algo}_tokens_per_s"] = n_tok / dt
        res[f"{algo}_blocks_per_s"] = sum(len(h) for h in hs) / dt
    cache = api.PrefixCache()
    hs = [api.prefix_block_hashes(t) for t in reqs]
    for r, h in enumerate(hs):
        cache.insert(h, lay.block_table[r, :len(h)])
    t0 = time.perf_counter()
    hits = sum(len(cache.longest_hit(h)) for h in hs)
    dt = time.perf_counter() - t0
    res["longest_hit_blocks_per_s"] = hits / dt
    res["longest_hit_calls_per_s"] = len(hs) / dt
    cache.close()
    return res


# --------------------------------------------------------------------------- CPU oracle leg

def _oracle_sample(name: str, n_requests: int, seed=None):
    """A bounded sample of the workload (first n requests) as host arrays for the oracle."""
    from paged_kv_cache_461_b200 import workloads as W
    lay = W.workload_layout(name, seed)
    idx = np.arange(min(n_requests, lay.num_seqs))
    sub = W.build_layout(name + "_sample", lay.ctx_lens[idx], lay.q_lens[idx], num_q_heads=lay.num_q_heads,
                         num_kv_heads=lay.num_kv_heads, head_dim=lay.head_dim, seed=lay.seed)
    vals = W.make_values_numpy(sub)
    return sub, vals


def cpu_oracle_run(name: str, target_s: float = 15.0, seed=None):
    """Time the oracle (as it stands) on a request sample sized for about target_s of CPU work."""
    import oracle
    from paged_kv_cache_461_b200 import workloads as W
    full = W.workload_layout(name, seed).num_seqs

    def run(n):
        sub, vals = _oracle_sample(name, n, seed)
        kc, vc = oracle.kv_write(vals.k_new, vals.v_new, sub.slot_mapping, vals.k_cache, vals.v_cache)
        t0 = time.perf_counter()
        oracle.attention_for(sub, kc, vc, vals.q)
        return sub, (kc, vc, vals.q), time.perf_counter() - t0

    sub, arrs, dt = run(min(8, full))
    n = int(min(full, max(sub.num_seqs, sub.num_seqs * target_s / max(dt, 1e-3))))
    if n > sub.num_seqs:
        sub, arrs, dt = run(n)
    cores = oracle.num_cores()

    # the same oracle on one thread, over the queries of the first m requests (about 3 s)
    def kv_bytes_of(m):
        return int(sub.seq_lens[:m].astype(np.int64).sum()) * sub.num_kv_heads * sub.head_dim * 2 * 2

    def run1(m):
        toks = np.arange(int(sub.query_start_loc[m]), dtype=np.int32)
        t0 = time.perf_counter()
        oracle.attention_for(sub, *arrs, token_list=toks, nthreads=1)
        return time.perf_counter() - t0

    m = min(2, sub.num_seqs)
    dt1 = run1(m)
    m2 = int(min(sub.num_seqs, max(m, m * 3.0 / max(dt1, 1e-3))))
    if m2 > m:
        m, dt1 = m2, run1(m2)
    return {"value": sub.kv_bytes() / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"first {sub.num_seqs} of the {full} requests of {name} "
                      f"({sub.kv_bytes() / 1e9:.3f} GB of KV, {dt:.2f} s, fp64, {cores} threads)",
            "single_thread": {"value": kv_bytes_of(m) / dt1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"queries of the first {m} requests of {name} "
                                        f"({kv_bytes_of(m) / 1e9:.3f} GB of KV, {dt1:.2f} s, fp64, 1 thread)"},
            "cpu_model": _cpu_model()}


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def reference_arm(args, ws, rank):
    """The reference arm: the fp64 oracle, as it stands, on this machine's host cores, over the whole workload
    (every request).  Rank 0 alone runs it (other ranks exit without work).  Each timed step is one oracle
    attention pass over the batch; the oracle's KV write (a pure function that returns copies of both pools)
    runs once before the steps and is timed on its own, outside the steps."""
    if rank != 0:
        return
    import oracle
    from paged_kv_cache_461_b200 import workloads as W
    full = W.workload_layout(args.workload)
    n_req = full.num_seqs if args.reference_requests <= 0 else min(args.reference_requests, full.num_seqs)
    sub, vals = _oracle_sample(args.workload, n_req)
    t0 = time.perf_counter()
    kc, vc = oracle.kv_write(vals.k_new, vals.v_new, sub.slot_mapping, vals.k_cache, vals.v_cache)
    write_s = time.perf_counter() - t0

    def step():
        oracle.attention_for(sub, kc, vc, vals.q)

    t0 = time.perf_counter()
    for _ in range(args.warmup):                      # untimed warm-up, bounded in time
        step()
        if time.perf_counter() - t0 > 30:
            break
    t_steps = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        t_steps.append(time.perf_counter() - t0)
        if sum(t_steps) > 120:
            break
    dt = statistics.mean(t_steps)
    v = sub.kv_bytes() / dt / 1e9
    cores = oracle.num_cores()
    which = f"all {sub.num_seqs}" if sub.num_seqs == full.num_seqs else f"the first {sub.num_seqs} of {full.num_seqs}"
    sample = f"{which} requests of {args.workload} ({sub.kv_bytes() / 1e9:.3f} GB of KV), each step one " \
             f"oracle attention pass (fp64, {cores} threads); the oracle's KV write timed once outside the steps"
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": len(t_steps),
            "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": job_config(full, args.gpus),
            "oracle_kv_write_ms": write_s * 1e3,
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample,
                             "cpu_model": _cpu_model()},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- small cases for ncu captures

def profile_case(kind: str, launches: int):
    """A reduced copy of a workload for ncu (same shapes, fewer requests, pool sized to fit):
    decode: the first 64 requests of the Llama-3-8B-shaped decode batch (~0.6 GB of KV, above L2);
    spec: the same 64 requests verifying 3 drafted tokens each (q_len 4, decode_max_query_len 4);
    prefill: the prefill chunks of the mixed 8192-token step alone;
    kvwrite: pa_kv_write of the mixed step's 8192 new tokens (pool sized to its requests, ~2 GB per cache);
    pack: pa_kv_pack of every block of the headline batch's first 64 requests.
    Runs 1 warm-up launch of pa_attention_mixed and then `launches` more."""
    import torch

    from paged_kv_cache_461_b200 import api, build
    from paged_kv_cache_461_b200 import workloads as W
    build.build()
    if kind in ("kvwrite", "pack"):
        # the mixed step's 8192-token KV write / whole-block pack of the headline batch's first 64 requests
        # (a pool sized to the requests' blocks, so the capture holds a few GB at most)
        lay = W.workload_layout(MIXED if kind == "kvwrite" else HEADLINE)
        idx = np.arange(64) if kind == "pack" else np.arange(lay.num_seqs)
        lay = W.build_layout(f"{lay.name}_{kind}_case", lay.ctx_lens[idx], lay.q_lens[idx],
                             num_q_heads=lay.num_q_heads, num_kv_heads=lay.num_kv_heads, head_dim=lay.head_dim,
                             seed=lay.seed)
        v = W.make_values_torch(lay, "cuda")
        slots = torch.from_numpy(lay.slot_mapping).cuda()
        nblk = (lay.seq_lens + 15) // 16
        ids = torch.from_numpy(np.concatenate([lay.block_table[r, :n] for r, n in enumerate(nblk)]).astype(np.int32)).cuda()
        staging = torch.empty((len(ids), 2, lay.num_kv_heads * 16 * lay.head_dim), dtype=torch.bfloat16, device="cuda")
        for _ in range(1 + launches):
            if kind == "kvwrite":
                api.kv_write(v.k_new, v.v_new, slots, v.k_cache, v.v_cache)
            else:
                api.kv_pack(v.k_cache, v.v_cache, ids, staging)
        torch.cuda.synchronize()
        print(json.dumps({"profile_case": kind, **lay.describe(), "blocks": len(ids),
                          "bytes_moved": 2 * staging.numel() * 2 if kind == "pack" else
                          4 * int((lay.slot_mapping >= 0).sum()) * lay.num_kv_heads * lay.head_dim * 2}))
        return
    full = W.workload_layout(MIXED if kind == "prefill" else HEADLINE)
    if kind in ("decode", "spec"):
        idx = np.arange(64)
    else:
        G = full.num_q_heads // full.num_kv_heads
        idx = np.nonzero(full.q_lens * G > 8)[0]
    q_lens = np.full(len(idx), 4, np.int32) if kind == "spec" else full.q_lens[idx]
    lay = W.build_layout(f"{full.name}_{kind}_case", full.ctx_lens[idx], q_lens,
                         num_q_heads=full.num_q_heads, num_kv_heads=full.num_kv_heads, head_dim=full.head_dim,
                         seed=full.seed)
    v = W.make_values_torch(lay, "cuda")
    qsl = torch.from_numpy(lay.query_start_loc).cuda()
    sl = torch.from_numpy(lay.seq_lens).cuda()
    bt = torch.from_numpy(lay.block_table).cuda()
    slots = torch.from_numpy(lay.slot_mapping).cuda()
    api.kv_write(v.k_new, v.v_new, slots, v.k_cache, v.v_cache)
    # the prefill chunks as a prefill-only batch, as bench.py times them; verify shapes on the decode kernel
    dq = {"prefill": -1, "spec": 4}.get(kind, 0)
    ws = api.alloc_workspace(lay.num_seqs, lay.num_tokens, lay.num_q_heads, v.k_cache, lay.max_seq_len,
                             decode_max_query_len=dq)
    out = torch.empty_like(v.q)
    for _ in range(1 + launches):
        api.attention_mixed(v.q, v.k_cache, v.v_cache, qsl, sl, bt, lay.max_query_len, lay.max_seq_len,
                            out=out, workspace=ws, decode_max_query_len=dq)
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": kind, **lay.describe(), "kv_bytes": lay.kv_bytes(),
                      "pool_bytes": 2 * v.k_cache.numel() * 2}))


def _summary(line: dict) -> dict:
    """The headline numbers of every part of the line in one short object, printed last."""
    r = lambda x, n=4: None if x is None else round(float(x), n)
    out = {"headline_gbs": r(line["value"], 1), "headline_frac": r(line["roofline"]["frac"]),
           "headline_ms_median": r(line["window"]["ms_per_step_median"], 5)}
    m = line.get("mixed_step")
    if m:
        out.update({"mixed_ms": r(m["ms_per_step"], 5), "mixed_tok_s": r(m["value"], 0),
                    "prefill_tflops": r(m["prefill_roofline"]["achieved"], 1),
                    "prefill_frac": r(m["prefill_roofline"]["frac"]),
                    "prefill_sustained_tflops": r(m["prefill_roofline"]["sustained"]["achieved"], 1),
                    "prefill_sustained_frac": r(m["prefill_roofline"]["sustained"]["frac"])})
    w = line.get("kv_write")
    if w:
        out.update({"kv_write_gbs": r(w["value"], 1), "kv_write_frac": r(w["frac"]),
                    "kv_write_vs_same_bytes_copy": r(w["same_bytes_device_copy"]["frac_of_it"])})
    f = line.get("follow_on")
    if f:
        for k, short in (("fused_kv_write_decode", "fused"), ("nhd_decode", "nhd"), ("kv_pack", "pack"),
                         ("kv_unpack", "unpack"), ("spec_verify_k3", "spec_k3")):
            if k in f:
                out[f"{short}_gbs"] = r(f[k]["value"], 1)
                out[f"{short}_frac"] = r(f[k]["frac"])
    o = line.get("other_workloads")
    if o:
        for k, short in (("long_context_decode", "long_ctx"), ("prefix_sharing", "prefix")):
            if k in o:
                out[f"{short}_gbs"] = r(o[k]["value"], 1)
                out[f"{short}_frac"] = r(o[k]["frac"])
    if "e2e" in line:
        out["e2e_gbs"] = r(line["e2e"]["value"], 1)
    if "cpu_baseline" in line:
        out["cpu_oracle_gbs"] = r(line["cpu_baseline"]["value"], 3)
    return out


# --------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-requests", type=int, default=0,
                    help="reference arm: time only the first N requests (0 = the whole workload)")
    ap.add_argument("--no-extras", action="store_true", help="headline only (no mixed step, e2e, prefill)")
    ap.add_argument("--profile-case", choices=["decode", "spec", "prefill", "kvwrite", "pack"],
                    help="run a small case of one kernel for an ncu capture and exit")
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case, args.steps)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"

    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        reference_arm(args, ws, rank)
        return

    import torch
    ws, rank, local = _dist_init()
    torch.cuda.set_device(local)
    from paged_kv_cache_461_b200 import build
    if rank == 0 or ws == 1:
        build.build()
    _barrier(ws)
    peaks = _peaks()

    st = Step(args.workload)
    sampler = ClockSampler(local)
    win = []
    ms_total = _time_region(st.step, args.steps, args.warmup, ws, window=win)
    # dominant kernel roofline: the attention launches (plan + decode with its split merge), events on their
    # stream, right after the timed steps (before the long window below warms the GPU into its power cap)
    att_steps = max(50, min(args.steps, 200))
    att_ms = _attention_only_ms(st, att_steps)
    # the same step back to back for about 0.3 s, each step on its own events: the median per-step time, and
    # enough clock samples to see the clocks the timed steps ran at
    w_med, w_mean, w_n, w_s = _window(st.step)
    clocks = sampler.stop(win[0], time.monotonic())
    clocks["note"] = "samples over the timed region, the attention-only launches and the 0.3 s window of the " \
                     "same step after them"
    value, ms_step = whole_job_value(st.kv_bytes, ms_total / args.steps, ws)

    achieved = st.kv_bytes / (att_ms * 1e-3) / 1e9
    traffic, _ = _traffic("decode_llama3_8b_decode", ["decode.cu", "ptx.cuh", "pa_internal.cuh"])
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "kernel": "pa_attention_mixed (plan_kernel + decode_kernel with its split merge)",
                "algorithmic_bytes_per_launch": st.kv_bytes, "ms_per_launch": att_ms,
                "peak_source": f"{peaks['source']} hbm_gbs (burst copy)"}

    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": job_config(st.lay, ws),
            "l2": f"inputs larger than L2 ({st.kv_bytes / 1e9:.2f} GB of KV read per step), no flush",
            "calls_per_step": "pa_attention_mixed_write (the KV write and the plan in one launch, then attention)",
            "window": {"ms_per_step_median": w_med, "ms_per_step_mean": w_mean, "steps": w_n, "seconds": w_s,
                       "value_median": ws * st.kv_bytes / (w_med * 1e-3) / 1e9},
            "roofline": roofline,
            "gpu_launches": st.launches_per_step * (args.steps + w_n + args.warmup) + (st.launches_per_step + 1) * att_steps,
            "clocks": clocks}

    if not args.no_extras:
        # every rank runs its replica end to end; the job's step time is the slowest rank's
        _barrier(ws)
        e_ms, h2d, d2h = _e2e(st, max(10, min(args.steps, 100)), args.warmup)
        e_val, e_ms = whole_job_value(st.kv_bytes, e_ms, ws)
        line["e2e"] = {"value": e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
                       "note": "pinned host buffers; every step's H2D and D2H inside the timed region, double-"
                               "buffered so step i+1's inputs and step i-1's output move while step i computes"}
    if not args.no_extras and rank == 0:
        line["follow_on"], n_l = _follow_on(st, max(10, min(args.steps, 50)), args.warmup, peaks)
        line["follow_on"]["prefix_hash"] = _prefix_hash_rate()
        line["other_workloads"], n_o = _other_workloads(max(10, min(args.steps, 30)), args.warmup, peaks)
        line["gpu_launches"] += n_o
        line["gpu_launches"] += n_l
    if not args.no_extras:
        del st
        torch.cuda.empty_cache()
        mx = Step(MIXED)
        pf_call = _prefill_only_call(mx)
        pf_ms = _prefill_burst(pf_call, 20, max(3, args.warmup))
        mk = max(10, min(args.steps, 100))
        m_ms = _max_over_ranks(_time_region(mx.step, mk, args.warmup, ws), ws) / mk
        pf_sus_ms, pf_sus_n, pf_clocks = _prefill_sustained(pf_call, pf_ms)
        pf_tf = mx.prefill_flops / (pf_ms * 1e-3) / 1e12
        pf_sus_tf = mx.prefill_flops / (pf_sus_ms * 1e-3) / 1e12
        line["mixed_step"] = {
            "value": ws * mx.lay.num_tokens / (m_ms * 1e-3), "unit": "tokens/s", "ms_per_step": m_ms,
            "workload": mx.lay.describe(), "kv_bytes_per_step": mx.kv_bytes,
            "prefill_flops_per_step": mx.prefill_flops,
            "prefill_roofline": {"bound": "tensor", "achieved": pf_tf, "peak": peaks["bf16_tflops"],
                                 "unit": "TFLOP/s", "frac": pf_tf / peaks["bf16_tflops"], "ms_per_launch": pf_ms,
                                 "launches": 20,
                                 "sustained": {"achieved": pf_sus_tf, "peak": peaks["bf16_tflops_sustained"],
                                               "frac": pf_sus_tf / peaks["bf16_tflops_sustained"],
                                               "ms_per_launch": pf_sus_ms, "launches": pf_sus_n,
                                               "window": "about 0.3 s back to back (power-capped clocks)",
                                               "clocks": pf_clocks},
                                 "kernel": "pa_attention_mixed on the prefill chunks alone, prefill-only mode (plan + prefill_kernel)",
                                 "peak_source": f"{peaks['source']} bf16_tflops (burst: 20 launches back to back, "
                                                f"~5 ms)"}}
        line["gpu_launches"] += mx.launches_per_step * mk + 2 * (20 + pf_sus_n)  # prefill-only: plan + prefill
        line["kv_write"], n_w = _kv_write_alone(mx, peaks)
        line["gpu_launches"] += n_w

    if ws == 1 and not args.no_cpu_baseline:
        # the oracle on this machine's host cores, at N = 1 only (a multi-GPU run would hold every GPU meanwhile)
        line["cpu_baseline"] = cpu_oracle_run(args.workload)
    line["summary"] = _summary(line)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
