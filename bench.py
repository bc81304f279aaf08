#!/usr/bin/env python
"""Benchmark of the decoder-block library on B200: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--only]

Headline (``value``): prefill tokens/s per layer of the LLaMA-2-7B-shaped
layer (dim 4096, 32/32 heads, hd 128, ffn 11008, bf16, causal prefill
1 x 2048).  One step = one ``llama_layer_prefill`` call over the whole batch:
RMSNorm, QKV GEMM, RoPE + KV append, causal flash attention, o_proj +
residual, RMSNorm, gate_up + SiLU·mul, down + residual.  The other workloads
(13B-shaped decode, 70B-shaped GQA prefill and decode, Phi-3-mini-shaped
whole model prefill and decode) are reported under ``workloads`` at N = 1.

Timing: W untimed warm-up steps, then K steps between a barrier plus
cudaDeviceSynchronize on both sides, CUDA events on the launching stream;
max over ranks.  Every step reads > 126 MB (the L2 size) of weights, so no
L2 flush is needed.  Per-kernel device times come from the library's own
tracer (CUDA events around each launch) in a second pass of K steps.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (the only reference this project has), on rank 0.
"""

from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

HEADLINE = "llama7b_prefill"
METRIC = "prefill & decode tokens/s per layer at 1 B200; % of TC / HBM roofline"
UNIT = "tokens/s/layer"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# ncu summary of the roofline kernel: its `traffic_bytes_per_launch` line is used
# only while `source_sha256` matches the kernel sources it was captured from
ROOFLINE_PROFILE = os.path.join(ROOT, "profiles", "gemm_gate_up_swiglu_llama7b_prefill.md")
KERNEL_SOURCES = ("llama_decoder_only_b200/csrc/gemm_tc.cuh", "llama_decoder_only_b200/csrc/common.cuh")


# ------------------------------------------------------------------ peaks, clocks

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha256():
    """sha256 over the sources of the tensor-core GEMM kernel (gemm_tc.cuh, common.cuh)."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def roofline_traffic():
    """(bytes per launch or None, note) from the committed ncu summary of the roofline kernel."""
    try:
        fields = {}
        with open(ROOFLINE_PROFILE) as f:
            for line in f:
                if ":" in line and line.split(":", 1)[0].strip() in ("traffic_bytes_per_launch", "source_sha256"):
                    k, v = line.split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        if fields.get("source_sha256") != kernel_source_sha256():
            return None, "null: the kernel sources changed since the ncu capture"
        return float(fields["traffic_bytes_per_launch"]), f"ncu capture in {os.path.relpath(ROOFLINE_PROFILE, ROOT)}"
    except Exception as e:  # missing or unreadable summary
        return None, f"null: {type(e).__name__}"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the GPU is under load."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.2)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.tmp.read())) if len(r) >= 9]
        os.unlink(self.tmp.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing

def spawn_ranks(n_gpus, argv):
    """Re-run this script as ``n_gpus`` ranks (one process per GPU) under
    torch.distributed.run on this node; returns the launcher's exit code."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n_gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    try:
        return subprocess.run(cmd, timeout=3600).returncode
    except subprocess.TimeoutExpired:
        return 124


def dist_init(n_gpus, backend="nccl"):
    """(rank, world, local rank) from the torchrun environment; one GPU per rank."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value, world, device="cuda"):
    """Largest ``value`` over all ranks (the job's time is the slowest rank's)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank, seconds_per_rank, world, device="cuda"):
    """Whole-job throughput: units of all ranks / the slowest rank's time."""
    slowest = max_over_ranks(seconds_per_rank, world, device)
    return units_per_rank * world / slowest, slowest


# ------------------------------------------------------------------ timing helpers

def timed(torch, fn, steps, warmup, world, between=None):
    """Device time (s) of ``steps`` calls of ``fn`` after ``warmup`` calls."""
    stream = torch.cuda.current_stream()
    for i in range(warmup):
        if between:
            between(i)
        fn(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        if between:
            between(i)
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3


def traced(L, torch, fn, steps, between=None):
    """Per-kernel device time over ``steps`` calls, from the library's tracer."""
    L.profile_read(reset=True)
    L.profile_enable(True)
    for i in range(steps):
        if between:
            between(i)
        fn(i)
    torch.cuda.synchronize()
    L.profile_enable(False)
    return L.profile_read(reset=True)


# ------------------------------------------------------------------ workloads

def gemm_flops_per_token(w):
    qkv = (w.n_heads + 2 * w.n_kv_heads) * w.head_dim
    return 2 * w.dim * (qkv + w.n_heads * w.head_dim + 2 * w.ffn_dim) + 2 * w.ffn_dim * w.dim


def attn_prefill_flops(w, B, L, p0=0):
    # causal pairs only: 4 * hd flops per (query, visible key, head)
    pairs = sum(p0 + t + 1 for t in range(L))
    return 4.0 * w.head_dim * w.n_heads * pairs * B


def layer_weight_bytes(w):
    qkv = (w.n_heads + 2 * w.n_kv_heads) * w.head_dim
    return 2 * w.dim * (qkv + w.n_heads * w.head_dim + 3 * w.ffn_dim)


def layer_weight_bytes_q4(w):
    """Bytes of a layer's seven projections in the 4-bit group-64 form: half a byte
    per weight plus a bf16 scale and offset per 64 weights."""
    params = layer_weight_bytes(w) // 2
    return params // 2 + (params // 64) * 4


def bench_prefill_layer(L, torch, w, steps, warmup, world, seed, with_e2e):
    from synth import device as sd
    dims = L.make_dims(w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim, w.eps, w.rope_theta,
                       w.rope_style, w.dtype)
    dev = sd.random_layer_on_device(w, seed)
    lw = L.layer_weights(dev)
    B, S = w.batch, w.prefill_len
    cache = L.KVCache(dims, B, S)
    ws = torch.zeros(L.workspace_size(dims, B, S), dtype=torch.uint8, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 1)
    x = torch.randn(B * S, w.dim, generator=g, device="cuda", dtype=torch.float32)
    y = torch.empty_like(x)

    def reset(_):
        cache.set_length(0)

    def step(_):
        L.layer_prefill(dims, lw, cache, B, S, x, y, ws)

    n0 = L.launch_count()
    t = timed(torch, step, steps, warmup, world, between=reset)
    launches = (L.launch_count() - n0) // (steps + warmup)
    kern = traced(L, torch, step, steps, between=reset)
    if L.device_status(ws) != 0:
        raise RuntimeError("device status error during the prefill bench")
    tokens = B * S
    res = {"tokens_per_step": tokens, "t_step_s": t / steps, "launches_per_step": launches,
           "kernels": {k: {"avg_us": 1e3 * ms / n, "launches": n // steps} for k, (ms, n) in kern.items()},
           "gemm_flops": gemm_flops_per_token(w) * tokens, "attn_flops": attn_prefill_flops(w, B, S)}
    if with_e2e:
        xh = torch.randn(B * S, w.dim, dtype=torch.float32).pin_memory()
        yh = torch.empty_like(xh).pin_memory()

        def e2e_step(_):
            x.copy_(xh, non_blocking=True)
            L.layer_prefill(dims, lw, cache, B, S, x, y, ws)
            yh.copy_(y, non_blocking=True)

        te = timed(torch, e2e_step, steps, warmup, world, between=reset)
        res["e2e_serial_t_step_s"] = te / steps
        res["e2e_t_step_s"] = pipelined_e2e(torch, L, dims, lw, cache, B, S, w.dim, ws, steps, warmup, world)
        res["h2d_bytes"] = xh.numel() * 4
        res["d2h_bytes"] = yh.numel() * 4
    del cache
    return res


def pipelined_e2e(torch, L, dims, lw, cache, B, S, dim, ws, steps, warmup, world):
    """Device time (s) per step of a pipelined host-to-host prefill loop.

    Every step copies its own input from pinned host memory and its result
    back, through the public ``layer_prefill`` call, as a serving loop would:
    copy-in, compute and copy-out run on three streams with double-buffered
    device and host buffers, so step i+1's upload and step i-1's download
    overlap step i's compute (PCIe is full duplex).  Events order each
    buffer's reuse.  Timed from the first upload to the last download.
    """
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    xd = [torch.empty(B * S, dim, device="cuda") for _ in range(2)]
    yd = [torch.empty(B * S, dim, device="cuda") for _ in range(2)]
    xh = [torch.randn(B * S, dim).pin_memory() for _ in range(2)]
    yh = [torch.empty(B * S, dim).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            k = i % 2
            if i >= 2:
                s_in.wait_event(ev_cmp[k])     # step i-2's compute is done with xd[k]
            with torch.cuda.stream(s_in):
                xd[k].copy_(xh[k], non_blocking=True)
            ev_in[k].record(s_in)
            s_cmp.wait_event(ev_in[k])
            if i >= 2:
                s_cmp.wait_event(ev_out[k])    # step i-2's download is done with yd[k]
            cache.set_length(0)
            L.layer_prefill(dims, lw, cache, B, S, xd[k], yd[k], ws, stream=s_cmp)
            ev_cmp[k].record(s_cmp)
            s_out.wait_event(ev_cmp[k])
            with torch.cuda.stream(s_out):
                yh[k].copy_(yd[k], non_blocking=True)
            ev_out[k].record(s_out)

    run(warmup)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    run(steps)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / steps


def bench_decode_layer(L, torch, w, steps, warmup, world, seed, q4=False):
    from synth import device as sd
    dims = L.make_dims(w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim, w.eps, w.rope_theta,
                       w.rope_style, w.dtype)
    if q4:
        dev = sd.random_q4_layer_on_device(w, seed)
        lw = L.layer_weights_q4(dev)
        layer_call = L.layer_decode_q4
    else:
        dev = sd.random_layer_on_device(w, seed)
        lw = L.layer_weights(dev)
        layer_call = L.layer_decode
    B, T0, nsteps = w.decode_batch, w.cache_len, w.decode_steps
    cap = T0 + nsteps
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 2)
    shape = (B, w.n_kv_heads, cap, w.head_dim)
    k = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)
    cache = L.KVCache(dims, B, cap, k=k, v=v)
    ws = torch.zeros(L.workspace_size(dims, B, 1), dtype=torch.uint8, device="cuda")
    xs = torch.randn(nsteps, B, w.dim, generator=g, device="cuda", dtype=torch.float32)
    y = torch.empty(B, w.dim, device="cuda", dtype=torch.float32)

    def pos(i):
        cache.set_length(T0 + (i % nsteps))

    def step(i):
        layer_call(dims, lw, cache, B, xs[i % nsteps], y, ws)

    n0 = L.launch_count()
    t = timed(torch, step, steps, warmup, world, between=pos)
    launches = (L.launch_count() - n0) // (steps + warmup)
    kern = traced(L, torch, step, steps, between=pos)
    if L.device_status(ws) != 0:
        raise RuntimeError("device status error during the decode bench")
    mean_T = sum(T0 + (i % nsteps) + 1 for i in range(steps)) / steps
    kv_bytes = 2 * B * w.n_kv_heads * mean_T * w.head_dim * 2
    return {"tokens_per_step": B, "t_step_s": t / steps, "launches_per_step": launches,
            "kernels": {kk: {"avg_us": 1e3 * ms / n, "launches": n // steps} for kk, (ms, n) in kern.items()},
            "weight_bytes": layer_weight_bytes_q4(w) if q4 else layer_weight_bytes(w), "kv_bytes": kv_bytes,
            "append_bytes": 2 * B * w.n_kv_heads * w.head_dim * 2}


def bench_model(L, torch, w, steps, warmup, world, seed, prefill_steps=None):
    from synth import device as sd
    dims = L.make_dims(w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim, w.eps, w.rope_theta,
                       w.rope_style, w.dtype)
    layers = [sd.random_layer_on_device(w, seed + 10 + i) for i in range(w.n_layers)]
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    emb = (torch.randn(w.vocab, w.dim, generator=g, device="cuda") * w.w_std).to(torch.bfloat16)
    lm = (torch.randn(w.vocab, w.dim, generator=g, device="cuda") * w.w_std).to(torch.bfloat16)
    fn = torch.ones(w.dim, device="cuda", dtype=torch.float32)
    model, keep = L.model_struct(dims, emb, fn, lm, layers)
    B, S, nsteps = w.batch, w.prefill_len, w.decode_steps
    cap = S + nsteps
    caches = [L.KVCache(dims, B, cap) for _ in range(w.n_layers)]
    ws = torch.zeros(max(L.model_workspace_size(model, B, S), L.model_workspace_size(model, B, 1)),
                     dtype=torch.uint8, device="cuda")
    prompt = torch.randint(0, w.vocab, (B, S), generator=g, device="cuda", dtype=torch.int32)
    forced = torch.randint(0, w.vocab, (nsteps, B), generator=g, device="cuda", dtype=torch.int32)
    ids = torch.empty(B, dtype=torch.int32, device="cuda")

    def reset_all(_):
        for c in caches:
            c.set_length(0)

    def prefill(_):
        L.model_forward(model, caches, prompt, B, S, None, ids, ws)

    n_pre = prefill_steps or max(1, steps // 4)
    tp = timed(torch, prefill, n_pre, max(3, warmup // 2), world, between=reset_all)
    kp = traced(L, torch, prefill, 1, between=reset_all)

    def pos(i):
        for c in caches:
            c.set_length(S + (i % nsteps))

    def decode(i):
        L.model_forward(model, caches, forced[i % nsteps], B, 1, None, ids, ws)

    td = timed(torch, decode, steps, warmup, world, between=pos)
    kd = traced(L, torch, decode, steps, between=pos)
    if L.device_status(ws) != 0:
        raise RuntimeError("device status error during the model bench")
    mean_T = sum(S + (i % nsteps) + 1 for i in range(steps)) / steps
    kv_bytes = w.n_layers * 2 * B * w.n_kv_heads * mean_T * w.head_dim * 2
    return {
        "prefill": {"tokens_per_step": B * S, "t_step_s": tp / n_pre,
                    "flops": w.n_layers * (gemm_flops_per_token(w) * B * S + attn_prefill_flops(w, B, S))
                    + 2 * B * w.dim * w.vocab,
                    "kernels": {k: {"total_us": 1e3 * ms, "launches": n} for k, (ms, n) in kp.items()}},
        "decode": {"tokens_per_step": B, "t_step_s": td / steps,
                   "bytes": w.n_layers * layer_weight_bytes(w) + 2 * w.vocab * w.dim + kv_bytes,
                   "kernels": {k: {"avg_us": 1e3 * ms / steps, "launches": n // steps}
                               for k, (ms, n) in kd.items()}},
    }


# ------------------------------------------------------------------ CPU oracle timing

def oracle_sample(tokens=256, repeats=None, budget_s=12.0):
    """fp64 oracle on the first ``tokens`` tokens of the headline layer (bounded CPU work)."""
    import numpy as np

    from oracle import block as ob
    w = synth.shrink(synth.WORKLOADS[HEADLINE], prefill_len=tokens)
    inp = synth.prefill_inputs(w, with_steps=False)
    W = {k: np.asarray(v, np.float64) for k, v in inp.weights.items()}
    d = ob.Dims(w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim, w.eps, w.rope_theta, w.rope_style)
    times = []
    t_start = time.perf_counter()
    while True:
        cache = ob.KVCache(1, w.n_kv_heads, w.head_dim, tokens)
        t0 = time.perf_counter()
        ob.layer_forward(d, W, inp.x, cache)
        times.append(time.perf_counter() - t0)
        if repeats is not None and len(times) >= repeats:
            break
        if repeats is None and time.perf_counter() - t_start > budget_s:
            break
    return tokens, times


def _fp64_layer(w, seed):
    """fp64 weights of workload ``w``'s layer shape for the CPU oracle's timing
    (the seeded recipe; values do not change the oracle's time)."""
    import numpy as np
    return {k: np.asarray(v, np.float64) for k, v in synth.layer_weights(w, np.random.default_rng(seed)).items()}


def _time_repeats(fn, budget_s):
    """Median wall time of ``fn()`` over repeats within ``budget_s`` (at least one)."""
    times = []
    t_start = time.perf_counter()
    while not times or time.perf_counter() - t_start < budget_s:
        t0 = time.perf_counter()
        fn()
        times.append(time.perf_counter() - t0)
    return statistics.median(times), len(times)


def oracle_workload_baselines(budget_s=3.0):
    """The fp64 oracle timed on a bounded sample of each non-headline workload
    (host cores; weights converted to fp64 outside the timed region).  Returns
    {workload key: cpu_baseline object} in the units of that workload's line."""
    import numpy as np

    from oracle import block as ob
    out = {}
    cores, model = cpu_threads(), cpu_model()

    def dims(w):
        return ob.Dims(w.dim, w.n_heads, w.n_kv_heads, w.head_dim, w.ffn_dim, w.eps, w.rope_theta, w.rope_style)

    def decode_sample(w, T0):
        W = _fp64_layer(w, w.seed)
        rng = np.random.default_rng(w.seed + 1)
        k0 = rng.standard_normal((1, w.n_kv_heads, T0, w.head_dim))
        v0 = rng.standard_normal((1, w.n_kv_heads, T0, w.head_dim))
        x = rng.standard_normal((1, 1, w.dim))

        def one():
            ob.layer_forward(dims(w), W, x, ob.KVCache(1, w.n_kv_heads, w.head_dim, T0 + 1, k0, v0))
        return one

    def prefill_sample(w, tokens):
        W = _fp64_layer(w, w.seed)
        x = np.random.default_rng(w.seed + 1).standard_normal((1, tokens, w.dim))

        def one():
            ob.layer_forward(dims(w), W, x, ob.KVCache(1, w.n_kv_heads, w.head_dim, tokens))
        return one

    W = synth.WORKLOADS
    t, n = _time_repeats(decode_sample(W["llama13b_decode"], 4096), budget_s)
    out["llama13b_decode/decode"] = {
        "value": 1.0 / t, "unit": "tokens/s/layer", "cores": cores, "kind": "oracle",
        "sample": f"fp64 oracle decode step of 1 of 16 sequences at cache length 4097, median of {n} ({model})"}
    t, n = _time_repeats(prefill_sample(W["gqa70b"], 256), budget_s)
    out["gqa70b/prefill"] = {
        "value": 256 / t, "unit": "tokens/s/layer", "cores": cores, "kind": "oracle",
        "sample": f"fp64 oracle prefill of the first 256 of 2 x 4096 tokens, median of {n} ({model})"}
    t, n = _time_repeats(decode_sample(W["gqa70b"], 4096), budget_s)
    out["gqa70b/decode"] = {
        "value": 1.0 / t, "unit": "tokens/s/layer", "cores": cores, "kind": "oracle",
        "sample": f"fp64 oracle decode step of 1 of 64 sequences at cache length 4097, median of {n} ({model})"}
    w = W["phi3mini_model"]
    t, n = _time_repeats(prefill_sample(w, 128), budget_s)
    out["phi3mini_model/prefill"] = {
        "value": 128 / (t * w.n_layers), "unit": "tokens/s (model)", "cores": cores, "kind": "oracle",
        "sample": f"fp64 oracle prefill of 128 of 8 x 512 tokens through ONE of the 32 layers, median of {n}, "
                  f"scaled by 32 layers (embedding and lm_head not timed) ({model})"}
    t, n = _time_repeats(decode_sample(w, 512), budget_s)
    out["phi3mini_model/decode"] = {
        "value": 1.0 / (t * w.n_layers), "unit": "tokens/s (model)", "cores": cores, "kind": "oracle",
        "sample": f"fp64 oracle decode step of 1 of 8 sequences at cache length 513 through ONE of the 32 layers, "
                  f"median of {n}, scaled by 32 layers ({model})"}
    return out


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_model():
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.startswith("Model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


# ------------------------------------------------------------------ main

def headline_config(w):
    return {"workload": f"{w.name}: LLaMA-2-7B-shaped layer (dim {w.dim}, {w.n_heads}/{w.n_kv_heads} heads, "
                        f"hd {w.head_dim}, ffn {w.ffn_dim}), bf16, causal prefill {w.batch} x {w.prefill_len}",
            "batch": w.batch, "seq_len": w.prefill_len, "layers_per_step": 1,
            "l2": "no flush: every step streams 405 MB of weights (> 126 MB L2)",
            "parallelism": "replicas (one independent layer per GPU)"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    w = synth.WORKLOADS[HEADLINE]
    tokens = 256
    _, times = oracle_sample(tokens, repeats=args.warmup + args.steps)
    timed_s = sum(times[args.warmup:])
    value = tokens * args.steps / timed_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * timed_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) inputs, N(0,0.02) weights)", "config": headline_config(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": f"fp64 oracle layer prefill of the first {tokens} of {w.prefill_len} tokens "
                                       f"per step ({cpu_model()})"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def run_fake(args):
    """Host-logic self-test of the multi-rank plumbing (no GPU, gloo): every rank
    'processes' 1000 units per step in (1 + rank) ms of sleep, timed on the host
    clock; the line carries the same aggregation as a real run."""
    rank, world, _ = dist_init(args.gpus, backend="gloo")
    for _ in range(args.warmup):
        time.sleep(0.001 * (1 + rank))
    barrier(world)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(0.001 * (1 + rank))
    elapsed = time.perf_counter() - t0
    barrier(world)
    value, slowest = aggregate_throughput(1000 * args.steps, elapsed, world, device="cpu")
    if rank == 0:
        print(json.dumps({"metric": "fake units/s", "value": value, "unit": "units/s", "n_gpus": world,
                          "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * slowest / args.steps,
                          "higher_is_better": True, "scaling": "weak", "data": "fake (host-logic self-test)",
                          "slowest_rank_s": slowest}))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--only", action="store_true", help="headline workload only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=None, choices=sorted(WORKLOAD_RUNNERS),
                    help="run one workload alone and print its own line (for profiling)")
    ap.add_argument("--fake-workload", action="store_true",
                    help="host-logic self-test of the multi-rank plumbing: no GPU, gloo, sleeps")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: re-run this command as N ranks on this node
        return spawn_ranks(args.gpus, sys.argv[1:])
    if args.fake_workload:
        return run_fake(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.workload:
        return run_single_workload(args)

    import torch

    import llama_decoder_only_b200 as L
    rank, world, local = dist_init(args.gpus)
    peaks, peak_src = load_peaks()
    sampler = ClockSampler(local)
    sampler.start()
    w = synth.WORKLOADS[HEADLINE]
    r = bench_prefill_layer(L, torch, w, args.steps, args.warmup, world, seed=100 + rank, with_e2e=True)
    value, slowest = aggregate_throughput(r["tokens_per_step"] * args.steps, r["t_step_s"] * args.steps, world)
    e2e_value, _ = aggregate_throughput(r["tokens_per_step"] * args.steps, r["e2e_t_step_s"] * args.steps, world)
    e2e_serial, _ = aggregate_throughput(r["tokens_per_step"] * args.steps, r["e2e_serial_t_step_s"] * args.steps,
                                         world)
    workloads = {}
    if world == 1 and not args.only:
        workloads = run_other_workloads(L, torch, args, peaks)
    clocks = sampler.stop()

    # roofline of the dominant kernel (the gate_up GEMM with the SiLU·mul epilogue)
    kg = r["kernels"].get("gemm_gate_up_swiglu")
    timed_region_s = r["t_step_s"] * args.steps
    peak_key = "bf16_tflops_sustained" if timed_region_s > 2.0 else "bf16_tflops"
    gu_flops = 2.0 * w.batch * w.prefill_len * 2 * w.ffn_dim * w.dim
    achieved = gu_flops / (kg["avg_us"] * 1e-6) / 1e12 if kg else None
    traffic, traffic_note = roofline_traffic()
    roofline = {"kernel": "gemm_gate_up_swiglu", "bound": "tensor", "achieved": achieved,
                "peak": peaks[peak_key], "unit": "TFLOP/s",
                "frac": achieved / peaks[peak_key] if achieved else None,
                "traffic": traffic, "traffic_source": traffic_note,
                "peak_source": f"{peak_key} ({'of measured' if peak_src == 'measured' else 'of fallback'})",
                "algorithmic_flops_per_launch": gu_flops}
    layer_flops = r["gemm_flops"] + r["attn_flops"]
    layer_tflops = layer_flops / r["t_step_s"] / 1e12

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        tokens, times = oracle_sample(256, budget_s=12.0)
        cpu = {"value": tokens / statistics.median(times), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
               "sample": f"fp64 oracle prefill of the first {tokens} of {w.prefill_len} tokens of the headline layer, "
                         f"median of {len(times)} runs ({cpu_model()})"}
        if workloads:
            for name, cb in oracle_workload_baselines().items():
                if name in workloads:
                    workloads[name]["cpu_baseline"] = cb

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * slowest / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) inputs, N(0,0.02) random-init weights of the layer's shape)",
            "config": headline_config(w),
            "layer_tflops": layer_tflops, "layer_frac_of_tensor_peak": layer_tflops / peaks[peak_key],
            "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": r["h2d_bytes"],
                    "d2h_bytes_per_step": r["d2h_bytes"],
                    "mode": "pipelined: copy-in, layer_prefill and copy-out on three streams, double-buffered",
                    "serial_value": e2e_serial},
            "gpu_launches": r["launches_per_step"] * args.steps,
            "kernels_us": {k: round(v["avg_us"], 2) for k, v in r["kernels"].items()},
            "clocks": clocks, "workloads": workloads,
        }
        dec = workloads.get("llama13b_decode/decode")
        if dec:
            line["decode"] = {"workload": "llama13b_decode: LLaMA-2-13B-shaped layer, bf16, batch 16, cache "
                                          "4096 -> 4224 over 128 steps, interleaved RoPE",
                              "value": dec["tokens_per_s_per_layer"], "unit": UNIT,
                              "frac_of_hbm_peak": dec["frac_of_hbm_peak"]}
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def _single_decode(L, torch, name, args, q4=False):
    r = bench_decode_layer(L, torch, synth.WORKLOADS[name], args.steps, args.warmup, 1, seed=11, q4=q4)
    by = r["weight_bytes"] + r["kv_bytes"] + r["append_bytes"]
    return {"metric": "decode tokens/s per layer", "unit": UNIT, "value": r["tokens_per_step"] / r["t_step_s"],
            "ms_per_step": 1e3 * r["t_step_s"], "gbs": by / r["t_step_s"] / 1e9,
            "kernels_us": {k: round(v["avg_us"], 2) for k, v in r["kernels"].items()}}


def _single_prefill(L, torch, name, args):
    w = synth.WORKLOADS[name]
    r = bench_prefill_layer(L, torch, w, args.steps, args.warmup, 1, seed=7, with_e2e=False)
    fl = r["gemm_flops"] + r["attn_flops"]
    return {"metric": "prefill tokens/s per layer", "unit": UNIT, "value": r["tokens_per_step"] / r["t_step_s"],
            "ms_per_step": 1e3 * r["t_step_s"], "tflops": fl / r["t_step_s"] / 1e12,
            "kernels_us": {k: round(v["avg_us"], 2) for k, v in r["kernels"].items()}}


def _single_model(L, torch, phase, args):
    r = bench_model(L, torch, synth.WORKLOADS["phi3mini_model"], args.steps, args.warmup, 1, seed=21)[phase]
    return {"metric": f"model {phase} tokens/s", "unit": "tokens/s", "value": r["tokens_per_step"] / r["t_step_s"],
            "ms_per_step": 1e3 * r["t_step_s"]}


WORKLOAD_RUNNERS = {
    "llama7b_prefill": lambda L, t, a: _single_prefill(L, t, "llama7b_prefill", a),
    "llama13b_decode": lambda L, t, a: _single_decode(L, t, "llama13b_decode", a),
    "gqa70b_prefill": lambda L, t, a: _single_prefill(L, t, "gqa70b", a),
    "gqa70b_decode": lambda L, t, a: _single_decode(L, t, "gqa70b", a),
    "llama13b_decode_q4": lambda L, t, a: _single_decode(L, t, "llama13b_decode", a, q4=True),
    "phi3_prefill": lambda L, t, a: _single_model(L, t, "prefill", a),
    "phi3_decode": lambda L, t, a: _single_model(L, t, "decode", a),
}


def run_single_workload(args):
    import torch

    import llama_decoder_only_b200 as L
    torch.cuda.set_device(0)
    line = {"workload": args.workload, "steps": args.steps, "warmup": args.warmup}
    line.update(WORKLOAD_RUNNERS[args.workload](L, torch, args))
    print(json.dumps(line))
    return 0


def run_other_workloads(L, torch, args, peaks):
    out = {}
    hbm = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops"] * 1e12
    for name in ("llama13b_decode", "gqa70b"):
        w = synth.WORKLOADS[name]
        if w.prefill_len:
            r = bench_prefill_layer(L, torch, w, max(3, args.steps // 3), args.warmup, 1, seed=7, with_e2e=False)
            fl = r["gemm_flops"] + r["attn_flops"]
            out[f"{name}/prefill"] = {
                "tokens_per_s_per_layer": r["tokens_per_step"] / r["t_step_s"], "ms_per_step": 1e3 * r["t_step_s"],
                "tflops": fl / r["t_step_s"] / 1e12, "frac_of_tensor_peak": fl / r["t_step_s"] / tc,
                "kernels_us": {k: round(v["avg_us"], 1) for k, v in r["kernels"].items()}}
        r = bench_decode_layer(L, torch, w, w.decode_steps, args.warmup, 1, seed=11)
        by = r["weight_bytes"] + r["kv_bytes"] + r["append_bytes"]
        out[f"{name}/decode"] = {
            "steps": w.decode_steps, "cache_lengths": [w.cache_len + 1, w.cache_len + w.decode_steps],
            "tokens_per_s_per_layer": r["tokens_per_step"] / r["t_step_s"], "ms_per_step": 1e3 * r["t_step_s"],
            "gbs": by / r["t_step_s"] / 1e9, "frac_of_hbm_peak": by / r["t_step_s"] / hbm,
            "kernels_us": {k: round(v["avg_us"], 1) for k, v in r["kernels"].items()}}
        torch.cuda.empty_cache()
    w = synth.WORKLOADS["llama13b_decode"]
    r = bench_decode_layer(L, torch, w, w.decode_steps, args.warmup, 1, seed=13, q4=True)
    by = r["weight_bytes"] + r["kv_bytes"] + r["append_bytes"]
    out["llama13b_decode_q4/decode"] = {
        "weights": "4-bit group-64 (codes + bf16 scale/offset per 64 weights)",
        "steps": w.decode_steps, "cache_lengths": [w.cache_len + 1, w.cache_len + w.decode_steps],
        "weight_bytes": r["weight_bytes"], "tokens_per_s_per_layer": r["tokens_per_step"] / r["t_step_s"],
        "ms_per_step": 1e3 * r["t_step_s"], "gbs": by / r["t_step_s"] / 1e9, "frac_of_hbm_peak": by / r["t_step_s"] / hbm,
        "kernels_us": {k: round(v["avg_us"], 1) for k, v in r["kernels"].items()}}
    torch.cuda.empty_cache()
    w = synth.WORKLOADS["phi3mini_model"]
    r = bench_model(L, torch, w, w.decode_steps, args.warmup, 1, seed=21, prefill_steps=max(3, args.steps // 4))
    p, d = r["prefill"], r["decode"]
    out["phi3mini_model/prefill"] = {"tokens_per_s_model": p["tokens_per_step"] / p["t_step_s"],
                                     "ms_per_step": 1e3 * p["t_step_s"],
                                     "tflops": p["flops"] / p["t_step_s"] / 1e12,
                                     "frac_of_tensor_peak": p["flops"] / p["t_step_s"] / tc}
    out["phi3mini_model/decode"] = {"steps": w.decode_steps,
                                    "cache_lengths": [w.prefill_len + 1, w.prefill_len + w.decode_steps],
                                    "tokens_per_s_model": d["tokens_per_step"] / d["t_step_s"],
                                    "ms_per_step": 1e3 * d["t_step_s"],
                                    "gbs": d["bytes"] / d["t_step_s"] / 1e9,
                                    "frac_of_hbm_peak": d["bytes"] / d["t_step_s"] / hbm,
                                    "kernels_us": {k: round(v["avg_us"], 1) for k, v in d["kernels"].items()}}
    torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    sys.exit(main())
