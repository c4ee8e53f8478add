"""Benchmark of the D-Quant compressed-KV hot path on B200.

One step = append one new token per sequence (dq_append_kv: rotate,
normalise, quantise, rANS-encode, drift into a container) + one decode step
of attention over the whole compressed context (dq_decode_attention: split-K
kernel decoding the containers in-kernel + combine kernel), on the serving
shape batch 128, 8 KV heads, 32 query heads, head_dim 128, 8192-token context
(the token appended each step is position 8191; the context is 8192 tokens).

Metric: compressed-KV decode attention throughput in KV tokens/s (B x context
per step); the HBM rate of the compressed bytes and the dominant kernel's
roofline fraction are reported beside it.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dq|reference]
                  [--workload NAME] [--paged] [--layers L] [--graph] [--prefill N_Q]
                  [--drift-mode 0|1]
--drift-mode 1 encodes with the rate-distortion fill after drift (the encode
report then shows its cost); --paged keeps the caches in page pools behind a
shuffled page table; --layers
runs an L-layer attention-only decode loop (one cache per layer); --graph also
times the step captured once as a CUDA graph and replayed. --prefill N_Q
switches to the chunked-prefill step (append an N_Q-token chunk to every
sequence, then causal attention of its queries over the compressed context)
and its own metric, query tokens/s, with a tensor-core roofline.
Under torchrun every rank runs an independent replica (no data-path
collective): value = all ranks' KV tokens / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "compressed-KV decode attention: KV tokens/s and HBM GB/s at B=128, 8K ctx"
UNIT = "KV tokens/s"
WORKLOAD = "serve_b128_t8k"
# Algorithmic work per token-head (one K and one V container), fixed
# convention: 128 symbols x 2 streams x (5.5 rANS decode ops + G multiply-adds)
# + 8 G softmax ops, counted in lane-ops (issue slots x 32).
RANS_OPS_PER_SYMBOL = 5.5
SOFTMAX_OPS_PER_HEAD = 8
# Encode (append) work per vector, same convention: 896 WHT + 256 norm/scale
# + 384 quantise + 128 x 8 rANS encode lane-ops.
ENCODE_OPS_PER_VECTOR = 2560
# Kernel launches of one step: dq_append_kv (1) + dq_decode_attention
# (prefix, split, combine).
LAUNCHES_PER_STEP = 4
# DRAM traffic of decode_split_kernel from one ncu capture (dram__bytes_read
# + dram__bytes_write) of the 32-sequence, 8192-token workload with 36-byte
# containers: 151.37 MB + 3.34 MB per launch over 32*8*8192 token-heads. It
# scales with the token-heads a launch processes (reads are the containers,
# writes the partial states). It belongs to one version of the kernel source:
# for any other, or other container sizes, traffic is reported as null.
# (Captured at source hash 5f062cef3d424eb2; the file has changed since in
# one comment only.)
DECODE_TRAFFIC = {"source": "decode_attention_dq_b200/csrc/dq_decode.cu",
                  "sha256_16": "2e1b65131b495877", "ck": 36, "cv": 36,
                  "bytes_per_token_head": (151.369216e6 + 3.344896e6) / (32 * 8 * 8192)}


def decode_traffic(token_heads, ck, cv):
    import hashlib
    t = DECODE_TRAFFIC
    try:
        with open(os.path.join(ROOT, t["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    if sha != t["sha256_16"] or (ck, cv) != (t["ck"], t["cv"]):
        return None
    return token_heads * t["bytes_per_token_head"]


def ops_per_token_head(G: int) -> float:
    return 2 * 128 * (RANS_OPS_PER_SYMBOL + G) + SOFTMAX_OPS_PER_HEAD * G


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def replica_workload(w, rank):
    """Each rank of a multi-GPU run is an independent replica with its own
    sequences (same shapes, its own seed); rank 0 keeps the workload's seed."""
    from decode_attention_dq_b200 import synth
    return w if rank == 0 else synth.scaled(w, seed=w.seed + 1000 * rank, name=w.name)


def max_over_ranks(values, dist, device):
    """Element-wise maximum of a list of floats over all ranks (the slowest
    rank's times); the values unchanged without a process group."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_rate(units_per_step_per_rank, world_size, ms_per_step):
    """Throughput of the whole job: every rank's units over the slowest
    rank's time per step."""
    return units_per_step_per_rank * world_size / (ms_per_step * 1e-3)


def dist_setup(args):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return ws, rank, local


def run_pipelined(nst, stream, n_in, n_out, h2d, compute, d2h, t_start=None, t_end=None):
    """nst end-to-end steps with the copies on their own streams, pipelined
    with the kernels on `stream`: step s+1's inputs go in (h2d(s) on an
    upload stream) and step s's output comes back (d2h(s) on a read-back
    stream) while kernels run. Events keep every dependency: compute(s)
    waits for its inputs; input buffer s % n_in is refilled only after the
    step that last read it has finished; output buffer s % n_out is rewritten
    only after its read-back; t_end (on `stream`) follows the last
    read-back, t_start precedes the first upload."""
    import torch

    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nst)]
    ev_done = [torch.cuda.Event() for _ in range(nst)]
    ev_out = [torch.cuda.Event() for _ in range(nst)]
    start = t_start if t_start is not None else torch.cuda.Event()
    start.record(stream)
    up.wait_event(start)
    down.wait_event(start)

    def upload(s):
        if s >= n_in:
            up.wait_event(ev_done[s - n_in])
        with torch.cuda.stream(up):
            h2d(s)
        ev_in[s].record(up)

    upload(0)
    for s in range(nst):
        if s + 1 < nst:
            upload(s + 1)
        stream.wait_event(ev_in[s])
        if s >= n_out:
            stream.wait_event(ev_out[s - n_out])
        compute(s)
        ev_done[s].record(stream)
        down.wait_event(ev_done[s])
        with torch.cuda.stream(down):
            d2h(s)
        ev_out[s].record(down)
    stream.wait_event(ev_out[nst - 1])
    if t_end is not None:
        t_end.record(stream)


def run_dq(args):
    import numpy as np
    import torch

    import decode_attention_dq_b200 as dq
    from decode_attention_dq_b200 import synth

    ws, rank, local = dist_setup(args)
    dist = None
    if ws > 1:
        import torch.distributed as dist
    w = replica_workload(synth.WORKLOADS[args.workload], rank)
    dev = torch.device("cuda", torch.cuda.current_device())
    tab = dq.dq_build_tables(n_kv_heads=w.Hkv, k_bits_per_value=w.k_bits, v_bits_per_value=w.v_bits,
                             drift_mode=args.drift_mode, k_rate_offset=args.k_rate_offset,
                             v_rate_offset=args.v_rate_offset)
    ck, cv = tab.k.container_bytes, tab.v.container_bytes
    T = w.T
    T_cap = (T + 31) // 32 * 32
    G = w.Hq // w.Hkv
    page_table = None
    if args.paged:
        # Pages of 32 tokens handed out in a shuffled order from one pool.
        max_pages = T_cap // 32
        num_pages = w.B * max_pages
        perm = np.random.default_rng(w.seed).permutation(num_pages).astype(np.int32)
        page_table = torch.from_numpy(perm.reshape(w.B, max_pages)).to(dev)
        kc = dq.new_pool(num_pages, w.Hkv, ck, dev)
        vc = dq.new_pool(num_pages, w.Hkv, cv, dev)
    else:
        kc = torch.zeros((w.B, w.Hkv, T_cap, ck), dtype=torch.uint8, device=dev)
        vc = torch.zeros((w.B, w.Hkv, T_cap, cv), dtype=torch.uint8, device=dev)
    prefill_stats = dq.new_stats(dev)
    t0 = time.time()
    enc_timings = []
    synth.prefill_cache(tab, w, kc, vc, T - 1, stats=prefill_stats, threads=args.threads,
                        timings=enc_timings, page_table=page_table)
    torch.cuda.synchronize()
    prefill_s = time.time() - t0
    pstats = dq.stats_dict(prefill_stats)
    enc_ms = sum(a.elapsed_time(b) for a, b, _ in enc_timings)
    enc_vectors = sum(n for _, _, n in enc_timings)  # per stream (K and V each)

    # Per-step inputs: a distinct new token and q for each step (host, pinned).
    nsteps_inputs = 4
    rows = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    host_k, host_v, host_q = [], [], []
    for s in range(nsteps_inputs):
        host_k.append(torch.from_numpy(synth.kv_block(w, "k", rows, n=1, step=s, threads=args.threads))
                      .to(w.torch_dtype).view(w.B, w.Hkv, 1, 128).pin_memory())
        host_v.append(torch.from_numpy(synth.kv_block(w, "v", rows, n=1, step=s, threads=args.threads))
                      .to(w.torch_dtype).view(w.B, w.Hkv, 1, 128).pin_memory())
        host_q.append(torch.from_numpy(synth.q_block(w, step=s)).to(w.torch_dtype).pin_memory())
    dev_k = [t.to(dev) for t in host_k]
    dev_v = [t.to(dev) for t in host_v]
    dev_q = [t.to(dev) for t in host_q]
    start = torch.full((w.B,), T - 1, dtype=torch.int32, device=dev)
    seq = torch.full((w.B,), T, dtype=torch.int32, device=dev)
    nbytes = dq.dq_decode_workspace_bytes(tab, w.B, w.Hq, w.Hkv, T)
    wsp = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=dev)
    out_host = torch.empty_like(out, device="cpu").pin_memory()
    stats = dq.new_stats(dev)
    stream = torch.cuda.current_stream()

    app_ws = torch.empty(max(16, dq.dq_append_workspace_bytes(tab, w.B, w.Hkv, 1)), dtype=torch.uint8,
                         device=dev)
    # Serving loop of L layers: one cache per layer (the same prefilled
    # contents), each step appends to and attends over every layer in turn.
    L = max(1, args.layers)
    caches = [(kc, vc)] + [(kc.clone(), vc.clone()) for _ in range(L - 1)]

    def append(i, layer, st):
        kl, vl = caches[layer]
        if page_table is None:
            dq.dq_append_kv(tab, dev_k[i], dev_v[i], start, kl, vl, stats=stats, stream=st, workspace=app_ws)
        else:
            dq.dq_append_kv_paged(tab, dev_k[i], dev_v[i], start, kl, vl, page_table, stats=stats,
                                  stream=st, workspace=app_ws)

    def decode(i, layer, st, o=None):
        kl, vl = caches[layer]
        o = out if o is None else o
        if page_table is None:
            dq.dq_decode_attention(tab, dev_q[i], kl, vl, seq, T, o, wsp, stats=stats, stream=st)
        else:
            dq.dq_decode_attention_paged(tab, dev_q[i], kl, vl, page_table, seq, T, o, wsp, stats=stats,
                                         stream=st)

    def step(s, ev=None, st=None):
        st = stream if st is None else st
        i = s % nsteps_inputs
        for layer in range(L):
            append(i, layer, st)
            if ev is not None:
                ev[layer][0].record(st)
            decode(i, layer, st)
            if ev is not None:
                ev[layer][1].record(st)

    def barrier():
        if dist is not None:
            dist.barrier()

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()

    # ---- timed region: device-resident inputs ----
    ev_dec = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(L)] for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for s in range(args.steps):
        step(s, ev_dec[s])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    elapsed_ms = e0.elapsed_time(e1)
    dec_ms = sum(a.elapsed_time(b) for evs in ev_dec for a, b in evs) / (args.steps * L)  # per decode call

    # ---- optional: the same step captured once as a CUDA graph and replayed ----
    graph_ms = None
    if args.graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(0, st=torch.cuda.current_stream())
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(args.steps):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        graph_ms = max_over_ranks([g0.elapsed_time(g1) / args.steps], dist, dev)[0]
        del g
    elapsed_ms, dec_ms = max_over_ranks([elapsed_ms, dec_ms], dist, dev)
    ms_per_step = elapsed_ms / args.steps
    kv_tokens_step = w.B * T * L
    value = whole_job_rate(kv_tokens_step, ws, ms_per_step)

    # ---- e2e: host buffers, copies inside the timed region ----
    # Every step copies its new K/V and q in from pinned host memory and its
    # output back, pipelined with the kernels (run_pipelined); the inputs
    # cycle over nsteps_inputs device buffers, the outputs over two.
    outs = [out, torch.empty_like(out)]
    outs_host = [out_host, torch.empty_like(out_host).pin_memory()]

    def e2e_h2d(s):
        i = s % nsteps_inputs
        dev_k[i].copy_(host_k[i], non_blocking=True)
        dev_v[i].copy_(host_v[i], non_blocking=True)
        dev_q[i].copy_(host_q[i], non_blocking=True)

    def e2e_compute(s):
        i = s % nsteps_inputs
        for layer in range(L):
            append(i, layer, stream)
            decode(i, layer, stream, outs[s % 2])

    def e2e_d2h(s):
        outs_host[s % 2].copy_(outs[s % 2], non_blocking=True)

    def run_e2e(nst, t_start=None, t_end=None):
        run_pipelined(nst, stream, nsteps_inputs, 2, e2e_h2d, e2e_compute, e2e_d2h, t_start, t_end)

    run_e2e(2)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run_e2e(args.steps, f0, f1)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks([f0.elapsed_time(f1)], dist, dev)[0]
    e2e_value = whole_job_rate(kv_tokens_step, ws, e2e_ms / args.steps)

    # ---- small-batch decode latency: the first 1 and 8 sequences of the same
    # cache, one dq_decode_attention call at a time with L2 flushed before
    # each (the regime in which the pages find D-Quant slower than BF16) ----
    small_batch = small_batch_latency(dq, tab, w, kc, vc, dev_q[0], seq, T, stream, dist, dev) \
        if (L == 1 and page_table is None) else None

    # ---- the long-context and low-budget workloads (device-timed, inputs
    # larger than L2); the serving caches stay resident meanwhile ----
    peaks, _src = measured_peaks()
    alu_peak_all = (torch.cuda.get_device_properties(dev).multi_processor_count * 128
                    * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12)
    long_context = budget_sweep = None
    if args.extra and L == 1 and page_table is None:
        long_context = long_context_report(dq, args, dev, stream, dist, alu_peak_all, peaks)
        budget_sweep = budget_sweep_report(dq, args, dev, stream, dist, alu_peak_all, peaks)

    # ---- chunked prefill over the same cache: the last n_q positions as a
    # chunk of queries (dq_prefill_attention), device-resident inputs ----
    prefill = None
    if args.prefill_chunk > 0 and L == 1 and T > args.prefill_chunk:
        n_q = args.prefill_chunk
        gq = torch.Generator(device=dev).manual_seed(w.seed)
        qc = torch.randn((w.B, n_q, w.Hq, 128), generator=gq, device=dev).to(w.torch_dtype)
        outc = torch.empty((w.B, n_q, w.Hq, 128), dtype=torch.float32, device=dev)
        qs0 = torch.full((w.B,), T - n_q, dtype=torch.int32, device=dev)
        pws = torch.empty(dq.dq_prefill_workspace_bytes(tab, w.B, w.Hkv, T_cap), dtype=torch.uint8, device=dev)

        def prefill_call():
            if page_table is None:
                dq.dq_prefill_attention(tab, qc, kc, vc, qs0, outc, workspace=pws, stats=stats)
            else:
                dq.dq_prefill_attention_paged(tab, qc, kc, vc, page_table, qs0, outc, workspace=pws, stats=stats)

        for _ in range(3):
            prefill_call()
        torch.cuda.synchronize()
        barrier()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        p0.record(stream)
        for _ in range(reps):
            prefill_call()
        p1.record(stream)
        torch.cuda.synchronize()
        barrier()
        pms = max_over_ranks([p0.elapsed_time(p1) / reps], dist, dev)[0]
        del pws
        prefill = {"chunk": n_q, "q_start": T - n_q, "ms": pms,
                   "query_tokens_per_s": whole_job_rate(w.B * n_q, ws, pms),
                   "useful_flops": chunk_pairs(w.B, w.Hq, T - n_q, n_q) * FLOPS_PER_PAIR,
                   "launches": 2 * reps}
    h2d = (host_k[0].numel() + host_v[0].numel() + host_q[0].numel()) * host_k[0].element_size()
    d2h = out_host.numel() * out_host.element_size()
    st = dq.stats_dict(stats)

    result = None
    if rank == 0:
        peaks, src = measured_peaks()
        sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
        clock_mhz = float(peaks.get("sm_max_mhz", 1965.0))
        alu_peak = sm_count * 128 * clock_mhz * 1e6 / 1e12  # T lane-ops/s
        token_heads = w.B * T * w.Hkv
        ops = token_heads * ops_per_token_head(G)
        achieved = ops / (dec_ms * 1e-3) / 1e12
        comp_bytes = token_heads * (ck + cv)
        hbm_gbs = comp_bytes / (dec_ms * 1e-3) / 1e9
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hkv": w.Hkv, "Hq": w.Hq, "head_dim": 128,
                       "context": T, "appended_per_step": 1, "input_dtype": w.dtype,
                       "k_bits_per_value": w.k_bits, "v_bits_per_value": w.v_bits,
                       "k_container_bytes": ck, "v_container_bytes": cv,
                       "l2": "inputs larger than L2 (%.0f MB of containers read per step)" % (comp_bytes / 1e6),
                       "cache": "paged: 32-token pages in a shuffled order" if args.paged else "contiguous",
                       "drift_mode": args.drift_mode,
                       "rate_offsets": [args.k_rate_offset, args.v_rate_offset],
                       "layers": L,
                       "parallelism": "replicas x%d" % ws},
            "hbm_gbs": hbm_gbs,
            "roofline": {"bound": "alu", "achieved": achieved, "peak": alu_peak, "unit": "Tlaneop/s",
                         "frac": achieved / alu_peak,
                         "traffic": None if args.paged else decode_traffic(token_heads, ck, cv),
                         "traffic_note": "decode_split_kernel DRAM bytes per launch, scaled from an ncu "
                                         "capture of the 32-sequence case by token-heads",
                         "algorithmic_bytes": comp_bytes,
                         "kernel": "decode_split_kernel + combine_kernel (dq_decode_attention)",
                         "kernel_ms": dec_ms, "peak_source": "%s clock, %d SMs x 128 lanes" % (src, sm_count),
                         "hbm": {"achieved_gbs": hbm_gbs, "peak_gbs": peaks.get("hbm_gbs"),
                                 "frac": hbm_gbs / float(peaks.get("hbm_gbs", 6650.0))}},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "copies": "every step's inputs in and output out, on upload and read-back streams "
                              "pipelined with the kernels"},
            "gpu_launches": LAUNCHES_PER_STEP * L * args.steps,
            "clocks": clk,
            "drift": {"prefill_k_syms_filled_pct": 100.0 * pstats["k_syms_filled"] / (token_heads * 128),
                      "prefill_v_syms_filled_pct": 100.0 * pstats["v_syms_filled"] / (token_heads * 128),
                      "prefill_k_syms_pct": 100.0 * pstats["k_syms_drifted"] / (token_heads * 128),
                      "prefill_v_syms_pct": 100.0 * pstats["v_syms_drifted"] / (token_heads * 128),
                      "prefill_k_cont_pct": 100.0 * pstats["k_cont_drifted"] / token_heads,
                      "prefill_v_cont_pct": 100.0 * pstats["v_cont_drifted"] / token_heads,
                      "fallbacks": pstats["overflow_fallbacks"]},
            "integrity_errors": st["integrity_errors"],
            "small_batch": small_batch,
            "long_context": long_context,
            "budget_sweep": budget_sweep,
            "prefill_s": prefill_s,
            "encode": encode_report(enc_ms, enc_vectors, w, ck, cv, alu_peak, peaks),
            "chunked_prefill": None if prefill is None else dict(
                prefill, what="dq_prefill_attention of the last %d positions of every sequence as a chunk of "
                              "queries over the %d-token compressed cache (random queries)" % (prefill["chunk"], T),
                tflops=prefill["useful_flops"] / (prefill["ms"] * 1e-3) / 1e12,
                roofline={"bound": "tensor", "peak": float(peaks.get("bf16_tflops", 1590.0)), "unit": "TFLOP/s",
                          "frac": prefill["useful_flops"] / (prefill["ms"] * 1e-3) / 1e12
                          / float(peaks.get("bf16_tflops", 1590.0))}),
            "serving": {"what": "attention-only decode loop over %d layer(s): append 1 token + decode "
                                "attention per layer, %d sequences of %d tokens" % (L, w.B, T),
                        "tokens_per_s": whole_job_rate(w.B, ws, ms_per_step),
                        "graph_ms_per_step": graph_ms,
                        "graph_tokens_per_s": None if graph_ms is None else whole_job_rate(w.B, ws, graph_ms)},
        }
        if ws == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(w, tab_seed=0, seconds=args.cpu_seconds,
                                                  rate_offsets=(args.k_rate_offset, args.v_rate_offset),
                                                  drift_mode=args.drift_mode)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def decode_ms(dq, tab, w, kc, vc, T, stream, reps=5):
    """Median device time (ms) of dq_decode_attention over the whole cache
    (inputs larger than L2), after two untimed calls."""
    import torch

    from decode_attention_dq_b200 import synth
    q = torch.from_numpy(synth.q_block(w)).to(device=kc.device, dtype=w.torch_dtype)
    seq = torch.full((w.B,), T, dtype=torch.int32, device=kc.device)
    ws = torch.empty(dq.dq_decode_workspace_bytes(tab, w.B, w.Hq, w.Hkv, T), dtype=torch.uint8, device=kc.device)
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device=kc.device)
    stats = dq.new_stats(kc.device)
    for _ in range(2):
        dq.dq_decode_attention(tab, q, kc, vc, seq, T, out, ws, stream=stream)
    evs = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dq.dq_decode_attention(tab, q, kc, vc, seq, T, out, ws, stats=stats, stream=stream)
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in evs), dq.stats_dict(stats)["integrity_errors"]


def decode_report(ms, w, T, ck, cv, alu_peak, peaks):
    G = w.Hq // w.Hkv
    token_heads = w.B * T * w.Hkv
    achieved = token_heads * ops_per_token_head(G) / (ms * 1e-3) / 1e12
    gbs = token_heads * (ck + cv) / (ms * 1e-3) / 1e9
    return {"decode_ms": ms, "kv_tokens_per_s": w.B * T / (ms * 1e-3), "hbm_gbs": gbs,
            "hbm_frac": gbs / float(peaks.get("hbm_gbs", 6650.0)),
            "roofline": {"bound": "alu", "achieved": achieved, "peak": alu_peak, "unit": "Tlaneop/s",
                         "frac": achieved / alu_peak}}


def long_context_report(dq, args, dev, stream, dist, alu_peak, peaks):
    """The long-context workload (4 sequences x 8 KV heads x 32 query heads,
    2.26 bit/value): the full 65536-token prefill append of all 4 sequences
    in one call (containers/s), then split-K decode attention over 65536 and
    131072 tokens."""
    import torch

    from decode_attention_dq_b200 import synth
    res = {"what": "4 sequences x 8 KV heads, 2.26 bit/value: one dq_append_kv of 65536 tokens per "
                   "sequence (encode), and dq_decode_attention over 65536 and 131072 tokens"}
    for name in ("long_b4_t64k", "long_b4_t128k"):
        w = replica_workload(synth.WORKLOADS[name], int(os.environ.get("RANK", "0")))
        tab = dq.dq_build_tables(n_kv_heads=w.Hkv, k_bits_per_value=w.k_bits, v_bits_per_value=w.v_bits)
        ck, cv = tab.k.container_bytes, tab.v.container_bytes
        kc = torch.zeros((w.B, w.Hkv, w.T, ck), dtype=torch.uint8, device=dev)
        vc = torch.zeros((w.B, w.Hkv, w.T, cv), dtype=torch.uint8, device=dev)
        timings = [] if w.T == 65536 else None
        synth.prefill_cache(tab, w, kc, vc, w.T, seqs_per_call=w.B, threads=args.threads, timings=timings)
        ms, bad = decode_ms(dq, tab, w, kc, vc, w.T, stream)
        enc = None
        if timings:
            enc_ms = sum(a.elapsed_time(b) for a, b, _ in timings)
            enc = max_over_ranks([enc_ms], dist, dev)[0]
        ms = max_over_ranks([ms], dist, dev)[0]
        r = dict(decode_report(ms, w, w.T, ck, cv, alu_peak, peaks), integrity_errors=bad)
        if enc is not None:
            n = sum(n for _, _, n in timings)
            r["prefill_encode"] = {"ms": enc, "containers_per_s": 2 * n / (enc * 1e-3),
                                   "tokens_per_sequence": w.T, "sequences": w.B}
        res[name] = r
        del kc, vc, tab
    return res


def budget_sweep_report(dq, args, dev, stream, dist, alu_peak, peaks):
    """The Llama-3.1-8B-shaped workload (32 sequences x 8 KV heads x 32 query
    heads x 32768 tokens) at 1.96, 2.26 and 3.0 bit/value: the same seeded
    K/V encoded with each budget's tables (drift rate per stream), then
    decode attention over the 32768 tokens."""
    import torch

    from decode_attention_dq_b200 import synth
    base = replica_workload(synth.WORKLOADS["llama_b32_t32k_2p26"], int(os.environ.get("RANK", "0")))
    budgets = (1.96, 2.26, 3.0)
    tabs = [dq.dq_build_tables(n_kv_heads=base.Hkv, k_bits_per_value=b, v_bits_per_value=b) for b in budgets]
    caches = [(torch.zeros((base.B, base.Hkv, base.T, t.k.container_bytes), dtype=torch.uint8, device=dev),
               torch.zeros((base.B, base.Hkv, base.T, t.v.container_bytes), dtype=torch.uint8, device=dev))
              for t in tabs]
    stats = [dq.new_stats(dev) for _ in tabs]
    # The same inputs for every budget: drawn once per batch of sequences.
    for b0 in range(0, base.B, 8):
        b1 = min(base.B, b0 + 8)
        rows = [(b, h) for b in range(b0, b1) for h in range(base.Hkv)]
        kt = torch.from_numpy(synth.kv_block(base, "k", rows, n=base.T, threads=args.threads)).to(
            device=dev, dtype=base.torch_dtype).view(b1 - b0, base.Hkv, base.T, 128)
        vt = torch.from_numpy(synth.kv_block(base, "v", rows, n=base.T, threads=args.threads)).to(
            device=dev, dtype=base.torch_dtype).view(b1 - b0, base.Hkv, base.T, 128)
        start = torch.zeros(b1 - b0, dtype=torch.int32, device=dev)
        for t, (kc, vc), st in zip(tabs, caches, stats):
            dq.dq_append_kv(t, kt, vt, start, kc[b0:b1], vc[b0:b1], stats=st)
    torch.cuda.synchronize()
    out = []
    n_sym = base.B * base.Hkv * base.T * 128
    n_cont = base.B * base.Hkv * base.T
    for bits, t, (kc, vc), st in zip(budgets, tabs, caches, stats):
        ms, bad = decode_ms(dq, t, base, kc, vc, base.T, stream)
        ms = max_over_ranks([ms], dist, dev)[0]
        sd = dq.stats_dict(st)
        out.append(dict(decode_report(ms, base, base.T, t.k.container_bytes, t.v.container_bytes, alu_peak, peaks),
                        bits_per_value=bits, k_container_bytes=t.k.container_bytes,
                        v_container_bytes=t.v.container_bytes,
                        k_drift_syms_pct=100.0 * sd["k_syms_drifted"] / n_sym,
                        v_drift_syms_pct=100.0 * sd["v_syms_drifted"] / n_sym,
                        k_drift_cont_pct=100.0 * sd["k_cont_drifted"] / n_cont,
                        v_drift_cont_pct=100.0 * sd["v_cont_drifted"] / n_cont,
                        fallbacks=sd["overflow_fallbacks"], integrity_errors=bad))
    del caches
    return {"what": "32 sequences x 8 KV heads x 32768 tokens, the same seeded K/V encoded at each budget; "
                    "drift rates over the whole prefill, then dq_decode_attention over all tokens",
            "budgets": out}


def small_batch_latency(dq, tab, w, kc, vc, q, seq, T, stream, dist, dev, reps=20):
    """Device time of one dq_decode_attention call (prefix, split and combine
    kernels) over the first B sequences of the cache, B = 1 and 8, with L2
    flushed (a 256 MB write) before every call; median over `reps` calls,
    slowest rank."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    res = {}
    for B in (1, 8):
        if B > w.B:
            continue
        wsb = torch.empty(dq.dq_decode_workspace_bytes(tab, B, w.Hq, w.Hkv, T), dtype=torch.uint8, device=dev)
        o = torch.empty((B, w.Hq, 128), dtype=torch.float32, device=dev)
        for _ in range(3):
            dq.dq_decode_attention(tab, q[:B], kc[:B], vc[:B], seq[:B], T, o, wsb, stream=stream)
        evs = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            dq.dq_decode_attention(tab, q[:B], kc[:B], vc[:B], seq[:B], T, o, wsb, stream=stream)
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize()
        us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3
        us = max_over_ranks([us], dist, dev)[0]
        res["b%d" % B] = {"decode_us": us, "kv_tokens_per_s": B * T / (us * 1e-6),
                          "sequences": B, "context": T}
    res["what"] = ("one dq_decode_attention call over the first B sequences of the benchmark cache, "
                   "L2 flushed before each call, median of %d" % reps)
    return res


def encode_report(enc_ms, enc_vectors, w, ck, cv, alu_peak, peaks):
    """Throughput of dq_append_kv over the prefill (device time of the append
    calls only; host generation of the inputs is outside the events)."""
    if enc_ms <= 0:
        return None
    containers = 2 * enc_vectors
    s = enc_ms * 1e-3
    in_bytes = containers * 128 * (2 if w.dtype == "bf16" else 4)
    out_bytes = enc_vectors * (ck + cv)
    achieved = containers * ENCODE_OPS_PER_VECTOR / s / 1e12
    return {"what": "prefill append of %d tokens x %d sequences x %d KV heads (K and V)"
                    % (w.T - 1, w.B, w.Hkv),
            "ms": enc_ms, "containers_per_s": containers / s,
            "hbm_gbs": (in_bytes + out_bytes) / s / 1e9,
            "roofline": {"bound": "alu", "achieved": achieved, "peak": alu_peak, "unit": "Tlaneop/s",
                         "frac": achieved / alu_peak,
                         "hbm_frac": (in_bytes + out_bytes) / s / 1e9 / float(peaks.get("hbm_gbs", 6650.0))}}


def oracle_sample_step(w, tabs, rows, cache_rows):
    """One bounded sample of the step on the host oracle: append one token to
    each sampled row and decode-attend over its full context."""
    import numpy as np
    from oracle import oracle as o

    G = w.Hq // w.Hkv
    for (b, h), (kc, vc) in zip(rows, cache_rows):
        from decode_attention_dq_b200 import synth
        k_new = synth.kv_row(w, "k", b, h, n=1, step=0)
        v_new = synth.kv_row(w, "v", b, h, n=1, step=0)
        kk, _, _, _ = o.encode_vectors(tabs.k, tabs.signs, k_new, np.array([h], np.int32), tabs.drift_mode)
        vv, _, _, _ = o.encode_vectors(tabs.v, tabs.signs, v_new, np.array([h], np.int32), tabs.drift_mode)
        kc[-1] = kk[0]
        vc[-1] = vv[0]
        q = synth.q_rows(w, b)[h * G:(h + 1) * G]
        qb = np.zeros((1, w.Hkv * G, 128))
        qb[0, h * G:(h + 1) * G] = q
        kfull = np.zeros((1, w.Hkv) + kc.shape, np.uint8)
        vfull = np.zeros((1, w.Hkv) + vc.shape, np.uint8)
        kfull[0, h] = kc
        vfull[0, h] = vc
        o.attention_fp64(tabs, qb, kfull, vfull, [kc.shape[0]], rows=[(0, h)])


def host_cpu():
    """Model string and usable core count of the host CPU."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    ncores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    return model, ncores


def cpu_baseline(w, tab_seed=0, seconds=15.0, max_rows=512, rate_offsets=(0.0, 0.0), drift_mode=0):
    """The oracle, as it stands, on the host: a bounded sample of the step,
    once on one thread (BLAS limited to one thread too) and once on all host
    cores (a thread per (sequence, KV head) row; the oracle's C calls and
    numpy's kernels release the GIL). Besides the step (append one token +
    decode attention), the two halves of the path are timed on their own:
    encode (containers/s over sampled rows' tokens) and fp64 decode
    attention (KV tokens/s)."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np
    from threadpoolctl import threadpool_limits

    from decode_attention_dq_b200 import synth
    from oracle import oracle as o

    tabs = o.Tables(w.Hkv, k_container_bytes=o.container_bytes(w.k_bits),
                    v_container_bytes=o.container_bytes(w.v_bits), sign_seed=tab_seed,
                    k_rate_offset=rate_offsets[0], v_rate_offset=rate_offsets[1], drift_mode=drift_mode)
    model, ncores = host_cpu()
    G = w.Hq // w.Hkv
    with threadpool_limits(limits=1):
        # Sampled rows' inputs and their oracle containers (setup, untimed
        # except for the encode measurement below, which re-encodes them).
        rng = np.random.default_rng(0)
        cand = [(int(b), int(h)) for b, h in zip(rng.integers(0, w.B, max_rows), rng.integers(0, w.Hkv, max_rows))]

        def inputs(bh):
            b, h = bh
            return synth.kv_row(w, "k", b, h), synth.kv_row(w, "v", b, h)

        def encode(bh, kv):
            h = bh[1]
            kc, _, _, _ = o.encode_vectors(tabs.k, tabs.signs, kv[0], np.full(w.T, h, np.int32), tabs.drift_mode)
            vc, _, _, _ = o.encode_vectors(tabs.v, tabs.signs, kv[1], np.full(w.T, h, np.int32), tabs.drift_mode)
            return kc, vc

        prepared = []
        t_setup = time.time()
        with ThreadPoolExecutor(ncores) as ex:
            for i in range(0, len(cand), ncores):
                chunk = cand[i:i + ncores]
                kvs = list(ex.map(inputs, chunk))
                conts = list(ex.map(encode, chunk, kvs))
                # The raw inputs (8 MB a row at 8K) are kept for the first 16
                # rows only, for the encode measurement.
                n0 = len(prepared)
                prepared.extend((bh, cc, kv if n0 + i < 16 else None)
                                for i, (bh, cc, kv) in enumerate(zip(chunk, conts, kvs)))
                if time.time() - t_setup > seconds:
                    break
        budget = seconds / 4
        # Step (append one token + attention over the row), one thread.
        done = 0
        t0 = time.time()
        for (bh, cc, _) in prepared:
            oracle_sample_step(w, tabs, [bh], [cc])
            done += 1
            if time.time() - t0 > budget:
                break
        dt = time.time() - t0
        # Encode alone: the rows' T tokens of K and V, one thread.
        enc_rows = 0
        t1 = time.time()
        for (bh, _, kv) in prepared:
            if kv is None:
                break
            encode(bh, kv)
            enc_rows += 1
            if time.time() - t1 > budget:
                break
        dt_enc = time.time() - t1
        # Decode attention alone: G query heads over the row's T tokens, one thread.
        dec_rows = 0
        t2 = time.time()
        for (bh, cc, _) in prepared:
            b, h = bh
            qb = np.zeros((1, w.Hq, 128))
            qb[0, h * G:(h + 1) * G] = synth.q_rows(w, b)[h * G:(h + 1) * G]
            kfull = np.zeros((1, w.Hkv) + cc[0].shape, np.uint8)
            vfull = np.zeros((1, w.Hkv) + cc[1].shape, np.uint8)
            kfull[0, h] = cc[0]
            vfull[0, h] = cc[1]
            o.attention_fp64(tabs, qb, kfull, vfull, [w.T], rows=[(0, h)])
            dec_rows += 1
            if time.time() - t2 > budget:
                break
        dt_dec = time.time() - t2
        # All cores, the step over the same rows.
        rows = prepared[:max(done, min(len(prepared), ncores))]
        t3 = time.time()
        with ThreadPoolExecutor(ncores) as ex:
            list(ex.map(lambda p: oracle_sample_step(w, tabs, [p[0]], [p[1]]), rows))
        dt_all = time.time() - t3
    per_row = w.T / w.Hkv  # one KV token = one position across all KV heads
    return {"value": done * per_row / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "cpu_model": model, "nproc": ncores,
            "sample": "%d (sequence, KV head) rows of %s: append 1 token + fp64 decode attention over %d "
                      "tokens each, one thread, %.1f s" % (done, w.name, w.T, dt),
            "encode": {"containers_per_s": enc_rows * 2 * w.T / dt_enc, "cores": 1,
                       "sample": "%d rows x %d tokens, K and V, one thread, %.1f s" % (enc_rows, w.T, dt_enc)},
            "decode": {"kv_tokens_per_s": dec_rows * per_row / dt_dec, "cores": 1,
                       "sample": "%d rows: %d query heads over %d tokens, fp64, one thread, %.1f s"
                                 % (dec_rows, G, w.T, dt_dec)},
            "all_cores": {"value": len(rows) * per_row / dt_all, "unit": UNIT, "cores": ncores,
                          "sample": "%d rows, one thread per row, %.1f s" % (len(rows), dt_all)}}


PREFILL_METRIC = "chunked-prefill attention over the compressed KV cache: query tokens/s"
PREFILL_UNIT = "query tokens/s"
# Useful tensor work per (query row, visible key): q.k and p.v, 128
# multiply-adds each.
FLOPS_PER_PAIR = 4 * 128
# Kernel launches of one prefill step: dq_append_kv of the chunk (encode +
# drift kernels; in drift mode 1 the drift kernel runs once per stream) and
# dq_prefill_attention (tile decode + attention kernels).
PREFILL_LAUNCHES_PER_STEP = 4


def prefill_launches_per_step(drift_mode):
    return PREFILL_LAUNCHES_PER_STEP + (1 if drift_mode == 1 else 0)


# DRAM traffic of prefill_kernel (the dominant kernel of the prefill step)
# from one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum, one
# pass) of `bench.py --prefill 512 --workload qwen3_8b_b16_t8k`: the decoded
# tiles read once (545 MB) plus the queries, and the fp32 output. Reported
# only for that workload and container size while the kernel source matches.
# (Captured at source hash ea5171e9edcc4ac1; the file has changed since in
# one comment only.)
PREFILL_TRAFFIC = {"source": "decode_attention_dq_b200/csrc/dq_prefill.cu", "sha256_16": "4c3e896135d811ad",
                   "workload": "qwen3_8b_b16_t8k", "chunk": 512, "ck": 36, "cv": 36,
                   "bytes": 617.33e6 + 129.95e6}


def prefill_traffic(workload, n_q, ck, cv):
    import hashlib
    t = PREFILL_TRAFFIC
    try:
        with open(os.path.join(ROOT, t["source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    if sha != t["sha256_16"] or (workload, n_q, ck, cv) != (t["workload"], t["chunk"], t["ck"], t["cv"]):
        return None
    return t["bytes"]


def chunk_pairs(B, Hq, q_start, n_q):
    """(query row, visible key) pairs of a causal chunk: sum over its query
    tokens i of (q_start + i + 1) keys, for every sequence and query head."""
    return B * Hq * (n_q * (q_start + 1) + n_q * (n_q - 1) // 2)


def run_prefill(args):
    """One step = append an n_q-token chunk to every sequence (dq_append_kv)
    + chunked-prefill attention of its n_q queries over the context, the
    chunk itself included (dq_prefill_attention); the chunk is the last
    n_q positions of the workload's context."""
    import numpy as np
    import torch

    import decode_attention_dq_b200 as dq
    from decode_attention_dq_b200 import synth

    ws, rank, local = dist_setup(args)
    dist = None
    if ws > 1:
        import torch.distributed as dist
    w = replica_workload(synth.WORKLOADS[args.workload], rank)
    dev = torch.device("cuda", torch.cuda.current_device())
    tab = dq.dq_build_tables(n_kv_heads=w.Hkv, k_bits_per_value=w.k_bits, v_bits_per_value=w.v_bits,
                             drift_mode=args.drift_mode, k_rate_offset=args.k_rate_offset,
                             v_rate_offset=args.v_rate_offset)
    ck, cv = tab.k.container_bytes, tab.v.container_bytes
    T, n_q = w.T, args.prefill
    q_start = T - n_q
    T_cap = (T + 31) // 32 * 32
    kc = torch.zeros((w.B, w.Hkv, T_cap, ck), dtype=torch.uint8, device=dev)
    vc = torch.zeros((w.B, w.Hkv, T_cap, cv), dtype=torch.uint8, device=dev)
    synth.prefill_cache(tab, w, kc, vc, q_start, threads=args.threads)
    rows = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    # The chunk's tokens: a seeded stream of their own (step index 1 of the
    # generator), and its queries.
    host_k = torch.from_numpy(synth.kv_block(w, "k", rows, n=n_q, step=1, threads=args.threads)
                              ).to(w.torch_dtype).view(w.B, w.Hkv, n_q, 128).pin_memory()
    host_v = torch.from_numpy(synth.kv_block(w, "v", rows, n=n_q, step=1, threads=args.threads)
                              ).to(w.torch_dtype).view(w.B, w.Hkv, n_q, 128).pin_memory()
    host_q = torch.from_numpy(synth.q_chunk(w, n_q)).to(w.torch_dtype).pin_memory()
    dk, dv, dqq = host_k.to(dev), host_v.to(dev), host_q.to(dev)
    out = torch.empty((w.B, n_q, w.Hq, 128), dtype=torch.float32, device=dev)
    out_host = torch.empty_like(out, device="cpu").pin_memory()
    start = torch.full((w.B,), q_start, dtype=torch.int32, device=dev)
    app_ws = torch.empty(max(16, dq.dq_append_workspace_bytes(tab, w.B, w.Hkv, n_q)), dtype=torch.uint8,
                         device=dev)
    pf_ws = torch.empty(dq.dq_prefill_workspace_bytes(tab, w.B, w.Hkv, T_cap), dtype=torch.uint8, device=dev)
    stats = dq.new_stats(dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        dq.dq_append_kv(tab, dk, dv, start, kc, vc, stats=stats, workspace=app_ws)
        if ev is not None:
            ev[0].record(stream)
        dq.dq_prefill_attention(tab, dqq, kc, vc, start, out, workspace=pf_ws, stats=stats)
        if ev is not None:
            ev[1].record(stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for s in range(args.steps):
        step(evs[s])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    elapsed_ms = e0.elapsed_time(e1)
    attn_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    elapsed_ms, attn_ms = max_over_ranks([elapsed_ms, attn_ms], dist, dev)
    ms_per_step = elapsed_ms / args.steps
    qtok = w.B * n_q
    value = whole_job_rate(qtok, ws, ms_per_step)

    # End to end: the chunk's K/V and q in from pinned host memory and the
    # output back every step, pipelined with the kernels (run_pipelined) over
    # two device buffer sets.
    bufs = [(dk, dv, dqq, out), (torch.empty_like(dk), torch.empty_like(dv), torch.empty_like(dqq),
                                 torch.empty_like(out))]
    outs_host = [out_host, torch.empty_like(out_host).pin_memory()]

    def e2e_h2d(s):
        bk, bv, bq, _ = bufs[s % 2]
        bk.copy_(host_k, non_blocking=True)
        bv.copy_(host_v, non_blocking=True)
        bq.copy_(host_q, non_blocking=True)

    def e2e_compute(s):
        bk, bv, bq, bo = bufs[s % 2]
        dq.dq_append_kv(tab, bk, bv, start, kc, vc, stats=stats, workspace=app_ws)
        dq.dq_prefill_attention(tab, bq, kc, vc, start, bo, workspace=pf_ws, stats=stats)

    def e2e_d2h(s):
        outs_host[s % 2].copy_(bufs[s % 2][3], non_blocking=True)

    run_pipelined(2, stream, 2, 2, e2e_h2d, e2e_compute, e2e_d2h)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run_pipelined(args.steps, stream, 2, 2, e2e_h2d, e2e_compute, e2e_d2h, f0, f1)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks([f0.elapsed_time(f1)], dist, dev)[0]
    st = dq.stats_dict(stats)
    result = None
    if rank == 0:
        peaks, src = measured_peaks()
        flops = chunk_pairs(w.B, w.Hq, q_start, n_q) * FLOPS_PER_PAIR
        achieved = flops / (attn_ms * 1e-3) / 1e12
        peak = float(peaks.get("bf16_tflops", 1590.0))
        peak_sus = float(peaks.get("bf16_tflops_sustained", peak))
        comp_bytes = w.B * w.Hkv * T * (ck + cv)
        io_bytes = 2 * dqq.numel() * dqq.element_size() + out.numel() * out.element_size()
        h2d = (host_k.numel() + host_v.numel() + host_q.numel()) * host_k.element_size()
        result = {
            "metric": PREFILL_METRIC, "value": value, "unit": PREFILL_UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16x2 tensor / f32", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hkv": w.Hkv, "Hq": w.Hq, "head_dim": 128,
                       "context": T, "chunk": n_q, "q_start": q_start, "input_dtype": w.dtype,
                       "k_container_bytes": ck, "v_container_bytes": cv, "drift_mode": args.drift_mode,
                       "rate_offsets": [args.k_rate_offset, args.v_rate_offset],
                       "l2": "inputs larger than L2 (%.0f MB of containers, %.0f MB of queries and outputs)"
                             % (comp_bytes / 1e6, io_bytes / 1e6),
                       "parallelism": "replicas x%d" % ws},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "frac_of_sustained": achieved / peak_sus,
                         "traffic": prefill_traffic(w.name, n_q, ck, cv),
                         "traffic_note": "prefill_kernel DRAM bytes per launch from one ncu capture of this "
                                         "workload; algorithmic bytes: containers once + q + out",
                         "algorithmic_bytes": comp_bytes + io_bytes,
                         "useful_flops": flops, "flops_convention": "4 x 128 per (query row, visible key)",
                         "kernel": "prefill_tiles_kernel + prefill_kernel (dq_prefill_attention)",
                         "kernel_ms": attn_ms,
                         "peak_source": "%s bf16 dense GEMM (fp16 runs at the same rate)" % src},
            "e2e": {"value": whole_job_rate(qtok, ws, e2e_ms / args.steps), "unit": PREFILL_UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
                    "copies": "every step's inputs in and output out, on upload and read-back streams "
                              "pipelined with the kernels"},
            "gpu_launches": prefill_launches_per_step(args.drift_mode) * args.steps,
            "clocks": clk,
            "integrity_errors": st["integrity_errors"], "wait_timeouts": st["wait_timeouts"],
        }
        if ws == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = prefill_cpu_baseline(w, n_q, seconds=args.cpu_seconds,
                                                          rate_offsets=(args.k_rate_offset, args.v_rate_offset),
                                                          drift_mode=args.drift_mode)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def prefill_row_inputs(w, bh, n_q):
    """The chunk's K, V and queries for one (sequence, KV head) row (host
    generation, done outside the timed region)."""
    import numpy as np

    from decode_attention_dq_b200 import synth
    b, h = bh
    G = w.Hq // w.Hkv
    q = np.zeros((1, n_q, w.Hq, 128))
    q[0, :, h * G:(h + 1) * G] = np.stack([synth.q_rows(w, b, i)[h * G:(h + 1) * G] for i in range(n_q)])
    return synth.kv_row(w, "k", b, h, n=n_q, step=1), synth.kv_row(w, "v", b, h, n=n_q, step=1), q


def oracle_prefill_row(w, tabs, bh, n_q, ctx, inputs):
    """The oracle's prefill step for one (sequence, KV head) row: encode the
    chunk's K and V, then fp64 causal attention of the chunk's queries (the G
    heads of this KV head) over context + chunk."""
    import numpy as np

    from oracle import oracle as o
    b, h = bh
    kc, vc = ctx
    k_new, v_new, q = inputs
    T = kc.shape[0]
    hh = np.full(n_q, h, np.int32)
    kk, _, _, _ = o.encode_vectors(tabs.k, tabs.signs, k_new, hh, tabs.drift_mode)
    vv, _, _, _ = o.encode_vectors(tabs.v, tabs.signs, v_new, hh, tabs.drift_mode)
    kfull = np.zeros((1, w.Hkv, T, kc.shape[1]), np.uint8)
    vfull = np.zeros((1, w.Hkv, T, vc.shape[1]), np.uint8)
    kfull[0, h, :T - n_q] = kc[:T - n_q]
    vfull[0, h, :T - n_q] = vc[:T - n_q]
    kfull[0, h, T - n_q:] = kk
    vfull[0, h, T - n_q:] = vv
    o.attention_prefill_fp64(tabs, q, kfull, vfull, [T - n_q], rows=[(0, h)])


def prefill_contexts(w, tabs, n_rows, seconds, n_q=0):
    """Oracle containers of the context of sampled rows and, with n_q, the
    rows' chunk inputs (setup, untimed): [((b, h), (kc, vc), inputs)]."""
    import numpy as np

    from decode_attention_dq_b200 import synth
    from oracle import oracle as o
    rows = [(s % w.B, (s * 3) % w.Hkv) for s in range(n_rows)]
    out = []
    t0 = time.time()
    for b, h in rows:
        K = synth.kv_row(w, "k", b, h)
        V = synth.kv_row(w, "v", b, h)
        kc, _, _, _ = o.encode_vectors(tabs.k, tabs.signs, K, np.full(w.T, h, np.int32), tabs.drift_mode)
        vc, _, _, _ = o.encode_vectors(tabs.v, tabs.signs, V, np.full(w.T, h, np.int32), tabs.drift_mode)
        out.append(((b, h), (kc, vc), prefill_row_inputs(w, (b, h), n_q) if n_q else None))
        if time.time() - t0 > seconds:
            break
    return out


def prefill_cpu_baseline(w, n_q, seconds=12.0, rate_offsets=(0.0, 0.0), drift_mode=0):
    """The oracle's prefill step on one host thread (BLAS limited to one
    thread), on a bounded sample of (sequence, KV head) rows."""
    from threadpoolctl import threadpool_limits

    from oracle import oracle as o
    tabs = o.Tables(w.Hkv, k_container_bytes=o.container_bytes(w.k_bits),
                    v_container_bytes=o.container_bytes(w.v_bits), k_rate_offset=rate_offsets[0],
                    v_rate_offset=rate_offsets[1], drift_mode=drift_mode)
    from concurrent.futures import ThreadPoolExecutor
    ncores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    with threadpool_limits(limits=1):
        ctx = prefill_contexts(w, tabs, 16, seconds / 2, n_q)
        done = 0
        t0 = time.time()
        for bh, cc, inp in ctx:
            oracle_prefill_row(w, tabs, bh, n_q, cc, inp)
            done += 1
            if time.time() - t0 > seconds / 2:
                break
        dt = time.time() - t0
        # All cores: a thread per row (the oracle's C calls and numpy release the GIL).
        rows = ctx[:max(done, min(len(ctx), ncores))]
        t1 = time.time()
        with ThreadPoolExecutor(ncores) as ex:
            list(ex.map(lambda p: oracle_prefill_row(w, tabs, p[0], n_q, p[1], p[2]), rows))
        dt_all = time.time() - t1
    return {"value": done * n_q / w.Hkv / dt, "unit": PREFILL_UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d (sequence, KV head) rows of %s: encode a %d-token chunk + fp64 causal attention of "
                      "its queries over %d tokens, one thread, %.1f s" % (done, w.name, n_q, w.T, dt),
            "all_cores": {"value": len(rows) * n_q / w.Hkv / dt_all, "unit": PREFILL_UNIT, "cores": ncores,
                          "sample": "%d rows, one thread per row, %.1f s" % (len(rows), dt_all)}}


def run_reference_prefill(args, w):
    """Reference arm of the prefill mode: the oracle's prefill step, one
    (sequence, KV head) row per step, one thread."""
    from threadpoolctl import threadpool_limits

    from oracle import oracle as o
    n_q = args.prefill
    tabs = o.Tables(w.Hkv, k_container_bytes=o.container_bytes(w.k_bits),
                    v_container_bytes=o.container_bytes(w.v_bits), k_rate_offset=args.k_rate_offset,
                    v_rate_offset=args.v_rate_offset, drift_mode=args.drift_mode)
    with threadpool_limits(limits=1):
        ctx = prefill_contexts(w, tabs, args.warmup + args.steps, 1e9, n_q)
        for i in range(args.warmup):
            oracle_prefill_row(w, tabs, ctx[i][0], n_q, ctx[i][1], ctx[i][2])
        t0 = time.time()
        for i in range(args.warmup, args.warmup + args.steps):
            oracle_prefill_row(w, tabs, ctx[i][0], n_q, ctx[i][1], ctx[i][2])
        dt = time.time() - t0
    value = args.steps * n_q / w.Hkv / dt
    sample = ("per step: one (sequence, KV head) row of %s, encode a %d-token chunk + fp64 causal attention "
              "over %d tokens, single thread" % (w.name, n_q, w.T))
    return {"impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": PREFILL_UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hkv": w.Hkv, "Hq": w.Hq, "head_dim": 128,
                       "context": w.T, "chunk": n_q, "sample_per_step": "one (sequence, KV head) row",
                       "drift_mode": args.drift_mode, "rate_offsets": [args.k_rate_offset, args.v_rate_offset]},
            "cpu_baseline": {"value": value, "unit": PREFILL_UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": PREFILL_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference(args):
    """Reference arm: the CPU oracle on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    from decode_attention_dq_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.prefill:
        return run_reference_prefill(args, w)
    import numpy as np
    from oracle import oracle as o
    tabs = o.Tables(w.Hkv, k_container_bytes=o.container_bytes(w.k_bits),
                    v_container_bytes=o.container_bytes(w.v_bits), k_rate_offset=args.k_rate_offset,
                    v_rate_offset=args.v_rate_offset, drift_mode=args.drift_mode)
    rows = [(s % w.B, (s * 3) % w.Hkv) for s in range(args.warmup + args.steps)]
    prepared = []
    for b, h in rows:
        K = synth.kv_row(w, "k", b, h)
        V = synth.kv_row(w, "v", b, h)
        kc, _, _, _ = o.encode_vectors(tabs.k, tabs.signs, K, np.full(w.T, h, np.int32), tabs.drift_mode)
        vc, _, _, _ = o.encode_vectors(tabs.v, tabs.signs, V, np.full(w.T, h, np.int32), tabs.drift_mode)
        prepared.append(((b, h), (kc, vc)))
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):  # one thread, BLAS included
        for i in range(args.warmup):
            oracle_sample_step(w, tabs, [prepared[i][0]], [prepared[i][1]])
        t0 = time.time()
        for i in range(args.warmup, args.warmup + args.steps):
            oracle_sample_step(w, tabs, [prepared[i][0]], [prepared[i][1]])
        dt = time.time() - t0
    kv_tokens = args.steps * w.T / w.Hkv
    value = kv_tokens / dt
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hkv": w.Hkv, "Hq": w.Hq, "head_dim": 128,
                       "context": w.T, "sample_per_step": "one (sequence, KV head) row",
                       "drift_mode": args.drift_mode, "rate_offsets": [args.k_rate_offset, args.v_rate_offset]},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": "per step: one (sequence, KV head) row of %s, append 1 token "
                                       "+ fp64 attention over %d tokens, single thread" % (w.name, w.T)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="dq", choices=["dq", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--threads", type=int, default=max(4, min(32, os.cpu_count() or 8)))
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", dest="extra", action="store_false",
                    help="skip the long-context and budget-sweep workloads")
    ap.add_argument("--paged", action="store_true", help="page pools and a shuffled page table")
    ap.add_argument("--layers", type=int, default=1, help="layers of the decode loop (one cache each)")
    ap.add_argument("--graph", action="store_true", help="also time the step captured as a CUDA graph")
    ap.add_argument("--prefill-chunk", type=int, default=512, metavar="N_Q",
                    help="also time chunked prefill of the last N_Q positions over the decode cache (0: off)")
    ap.add_argument("--k-rate-offset", type=float, default=0.0,
                    help="K table target rate above the container's nominal rate (bit/value)")
    ap.add_argument("--v-rate-offset", type=float, default=0.0,
                    help="V table target rate above the container's nominal rate (bit/value)")
    ap.add_argument("--drift-mode", type=int, default=0, choices=[0, 1],
                    help="0: drift only (default); 1: drift, then the rate-distortion fill")
    ap.add_argument("--prefill", type=int, default=0, metavar="N_Q",
                    help="chunked-prefill mode: append an N_Q-token chunk and attend its queries causally")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        res = run_reference(args)
    else:
        res = run_prefill(args) if args.prefill else run_dq(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
