"""GQLA decode-attention benchmark (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--sq 1|2] [--impl ours|reference]

Workload: the LLaMA-3-8B-shaped GQLA layer (n_h 32, G 8, d_nope 128, d_rope
64, d_v 128, r 512), batch 32, uniform context 8192, s_q new tokens per
sequence, bf16, synthetic seeded inputs.  One step is one pass of the whole
decode hot path over that batch: the decode-time expansion of the s_q new
tokens into the per-group cache, the MQA-absorb decode and the GQA decode
(both paths produce the batch's B*s_q output tokens).  value = decoded tokens
(B*s_q per step, per GPU) / device time.  Under torchrun every rank decodes
its own batch (weak scaling; sequences are independent, no data-path
collective); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the reference arm of this build)
on the same workload, one bounded sample of (sequence, group) units per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attention tokens/s per layer and % of roofline (HBM GB/s or TC util), 1×B200"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--sq", type=int, default=1, choices=[1, 2])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches only")
    ap.add_argument("--tp", action="store_true",
                    help="with --gpus N > 1: split the groups of one batch over the ranks (strong scaling) "
                         "instead of giving every rank its own batch")
    ap.add_argument("--sweep", choices=["crossover", "context", "ragged", "capacity"],
                    help="instead of the headline line, time both decode paths over a workload sweep "
                         "(one JSON line per point)")
    return ap.parse_args()


def workload(s_q):
    from latent_kv_cache_flash_b200 import synth
    return synth.llama3_8b(s_q=s_q)


def algorithmic(wl):
    """Per-step algorithmic bytes and flops of each path (the method's own
    traffic: cache bytes read once per step, q/out/weights ignored)."""
    d = wl.dims
    T = wl.batch * wl.seq_len
    keys = sum(wl.seq_len - d.s_q + i + 1 for i in range(d.s_q)) * wl.batch   # (query, key) pairs per head
    absorb_bytes = 2 * T * (d.r + d.d_rope)
    absorb_flops = d.n_h * keys * 2 * (2 * d.r + d.d_rope) + wl.batch * d.s_q * d.n_h * 2 * d.r * (d.d_nope + d.d_v)
    gqa_bytes = 2 * T * d.G * (d.d_qk + d.d_v)
    gqa_flops = d.n_h * keys * 2 * (d.d_qk + d.d_v)
    gqa_shared_bytes = 2 * T * (d.G * (d.d_nope + d.d_v) + d.d_rope)
    return dict(absorb_bytes=absorb_bytes, absorb_flops=absorb_flops, gqa_bytes=gqa_bytes, gqa_flops=gqa_flops,
                gqa_shared_bytes=gqa_shared_bytes)


# ---------------------------------------------------------------- clocks ---
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.idx = gpu_index
        self.path = os.path.join(ROOT, "gpurun_out", "clocks_bench.csv") if os.path.isdir(
            os.path.join(ROOT, "gpurun_out")) else "/tmp/gqla_clocks.csv"

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-i", str(self.idx), "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------- cpu baseline ---
def oracle_sample(inp, units, both_forms=True):
    """Runs the oracle on (sequence, group) units; returns seconds."""
    import numpy as np
    from oracle import gqla_oracle as O
    d = inp.dims
    W_uk = inp.W_uk.double().cpu().numpy()
    W_uv = inp.W_uv.double().cpu().numpy()
    t0 = time.perf_counter()
    for b, g in units:
        rows = inp.logical_latent(b).double().cpu().numpy()
        qb = inp.q[b].double().cpu().numpy()
        L = inp.seq_lens_host[b]
        O.decode_sequence_gqa(qb, rows[:, :d.r], rows[:, d.r:], W_uk, W_uv, L, d.softmax_scale, groups=[g])
        if both_forms:
            O.decode_sequence_absorb(qb, rows[:, :d.r], rows[:, d.r:], W_uk, W_uv, L, d.softmax_scale, groups=[g])
    return time.perf_counter() - t0


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(inp, budget_s=12.0):
    wl = inp.wl
    d = wl.dims
    all_units = [(b, g) for b in range(wl.batch) for g in range(d.G)]
    import random
    rnd = random.Random(0)
    rnd.shuffle(all_units)
    done, spent = 0, 0.0
    while done < len(all_units) and (spent < budget_s or done < 2):
        spent += oracle_sample(inp, [all_units[done]])
        done += 1
    per_step = spent / done * len(all_units)
    return {"value": wl.batch * d.s_q / per_step, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": "%d of %d (sequence, group) units of %s (B%d L%d s_q%d), fp64 expanded and absorb forms, "
                      "%.1f s, extrapolated linearly to the whole batch" % (
                          done, len(all_units), wl.name, wl.batch, wl.seq_len, d.s_q, spent)}


# ----------------------------------------------------------- reference ---
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import torch
    from latent_kv_cache_flash_b200 import synth
    wl = workload(args.sq)
    inp = synth.make_inputs(wl, "cpu")
    d = wl.dims
    all_units = [(b, g) for b in range(wl.batch) for g in range(d.G)]
    # one unit per step keeps the whole run within a few minutes
    for w in range(args.warmup):
        oracle_sample(inp, [all_units[w % len(all_units)]])
    t = 0.0
    for s in range(args.steps):
        t += oracle_sample(inp, [all_units[(args.warmup + s) % len(all_units)]])
    per_unit = t / args.steps
    step_s = per_unit * len(all_units)
    value = wl.batch * d.s_q / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "%s B%d L%d s_q%d" % (wl.name, wl.batch, wl.seq_len, d.s_q), "batch": wl.batch,
                       "seq_len": wl.seq_len, "s_q": d.s_q, "n_h": d.n_h, "G": d.G, "r": d.r},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": "one (sequence, group) unit per step, fp64 expanded and absorb forms, "
                                       "extrapolated to %d units per step" % len(all_units)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ours ---
def kernel_sha(files):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "latent_kv_cache_flash_b200", "csrc")
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(name):
    """DRAM bytes per launch from the committed ncu record of this kernel, or
    None when the kernel's sources changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        rec = json.load(open(p)).get(name)
        if not rec or rec.get("source_sha") != kernel_sha(rec["files"]):
            return None
    except Exception:
        return None
    return rec.get("bytes_per_launch")


def run_ours(args):
    import torch
    import torch.distributed as dist
    from latent_kv_cache_flash_b200 import build, gqla, synth

    from latent_kv_cache_flash_b200 import multi
    rank, local, world = multi.rank_info()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (no CPU fallback)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    build.build()
    hbm, tf_burst, tf_sust, peak_src = load_peaks()

    wl = workload(args.sq)
    tp = args.tp and world > 1
    if not tp:
        wl.seed = multi.rank_seed(wl.seed, rank)   # replicas: every rank its own batch
    inp = synth.make_inputs(wl, dev)
    if tp:
        inp = multi.tp_shard(inp, world, rank)    # the same batch; this rank's groups and heads
        wl = inp.wl
    d = wl.dims
    dims = gqla.make_dims(d)
    lay = gqla.make_layout(inp.seq_lens, inp.max_seq_len, 0, inp.capacity, None, 0)
    ks, vs = synth.expanded_pool_shapes(inp)
    kp = torch.empty(ks, dtype=d.torch_dtype, device=dev)
    vp = torch.empty(vs, dtype=d.torch_dtype, device=dev)
    B = wl.batch
    out_a = torch.empty((B, d.s_q, d.n_h, d.d_v), dtype=d.torch_dtype, device=dev)
    out_g = torch.empty_like(out_a)
    lse_a = torch.empty((B, d.s_q, d.n_h), device=dev)
    lse_g = torch.empty_like(lse_a)
    # the absorb workspace sized for any split count the step may use
    ws_a = gqla.workspace_for(dims, lay, 8, gqla.GQLA_PATH_ABSORB, dev)
    ws_a0 = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_ABSORB, dev)
    if ws_a0.numel() > ws_a.numel():
        ws_a = ws_a0
    del ws_a0
    absorb_splits = [0]            # 0 = the library's plan for the whole GPU
    gqa_splits = [0]
    ws_g = gqla.workspace_for(dims, lay, 8, gqla.GQLA_PATH_GQA, dev)
    ws_g0 = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_GQA, dev)
    if ws_g0.numel() > ws_g.numel():
        ws_g = ws_g0
    del ws_g0
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # the resident per-group cache of all tokens (a prefill-time cost, timed on its own)
    gqla.gqla_expand_cache(dims, lay, inp.latent, inp.W_uk, inp.W_uv, kp, vp, 0, status)
    # the step's new tokens [c_KV ; k_rope], resident on the device; each step
    # writes them into the latent pool (they are the rows already there, so
    # every step sees the same cache)
    Lmax = wl.seq_len
    new_rows = inp.latent[:, Lmax - d.s_q:Lmax].contiguous()

    def append_latent():
        gqla.gqla_append_tokens(dims, lay, new_rows, inp.latent, dev_status=status)

    def append():
        # the new rows into the latent pool, then their expansion into the per-group pools
        gqla.gqla_append_tokens(dims, lay, new_rows, inp.latent, inp.W_uk, inp.W_uv, kp, vp, dev_status=status)

    def expand_new():
        # the new rows' expansion alone (no latent pool argument)
        gqla.gqla_append_tokens(dims, lay, new_rows, None, inp.W_uk, inp.W_uv, kp, vp, dev_status=status)

    def expand_tail():
        gqla.gqla_expand_cache(dims, lay, inp.latent, inp.W_uk, inp.W_uv, kp, vp, d.s_q, status)

    def absorb():
        gqla.gqla_decode_absorb(dims, lay, inp.q, inp.latent, inp.W_uk, inp.W_uv, out_a, lse_a, absorb_splits[0],
                                ws_a, status)

    def gqa():
        gqla.gqla_decode_gqa(dims, lay, inp.q, kp, vp, out_g, lse_g, gqa_splits[0], ws_g, status)

    def step():
        append()
        absorb()
        gqa()

    # The two paths of a step share no data once the new tokens are in the
    # pools: the absorb path runs on a second stream, forked from and joined
    # back into the main one, so its CTAs and the GQA path's share the machine.
    side = torch.cuda.Stream(dev)

    def step_overlapped(after_absorb=None, after_gqa=None):
        main = torch.cuda.current_stream(dev)   # the capture stream while a graph is recorded
        append_latent()                         # what the absorb path needs ...
        fork = torch.cuda.Event()
        fork.record(main)
        side.wait_event(fork)
        with torch.cuda.stream(side):
            absorb()
            if after_absorb:
                after_absorb()                  # e.g. its output's copy to the host, on the same stream
        expand_new()                            # ... and what the GQA path needs, beside the absorb call
        gqa()
        if after_gqa:
            after_gqa()
        join = torch.cuda.Event()
        join.record(side)
        main.wait_event(join)

    barrier = multi.barrier

    def timed(fn, n):
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return multi.max_over_ranks(e0.elapsed_time(e1), dev)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    n0 = gqla.gqla_launch_counter()
    eager_ms = timed(step, args.steps) / args.steps
    launches = gqla.gqla_launch_counter() - n0
    # the same step captured once as a CUDA graph and replayed (no host
    # launch gaps between the kernels); every kernel still runs each step
    graph = None
    tuned = None
    if not args.no_graph:
        def capture():
            for _ in range(3):
                step_overlapped()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step_overlapped()
            for _ in range(3):
                g.replay()
            return g

        # The split plan of a call assumes it has the whole GPU; in the
        # overlapped step the two decode calls share it, so their split counts
        # are tuned here: each candidate pair's graph is timed (outside the
        # reported region) and the fastest pair is kept.
        tuned = {}
        plan_a = gqla.gqla_num_splits(dims, lay, 0, gqla.GQLA_PATH_ABSORB)
        plan_g = gqla.gqla_num_splits(dims, lay, 0, gqla.GQLA_PATH_GQA)
        for ca in [0] + [c for c in (1, 2, 4) if c != plan_a]:
            for cg in [0] + [c for c in (1, 2, 4, 8) if c != plan_g]:
                absorb_splits[0], gqa_splits[0] = ca, cg
                g = capture()
                tuned[(ca, cg)] = timed(g.replay, 30) / 30
                del g
        absorb_splits[0], gqa_splits[0] = min(tuned, key=tuned.get)
        graph = capture()
        ms_step = timed(graph.replay, args.steps) / args.steps
    else:
        ms_step = eager_ms
    # per-call breakdown (each over at least ~0.3 s of device time)
    reps = args.steps if args.no_clocks else max(args.steps, int(300.0 / max(ms_step, 1e-3)))
    step_splits = (absorb_splits[0], gqa_splits[0])
    absorb_splits[0] = gqa_splits[0] = 0   # alone, each call takes the library's own plan
    ms_absorb = timed(absorb, reps) / reps
    ms_gqa = timed(gqa, reps) / reps
    ms_tail = timed(expand_tail, reps) / reps
    ms_append = timed(append_latent, reps) / reps
    ms_append_expand = timed(append, reps) / reps
    ms_expand_full = timed(lambda: gqla.gqla_expand_cache(dims, lay, inp.latent, inp.W_uk, inp.W_uv, kp, vp, 0,
                                                          status), 10) / 10
    # the GQA call over the same cache with the RoPE key stored once per token
    # row (a second, smaller K pool; V is shared)
    dims_s = gqla.make_dims(dataclasses.replace(d, k_shared_rope=True))
    kp_s = torch.empty(tuple(ks[:2]) + (d.G * d.d_nope + d.d_rope,), dtype=d.torch_dtype, device=dev)
    gqla.gqla_expand_cache(dims_s, lay, inp.latent, inp.W_uk, inp.W_uv, kp_s, vp, 0, status)
    ms_gqa_s = timed(lambda: gqla.gqla_decode_gqa(dims_s, lay, inp.q, kp_s, vp, out_g, lse_g, 0, ws_g, status),
                     reps) / reps
    del kp_s

    # end to end through the public API with host buffers: the step's new
    # inputs (queries and the new tokens' latent rows) go host->device, both
    # paths' outputs come back device->host, inside the timed region
    q_host = inp.q.cpu().pin_memory()
    new_rows_host = new_rows.cpu().pin_memory()
    out_host = torch.empty((2,) + tuple(out_a.shape), dtype=out_a.dtype).pin_memory()

    def e2e_body(run_step):
        inp.q.copy_(q_host, non_blocking=True)
        new_rows.copy_(new_rows_host, non_blocking=True)
        run_step()
        out_host[0].copy_(out_a, non_blocking=True)
        out_host[1].copy_(out_g, non_blocking=True)

    def e2e_body_overlapped():
        # each path's output goes to the host as soon as that path is done
        inp.q.copy_(q_host, non_blocking=True)
        new_rows.copy_(new_rows_host, non_blocking=True)
        step_overlapped(after_absorb=lambda: out_host[0].copy_(out_a, non_blocking=True),
                        after_gqa=lambda: out_host[1].copy_(out_g, non_blocking=True))

    absorb_splits[0], gqa_splits[0] = step_splits
    # the copies and the step's calls recorded once as a CUDA graph (the copies
    # read and write the pinned host buffers on every replay), then one replay
    # and a host wait per step
    e2e_graph = None
    if graph is not None:
        torch.cuda.synchronize()
        e2e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e2e_graph):
            e2e_body_overlapped()

    def e2e_step():
        if e2e_graph is not None:
            e2e_graph.replay()
        else:
            e2e_body(step)
        torch.cuda.current_stream(dev).synchronize()

    for _ in range(3):
        e2e_step()
    e2e_ms = timed(e2e_step, args.steps) / args.steps
    clk = clocks.stop() if clocks else None
    torch.cuda.synchronize()
    st = int(status.item())
    if st != 0:
        raise SystemExit("device status 0x%x during the bench" % st)

    alg = algorithmic(wl)
    tokens = B * d.s_q
    # replicas decode world batches per step; tensor-parallel ranks share one
    value = multi.job_tokens_per_s(tokens, 1, 1 if tp else world, ms_step)
    # dominant kernel: the slower decode call of the step
    if ms_gqa >= ms_absorb:
        name, ms_dom, bytes_dom = "gqla_decode_gqa", ms_gqa, alg["gqa_bytes"]
        roof = {"bound": "hbm", "achieved": bytes_dom / (ms_dom * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s"}
    else:
        name, ms_dom = "gqla_decode_absorb", ms_absorb
        t_hbm = alg["absorb_bytes"] / (hbm * 1e9)
        t_tc = alg["absorb_flops"] / (tf_burst * 1e12)
        if t_hbm >= t_tc:
            roof = {"bound": "hbm", "achieved": alg["absorb_bytes"] / (ms_dom * 1e-3) / 1e9, "peak": hbm,
                    "unit": "GB/s"}
        else:
            roof = {"bound": "tensor", "achieved": alg["absorb_flops"] / (ms_dom * 1e-3) / 1e12, "peak": tf_burst,
                    "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(name)
    roof["kernel"] = name
    roof["peak_source"] = peak_src

    def path_entry(ms, nbytes, flops):
        t_roof = max(nbytes / (hbm * 1e9), flops / (tf_burst * 1e12))
        return {"ms": ms, "tokens_per_s": tokens / (ms * 1e-3), "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
                "tflops": flops / (ms * 1e-3) / 1e12, "roofline_frac": t_roof / (ms * 1e-3),
                "bound": "hbm" if nbytes / (hbm * 1e9) >= flops / (tf_burst * 1e12) else "tensor"}

    T = B * wl.seq_len
    exp_flops = 2 * T * d.r * d.G * (d.d_nope + d.d_v)
    exp_bytes = 2 * T * (d.r + d.d_rope) + 2 * T * d.G * (d.d_qk + d.d_v)
    h2d = q_host.numel() * q_host.element_size() + new_rows_host.numel() * new_rows_host.element_size()
    d2h = out_host.numel() * out_host.element_size()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if tp else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Gaussian, random-init weights)",
        "config": {"workload": "%s B%d L%d s_q%d" % (wl.name, B, wl.seq_len, d.s_q), "batch": B,
                   "seq_len": wl.seq_len, "s_q": d.s_q, "n_h": d.n_h, "G": d.G, "d_nope": d.d_nope,
                   "d_rope": d.d_rope, "d_v": d.d_v, "r": d.r,
                   "step": ("append the s_q new tokens (latent rows + their per-group expansion) + absorb "
                            "decode + GQA decode"),
                   "launch": ("cuda_graph replay of the step; absorb path on a second stream, overlapped with "
                              "the tail expansion + GQA path") if graph is not None else "eager, sequential",
                   "eager_ms_per_step": eager_ms,
                   "l2": "no flush: inputs larger than L2 (latent %.0f MB, expanded cache %.0f MB)" % (
                       alg["absorb_bytes"] / 1e6, alg["gqa_bytes"] / 1e6),
                   "parallelism": ("tp%d over groups (each rank: G/%d groups and their heads; no collective "
                                   "inside attention)" % (world, world)) if tp else
                                  "replicas x%d (batch-sharded, no collective)" % world},
        "roofline": roof,
        "e2e": {"value": (1 if tp else world) * tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                "launch": ("one CUDA graph replay (H2D copies, the step's calls, D2H copies) and a host wait per "
                           "step") if e2e_graph is not None else "eager calls and a host wait per step",
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clk,
        "paths": {"absorb": path_entry(ms_absorb, alg["absorb_bytes"], alg["absorb_flops"]),
                  "gqa": path_entry(ms_gqa, alg["gqa_bytes"], alg["gqa_flops"]),
                  "gqa_shared_rope": path_entry(ms_gqa_s, alg["gqa_shared_bytes"], alg["gqa_flops"]),
                  "expand_tail": {"ms": ms_tail},
                  "append_latent": {"ms": ms_append},
                  "append_and_expand": {"ms": ms_append_expand},
                  "expand_full_cache": {"ms": ms_expand_full, "tflops": exp_flops / (ms_expand_full * 1e-3) / 1e12,
                                        "hbm_gbs": exp_bytes / (ms_expand_full * 1e-3) / 1e9,
                                        "tc_frac": exp_flops / (ms_expand_full * 1e-3) / (tf_burst * 1e12)}},
        "splits": {"absorb": gqla.gqla_num_splits(dims, lay, 0, gqla.GQLA_PATH_ABSORB),
                   "in_overlapped_step": {
                       "absorb": gqla.gqla_num_splits(dims, lay, absorb_splits[0], gqla.GQLA_PATH_ABSORB),
                       "gqa": gqla.gqla_num_splits(dims, lay, gqa_splits[0], gqla.GQLA_PATH_GQA)},
                   "step_tuning_ms": ({"absorb %s, gqa %s" % (k[0] or "plan", k[1] or "plan"): v
                                       for k, v in tuned.items()} if tuned else None),
                   "gqa": gqla.gqla_num_splits(dims, lay, 0, gqla.GQLA_PATH_GQA)},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        inp_cpu = inp
        line["cpu_baseline"] = cpu_baseline(inp_cpu)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph, e2e_graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def time_paths(inp, reps, hbm, tf_burst, expand=True):
    """Device time of one absorb call and one GQA call on resident inputs.
    With expand=False the per-group pools are filled with seeded random bf16
    instead of the expansion (decode time does not depend on the values)."""
    import torch
    from latent_kv_cache_flash_b200 import gqla, synth
    d = inp.dims
    dev = inp.q.device
    dims = gqla.make_dims(d)
    lay = gqla.make_layout(inp.seq_lens, inp.max_seq_len, inp.wl.page_size,
                           inp.capacity if inp.wl.page_size == 0 else 0, inp.block_table, inp.num_pages)
    ks, vs = synth.expanded_pool_shapes(inp)
    if expand:
        kp = torch.empty(ks, dtype=d.torch_dtype, device=dev)
        vp = torch.empty(vs, dtype=d.torch_dtype, device=dev)
        gqla.gqla_expand_cache(dims, lay, inp.latent, inp.W_uk, inp.W_uv, kp, vp)
    else:
        g = torch.Generator(device=dev)
        g.manual_seed(1)
        kp = synth._randn_chunked(ks, g, dev, d.torch_dtype)
        vp = synth._randn_chunked(vs, g, dev, d.torch_dtype)
    B = inp.wl.batch
    out = torch.empty((B, d.s_q, d.n_h, d.d_v), dtype=d.torch_dtype, device=dev)
    lse = torch.empty((B, d.s_q, d.n_h), device=dev)
    ws_a = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_ABSORB, dev)
    ws_g = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_GQA, dev)
    res = {}
    lens = inp.seq_lens_host
    T = sum(lens)
    keys = sum(sum(L - d.s_q + i + 1 for i in range(d.s_q)) for L in lens)
    gqa_flops = d.n_h * keys * 2 * (d.d_qk + d.d_v)
    work = {"absorb": (2 * T * (d.r + d.d_rope), d.n_h * keys * 2 * (2 * d.r + d.d_rope)),
            "gqa": (2 * T * d.G * (d.d_qk + d.d_v), gqa_flops),
            "gqa_shared_rope": (2 * T * (d.G * (d.d_nope + d.d_v) + d.d_rope), gqa_flops)}
    dims_s = gqla.make_dims(dataclasses.replace(d, k_shared_rope=True))
    pools = {"kp": kp}

    def shared_pool():
        # the shared-RoPE K pool replaces the per-group one (one K pool resident at a time)
        pools.pop("kp", None)
        ks_s = tuple(ks[:2]) + (d.G * d.d_nope + d.d_rope,)
        if expand:
            kp_s = torch.empty(ks_s, dtype=d.torch_dtype, device=dev)
            gqla.gqla_expand_cache(dims_s, lay, inp.latent, inp.W_uk, inp.W_uv, kp_s, vp)
        else:
            kp_s = synth._randn_chunked(ks_s, g, dev, d.torch_dtype)
        pools["kp_s"] = kp_s

    calls = {"absorb": lambda: gqla.gqla_decode_absorb(dims, lay, inp.q, inp.latent, inp.W_uk, inp.W_uv, out, lse,
                                                        0, ws_a),
             "gqa": lambda: gqla.gqla_decode_gqa(dims, lay, inp.q, pools["kp"], vp, out, lse, 0, ws_g),
             "gqa_shared_rope": lambda: gqla.gqla_decode_gqa(dims_s, lay, inp.q, pools["kp_s"], vp, out, lse, 0,
                                                             ws_g)}
    del kp
    for name, fn in calls.items():
        if name == "gqa_shared_rope":
            shared_pool()
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        nbytes, flops = work[name]
        t_hbm, t_tc = nbytes / (hbm * 1e9), flops / (tf_burst * 1e12)
        res[name] = {"ms": ms, "tokens_per_s": B * d.s_q / (ms * 1e-3), "bound": "hbm" if t_hbm >= t_tc else "tensor",
                     "roofline_frac": max(t_hbm, t_tc) / (ms * 1e-3), "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
                     "tflops": flops / (ms * 1e-3) / 1e12,
                     "splits": gqla.gqla_num_splits(dims, lay, 0, 0 if name == "absorb" else 1)}
    pools.clear()
    del vp
    return res


def capacity_point(d, L, budget_bytes, path, reps, hbm, tf_burst, max_batch=4096):
    """Largest batch of L-token sequences whose cache for this path fits in
    budget_bytes, and one decode call's device time at that batch.  Only the
    path's own cache is allocated (filled with seeded random bf16: decode time
    does not depend on the values)."""
    import torch
    from latent_kv_cache_flash_b200 import gqla, synth
    dev = torch.device("cuda")
    dd = dataclasses.replace(d, k_shared_rope=(path == "gqa_shared_rope"))
    dims = gqla.make_dims(dd)
    per_token = gqla.gqla_cache_bytes_per_token(dims, gqla.GQLA_PATH_ABSORB if path == "absorb" else gqla.GQLA_PATH_GQA)
    B = min(max_batch, int(budget_bytes // (per_token * L)))
    if B < 1:
        return {"batch": 0}
    g = torch.Generator(device=dev)
    g.manual_seed(2)
    lens = torch.full((B,), L, dtype=torch.int32, device=dev)
    lay = gqla.make_layout(lens, L, 0, L)
    q = synth._randn_chunked((B, d.s_q, d.n_h, d.d_qk), g, dev, d.torch_dtype)
    out = torch.empty((B, d.s_q, d.n_h, d.d_v), dtype=d.torch_dtype, device=dev)
    lse = torch.empty((B, d.s_q, d.n_h), device=dev)
    keys = B * sum(L - d.s_q + i + 1 for i in range(d.s_q))
    if path == "absorb":
        latent = synth._randn_chunked((B, L, d.r + d.d_rope), g, dev, d.torch_dtype)
        W_uk = synth._randn_chunked((d.G, d.r, d.d_nope), g, dev, d.torch_dtype)
        W_uv = synth._randn_chunked((d.G, d.r, d.d_v), g, dev, d.torch_dtype)
        ws = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_ABSORB, dev)
        fn = lambda: gqla.gqla_decode_absorb(dims, lay, q, latent, W_uk, W_uv, out, lse, 0, ws)
        flops = d.n_h * keys * 2 * (2 * d.r + d.d_rope)
        pools = (latent,)
    else:
        kw = d.G * d.d_nope + d.d_rope if dd.k_shared_rope else d.G * d.d_qk
        kp = synth._randn_chunked((B, L, kw), g, dev, d.torch_dtype)
        vp = synth._randn_chunked((B, L, d.G * d.d_v), g, dev, d.torch_dtype)
        ws = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_GQA, dev)
        fn = lambda: gqla.gqla_decode_gqa(dims, lay, q, kp, vp, out, lse, 0, ws)
        flops = d.n_h * keys * 2 * (d.d_qk + d.d_v)
        pools = (kp, vp)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = per_token * L * B
    t_roof = max(nbytes / (hbm * 1e9), flops / (tf_burst * 1e12))
    del pools
    return {"batch": B, "cache_bytes": nbytes, "ms": ms, "tokens_per_s": B * d.s_q / (ms * 1e-3),
            "roofline_frac": t_roof / (ms * 1e-3)}


def run_capacity(args):
    """Capacity-tuned comparison: under one cache budget per GPU for this
    layer, each path decodes the largest batch that fits.  The DeepSeek-V3
    layer whole on one GPU, and one rank's share of it under 8-way group
    tensor parallelism (16 heads, 2 groups; the absorb path keeps the whole
    latent cache on every rank)."""
    import torch
    from latent_kv_cache_flash_b200 import build, synth
    build.build()
    hbm, tf_burst, _, _ = load_peaks()
    budget = 16 * 2 ** 30
    layers = [("DeepSeek-V3 layer, one GPU", synth.Dims(n_h=128, G=16, d_nope=128, d_rope=64, d_v=128, r=512)),
              ("DeepSeek-V3 layer, one rank of 8-way group TP",
               synth.Dims(n_h=16, G=2, d_nope=128, d_rope=64, d_v=128, r=512))]
    for name, d in layers:
        for L in (8192, 32768):
            line = {"sweep": "capacity", "layer": name, "n_h": d.n_h, "G": d.G, "s_q": d.s_q, "seq_len": L,
                    "budget_bytes": budget}
            for path in ("absorb", "gqa", "gqa_shared_rope"):
                line[path] = capacity_point(d, L, budget, path, max(5, args.steps // 10), hbm, tf_burst)
                torch.cuda.empty_cache()
            ok = {k: v for k, v in line.items() if isinstance(v, dict) and v.get("batch")}
            line["fastest_at_capacity"] = max(ok, key=lambda k: ok[k]["tokens_per_s"])
            print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """Both decode paths over the crossover, context or ragged workloads."""
    import torch
    from latent_kv_cache_flash_b200 import build, synth
    build.build()
    hbm, tf_burst, _, _ = load_peaks()
    if args.sweep == "capacity":
        return run_capacity(args)
    if args.sweep == "crossover":
        points = [synth.crossover(G, s_q) for G in (1, 2, 4, 8, 16, 32, 128) for s_q in (1, 2, 4)]
    elif args.sweep == "context":
        points = [synth.dsv3(seq_len=L, s_q=s_q) for L in (8192, 16384, 32768, 65536) for s_q in (1, 2)]
    else:
        points = [synth.ragged_paged()]
    from latent_kv_cache_flash_b200 import gqla
    for wl in points:
        inp = synth.make_inputs(wl, "cuda")
        res = time_paths(inp, max(5, args.steps // 10), hbm, tf_burst, expand=False)
        d = wl.dims
        lay = gqla.make_layout(inp.seq_lens, inp.max_seq_len, wl.page_size,
                               inp.capacity if wl.page_size == 0 else 0, inp.block_table, inp.num_pages)
        sel = gqla.gqla_select_path(gqla.make_dims(d), lay, sum(inp.seq_lens_host))
        line = {"sweep": args.sweep, "workload": wl.name, "G": d.G, "s_q": d.s_q, "batch": wl.batch,
                "seq_len": wl.seq_len if wl.ragged is None else "ragged %d..%d" % wl.ragged,
                "page_size": wl.page_size, "absorb": res["absorb"], "gqa": res["gqa"],
                "gqa_shared_rope": res["gqa_shared_rope"],
                "faster": "absorb" if res["absorb"]["ms"] < res["gqa"]["ms"] else "gqa",
                "fastest": min(res, key=lambda k: res[k]["ms"]),
                "selector": {"path": "gqa" if sel[0] == gqla.GQLA_PATH_GQA else "absorb",
                             "absorb_ms": sel[1] * 1e-3, "gqa_ms": sel[2] * 1e-3},
                "pools": "expanded pools filled with seeded random bf16 (decode timing only)"}
        print(json.dumps(line), flush=True)
        del inp
        torch.cuda.empty_cache()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
