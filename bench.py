"""GQLA decode-attention benchmark (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload dsv3_64k|llama3_8b] [--sq 1|2]
                    [--impl ours|reference] [--sweep crossover|context|ragged|capacity]

Default workload: the DeepSeek-V3-shaped GQLA layer (n_h 128, G 16, d_nope
128, d_rope 64, d_v 128, r 512), batch 64, uniform context 65536, s_q new
tokens per sequence, bf16, synthetic seeded inputs: the largest single-GPU
configuration of the decode study.  --workload llama3_8b selects the
LLaMA-3-8B-shaped layer (n_h 32, G 8), batch 32, context 8192.

One step is one decode step of that batch: the s_q new tokens' latent rows
are written into the latent pool, their expansion is written into the
per-group pools (which the GQA path reads and a runtime keeps current so it
can switch paths), and the decode path the library's selector picks for the
workload runs over the whole cache (append, expansion, decode: the hot path
of one step).  The other path is timed on the same inputs and reported under
"paths".  value = decoded tokens (B*s_q per step per GPU) / device time.
Under torchrun every rank decodes its own batch (weak scaling; sequences are
independent, no data-path collective); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the bench's reference arm)
on the same workload: each step decodes one (sequence, group) unit of the
batch, and its rate is scaled by the batch's number of such units.
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
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode attention tokens/s per layer and % of roofline (HBM GB/s or TC util), 1×B200"
WORKLOADS = ("dsv3_64k", "llama3_8b")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="dsv3_64k", choices=WORKLOADS)
    ap.add_argument("--sq", type=int, default=1, choices=[1, 2, 3, 4])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", choices=["select", "absorb", "gqa"], default="select",
                    help="decode path of the step: the library's selector (default) or a fixed one")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches only")
    ap.add_argument("--tp", action="store_true",
                    help="with --gpus N > 1: split the groups of one batch over the ranks (strong scaling) "
                         "instead of giving every rank its own batch")
    ap.add_argument("--once", choices=["absorb", "gqa"],
                    help="profiling case: build a DeepSeek-V3-shaped batch of --batch sequences of --seq-len "
                         "tokens with --groups groups, run --warmup calls of this path, then one more, and exit")
    ap.add_argument("--batch", type=int, default=8)
    ap.add_argument("--seq-len", type=int, default=8192)
    ap.add_argument("--groups", type=int, default=16)
    ap.add_argument("--sweep", choices=["crossover", "context", "ragged", "capacity"],
                    help="instead of the headline line, time both decode paths over a workload sweep "
                         "(one JSON line per point)")
    return ap.parse_args()


def workload(name, s_q):
    from latent_kv_cache_flash_b200 import synth
    if name == "llama3_8b":
        return synth.llama3_8b(s_q=s_q)
    return synth.dsv3(seq_len=65536, s_q=s_q)


def bench_config(wl, world=1, tp=False):
    """The workload's description, the same dict in both arms of the bench."""
    d = wl.dims
    T = wl.batch * wl.seq_len
    return {"workload": "%s B%d L%d s_q%d" % (wl.name, wl.batch, wl.seq_len, d.s_q), "batch": wl.batch,
            "seq_len": wl.seq_len, "s_q": d.s_q, "n_h": d.n_h, "G": d.G, "d_nope": d.d_nope,
            "d_rope": d.d_rope, "d_v": d.d_v, "r": d.r, "dtype": d.dtype,
            "l2": "no flush: inputs larger than L2 (latent cache %.0f MB, expanded cache %.0f MB)" % (
                2 * T * (d.r + d.d_rope) / 1e6, 2 * T * d.G * (d.d_qk + d.d_v) / 1e6),
            "parallelism": ("tp%d over groups (each rank: G/%d groups and their heads; no collective inside "
                            "attention)" % (world, world)) if tp else
                           "replicas x%d (batch-sharded, no collective)" % world}


def algorithmic(wl):
    """Per-step algorithmic bytes and flops (the method's own traffic: every
    cached byte a path reads once per step; q, out and weights ignored) of
    each decode path, of the new tokens' append and expansion, and of the
    whole-cache expansion."""
    d = wl.dims
    B = wl.batch
    T = B * wl.seq_len
    keys = sum(wl.seq_len - d.s_q + i + 1 for i in range(d.s_q)) * B   # (query, key) pairs per head
    E = d.r + d.d_rope
    new = B * d.s_q
    return dict(
        absorb_bytes=2 * T * E,
        absorb_flops=d.n_h * keys * 2 * (2 * d.r + d.d_rope) + new * d.n_h * 2 * d.r * (d.d_nope + d.d_v),
        gqa_bytes=2 * T * d.G * (d.d_qk + d.d_v),
        gqa_flops=d.n_h * keys * 2 * (d.d_qk + d.d_v),
        gqa_shared_bytes=2 * T * (d.G * (d.d_nope + d.d_v) + d.d_rope),
        # new rows written into the latent pool; then read, expanded and written per group
        append_bytes=2 * new * E,
        expand_new_bytes=2 * new * E + 2 * new * d.G * (d.d_qk + d.d_v),
        expand_new_flops=2 * new * d.r * d.G * (d.d_nope + d.d_v),
        expand_full_bytes=2 * T * E + 2 * T * d.G * (d.d_qk + d.d_v),
        expand_full_flops=2 * T * d.r * d.G * (d.d_nope + d.d_v))


def roof_time(nbytes, flops, hbm, tf):
    """Roofline time (s) and its binding resource."""
    t_hbm, t_tc = nbytes / (hbm * 1e9), flops / (tf * 1e12)
    return max(t_hbm, t_tc), ("hbm" if t_hbm >= t_tc else "tensor")


# ---------------------------------------------------------------- clocks ---
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.idx = gpu_index
        fd, self.path = tempfile.mkstemp(prefix="gqla_clocks_", suffix=".csv")
        os.close(fd)

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
        sm, power, mx, reasons = [], [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
                power.append(float(p[3]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# --------------------------------------------------------- cpu baseline ---
def oracle_unit(inp, unit):
    """The oracle's decode of one (sequence, group) unit in the expanded form
    (the definition); returns seconds."""
    from oracle import gqla_oracle as O
    d = inp.dims
    b, g = unit
    W_uk = inp.W_uk.double().cpu().numpy()
    W_uv = inp.W_uv.double().cpu().numpy()
    rows = inp.logical_latent(b).double().cpu().numpy()
    qb = inp.q[b].double().cpu().numpy()
    L = inp.seq_lens_host[b]
    t0 = time.perf_counter()
    O.decode_sequence_gqa(qb, rows[:, :d.r], rows[:, d.r:], W_uk, W_uv, L, d.softmax_scale, groups=[g])
    return time.perf_counter() - t0


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def shuffled_units(wl):
    import random
    units = [(b, g) for b in range(wl.batch) for g in range(wl.dims.G)]
    random.Random(0).shuffle(units)
    return units


def cpu_baseline(inp, budget_s=12.0):
    wl = inp.wl
    d = wl.dims
    units = shuffled_units(wl)
    done, spent = 0, 0.0
    while done < len(units) and (spent < budget_s or done < 2):
        spent += oracle_unit(inp, units[done])
        done += 1
    per_step = spent / done * len(units)
    return {"value": wl.batch * d.s_q / per_step, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": "%d of the %d (sequence, group) units of %s (B%d L%d s_q%d) decoded by the fp64 oracle "
                      "(expanded form, the definition) in %.1f s; the rate is scaled to the whole batch" % (
                          done, len(units), wl.name, wl.batch, wl.seq_len, d.s_q, spent)}


# ----------------------------------------------------------- reference ---
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    from latent_kv_cache_flash_b200 import synth
    wl = workload(args.workload, args.sq)
    inp = synth.make_inputs(wl, "cpu")
    d = wl.dims
    units = shuffled_units(wl)
    for w in range(args.warmup):
        oracle_unit(inp, units[w % len(units)])
    times = []
    for s in range(args.steps):
        times.append(oracle_unit(inp, units[(args.warmup + s) % len(units)]))
    step_s = sum(times) / len(times)
    # one unit of the B*G per step: the batch's tokens scaled by that share
    value = wl.batch * d.s_q / len(units) / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Gaussian, "
            "random-init weights)", "config": bench_config(wl, world, args.tp),
            "step": ("one (sequence, group) unit of the batch decoded by the fp64 oracle (expanded form); "
                     "ms_per_step is that measured time, value scales its rate by the %d units of the batch"
                     % len(units)),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": "one of the %d (sequence, group) units per step, %d steps, fp64 expanded "
                                       "form, on rank 0's host cores" % (len(units), args.steps)},
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


def recorded_traffic(name, workload_name):
    """DRAM bytes per launch from the committed ncu record of this call on
    this workload, or None when the kernels' sources changed since the
    counters were taken (or none were taken)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        rec = json.load(open(p)).get("%s @ %s" % (name, workload_name))
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

    wl = workload(args.workload, args.sq)
    tp = args.tp and world > 1
    config = bench_config(wl, world, tp)
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
    out = torch.empty((B, d.s_q, d.n_h, d.d_v), dtype=d.torch_dtype, device=dev)
    lse = torch.empty((B, d.s_q, d.n_h), device=dev)
    ws_a = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_ABSORB, dev)
    ws_g = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_GQA, dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # the resident per-group cache of all tokens (a prefill-time cost, timed on its own)
    gqla.gqla_expand_cache(dims, lay, inp.latent, inp.W_uk, inp.W_uv, kp, vp, 0, status)
    # the step's new tokens [c_KV ; k_rope], resident on the device; each step
    # writes them into the latent pool (they are the rows already there, so
    # every step sees the same cache)
    Lmax = wl.seq_len
    new_rows = inp.latent[:, Lmax - d.s_q:Lmax].contiguous()

    sel_path, sel_absorb_us, sel_gqa_us = gqla.gqla_select_path(dims, lay, sum(inp.seq_lens_host))
    if args.path == "absorb":
        path = gqla.GQLA_PATH_ABSORB
    elif args.path == "gqa":
        path = gqla.GQLA_PATH_GQA
    else:
        path = sel_path
    path_name = "absorb" if path == gqla.GQLA_PATH_ABSORB else "gqa"

    def append_latent():
        gqla.gqla_append_tokens(dims, lay, new_rows, inp.latent, dev_status=status)

    def expand_new():
        # the new rows' expansion alone (no latent pool argument): dense rows,
        # many sequences' new tokens to one 128-row tensor-core tile
        gqla.gqla_append_tokens(dims, lay, new_rows, None, inp.W_uk, inp.W_uv, kp, vp, dev_status=status)

    def absorb():
        gqla.gqla_decode_absorb(dims, lay, inp.q, inp.latent, inp.W_uk, inp.W_uv, out, lse, 0, ws_a, status)

    def gqa():
        gqla.gqla_decode_gqa(dims, lay, inp.q, kp, vp, out, lse, 0, ws_g, status)

    decode = absorb if path == gqla.GQLA_PATH_ABSORB else gqa

    def step():
        append_latent()
        expand_new()
        decode()

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

    # eager timed region: every C-ABI call made on every step; CUDA events
    # around the decode call of each step (the dominant call) on its stream
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]

    def eager_steps():
        for i in range(args.steps):
            append_latent()
            expand_new()
            ev[i][0].record(stream)
            decode()
            ev[i][1].record(stream)

    n0 = gqla.gqla_launch_counter()
    eager_ms = timed(eager_steps, 1) / args.steps
    launches = gqla.gqla_launch_counter() - n0
    ms_decode_live = multi.max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, dev)

    # the same step captured once as a CUDA graph and replayed (no host
    # launch gaps between the kernels); every kernel still runs each step
    graph = None
    if not args.no_graph:
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        ms_step = timed(graph.replay, args.steps) / args.steps
    else:
        ms_step = eager_ms

    # end to end through the public API with host buffers: the step's inputs
    # (queries and the new tokens' latent rows) go host->device from pinned
    # memory, and the step's result (out and lse) comes back device->host,
    # inside the timed region; every C-ABI call is made on every step, then
    # the host waits for the step
    # (measured right after the step, before the per-call breakdown and the
    # whole-cache expansion heat the GPU into its power cap)
    q_host = inp.q.cpu().pin_memory()
    new_rows_host = new_rows.cpu().pin_memory()
    out_host = torch.empty(tuple(out.shape), dtype=out.dtype).pin_memory()
    lse_host = torch.empty(tuple(lse.shape), dtype=lse.dtype).pin_memory()

    def e2e_body():
        inp.q.copy_(q_host, non_blocking=True)
        new_rows.copy_(new_rows_host, non_blocking=True)
        step()
        out_host.copy_(out, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    def e2e_step():
        e2e_body()
        stream.synchronize()

    for _ in range(3):
        e2e_step()
    e2e_serial_ms = timed(e2e_step, args.steps) / args.steps

    # the same calls pipelined as a serving loop runs them: two sets of device
    # staging buffers, step i+1's inputs copied in (own stream) while step i
    # computes, step i's result copied out (own stream) while step i+1
    # computes; every step's copies stay inside the timed region and the host
    # holds each step's result before the loop ends
    q2 = [inp.q, torch.empty_like(inp.q)]
    rows2 = [new_rows, torch.empty_like(new_rows)]
    out2 = [out, torch.empty_like(out)]
    lse2 = [lse, torch.empty_like(lse)]
    out_host2 = [out_host, torch.empty(tuple(out.shape), dtype=out.dtype).pin_memory()]
    lse_host2 = [lse_host, torch.empty(tuple(lse.shape), dtype=lse.dtype).pin_memory()]
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event(), torch.cuda.Event()]
    ev_done = [torch.cuda.Event(), torch.cuda.Event()]
    ev_out = [torch.cuda.Event(), torch.cuda.Event()]

    def step_on(k):
        gqla.gqla_append_tokens(dims, lay, rows2[k], inp.latent, dev_status=status)
        gqla.gqla_append_tokens(dims, lay, rows2[k], None, inp.W_uk, inp.W_uv, kp, vp, dev_status=status)
        if path == gqla.GQLA_PATH_ABSORB:
            gqla.gqla_decode_absorb(dims, lay, q2[k], inp.latent, inp.W_uk, inp.W_uv, out2[k], lse2[k], 0, ws_a,
                                    status)
        else:
            gqla.gqla_decode_gqa(dims, lay, q2[k], kp, vp, out2[k], lse2[k], 0, ws_g, status)

    def e2e_pipelined(n):
        for i in range(n):
            k = i & 1
            with torch.cuda.stream(h2d_stream):
                h2d_stream.wait_event(ev_done[k])          # step i-2 has finished with these buffers
                q2[k].copy_(q_host, non_blocking=True)
                rows2[k].copy_(new_rows_host, non_blocking=True)
                ev_in[k].record(h2d_stream)
            stream.wait_event(ev_in[k])
            stream.wait_event(ev_out[k])                   # step i-2's result is out before it is overwritten
            step_on(k)
            ev_done[k].record(stream)
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(ev_done[k])
                out_host2[k].copy_(out2[k], non_blocking=True)
                lse_host2[k].copy_(lse2[k], non_blocking=True)
                ev_out[k].record(d2h_stream)
            if i >= 1:
                ev_out[k ^ 1].synchronize()                # the host holds step i-1's result
        ev_out[(n - 1) & 1].synchronize()

    e2e_pipelined(3)
    torch.cuda.synchronize()
    e2e_ms = timed(lambda: e2e_pipelined(args.steps), 1) / args.steps
    # both buffer sets hold what the plain step computes from the same inputs
    step()
    torch.cuda.synchronize()
    for k in (0, 1):
        if not (torch.equal(out_host2[k], out.cpu()) and torch.equal(lse_host2[k], lse.cpu())):
            raise SystemExit("pipelined end-to-end step %d differs from the step's own result" % k)
    # the same, recorded once as a CUDA graph (copies included) and replayed
    e2e_graph_ms = None
    if not args.no_graph:
        torch.cuda.synchronize()
        e2e_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(e2e_graph):
            e2e_body()

        def e2e_graph_step():
            e2e_graph.replay()
            stream.synchronize()

        for _ in range(3):
            e2e_graph_step()
        e2e_graph_ms = timed(e2e_graph_step, args.steps) / args.steps
        del e2e_graph

    # per-call breakdown (each over at least ~0.3 s of device time)
    reps = args.steps if args.no_clocks else max(args.steps, int(300.0 / max(ms_step, 1e-3)))
    ms_absorb = timed(absorb, reps) / reps
    ms_gqa = timed(gqa, reps) / reps
    ms_append = timed(append_latent, reps) / reps
    ms_expand_new = timed(expand_new, reps) / reps
    n_full = 5 if wl.seq_len * B > 1 << 20 else 10
    ms_expand_full = timed(lambda: gqla.gqla_expand_cache(dims, lay, inp.latent, inp.W_uk, inp.W_uv, kp, vp, 0,
                                                          status), n_full) / n_full
    # the GQA call over the same cache with the RoPE key stored once per token
    # row (a smaller K pool; V is shared); the per-group K pool is released first
    dims_s = gqla.make_dims(dataclasses.replace(d, k_shared_rope=True))
    del graph
    graph = None
    kp_shape = tuple(ks[:2]) + (d.G * d.d_nope + d.d_rope,)
    del kp
    torch.cuda.empty_cache()
    kp_s = torch.empty(kp_shape, dtype=d.torch_dtype, device=dev)
    gqla.gqla_expand_cache(dims_s, lay, inp.latent, inp.W_uk, inp.W_uv, kp_s, vp, 0, status)
    ms_gqa_s = timed(lambda: gqla.gqla_decode_gqa(dims_s, lay, inp.q, kp_s, vp, out, lse, 0, ws_g, status),
                     reps) / reps
    del kp_s
    torch.cuda.empty_cache()

    clk = clocks.stop() if clocks else None
    torch.cuda.synchronize()
    st = int(status.item())
    if st != 0:
        raise SystemExit("device status 0x%x during the bench" % st)

    alg = algorithmic(wl)
    tokens = B * d.s_q
    # replicas decode world batches per step; tensor-parallel ranks share one
    job = 1 if tp else world
    value = multi.job_tokens_per_s(tokens, 1, job, ms_step)
    dec_bytes = alg["absorb_bytes"] if path == gqla.GQLA_PATH_ABSORB else alg["gqa_bytes"]
    dec_flops = alg["absorb_flops"] if path == gqla.GQLA_PATH_ABSORB else alg["gqa_flops"]
    # dominant call: the step's decode call, timed live in the eager timed region
    t_roof, bound = roof_time(dec_bytes, dec_flops, hbm, tf_burst)
    call = "gqla_decode_%s" % path_name
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": dec_bytes / (ms_decode_live * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": dec_flops / (ms_decode_live * 1e-3) / 1e12, "peak": tf_burst,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(call, config["workload"])
    roof["kernel"] = call + (" (one call: absorbed-query GEMM, latent decode, split merge, up-projection)"
                             if path == gqla.GQLA_PATH_ABSORB else " (one call: decode and split merge)")
    roof["ms_per_launch"] = ms_decode_live
    roof["algorithmic_bytes"] = dec_bytes
    roof["algorithmic_flops"] = dec_flops
    roof["roofline_ms"] = t_roof * 1e3
    roof["peak_source"] = peak_src + " (MEASURED_PEAKS.json: copy GB/s, cuBLAS bf16 burst TFLOP/s)"
    # the step's own roofline: everything the step reads, writes and computes
    step_bytes = alg["append_bytes"] + alg["expand_new_bytes"] + dec_bytes
    step_flops = alg["expand_new_flops"] + dec_flops
    t_step_roof, step_bound = roof_time(step_bytes, step_flops, hbm, tf_burst)

    def path_entry(ms, nbytes, flops):
        t, bnd = roof_time(nbytes, flops, hbm, tf_burst)
        e = {"ms": ms, "tokens_per_s": tokens / (ms * 1e-3), "hbm_gbs": nbytes / (ms * 1e-3) / 1e9,
             "tflops": flops / (ms * 1e-3) / 1e12, "roofline_frac": t / (ms * 1e-3), "bound": bnd}
        if t / (ms * 1e-3) > 1.0:
            e["note"] = ("above 1: the HBM peak is a copy's rate (reads and writes with their turnarounds); "
                         "this call is a pure read stream")
        return e

    h2d = q_host.numel() * q_host.element_size() + new_rows_host.numel() * new_rows_host.element_size()
    d2h = out_host.numel() * out_host.element_size() + lse_host.numel() * lse_host.element_size()
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if tp else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Gaussian, random-init weights)",
        "config": config,
        "step": {"path": path_name,
                 "selector": {"path": "absorb" if sel_path == gqla.GQLA_PATH_ABSORB else "gqa",
                              "predicted_absorb_ms": sel_absorb_us * 1e-3, "predicted_gqa_ms": sel_gqa_us * 1e-3},
                 "calls": ["gqla_append_tokens (new latent rows)", "gqla_append_tokens (their expansion)", call],
                 "launch": "cuda_graph replay of the step" if not args.no_graph else "eager",
                 "eager_ms_per_step": eager_ms,
                 "roofline": {"bound": step_bound, "bytes": step_bytes, "flops": step_flops,
                              "roofline_ms": t_step_roof * 1e3, "frac": t_step_roof / (ms_step * 1e-3)}},
        "roofline": roof,
        "e2e": {"value": job * tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                "launch": "every C-ABI call of the step made eagerly each step; the step's inputs copied in "
                          "and its result copied out on their own streams, overlapping the neighbouring "
                          "steps (double-buffered); the host holds every step's result",
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "e2e_serial": {"value": job * tokens / (e2e_serial_ms * 1e-3), "unit": "tokens/s",
                       "launch": "the same calls and copies on one stream, the host waiting for each step "
                                 "before the next", "ms_per_step": e2e_serial_ms,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "e2e_graph": ({"value": job * tokens / (e2e_graph_ms * 1e-3), "unit": "tokens/s",
                       "launch": "one CUDA graph replay (H2D copies, the step's calls, D2H copies) and a host "
                                 "wait per step", "ms_per_step": e2e_graph_ms,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h} if e2e_graph_ms else None),
        "gpu_launches": launches,
        "gpu_launches_per_step": launches / args.steps,
        "clocks": clk,
        "paths": {"absorb": path_entry(ms_absorb, alg["absorb_bytes"], alg["absorb_flops"]),
                  "gqa": path_entry(ms_gqa, alg["gqa_bytes"], alg["gqa_flops"]),
                  "gqa_shared_rope": path_entry(ms_gqa_s, alg["gqa_shared_bytes"], alg["gqa_flops"]),
                  "append_latent": {"ms": ms_append},
                  "expand_new_tokens": path_entry(ms_expand_new, alg["expand_new_bytes"], alg["expand_new_flops"]),
                  "expand_full_cache": path_entry(ms_expand_full, alg["expand_full_bytes"],
                                                  alg["expand_full_flops"])},
        "splits": {"absorb": gqla.gqla_num_splits(dims, lay, 0, gqla.GQLA_PATH_ABSORB),
                   "gqa": gqla.gqla_num_splits(dims, lay, 0, gqla.GQLA_PATH_GQA)},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp)
    if rank == 0:
        print(json.dumps(line), flush=True)
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


def run_once(args):
    """A few calls of one decode path on a small case (for ncu captures)."""
    import torch
    from latent_kv_cache_flash_b200 import build, gqla, synth
    build.build()
    wl = synth.dsv3(seq_len=args.seq_len, s_q=args.sq, batch=args.batch, G=args.groups)
    inp = synth.make_inputs(wl, "cuda")
    d = wl.dims
    dims = gqla.make_dims(d)
    lay = gqla.make_layout(inp.seq_lens, inp.max_seq_len, 0, inp.capacity)
    out = torch.empty((wl.batch, d.s_q, d.n_h, d.d_v), dtype=d.torch_dtype, device="cuda")
    lse = torch.empty((wl.batch, d.s_q, d.n_h), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if args.once == "absorb":
        ws = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_ABSORB, "cuda")
        fn = lambda: gqla.gqla_decode_absorb(dims, lay, inp.q, inp.latent, inp.W_uk, inp.W_uv, out, lse, 0, ws,
                                             status)
    else:
        ks, vs = synth.expanded_pool_shapes(inp)
        kp = torch.empty(ks, dtype=d.torch_dtype, device="cuda")
        vp = torch.empty(vs, dtype=d.torch_dtype, device="cuda")
        gqla.gqla_expand_cache(dims, lay, inp.latent, inp.W_uk, inp.W_uv, kp, vp, 0, status)
        ws = gqla.workspace_for(dims, lay, 0, gqla.GQLA_PATH_GQA, "cuda")
        fn = lambda: gqla.gqla_decode_gqa(dims, lay, inp.q, kp, vp, out, lse, 0, ws, status)
    for _ in range(args.warmup + 1):
        fn()
    torch.cuda.synchronize()
    st = int(status.item())
    path = gqla.GQLA_PATH_ABSORB if args.once == "absorb" else gqla.GQLA_PATH_GQA
    print(json.dumps({"once": args.once, "workload": "%s B%d L%d G%d s_q%d" % (wl.name, wl.batch, wl.seq_len, d.G,
                                                                                  d.s_q),
                      "splits": gqla.gqla_num_splits(dims, lay, 0, path), "calls": args.warmup + 1,
                      "status": st}))
    return 0 if st == 0 else 1


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.once:
        return run_once(args)
    if args.sweep:
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
