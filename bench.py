"""Benchmark of one decode step of attention against a paged KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload batch10] [--layers L] [--splits S]

A step is one pass of the whole hot path over one batch: for every layer, RoPE on
the new token's q and k, the KV append through the slot mapping, and paged decode
attention (one streaming kernel that also merges cut segments).  The default workload is the batch-10,
32-layer, 32-head, head_dim-128, fp16 decode step with context lengths uniform in
[128, 2048] and 16-token pages interleaved across the requests.

Prints one JSON line.  `value` is KV-read throughput (algorithmic K+V bytes the
attention must read, per second) of whole steps timed with CUDA events, inputs
resident in HBM; `e2e` is the same metric with each step's inputs copied from
pinned host memory and its outputs read back inside the timed region; `roofline`
is the attention call alone, timed per launch, against the measured HBM copy
bandwidth.  With --impl reference the fp64 CPU oracle is timed instead, on a
bounded sample of the same workload.
"""
import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
METRIC = "paged decode-attention KV-read GB/s (% of HBM peak); us per layer-step"
UNIT = "GB/s"
INPUT_SETS = 4           # distinct per-step q/k/v sets (one captured step each) cycled through


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=synth.WORKLOADS, default="batch10")
    ap.add_argument("--layers", type=int, default=None, help="override the workload's layer count")
    ap.add_argument("--splits", type=int, default=0, help="attention work partitions (0 = auto)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the CPU-baseline sample")
    ap.add_argument("--op", choices=("decode", "rms_norm", "prefill"), default="decode",
                    help="decode: the decode step (default); rms_norm / prefill: that kernel alone")
    ap.add_argument("--chunk", type=int, default=512, help="prefill: new tokens per sequence")
    ap.add_argument("--no-fused", action="store_true",
                    help="decode: RoPE + append and attention as two launches per layer even where the fused "
                         "layer kernel is used (one query head per kv head)")
    ap.add_argument("--kv", choices=("native", "int8"), default="native",
                    help="decode: page storage -- the workload's 16-bit type, or int8 codes with a fp32 "
                         "scale per (token, head) row")
    return ap.parse_args(argv)


# ------------------------------------------------------------------ helpers
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_digest():
    h = hashlib.sha256()
    for name in ("decode_attention.cuh", "decode_attention_mma.cuh", "decode_attention_i8.cuh", "pkv_device.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_460_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def kv_bytes_per_layer(s, kv):
    """Algorithmic KV bytes one attention call reads: every cached token's K and V row of
    every kv head -- head_dim elements, or head_dim int8 codes plus a 4-byte scale."""
    if kv == "int8":
        return int(s.context_lens.astype(np.int64).sum()) * s.kv_heads * 2 * (s.head_dim + 4)
    return s.kv_bytes_read()


def profiled_traffic(workload, kv="native"):
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken
    on the kernel source as it is now (else None)."""
    name = workload if kv == "native" else "int8_" + workload
    path = os.path.join(ROOT, "profiles", "decode_attention_%s.md" % name)
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith("- "):
                k, v = line.strip()[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_digest") != kernel_source_digest():
        return None
    try:
        return int(float(vals["dram_bytes_per_attention_call"]))
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed regions run."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.device_index = device_index
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit("--gpus %d but WORLD_SIZE %d" % (args.gpus, world))
    return world, rank, local


def throughput(world, bytes_per_step, steps, ms):
    """Whole-job GB/s: the bytes of all `world` replicas over the slowest rank's time."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def max_over_ranks(value, world, device=None):
    """Max of a per-rank float across the process group (the identity with one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle timing
def host_cpu():
    """(usable host cores, CPU model name)."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return cores, model


def time_oracle_sample(s, seconds, seed=0, kv="native", all_cores=True):
    """Time the fp64 oracle on batches of random (sequence, kv head) pairs of the workload
    (each pair a standalone sequence with the group's query heads; inputs drawn outside the
    timed calls) until about `seconds` of single-thread time.  Each batch runs twice: the
    plain build on one thread, then the OpenMP build with its pairs spread over every host
    core.  Returns a dict with both legs' GB/s of algorithmic KV bytes."""
    import oracle
    r = np.random.Generator(np.random.PCG64(seed))
    G = s.q_heads // s.kv_heads
    live = np.nonzero(s.context_lens > 0)[0]
    scale = 1.0 / math.sqrt(s.head_dim)
    cores, model = host_cpu()
    threads = oracle.set_threads(cores) if all_cores else 1
    row_bytes = 2 * (s.head_dim + 4) if kv == "int8" else 2 * s.head_dim * s.elt_bytes
    mean_len = float(s.context_lens[live].mean())
    # pairs per batch: about a second of single-thread work (the oracle reads ~0.1 GB/s),
    # less for a short budget; at least two per thread, at most 1 GB of pages
    target = min(0.15e9, max(2e6, 0.1e9 * seconds))
    want = max(2 * threads, int(target / (mean_len * row_bytes)))
    n_pairs = max(1, min(want, int(1e9 / (float(s.context_lens.max()) * row_bytes))))
    t1 = tn = 0.0
    nbytes = 0
    batches = 0
    while t1 < seconds:
        pairs = [(int(r.choice(live)), int(r.integers(0, s.kv_heads))) for _ in range(n_pairs)]
        m = synth.pair_batch_numpy(s, pairs, int(r.integers(1 << 30)), kv)
        hp = [(i, h) for i in range(n_pairs) for h in range(G)]
        if kv == "int8":
            args = (m["q"], m["k_codes"], m["v_codes"], m["k_scales"], m["v_scales"], m["block_tables"],
                    m["context_lens"], scale, s.dtype, hp)
            fn = oracle.decode_attention_i8_pairs
        else:
            args = (m["q"], m["k"], m["v"], m["block_tables"], m["context_lens"], scale, s.dtype, hp)
            fn = oracle.decode_attention_pairs
        t0 = time.perf_counter()
        fn(*args)
        t1 += time.perf_counter() - t0
        if all_cores:
            t0 = time.perf_counter()
            fn(*args, omp=True)
            tn += time.perf_counter() - t0
        nbytes += int(m["context_lens"].astype(np.int64).sum()) * row_bytes
        batches += 1
    desc = "%d batches of %d random (sequence, kv head) pairs of one %s layer (%d query heads each%s); " \
           "one thread: %.1f s" % (batches, n_pairs, s.name, G, ", int8 pages" if kv == "int8" else "", t1)
    res = {"single": nbytes / t1 / 1e9, "cores_available": cores, "cpu_model": model, "sample": desc}
    if all_cores:
        res["all"] = nbytes / tn / 1e9
        res["threads"] = threads
        res["sample"] += "; %d threads: %.1f s" % (threads, tn)
    return res


def cpu_baseline_entry(res, unit):
    """The bench line's cpu_baseline: the all-core leg, the single-thread leg beside it."""
    return {"value": res.get("all", res["single"]), "unit": unit, "cores": res.get("threads", 1), "kind": "oracle",
            "sample": res["sample"], "cpu_model": res["cpu_model"], "cores_available": res["cores_available"],
            "single_thread": {"value": res["single"], "unit": unit, "cores": 1}}


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    s = synth.spec(args.workload, num_layers=args.layers)
    per_step = max(0.05, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup):
        time_oracle_sample(s, per_step, seed=i, kv=args.kv, all_cores=False)
    vals, t_all, last = [], 0.0, None
    for i in range(args.steps):
        t0 = time.perf_counter()
        last = time_oracle_sample(s, per_step, seed=1000 + i, kv=args.kv)
        t_all += time.perf_counter() - t0
        vals.append(last["all"])
    value = float(np.mean(vals))
    cpu = cpu_baseline_entry(last, UNIT)
    cpu["value"] = value
    cpu["sample"] = "each step: " + cpu["sample"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * t_all / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(s, args),
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(s, args):
    kv = getattr(args, "kv", "native")
    per_layer = kv_bytes_per_layer(s, kv)
    pages = s.dtype if kv == "native" else "int8 pages (fp32 row scales), %s activations" % s.dtype
    return {"workload": "%s: batch %d, %d layers, %d q / %d kv heads, head_dim %d, page %d, %s, context %d..%d"
                        % (s.name, s.batch, s.num_layers, s.q_heads, s.kv_heads, s.head_dim, s.page_size, pages,
                           int(s.context_lens.min()), int(s.context_lens.max())),
            "batch": s.batch, "layers": s.num_layers, "q_heads": s.q_heads, "kv_heads": s.kv_heads,
            "head_dim": s.head_dim, "page_size": s.page_size, "kv_storage": "int8" if kv == "int8" else s.dtype,
            "kv_bytes_per_layer": per_layer, "kv_bytes_per_step": per_layer * s.num_layers,
            "parallelism": "replicas" if args.gpus > 1 else "single",
            "l2": "inputs larger than L2: each step streams %d layer caches (%.2f GB of K+V)"
                  % (s.num_layers, per_layer * s.num_layers / 1e9)
                  if per_layer * s.num_layers > 2 * 126e6
                  else "L2 flushed (256 MB memset) before every timed step, outside the timed intervals"}


# ------------------------------------------------------------------ GPU run
def run_ours(args):
    import torch
    import paged_kv_cache_460_b200 as pkv
    from paged_kv_cache_460_b200.step import DecodeStep

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))

    s = synth.spec(args.workload, num_layers=args.layers)
    L = s.num_layers
    if args.kv == "int8":
        kc, vc, ksc, vsc = synth.pool_values_i8_torch(s, dev)
        pool = pkv.KVPool(kc, vc, ksc, vsc, dtype=torch.float16 if s.dtype == "f16" else torch.bfloat16)
    else:
        kp, vp = synth.pool_values_torch(s, dev)
        pool = pkv.KVPool(kp, vp)
    layer_bytes = kv_bytes_per_layer(s, args.kv)
    qs, ks, vs = synth.step_values_torch(s, INPUT_SETS, dev)
    # the fused layer where it measured faster: one query head per kv head (16-bit or int8
    # pages); with grouped heads every segment turns G q rows in-kernel and it loses
    fused = not args.no_fused and s.q_heads == s.kv_heads
    steps = []
    for j in range(INPUT_SETS):
        st = DecodeStep(pool, s.batch, s.q_heads, s.max_pages, theta=s.theta, num_splits=args.splits, device=dev,
                        fused=fused)
        st.set_metadata(s.block_tables, s.context_lens, non_blocking=False)
        st.q.copy_(qs[j])
        st.k.copy_(ks[j])
        st.v.copy_(vs[j])
        steps.append(st)
    del qs, ks, vs
    small = layer_bytes * L < 2 * 126e6
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev) if small else None

    def sync_all():
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    # warm-up: eager steps (sets kernel attributes), then graph capture and replays
    for i in range(args.warmup):
        steps[i % INPUT_SETS].eager()
    for st in steps:
        st.capture()
    attn = torch.cuda.CUDAGraph()                 # the 32 attention (fused: layer) calls of one step alone
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs), torch.cuda.graph(attn, stream=cs):
        st0 = steps[0]
        for layer in range(L):
            if fused:                               # the angle table of st0 is current
                pkv.paged_decode_layer(pool, layer, st0.out[layer], st0.q[layer], st0.k[layer], st0.v[layer],
                                       st0.rope, st0.block_tables, st0.context_lens, st0.scale,
                                       num_splits=st0.num_splits, workspace=st0.workspace)
            else:
                pkv.paged_decode_attention(pool, layer, st0.out[layer], st0.q[layer], st0.block_tables,
                                           st0.context_lens, st0.scale, num_splits=st0.num_splits,
                                           workspace=st0.workspace)
    torch.cuda.current_stream().wait_stream(cs)
    for i in range(args.warmup):
        steps[i % INPUT_SETS].replay()
        attn.replay()
    sync_all()

    stream = torch.cuda.current_stream()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    def timed(run):
        """Device time of `args.steps` calls of run(i).  A workload that fits in L2 gets
        the cache flushed before every call, outside the timed intervals."""
        sync_all()
        if flush is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(args.steps):
                run(i)
            e1.record(stream)
            sync_all()
            return e0.elapsed_time(e1)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            run(i)
            evs[i][1].record(stream)
        sync_all()
        return sum(a.elapsed_time(b) for a, b in evs)

    # ---- phase A: whole steps (headline value), one graph launch per step
    ms_total = max_over_ranks(timed(lambda i: steps[i % INPUT_SETS].replay()), world, dev)
    # ---- phase B: the attention calls alone (roofline of the dominant kernel)
    attn_ms_mean = max_over_ranks(timed(lambda i: attn.replay()), world, dev) / (args.steps * L)
    clk = clocks.stop()

    # ---- e2e through the public API: pinned host buffers in and out, one DecodeStep.run per
    #      step (its graph carries the copies, overlapped with the kernels)
    e2e = None
    if not args.no_e2e:
        st = steps[0]
        tdt = st.q.dtype
        hq = torch.empty(st.q.shape, dtype=tdt).pin_memory()
        hk = torch.empty(st.k.shape, dtype=tdt).pin_memory()
        hv = torch.empty(st.v.shape, dtype=tdt).pin_memory()
        hq.copy_(st.q)
        hk.copy_(st.k)
        hv.copy_(st.v)
        hout = torch.empty(st.out.shape, dtype=tdt).pin_memory()
        hbt = torch.from_numpy(s.block_tables).pin_memory()
        hcl = torch.from_numpy(s.context_lens).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hbt, hcl))
        d2h = hout.numel() * hout.element_size()
        for _ in range(max(1, args.warmup)):
            st.set_metadata(hbt, hcl)
            st.run(hq, hk, hv, hout)
        sync_all()
        n_e2e = max(1, args.steps // 2)

        def e2e_step(i):
            st.set_metadata(hbt, hcl)
            st.run(hq, hk, hv, hout)

        saved, args.steps = args.steps, n_e2e
        ms_e2e = max_over_ranks(timed(e2e_step), world, dev)
        args.steps = saved
        e2e = {"value": throughput(world, layer_bytes * L, n_e2e, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e / n_e2e}

    err = pkv.kv_get_device_error()
    if err:
        raise SystemExit("device error word 0x%x after the benchmark" % err)

    if rank == 0:
        per_step_ms = ms_total / args.steps
        value = throughput(world, layer_bytes * L, args.steps, ms_total)
        peak, peak_kind = measured_peaks()
        achieved = layer_bytes / (attn_ms_mean * 1e-3) / 1e9
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline_entry(time_oracle_sample(s, args.cpu_seconds, kv=args.kv), UNIT)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": per_step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": s.dtype, "data": "synthetic", "config": workload_config(s, args),
            "us_per_layer_step": 1000.0 * per_step_ms / L,
            "attention_us_per_layer": 1000.0 * attn_ms_mean,
            "pct_of_8tbs": 100.0 * value / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(args.workload, args.kv),
                         "peak_source": "%s copy bandwidth" % peak_kind,
                         "kernel": ("paged_decode_layer (RoPE + append + attention, one kernel per layer)"
                                    if fused else "paged_decode_attention (one kernel per call)"),
                         "frac_of_8tbs": achieved / NOMINAL_HBM_GBS},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * steps[0].kernels_per_step * world,
            "num_splits": args.splits or pkv.pkv_decode_auto_splits(pool, s.batch, s.max_pages, s.q_heads),
            "cluster": 0 if args.splits else pkv.pkv_decode_cluster_size(pool, s.batch, s.max_pages, s.q_heads),
            "launch": "one CUDA graph per step (%d kernels%s)" % (
                steps[0].kernels_per_step, ": an angle table, then one fused kernel per layer" if fused else ""),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    for st in steps:
        st.graph = None
    attn = None
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


def run_rms_norm(args):
    """RMSNorm (fused residual add) on the decode hidden state of the workload's batch:
    rows = batch, hidden = q_heads * head_dim; 32 calls per step (one per layer) in a graph."""
    import torch
    import paged_kv_cache_460_b200 as pkv
    s = synth.spec(args.workload, num_layers=args.layers)
    dev = torch.device("cuda", 0)
    tdt = torch.float16 if s.dtype == "f16" else torch.bfloat16
    rows, hidden, L = s.batch, s.q_heads * s.head_dim, s.num_layers
    g = torch.Generator(device=dev)
    g.manual_seed(4242)
    x = torch.randn((L, rows, hidden), generator=g, device=dev).to(tdt)
    res = torch.randn((L, rows, hidden), generator=g, device=dev).to(tdt)
    w = torch.randn((L, hidden), generator=g, device=dev).to(tdt)
    out = torch.empty_like(x)
    for layer in range(L):
        pkv.rms_norm(out[layer], x[layer], w[layer], 1e-6, residual=res[layer])
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs), torch.cuda.graph(graph, stream=cs):
        for layer in range(L):
            pkv.rms_norm(out[layer], x[layer], w[layer], 1e-6, residual=res[layer])
    torch.cuda.current_stream().wait_stream(cs)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    per_call_us = 1000.0 * ms / (args.steps * L)
    bytes_per_call = (4 * rows * hidden + hidden) * 2          # x, residual in; residual, out back; weight
    print(json.dumps({"metric": "rms_norm (fused residual) us per call", "value": per_call_us, "unit": "us",
                      "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
                      "config": {"workload": "rows %d x hidden %d, %s" % (rows, hidden, s.dtype)},
                      "bytes_per_call": bytes_per_call, "GB_per_s": bytes_per_call / (per_call_us * 1e-6) / 1e9,
                      "gpu_launches": args.steps * L}), flush=True)
    return 0


def run_prefill(args):
    """Chunked prefill attention on the workload's sequences: the last `--chunk` tokens of
    each context are the chunk (causal over the whole cached prefix); 32 calls per step, one
    per layer, in a graph.  Reports us per call and tensor TFLOP/s (4 flops per q.k / p.V
    multiply-add pair element) against the measured bf16 GEMM peak."""
    import torch
    import paged_kv_cache_460_b200 as pkv
    s = synth.spec(args.workload, num_layers=args.layers)
    dev = torch.device("cuda", 0)
    tdt = torch.float16 if s.dtype == "f16" else torch.bfloat16
    L = s.num_layers
    kp, vp = synth.pool_values_torch(s, dev)
    pool = pkv.KVPool(kp, vp)
    ctx = s.context_lens.astype(np.int64)
    chunk = np.minimum(ctx, args.chunk)
    cu_q = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int32)
    total = int(cu_q[-1])
    g = torch.Generator(device=dev)
    g.manual_seed(5150)
    q = torch.randn((L, total, s.q_heads, s.head_dim), generator=g, device=dev).to(tdt)
    out = torch.empty_like(q)
    cu_t = torch.from_numpy(cu_q).to(dev)
    bt = torch.from_numpy(s.block_tables).to(dev)
    cl = torch.from_numpy(s.context_lens).to(dev)
    scale = 1.0 / math.sqrt(s.head_dim)

    def step():
        for layer in range(L):
            pkv.paged_prefill_attention(pool, layer, out[layer], q[layer], cu_t, bt, cl, scale)

    step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs), torch.cuda.graph(graph, stream=cs):
        step()
    torch.cuda.current_stream().wait_stream(cs)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    per_call_us = 1000.0 * e0.elapsed_time(e1) / (args.steps * L)
    # visible keys of row i of sequence b: L_b - n_b + i + 1
    keys = sum(int(n) * int(c - n) + int(n) * (int(n) + 1) // 2 for c, n in zip(ctx, chunk))
    flops = 4.0 * keys * s.head_dim * s.q_heads
    tflops = flops / (per_call_us * 1e-6) / 1e12
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak = float(json.load(f)["bf16_tflops"])
        kind = "measured"
    except Exception:
        peak, kind = 1590.0, "fallback"
    print(json.dumps({"metric": "paged chunked-prefill attention us per call", "value": per_call_us, "unit": "us",
                      "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
                      "config": {"workload": "%s contexts, last %d tokens of each as the chunk (%d rows), %d q / %d kv "
                                             "heads, d %d, page %d, %s" % (s.name, args.chunk, total, s.q_heads,
                                                                          s.kv_heads, s.head_dim, s.page_size,
                                                                          s.dtype)},
                      "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                                   "frac": tflops / peak, "peak_source": "%s bf16 GEMM" % kind},
                      "gpu_launches": args.steps * L}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "rms_norm":
        return run_rms_norm(args)
    if args.op == "prefill":
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
