"""Benchmark of the graded bit-plane VMM (GRINQH decode hot path) on B200.

Workload (default): the seven decode linears of a Llama3-8B-shaped layer
(q/o 4096x4096, k/v 4096x1024, gate/up 4096x14336, down 14336x4096), batch 1,
weights ~N(0, 0.02) RTN-8 packed as bit planes, fp16 activations ~N(0,1) with a
fixed 1% of channels scaled x20, thresholds calibrated (128 vectors, classes
{0,2,3,4,8}, maximum-entropy P) for average widths 4, 3 and 2 bits.

One step = grinqh_select + grinqh_vmm for each of the 7 linears at each of the 3
widths (21 pairs), every pair on its own packed copy of its layer (6 copies of
the layer in HBM, ~1.3 GB, far above the 126 MB L2), replayed from a CUDA graph.
value = microseconds per select+VMM pair (lower is better).

The roofline entry is for grinqh_vmm alone, timed by a graph of the 21 VMMs with
CUDA events on the launching stream; achieved GB/s counts the algorithmic bytes
of each call: planes sum_k b_k N/8, scale/zero 4 bytes per (active row, 128
columns), x (2K), the channel list (4 per active row) and y (4N).

`--impl reference` times the fp64 CPU oracle (the only reference there is) on a
bounded sample of the same workload on the host cores.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs per batch-1 VMM and effective HBM GB/s (% of peak) vs average bits"
UNIT = "µs"
TARGETS = (4.0, 3.0, 2.0)
WORKLOAD = "llama3-8b decode linears (q,k,v,o,gate,up,down), batch 1, avg bits 4/3/2"
# Stored code width and class set of the workload: b_max = 8 with classes
# {0,2,3,4,8} by default; --bmax 4 or 6 stores b_max-bit codes and grades into
# the paper's even classes {0, 2, ..., b_max} (Section 3.3, b_max in {4, 6, 8}).
BMAX = 8
CLASSES = None   # set in main()
# Layer family: "llama3" (Llama3-8B shapes, weights N(0, 0.02), outlier
# activations, average bits 4/3/2) or "qwen3" (Qwen3-8B shapes, weights with a
# log-uniform per-row std in [0.005, 0.05], Student-t(3) activations, 4/3).
FAMILY = "llama3"


def _family(wl):
    """(shapes, activation draw (K, count, key) -> uint16 bits) of FAMILY."""
    if FAMILY == "qwen3":
        return wl.QWEN3_8B, (lambda K, count, key, li: wl.activations_student_t(K, count, key=key))
    return wl.LLAMA3_8B, (lambda K, count, key, li: wl.activations_outlier(K, count, key=key, chan_key=(1, 0, li)))


def _weights(torch, gen, K, N, dev):
    """Weights of one linear on the GPU from the seeded generator `gen`."""
    W = torch.randn(K, N, generator=gen, device=dev, dtype=torch.float32)
    if FAMILY == "qwen3":
        u = torch.rand(K, 1, generator=gen, device=dev, dtype=torch.float64)
        sig = torch.exp(np.log(0.005) + u * (np.log(0.05) - np.log(0.005))).float()
        return W * sig
    return W * 0.02


def kernel_source_hash():
    """sha256 of the VMM kernel sources (vmm.cu, common.cuh): the key under which a
    traffic capture is valid."""
    import hashlib
    h = hashlib.sha256()
    for f in ("vmm.cu", "common.cuh"):
        with open(os.path.join(ROOT, "activation_graded_bit_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms in the background."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                v = [t.strip() for t in line.split(",")]
                if len(v) >= 9:
                    rows.append(v)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# replicas: every rank runs the whole workload on its own GPU (no exchange on
# the data path); the job's time is the slowest rank's
# ---------------------------------------------------------------------------
def max_over_ranks(value, world, dist_mod=None, device="cpu"):
    """The largest `value` over all ranks, on every rank (value itself when world == 1)."""
    if world <= 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())


def per_pair_us(ms_total, steps, pairs_per_step, world):
    """Whole-job microseconds per select+VMM pair: the slowest rank's time for
    `steps` steps over the pairs that all ranks processed in that time."""
    return ms_total * 1e3 / (steps * pairs_per_step * world)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def build_workload(g, wl, torch, dev, copies=2):
    """Pack `copies` x 3 (one per width) copies of the 7 linears, calibrate per
    linear and width, and draw one input vector per pair."""
    classes = CLASSES
    pairs = []
    gen = torch.Generator(device=dev)
    shapes, draw = _family(wl)
    for li, (name, K, N) in enumerate(shapes):
        Xc = draw(K, 128, (1, 0, li, 1), li)
        Xc_d = torch.from_numpy(Xc.view(np.int16)).to(dev)
        th = {}
        for t in TARGETS:
            th[t] = g.calibrate(Xc_d, classes, P=None, target_bits=t)
        for c in range(copies):
            for ti, t in enumerate(TARGETS):
                gen.manual_seed(1_000_003 * (li + 1) + 7919 * c + 31 * ti)
                W = _weights(torch, gen, K, N, dev)
                p = g.pack(W, b_max=BMAX)
                del W
                x = draw(K, 1, (1, c, li, 2 + ti), li)[0]
                x_d = torch.from_numpy(x.view(np.int16)).to(dev)
                sel = g.select(x_d, th[t], classes)
                pairs.append(dict(name=name, K=K, N=N, target=t, copy=c, packed=p, x=x_d, x_host=x,
                                  th=th[t], sel=sel, ws=g.vmm_workspace(p.layout, dev),
                                  y=torch.empty(N, dtype=torch.float32, device=dev)))
    torch.cuda.synchronize()
    return pairs


def algorithmic_bytes(pair):
    bits = pair["sel"].bits.cpu().numpy().astype(np.int64)
    K, N = pair["K"], pair["N"]
    active = int((bits > 0).sum())
    ng = (N + 127) // 128
    planes = int(bits.sum()) * N / 8.0
    meta = 4.0 * ng * active
    total = planes + meta + 2.0 * K + 4.0 * active + 4.0 * N
    return planes, total, float(bits.mean()), active / K


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from activation_graded_bit_b200 import grinqh as g
    from activation_graded_bit_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    pairs = build_workload(g, wl, torch, dev, copies=args.copies)
    groups = {}
    for pr in pairs:
        groups.setdefault(pr["copy"], []).append(pr)
    copies = sorted(groups)

    stream = torch.cuda.Stream(device=dev)

    def step_pairs(c):
        for pr in groups[c]:
            g.select(pr["x"], pr["th"], CLASSES, out=pr["sel"], stream=stream)
            g.vmm(pr["packed"], pr["x"], pr["sel"], pr["ws"], y=pr["y"], stream=stream)

    def vmm_only(c):
        for pr in groups[c]:
            g.vmm(pr["packed"], pr["x"], pr["sel"], pr["ws"], y=pr["y"], stream=stream)

    # the same graded products through the one-call entry point (grading inside
    # the VMM kernel, no channel lists): reported beside the headline
    def fused_pairs(c):
        for pr in groups[c]:
            g.select_vmm(pr["packed"], pr["x"], pr["th"], CLASSES, pr["ws"], y=pr["y"], stream=stream)

    # e2e: a step's inputs come from pinned host memory in one copy and its
    # outputs go back in one copy: every pair's x and y are views into one
    # device buffer per step (offsets are multiples of 16 bytes)
    io = {}
    for c in copies:
        grp = groups[c]
        xs_dev = torch.empty(sum(pr["K"] for pr in grp), dtype=torch.int16, device=dev)
        ys_dev = torch.empty(sum(pr["N"] for pr in grp), dtype=torch.float32, device=dev)
        xo = yo = 0
        for pr in grp:
            xv = xs_dev[xo:xo + pr["K"]]
            xv.copy_(pr["x"])
            pr["x"] = xv
            pr["y"] = ys_dev[yo:yo + pr["N"]]
            xo += pr["K"]
            yo += pr["N"]
        xs_pin = torch.from_numpy(np.concatenate([pr["x_host"] for pr in grp]).view(np.int16).copy()).pin_memory()
        ys_pin = torch.empty(ys_dev.numel(), dtype=torch.float32).pin_memory()
        io[c] = (xs_dev, ys_dev, xs_pin, ys_pin)
    torch.cuda.synchronize()

    def e2e_pairs(c):
        xs_dev, ys_dev, xs_pin, ys_pin = io[c]
        xs_dev.copy_(xs_pin, non_blocking=True)
        for pr in groups[c]:
            g.select(pr["x"], pr["th"], CLASSES, out=pr["sel"], stream=stream)
            g.vmm(pr["packed"], pr["x"], pr["sel"], pr["ws"], y=pr["y"], stream=stream)
        ys_pin.copy_(ys_dev, non_blocking=True)

    def capture(fn):
        graphs = {}
        with torch.cuda.stream(stream):
            for c in copies:
                fn(c)  # eager warm-up outside capture
            torch.cuda.synchronize()
            for c in copies:
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    fn(c)
                graphs[c] = gr
        torch.cuda.synchronize()
        return graphs

    # the layers the 75%-of-HBM target is stated for: at least 4096 x 4096, 3-4
    # average bits (q, o, gate, up, down at targets 4 and 3)
    def big(pr):
        return pr["K"] >= 4096 and pr["N"] >= 4096 and pr["target"] >= 3.0

    def vmm_big(c):
        for pr in groups[c]:
            if big(pr):
                g.vmm(pr["packed"], pr["x"], pr["sel"], pr["ws"], y=pr["y"], stream=stream)

    g_step = capture(step_pairs)
    g_vmm = capture(vmm_only)
    g_big = capture(vmm_big)
    g_e2e = capture(e2e_pairs)
    g_fused = capture(fused_pairs)

    def timed(graphs, steps, warmup):
        with torch.cuda.stream(stream):
            for i in range(warmup):
                graphs[copies[i % len(copies)]].replay()
        stream.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(steps):
                graphs[copies[i % len(copies)]].replay()
            e1.record(stream)
        stream.synchronize()
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev)
        if world > 1:
            dist.barrier()
        return ms

    n_pairs = len(groups[copies[0]])
    with ClockSampler(local) as clk:
        ms_step = timed(g_step, args.steps, args.warmup)
    clocks = clk.summary()
    ms_vmm = timed(g_vmm, args.steps, args.warmup)
    ms_e2e = timed(g_e2e, args.steps, args.warmup)
    ms_fused = timed(g_fused, args.steps, args.warmup)
    ms_big = timed(g_big, args.steps, args.warmup)

    # correctness spot check of the timed path (one pair) before reporting
    torch.cuda.synchronize()
    y0 = pairs[0]["y"]
    assert bool(torch.isfinite(y0).all()), "non-finite y"

    points = []
    tot_alg = 0.0
    tot_planes = 0.0
    for pr in groups[copies[0]]:
        planes, total, mean_bits, active = algorithmic_bytes(pr)
        tot_alg += total
        tot_planes += planes
        points.append(dict(linear=pr["name"], K=pr["K"], N=pr["N"], target_bits=pr["target"],
                           mean_bits=round(mean_bits, 4), active_frac=round(active, 4),
                           planes_bytes=int(planes), alg_bytes=int(total)))
    peak, peak_kind = _peaks()
    big_pairs = [pr for pr in groups[copies[0]] if big(pr)]
    big_alg = sum(algorithmic_bytes(pr)[1] for pr in big_pairs)
    achieved_big = big_alg * args.steps / (ms_big * 1e-3) / 1e9
    us_pair = ms_step * 1e3 / (args.steps * n_pairs)
    us_vmm = ms_vmm * 1e3 / (args.steps * n_pairs)
    achieved = tot_alg * args.steps / (ms_vmm * 1e-3) / 1e9
    us_fused = ms_fused * 1e3 / (args.steps * n_pairs)
    achieved_fused = tot_alg * args.steps / (ms_fused * 1e-3) / 1e9
    value = per_pair_us(ms_step, args.steps, n_pairs, world)
    e2e_us = per_pair_us(ms_e2e, args.steps, n_pairs, world)
    h2d = sum(2 * pr["K"] for pr in groups[copies[0]])
    d2h = sum(4 * pr["N"] for pr in groups[copies[0]])

    # select + vmm per pair, plus the partial-sum kernel when the layer has more
    # than one row split (the workspace then holds R x n_tiles x 1024 partials)
    launches_per_step = 0
    for pr in groups[copies[0]]:
        L = pr["packed"].layout
        launches_per_step += 2 + (1 if pr["ws"].numel() > 16 + L.n_tiles * 4096 else 0)

    # DRAM traffic per step comes from an ncu capture (profiles/vmm_traffic.json)
    # of the default workload; it is reported only when that capture was taken on
    # the kernel source that runs now (same hash), else null
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "vmm_traffic.json")
    if os.path.exists(tpath) and FAMILY == "llama3" and BMAX == 8:
        try:
            tj = json.load(open(tpath))
            if tj.get("kernel_source_sha256") == kernel_source_hash():
                traffic = tj.get("bytes_per_launch_scaled")
        except Exception:
            traffic = None

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(args)
        out = {
            "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step / args.steps, 6), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "u8 planes, fp32 accumulate", "data": "synthetic",
            "config": _config(n_pairs),
            "parallelism": "replicas only" if world > 1 else "single GPU",
            "resident_bytes": int(sum(pr["packed"].packed.numel() for pr in pairs)),
            "vmm_us": round(us_vmm, 4), "select_plus_vmm_us": round(us_pair, 4),
            "select_vmm_fused": {"us": round(us_fused, 4), "achieved": round(achieved_fused, 1), "unit": "GB/s",
                                 "frac": round(achieved_fused / peak, 4),
                                 "what": "grinqh_select_vmm per (linear, width): grading inside the VMM "
                                         "kernel, no channel lists, same y within the bound"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                         "kernel": "grinqh vmm_kernel"},
            "roofline_target_layers": {
                "what": "grinqh_vmm on the layers of at least 4096 x 4096 at 3-4 average bits (q, o, gate, up, "
                        "down at targets 4 and 3): algorithmic bytes / time of a graph of those %d calls" % len(big_pairs),
                "us_per_vmm": round(ms_big * 1e3 / (args.steps * len(big_pairs)), 4),
                "achieved": round(achieved_big, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved_big / peak, 4), "peak_kind": peak_kind},
            "points": points,
            "e2e": {"value": round(e2e_us, 4), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
        }
        if cpu is not None:
            out["cpu_baseline"] = cpu
        print(json.dumps(out))
    # release graphs before tearing down the process group
    del g_step, g_vmm, g_e2e, g_big
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# oracle timing (host cores)
# ---------------------------------------------------------------------------
def _oracle_sample(budget_s, nthreads):
    """Time oracle select + vmm on a bounded sample of the workload's pairs."""
    import oracle
    from activation_graded_bit_b200 import workloads as wl
    classes = np.array(CLASSES, np.uint8)
    done = 0
    secs = 0.0
    names = []
    t_start = time.time()
    shapes, draw = _family(wl)
    for li, (name, K, N) in enumerate(shapes):
        if time.time() - t_start > budget_s:
            break
        # untimed setup: weights, RTN codes, thresholds of this linear
        W = (wl.weights_rowstd_loguniform(K, N, key=(1, 9, li, 0)) if FAMILY == "qwen3"
             else wl.weights_gaussian(K, N, key=(1, 9, li, 0)))
        q, s, z = oracle.rtn_quantize(W, BMAX)
        del W
        Xc = draw(K, 32, (1, 0, li, 1), li)
        for ti, t in enumerate(TARGETS):
            th = oracle.thresholds(Xc, oracle.maxent_distribution(classes, t))
            x = draw(K, 1, (1, 0, li, 2 + ti), li)[0]
            t0 = time.perf_counter()
            bits, idx, off = oracle.select(x, th, classes)
            oracle.vmm(x, q, s, z, bits, nthreads=nthreads, bmax=BMAX)
            secs += time.perf_counter() - t0
            done += 1
            names.append("%s@%g" % (name, t))
            if time.time() - t_start > budget_s:
                break
    return done, secs, names


def _cpu_model():
    """The host CPU's model name (first 'model name' line of /proc/cpuinfo), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(args):
    nthreads = os.cpu_count() or 1
    done, secs, names = _oracle_sample(args.cpu_budget, nthreads)
    # the same oracle on one thread, on a shorter bounded sample (the first pairs)
    done1, secs1, names1 = _oracle_sample(min(5.0, args.cpu_budget / 4.0), 1)
    return {"value": round(secs * 1e6 / max(done, 1), 1), "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "sample": "fp64 oracle select+vmm on %d of the %d (linear, width) pairs: %s" % (
                done, 7 * len(TARGETS), ", ".join(names)),
            "single_thread": {"value": round(secs1 * 1e6 / max(done1, 1), 1), "unit": UNIT, "cores": 1,
                              "sample": ", ".join(names1)},
            "cpu_model": _cpu_model()}


def _config(n_pairs):
    """The workload description both arms print (the same dict: same config)."""
    return {"workload": WORKLOAD, "pairs_per_step": n_pairs, "classes": list(CLASSES), "b_max": BMAX,
            "l2": "inputs larger than L2: every pair of a step reads its own packed copy of its layer, "
                  "the copies rotate"}


def _oracle_pairs(cols):
    """Untimed setup of the reference arm: for each of the 21 (linear, width)
    pairs of a step, the same weights, thresholds and activation vector as the
    CPU baseline draws, RTN codes of a column sample (`cols` columns as whole
    128-column groups spread over the layer, the last group included)."""
    import oracle
    from activation_graded_bit_b200 import workloads as wl
    classes = np.array(CLASSES, np.uint8)
    shapes, draw = _family(wl)
    pairs = []
    for li, (name, K, N) in enumerate(shapes):
        W = (wl.weights_rowstd_loguniform(K, N, key=(1, 9, li, 0)) if FAMILY == "qwen3"
             else wl.weights_gaussian(K, N, key=(1, 9, li, 0)))
        ng = (N + 127) // 128
        take = max(1, min(ng, cols // 128))
        groups = sorted(set(np.linspace(0, ng - 1, take).round().astype(int).tolist()))
        sel_cols = np.concatenate([np.arange(128 * g, min(N, 128 * g + 128)) for g in groups])
        q, s, z = oracle.rtn_quantize(np.ascontiguousarray(W[:, sel_cols]), BMAX)
        del W
        Xc = draw(K, 32, (1, 0, li, 1), li)
        for ti, t in enumerate(TARGETS):
            th = oracle.thresholds(Xc, oracle.maxent_distribution(classes, t))
            x = draw(K, 1, (1, 0, li, 2 + ti), li)[0]
            pairs.append(dict(name="%s@%g" % (name, t), x=x, th=th, q=q, s=s, z=z, N=N, n=len(sel_cols)))
    return pairs


def run_reference(args):
    """The reference arm: the fp64 CPU oracle (select + VMM) on every one of the
    step's 21 (linear, width) pairs, each step. Selection runs on the whole
    vector; the VMM on a column sample of each layer, its time scaled by
    N / sampled columns (the oracle's VMM time is linear in the columns it
    computes). value = mean microseconds per pair, like the GPU arm."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    nthreads = os.cpu_count() or 1
    cols = 1024
    pairs = _oracle_pairs(cols)
    classes = np.array(CLASSES, np.uint8)
    per_step = []
    for i in range(args.warmup + args.steps):
        tot = 0.0
        for pr in pairs:
            t0 = time.perf_counter()
            bits, idx, off = oracle.select(pr["x"], pr["th"], classes)
            t1 = time.perf_counter()
            oracle.vmm(pr["x"], pr["q"], pr["s"], pr["z"], bits, nthreads=nthreads, bmax=BMAX)
            t2 = time.perf_counter()
            tot += (t1 - t0) + (t2 - t1) * pr["N"] / pr["n"]
        if i >= args.warmup:
            per_step.append(tot / len(pairs))
    v = statistics.mean(per_step) * 1e6
    sample = ("fp64 oracle select (whole x) + vmm on %d-column samples of each layer (time scaled by N/%d), "
              "all %d (linear, width) pairs every step" % (cols, cols, len(pairs)))
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": UNIT, "n_gpus": 0,
           "steps": args.steps, "warmup": args.warmup, "higher_is_better": False, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": _config(len(pairs)), "parallelism": "host cores",
           "cpu_baseline": {"value": round(v, 1), "unit": UNIT, "cores": nthreads, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(v, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out))


def run_profile_case(args):
    """One (linear, width) pair, `--iters` eager select+vmm calls (select+vmm_lut
    over synthetic table codes with --lut), no timing: the small case that ncu
    captures."""
    import torch
    from activation_graded_bit_b200 import grinqh as g
    from activation_graded_bit_b200 import workloads as wl
    shapes = {name: (li, K, N) for li, (name, K, N) in enumerate(wl.LLAMA3_8B)}
    li, K, N = shapes[args.profile]
    dev = torch.device("cuda", 0)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1_000_003 * (li + 1))
    W = torch.randn(K, N, generator=gen, device=dev, dtype=torch.float32) * 0.02
    p = g.pack(W)
    del W
    Xc = wl.activations_outlier(K, 128, key=(1, 0, li, 1), chan_key=(1, 0, li))
    th = g.calibrate(torch.from_numpy(Xc.view(np.int16)).to(dev), wl.CLASSES, P=None, target_bits=args.bits)
    x = wl.activations_outlier(K, 1, key=(1, 0, li, 2), chan_key=(1, 0, li))[0]
    x_d = torch.from_numpy(x.view(np.int16)).to(dev)
    ws = g.vmm_workspace(p.layout, dev)
    y = torch.empty(N, dtype=torch.float32, device=dev)
    sel = g.empty_selection(K, wl.CLASSES, dev)
    if args.prefill or args.batch:
        _profile_tc(args, g, wl, p, th, K, N, li, dev)
        return
    if args.lut:
        # nested table codes on the same layer: synthetic codes and tables
        codes = torch.randint(0, 256, (K, N), generator=gen, device=dev, dtype=torch.uint8)
        p = g.pack_codes(codes)
        del codes
        lut = torch.randn((K, 512), generator=gen, device=dev).half().view(torch.int16).contiguous()
    for _ in range(args.iters):
        g.select(x_d, th, wl.CLASSES, out=sel)
        if args.lut:
            g.vmm_lut(p, lut, x_d, sel, ws, y=y)
        else:
            g.vmm(p, x_d, sel, ws, y=y)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y).all())
    # the counts a capture is divided by: (row, tile) records of nonzero width and
    # the algorithmic bytes of one call (planes of the selected widths, the
    # records' scale/zero words, x, the channel list and y)
    bits = sel.bits.cpu().numpy().astype(np.int64)
    active = int((bits > 0).sum())
    alg = bits.sum() * N / 8.0 + 4.0 * ((N + 127) // 128) * active + 2.0 * K + 4.0 * active + 4.0 * N
    print("profile case %s @ %g bits: %d select+%s calls; %d active rows, %d records, %d algorithmic bytes"
          % (args.profile, args.bits, args.iters, "vmm_lut" if args.lut else "vmm", active,
             active * p.layout.n_tiles, int(alg)))


def _profile_tc(args, g, wl, p, th, K, N, li, dev):
    """The tensor-core kernels' small case: `--iters` eager grinqh_prefill_tc calls
    (with --prefill) or grinqh_select_vmm_batch_tc calls (with --batch) on one
    linear at `--tokens` tokens, and the flop and algorithmic byte counts a
    capture is divided by."""
    import torch
    T = args.tokens if args.tokens else (2048 if args.prefill else 16)
    X = wl.activations_outlier(K, T, key=(1, 1, li, T), chan_key=(1, 0, li))
    X_d = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).to(dev)
    Y = torch.empty((T, N), dtype=torch.float32, device=dev)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    for _ in range(args.iters):
        if args.prefill:
            g.prefill_tc(p, X_d, status, Y=Y)
        else:
            g.select_vmm_batch_tc(p, X_d, th, wl.CLASSES, status, Y=Y)
    torch.cuda.synchronize()
    assert int(status.count_nonzero()) == 0 and bool(torch.isfinite(Y).all())
    # prefill: every row at b_max, 2 T K N flops; planes + scale/zero words read
    # once, X read, Y written. batch: the rows some token grades nonzero, read once.
    alg = p.packed.numel() + 2.0 * K * T + 4.0 * N * T
    print("profile case %s %s: %d calls at %d tokens; %.4g flops per call (2 T K N), %d algorithmic bytes"
          % (args.profile, "prefill_tc" if args.prefill else "select_vmm_batch_tc @ %g bits" % args.bits,
             args.iters, T, 2.0 * T * K * N, int(alg)))


# ---------------------------------------------------------------------------
# extra measurements: the average-bit sweep and the 32-layer linear stack
# ---------------------------------------------------------------------------
def _graph_time_us(torch, stream, fn, reps, warmup=3):
    """Mean microseconds of one fn(stream) call, replayed from a CUDA graph of
    `reps` calls, timed with events on the stream (median of 5 replays)."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            fn(stream)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for _ in range(reps):
                fn(stream)
        gr.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(5):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            gr.replay()
            e1.record(stream)
            stream.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3 / reps)
    del gr
    return statistics.median(ts)


def run_sweep(args):
    """Average-bit sweep: microseconds, effective GB/s and roofline fraction of
    the VMM (and of select+VMM and the fused call) against the achieved mean
    width, with a least-squares line t = a + b * mean_bits per shape and
    activation distribution. Shapes: the 14336x4096 down-proj layer (Gaussian
    and SiLU(a)*b activations) and the pages' isolated-kernel matrix 16384x4096
    (Section 4 "Setup for Kernel Benchmarking", Appendix C.2 Fig. 11; Gaussian
    activations), the latter also at the figure's configuration: b_max 8, target
    4 bits, uniformly distributed thresholds, read as the five even widths
    {0, 2, 4, 6, 8} with equal shares (mean width 4)."""
    import torch
    from activation_graded_bit_b200 import grinqh as g
    from activation_graded_bit_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    peak, peak_kind = _peaks()
    points = []
    fits = {}
    shapes = (("down_proj 14336x4096", 14336, 4096, ("gaussian", "silu_gated")),
              ("isolated 16384x4096", 16384, 4096, ("gaussian",)))
    for si, (label, K, N, dists) in enumerate(shapes):
        copies = []
        for c in range(6):   # 6 packed copies (>= 360 MB): a replay of one point never finds the weights in L2
            gen = torch.Generator(device=dev)
            gen.manual_seed(3_000_017 + 101 * si + c)
            copies.append(g.pack(torch.randn(K, N, generator=gen, device=dev, dtype=torch.float32) * 0.02))
        ws = g.vmm_workspace(copies[0].layout, dev)
        y = torch.empty(N, dtype=torch.float32, device=dev)
        runs = [(d, wl.CLASSES, t, None) for d in dists for t in (0.5, 1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 8.0)]
        if si == 1:
            runs.append(("gaussian", (0, 2, 4, 6, 8), 4.0, [0.2] * 5))   # Fig. 11's configuration
        for dist, classes, t, P in runs:
            gen_x = wl.activations_gaussian if dist == "gaussian" else wl.activations_silu_gated
            Xc = torch.from_numpy(gen_x(K, 128, key=(3, 1, dist == "gaussian", si)).view(np.int16)).to(dev)
            x = torch.from_numpy(gen_x(K, 1, key=(3, 2, dist == "gaussian", si))[0].view(np.int16)).to(dev)
            th = (g.calibrate(Xc, classes, P=np.array(P, np.float64)) if P is not None
                  else g.calibrate(Xc, classes, target_bits=t))
            sel = g.select(x, th, classes)
            torch.cuda.synchronize()
            bits = sel.bits.cpu().numpy().astype(np.int64)
            active = int((bits > 0).sum())
            alg = bits.sum() * N / 8.0 + 4.0 * ((N + 127) // 128) * active + 2.0 * K + 4.0 * active + 4.0 * N

            def vmm_only(st, sel=sel):
                for p in copies:
                    g.vmm(p, x, sel, ws, y=y, stream=st)

            def pair(st, sel=sel, th=th, classes=classes):
                for p in copies:
                    g.select(x, th, classes, out=sel, stream=st)
                    g.vmm(p, x, sel, ws, y=y, stream=st)

            def fused(st, th=th, classes=classes):
                for p in copies:
                    g.select_vmm(p, x, th, classes, ws, y=y, stream=st)
            tv = _graph_time_us(torch, stream, vmm_only, reps=8) / len(copies)
            tp = _graph_time_us(torch, stream, pair, reps=8) / len(copies)
            tf = _graph_time_us(torch, stream, fused, reps=8) / len(copies)
            points.append(dict(shape=label, K=K, N=N, dist=dist, classes=list(classes), target_bits=t,
                               thresholds="uniform shares" if P is not None else "maximum entropy",
                               mean_bits=round(float(bits.mean()), 4), active_frac=round(active / K, 4),
                               alg_bytes=int(alg), vmm_us=round(tv, 3), select_plus_vmm_us=round(tp, 3),
                               select_vmm_fused_us=round(tf, 3), gbs=round(alg / (tv * 1e-6) / 1e9, 1),
                               frac=round(alg / (tv * 1e-6) / 1e9 / peak, 4)))
        for dist in dists:
            pts = [q for q in points if q["shape"] == label and q["dist"] == dist and q["thresholds"] != "uniform shares"]
            xb = np.array([q["mean_bits"] for q in pts])
            tt = np.array([q["vmm_us"] for q in pts])
            slope, icpt = np.polyfit(xb, tt, 1)
            pred = icpt + slope * xb
            r2 = 1.0 - float(((tt - pred) ** 2).sum() / ((tt - tt.mean()) ** 2).sum())
            fits["%s %s" % (label, dist)] = dict(us_per_bit=round(float(slope), 4), us_at_0_bits=round(float(icpt), 4),
                                                 r2=round(r2, 5))
        del copies
        torch.cuda.empty_cache()
    print(json.dumps({"metric": "vmm us, effective GB/s and roofline fraction vs average bits", "unit": UNIT,
                      "higher_is_better": False, "data": "synthetic", "peak": peak, "peak_kind": peak_kind,
                      "config": {"workload": "14336x4096 and 16384x4096 layers, 6 packed copies rotated per shape"},
                      "points": points, "linear_fit": fits}))


def run_stack(args):
    """The 32-layer Llama3-8B linear stack (7 linears per layer), batch-1 decode
    at 3 average bits: select + VMM for all 224 linears of a step chained on one
    stream; tokens/s = steps / time. Activations rotate over 8 seeded sets (one
    graph each): per layer one x for q/k/v, one for o, one for gate/up, one for
    down. Measured twice: as 7 separate linears with thresholds calibrated per
    linear, and grouped the way a serving stack packs them, with the linears
    that read the same x concatenated along N ([q|k|v] 4096 x 6144, [gate|up]
    4096 x 28672; the same weights) and one set of thresholds per input vector
    (Section 3.2 computes a layer's thresholds from the activations that enter
    it, so linears reading the same x share them): 4 select + VMM pairs per
    layer instead of 7."""
    import torch
    from activation_graded_bit_b200 import grinqh as g
    from activation_graded_bit_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    classes = wl.CLASSES
    n_layers, n_sets = 32, 8
    src = {"q_proj": 0, "k_proj": 0, "v_proj": 0, "o_proj": 1, "gate_proj": 2, "up_proj": 2, "down_proj": 3}
    lin, grp = [], []
    for layer in range(n_layers):
        Ws = {}
        for li, (name, K, N) in enumerate(wl.LLAMA3_8B):
            gen = torch.Generator(device=dev)
            gen.manual_seed(4_000_037 * (layer + 1) + li)
            Ws[name] = torch.randn(K, N, generator=gen, device=dev, dtype=torch.float32) * 0.02
            p = g.pack(Ws[name])
            Xc = wl.activations_outlier(K, 128, key=(4, layer, li, 1), chan_key=(4, layer, li))
            th = g.calibrate(torch.from_numpy(Xc.view(np.int16)).to(dev), classes, target_bits=3.0)
            lin.append(dict(layer=layer, name=name, K=K, N=N, p=p, th=th, sel=g.empty_selection(K, classes, dev),
                            ws=g.vmm_workspace(p.layout, dev), y=torch.empty(N, dtype=torch.float32, device=dev)))
        for sname, names in ((0, ("q_proj", "k_proj", "v_proj")), (1, ("o_proj",)), (2, ("gate_proj", "up_proj")),
                             (3, ("down_proj",))):
            W = torch.cat([Ws[nm] for nm in names], dim=1).contiguous()
            K, N = W.shape
            p = g.pack(W)
            del W
            Xc = wl.activations_outlier(K, 128, key=(4, layer, 100 + sname, 1), chan_key=(4, layer, 0))
            th = g.calibrate(torch.from_numpy(Xc.view(np.int16)).to(dev), classes, target_bits=3.0)
            grp.append(dict(layer=layer, src=sname, K=K, N=N, p=p, th=th, sel=g.empty_selection(K, classes, dev),
                            ws=g.vmm_workspace(p.layout, dev), y=torch.empty(N, dtype=torch.float32, device=dev)))
        del Ws
    # x[set][layer][source]
    xs = [[[torch.from_numpy(wl.activations_outlier(14336 if s == 3 else 4096, 1, key=(4, 9, k, layer, s),
                                                    chan_key=(4, layer, 0))[0].view(np.int16)).to(dev)
            for s in range(4)] for layer in range(n_layers)] for k in range(n_sets)]
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device=dev)

    def step_sep(st, k):
        for d in lin:
            x = xs[k][d["layer"]][src[d["name"]]]
            g.select(x, d["th"], classes, out=d["sel"], stream=st)
            g.vmm(d["p"], x, d["sel"], d["ws"], y=d["y"], stream=st)

    def step_grp(st, k):
        for d in grp:
            x = xs[k][d["layer"]][d["src"]]
            g.select(x, d["th"], classes, out=d["sel"], stream=st)
            g.vmm(d["p"], x, d["sel"], d["ws"], y=d["y"], stream=st)

    def step_grp_fused(st, k):
        for d in grp:
            g.select_vmm(d["p"], xs[k][d["layer"]][d["src"]], d["th"], classes, d["ws"], y=d["y"], stream=st)

    def tokens_per_s(step):
        graphs = []
        with torch.cuda.stream(stream):
            for k in range(n_sets):
                step(stream, k)
            torch.cuda.synchronize()
            for k in range(n_sets):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    step(stream, k)
                graphs.append(gr)
            for i in range(max(args.warmup, 3)):
                graphs[i % n_sets].replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(args.stack_steps):
                graphs[i % n_sets].replay()
            e1.record(stream)
        stream.synchronize()
        ms = e0.elapsed_time(e1)
        del graphs
        return ms

    ms = tokens_per_s(step_sep)
    ms_g = tokens_per_s(step_grp)
    ms_gf = tokens_per_s(step_grp_fused)
    assert all(bool(torch.isfinite(d["y"]).all()) for d in lin[:7] + grp[:4])
    packed_gb = sum(d["p"].packed.numel() for d in lin) / 1e9
    print(json.dumps({"metric": "linear-stack tokens/s (32 x 7 Llama3-8B linears, batch 1, 3 average bits)",
                      "value": round(args.stack_steps / (ms * 1e-3), 2), "unit": "tokens/s", "higher_is_better": True,
                      "steps": args.stack_steps, "warmup": max(args.warmup, 3), "ms_per_token": round(ms / args.stack_steps, 4),
                      "data": "synthetic", "config": {"workload": "32-layer Llama3-8B linear stack, %.2f GB packed, "
                                                      "8 activation sets rotated, thresholds per linear" % packed_gb},
                      "gpu_launches_per_token": 2 * len(lin) + sum(1 for d in lin if d["ws"].numel() > 16),
                      "grouped": {"value": round(args.stack_steps / (ms_g * 1e-3), 2), "unit": "tokens/s",
                                  "ms_per_token": round(ms_g / args.stack_steps, 4),
                                  "what": "same weights, [q|k|v] and [gate|up] concatenated along N, thresholds "
                                          "per input vector: 4 select + VMM pairs per layer",
                                  "gpu_launches_per_token": 2 * len(grp) + sum(1 for d in grp if d["ws"].numel() > 16)},
                      "grouped_fused": {"value": round(args.stack_steps / (ms_gf * 1e-3), 2), "unit": "tokens/s",
                                        "ms_per_token": round(ms_gf / args.stack_steps, 4),
                                        "what": "the grouped stack through grinqh_select_vmm (grading inside the "
                                                "VMM kernel, no channel lists): 4 calls per layer",
                                        "gpu_launches_per_token": len(grp) + sum(1 for d in grp if d["ws"].numel() > 16)}}))

def run_batch(args):
    """Batch > 1 on the Llama3-8B step (21 (linear, width) pairs, two packed copies
    rotated): for T tokens per call, microseconds per call and per token,
    graph-replayed, through grinqh_select_vmm_batch (every token graded and rebuilt
    as at batch one) and through grinqh_select_vmm_batch_tc (rows rebuilt once for
    all tokens, width classes as tensor-core MMAs); the T activation vectors of a
    pair are drawn like the batch-1 ones."""
    import torch
    from activation_graded_bit_b200 import grinqh as g
    from activation_graded_bit_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    pairs = build_workload(g, wl, torch, dev, copies=2)
    groups = {}
    for pr in pairs:
        groups.setdefault(pr["copy"], []).append(pr)
    copies = sorted(groups)
    stream = torch.cuda.Stream(device=dev)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    out = []

    def timed(step):
        graphs = {}
        with torch.cuda.stream(stream):
            for c in copies:
                step(c)
            torch.cuda.synchronize()
            for c in copies:
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    step(c)
                graphs[c] = gr
            for i in range(args.warmup):
                graphs[copies[i % len(copies)]].replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            steps = max(args.steps // 10, 20)
            e0.record(stream)
            for i in range(steps):
                graphs[copies[i % len(copies)]].replay()
            e1.record(stream)
        stream.synchronize()
        del graphs
        return e0.elapsed_time(e1) * 1e3 / (steps * len(groups[copies[0]]))

    for T in (1, 2, 4, 8, 16, 32, 64):
        for pr in pairs:
            X = wl.activations_outlier(pr["K"], T, key=(7, pr["copy"], T, pr["K"], pr["N"], int(pr["target"])),
                                       chan_key=(1, 0, 0))
            pr["X"] = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).to(dev)
            pr["Y"] = torch.empty((T, pr["N"]), dtype=torch.float32, device=dev)
            pr["wsT"] = g.vmm_batch_workspace(pr["packed"].layout, T, dev)

        def step(c):
            for pr in groups[c]:
                g.select_vmm_batch(pr["packed"], pr["X"], pr["th"], CLASSES, pr["wsT"], Y=pr["Y"], stream=stream)

        def step_tc(c):
            for pr in groups[c]:
                g.select_vmm_batch_tc(pr["packed"], pr["X"], pr["th"], CLASSES, status, Y=pr["Y"], stream=stream)
        us_call = timed(step)
        us_tc = timed(step_tc)
        torch.cuda.synchronize()
        assert int(status.count_nonzero()) == 0, "the tensor-core batch reported a status"
        out.append({"tokens": T, "us_per_call": round(us_call, 3), "us_per_token": round(us_call / T, 3),
                    "tc_us_per_call": round(us_tc, 3), "tc_us_per_token": round(us_tc / T, 3)})
        assert all(bool(torch.isfinite(pr["Y"]).all()) for pr in groups[copies[0]])
    print(json.dumps({"metric": "batched graded VMM: us per (linear, width) call and per token vs batch size "
                                "(per-token kernel and tensor-core kernel)",
                      "unit": "µs", "higher_is_better": False, "data": "synthetic",
                      "config": {"workload": WORKLOAD.replace("batch 1", "batch 1..64"), "classes": list(CLASSES),
                                 "b_max": BMAX, "l2": "two packed copies of the layer set rotate"},
                      "points": out}))


def run_lut(args):
    """Nested look-up-table codes through grinqh_vmm_lut on the decode step (the
    same 21 (linear, width) pairs, selections and two rotated copies as the main
    run): synthetic b_max-bit codes and binary16 tables (timing does not depend
    on their values), microseconds per VMM and per select+VMM pair, graph-replayed,
    with grinqh_vmm on the uniform codes of the same pairs timed beside it."""
    import torch
    from activation_graded_bit_b200 import grinqh as g
    from activation_graded_bit_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    pairs = build_workload(g, wl, torch, dev, copies=2)
    gen = torch.Generator(device=dev)
    E = 1 << (BMAX + 1)
    tot_alg = 0.0
    for i, pr in enumerate(pairs):
        K, N = pr["K"], pr["N"]
        gen.manual_seed(2_000_003 + 7919 * i)
        codes = torch.randint(0, 1 << BMAX, (K, N), generator=gen, device=dev, dtype=torch.uint8)
        pr["packed_lut"] = g.pack_codes(codes, b_max=BMAX)
        del codes
        pr["lut"] = torch.randn((K, E), generator=gen, device=dev).half().view(torch.int16).contiguous()
        if pr["copy"] == 0:
            bits = pr["sel"].bits.cpu().numpy().astype(np.int64)
            active = bits > 0
            # planes + each active row's width-b table once + x + channel list + y
            tot_alg += (bits.sum() * N / 8.0 + float((2 << bits[active]).sum()) + 2.0 * K
                        + 4.0 * int(active.sum()) + 4.0 * N)
    torch.cuda.synchronize()
    groups = {}
    for pr in pairs:
        groups.setdefault(pr["copy"], []).append(pr)
    copies = sorted(groups)
    n_pairs = len(groups[copies[0]])
    stream = torch.cuda.Stream(device=dev)

    def graphs_of(fn):
        out = {}
        with torch.cuda.stream(stream):
            for c in copies:
                fn(c)
            torch.cuda.synchronize()
            for c in copies:
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    fn(c)
                out[c] = gr
        torch.cuda.synchronize()
        return out

    def lut_only(c):
        for pr in groups[c]:
            g.vmm_lut(pr["packed_lut"], pr["lut"], pr["x"], pr["sel"], pr["ws"], y=pr["y"], stream=stream)

    def lut_pairs(c):
        for pr in groups[c]:
            g.select(pr["x"], pr["th"], CLASSES, out=pr["sel"], stream=stream)
            g.vmm_lut(pr["packed_lut"], pr["lut"], pr["x"], pr["sel"], pr["ws"], y=pr["y"], stream=stream)

    def uniform_only(c):
        for pr in groups[c]:
            g.vmm(pr["packed"], pr["x"], pr["sel"], pr["ws"], y=pr["y"], stream=stream)

    def timed(graphs):
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                graphs[copies[i % len(copies)]].replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(args.steps):
                graphs[copies[i % len(copies)]].replay()
            e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1) * 1e3 / (args.steps * n_pairs)

    us_lut = timed(graphs_of(lut_only))
    us_pair = timed(graphs_of(lut_pairs))
    us_uni = timed(graphs_of(uniform_only))
    assert all(bool(torch.isfinite(pr["y"]).all()) for pr in pairs)
    peak, peak_kind = _peaks()
    achieved = tot_alg / n_pairs / (us_lut * 1e-6) / 1e9
    print(json.dumps({"metric": "grinqh_vmm_lut: µs per batch-1 VMM over nested look-up-table codes",
                      "value": round(us_lut, 4), "unit": "µs", "higher_is_better": False, "steps": args.steps,
                      "warmup": args.warmup, "data": "synthetic codes and tables",
                      "config": {"workload": WORKLOAD, "classes": list(CLASSES), "b_max": BMAX,
                                 "l2": "two packed copies of the layer set rotate (inputs larger than L2)"},
                      "select_plus_vmm_lut_us": round(us_pair, 4), "vmm_uniform_us_same_run": round(us_uni, 4),
                      "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                                   "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                                   "bytes_per_step": tot_alg}}))


def run_cold(args):
    """Isolated cold calls: for every (linear, width) pair of the decode step, one
    grinqh_select and one grinqh_vmm (with its partial sums) right after a write of
    twice the L2 size, each bracketed by CUDA events on the launching stream;
    median over `--iters` repetitions per pair (one untimed first repetition)."""
    import torch
    from activation_graded_bit_b200 import grinqh as g
    from activation_graded_bit_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    pairs = build_workload(g, wl, torch, dev, copies=1)
    stream = torch.cuda.Stream(device=dev)
    l2 = int(torch.cuda.get_device_properties(dev).L2_cache_size)
    flush = torch.empty(max(2 * l2 // 4, 1 << 20), dtype=torch.float32, device=dev)
    reps = max(args.iters, 5)
    peak, peak_kind = _peaks()
    points = []
    for pr in pairs:
        t_sel, t_vmm = [], []
        for r in range(reps + 1):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e2 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                flush.fill_(float(r))
                e0.record(stream)
                g.select(pr["x"], pr["th"], CLASSES, out=pr["sel"], stream=stream)
                e1.record(stream)
                g.vmm(pr["packed"], pr["x"], pr["sel"], pr["ws"], y=pr["y"], stream=stream)
                e2.record(stream)
            stream.synchronize()
            if r > 0:
                t_sel.append(e0.elapsed_time(e1) * 1e3)
                t_vmm.append(e1.elapsed_time(e2) * 1e3)
        tv = statistics.median(t_vmm)
        alg = algorithmic_bytes(pr)[1]
        points.append({"linear": pr["name"], "K": pr["K"], "N": pr["N"], "target_bits": pr["target"],
                       "select_us": round(statistics.median(t_sel), 3), "vmm_us": round(tv, 3),
                       "alg_bytes": int(alg), "frac": round(alg / (tv * 1e-6) / 1e9 / peak, 4)})
    assert all(bool(torch.isfinite(pr["y"]).all()) for pr in pairs)
    n = len(points)
    print(json.dumps({"metric": "isolated cold select and VMM: µs per call after an L2 flush",
                      "unit": "µs", "higher_is_better": False, "data": "synthetic",
                      "config": {"workload": WORKLOAD, "classes": list(CLASSES), "b_max": BMAX,
                                 "l2": "%d bytes written before every call pair (2x L2)" % (4 * flush.numel()),
                                 "repetitions": reps},
                      "peak": peak, "peak_kind": peak_kind,
                      "select_us_mean": round(sum(p["select_us"] for p in points) / n, 3),
                      "vmm_us_mean": round(sum(p["vmm_us"] for p in points) / n, 3),
                      "points": points}))


def run_prefill(args):
    """The prefill path on the Llama3-8B linears (Section 4 of the paper: unpack at
    full b_max precision, then a dense product): for T tokens, microseconds of the
    fused tensor-core product grinqh_prefill_tc (weights rebuilt into the MMA's
    operand tiles), of grinqh_dequant alone and of grinqh_prefill (dequant + library
    fp16 GEMM), TFLOP/s of each (2 T K N flops) against the measured bf16 GEMM peak
    (binary16 runs at the bf16 rate), and the dequant's GB/s (plane and scale/zero
    bytes read + 2 K N written) against the measured copy bandwidth. Graph-replayed
    over two packed copies."""
    import torch
    from activation_graded_bit_b200 import grinqh as g
    from activation_graded_bit_b200 import workloads as wl
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device=dev)
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        pass
    tflops_peak = float(peaks.get("bf16_tflops", 1590.0))
    tflops_sust = float(peaks.get("bf16_tflops_sustained", 1400.0))
    hbm_peak, hbm_kind = _peaks()
    lin = []
    for li, (name, K, N) in enumerate(wl.LLAMA3_8B):
        ps = []
        for c in range(2):
            gen = torch.Generator(device=dev)
            gen.manual_seed(6_000_011 * (li + 1) + c)
            ps.append(g.pack(torch.randn(K, N, generator=gen, device=dev, dtype=torch.float32) * 0.02))
        lin.append(dict(name=name, K=K, N=N, p=ps, W16=[torch.empty((K, N), dtype=torch.float16, device=dev)
                                                         for _ in range(2)]))
    out = []
    for T in (512, 2048):
        for d in lin:
            X = wl.activations_outlier(d["K"], T, key=(6, T, d["K"], d["N"]), chan_key=(6, d["K"]))
            d["X"] = torch.from_numpy(np.ascontiguousarray(X).view(np.int16)).to(dev)
            d["Y"] = torch.empty((T, d["N"]), dtype=torch.float32, device=dev)

        def timed(fn, reps=20):
            with torch.cuda.stream(stream):
                fn(0)
                fn(1)
                torch.cuda.synchronize()
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=stream):
                    for r in range(reps):
                        fn(r % 2)
                gr.replay()
                torch.cuda.synchronize()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                gr.replay()
                e1.record(stream)
            stream.synchronize()
            del gr
            return e0.elapsed_time(e1) * 1e3 / reps

        status = torch.zeros(4, dtype=torch.int32, device=dev)
        for d in lin:
            K, N = d["K"], d["N"]
            us_tc = timed(lambda c: g.prefill_tc(d["p"][c], d["X"], status, Y=d["Y"], stream=stream))
            us_deq = timed(lambda c: g.dequant(d["p"][c], out=d["W16"][c], stream=stream))
            us_all = timed(lambda c: g.prefill(d["p"][c], d["X"], Y=d["Y"], W16=d["W16"][c], stream=stream))
            flops = 2.0 * T * K * N
            deq_bytes = d["p"][0].packed.numel() + 2.0 * K * N
            out.append({"linear": d["name"], "K": K, "N": N, "tokens": T,
                        "prefill_tc_us": round(us_tc, 2), "tc_tflops": round(flops / (us_tc * 1e-6) / 1e12, 1),
                        "tc_frac": round(flops / (us_tc * 1e-6) / 1e12 / tflops_peak, 4),
                        "tc_frac_sustained": round(flops / (us_tc * 1e-6) / 1e12 / tflops_sust, 4),
                        "dequant_gemm_us": round(us_all, 2),
                        "dequant_us": round(us_deq, 2), "tflops": round(flops / (us_all * 1e-6) / 1e12, 1),
                        "tflops_frac": round(flops / (us_all * 1e-6) / 1e12 / tflops_peak, 4),
                        "dequant_gbs": round(deq_bytes / (us_deq * 1e-6) / 1e9, 1),
                        "dequant_frac": round(deq_bytes / (us_deq * 1e-6) / 1e9 / hbm_peak, 4)})
        torch.cuda.synchronize()
        assert int(status.count_nonzero()) == 0, "a wait inside the tensor-core prefill gave up"
    print(json.dumps({"metric": "prefill: us per linear and TFLOP/s of the fused tensor-core product "
                                "(grinqh_prefill_tc) and of dequant + library fp16 GEMM (grinqh_prefill)",
                      "unit": "µs", "higher_is_better": False, "data": "synthetic",
                      "peak_tflops": tflops_peak, "peak_tflops_sustained": tflops_sust, "peak_gbs": hbm_peak,
                      "peak_kind": hbm_kind,
                      "config": {"workload": "llama3-8b linears, prefill of 512 and 2048 tokens, b_max 8 codes, "
                                             "two packed copies rotated"},
                      "points": out}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--copies", type=int, default=2)
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", default=None, help="linear name: run one small case for ncu and exit")
    ap.add_argument("--bits", type=float, default=4.0)
    ap.add_argument("--tokens", type=int, default=0,
                    help="with --profile and --prefill or --batch: tokens per call (default 2048 or 16)")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--sweep", action="store_true", help="average-bit sweep on a 14336x4096 layer (one JSON line)")
    ap.add_argument("--stack", action="store_true", help="32-layer linear stack tokens/s (one JSON line)")
    ap.add_argument("--stack-steps", type=int, default=256)
    ap.add_argument("--batch", action="store_true", help="batch 1..16 through the batched fused call (one JSON line)")
    ap.add_argument("--prefill", action="store_true", help="prefill path: dequant + GEMM on the linears (one JSON line)")
    ap.add_argument("--lut", action="store_true", help="nested look-up-table codes through grinqh_vmm_lut (one JSON line)")
    ap.add_argument("--cold", action="store_true", help="isolated cold select and VMM after an L2 flush (one JSON line)")
    ap.add_argument("--bmax", type=int, default=8, choices=(4, 6, 8),
                    help="stored code width; 4 or 6 grade into the classes {0, 2, ..., b_max}")
    ap.add_argument("--family", default="llama3", choices=("llama3", "qwen3"),
                    help="layer family of the main run: Llama3-8B (default) or Qwen3-8B shapes and distributions")
    args = ap.parse_args()
    global BMAX, CLASSES, WORKLOAD, FAMILY, TARGETS
    FAMILY = args.family
    if FAMILY == "qwen3":
        TARGETS = (4.0, 3.0)
        WORKLOAD = ("qwen3-8b decode linears (q,k,v,o,gate,up,down), batch 1, avg bits 4/3, row-std log-uniform "
                    "weights, student-t activations")
    from activation_graded_bit_b200 import workloads as wl
    BMAX = args.bmax
    CLASSES = tuple(wl.CLASSES) if BMAX == 8 else tuple(range(0, BMAX + 1, 2))
    if BMAX != 8:
        WORKLOAD = WORKLOAD + ", b_max %d codes, classes %s" % (BMAX, "/".join(map(str, CLASSES)))
    if args.warmup < 3:
        args.warmup = 3
    if args.profile:
        run_profile_case(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.stack:
        run_stack(args)
        return
    if args.batch:
        run_batch(args)
        return
    if args.prefill:
        run_prefill(args)
        return
    if args.lut:
        run_lut(args)
        return
    if args.cold:
        run_cold(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
