"""Benchmark: fused row normalization on B200, one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole hot path over the large bf16 workloads:
  dual q/k head RMSNorm   q [8192, 32, 128] + k [8192, 8, 128]  (one launch)
  RMSNorm                 [16, 4096, 4096]
  LayerNorm               [65536, D] for D in 768, 1000, 4097, 8192, 16384
i.e. 7 launches, 720,896 normalized rows and ~9.2 GB of algorithmic HBM
traffic per step. Inputs live in HBM before timing starts (seeded, drawn on
the device). Every step reads ~4.6 GB, far more than the 126 MB L2, so no
L2 flush is needed between steps. The device time of K steps is taken with
CUDA events on the launching stream, bracketed by a barrier and a
synchronize, and the maximum over ranks is reported.

Multi-GPU (torchrun): each rank normalizes its own copy of the workload (weak
scaling; rows are independent, so there is no data-path collective); the
only collective is the max-over-ranks of the timings.

--impl reference runs the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workloads per step (rank 0 only).
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from transformer_row_normalization_b200 import workloads as wl  # noqa: E402

METRIC = "normalized rows/sec and achieved HBM GB/s as % of B200 peak, 1 GPU"
FALLBACK_HBM_GBS = 6650.0
CSRC = os.path.join(ROOT, "transformer_row_normalization_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------------------
# distributed plumbing (host logic; covered by tests on gloo)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(value, dist, device):
    """The maximum of a float over all ranks (the value itself at N=1)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_seed(seed, rank):
    """Each rank draws its own inputs (same recipe, different seed)."""
    return seed + 1000 * rank


# ---------------------------------------------------------------------------
# measured peaks, clocks, profile bookkeeping


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def source_digest():
    """Digest of the sources the kernels are built from: the CUDA sources
    and the C-ABI header."""
    h = hashlib.sha256()
    for d in (CSRC, INCLUDE):
        for name in sorted(os.listdir(d)):
            if name.endswith((".cu", ".cuh", ".h")):
                with open(os.path.join(d, name), "rb") as f:
                    h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name):
    """DRAM bytes per launch from an ncu capture recorded in
    profiles/ncu_traffic.json, if that capture was taken of the current
    kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(workload_name)
    if not e or e.get("source_digest") != source_digest():
        return None
    return e.get("traffic_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed
    region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.target = None
        try:
            p = torch.cuda.get_device_properties(device)
            self.target = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            self.target = str(device.index or 0)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", self.target],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return self.parse(out)

    @staticmethod
    def parse(text):
        """Median SM clock, max clock, peak power and the throttle reasons
        seen in nvidia-smi CSV samples of FIELDS."""
        rows = [[c.strip() for c in l.split(",")] for l in text.strip().splitlines()
                if l.count(",") >= 7]
        rows = [r for r in rows if r[0].replace(".", "", 1).isdigit()]
        if not rows:
            return None
        sm = [float(r[0]) for r in rows]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[4:8]) if v == "Active"})
        power = [float(r[2]) for r in rows if r[2].replace(".", "", 1).isdigit()]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][1]),
                "power_w_max": max(power) if power else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# the step


class Step:
    """Workloads (by default the large bf16 suite) on one device, with outputs
    preallocated."""

    def __init__(self, device, rank, names=wl.LARGE_SUITE):
        import transformer_row_normalization_b200 as rn
        self.rn = rn
        self.device = device
        self.items = []
        for name in names:
            w = wl.WORKLOADS[name]
            rw = wl.Workload(w.name, w.op, w.dtype, w.shape, w.eps, rank_seed(w.seed, rank),
                             k_shape=w.k_shape)
            a = wl.make_inputs(rw, device=device)
            if w.op == "dual":
                out = (torch.empty_like(a["q"]), torch.empty_like(a["k"]))
            else:
                out = (torch.empty_like(a["x"]),)
            self.items.append((w, a, out))
        torch.cuda.synchronize(device)

    @property
    def rows(self):
        return sum(w.total_rows for w, _, _ in self.items)

    @property
    def bytes(self):
        return sum(w.algorithmic_bytes() for w, _, _ in self.items)

    def launch(self, i, stream=None):
        w, a, out = self.items[i]
        rn = self.rn
        if w.op == "dual":
            rn.dual_head_rms_norm(a["q"], a["k"], a["wq"], a["wk"], w.eps, out_q=out[0],
                                  out_k=out[1], stream=stream)
        elif w.op == "rms":
            rn.rms_norm(a["x"], a["w"], w.eps, out=out[0], stream=stream)
        else:
            rn.layer_norm(a["x"], a["w"], a["b"], w.eps, out=out[0], stream=stream)

    def run(self, stream=None):
        for i in range(len(self.items)):
            self.launch(i, stream)


def time_steps(step, k, stream):
    """Device time of k steps (ms) and per-launch times (ms, per workload,
    averaged), all from CUDA events on `stream`."""
    n = len(step.items)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(k)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for s in range(k):
            ev[s][0].record(stream)
            for i in range(n):
                step.launch(i, stream)
                ev[s][i + 1].record(stream)
        end.record(stream)
    end.synchronize()
    total = start.elapsed_time(end)
    per = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(k)) / k for i in range(n)]
    return total, per


def chunk_views(w, a, out, chunks):
    """Row chunks of one workload: per chunk, (device input views, device
    output views) as [rows, dim] slices; the dual workload is cut by tokens
    (its q and k rows together)."""
    if w.op == "dual":
        q, k = a["q"], a["k"]
        tokens = q.shape[0]
        step = -(-tokens // chunks)
        res = []
        for t0 in range(0, tokens, step):
            t1 = min(tokens, t0 + step)
            res.append(((q[t0:t1], k[t0:t1]), (out[0][t0:t1], out[1][t0:t1])))
        return res
    x = a["x"].reshape(-1, w.dim)
    y = out[0].reshape(-1, w.dim)
    step = -(-x.shape[0] // chunks)
    return [((x[r0:r0 + step],), (y[r0:r0 + step],)) for r0 in range(0, x.shape[0], step)]


def launch_chunk(rn, w, a, ins, outs, stream):
    """The public call of workload w on one chunk of its rows."""
    if w.op == "dual":
        rn.dual_head_rms_norm(ins[0], ins[1], a["wq"], a["wk"], w.eps, out_q=outs[0],
                              out_k=outs[1], stream=stream)
    elif w.op == "rms":
        rn.rms_norm(ins[0], a["w"], w.eps, out=outs[0], stream=stream)
    else:
        rn.layer_norm(ins[0], a["w"], a["b"], w.eps, out=outs[0], stream=stream)


def time_e2e(step, k, stream, chunks=8):
    """Through the public API with HOST buffers: every step copies each
    workload's inputs from pinned host memory to the device, normalizes, and
    copies the outputs back to pinned host memory. Each workload runs in
    `chunks` row chunks pipelined over three streams (host-to-device copies,
    kernels, device-to-host copies), so both PCIe directions and the kernels
    overlap; a chunk's kernel waits for its inputs, its read-back for its
    kernel, and its next upload for the previous step's kernel on it (the
    next kernel likewise waits for the previous read-back)."""
    dev = step.device
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    host_in, host_out = [], []
    h2d = d2h = 0
    for w, a, out in step.items:
        hi = {key: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for key, t in a.items()}
        for key, t in a.items():
            hi[key].copy_(t)
        ho = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in out]
        host_in.append(hi)
        host_out.append(ho)
        h2d += sum(t.numel() * t.element_size() for t in a.values())
        d2h += sum(t.numel() * t.element_size() for t in out)
    # (device views, host views) of every chunk of every workload
    plan = []
    for i, (w, a, out) in enumerate(step.items):
        ho = [t for t in host_out[i]]
        hi = {key: t for key, t in host_in[i].items()}
        dev_chunks = chunk_views(w, a, out, chunks)
        host_chunks = chunk_views(w, hi, ho, chunks)
        vec = [key for key in a if key in ("w", "b", "wq", "wk")]
        plan.append((w, a, [(d, h) for d, h in zip(dev_chunks, host_chunks)], vec, i))
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    last_kernel, last_read = {}, {}
    start.record(stream)
    up.wait_stream(stream)
    down.wait_stream(stream)
    for _ in range(k):
        for w, a, chunk_list, vec, i in plan:
            for c, ((d_in, d_out), (h_in, h_out)) in enumerate(chunk_list):
                key = (i, c)
                with torch.cuda.stream(up):
                    if key in last_kernel:
                        up.wait_event(last_kernel[key])
                    if c == 0:
                        for name in vec:
                            a[name].copy_(host_in[i][name], non_blocking=True)
                    for dst, src in zip(d_in, h_in):
                        dst.copy_(src, non_blocking=True)
                    loaded = torch.cuda.Event()
                    loaded.record(up)
                stream.wait_event(loaded)
                if key in last_read:
                    stream.wait_event(last_read[key])
                launch_chunk(step.rn, w, a, d_in, d_out, stream)
                done = torch.cuda.Event()
                done.record(stream)
                last_kernel[key] = done
                with torch.cuda.stream(down):
                    down.wait_event(done)
                    for dst, src in zip(h_out, d_out):
                        dst.copy_(src, non_blocking=True)
                    read = torch.cuda.Event()
                    read.record(down)
                last_read[key] = read
    stream.wait_stream(down)
    stream.wait_stream(up)
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end), h2d, d2h


def cpu_baseline(step, chunk_rows=2048, single_share=16):
    """The fp64 oracle on the host cores over every row of one step (copied
    from the device in chunks of `chunk_rows` rows; only the oracle calls are
    timed), and on one thread over the first 1/`single_share` of each
    workload's rows (the step's row mix, a bounded sample)."""
    import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    # warm-up (page faults, thread pool) on a few rows
    w0, a0, _ = step.items[1]
    oracle.rms_norm(a0["x"].reshape(-1, w0.dim)[:64].cpu(), a0["w"].cpu(), w0.eps, nthreads=cores)

    def parts_of(w, a):
        if w.op == "dual":
            return ([(a["q"].reshape(-1, w.dim), a["wq"]),
                     (a["k"].reshape(-1, w.k_shape[-1]), a["wk"])], None)
        return [(a["x"].reshape(-1, w.dim), a["w"])], (a["b"].cpu() if "b" in a else None)

    def run(w, xc, wt, bias, n):
        t0 = time.perf_counter()
        if w.op == "ln":
            oracle.layer_norm(xc, wt, bias, w.eps, nthreads=n)
        else:
            oracle.rms_norm(xc, wt, w.eps, nthreads=n)
        return time.perf_counter() - t0

    busy = busy1 = 0.0
    rows = rows1 = 0
    for w, a, _ in step.items:
        parts, bias = parts_of(w, a)
        for x, wt in parts:
            wt = wt.cpu()
            for r0 in range(0, x.shape[0], chunk_rows):
                xc = x[r0:r0 + chunk_rows].cpu()
                busy += run(w, xc, wt, bias, cores)
                rows += xc.shape[0]
            xc = x[:max(1, x.shape[0] // single_share)].cpu()
            busy1 += run(w, xc, wt, bias, 1)
            rows1 += xc.shape[0]
    return {"value": round(rows / busy, 1), "unit": "rows/s", "cores": cores, "kind": "oracle",
            "sample": f"one full step ({rows} rows, every workload), fp64, {cores} threads, "
                      f"{busy:.1f} s of oracle time",
            "single_thread": {"value": round(rows1 / busy1, 1), "unit": "rows/s", "cores": 1,
                              "sample": f"the first 1/{single_share} of each workload's rows "
                                        f"({rows1} rows), fp64, 1 thread, {busy1:.1f} s"}}


def time_fused(device, rank, dist, peak, reps=30, oracle_rows=2048):
    """The extensions (residual-add RMSNorm, gated RMSNorm, dual head RMSNorm +
    RoPE, rows streamed past the register kernels' width), measured beside the
    step: the median CUDA-event time of single launches on the
    launching stream, each after a 256 MB read that evicts L2 (max over
    ranks), and on rank 0 the fp64 oracle's rows/s on the first
    `oracle_rows` rows on all host cores."""
    import transformer_row_normalization_b200 as rn
    evict = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    out = []
    for name in wl.FUSED_SUITE:
        w = wl.WORKLOADS[name]
        rw = wl.Workload(w.name, w.op, w.dtype, w.shape, w.eps, rank_seed(w.seed, rank),
                         k_shape=w.k_shape, meta=w.meta)
        a = wl.make_inputs(rw, device=device)
        if w.op in ("rms", "ln"):
            y = torch.empty_like(a["x"])

            def launch():
                if w.op == "ln":
                    rn.layer_norm(a["x"], a["w"], a["b"], w.eps, out=y)
                else:
                    rn.rms_norm(a["x"], a["w"], w.eps, out=y)
        elif w.op == "dual_rope":
            table = rn.rope_table(w.meta["rope_dims"], w.shape[0], base=w.meta["rope_base"],
                                  device=device)
            yq, yk = torch.empty_like(a["q"]), torch.empty_like(a["k"])

            def launch():
                rn.dual_head_rms_norm_rope(a["q"], a["k"], a["wq"], a["wk"], w.eps, table, 0,
                                           w.meta["rope_dims"], out_q=yq, out_k=yk)
        else:
            second = a["r"] if w.op == "add_rms" else a["z"]
            y, h = torch.empty_like(a["x"]), torch.empty_like(a["x"])

            def launch():
                if w.op == "add_rms":
                    rn.add_rms_norm(a["x"], second, a["w"], w.eps, out=y, out_h=h)
                else:
                    rn.gated_rms_norm(a["x"], second, a["w"], w.eps, out=y)

        for _ in range(3):
            launch()
        # all reps queued before any is read back: the host stays ahead of the
        # GPU (each eviction read takes ~40 us), so no launch waits on the host
        # inside its event pair
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for s, e in ev:
            evict.sum()
            s.record()
            launch()
            e.record()
        torch.cuda.synchronize(device)
        times = [s.elapsed_time(e) for s, e in ev]
        t = max_over_ranks(sorted(times)[len(times) // 2], dist, device)
        g = w.algorithmic_bytes() / (t * 1e-3) / 1e9
        item = {"workload": name, "us": round(t * 1e3, 2),
                "rows_per_s": round(w.total_rows / (t * 1e-3)), "gbs": round(g, 1),
                "frac": round(g / peak, 4), "algorithmic_bytes": w.algorithmic_bytes()}
        if rank == 0:
            import oracle
            if w.op in ("rms", "ln"):
                nr = max(1, oracle_rows // 256)  # 65536-wide rows: a few MB of oracle work
                xs = a["x"].reshape(-1, w.dim)[:nr].cpu()
                args = ((xs, a["w"].cpu(), a["b"].cpu(), w.eps) if w.op == "ln"
                        else (xs, a["w"].cpu(), w.eps))
                fn = oracle.layer_norm if w.op == "ln" else oracle.rms_norm
                nrows = nr
            elif w.op == "dual_rope":
                # whole tokens: oracle_rows // 40 tokens of 32 query + 8 key heads
                nt = max(1, oracle_rows // 40)
                args = (a["q"].reshape(-1, w.dim)[:nt * 32].cpu(),
                        a["k"].reshape(-1, w.dim)[:nt * 8].cpu(), a["wq"].cpu(), a["wk"].cpu(),
                        w.eps, 32, 8, 0, w.meta["rope_dims"])
                fn, nrows = oracle.dual_head_rms_norm_rope, nt * 40
            else:
                x = a["x"].reshape(-1, w.dim)[:oracle_rows].cpu()
                x2 = second.reshape(-1, w.dim)[:oracle_rows].cpu()
                args = (x, x2, a["w"].cpu(), w.eps)
                fn = oracle.add_rms_norm if w.op == "add_rms" else oracle.gated_rms_norm
                nrows = x.shape[0]
            fn(*args, nthreads=cores)  # warm-up
            t0 = time.perf_counter()
            fn(*args, nthreads=cores)
            busy = time.perf_counter() - t0
            item["oracle_rows_per_s"] = round(nrows / busy, 1)
        out.append(item)
    return {"workloads": out, "cores": cores,
            "timing": f"median of {reps} single launches (queued back to back), each after "
                      "a 256 MB read that evicts L2; oracle on the first "
                      f"{oracle_rows} rows, fp64, {cores} threads"}


def time_configs(step, small, device, dist, peak, reps=30, burst=100):
    """Every config alone, cold and warm: min and median of `reps` CUDA-event
    timings on the launching stream after 3 warm-up launches. Cold: each rep
    follows a 256 MB read (over twice the 126 MB L2), which evicts the
    config's data and leaves L2 clean; a flush by writing would leave ~126 MB
    of dirty lines for the timed launch to write back. Warm: no flush; each
    rep times one launch of a large config right after another, or one replay
    of a CUDA graph of `burst` launches of a small one (per-launch time =
    total / burst; eager Python launches of a few-microsecond kernel would
    time the host). Large configs carry a roofline fraction (cold median); the
    small ones fit in L2 and are launch-bound, so they carry none. Max over
    ranks."""
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    out = []
    for st, large in ((step, True), (small, False)):
        for i, (w, _, _) in enumerate(st.items):
            for _ in range(3):
                st.launch(i)
            n = 1 if large else burst
            graph = None
            if not large:
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph):
                    for _ in range(n):
                        st.launch(i)
                graph.replay()
            cold = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(reps)]
            for a, b in cold:
                flush.sum()
                a.record(stream)
                st.launch(i)
                b.record(stream)
            warm = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(reps)]
            for a, b in warm:
                a.record(stream)
                if graph is not None:
                    graph.replay()
                else:
                    st.launch(i)
                b.record(stream)
            torch.cuda.synchronize(device)
            del graph
            tc = sorted(a.elapsed_time(b) * 1e3 for a, b in cold)
            tw = sorted(a.elapsed_time(b) * 1e3 / n for a, b in warm)
            tc = [max_over_ranks(t, dist, device) for t in (tc[0], tc[len(tc) // 2])]
            tw = [max_over_ranks(t, dist, device) for t in (tw[0], tw[len(tw) // 2])]
            item = {"workload": w.name, "us_cold_min": round(tc[0], 2),
                    "us_cold_median": round(tc[1], 2), "us_warm_min": round(tw[0], 2),
                    "us_warm_median": round(tw[1], 2),
                    "rows_per_s_cold": round(w.total_rows / (tc[1] * 1e-6)),
                    "rows_per_s_warm": round(w.total_rows / (tw[1] * 1e-6))}
            if large:
                g = w.algorithmic_bytes() / (tc[1] * 1e-6) / 1e9
                item["gbs_cold"] = round(g, 1)
                item["frac_cold"] = round(g / peak, 4)
            out.append(item)
    return {"items": out,
            "timing": f"min and median of {reps} reps after 3 warm-up launches; cold: each "
                      "rep after a 256 MB read that evicts L2; warm: no flush, small configs "
                      f"timed as one replay of a CUDA graph of {burst} launches"}


# ---------------------------------------------------------------------------


def config_dict(rows, nbytes, world, path=0):
    return {
        "workload": "large bf16 suite: dual q/k head RMSNorm q[8192,32,128]+k[8192,8,128] "
                    "(1 launch); RMSNorm [16,4096,4096] with 1% x50 outliers; LayerNorm "
                    "[65536,D] D in {768,1000,4097,8192,16384} with constant rows",
        "rows_per_step": rows,
        "algorithmic_bytes_per_step": nbytes,
        "launches_per_step": 7,
        "l2": "no flush: each step reads ~4.6 GB and writes ~4.6 GB (126 MB L2)",
        "parallelism": f"dp{world} (weak: each rank its own copy of the suite)",
        "kernel_path": path,
    }


def run_ours(args):
    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    peak, peak_kind = measured_peak()
    step = Step(device, rank)
    step.rn.set_path_override(args.path)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step.run(stream)
    stream.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize(device)
    clocks = ClockSampler(device) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.2)
    total_ms, per_ms = time_steps(step, args.steps, stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop() if clocks else None
    barrier(dist, device)
    total_ms = max_over_ranks(total_ms, dist, device)
    per_ms = [max_over_ranks(t, dist, device) for t in per_ms]

    rows = step.rows
    nbytes = step.bytes
    seconds = total_ms / 1e3
    value = world * rows * args.steps / seconds
    gbs = nbytes * args.steps / seconds / 1e9

    per_config = []
    for (w, _, _), t in zip(step.items, per_ms):
        g = w.algorithmic_bytes() / (t * 1e-3) / 1e9
        per_config.append({"workload": w.name, "us": round(t * 1e3, 2),
                           "rows_per_s": round(w.total_rows / (t * 1e-3)),
                           "gbs": round(g, 1), "frac": round(g / peak, 4)})
    dom = max(range(len(per_ms)), key=lambda i: per_ms[i])
    dw = step.items[dom][0]
    achieved = dw.algorithmic_bytes() / (per_ms[dom] * 1e-3) / 1e9
    traffic = recorded_traffic(dw.name)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "kernel_workload": dw.name, "peak_source": peak_kind,
                "algorithmic_bytes_per_launch": dw.algorithmic_bytes(),
                "us_per_launch": round(per_ms[dom] * 1e3, 2),
                "frac_is": "in-step average: CUDA events between the kernel's back-to-back "
                           "launches inside the timed region, averaged over its launches",
                "sm_mhz": clk["sm_mhz"] if clk else None}

    e2e_steps = max(1, min(3, args.steps))
    e2e_ms, h2d, d2h = time_e2e(step, e2e_steps, stream)
    e2e_ms = max_over_ranks(e2e_ms, dist, device)
    e2e = {"value": world * rows * e2e_steps / (e2e_ms / 1e3), "unit": "rows/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "pipeline": "8 row chunks per workload over three streams: uploads, kernels, "
                       "read-backs"}

    fused = time_fused(device, rank, dist, peak)
    configs = time_configs(step, Step(device, rank, wl.SMALL_SUITE), device, dist, peak)
    base = cpu_baseline(step) if (rank == 0 and world == 1) else None
    # the same kernel timed alone, cold (after an L2-evicting read), beside the
    # in-step figure that `frac` uses
    for item in configs["items"]:
        if item["workload"] == dw.name:
            roofline["cold_median_us"] = item["us_cold_median"]
            roofline["frac_cold"] = item.get("frac_cold")
    if dist is not None:
        barrier(dist, device)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "rows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded on the device with the workloads' shapes and distributions",
            "config": config_dict(rows, nbytes, world, args.path),
            "hbm": {"gbs": round(gbs, 1), "peak_gbs": peak, "frac": round(gbs / peak, 4),
                    "peak_source": peak_kind},
            "roofline": roofline, "cpu_baseline": base, "e2e": e2e,
            "gpu_launches": 7 * args.steps, "clocks": clk, "per_config": per_config,
            "configs": configs, "fused": fused,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_reference(args):
    """The fp64 oracle on the host cores, each step a bounded sample of the
    workloads (rows_per_workload rows of each)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    samples = []
    per_wl = max(4, min(64, 6000 // max(1, args.steps + args.warmup)))
    for name in wl.LARGE_SUITE:
        w = wl.WORKLOADS[name]
        if w.op == "dual":
            sw = wl.Workload(w.name, w.op, w.dtype, (per_wl, 32, 128), w.eps, w.seed,
                             k_shape=(per_wl, 8, 128))
        else:
            sw = wl.Workload(w.name, w.op, w.dtype, (per_wl * 4, w.dim), w.eps, w.seed)
        samples.append((sw, wl.make_inputs(sw)))

    def one_step():
        n = 0
        for sw, a in samples:
            if sw.op == "dual":
                oracle.dual_head_rms_norm(a["q"].reshape(-1, 128), a["k"].reshape(-1, 128),
                                          a["wq"], a["wk"], sw.eps, nthreads=cores)
            elif sw.op == "rms":
                oracle.rms_norm(a["x"], a["w"], sw.eps, nthreads=cores)
            else:
                oracle.layer_norm(a["x"], a["w"], a["b"], sw.eps, nthreads=cores)
            n += sw.total_rows
        return n

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    rows = 0
    for _ in range(args.steps):
        rows += one_step()
    dt = time.perf_counter() - t0
    value = rows / dt
    sample = (f"per step {rows // args.steps} rows: {per_wl * 40} dual head rows and "
              f"{per_wl * 4} rows of each other workload, fp64, {cores} threads")
    full_rows = sum(wl.WORKLOADS[n].total_rows for n in wl.LARGE_SUITE)
    full_bytes = sum(wl.WORKLOADS[n].algorithmic_bytes() for n in wl.LARGE_SUITE)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": "rows/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded on the host with the workloads' shapes and distributions",
        "config": config_dict(full_rows, full_bytes, world),
        "cpu_baseline": {"value": round(value, 1), "unit": "rows/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 1), "unit": "rows/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """One workload, launched --steps times after --warmup launches, for
    profiler captures: OP:DTYPE:ROWS:DIM with OP one of rms, ln, add_rms,
    gated_rms, dual, dual_rope (for the dual ops ROWS counts tokens of 32
    query and 8 key heads of DIM columns; RoPE rotates all DIM columns,
    split-half, base 10000, positions 0..ROWS-1). Prints the median
    CUDA-event time per launch (each launch after a 256 MB read that evicts
    L2) on stderr; this is not the benchmark line."""
    import transformer_row_normalization_b200 as rn
    op, dt, rows, dim = args.profile_case.split(":")
    dtype = torch.bfloat16 if dt == "bf16" else torch.float32
    rows, dim = int(rows), int(dim)
    device = torch.device("cuda", 0)
    rn.set_path_override(args.path)
    if op in ("dual", "dual_rope"):
        q = wl.random_rows(rows * 32, dim, dtype, seed=1, device=device)
        k = wl.random_rows(rows * 8, dim, dtype, seed=2, device=device)
        wq = wl.random_vector(dim, dtype, seed=3, device=device)
        wk = wl.random_vector(dim, dtype, seed=4, device=device)
        yq, yk = torch.empty_like(q), torch.empty_like(k)
        table = rn.rope_table(dim, rows, device=device) if op == "dual_rope" else None
        plan = rn.plan(rn.RN_OP_DUAL, q, weight=wq, bias=wk, k=k)

        def launch():
            if op == "dual":
                rn.dual_head_rms_norm(q, k, wq, wk, 1e-6, out_q=yq, out_k=yk)
            else:
                rn.dual_head_rms_norm_rope(q, k, wq, wk, 1e-6, table, 0, dim, heads_q=32,
                                           heads_k=8, out_q=yq, out_k=yk)
    else:
        x = wl.random_rows(rows, dim, dtype, seed=1, device=device, mean=0.5, std=2.0)
        w = wl.random_vector(dim, dtype, seed=2, device=device)
        b = wl.random_vector(dim, dtype, seed=3, device=device, mean=0.0, std=0.1)
        x2 = wl.random_rows(rows, dim, dtype, seed=4, device=device)
        y, h = torch.empty_like(x), torch.empty_like(x)
        plan = rn.plan(rn.RN_OP_LN if op == "ln" else rn.RN_OP_RMS, x, weight=w,
                       bias=b if op == "ln" else None)

        def launch():
            if op == "rms":
                rn.rms_norm(x, w, 1e-5, out=y)
            elif op == "ln":
                rn.layer_norm(x, w, b, 1e-5, out=y)
            elif op == "add_rms":
                rn.add_rms_norm(x, x2, w, 1e-5, out=y, out_h=h)
            else:
                rn.gated_rms_norm(x, x2, w, 1e-5, out=y)
    evict = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
    times = []
    for i in range(args.warmup + args.steps):
        evict.sum()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        launch()
        e.record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            times.append(s.elapsed_time(e) * 1e3)
    log(f"{args.profile_case} path={args.path} median {sorted(times)[len(times) // 2]:.1f} us "
        f"plan={plan} timeouts={rn.device_error_count()}")


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--profile-case", default=None,
                    help="OP:DTYPE:ROWS:DIM -- launch one workload for a profiler capture")
    ap.add_argument("--path", type=int, default=0,
                    help="kernel choice: 0 automatic, 1 register, 2 per-warp bulk-copy rings, "
                         "3 register with prefetch of the rows ahead")
    args = ap.parse_args(argv)
    if args.profile_case:
        return run_profile_case(args)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, _, _ = dist_env()
    if world != args.gpus and world > 1:
        log(f"note: WORLD_SIZE={world} but --gpus {args.gpus}")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
