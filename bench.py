"""Benchmark of the streaming KV-cache attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload ID]

A step is one window step of the whole hot path over every layer of the
workload: one kv_stream_insert launch for all layers (fs_stream_insert_batch:
each layer's new frame of each view plus the text, evicting each view's oldest
frame and rotating the new keys once), then, per layer, stream_attn of the
step's queries against the layer's cache. Default workload: the
driving-shaped window (4 cameras x 4 frames x 180 tokens + 256 text tokens,
36 layers, H=32, Hkv=8, d=128), synthetic seeded inputs resident in HBM before
timing. The same run also times one layer of the wide window (7 cameras x 8
frames x 256 tokens + 512 text) for its stream_attn and insert roofline.

Prints ONE JSON line (rank 0). ``value`` is algorithmic attention TFLOP/s of the
whole job (4*d*H per visible query-key pair, summed over layers and ranks),
timed on the device with CUDA events between two barriers, max over ranks.
Under torchrun each rank runs its own replica of the workload (weak scaling,
no data-path collective).
"""
from __future__ import annotations

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

METRIC = "stream-attn TFLOP/s & µs/window-step (4 cams×4 frames); % of B200 BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0
KERNEL_SOURCES = ["streaming_kv_cache_stream_b200/csrc/stream_attn.cu",
                  "streaming_kv_cache_stream_b200/csrc/sm100.cuh",
                  "streaming_kv_cache_stream_b200/csrc/fs_internal.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "stream_attn_traffic.txt")


# ------------------------------------------------------------------ helpers

def visible_pairs_step(V, T, n, X):
    """Visible (query, key) pairs of one window step: view v's new-frame token i
    sees v*T*n + (T-1)*n + i + 1 keys, text token j sees V*T*n + j + 1."""
    frames = V * n * ((T - 1) * n + 1) + T * n * n * V * (V - 1) // 2 + V * n * (n - 1) // 2
    text = X * (V * T * n + 1) + X * (X - 1) // 2
    return frames + text


def step_flops(wl):
    return 4.0 * wl.d * wl.H * visible_pairs_step(wl.views, wl.frames, wl.tok_per_frame, wl.text_len)


def verify_flops(wl):
    """Algorithmic FLOPs of one drafted-block verify call: block token t sees the
    L window keys and block tokens 0..t."""
    return 4.0 * wl.d * wl.H * sum(wl.window_len + t + 1 for t in range(wl.verify_tokens))


def frame_flops(wl, heads=None):
    """Algorithmic FLOPs of one encoder-attention call over the newest frame of
    every view: each of a view's n tokens sees all n (QK^T and PV, 2 each per
    element), 4 d H n^2 per view."""
    from streaming_kv_cache_stream_b200.inputs import FRAME_HEADS

    h = heads or FRAME_HEADS
    return 4.0 * h["d"] * h["H"] * wl.views * wl.tok_per_frame ** 2


def insert_algorithmic_bytes(wl):
    """Bytes one layer's window-step insert must move: read the step's K and V
    (bf16) and write them into the ring, i.e. 2 tensors x (read + write) x
    N_new x Hkv x d x 2 bytes."""
    return 8.0 * wl.step_tokens * wl.Hkv * wl.d


def insert_implementation_bytes(wl):
    """Bytes kv_stream_insert moves for one layer's window step as built: the
    algorithmic bytes plus the rotated operands of the new rows (K hi, K lo,
    V as fp16), and, amortised over R = 16 steps, the re-base pass (read the
    kept rows' K and V, write the operands of every window row)."""
    new = wl.step_tokens * wl.Hkv * wl.d * (8 + 6)
    kept = wl.window_len - wl.step_tokens
    rebase = (kept * 4 + wl.window_len * 6) * wl.Hkv * wl.d
    return float(new + rebase / 16.0)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_id):
    """DRAM bytes per stream_attn launch from a committed ncu summary, if it was
    taken on the current kernel source and this workload; else None."""
    try:
        kv = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    kv[k.strip()] = v.strip()
        if kv.get("kernel_sha256_16") != kernel_hash() or kv.get("workload_id") != str(workload_id):
            return None
        return float(kv["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling; only samples taken inside the timed
    window (host wall-clock marks) are summarised."""

    QUERY = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu):
        self.gpu = gpu
        self.proc = None
        self.t0 = self.t1 = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(1.0)  # let nvidia-smi start sampling before the timed region
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.05)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        import datetime

        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            if self.t0 is None or not (self.t0 - 0.02 <= ts <= self.t1 + 0.02):
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["no samples inside the timed region"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


def gpu_id(dev):
    """nvidia-smi id of a torch device: its UUID when torch exposes it."""
    import torch

    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


def dist_setup(n_gpus, backend=None):
    """Rank, world and local rank from the torchrun environment; joins the
    process group when world > 1 (NCCL on GPUs; gloo when CUDA is absent, which
    the CPU tests use). Returns (world, rank, local)."""
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    backend = backend or ("nccl" if cuda else "gloo")
    if world > 1:
        import datetime

        import torch.distributed as dist

        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif cuda:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch

    if world > 1:
        import torch.distributed as dist

        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x, world):
    """The largest of every rank's x (every rank gets it): device times are
    reported as the slowest rank's."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank, ms, world):
    """Whole-job throughput of weak-scaling replicas: every rank did
    flops_per_rank in (at most) ms, the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


# ----------------------------------------------------------- CPU oracle leg

def blas_info():
    """(threads, "library version") of numpy's BLAS, from threadpoolctl."""
    try:
        from threadpoolctl import threadpool_info

        blas = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if blas:
            b = blas[0]
            return int(b.get("num_threads", 1)), f"{b.get('internal_api', '?')} {b.get('version', '?')}"
    except Exception:
        pass
    return os.cpu_count() or 1, "unknown"


def oracle_timing(wid, target_s=15.0, max_units=64):
    """Times the fp64 CPU oracle (as it stands) on window steps of this workload.

    Returns (seconds, algorithmic flops, layer-steps done, threads used)."""
    import numpy as np

    from oracle import StreamOracle, bf16_bits_to_f64
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS, window_inputs

    wl = WORKLOADS[wid]
    threads, _ = blas_info()
    fl = step_flops(wl)
    total_s, units, layer = 0.0, 0, 0
    while units < max_units and total_s < target_s:
        orc = StreamOracle(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d, wl.rope_base)
        pre = window_inputs(wid, layer % wl.layers, 0)
        orc.win.prefill(bf16_bits_to_f64(pre["K"]), bf16_bits_to_f64(pre["V"]))  # untimed setup
        inp = window_inputs(wid, layer % wl.layers, 1)
        f = {x: bf16_bits_to_f64(inp[x]) for x in ("Q", "K", "V")}
        t0 = time.perf_counter()
        orc.step(f["Q"], f["K"], f["V"])
        total_s += time.perf_counter() - t0
        units += 1
        layer += 1
    return total_s, fl * units, units, threads


# --------------------------------------------------------------- GPU leg

def l2_flusher(dev):
    """Reading a 256 MB buffer evicts the 126 MB L2 between timed launches. A
    read leaves clean lines behind (a write-based flush would leave 126 MB of
    dirty lines that the next kernel pays to write back)."""
    import torch

    buf = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        torch.sum(buf, dim=0, out=sink)
    return flush


def choose_peak(peaks, clocks):
    """The bf16 peak that applies to a kernel timed inside this run: the burst
    figure when the SM clock held its maximum with no power cap, else the
    sustained (power-capped) one."""
    burst = float(peaks.get("bf16_tflops"))
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    sm, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = "sw_power_cap" in (clocks.get("reasons") or [])
    if sm and mx and sm >= 0.95 * mx and not capped:
        return burst, "bf16_tflops (burst: SM clock at its maximum, no power cap during the timed region)"
    return sustained, "bf16_tflops_sustained (SM clock below maximum or power-capped during the timed region)"


def time_single_layer(wid, steps, warmup, dev):
    """One layer of a workload, window steps with L2 flushed before each: CUDA
    events around fs_stream_insert and around fs_stream_attend (one launch
    each). Returns per-launch microseconds (lists)."""
    import numpy as np
    import torch

    from streaming_kv_cache_stream_b200.abi import Stream
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS, window_inputs

    wl = WORKLOADS[wid]

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    s = Stream(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d, wl.rope_base)
    pre = window_inputs(wid, 0, 0)
    q = to_dev(pre["Q"])
    s.insert(to_dev(pre["K"]), to_dev(pre["V"]))
    s.attend(q, torch.empty(q.shape, dtype=torch.float32, device=dev))
    del q
    sets = 2
    inputs = [{x: to_dev(window_inputs(wid, 0, 1 + k)[x]) for x in ("Q", "K", "V")} for k in range(sets)]
    out = torch.empty((wl.step_tokens, wl.H, wl.d), dtype=torch.float32, device=dev)
    flush = l2_flusher(dev)
    stream = torch.cuda.current_stream()
    ins, att = [], []
    for k in range(warmup + steps):
        inp = inputs[k % sets]
        flush()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        s.insert(inp["K"], inp["V"])
        ev[1].record(stream)
        s.attend(inp["Q"], out)
        ev[2].record(stream)
        if k >= warmup:
            att.append(ev)
    torch.cuda.synchronize()
    s.sync()
    ins = [e[0].elapsed_time(e[1]) * 1e3 for e in att]
    att_us = [e[1].elapsed_time(e[2]) * 1e3 for e in att]
    s.close()
    del inputs, out
    torch.cuda.empty_cache()
    return ins, att_us


def time_frame_attention(wid, calls, dev):
    """fs_frame_attend on the newest frame of every view of a workload (encoder
    heads of inputs.FRAME_HEADS): CUDA events around replays of a graph of 10 calls.
    Returns (per-call microseconds, algorithmic FLOPs per call)."""
    import numpy as np
    import torch

    from streaming_kv_cache_stream_b200.abi import Stream
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS, frame_inputs

    wl = WORKLOADS[wid]

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    s = Stream(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d, wl.rope_base)
    b = {x: to_dev(v) for x, v in frame_inputs(wid, 0, 1).items()}
    out = torch.empty(b["Q"].shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(5):
        s.frame_attend(b["Q"], b["K"], b["V"], out)
    torch.cuda.synchronize()
    # Replayed from a CUDA graph of 10 calls (the encoder layer runs under CUDA
    # graphs in the pages' system; per-call Python dispatch would dominate).
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(10):
            s.frame_attend(b["Q"], b["K"], b["V"], out)
    graph.replay()
    torch.cuda.synchronize()
    ev = []
    for _ in range(calls):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        ev.append((e0, e1))
    torch.cuda.synchronize()
    del graph
    s.sync()
    s.close()
    us = [a.elapsed_time(c) * 1e3 / 10 for a, c in ev]
    return us, frame_flops(wl)


def time_kv_proj(wid, steps, warmup, dev):
    """fs_stream_insert_proj for every layer of a workload's window step, each
    layer with its own hidden states and weight (d_model = H*d), launched back
    to back as a model's step would: CUDA events around each step's calls.
    Returns (per-call microseconds per step, algorithmic FLOPs per call, bytes
    per call)."""
    import numpy as np
    import torch

    from streaming_kv_cache_stream_b200.abi import Stream
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS, hidden_inputs, proj_weight

    wl = WORKLOADS[wid]
    dm = wl.H * wl.d
    layers = wl.layers

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    hs = [Stream(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d, wl.rope_base)
          for _ in range(layers)]
    Ws = [to_dev(proj_weight(wid, l, dm)) for l in range(layers)]
    for l, s in enumerate(hs):
        s.insert_proj(to_dev(hidden_inputs(wid, l, 0, dm)), Ws[l])
    Xs = [to_dev(hidden_inputs(wid, l, 1, dm)) for l in range(layers)]
    stream = torch.cuda.current_stream()
    ev = []
    for k in range(warmup + steps):  # fewer steps than the re-base interval (16): no re-rotation pass
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for l, s in enumerate(hs):
            s.insert_proj(Xs[l], Ws[l])
        e1.record(stream)
        if k >= warmup:
            ev.append((e0, e1))
    torch.cuda.synchronize()
    for s in hs:
        s.sync()
        s.close()
    us = [a.elapsed_time(c) * 1e3 / layers for a, c in ev]
    N, outs = wl.step_tokens, 2 * wl.Hkv * wl.d
    flops = 2.0 * N * outs * dm
    nbytes = 2 * (N * dm + outs * dm + N * outs)  # X, W read; K, V written (bf16)
    del Xs, Ws
    torch.cuda.empty_cache()
    return us, flops, nbytes


def run_ours(args):
    import numpy as np
    import torch

    from streaming_kv_cache_stream_b200.abi import Stream, insert_batch, load
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS, window_inputs

    world, rank, local = dist_setup(args.gpus)
    load()
    wid = args.workload
    wl = WORKLOADS[wid]
    layers = wl.layers
    dev = torch.device("cuda", local if world > 1 else 0)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    streams = [Stream(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d, wl.rope_base)
               for _ in range(layers)]
    # prefill (the stream's first call), untimed
    for l, s in enumerate(streams):
        inp = window_inputs(wid, l, 0)
        q = to_dev(inp["Q"])
        out = torch.empty(q.shape, dtype=torch.float32, device=dev)
        s.insert(to_dev(inp["K"]), to_dev(inp["V"]))
        s.attend(q, out)
        del q, out
    torch.cuda.synchronize()
    # step inputs resident in HBM: `sets` distinct input sets per layer, cycled
    sets = 2
    inputs = [[{x: to_dev(window_inputs(wid, l, 1 + k)[x]) for x in ("Q", "K", "V")} for k in range(sets)]
              for l in range(layers)]
    nq = wl.step_tokens
    outs = [torch.empty((nq, wl.H, wl.d), dtype=torch.float32, device=dev) for _ in range(layers)]
    stream = torch.cuda.current_stream()

    def step(k, ev=None):
        # Events go around the step's one insert launch (all layers) and around
        # one layer's attention (layer k mod layers): every kernel is still
        # timed inside the timed region, while the other layers' attention
        # launches follow each other with nothing in between.
        sample = k % len(streams)
        cur = [inputs[l][k % sets] for l in range(layers)]
        if ev is not None:
            ev[0].record(stream)
        insert_batch(streams, [c["K"] for c in cur], [c["V"] for c in cur])
        if ev is not None:
            ev[1].record(stream)
        for l, s in enumerate(streams):
            timed = ev is not None and l == sample
            if timed:
                ev[2].record(stream)
            s.attend(cur[l]["Q"], outs[l])
            if timed:
                ev[3].record(stream)

    clk = ClockSampler(gpu_id(dev))
    clk.start()
    for k in range(args.warmup):
        step(k)
    torch.cuda.synchronize()
    launches0 = sum(s.info().launches for s in streams)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    clk.mark_start()
    start.record(stream)
    for k in range(args.steps):
        step(args.warmup + k, evs[k])
    end.record(stream)
    torch.cuda.synchronize()
    clk.mark_end()
    clk.stop()
    barrier(world)
    for s in streams:
        s.sync()  # raises on a device-side error flag (timeout, range)
    launches = sum(s.info().launches for s in streams) - launches0
    elapsed_ms = max_over_ranks(start.elapsed_time(end), world)
    ins_us = [evs[k][0].elapsed_time(evs[k][1]) * 1e3 for k in range(args.steps)]
    att_us = [evs[k][2].elapsed_time(evs[k][3]) * 1e3 for k in range(args.steps)]

    fl_layer = step_flops(wl)
    ms_per_step = elapsed_ms / args.steps
    value = job_tflops(fl_layer * layers, ms_per_step, world)
    att_mean, att_med = statistics.mean(att_us), statistics.median(att_us)
    att_tflops = fl_layer / (att_mean * 1e-6) / 1e12
    ins_mean, ins_med = statistics.mean(ins_us), statistics.median(ins_us)
    ins_alg = insert_algorithmic_bytes(wl) * layers
    ins_impl = insert_implementation_bytes(wl) * layers
    peaks, src = load_peaks()
    hbm = float(peaks.get("hbm_gbs"))
    clocks = clk.summary()
    peak_t, peak_why = choose_peak(peaks, clocks)

    # ---- one layer of the wide window (the largest-query config), same process
    wide = None
    if rank == 0 and not args.no_wide and wid != 4 and 4 in WORKLOADS:
        w4 = WORKLOADS[4]
        wi, wa = time_single_layer(4, steps=10, warmup=3, dev=dev)
        fl4 = step_flops(w4)
        b4 = insert_algorithmic_bytes(w4)
        wide = {
            "workload": f"{w4.name} window: {w4.views} cams x {w4.frames} frames x {w4.tok_per_frame} tok + "
                        f"{w4.text_len} text, 1 layer, H{w4.H}/Hkv{w4.Hkv}/d{w4.d}, 1% of K rows x8",
            "steps": len(wa), "l2": "flushed (256 MB write) before every step",
            "stream_attn_us_median": round(statistics.median(wa), 2),
            "stream_attn_us_mean": round(statistics.mean(wa), 2),
            "stream_attn_tflops": round(fl4 / (statistics.median(wa) * 1e-6) / 1e12, 2),
            "stream_attn_frac_of_burst": round(fl4 / (statistics.median(wa) * 1e-6) / 1e12
                                               / float(peaks.get("bf16_tflops")), 4),
            "stream_attn_frac_of_nominal_2250": round(fl4 / (statistics.median(wa) * 1e-6) / 1e12
                                                      / NOMINAL_BF16_TFLOPS, 4),
            "insert_us_median": round(statistics.median(wi), 2),
            "insert_algorithmic_bytes": b4,
            "insert_gbs": round(b4 / (statistics.median(wi) * 1e-6) / 1e9, 1),
            "insert_frac_of_measured_hbm": round(b4 / (statistics.median(wi) * 1e-6) / 1e9 / hbm, 4),
            "insert_frac_of_nominal_8000": round(b4 / (statistics.median(wi) * 1e-6) / 1e9 / 8000.0, 4),
        }

    # ---- the vision encoder's attention over the newest frames (same views and frame length)
    frame = None
    if rank == 0 and not args.no_wide:
        fu, ffl = time_frame_attention(wid, 20, dev)
        from streaming_kv_cache_stream_b200.inputs import FRAME_HEADS

        frame = {
            "kernel": "frame_attn",
            "shape": f"{wl.views} views x {wl.tok_per_frame} tokens, encoder heads H{FRAME_HEADS['H']}/"
                     f"Hkv{FRAME_HEADS['Hkv']}/d{FRAME_HEADS['d']}, bidirectional within each frame",
            "us_per_call_median": round(statistics.median(fu), 2),
            "algorithmic_mflop_per_call": round(ffl / 1e6, 2),
            "tflops": round(ffl / (statistics.median(fu) * 1e-6) / 1e12, 3),
            "l2": "inputs L2-resident (2 MB, as produced by the encoder's previous layer)",
        }

    # ---- the K/V projection fused with the ring insert (one layer's window step)
    proj = None
    if rank == 0 and not args.no_wide:
        pu, pfl, pb = time_kv_proj(wid, 8, 3, dev)
        pmed = statistics.median(pu)
        proj = {
            "kernel": "kv_proj",
            "bound": "tensor",
            "shape": f"X [{wl.step_tokens} x {wl.H * wl.d}] x W^T [{wl.H * wl.d} x {2 * wl.Hkv * wl.d}] bf16, "
                     "epilogue writes the ring slots (bf16) and the rotated fp16 operands",
            "us_per_call_median": round(pmed, 2),
            "us_per_call_mean": round(statistics.mean(pu), 2),
            "algorithmic_gflop_per_call": round(pfl / 1e9, 4),
            "tflops": round(pfl / (pmed * 1e-6) / 1e12, 2),
            "frac_of_burst": round(pfl / (pmed * 1e-6) / 1e12 / float(peaks.get("bf16_tflops")), 4),
            "hbm_floor_us": round(pb / (hbm * 1e3), 2),
            "l2": "every layer's own X and W (%d MiB per step): no reuse across calls" % (
                wl.layers * 2 * (wl.step_tokens + 2 * wl.Hkv * wl.d) * wl.H * wl.d // 2 ** 20),
            "timing": "CUDA events around the %d calls of a step (one per layer, back to back), per call" % wl.layers,
        }

    # ---- drafted-block verification against the medium window's cache (the
    # verify workload), replayed from a CUDA graph
    verify = None
    vid = 5
    if rank == 0 and not args.no_wide and vid in WORKLOADS:
        vs, vblocks = verify_stream(vid, dev)
        vus = time_verify_graph(vs, vblocks, 8, dev)
        vs.sync()
        vs.close()
        vwl = WORKLOADS[vid]
        vfl = verify_flops(vwl)
        verify = {
            "kernel": "verify_attn",
            "shape": f"{vwl.verify_tokens}-token drafted blocks after the text of the medium window "
                     f"(L = {vwl.window_len}, H{vwl.H}/Hkv{vwl.Hkv}/d{vwl.d})",
            "us_per_call_graph": round(vus, 2),
            "algorithmic_mflop_per_call": round(vfl / 1e6, 2),
            "tflops": round(vfl / (vus * 1e-6) / 1e12, 3),
            "timing": "CUDA events around 8 replays of a graph of 16 calls",
        }

    # ---- end to end through the public C ABI with host buffers
    e2e_steps = max(1, min(args.steps, 5))
    pin = [{x: torch.from_numpy(np.ascontiguousarray(window_inputs(wid, l, 1)[x]).view(np.int16)).pin_memory()
            for x in ("Q", "K", "V")} for l in range(layers)]
    pin_out = [torch.empty((nq, wl.H, wl.d), dtype=torch.float32).pin_memory() for _ in range(layers)]
    for l, s in enumerate(streams):  # first call sizes the staging buffers and copy streams, untimed
        s.step_host(pin[l]["K"], pin[l]["V"], pin[l]["Q"], pin_out[l])
    for s in streams:
        s.sync()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(e2e_steps):
        for l, s in enumerate(streams):
            s.step_host(pin[l]["K"], pin[l]["V"], pin[l]["Q"], pin_out[l])
    for s in streams:
        s.sync()  # the downloads run on the handles' copy streams
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    h2d = layers * (2 * wl.step_tokens * wl.Hkv * wl.d * 2 + nq * wl.H * wl.d * 2)
    d2h = layers * nq * wl.H * wl.d * 4

    result = None
    if rank == 0:
        traffic = recorded_traffic(wid)
        result = {
            "metric": METRIC,
            "value": round(value, 3),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 5),
            "us_per_window_step": round(ms_per_step * 1e3, 2),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f16",
            "precision": "bf16 inputs; rotated Q/K as fp16 hi+lo (3 MMAs), P and V fp16, fp32 accumulate, fp32 out; "
                         "supported input range |V|<=65504, |K|<=46318, checked on the device",
            "data": "synthetic",
            "config": {
                "workload": f"{wl.name} window: {wl.views} cams x {wl.frames} frames x {wl.tok_per_frame} tok "
                            f"+ {wl.text_len} text, {wl.layers} layers, H{wl.H}/Hkv{wl.Hkv}/d{wl.d}",
                "workload_id": wid,
                "layers": layers,
                "window_len": wl.window_len,
                "queries_per_step": nq,
                "algorithmic_gflop_per_layer_step": round(fl_layer / 1e9, 4),
                "l2": "inputs larger than L2: each step streams ~%.2f GB of per-layer inputs, caches and outputs"
                      % (layers * (wl.step_tokens * (2 * wl.Hkv + wl.H) * wl.d * 2 + nq * wl.H * wl.d * 4
                                   + 3 * wl.window_len * wl.Hkv * wl.d * 2) / 1e9),
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "kernel_timing": "CUDA events around the step's insert launch (all layers) and around one layer's "
                                 "attention per timed step (layer = step mod layers)",
            },
            "roofline": {
                "bound": "tensor",
                "kernel": "stream_attn",
                "achieved": round(att_tflops, 2),
                "peak": peak_t,
                "peak_source": f"{src} {peak_why}",
                "unit": "TFLOP/s",
                "frac": round(att_tflops / peak_t, 4),
                "frac_of_burst": round(att_tflops / float(peaks.get("bf16_tflops")), 4),
                "frac_of_sustained": round(att_tflops / float(peaks.get("bf16_tflops_sustained",
                                                                       peaks.get("bf16_tflops"))), 4),
                "frac_of_nominal_2250": round(att_tflops / NOMINAL_BF16_TFLOPS, 4),
                "traffic": traffic,
                "us_per_launch": round(att_mean, 2),
                "us_per_launch_median": round(att_med, 2),
                "algorithmic_gflop_per_launch": round(fl_layer / 1e9, 4),
            },
            "insert": {
                "kernel": "kv_stream_insert",
                "bound": "hbm",
                "layers_per_launch": layers,
                "us_per_launch": round(ins_mean, 2),
                "us_per_launch_median": round(ins_med, 2),
                "us_per_layer": round(ins_mean / layers, 3),
                "bytes_per_launch": ins_alg,
                "bytes_definition": "algorithmic: read the step's K and V and write them into the ring (bf16)",
                "achieved_gbs": round(ins_alg / (ins_mean * 1e-6) / 1e9, 1),
                "peak_gbs": hbm,
                "frac": round(ins_alg / (ins_mean * 1e-6) / 1e9 / hbm, 4),
                "frac_of_nominal_8000": round(ins_alg / (ins_mean * 1e-6) / 1e9 / 8000.0, 4),
                "traffic": ins_impl,
                "traffic_definition": "bytes the kernel moves as built: algorithmic + fp16 hi/lo/V operands of the "
                                      "new rows + the re-base pass amortised over 16 steps",
            },
            "wide_window": wide,
            "frame_encoder": frame,
            "kv_proj": proj,
            "verify_block": verify,
            "e2e": {
                "value": round(world * fl_layer * layers / (e2e_ms * 1e-3) / 1e12, 3),
                "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "api": "fs_stream_step_host per layer, pinned host buffers (uploads, kernels and downloads on "
                       "three streams)",
            },
            "gpu_launches": launches,
            "clocks": clocks,
        }
    for s in streams:
        s.close()
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    return result


def verify_stream(wid, dev):
    """A stream holding the verify workload's cache (the medium window after its
    steps) and device copies of a few drafted blocks."""
    import numpy as np
    import torch

    from streaming_kv_cache_stream_b200.abi import Stream
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS, verify_inputs, window_inputs

    wl = WORKLOADS[wid]

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    s = Stream(wl.views, wl.frames, wl.tok_per_frame, wl.text_len, wl.H, wl.Hkv, wl.d, wl.rope_base)
    for k in range(wl.steps + 1):  # the cache the drafted blocks are checked against
        inp = window_inputs(wid, 0, k)
        q = to_dev(inp["Q"])
        s.insert(to_dev(inp["K"]), to_dev(inp["V"]))
        s.attend(q, torch.empty(q.shape, dtype=torch.float32, device=dev))
    blocks = [{x: to_dev(verify_inputs(wid, c)[x]) for x in ("Q", "K", "V")} for c in range(4)]
    return s, blocks


def time_verify_graph(s, blocks, replays, dev, calls=16):
    """fs_stream_attend_ext calls replayed from a CUDA graph of `calls` calls (the
    pages run the decode loop under CUDA graphs): device microseconds per call."""
    import torch

    nx, H, d = blocks[0]["Q"].shape
    gouts = [torch.empty((nx, H, d), dtype=torch.float32, device=dev) for _ in range(2)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for c in range(calls):
            b = blocks[c % len(blocks)]
            s.attend_ext(b["Q"], b["K"], b["V"], gouts[c % 2])
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for _ in range(replays):
        graph.replay()
    g1.record(stream)
    torch.cuda.synchronize()
    del graph
    return g0.elapsed_time(g1) * 1e3 / (replays * calls)


def run_verify(args):
    """Drafted-block verify calls (workload 5): fs_stream_attend_ext of 8-token
    blocks against the medium window's cache after one step, inputs resident;
    a "step" is one verify call. The e2e leg copies each block from pinned host
    memory and the output back inside the timed region."""
    import numpy as np
    import torch

    from streaming_kv_cache_stream_b200.abi import load
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS, verify_inputs

    world, rank, local = dist_setup(args.gpus)
    load()
    wid = args.workload
    wl = WORKLOADS[wid]
    dev = torch.device("cuda", local if world > 1 else 0)

    s, blocks = verify_stream(wid, dev)
    sets = len(blocks)
    nx = wl.verify_tokens
    out = torch.empty((nx, wl.H, wl.d), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    clk = ClockSampler(gpu_id(dev))
    clk.start()
    for k in range(args.warmup):
        b = blocks[k % sets]
        s.attend_ext(b["Q"], b["K"], b["V"], out)
    torch.cuda.synchronize()
    launches0 = s.info().launches
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    clk.mark_start()
    start.record(stream)
    for k in range(args.steps):
        b = blocks[k % sets]
        s.attend_ext(b["Q"], b["K"], b["V"], out)
    end.record(stream)
    torch.cuda.synchronize()
    clk.mark_end()
    clk.stop()
    barrier(world)
    launches = s.info().launches - launches0
    ms = max_over_ranks(start.elapsed_time(end), world) / args.steps
    L = wl.window_len
    fl = verify_flops(wl)
    # end to end: pinned host block in, result out, inside the timed region
    pin = [{x: torch.from_numpy(np.ascontiguousarray(verify_inputs(wid, c)[x]).view(np.int16)).pin_memory()
            for x in ("Q", "K", "V")} for c in range(sets)]
    pin_out = torch.empty((nx, wl.H, wl.d), dtype=torch.float32).pin_memory()
    dq, dk, dv = (torch.empty_like(blocks[0][x]) for x in ("Q", "K", "V"))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, min(args.steps, 64))
    e0.record(stream)
    for k in range(n_e2e):
        hb = pin[k % sets]
        dq.copy_(hb["Q"], non_blocking=True)
        dk.copy_(hb["K"], non_blocking=True)
        dv.copy_(hb["V"], non_blocking=True)
        s.attend_ext(dq, dk, dv, out)
        pin_out.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / n_e2e
    # The same calls replayed from a CUDA graph: the device time per call
    # without host dispatch.
    graph_ms = max_over_ranks(time_verify_graph(s, blocks, max(1, args.steps // 16), dev) / 1e3, world)
    s.sync()
    s.close()
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    h2d = int(dq.numel() + dk.numel() + dv.numel()) * 2
    return {
        "metric": METRIC,
        "value": round(world * fl / (ms * 1e-3) / 1e12, 4),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms, 5),
        "us_per_verify_call": round(ms * 1e3, 2),
        "us_per_verify_call_graph": round(graph_ms * 1e3, 2),
        "tflops_graph": round(fl / (graph_ms * 1e-3) / 1e12, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16",
        "data": "synthetic",
        "config": {"workload": f"verify: {nx}-token drafted blocks after the text of the medium window "
                               f"(L = {L}, H{wl.H}/Hkv{wl.Hkv}/d{wl.d})", "workload_id": wid,
                   "algorithmic_mflop_per_call": round(fl / 1e6, 2),
                   "l2": "operands of one call fit in L2 (latency-bound shape)"},
        "e2e": {"value": round(world * fl / (e2e_ms * 1e-3) / 1e12, 4), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": int(out.numel()) * 4, "api": "Stream.attend_ext after pinned host copies"},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }


def run_reference(args):
    """The oracle arm: the fp64 CPU oracle, as it stands, on host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS

    wid = args.workload
    wl = WORKLOADS[wid]
    times = []
    flops = 0.0
    threads = 1
    units_total = 0
    # Bounded: the whole run stays within a few minutes (about 150 s of timed
    # oracle work however many steps are asked for).
    per_step_s = min(8.0, 150.0 / max(1, args.steps))
    for _ in range(min(args.warmup, 3)):
        oracle_timing(wid, target_s=0.0, max_units=1)
    for _ in range(args.steps):
        s, fl, units, threads = oracle_timing(wid, target_s=per_step_s, max_units=36)
        times.append(s)
        flops += fl
        units_total += units
    total = sum(times)
    value = flops / total / 1e12
    per_layer_ms = total / units_total * 1e3
    sample = (f"{units_total} layer-steps of the workload (one window step of one layer each: "
              f"{wl.step_tokens} queries x {wl.window_len} keys, all {wl.H} heads), fp64 numpy")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": per_layer_ms * wl.layers,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{wl.name} window, {wl.layers} layers", "workload_id": wid,
                   "note": "ms_per_step scales the per-layer time by the layer count"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample,
                         "blas": blas_info()[1]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-wide", action="store_true", help="skip the one-layer wide-window timing")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        res = run_reference(args)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    from streaming_kv_cache_stream_b200.inputs import WORKLOADS as _W

    if _W[args.workload].verify_calls:
        res = run_verify(args)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    res = run_ours(args)
    if res is not None:
        if res["n_gpus"] == 1 and not args.no_cpu_baseline:
            s, fl, units, threads = oracle_timing(args.workload, target_s=15.0, max_units=36)
            from streaming_kv_cache_stream_b200.inputs import WORKLOADS

            wl = WORKLOADS[args.workload]
            res["cpu_baseline"] = {
                "value": round(fl / s / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                "blas": blas_info()[1],
                "sample": f"{units} layer-steps ({wl.step_tokens} queries x {wl.window_len} keys, {wl.H} heads each), "
                          f"{s:.1f} s of fp64 numpy",
            }
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
