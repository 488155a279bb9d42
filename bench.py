"""Benchmark of the routed-expert MoE layer over 4-bit codebook weights.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_t1|decode_t8|decode_t64|prefill_t2048|prefill_t8192]

One step = one pass of the whole layer (route -> gate/up + SwiGLU -> down ->
combine) over one batch of synthetic GLM-5.2-shaped input (hidden 6144,
intermediate 2048, 256 experts, top-8; 4-bit Lloyd codebook + E8M0/32
weights).  The default workload is decode at T=1.  Inputs rotate over 8
seeded batches resident in HBM.  The timed K steps run back to back between
one pair of CUDA events with no L2 flush: each step's expert weights exceed
L2 (8 experts x 20 MB at T=1; all 256 experts at prefill sizes) and
consecutive steps route to different experts.  The same steps are also timed
one at a time with L2 flushed before each, outside the step's own events (a
256 MiB write, then a 256 MiB read of a second buffer), reported as
"flushed".  Prints one JSON line (rank 0).

--impl reference times the fp64 CPU oracle on the host cores on the same
workload, each step a bounded sample (one expert's contribution for one
token, over a slice of the intermediate channels, on every thread).

N > 1: independent replicas, one per GPU (the layer is single-GPU); the
device time is the max over ranks; value = tokens of all ranks / that time.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from bit_codebook_quantized_router_b200 import inputs  # noqa: E402

METRIC = "MoE layer tokens/s"
UNIT = "tokens/s"
FLUSH_BYTES = 256 << 20
ROTATE = 8
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def workload_desc(w: inputs.Workload) -> dict:
    sh = w.shape
    kind = "GLM-5.2-shaped" if sh == inputs.GLM else "small"
    d = {"workload": f"{w.name}: {kind} routed-expert MoE layer, T={w.T}, H={sh.H}, I={sh.I}, "
                     f"E={sh.E}, top-{sh.k}, 4-bit Lloyd-codebook codes + E8M0 scale per 32",
         "T": w.T, "H": sh.H, "I": sh.I, "E": sh.E, "top_k": sh.k,
         "routing": "zipf-skewed" if w.zipf else "uniform random",
         "tables": "lloyd + e2m1 (5 experts)" if w.mixed_tables else "lloyd",
         "inputs": f"{ROTATE} rotating seeded batches, resident in HBM",
         "l2": "inputs larger than L2: the timed steps run back to back with no flush; each step's "
               "expert weights exceed L2 and consecutive steps route to different experts ('flushed' "
               "repeats the steps one at a time with a 256 MiB write + 256 MiB read flush before each)"}
    return d


def expert_bytes(sh: inputs.Shape) -> tuple[int, int]:
    """(gate+up bytes, down bytes) of one expert: codes + E8M0 scales."""
    gu = 2 * sh.I * (sh.H // 2 + sh.H // 32)
    dn = sh.H * (sh.I // 2 + sh.I // 32)
    return gu, dn


FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def load_sustained_tflops():
    """The bf16 GEMM peak under the power cap (a seconds-long loop)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f).get("bf16_tflops_sustained", FALLBACK_BF16_TFLOPS_SUSTAINED)
    return FALLBACK_BF16_TFLOPS_SUSTAINED


def max_over_ranks(ms: float, device) -> float:
    """The job's device time: the slowest rank's.  Every rank calls it at the
    same point (an all-reduce with op MAX when more than one rank runs)."""
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: the tokens every rank processed over the slowest
    rank's time (replicas: each rank runs its own batches)."""
    return tokens_per_step * steps * world / (max_ms / 1e3)


def source_digest(files) -> str:
    """Digest of the kernel sources as compiled: line comments and blank lines
    do not count, so a comment edit keeps a profile's figures valid."""
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            text = re.sub(r"//[^\n]*", "", fh.read())
        h.update("\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip()).encode())
    return h.hexdigest()[:16]


def profile_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel_key)
    if not d:
        return None
    if d.get("source_digest") != source_digest(d.get("sources", [])):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, index: int, period_s: float = 0.002):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return self
        names = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                 "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                    r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                    for n, bit in names.items():
                        if r & bit:
                            self.reasons.add(n)
                except Exception:
                    pass
                time.sleep(self.period)

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()
        return False

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline of our arm)
# ---------------------------------------------------------------------------

def oracle_sample_layer(w, x_bits, lg, tokens, device):
    """Oracle layer with the experts the sampled tokens route to, packed by the
    oracle itself from the same bf16 weights (setup, not timed)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    ids, wts = oracle.route(lg[tokens], w.shape.k)
    experts = sorted(set(ids.reshape(-1).tolist()))
    tables, tid = inputs.layer_tables(w)
    sh = w.shape
    L = oracle.Layer(sh.E, sh.H, sh.I, tables, tid)

    def job(e_blobs):
        e, blobs = e_blobs
        out = []
        for proj in inputs.PROJECTIONS:
            N, K = inputs.proj_shape(sh, proj)
            c, s = oracle.pack(blobs[proj][None], tables, tid[e:e + 1], 1, N, K)
            out += [c[0], s[0]]
        return e, out

    jobs = [(e, {p: inputs.bf16_bits(inputs.expert_weight(w, e, p, device=device)) for p in inputs.PROJECTIONS})
            for e in experts]
    with ThreadPoolExecutor(max_workers=os.cpu_count()) as ex:
        for e, parts in ex.map(job, jobs):
            L.set_expert(e, *parts)
    return L, ids, wts


def time_oracle_units(L, x_bits, units, threads):
    """Run oracle units (token, slot, i0, i1) on `threads` threads; wall time."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(lambda u: oracle.expert_partial(L, u[1], x_bits[u[0]], u[2], u[3]), units))
    return time.perf_counter() - t0


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    sh = w.shape
    x_bits = inputs.bf16_bits(inputs.activations(w))
    lg = inputs.router_logits(w).numpy()
    threads = max(1, os.cpu_count() or 1)
    tokens = list(range(min(w.T, 4)))
    L, ids, wts = oracle_sample_layer(w, x_bits, lg, tokens, "cpu")
    # calibrate one unit (one token, one expert, I/8 channels) to size a step
    t_cal = time_oracle_units(L, x_bits, [(0, int(ids[0, 0]), 0, sh.I // 8)], 1) * 8
    budget = 150.0
    q = 1
    while q < sh.I // 32 and (args.steps + args.warmup) * t_cal / q > budget:
        q *= 2
    chunk = sh.I // q

    def step_units(s):
        # `threads` units per step, walking (token, slot, chunk) in order
        out = []
        for u in range(threads):
            n = s * threads + u
            t = tokens[(n // (sh.k * q)) % len(tokens)]
            j = (n // q) % sh.k
            c = n % q
            out.append((t, int(ids[tokens.index(t), j]), c * chunk, (c + 1) * chunk))
        return out

    for s in range(args.warmup):
        time_oracle_units(L, x_bits, step_units(s), threads)
    times = [time_oracle_units(L, x_bits, step_units(args.warmup + s), threads) for s in range(args.steps)]
    tokens_per_step = threads / (sh.k * q)
    total = sum(times)
    value = tokens_per_step * args.steps / total
    sample = (f"each step: {threads} units of one token x one routed expert x {chunk} of {sh.I} intermediate "
              f"channels ({tokens_per_step:.4g} token-equivalents), fp64 oracle, {len(tokens)} sampled tokens")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(workload_desc(w), parallelism=f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline(w, x_bits, lg):
    """The oracle on this host's cores: 2 tokens (1 at T=1) x all their routed
    experts, full channels, each (token, expert) split over intermediate
    channel ranges so that every core has work."""
    import oracle
    oracle.build()
    sh = w.shape
    tokens = [0, 1] if w.T > 1 else [0]
    L, ids, _ = oracle_sample_layer(w, x_bits, lg, tokens, "cuda")
    cores = max(1, os.cpu_count() or 1)
    pairs = [(t, int(ids[i, j])) for i, t in enumerate(tokens) for j in range(sh.k)]
    q = 1
    while len(pairs) * q < cores and q < sh.I // 32:
        q *= 2
    chunk = sh.I // q
    units = [(t, e, c * chunk, (c + 1) * chunk) for t, e in pairs for c in range(q)]
    threads = min(len(units), cores)
    # repeated until about 10 s of wall time have been measured
    dt, reps = 0.0, 0
    while dt < 10.0 and reps < 200:
        dt += time_oracle_units(L, x_bits, units, threads)
        reps += 1
    # the same per-token code on one thread: the first token's units, about 5 s
    one = [u for u in units if u[0] == tokens[0]]
    dt1, reps1 = 0.0, 0
    while dt1 < 5.0 and reps1 < 100:
        dt1 += time_oracle_units(L, x_bits, one, 1)
        reps1 += 1
    return {"value": reps * len(tokens) / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{len(tokens)} token(s) x {sh.k} routed experts, full layer arithmetic in fp64, "
                      f"each (token, expert) in {q} channel ranges of {chunk} over {threads} threads, "
                      f"repeated {reps} times ({dt:.1f} s)",
            "single_thread": {"value": reps1 / dt1, "unit": UNIT, "cores": 1, "kind": "oracle",
                              "sample": f"1 token x {sh.k} routed experts, full layer arithmetic in fp64 on "
                                        f"one thread, repeated {reps1} times ({dt1:.1f} s)"}}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def build_device_layer(w):
    import bit_codebook_quantized_router_b200 as q4
    sh = w.shape
    tables, tid = inputs.layer_tables(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    parts = {}
    for proj in inputs.PROJECTIONS:
        N, K = inputs.proj_shape(sh, proj)
        big = torch.empty((sh.E, N, K), dtype=torch.bfloat16, device="cuda")
        for e in range(sh.E):
            big[e] = inputs.expert_weight(w, e, proj, device="cuda")
        parts[proj] = q4.pack(big, tables, tid, status=status)
        del big
    torch.cuda.empty_cache()
    assert q4.lib().moe_q4_read_status(q4._lib._ptr(status), q4._lib._stream()) == 0
    return q4.Layer(*parts["gate"], *parts["up"], *parts["down"], tables, tid)


# kernels between the forward_stages events, in launch order
KERNELS = [("route", "routing + grouping", None),
           ("gather", "gather of activation rows", None),
           ("gate_up_tc", "tc_gemm_kernel<gate/up> (tensor-core gate/up + SwiGLU)", "tensor"),
           ("gate_up_small", "dk_kernel<gate/up> (small-M gate/up + SwiGLU)", "hbm"),
           ("down_tc", "tc_gemm_kernel<down> (tensor-core down)", "tensor"),
           ("down_small", "dk_kernel<down> (small-M down)", "hbm"),
           ("combine", "combine", None)]
SMALL_M_MAX_ROWS = 16


def kernel_work(sh: inputs.Shape, T: int, counts) -> dict:
    """Algorithmic work of each GEMM kernel for one batch, from its routing
    counts: bytes for the small-M kernels (packed weights of their experts,
    activation rows read, results written), FLOPs for the tensor-core ones."""
    gu, dn = expert_bytes(sh)
    c = np.asarray(counts)
    small = (c > 0) & (c <= SMALL_M_MAX_ROWS)
    big = c > SMALL_M_MAX_ROWS
    rs, rb = int(c[small].sum()), int(c[big].sum())
    return {"gate_up_small": small.sum() * gu + rs * sh.H * 2 + rs * sh.I * 2 * 2,
            "down_small": small.sum() * dn + rs * sh.I * 2 * 2 + rs * sh.H * 4,
            "gate_up_tc": 2.0 * rb * 2 * sh.I * sh.H,
            "down_tc": 2.0 * rb * sh.H * sh.I}


# datasheet figures the fractions are also reported against: HBM3e 8 TB/s,
# dense bf16 2.25 PFLOP/s (the measured peaks are the roofline's denominators)
DATASHEET_HBM_GBS = 8000.0
DATASHEET_BF16_TFLOPS = 2250.0


def roofline(work, kern_ms, n_prof, hbm_peak, tf_peak, peak_src):
    """Achieved rate of every GEMM kernel (algorithmic work / event time,
    summed over the profiled steps) and the roofline entry of the dominant
    one (largest total time)."""
    kernels = {}
    for j, (key, name, bound) in enumerate(KERNELS):
        ms = float(kern_ms[:, j].sum())
        ent = {"name": name, "mean_ms": ms / n_prof}
        if bound is not None:
            tot = float(sum(work[i % ROTATE][key] for i in range(n_prof)))
            if bound == "hbm":
                ach = tot / (ms / 1e3) / 1e9 if ms > 0 else 0.0
                ent.update(bound="hbm", achieved=ach, unit="GB/s", peak=hbm_peak, frac=ach / hbm_peak,
                           frac_of_datasheet=ach / DATASHEET_HBM_GBS,
                           algorithmic_per_launch=tot / n_prof)
            else:
                ach = tot / (ms / 1e3) / 1e12 if ms > 0 else 0.0
                ent.update(bound="tensor", achieved=ach, unit="TFLOP/s", peak=tf_peak, frac=ach / tf_peak,
                           frac_of_datasheet=ach / DATASHEET_BF16_TFLOPS,
                           algorithmic_per_launch=tot / n_prof)
        kernels[key] = ent
    gemms = [k for k, _, b in KERNELS if b is not None and kernels[k]["algorithmic_per_launch"] > 0]
    dom = max(gemms, key=lambda k: kernels[k]["mean_ms"])
    d = kernels[dom]
    roof = {"kernel": d["name"], "bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"],
            "unit": d["unit"], "frac": d["frac"], "frac_of_datasheet": d["frac_of_datasheet"], "peak_source": peak_src,
            "traffic": profile_traffic(dom), "algorithmic_per_launch": d["algorithmic_per_launch"],
            "launch_ms": d["mean_ms"]}
    return roof, kernels



def measure_graph(q4, layer, xs, lgs, k, out, ws, flush_l2, steps, stream):
    """The same forward replayed from CUDA graphs (one per rotating batch):
    launch gaps between the kernels disappear.  Returns (ms_per_step, None) or
    (None, reason)."""
    try:
        graphs = []
        for v in range(ROTATE):
            q4.forward(layer, xs[v], lgs[v], k, out=out, ws=ws)  # warm (host-side lookups)
        torch.cuda.synchronize()
        for v in range(ROTATE):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                q4.forward(layer, xs[v], lgs[v], k, out=out, ws=ws)
            graphs.append(g)
        for v in range(ROTATE):
            graphs[v].replay()
        torch.cuda.synchronize()
        if q4.forward_status(ws) != 0:
            return None, "device status after graph replay"
        st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            flush_l2(i)
            st[i].record(stream)
            graphs[i % ROTATE].replay()
            en[i].record(stream)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in zip(st, en)) / steps
        del graphs
        return ms, None
    except Exception as exc:  # capture unsupported here: report, do not fail the run
        torch.cuda.synchronize()
        return None, f"{type(exc).__name__}: {exc}"[:200]


def measure_dequant(q4, layer, hbm_peak, flush_l2, stream, reps=5):
    """Standalone full-layer dequant: every expert's gate, up and down to bf16
    (three calls, preallocated outputs).  Algorithmic bytes = packed codes +
    scales read + bf16 written."""
    parts = [(layer.gate_w, layer.gate_s), (layer.up_w, layer.up_s), (layer.down_w, layer.down_s)]
    outs = [torch.empty((c.shape[0], c.shape[1], c.shape[2] * 2), dtype=torch.bfloat16, device=c.device)
            for c, _ in parts]
    nbytes = sum(c.numel() + s.numel() + o.numel() * 2 for (c, s), o in zip(parts, outs))

    def run():
        for (c, s), o in zip(parts, outs):
            q4.dequant(c, s, layer.tables, layer.table_id, out=o)

    for _ in range(3):
        run()
    torch.cuda.synchronize()
    st = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    for i in range(reps):
        flush_l2(i)
        st[i].record(stream)
        run()
        en[i].record(stream)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in zip(st, en)) / reps
    del outs
    torch.cuda.empty_cache()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"kernel": "dequant_kernel (all 256 x 3 projections -> bf16)", "bytes": nbytes, "ms": ms,
            "gbs": gbs, "frac": gbs / hbm_peak, "frac_of_datasheet": gbs / DATASHEET_HBM_GBS}


def measure_lloyd(q4, w, hbm_peak, flush_l2, stream, reps=3, max_iter=100):
    """The layer's weighted Lloyd-Max grid fit on the GPU: one pass over all
    the layer's bf16 expert weights (gate, up, down of every expert) into the
    ratio histogram, then the Lloyd steps on it.  Algorithmic bytes: the bf16
    weights read once."""
    sh = w.shape
    grid0 = inputs.lloyd_max_grid()
    projs = []
    for proj in inputs.PROJECTIONS:
        N, K = inputs.proj_shape(sh, proj)
        big = torch.empty((sh.E, N, K), dtype=torch.bfloat16, device="cuda")
        for e in range(sh.E):
            big[e] = inputs.expert_weight(w, e, proj, device="cuda")
        projs.append(big)
    nbytes = sum(p.numel() * 2 for p in projs)
    g, it, st = q4.lloyd_fit(projs, grid0, max_iter=max_iter)  # warm
    torch.cuda.synchronize()
    ok = st == 0
    need = int(q4.lib().moe_q4_lloyd_workspace(np.ascontiguousarray(grid0, np.float32).ctypes.data))
    ws = q4.alloc_workspace(need)
    g0 = np.ascontiguousarray(grid0, np.float32)
    grid = torch.empty(8, dtype=torch.float32, device="cuda")
    iters = torch.empty(1, dtype=torch.int32, device="cuda")
    L = q4.lib()
    sid = ctypes.c_void_p(stream.cuda_stream)
    hist_ms, solve_ms = [], []
    for i in range(reps):
        flush_l2(i)
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record(stream)
        for j, p in enumerate(projs):
            L.moe_q4_lloyd_hist(ctypes.c_void_p(p.data_ptr()), p.numel() // 32, g0.ctypes.data, 1 if j == 0 else 0,
                                ctypes.c_void_p(ws.data_ptr()), ws.numel(), sid)
        e1.record(stream)
        L.moe_q4_lloyd_solve(g0.ctypes.data, max_iter, ctypes.c_double(1e-12), ctypes.c_void_p(grid.data_ptr()),
                             ctypes.c_void_p(iters.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(), sid)
        e2.record(stream)
        torch.cuda.synchronize()
        hist_ms.append(e0.elapsed_time(e1))
        solve_ms.append(e1.elapsed_time(e2))
    ok = ok and torch.equal(grid, g) and int(iters.item()) == int(it.item())
    del projs
    torch.cuda.empty_cache()
    hm, sm = float(np.median(hist_ms)), float(np.median(solve_ms))
    gbs = nbytes / (hm / 1e3) / 1e9
    return {"kernel": "lloyd_hist_kernel (ratio histogram over all 256 x 3 projections) + lloyd_solve_kernel",
            "bytes": nbytes, "hist_ms": hm, "solve_ms": sm, "iters": int(it.item()),
            "grid": [float(v) for v in g.cpu().numpy()], "gbs": gbs, "frac": gbs / hbm_peak,
            "frac_of_datasheet": gbs / DATASHEET_HBM_GBS, "status_ok": bool(ok)}


def measure_shared(q4, w, layer, xs, lgs, hbm_peak, flush_l2, stream, steps=50):
    """The layer with its BF16 shared expert (moe_q4_forward_ex): the same
    steps back to back; bytes = the routed experts touched + the shared
    expert's BF16 weights (3 I H * 2) + x and out."""
    sh = w.shape
    gu, dn = inputs.shared_expert_weights(w, device="cuda")
    shared = q4.Shared(gu, dn)
    T, k = w.T, sh.k
    ws = q4.alloc_workspace(q4.forward_ex_workspace(layer, shared, T, k))
    out = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
    for i in range(5):
        q4.forward_ex(layer, shared, xs[i % ROTATE], lgs[i % ROTATE], k, out=out, ws=ws)
    torch.cuda.synchronize()
    ok = q4.forward_status(ws) == 0
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    # back to back behind a device-side sleep, as the main timed loop: the host
    # enqueues every step before the GPU reaches the first
    torch.cuda._sleep(int(steps * 400_000))
    a.record(stream)
    for i in range(steps):
        q4.forward_ex(layer, shared, xs[i % ROTATE], lgs[i % ROTATE], k, out=out, ws=ws)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    touched = float(np.mean([torch.unique(torch.topk(l, k, dim=1).indices).numel() for l in lgs]))
    gu_b, dn_b = expert_bytes(sh)
    nbytes = touched * (gu_b + dn_b) + 3 * sh.I * sh.H * 2 + T * sh.H * 2 * 2
    gbs = nbytes / (ms / 1e3) / 1e9
    del ws, shared, gu, dn
    return {"kernel": "forward with the shared expert: routed kernels + sx_gemm_kernel<2> (merged gate+up, SwiGLU) + "
                      "sx_gemm_kernel<1> (down) (+ split reduction) + combine",
            "ms_per_step": ms, "value": T / (ms / 1e3), "unit": UNIT, "bytes_per_step": nbytes, "gbs": gbs,
            "frac_of_peak": gbs / hbm_peak, "status_ok": bool(ok),
            "shared_bytes": 3 * sh.I * sh.H * 2}


def measure_gated(q4, w, layer, xs, stream, steps=50):
    """The layer from the hidden states (moe_q4_forward_gated): the bf16
    router gate, the routing and the routed experts, steps back to back.
    The logits-input forward is timed on the same router logits (the same
    routing) beside it: `router_added_ms` is the difference."""
    sh = w.shape
    gate = inputs.router_weight(w, device="cuda")
    T, k = w.T, sh.k
    ws = q4.alloc_workspace(q4.forward_gated_workspace(layer, None, T, k))
    out = torch.empty((T, sh.H), dtype=torch.bfloat16, device="cuda")
    lgs = [q4.router(x, gate) for x in xs]
    runs = {"gated": lambda i: q4.forward_gated(layer, None, gate, xs[i % ROTATE], k, out=out, ws=ws),
            "plain": lambda i: q4.forward(layer, xs[i % ROTATE], lgs[i % ROTATE], k, out=out, ws=ws)}
    ms = {}
    for name, run in runs.items():
        for i in range(5):
            run(i)
        torch.cuda.synchronize()
        assert q4.forward_status(ws) == 0
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(int(steps * 400_000))
        a.record(stream)
        for i in range(steps):
            run(i)
        b.record(stream)
        torch.cuda.synchronize()
        ms[name] = a.elapsed_time(b) / steps
    ok = q4.forward_status(ws) == 0
    touched = float(np.mean([torch.unique(torch.topk(l, k, dim=1).indices).numel() for l in lgs]))
    fused = T <= 32 and sh.H % 128 == 0 and T * k <= 4096
    first = ("router_route_kernel (router gate + routing + grouping, one clustered launch)" if fused else
             "router kernels, then the routing kernels")
    del ws, gate, out, lgs
    return {"kernel": first + ", then the layer's kernels", "ms_per_step": ms["gated"],
            "value": T / (ms["gated"] / 1e3), "unit": UNIT, "logits_input_ms_per_step": ms["plain"],
            "router_added_ms": ms["gated"] - ms["plain"], "touched_experts": touched, "status_ok": bool(ok),
            "note": "routing from a random bf16 gate (no Zipf skew); both steps on the same logits"}


def measure_router(q4, w, xs, hbm_peak, tf_peak, flush_l2, stream, reps=20):
    """The router gate ahead of the layer (moe_q4_router): bf16 x [T, H] times
    the bf16 gate [E, H] -> fp32 logits.  Algorithmic work: the gate and x read
    and the logits written (bytes), 2 T E H flop; reported against the HBM
    roofline at decode sizes and the tensor roofline at prefill sizes."""
    sh = w.shape
    gate = inputs.router_weight(w, device="cuda")
    T = xs[0].shape[0]
    out = torch.empty((T, sh.E), dtype=torch.float32, device="cuda")
    need = q4.router_workspace(T, sh.H, sh.E)
    ws = q4.alloc_workspace(need) if need else None
    for i in range(3):
        q4.router(xs[i % len(xs)], gate, out=out, ws=ws)
    torch.cuda.synchronize()
    # back to back behind a device-side sleep (the host enqueues every call
    # before the GPU reaches the first: its launch overhead is not timed);
    # the rotating x batches and the 3 MB gate stay in L2 between calls
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(int(reps * 400_000))
    a.record(stream)
    for i in range(reps):
        q4.router(xs[i % len(xs)], gate, out=out, ws=ws)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / reps
    nbytes = sh.E * sh.H * 2 + T * sh.H * 2 + T * sh.E * 4
    flop = 2.0 * T * sh.E * sh.H
    gbs = nbytes / (ms / 1e3) / 1e9
    tfs = flop / (ms / 1e3) / 1e12
    hbm_bound = T <= 256
    if T <= 32 and sh.H % 128 == 0:
        kernel, how = "router_few_kernel (one clustered launch)", "mma.sync bf16"
    elif sh.E % 128 == 0 and sh.H % 64 == 0:
        kernel, how = "sx_gemm_kernel<1> (tcgen05 dense GEMM) + sx_reduce_kernel (K split)", "tcgen05 bf16"
    else:
        kernel, how = "router_kernel" + (" + router_reduce_kernel (K split)" if need else ""), "mma.sync bf16"
    return {"kernel": kernel, "ms": ms, "bytes": nbytes,
            "flop": flop, "gbs": gbs, "tflops": tfs, "bound": "hbm" if hbm_bound else "tensor",
            "frac": gbs / hbm_peak if hbm_bound else tfs / tf_peak,
            "frac_of_datasheet": gbs / DATASHEET_HBM_GBS if hbm_bound else tfs / DATASHEET_BF16_TFLOPS,
            "note": how + " GEMM; not part of the step (the layer's input is the logits)"}


def measure_workload(q4, w, args, steps, warmup, world, dev, local, stream, flush_l2, barrier, full):
    """Build workload w's layer and time its forward: K steps back to back
    (the value), per-kernel times, the host-buffer entry point (e2e) and SM
    clocks; with `full`, also the flushed one-at-a-time steps, CUDA-graph
    replay, the full-layer dequant and the router gate.  Returns the fields
    of a bench line (without cpu_baseline)."""
    sh = w.shape
    T, k = w.T, sh.k
    layer = build_device_layer(w)
    xs = [inputs.activations(w, device="cuda", variant=v) for v in range(ROTATE)]
    lgs = [inputs.router_logits(w, device="cuda", variant=v) for v in range(ROTATE)]
    # distinct experts touched per batch (for the algorithmic bytes)
    touched, counts = [], []
    for lg in lgs:
        ids = torch.topk(lg, k, dim=1).indices
        touched.append(int(torch.unique(ids).numel()))
        counts.append(torch.bincount(ids.reshape(-1), minlength=sh.E).cpu().numpy())
    ws = q4.alloc_workspace(q4.forward_workspace(layer, T, k))
    out = torch.empty((T, sh.H), dtype=torch.bfloat16, device=dev)

    for i in range(warmup):
        q4.forward(layer, xs[i % ROTATE], lgs[i % ROTATE], k, out=out, ws=ws)
    torch.cuda.synchronize()
    assert q4.forward_status(ws) == 0

    # Timed: the K steps back to back between one pair of events, no flush.
    # Every step's expert weights alone exceed L2 (8 experts x 20 MB at T=1
    # against 126 MB) and consecutive steps route to different experts, so
    # each step streams its weights from HBM.  A device-side sleep ahead of
    # the first event lets the host enqueue all K steps before the GPU gets
    # to them (the host never starves the timed region).
    t_beg = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        torch.cuda._sleep(int(min(steps, 2000) * 400_000))  # about 0.2 ms per step at 2 GHz
        t_beg.record(stream)
        h0 = time.perf_counter()
        for i in range(steps):
            q4.forward(layer, xs[i % ROTATE], lgs[i % ROTATE], k, out=out, ws=ws)
        enqueue_ms = (time.perf_counter() - h0) * 1e3
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = max_over_ranks(t_beg.elapsed_time(t_end), dev)
    value = job_tokens_per_s(T, steps, world, total_ms)
    assert q4.forward_status(ws) == 0

    flushed_ms = None
    if full:
        # the same steps one at a time, L2 flushed before each, outside its events
        n_fl = min(steps, 200)
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_fl)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_fl)]
        torch.cuda.synchronize()
        for i in range(n_fl):
            flush_l2(i)
            starts[i].record(stream)
            q4.forward(layer, xs[i % ROTATE], lgs[i % ROTATE], k, out=out, ws=ws)
            ends[i].record(stream)
        torch.cuda.synchronize()
        flushed_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / n_fl, dev)

    # per-kernel times (separate pass, events between the kernels)
    n_prof = min(steps, 100)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(n_prof)]
    for row in evs:  # torch creates the CUDA event on first record
        for ev in row:
            ev.record(stream)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk_k:
        for i in range(n_prof):
            flush_l2(i)
            q4.forward_stages(layer, xs[i % ROTATE], lgs[i % ROTATE], k, out, ws, evs[i])
        torch.cuda.synchronize()
    kern_ms = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(7)] for i in range(n_prof)])
    assert q4.forward_status(ws) == 0

    # e2e through the host-buffer entry points (pinned host memory): every
    # step copies its x and logits host->device and its output device->host
    # inside the timed region.  Throughput (the e2e value): the steps enqueued
    # back to back with moe_q4_forward_host_async between one pair of events
    # behind a device-side sleep, as the main timed loop (no flush: the
    # rotating batches' weights exceed L2), the device status read once at
    # the end.  Latency (e2e_sync): moe_q4_forward_host, which waits for its
    # own work, one call at a time after an L2 flush.
    n_e2e = min(steps, 200)
    xh = [x.cpu().pin_memory() for x in xs]
    lh = [l.cpu().pin_memory() for l in lgs]
    ohs = [torch.empty((T, sh.H), dtype=torch.bfloat16).pin_memory() for _ in range(ROTATE)]
    wsh = q4.alloc_workspace(q4.forward_host_workspace(layer, T, k))
    for i in range(3):
        q4.forward_host(layer, xh[i % ROTATE], lh[i % ROTATE], k, ohs[0], wsh)
    ta, tb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    torch.cuda._sleep(int(min(n_e2e, 2000) * 400_000))
    ta.record(stream)
    for i in range(n_e2e):
        q4.forward_host_async(layer, xh[i % ROTATE], lh[i % ROTATE], k, ohs[i % ROTATE], wsh)
    tb.record(stream)
    assert q4.forward_status(wsh) == 0
    barrier()
    e2e_ms = max_over_ranks(ta.elapsed_time(tb), dev)
    e2e_value = job_tokens_per_s(T, n_e2e, world, e2e_ms)
    n_sync = min(n_e2e, 100)
    e_s = [torch.cuda.Event(enable_timing=True) for _ in range(n_sync)]
    e_e = [torch.cuda.Event(enable_timing=True) for _ in range(n_sync)]
    torch.cuda.synchronize()
    for i in range(n_sync):
        flush_l2(i)
        e_s[i].record(stream)
        st = q4.forward_host(layer, xh[i % ROTATE], lh[i % ROTATE], k, ohs[0], wsh)
        e_e[i].record(stream)
        assert st == 0
    torch.cuda.synchronize()
    e2e_sync_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_s, e_e)), dev)
    e2e_sync_value = job_tokens_per_s(T, n_sync, world, e2e_sync_ms)
    del wsh

    hbm_peak, tf_peak, peak_src = load_peaks()
    # The tensor-core kernels' denominator follows the regime the per-kernel
    # timing ran in: the burst GEMM peak while the SM clock held its maximum,
    # the sustained one (the power cap's) when the clock fell below 90% of it
    # during that loop.  Both fractions are reported.
    ck = clk_k.summary()
    tf_burst, tf_sust = tf_peak, load_sustained_tflops()
    capped = bool(ck.get("sm_mhz") and ck.get("sm_max_mhz") and ck["sm_mhz"] < 0.9 * ck["sm_max_mhz"])
    tf_peak = tf_sust if capped else tf_burst
    work = [kernel_work(sh, T, c) for c in counts]
    roof, kernels = roofline(work, kern_ms, n_prof, hbm_peak, tf_peak, peak_src)
    for ent in list(kernels.values()) + [roof]:
        if ent.get("bound") == "tensor":
            ent["peak_regime"] = "sustained" if capped else "burst"
            ent["frac_of_burst"] = ent["achieved"] / tf_burst
            ent["frac_of_sustained"] = ent["achieved"] / tf_sust
    gu, dn = expert_bytes(sh)
    layer_bytes = float(np.mean(touched)) * (gu + dn) + T * sh.H * 2 * 2
    # our kernels per forward: route (1 fused for T <= 256, else 2), small-M
    # gate/up and down, combine, and for T > 16 the gather and the two
    # tensor-core GEMMs
    kernels_per_step = (1 if T <= 256 else 2) + 3 + (3 if T > 16 else 0)
    res = {
        "value": value, "ms_per_step": total_ms / steps, "steps": steps, "warmup": warmup,
        "config": dict(workload_desc(w), parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        "roofline": roof,
        "kernels": kernels,
        "layer_hbm": {"touched_experts": float(np.mean(touched)), "bytes_per_step": layer_bytes,
                      "gbs": layer_bytes / (total_ms / steps / 1e3) / 1e9,
                      "frac_of_peak": layer_bytes / (total_ms / steps / 1e3) / 1e9 / hbm_peak,
                      "frac_of_datasheet": layer_bytes / (total_ms / steps / 1e3) / 1e9 / DATASHEET_HBM_GBS},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": T * sh.H * 2 + T * sh.E * 4,
                "d2h_bytes_per_step": T * sh.H * 2,
                "api": "moe_q4_forward_host_async, steps back to back, status read at the end"},
        "e2e_sync": {"value": e2e_sync_value, "unit": UNIT,
                     "api": "moe_q4_forward_host (waits for each call), one call at a time after an L2 flush"},
        "enqueue_ms": enqueue_ms,
        "gpu_launches": kernels_per_step * steps,
        "clocks": clk.summary(),
        "clocks_kernel_timing": ck,
    }
    res["router"] = measure_router(q4, w, xs, hbm_peak, tf_peak, flush_l2, stream)
    res["shared_expert"] = measure_shared(q4, w, layer, xs, lgs, hbm_peak, flush_l2, stream,
                                          steps=min(steps, 50))
    res["gated"] = measure_gated(q4, w, layer, xs, stream, steps=min(steps, 50))
    if full:
        res["flushed"] = {"value": T * world / (flushed_ms / 1e3), "unit": UNIT, "ms_per_step": flushed_ms,
                          "steps": n_fl,
                          "note": "each step alone between its own events, L2 flushed before it (outside the events)"}
        graph_ms, graph_why = measure_graph(q4, layer, xs, lgs, k, out, ws, flush_l2, min(steps, 200), stream)
        res["graph"] = ({"value": T * world / (graph_ms / 1e3), "unit": UNIT, "ms_per_step": graph_ms,
                         "note": "same forward replayed from CUDA graphs, L2 flushed outside the events"}
                        if graph_ms else {"value": None, "unavailable": graph_why})
        res["dequant"] = measure_dequant(q4, layer, hbm_peak, flush_l2, stream) if not args.no_dequant else None
        if not args.no_lloyd:
            res["lloyd"] = measure_lloyd(q4, w, hbm_peak, flush_l2, stream)
        res["_cpu_inputs"] = (inputs.bf16_bits(xs[0]), lgs[0].cpu().numpy())
    del layer, xs, lgs, ws, out
    torch.cuda.empty_cache()
    return res


# workloads timed in the same run beside the primary one (one GPU only): the
# second decode size and the tensor-core prefill size of the performance bars
EXTRA_WORKLOADS = ("decode_t8", "prefill_t2048")
EXTRA_STEPS = 50


def run_ours(args, w):
    import torch.distributed as dist

    import bit_codebook_quantized_router_b200 as q4
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    scrub = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2(i):
        flush.fill_(i & 0xFF)
        scrub.sum()

    def barrier():
        if world > 1:
            dist.barrier()

    res = measure_workload(q4, w, args, args.steps, args.warmup, world, dev, local, stream, flush_l2, barrier,
                           full=True)
    x_bits, lg0 = res.pop("_cpu_inputs")
    line = {"metric": METRIC, "value": res.pop("value"), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": res.pop("ms_per_step"), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic"}
    res.pop("steps")
    res.pop("warmup")
    line.update(res)
    if world == 1 and not args.no_extra:
        extra = {}
        for name in EXTRA_WORKLOADS:
            if name == w.name:
                continue
            we = inputs.WORKLOADS[name]
            if args.experts:
                import dataclasses
                we = dataclasses.replace(we, shape=dataclasses.replace(we.shape, E=args.experts))
            r = measure_workload(q4, we, args, min(args.steps, EXTRA_STEPS), args.warmup, world, dev, local,
                                 stream, flush_l2, barrier, full=False)
            r["metric"], r["unit"] = METRIC, UNIT
            extra[name] = r
        line["workloads"] = extra
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, x_bits, lg0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_t1", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dequant", action="store_true", help="skip the standalone full-layer dequant measurement")
    ap.add_argument("--no-lloyd", action="store_true", help="skip the GPU grid-fit measurement")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (not also decode_t8 and prefill_t2048 in the same line)")
    ap.add_argument("--experts", type=int, default=0,
                    help="layer with this many experts (same H, I, top-k) instead of the workload's; "
                         "for small profiling captures")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = inputs.WORKLOADS[args.workload]
    if args.experts:
        import dataclasses
        w = dataclasses.replace(w, shape=dataclasses.replace(w.shape, E=args.experts))
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
