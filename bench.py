"""Benchmark of the POET-X layer hot path on B200: forward + backward of the
Llama-8B decoder block's seven linears (q, k, v, o, gate, up, down; b = 256,
16384 tokens per GPU), CNP build and CNP backward included, merge excluded.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl poetx|reference]

One step = the G_R, G_P blocks of every linear built from the packed triangles
(one batched CNP build), the forwards (saving Y and the gathered input), the
backwards in reverse order (dx and the token sums dG of both sides), then one
batched CNP backward from the dG of all linears to their packed dq.  The
headline step is input-centric (the write-up's section 1): every block product
acts on token rows and no transformed weight is formed; the weight-fold and
weight-centric evaluations are reported as labelled variants.  With N > 1
ranks each linear's dG is summed across ranks (NCCL all-reduce, the
data-parallel exchange) as soon as its backward is done, overlapped with the
next linear's backward; the CNP backward is linear in dG, so this gives the
summed dq.  Each rank processes its own 16384 tokens (weak
scaling).  Inputs are synthetic (seeded normal activations / gradients,
N(0, 0.02^2) weights, N(0, 0.01^2) triangles, seeded permutations), drawn on
the device; q, k, v read one input and gate, up another, as in the decoder
block; every tensor of the working set is larger than L2.

The JSON line also carries: the end-to-end rate through the Python API with
every step's inputs copied from pinned host memory and the dq read back
("e2e"); the stage breakdown from the library's profiler; the dominant
kernel's roofline; nvidia-smi clocks, reasons and power stamped inside the
timed region; the folded / mem / POET-XQ variants and the optimizer step, each
variant timed right after a fresh timing of the plain step; the merge of all
seven linears; and ("configs") the single-layer workloads attn3b, up8b and
down13b (step rate, W0 roofline, CNP build and backward microbenchmark, the
down13b merge) and the 8B block's batched CNP microbenchmark.

--impl reference times the float64 CPU oracle (oracle/) on the host cores on
a bounded token sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import poetx_inputs as pi  # noqa: E402

METRIC = "POET-X layer fwd+bwd tokens/s (Llama-8B shapes, b=256); % bf16 tensor peak"
WORKLOAD = "block8b"
# DRAM bytes (read + write) per launch of the dominant kernel -- the forward
# W0 GEMM (CTA-pair kernel) at M = 16384, N = 14336, K = 4096 -- from an ncu
# capture of that kernel and shape (dram__bytes_read.sum +
# dram__bytes_write.sum); reset to None whenever the kernel changes until it
# is captured again.
W0_GEMM_TRAFFIC_BYTES = 948963840 + 455262208
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0   # B200 dense bf16 tensor-core peak (datasheet, no sparsity)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def config_block(cfg: pi.Config, n_gpus: int) -> dict:
    return {"workload": f"{cfg.name}: {cfg.description}",
            "linears": [f"{nm} {m}x{n}" for nm, m, n in cfg.layers],
            "tokens_per_gpu": cfg.T, "global_batch": cfg.T * n_gpus, "seq_len": 2048, "b": cfg.b,
            "parallelism": f"dp{n_gpus}",
            "shared_inputs": [",".join(cfg.layers[i][0] for i in range(len(cfg.layers)) if cfg.x_source(i) == j)
                              for j in sorted({cfg.x_source(i) for i in range(len(cfg.layers))})
                              if sum(cfg.x_source(i) == j for i in range(len(cfg.layers))) > 1],
            "l2": "no flush: every input and intermediate is larger than the 126 MB L2"}


# ---------------------------------------------------------------- distributed helpers
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(
        os.environ.get("LOCAL_RANK", "0"))


def reduce_max(value: float, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_grads(flat) -> None:
    """Sum the packed gradients of every linear across data-parallel ranks."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM)


def allreduce_start(t):
    """Start summing `t` across data-parallel ranks without waiting (the
    collective runs on the communication stream while later kernels run);
    returns a handle for allreduce_finish, or None with a single rank."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        return dist.all_reduce(t, op=dist.ReduceOp.SUM, async_op=True)
    return None


def allreduce_finish(handles) -> None:
    """Make the current stream wait for every started all-reduce."""
    for h in handles:
        if h is not None:
            h.wait()


def barrier(device) -> None:
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier(device_ids=[device.index] if device.type == "cuda" else None)
    if device.type == "cuda":
        torch.cuda.synchronize(device)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples around the timed region.
    Each sample carries nvidia-smi's own timestamp; `mark_begin` / `mark_end`
    bracket the region on the host clock and only the samples inside it count
    as "under load" (the median clock, the instantaneous power)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw.instant,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None
        self.t_begin = None
        self.t_end = None

    def start(self):
        fields = self.FIELDS
        try:
            # drivers without the instantaneous power field: the averaged one
            probe = subprocess.run(["nvidia-smi", f"--query-gpu={fields}", "--format=csv,noheader,nounits", "-i",
                                    self.gpu_id], capture_output=True, text=True, timeout=20)
            if probe.returncode != 0:
                fields = fields.replace("power.draw.instant", "power.draw")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", self.gpu_id], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except (OSError, subprocess.TimeoutExpired):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark_begin(self):
        self.t_begin = time.time()

    def mark_end(self):
        self.t_end = time.time()

    @staticmethod
    def parse(lines, t_begin=None, t_end=None) -> dict:
        """Samples -> the clocks record.  Samples outside [t_begin, t_end]
        (when both are given and at least one sample falls inside) are
        dropped; reasons are collected over the kept samples."""
        rows = []
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            try:
                sm, smax = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            try:
                power = float(parts[4])
            except ValueError:
                power = None
            rows.append((ts, sm, smax, power, parts[6:10]))
        inside = rows
        if t_begin is not None and t_end is not None:
            sel = [r for r in rows if r[0] is not None and t_begin <= r[0] <= t_end]
            if sel:
                inside = sel
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}
        reasons = set()
        for r in inside:
            for name, v in zip(ClockSampler.NAMES, r[4]):
                if v.lower() == "active":
                    reasons.add(name)
        powers = [r[3] for r in inside if r[3] is not None]
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside), "samples_total": len(rows),
                "sm_mhz_min": min(r[1] for r in inside),
                "power_w_median": statistics.median(powers) if powers else None,
                "power_w_max": max(powers) if powers else None,
                "window": "samples stamped inside the timed region" if inside is not rows else "all samples"}

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)  # the sample that covers the region's end
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        return self.parse(self.lines, self.t_begin, self.t_end)


# ---------------------------------------------------------------- POET-X arm
def build_block(cfg: pi.Config, device, rank: int, fold: int = 0):
    import torch
    import orthogonal_equivalence_b200 as px
    layers = []
    for li, (name, m, n) in enumerate(cfg.layers):
        g = torch.Generator(device=device)
        g.manual_seed(pi.seed_of(cfg, li, "W0"))
        W0lin = (torch.randn((n, m), generator=g, device=device, dtype=torch.float32) * 0.02).to(torch.bfloat16)
        gc = torch.Generator()
        gc.manual_seed(pi.seed_of(cfg, li, "permR"))
        permR = torch.randperm(m, generator=gc).to(torch.int32)
        gc.manual_seed(pi.seed_of(cfg, li, "permP"))
        permP = torch.randperm(n, generator=gc).to(torch.int32)
        tri = cfg.b * (cfg.b - 1) // 2
        g.manual_seed(pi.seed_of(cfg, li, "qR"))
        qR = torch.randn((m // cfg.b, tri), generator=g, device=device) * cfg.sigma_q
        g.manual_seed(pi.seed_of(cfg, li, "qP"))
        qP = torch.randn((n // cfg.b, tri), generator=g, device=device) * cfg.sigma_q
        L = px.PoetxLinear(m, n, cfg.b, px.POETX_BF16, device=device, fold=fold)
        L.load(W0lin, permR, permP, qR, qP)
        del W0lin
        # per-rank data (each data-parallel rank sees its own tokens); linears
        # of a block that read the same hidden state share one x
        src = cfg.x_source(li)
        if src != li:
            x = layers[src]["x"]
        else:
            g.manual_seed(pi.seed_of(cfg, li, "x") + 7919 * rank)
            x = torch.randn((cfg.T, m), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
        g.manual_seed(pi.seed_of(cfg, li, "dz") + 7919 * rank)
        dz = torch.randn((cfg.T, n), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
        layers.append({"L": L, "x": x, "dz": dz, "m": m, "n": n, "x_src": src})
    group = px.LayerGroup([l["L"] for l in layers])
    group.flatten_params()
    dG = group.dG_buffer()
    off = 0
    for l, (dGR, dGP) in zip(layers, group.dG_views(dG)):
        l["group"] = group
        l["dGR"], l["dGP"] = dGR, dGP
        l["dG_all"] = dG[off:off + dGR.shape[0] + dGP.shape[0]]  # both sides, contiguous
        off += dGR.shape[0] + dGP.shape[0]
    layers[0]["dG"] = dG
    # outputs and saved activations, allocated once
    nq = sum(l["L"].qR.numel() + l["L"].qP.numel() for l in layers)
    flat = torch.zeros(nq, dtype=torch.float32, device=device)
    off = 0
    for l in layers:
        L = l["L"]
        l["z"] = torch.empty((cfg.T, l["n"]), dtype=torch.bfloat16, device=device)
        l["y"] = torch.empty((cfg.T, l["n"]), dtype=torch.bfloat16, device=device)
        l["xg"] = torch.empty((cfg.T, l["m"]), dtype=torch.bfloat16, device=device)
        l["dx"] = torch.empty((cfg.T, l["m"]), dtype=torch.bfloat16, device=device)
        l["dqR"] = flat[off:off + L.qR.numel()].view_as(L.qR)
        off += L.qR.numel()
        l["dqP"] = flat[off:off + L.qP.numel()].view_as(L.qP)
        off += L.qP.numel()
    return layers, flat


def run_step(layers, flat, mem: bool = False, xs=None, dzs=None, ready=None) -> None:
    """One step: G of every linear from its packed triangles (one batched CNP
    build); the forwards, which keep Y and Xg = x[:, permR] for the backward
    (with `mem`, nothing: the backward recomputes Y); the backwards in reverse
    order down to dx and the token sums dG; one batched CNP backward from the
    dG of all linears to their packed dq; the data-parallel gradient sum.
    `xs`, `dzs` replace the resident inputs; `ready(i, kind)` is called before
    linear i first reads x ("x") or dz ("dz")."""
    group = layers[0]["group"]
    group.build()
    for i, l in enumerate(layers):
        x = l["x"] if xs is None else xs[i]
        if ready:
            ready(i, "x")
        if mem:
            l["L"].forward(x, save=False, z=l["z"])
            l["saved"] = None
        else:
            l["saved"] = l["L"].forward(x, save_xg=True, z=l["z"], y=l["y"], xg=l["xg"])[1]
    pending = []
    for i in reversed(range(len(layers))):
        l = layers[i]
        if ready:
            ready(i, "dz")
        l["L"].backward_dG(l["x"] if xs is None else xs[i], l["saved"], l["dz"] if dzs is None else dzs[i],
                           l["dGR"], l["dGP"], dx=l["dx"])
        if ready:
            ready(i, "done")
        # the data-parallel exchange: this linear's dG summed across ranks
        # while the next linear's backward runs (dq is linear in dG)
        pending.append(allreduce_start(l["dG_all"]))
    allreduce_finish(pending)
    group.cnp_backward(layers[0]["dG"], flat)


def time_per_call(fn, k: int, device, stream) -> float:
    """Mean device ms of fn() over k calls: CUDA events on the launching
    stream between barriers + synchronizes, max over ranks."""
    import torch
    barrier(device)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(k):
        fn()
    b_.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    return reduce_max(a.elapsed_time(b_), device) / k


def dominant_w0(cfg: pi.Config, records):
    """The dominant kernel: the forward W0 GEMM (Y = U W~, M = T, N = n,
    K = m) of the linears with the largest m x n and that exact shape.
    Returns ((m, n), those linears, their per-launch ms from the profiler's
    records of whole input-centric steps, whose W0 launches come forward in
    layer order, then backward in reverse order)."""
    L = len(cfg.layers)
    big = max(m * n for _, m, n in cfg.layers)
    shape = next((m, n) for _, m, n in cfg.layers if m * n == big)
    dom_layers = [i for i, (_, m, n) in enumerate(cfg.layers) if (m, n) == shape]
    w0_rec = [ms for st, ms in records if st == "w0_gemm"]
    dom_ms = [ms for k, ms in enumerate(w0_rec) if (k % (2 * L)) < L and (k % (2 * L)) in dom_layers]
    return shape, dom_layers, dom_ms


def time_merges(cfg: pi.Config, plist, device, stream, k: int = 3) -> dict:
    """One merge (W0 <- R W0 P into a scratch weight, q = 0, G = I) of every
    layer in `plist`, timed over k repetitions (the merge's arithmetic does
    not depend on the values, so the repetitions that start from q = 0 cost
    the same).  Algorithmic work per layer: 4 n m b flops (the two block
    products) and 4 n m bytes (the bf16 weight read and written)."""
    import torch
    import orthogonal_equivalence_b200 as px
    nb = max(px.poetx_merge_workspace_bytes(L.abi()) for L in plist)
    ws = torch.empty(nb, dtype=torch.uint8, device=device)
    W_out = torch.empty(max(L.m * L.n for L in plist), dtype=torch.bfloat16, device=device)
    perms = []
    for i, L in enumerate(plist):
        newR, newP = pi.merge_perms(cfg, i, 1, L.m, L.n)
        perms.append((torch.from_numpy(newR).to(device), torch.from_numpy(newP).to(device)))

    def merge_all():
        for L, (newR, newP) in zip(plist, perms):
            px.poetx_merge(L.abi(), newR, newP, W_out, ws, nb)

    merge_all()
    ms = time_per_call(merge_all, k, device, stream)
    flops = sum(4.0 * L.n * L.m * L.b for L in plist)
    nbytes = sum(4.0 * L.n * L.m for L in plist)
    return {"layers": [f"{L.m}x{L.n}" for L in plist], "ms": ms, "tflops": flops / (ms / 1e3) / 1e12,
            "algorithmic_gbs": nbytes / (ms / 1e3) / 1e9,
            "note": "one merge of every listed linear: W0 <- R W0 P re-framed into new permutations, q = 0, G = I"}


def cnp_microbench(cfg: pi.Config, device, stream, k: int = 20) -> dict:
    """The Cayley-Neumann build of G_R, G_P of every linear of `cfg` (one
    batch) and its backward from dG to the packed dq (one batch), timed
    separately over k calls each.  Algorithmic flops per block: 4 b^3 for the
    build (S = Q Q, then (2Q + S) S), 8 b^3 for the backward."""
    import torch
    import orthogonal_equivalence_b200 as px
    b = cfg.b
    Ls = []
    for li, (_, m, n) in enumerate(cfg.layers):
        L = px.PoetxLinear(m, n, b, px.POETX_BF16, device=device)
        g = torch.Generator(device=device)
        g.manual_seed(pi.seed_of(cfg, li, "qR"))
        L.qR.copy_(torch.randn(L.qR.shape, generator=g, device=device) * cfg.sigma_q)
        g.manual_seed(pi.seed_of(cfg, li, "qP"))
        L.qP.copy_(torch.randn(L.qP.shape, generator=g, device=device) * cfg.sigma_q)
        Ls.append(L)
    group = px.LayerGroup(Ls)
    q = group.flatten_params()
    dG = group.dG_buffer()
    g = torch.Generator(device=device)
    g.manual_seed(pi.seed_of(cfg, 0, "dz"))
    dG.copy_(torch.randn(dG.shape, generator=g, device=device))
    dq = torch.empty_like(q)
    nblk = dG.shape[0]
    group.build()
    group.cnp_backward(dG, dq)
    build_ms = time_per_call(group.build, k, device, stream)
    bwd_ms = time_per_call(lambda: group.cnp_backward(dG, dq), k, device, stream)
    return {"blocks": int(nblk), "b": b, "build_us": build_ms * 1e3, "backward_us": bwd_ms * 1e3,
            "build_tflops": 4.0 * b ** 3 * nblk / (build_ms / 1e3) / 1e12,
            "backward_tflops": 8.0 * b ** 3 * nblk / (bwd_ms / 1e3) / 1e12,
            "path": "fused CTA-pair kernel (bf16 operands, fp32 accumulate)" if b == 256 else
                    "batched tcgen05 GEMM chain (tf32 operands, fp32 accumulate)",
            "note": "q ~ N(0, sigma^2) of the workload, dG ~ N(0, 1); k calls of each, CUDA events"}


def measure_layer_config(name: str, args, device, stream, peaks) -> dict:
    """One single-layer workload (input-centric): the step of run_step on its
    own layer, timed like the headline, plus its W0 GEMM roofline, the CNP
    microbench of its blocks and (down13b) its merge."""
    import torch
    import orthogonal_equivalence_b200 as px
    cfg = pi.CONFIGS[name]
    layers, flat = build_block(cfg, device, 0)
    for _ in range(3):
        run_step(layers, flat)
    k = max(3, min(args.steps, 10))
    ms = time_per_call(lambda: run_step(layers, flat), k, device, stream)
    px.poetx_profile_begin()
    for _ in range(2):
        run_step(layers, flat)
    torch.cuda.synchronize(device)
    stages = px.poetx_profile_end()
    records = px.poetx_profile_records()
    shape, _, dom_ms = dominant_w0(cfg, records)
    dom_flops = 2.0 * cfg.T * shape[0] * shape[1]
    w0 = dom_flops / (statistics.mean(dom_ms) / 1e3) / 1e12 if dom_ms else None
    tflops = cfg.flops_per_step() / (ms / 1e3) / 1e12
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    out = {"workload": cfg.description, "tokens_per_s": cfg.T / (ms / 1e3), "ms_per_step": ms, "steps": k,
           "tflops": tflops, "pct_bf16_peak_nominal": 100.0 * tflops / NOMINAL_BF16_TFLOPS,
           "stages_ms_per_step": {s_: v[0] / 2 for s_, v in stages.items() if v[1]},
           "w0_forward": {"M": cfg.T, "N": shape[1], "K": shape[0], "tflops": w0,
                          "frac_of_measured_burst": (w0 / burst) if w0 else None,
                          "frac_of_nominal": (w0 / NOMINAL_BF16_TFLOPS) if w0 else None}}
    plist = [l["L"] for l in layers]
    for l in layers:
        del l["L"]
    del layers, flat
    out["cnp"] = cnp_microbench(cfg, device, stream)
    if name == "down13b":
        out["merge"] = time_merges(cfg, plist, device, stream)
    del plist
    torch.cuda.empty_cache()
    return out


def bench_poetx(args, cfg: pi.Config) -> dict:
    import torch
    import torch.distributed as dist
    import orthogonal_equivalence_b200 as px
    from orthogonal_equivalence_b200 import build as pbuild

    rank, world, local = dist_env()
    if world > 1:
        # NVSwitch multicast (NVLS) off unless the caller sets it: the exchange
        # is a few tens of MB overlapped with the backward, and a rank that
        # exits while bound to a multicast object can disturb its peers
        os.environ.setdefault("NCCL_NVLS_ENABLE", "0")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if rank == 0:
        pbuild.build()
    if world > 1:
        dist.barrier(device_ids=[local])
    px.lib()

    layers, flat = build_block(cfg, device, rank)
    torch.cuda.synchronize(device)
    for _ in range(args.warmup):
        run_step(layers, flat)
    barrier(device)

    props = torch.cuda.get_device_properties(device)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid else str(local))
    sampler.start()
    time.sleep(0.3)
    stream = torch.cuda.current_stream(device)
    # Timed region: K steps, CUDA events on the launching stream only at its
    # ends (value, ms_per_step).
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    sampler.mark_begin()
    start.record(stream)
    for _ in range(args.steps):
        run_step(layers, flat)
    end.record(stream)
    torch.cuda.synchronize(device)
    sampler.mark_end()
    barrier(device)
    clocks = sampler.stop()
    ms_local = start.elapsed_time(end)
    ms_total = reduce_max(ms_local, device)

    # Profiled timed region: the same K steps again with the library's stage
    # profiler on (a CUDA event pair around every launch on its stream): the
    # stage breakdown, the launch count and the dominant kernel's per-launch
    # times for the roofline.  The events cost a few microseconds per launch,
    # which is why the headline value comes from the region above.
    barrier(device)
    px.poetx_profile_begin()
    p_start, p_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p_start.record(stream)
    for _ in range(args.steps):
        run_step(layers, flat)
    p_end.record(stream)
    torch.cuda.synchronize(device)
    stages = px.poetx_profile_end()
    records = px.poetx_profile_records()
    barrier(device)
    ms_profiled = reduce_max(p_start.elapsed_time(p_end), device)

    # End to end through the public API: every step copies its inputs (each
    # distinct x, which q/k/v and gate/up share, and the dz of every linear)
    # from pinned host memory and reads the packed gradients back.  The
    # copies run on their own stream into two alternating sets of device
    # buffers, so step s+1's inputs stream in while step s computes; each
    # linear waits only for its own inputs.
    e2e = None
    if not args.no_e2e:
        srcs = sorted({l["x_src"] for l in layers})
        host_x = {j: layers[j]["x"].cpu().pin_memory() for j in srcs}
        host_dz = [l["dz"].cpu().pin_memory() for l in layers]
        host_dq = torch.empty(flat.numel(), dtype=torch.float32).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in list(host_x.values()) + host_dz)
        d2h = host_dq.numel() * 4
        e_steps = max(2, min(args.steps, 6))
        copy_stream = torch.cuda.Stream(device)
        dev_x = [{j: layers[j]["x"] for j in srcs}, {j: torch.empty_like(layers[j]["x"]) for j in srcs}]
        dev_dz = [[l["dz"] for l in layers], [torch.empty_like(l["dz"]) for l in layers]]
        readers = {j: [i for i, l in enumerate(layers) if l["x_src"] == j] for j in srcs}
        ev = lambda: torch.cuda.Event()  # noqa: E731
        x_ready = [{j: ev() for j in srcs} for _ in range(2)]
        dz_ready = [[ev() for _ in layers] for _ in range(2)]
        consumed = [[ev() for _ in layers] for _ in range(2)]
        for k in range(2):
            for e in consumed[k]:
                e.record(stream)

        def e2e_step(k):
            with torch.cuda.stream(copy_stream):
                for j in srcs:
                    for i in readers[j]:
                        copy_stream.wait_event(consumed[k][i])
                    dev_x[k][j].copy_(host_x[j], non_blocking=True)
                    x_ready[k][j].record(copy_stream)
                for i in reversed(range(len(layers))):
                    dev_dz[k][i].copy_(host_dz[i], non_blocking=True)
                    dz_ready[k][i].record(copy_stream)

            def ready(i, kind):
                if kind == "x":
                    stream.wait_event(x_ready[k][layers[i]["x_src"]])
                elif kind == "dz":
                    stream.wait_event(dz_ready[k][i])
                else:
                    consumed[k][i].record(stream)

            xs = [dev_x[k][l["x_src"]] for l in layers]
            run_step(layers, flat, xs=xs, dzs=dev_dz[k], ready=ready)
            host_dq.copy_(flat, non_blocking=True)

        e2e_step(0)
        e2e_step(1)
        barrier(device)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        copy_stream.wait_event(s2)
        for it in range(e_steps):
            e2e_step(it % 2)
        e2.record(stream)
        torch.cuda.synchronize(device)
        e_ms = reduce_max(s2.elapsed_time(e2), device)
        e2e = {"value": world * cfg.T * e_steps / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": e_steps,
               "h2d_gbs": h2d * e_steps / (e_ms / 1e3) / 1e9}
    # Variants of the same step (see the POET-X write-up's three variants and
    # its optimizer), each timed right after the plain step over the same
    # number of steps ("base_ms_per_step"), so that the pair shares the
    # board's power and thermal state (it drifts over a run at the cap):
    #   folded     - both per-step weight folds (POETX_FOLD_R | POETX_FOLD_P):
    #                G_R applied to the weight rows in the forward, G_P in the
    #                backward (transient weight-sized copies, not input-centric)
    #   mem        - nothing kept between forward and backward but x; the
    #                backward recomputes Y (input-centric throughout)
    #   mem_folded - mem with every fold, so the forward that saves nothing is
    #                the weight-centric single GEMM
    #   optimizer_step - AdamW on all packed triangles + batched CNP rebuild
    #   xq         - weights kept as int8 codes, dequantized before each use
    variants = None
    merge_block = None
    if not args.no_variants:
        def timed(fn, k):
            return time_per_call(fn, k, device, stream)

        def set_fold(f):
            for l in layers:
                l["L"].fold = f

        base = lambda: run_step(layers, flat)  # noqa: E731
        step_mem = lambda: run_step(layers, flat, mem=True)  # noqa: E731
        variants = {}
        transient = int(max(2 * l["m"] * l["n"] for l in layers))
        for vname, fold, fn, note in (
                ("folded", px.POETX_FOLD_ALL, base,
                 "G_R folded into the weight rows in the forward (T > n), G_P in the backward (T > m): "
                 "weight-sized transient copies in the existing workspace; not input-centric"),
                ("mem", 0, step_mem, "backward recomputes Y; no [T][n] activation kept; input-centric"),
                ("mem_folded", px.POETX_FOLD_ALL, step_mem,
                 "mem with every fold: the forward that saves nothing is one GEMM on the whole transformed "
                 "weight (weight-centric)")):
            set_fold(fold)
            fn()
            set_fold(0)
            ms_b = timed(base, args.steps)
            set_fold(fold)
            ms = timed(fn, args.steps)
            set_fold(0)
            variants[vname] = {"tokens_per_s": world * cfg.T / (ms / 1e3), "ms_per_step": ms,
                               "base_ms_per_step": ms_b, "fold": fold, "note": note}
            if fold:
                variants[vname]["transient_weight_bytes"] = transient
                variants[vname]["extra_workspace_bytes"] = 0
        group = layers[0]["group"]
        opt = lambda: group.optimizer_step(flat, 1e-4, weight_decay=0.0)  # noqa: E731
        opt()
        ms = timed(opt, args.steps)
        variants["optimizer_step"] = {"ms_per_step": ms, "params": int(group.q.numel()),
                                      "note": "AdamW on every packed triangle + batched CNP rebuild of every G"}
        ms_b = timed(base, args.steps)
        scratch = torch.empty(max(l["m"] * l["n"] for l in layers), dtype=torch.bfloat16, device=device)
        saved_W = [l["L"].W for l in layers]
        for l in layers:
            l["L"].quantize_weight(scratch)
        run_step(layers, flat)
        ms = timed(base, args.steps)
        # stage breakdown of the same step (library profiler, a few steps)
        px.poetx_profile_begin()
        for _ in range(3):
            run_step(layers, flat)
        torch.cuda.synchronize(device)
        xq_stages = px.poetx_profile_end()
        variants["xq"] = {"tokens_per_s": world * cfg.T / (ms / 1e3), "ms_per_step": ms, "base_ms_per_step": ms_b,
                          "weight_bytes": int(sum(l["m"] * l["n"] + 4 * l["n"] for l in layers)),
                          "stages_ms_per_step": {k: v[0] / 3 for k, v in xq_stages.items() if v[1]},
                          "note": "int8 per-row weights, dequantized into one shared scratch before each use"}
        for l, W in zip(layers, saved_W):
            l["L"].Wq = None
            l["L"].W = W
        del scratch
        # the merge of all linears of the block (it resets q and G, so it runs last)
        merge_block = time_merges(cfg, [l["L"] for l in layers], device, stream)
    device_error = px.poetx_device_error()

    peaks, peak_src = measured_peaks()
    ms_step = ms_total / args.steps
    flops_step = cfg.flops_per_step()
    w0_ms, w0_launches = stages["w0_gemm"]
    w0_flops = cfg.gemm_flops_per_step() * args.steps  # 2Tmn forward + 2Tmn backward per linear
    peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    shape, dom_layers, dom_ms = dominant_w0(cfg, records)
    dom_flops = 2.0 * cfg.T * shape[0] * shape[1]
    achieved = dom_flops / (statistics.mean(dom_ms) / 1e3) / 1e12 if dom_ms else None
    total_launches = int(sum(c for _, c in stages.values()))
    tflops = flops_step / (ms_step / 1e3) / 1e12
    res = {
        "metric": METRIC,
        "value": world * cfg.T * args.steps / (ms_total / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded normal activations and gradients; random-init N(0,0.02^2) weights)",
        "config": config_block(cfg, world),
        "evaluation": "input-centric (every block product on token rows; no transformed weight formed)",
        "tflops_per_gpu": tflops,
        "pct_bf16_peak": 100.0 * tflops / NOMINAL_BF16_TFLOPS,
        "pct_bf16_peak_of": f"nominal B200 dense bf16 peak, {NOMINAL_BF16_TFLOPS:.0f} TFLOP/s",
        "pct_bf16_peak_measured": {"burst": 100.0 * tflops / peak_burst, "sustained": 100.0 * tflops / peak_sus,
                                   "source": f"{peak_src} bf16_tflops / bf16_tflops_sustained (cuBLAS GEMM)"},
        "roofline": {"kernel": f"w0_gemm forward, M={cfg.T} N={shape[1]} K={shape[0]} "
                               f"(layers {[cfg.layers[i][0] for i in dom_layers]})",
                     "bound": "tensor", "achieved": achieved,
                     "peak": peak_sus, "unit": "TFLOP/s",
                     "frac": (achieved / peak_sus) if achieved else None,
                     "traffic": W0_GEMM_TRAFFIC_BYTES if (cfg.name, cfg.T) == ("block8b", 16384) else None,
                     "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)",
                     "frac_of_burst": (achieved / peak_burst) if achieved else None,
                     "frac_of_nominal": (achieved / NOMINAL_BF16_TFLOPS) if achieved else None,
                     "launches": len(dom_ms),
                     "algorithmic_flops_per_launch": dom_flops,
                     "algorithmic_bytes_per_launch": 2.0 * (cfg.T * shape[0] + shape[0] * shape[1] + cfg.T * shape[1]),
                     "note": "achieved = 2*T*m*n per launch / mean CUDA-event launch time over the timed region; "
                             "traffic = DRAM bytes per launch of the same kernel and shape from an ncu capture; "
                             "frac divides by the measured sustained cuBLAS peak, frac_of_burst by the measured "
                             "burst peak, frac_of_nominal by the 2250 TFLOP/s datasheet figure"},
        "w0_stage": {"tflops": w0_flops / (w0_ms / 1e3) / 1e12 if w0_ms > 0 else None, "launches": w0_launches,
                     "note": "all forward and backward W0 GEMM launches of the step"},
        "stages_ms_per_step": {k: v[0] / args.steps for k, v in stages.items()},
        "profiled_ms_per_step": ms_profiled / args.steps,
        "gpu_launches": total_launches,
        "clocks": clocks,
        "e2e": e2e,
        "variants": variants,
        "merge": merge_block,
        "device_error": device_error,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, args.cpu_tokens)
        res["cpu_baseline_1core"] = cpu_baseline(cfg, args.cpu_tokens_1core, threads=1)
    for l in layers:
        del l["L"]
    del layers, flat
    if not args.no_configs and world == 1:
        torch.cuda.empty_cache()
        res["configs"] = {name: measure_layer_config(name, args, device, stream, peaks)
                          for name in ("attn3b", "up8b", "down13b")}
        res["configs"]["block8b"] = {"cnp": cnp_microbench(cfg, device, stream)}
        res["device_error"] = res["device_error"] | px.poetx_device_error()
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return res if rank == 0 else None


# ---------------------------------------------------------------- oracle (CPU) arm
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_step(cfg: pi.Config, inputs) -> None:
    import oracle
    for inp in inputs:
        W0 = inp.W0lin64.T
        GR = oracle.cnp_blocks(inp.qR, inp.b)
        GP = oracle.cnp_blocks(inp.qP, inp.b)
        oracle.forward(inp.x64, W0, inp.permR, GR, inp.permP, GP)
        oracle.layer_backward(inp.x64, W0, inp.permR, inp.qR, inp.permP, inp.qP, inp.b, inp.dz64)


def oracle_inputs(cfg: pi.Config, tokens: int):
    return [pi.layer_inputs(cfg, li, T=tokens) for li in range(len(cfg.layers))]


def cpu_baseline(cfg: pi.Config, tokens: int, threads: int | None = None) -> dict:
    """The oracle as it stands on the host cores (all BLAS threads, or
    `threads`), one step on a `tokens`-row sample of the workload."""
    inputs = oracle_inputs(cfg, tokens)
    if threads is not None:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(threads):
            t0 = time.perf_counter()
            oracle_step(cfg, inputs)
            dt = time.perf_counter() - t0
        cores = threads
    else:
        t0 = time.perf_counter()
        oracle_step(cfg, inputs)
        dt = time.perf_counter() - t0
        cores = blas_threads()
    return {"value": tokens / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{tokens} of {cfg.T} tokens through all {len(cfg.layers)} linears (forward, backward, "
                      f"CNP build and backward, float64), one step, {dt:.1f} s"}


def bench_reference(args, cfg: pi.Config) -> dict:
    rank, world, _ = dist_env()
    if rank != 0:
        return None
    tokens = args.ref_tokens
    inputs = oracle_inputs(cfg, tokens)
    for _ in range(args.warmup):
        oracle_step(cfg, inputs)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(cfg, inputs)
    dt = time.perf_counter() - t0
    value = tokens * args.steps / dt
    sample = (f"{tokens} of {cfg.T} tokens per step through all {len(cfg.layers)} linears (forward, backward, "
              f"CNP build and backward, float64)")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, poetx_inputs recipe)", "config": config_block(cfg, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["poetx", "reference"], default="poetx")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(pi.CONFIGS))
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's tokens per GPU (smaller cases for profiler captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the folded / mem / xq / optimizer-step timings and the merge")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the single-layer workloads (attn3b, up8b, down13b) and the CNP microbenchmarks")
    ap.add_argument("--cpu-tokens", type=int, default=512, help="token sample of the CPU-baseline leg")
    ap.add_argument("--cpu-tokens-1core", type=int, default=64, help="token sample of the one-core CPU baseline")
    ap.add_argument("--ref-tokens", type=int, default=64, help="token sample per step of --impl reference")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = pi.CONFIGS[args.workload]
    if args.tokens is not None:
        import dataclasses
        cfg = dataclasses.replace(cfg, T=args.tokens)
    res = bench_reference(args, cfg) if args.impl == "reference" else bench_poetx(args, cfg)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
