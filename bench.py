#!/usr/bin/env python3
"""Benchmark of the windowed atom attention forward pass on B200.

One step = one forward pass of the whole block (usability + conditioning, projections,
slot-gathered attention, transition, encoder pooling / decoder readout) over one
synthetic batch, through the C ABI. Prints ONE JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the float64 CPU oracle on the host cores

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own seeded batch
(independent problems, no collective on the data path: weak scaling); timing is the
max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_windowed_atom_b200 import workloads  # noqa: E402

DEFAULT_WORKLOAD = "esm_encoder_bf16_b2_a32768"
METRIC = "atom-encoder atoms/s and attention entries/s (A·H·K); % of HBM roofline"
FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0            # burst
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0  # seconds-long loop under the power cap


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["atomenc", "reference"], default="atomenc")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=workloads.WORKLOAD_ORDER)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="host seconds for the oracle baseline sample")
    p.add_argument("--op", choices=["block", "single_to_pair"], default="block",
                   help="block: the atom attention block (default); single_to_pair: the pair "
                        "feature pass, B=1 N=384 C=128 2H=64 D=128 with output_norm")
    return p.parse_args()


# ----------------------------------------------------------------------------- helpers

def attention_bytes(spec: workloads.WorkloadSpec) -> int:
    """Algorithmic HBM bytes of one slot-attention launch: key_index (int64) and
    window_mask read once per slot, AF3 pair rows (storage type) once per slot, the
    usable flag once per atom, Q, K, V and value-gate logits read once per atom and the
    gated output written once per atom (storage type), the attention weights written
    once (storage type)."""
    s = 2 if spec.dtype == "bfloat16" else 4
    slots = spec.B * spec.A * spec.K
    hd = spec.H * spec.D
    b = slots * (8 + 1)
    if spec.style == "af3":
        b += slots * spec.P * s
    b += spec.B * spec.A * (1 + 5 * hd * s)
    b += spec.B * spec.H * spec.A * spec.K * s
    return b


def dense_flops(spec: workloads.WorkloadSpec) -> int:
    """Algorithmic flops of the dense projections of one forward (2 per multiply-add):
    conditioning (AF3: 3 scale + 3 shift + 2 gate blocks of C columns; ESMFold2: the six
    w_mod blocks), Q/K/V/value gate, attention out-projection, SwiGLU gate/up and
    w_ff_out, and the encoder's pooling projection or the decoder's token projection
    (per token) and readout."""
    C, S, HD, M, U, V = spec.C, spec.S, spec.H * spec.D, spec.M, spec.U, spec.V
    per_atom = 2 * S * (8 * C if spec.style == "af3" else 6 * C)
    per_atom += 2 * C * 4 * HD + 2 * HD * C + 2 * C * 2 * M + 2 * M * C
    per_atom += 2 * C * U if spec.stage == "encoder" else 2 * C * 3
    total = per_atom * spec.B * spec.A
    if spec.stage == "decoder":
        total += 2 * V * C * spec.B * spec.T
    return total


def storage_dtype(spec) -> str:
    return "bf16" if spec.dtype == "bfloat16" else "f32"


def config_of(spec, world):
    return {
        "workload": spec.name, "description": spec.description, "style": spec.style,
        "stage": spec.stage, "storage": "bf16" if spec.dtype == "bfloat16" else "fp32",
        "B": spec.B, "A": spec.A, "T": spec.T, "K": spec.K, "C": spec.C, "S": spec.S,
        "H": spec.H, "D": spec.D, "P": spec.P, "M": spec.M, "U": spec.U, "V": spec.V,
        "radius": spec.radius, "atoms_per_step": spec.atoms * world,
        "entries_per_step": spec.entries * world,
        "l2": f"flushed before every timed step ({FLUSH_BYTES >> 20} MiB write)",
        "parallelism": f"replicas x{world} (independent batches per GPU)",
    }


def load_peaks():
    """(hbm GB/s, bf16 TFLOP/s sustained, source) from MEASURED_PEAKS.json, else the
    fallbacks measured earlier on this machine."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        hbm = float(pk["hbm_gbs"])
        tf = pk.get("bf16_tflops_sustained", pk.get("bf16_tflops"))
        tf = float(tf) if tf is not None else FALLBACK_BF16_TFLOPS_SUSTAINED
        return hbm, tf, "measured (MEASURED_PEAKS.json: hbm_gbs STREAM-style copy, bf16_tflops_sustained cuBLAS loop)"
    except Exception:
        return (FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS_SUSTAINED,
                "fallback (6.65 TB/s and 1.4 PFLOP/s sustained, earlier measurements on this pool)")


def attention_kernel(spec) -> str:
    """The attention kernel the library launches for this shape: the row-gather kernel
    for bf16 storage (float32: problems of at most 1024 atoms) when H*D = 128, a head
    spans a whole number of 16-channel lane groups (D a multiple of 16, at most 8
    heads), K <= 128 and (AF3) P <= 32; the per-(query, head) kernel otherwise (the same
    rule as the workspace plan of the C library)."""
    hd = spec.H * spec.D
    lc = hd // 8
    rg = ((spec.dtype == "bfloat16" or spec.B * spec.A <= 1024) and hd == 128 and spec.D >= lc and spec.D % lc == 0
          and hd // spec.D <= 8 and spec.K <= 128 and (spec.style != "af3" or spec.P <= 32))
    return "k_attn_rows" if rg else "k_slot_attention"


KERNEL_SOURCES = {"k_attn_rows": ("attn_rows.cuh", "common.cuh"),
                  "k_slot_attention": ("attention.cuh", "common.cuh")}


def kernel_source_sha(kernel: str = "k_attn_rows") -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "sparse_windowed_atom_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str = "k_attn_rows"):
    """DRAM bytes per attention launch from a committed ncu summary, if it was taken on
    the current source of that kernel for this workload; else None."""
    path = os.path.join(ROOT, "profiles", f"traffic_{kernel}.txt")
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha(kernel)
    with open(path) as f:
        for line in f:
            if line.startswith("#") or "=" not in line:
                continue
            kv = dict(x.split("=", 1) for x in line.split())
            if kv.get("workload") == workload and kv.get("source_sha") == sha:
                return int(kv["dram_bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_uuid: str | None):
        self.samples = []
        self.t0 = self.t1 = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if device_uuid:
            cmd[1:1] = ["-i", device_uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.samples.append((time.monotonic(), parts))

    def start(self):
        self.t0 = time.monotonic()

    def stop(self):
        self.t1 = time.monotonic()
        time.sleep(0.25)
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        inside = [p for t, p in self.samples if self.t0 - 0.15 <= t <= self.t1 + 0.15]
        note = "timed region"
        if not inside:
            # a timed region shorter than the sampling period: take the nearest samples
            inside = [p for t, p in sorted(self.samples, key=lambda s: abs(s[0] - self.t1))[:3]]
            note = "nearest samples (timed region shorter than the 100 ms sampling period)"

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[0]) for p in inside if num(p[0]) is not None]
        mx = [num(p[1]) for p in inside if num(p[1]) is not None]
        reasons = set()
        for p in inside:
            for name, val in zip(self.NAMES, p[4:8]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(inside), "window": note}


# ----------------------------------------------------------------------------- CPU oracle

def oracle_rate(spec, budget_s: float, seed: int = 0, threads: str = "all"):
    """Time the float64 oracle (as it stands) on a bounded sample of the workload:
    batch element 0, the first n query atoms (n doubled until the budget is used),
    repeated until budget_s. threads="all" runs the OpenMP build of the same source on
    every host core, "one" the one-thread build. Returns (atoms/s, sample, seconds,
    threads used)."""
    import oracle
    w = workloads.make_inputs(spec.replace(B=1), seed=seed)
    f64 = lambda d: {k: v.astype(np.float64) for k, v in d.items()}
    act, prm = f64(w["activations"]), f64(w["parameters"])
    n = min(spec.A, 1024)
    done, spent, passes = 0, 0.0, 0
    while spent < budget_s:
        sel = np.zeros((1, spec.A), bool)
        sel[0, :n] = True
        t = time.perf_counter()
        oracle.windowed_atom_attention(act, prm, w["masks"], w["structure"], eps=spec.eps,
                                       style=spec.style, stage=spec.stage, radius=spec.radius,
                                       query_select=None if n == spec.A else sel,
                                       threads=threads)
        dt = time.perf_counter() - t
        spent += dt
        done += n
        passes += 1
        if dt < budget_s / 6 and n < spec.A:
            n = min(spec.A, n * 2)
    cores = oracle.threads_used(threads)
    sample = (f"batch element 0 of {spec.name}: {passes} oracle passes over the first "
              f"<= {n} of {spec.A} query atoms ({done} atoms total), {cores} host thread(s)")
    return done / spent, sample, spent, cores


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    spec = workloads.WORKLOADS[args.workload]
    steps, warm = args.steps, args.warmup
    per_step = max(0.5, min(8.0, 150.0 / max(1, steps + warm)))
    for _ in range(warm):
        oracle_rate(spec, per_step / 4)
    total_atoms, total_s, sample, cores = 0.0, 0.0, "", 1
    for _ in range(steps):
        r, sample, s, cores = oracle_rate(spec, per_step)
        total_atoms += r * s
        total_s += s
    rate = total_atoms / total_s
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "atoms/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warm, "ms_per_step": 1e3 * total_s / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": config_of(spec, 1),
        "entries_per_s": rate * spec.H * spec.K,
        "cpu_baseline": {"value": rate, "unit": "atoms/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {sample}"},
        "e2e": {"value": rate, "unit": "atoms/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- ranks

class Ranks:
    """One process per GPU (torchrun env: RANK, LOCAL_RANK, WORLD_SIZE, MASTER_*).
    Every rank runs its own replica of the workload on its own seeded batch; the only
    collectives are the barrier around the timed region and the max over ranks of the
    device time (no collective on the data path)."""

    def __init__(self, backend: str = "nccl", device=None, timeout_s: int = 120):
        import torch
        import torch.distributed as dist
        self.dist, self.torch = dist, torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device if device is not None else torch.device("cpu")
        if self.world > 1:
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)

    def seed(self) -> int:
        return self.rank

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, x: float) -> float:
        if self.world == 1:
            return x
        t = self.torch.tensor([x], dtype=self.torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def job_rate(self, units_per_rank: float, ms_per_step: float) -> float:
        """Whole-job throughput: the units every rank processed per step over the
        slowest rank's time per step."""
        return units_per_rank * self.world / (ms_per_step / 1e3)

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


# ----------------------------------------------------------------------------- GPU arm

def run_atomenc(args):
    import torch

    from sparse_windowed_atom_b200 import atomenc

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU path exists)")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    barrier, max_over_ranks = ranks.barrier, ranks.max

    spec = workloads.WORKLOADS[args.workload]
    w = workloads.make_inputs(spec, seed=ranks.seed())
    fdt = torch.bfloat16 if spec.dtype == "bfloat16" else torch.float32
    host = {}
    for grp in ("activations", "parameters"):
        for k, v in w[grp].items():
            host[k] = torch.from_numpy(np.ascontiguousarray(v)).to(fdt)
    for grp in ("masks", "structure"):
        for k, v in w[grp].items():
            host[k] = torch.from_numpy(np.ascontiguousarray(v))
    pnames = set(w["parameters"])
    devt = {k: v.to(dev) for k, v in host.items()}
    inputs = {k: v for k, v in devt.items() if k not in pnames}
    params = {k: v for k, v in devt.items() if k in pnames}
    outs = {k: torch.empty(s, dtype=fdt, device=dev)
            for k, s in atomenc.output_shapes(spec.style, spec.stage, inputs, params).items()}
    ws = torch.empty(atomenc.atomenc_workspace_size(spec.style, spec.stage, inputs, params, outs),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    nph = atomenc.NUM_PHASES + 1
    K, W = args.steps, args.warmup

    def make_events(n):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nph)] for _ in range(n)]
        for row in evs:
            for e in row:
                e.record(stream)
        return evs

    def fwd(evrow):
        return atomenc.atomenc_forward_profiled(spec.style, spec.stage, inputs, params, spec.eps,
                                                spec.radius, outs, ws, evrow, stream)

    fwd_plain = atomenc.Forward(spec.style, spec.stage, inputs, params, spec.eps, spec.radius,
                                outs, ws, stream)

    warm_ev = make_events(1)[0]
    per_step_launches = 0
    for _ in range(W):
        flush.zero_()
        per_step_launches = fwd(warm_ev)
    evs = make_events(K)
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    torch.cuda.synchronize(dev)
    status = atomenc.atomenc_get_status(ws, stream)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    time.sleep(0.3)
    # ---- the timed steps: one forward per step through the C ABI, events only around it
    # (kernels of a step follow each other with programmatic dependent launch)
    barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    host_s = 0.0
    for i in range(K):
        flush.zero_()
        step_ev[i][0].record(stream)
        h0 = time.perf_counter()
        fwd_plain()
        host_s += time.perf_counter() - h0
        step_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    sampler.stop()
    launches = per_step_launches * K

    # ---- prepared weights: the same steps through atomenc_forward_prepared with the weight
    # images built once beforehand (outside the timed steps; the headline value above
    # rebuilds them inside every step)
    image = atomenc.atomenc_prepare_weights(spec.style, spec.stage, inputs, params, outs,
                                            stream=stream)
    ws_p = torch.empty(atomenc.atomenc_prepared_workspace_size(spec.style, spec.stage, inputs,
                                                               params, outs),
                       dtype=torch.uint8, device=dev)
    fwd_prep = atomenc.Forward(spec.style, spec.stage, inputs, params, spec.eps, spec.radius,
                               outs, ws_p, stream, image=image)
    for _ in range(W):
        flush.zero_()
        fwd_prep()
    prep_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        flush.zero_()
        prep_ev[i][0].record(stream)
        fwd_prep()
        prep_ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    prep_status = atomenc.atomenc_get_status(ws_p, stream)
    prep_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in prep_ev)) / K

    # ---- phase pass: the same steps again with an event at every phase boundary (these
    # events serialise the phases); gives the breakdown and the attention kernel's time
    barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        flush.zero_()
        fwd(evs[i])
    torch.cuda.synchronize(dev)
    barrier()

    # ---- traced pass: the same steps again with an event after every kernel (these
    # events serialise the kernels); gives each kernel's own device time
    nk = atomenc.MAX_LAUNCHES + 1
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk)] for _ in range(K)]
    for row in kev:
        for e in row:
            e.record(stream)
    barrier()
    torch.cuda.synchronize(dev)
    kinds = []
    for i in range(K):
        flush.zero_()
        kinds = atomenc.atomenc_forward_traced(spec.style, spec.stage, inputs, params, spec.eps,
                                               spec.radius, outs, ws, kev[i], stream)
    torch.cuda.synchronize(dev)
    barrier()
    kernel_ms = [statistics.fmean(kev[i][j].elapsed_time(kev[i][j + 1]) for i in range(K))
                 for j in range(len(kinds))]
    by_kind = {}
    for kd, t in zip(kinds, kernel_ms):
        by_kind[kd] = by_kind.get(kd, 0.0) + t

    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    phase_ms = [statistics.fmean(evs[i][p].elapsed_time(evs[i][p + 1]) for i in range(K))
                for p in range(atomenc.NUM_PHASES)]
    phased_step_ms = statistics.fmean(evs[i][0].elapsed_time(evs[i][nph - 1]) for i in range(K))
    total_ms = max_over_ranks(sum(step_ms))
    ms_per_step = total_ms / K
    atoms = spec.atoms * world
    value = ranks.job_rate(spec.atoms, ms_per_step)

    # ---- roofline of the attention kernel (its own device time, traced pass)
    attn_ms = max_over_ranks(by_kind.get("attention", phase_ms[3]))
    hbm_peak, tc_peak, peak_src = load_peaks()
    abytes = attention_bytes(spec)
    achieved = abytes / (attn_ms / 1e3) / 1e9
    dominant = max(range(atomenc.NUM_PHASES), key=lambda p: phase_ms[p])
    akernel = attention_kernel(spec)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": recorded_traffic(spec.name, akernel),
                "kernel": akernel, "bytes_per_launch": abytes,
                "avg_launch_ms": attn_ms, "peak_source": peak_src,
                "frac_of_8TBs": achieved / 8000.0}
    # ---- the dense projections on the tensor cores: algorithmic flops over the summed
    # device time of the tcgen05 kernels (projection GEMMs and the fused tail)
    tc_ms = max_over_ranks(by_kind.get("gemm", 0.0) + by_kind.get("transition", 0.0))
    flops = dense_flops(spec)
    tc_ach = flops / (tc_ms / 1e3) / 1e12 if tc_ms > 0 else 0.0
    roofline_tc = {"bound": "tensor", "achieved": tc_ach, "peak": tc_peak, "unit": "TFLOP/s",
                   "frac": tc_ach / tc_peak, "traffic": None,
                   "kernels": "k_gemm_rows + k_transition (tcgen05)",
                   "flops_per_step": flops, "ms_per_step": tc_ms, "peak_source": peak_src,
                   "products": ("three bf16 tcgen05 products per float32 product (hi*hi + hi*lo "
                                "+ lo*hi); the flops counted are the algorithmic ones"
                                if spec.dtype == "float32" else
                                "bf16 operands, float32 accumulation")}

    # ---- end to end: pinned host inputs -> device, forward, outputs -> pinned host, every
    # step through the public API. Two buffer sets and three streams: the host->device
    # copies of step i+1 and the device->host copies of step i-1 overlap the forward of
    # step i (each copy and forward waits for the events that make its buffers free).
    e2e = None
    if not args.no_e2e:
        # every input in one pinned host buffer and every output in one device buffer (each
        # tensor at a 256-byte aligned offset), so a step is one copy in and one copy out
        def packed(shapes, device, pin=False):
            offs, cur = {}, 0
            for k, (shape, dtype) in shapes.items():
                offs[k] = cur
                n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
                cur += (n + 255) // 256 * 256
            buf = torch.empty(cur, dtype=torch.uint8, device=device, pin_memory=pin)
            views = {}
            for k, (shape, dtype) in shapes.items():
                n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
                views[k] = buf[offs[k]:offs[k] + n].view(dtype).view(shape)
            return buf, views

        in_shapes = {k: (tuple(v.shape), v.dtype) for k, v in host.items()}
        out_shapes = {k: (tuple(v.shape), v.dtype) for k, v in outs.items()}
        hin_buf, hin = packed(in_shapes, "cpu", pin=True)
        for k, v in host.items():
            hin[k].copy_(v)
        h2d = hin_buf.numel()
        ke = max(4, min(K, 20))
        s_in, s_out, comp = torch.cuda.Stream(dev), torch.cuda.Stream(dev), stream
        sets = []
        for _ in range(2):
            din_buf, dt = packed(in_shapes, dev)
            dout_buf, do = packed(out_shapes, dev)
            fwd_b = atomenc.Forward(spec.style, spec.stage,
                                    {k: v for k, v in dt.items() if k not in pnames},
                                    {k: v for k, v in dt.items() if k in pnames},
                                    spec.eps, spec.radius, do, torch.empty_like(ws), comp)
            sets.append({"din": din_buf, "dout": dout_buf, "fwd": fwd_b,
                         "hout": torch.empty(dout_buf.numel(), dtype=torch.uint8, pin_memory=True),
                         "copied_in": torch.cuda.Event(), "computed": torch.cuda.Event(),
                         "copied_out": torch.cuda.Event(), "used": False})
        d2h = sets[0]["dout"].numel()

        def e2e_step(i):
            S = sets[i % 2]
            with torch.cuda.stream(s_in):
                if S["used"]:
                    s_in.wait_event(S["computed"])        # its inputs were consumed
                S["din"].copy_(hin_buf, non_blocking=True)
                S["copied_in"].record(s_in)
            comp.wait_event(S["copied_in"])
            if S["used"]:
                comp.wait_event(S["copied_out"])          # its outputs were read back
            S["fwd"]()
            S["computed"].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(S["computed"])
                S["hout"].copy_(S["dout"], non_blocking=True)
                S["copied_out"].record(s_out)
            S["used"] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(ke):
            e2e_step(i)
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1)) / ke
        e2e = {"value": ranks.job_rate(spec.atoms, e_ms), "unit": "atoms/s", "h2d_bytes_per_step": h2d * world,
               "d2h_bytes_per_step": d2h * world, "ms_per_step": e_ms, "steps": ke,
               "pipeline": "inputs packed in one pinned buffer, outputs in one device buffer (one copy each way per step); two buffer sets, so the copies of neighbouring steps overlap the forward"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, sample, spent, cores = oracle_rate(spec, args.cpu_seconds, threads="all")
        rate1, sample1, spent1, _ = oracle_rate(spec, max(2.0, args.cpu_seconds / 3), threads="one")
        cpu = {"value": rate, "unit": "atoms/s", "cores": cores, "kind": "oracle", "sample": sample,
               "seconds": spent, "one_core": {"value": rate1, "cores": 1, "sample": sample1,
                                              "seconds": spent1}}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "atoms/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": storage_dtype(spec),
            "data": "synthetic (seeded workload generator; no dataset)",
            "config": config_of(spec, world),
            "entries_per_s": ranks.job_rate(spec.entries, ms_per_step),
            "roofline": roofline, "roofline_projections": roofline_tc,
            "cpu_baseline": cpu, "e2e": e2e,
            "kernel_ms": {k: v for k, v in sorted(by_kind.items())},
            "kernel_launches": kinds,
            "launch_ms": kernel_ms,
            "gpu_launches": launches,
            "clocks": sampler.summary(),
            "phase_ms": dict(zip(atomenc.PHASES, phase_ms)),
            "phase_pass_ms_per_step": phased_step_ms,
            "host_us_per_call": 1e6 * host_s / K,
            "dominant_phase": atomenc.PHASES[dominant],
            "device_status": status,
            "prepared_weights": {
                "value": ranks.job_rate(spec.atoms, prep_ms), "unit": "atoms/s",
                "ms_per_step": prep_ms, "device_status": prep_status,
                "note": ("atomenc_forward_prepared: weight images built once by "
                         "atomenc_prepare_weights outside the timed steps; every other step "
                         "of the pass inside them"),
            },
        }
        print(json.dumps(line), flush=True)
    ranks.close()
    return 0


def run_single_to_pair(args):
    """Pair features of one N=384 chain (synthetic, seeded): pairs/s of device time, and the
    pass's HBM roofline (x read once; pair_features and output written once)."""
    import torch
    from sparse_windowed_atom_b200 import atomenc
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU path exists)")
    dev = torch.device("cuda", 0)
    B, N, C, H, Dp = 1, 384, 128, 32, 128
    rng = np.random.default_rng(0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device=dev, dtype=torch.float32)
    act = {"x": t(rng.normal(size=(B, N, C)))}
    prm = {"weight": t(rng.normal(size=(C, 2 * H)) / np.sqrt(C)), "bias": t(0.1 * rng.normal(size=2 * H)),
           "norm_scale": t(1 + 0.1 * rng.normal(size=C)), "norm_bias": t(0.1 * rng.normal(size=C)),
           "out_weight": t(rng.normal(size=(2 * H, Dp)) / np.sqrt(2 * H)), "out_bias": t(0.1 * rng.normal(size=Dp)),
           "output_scale": t(1 + 0.1 * rng.normal(size=Dp)), "output_bias": t(0.1 * rng.normal(size=Dp))}
    msk = {"mask": torch.from_numpy(rng.random((B, N)) < 0.95).to(dev)}
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    ws = None
    for _ in range(args.warmup):
        flush.zero_()
        pf, out = atomenc.single_to_pair(act, prm, msk, eps=1e-5, output_norm=True, workspace=ws)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record()
        atomenc.single_to_pair(act, prm, msk, eps=1e-5, output_norm=True, workspace=ws)
        evs[i][1].record()
    torch.cuda.synchronize()
    ms = statistics.fmean(a.elapsed_time(b) for a, b in evs)
    nbytes = B * N * C * 4 + B * N * N * (2 * H + Dp) * 4
    peak, _, src = load_peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    print(json.dumps({"op": "single_to_pair", "metric": "pair features: token pairs/s", "unit": "pairs/s",
                      "value": B * N * N / (ms / 1e3), "ms_per_step": ms, "steps": args.steps,
                      "warmup": args.warmup, "dtype": "f32", "data": "synthetic (seeded)",
                      "config": {"B": B, "N": N, "C": C, "2H": 2 * H, "D": Dp, "output_norm": True,
                                 "l2": f"flushed before every timed step ({FLUSH_BYTES >> 20} MiB write)"},
                      "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                                   "frac": achieved / peak, "bytes_per_step": nbytes, "peak_source": src},
                      "higher_is_better": True}), flush=True)
    return 0


def main():
    args = parse_args()
    if args.op == "single_to_pair":
        return run_single_to_pair(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_atomenc(args)


if __name__ == "__main__":
    sys.exit(main())
