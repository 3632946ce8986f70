"""Decode state-update throughput of DeltaLog on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--L 16] [--merge fused|separate]
                    [--impl ours|reference] [--sweep]

Workload: GDN decode, B=512 sequences, H=32 heads, d_k=d_v=128, fp32 state
(1 GiB), bf16 q/k/v, ragged batch whose sequences start at log fill offsets
U{0..L-1} (so merges are staggered), L=16.  One step = one decode step of the
whole batch (one layer, all heads) including the merges it triggers; the
timed loop cycles a device ring of 16 pre-drawn steps.  tokens/s = B * K /
time.  The state (1 GiB) is far larger than L2 (126 MB), so no L2 flush is
needed between steps.

The JSON line also carries: the roofline of the dominant kernel (the step
kernel, HBM-bound: algorithmic bytes per launch / its mean CUDA-event
duration, against the measured copy bandwidth), the eager dense step kernel
timed the same way, an end-to-end figure (host inputs in pinned memory
copied in and o copied out every step), the fp64 CPU oracle timed on a
bounded sample of the same workload, and SM clocks sampled during the timed
region.

With --gpus N > 1 (one process per GPU under torchrun) every rank decodes its
own B=512 batch (weak scaling, no data-path collective); the time is the
maximum over ranks and the value counts all ranks' tokens.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_attention_recurrent_deltalog_b200 import workloads as wl  # noqa: E402

METRIC = "decode state-update tokens/s (B=512,H=32,d=128); HBM GB/s vs 8 TB/s peak"
UNIT = "tokens/s"
RING = 16
HOLD_CYCLES = 1_000_000  # ~0.5 ms of GPU spin before a device-timed region starts


def hold_stream():
    """A short GPU spin queued just before a device-timed region's start
    event (and outside it): it holds the stream while the host queues the
    region's first launches, so the region times its launches back to back
    and not the host's latency to issue the first one after a synchronize
    (nvbench's blocking-kernel practice).  The end-to-end region, whose host
    copies belong to what it measures, does not use it.  Without torch's
    spin helper the region simply starts unheld (slightly conservative)."""
    sleep = getattr(torch.cuda, "_sleep", None)
    if sleep is not None:
        sleep(HOLD_CYCLES)
L2_BYTES = 126 * 2**20
FALLBACK_HBM_GBS = 6650.0

# Sources of each kernel: a DRAM traffic figure taken by ncu (a JSON record
# under profiles/) is reported only while the sources it was taken from are
# unchanged.
_CSRC = "linear_attention_recurrent_deltalog_b200/csrc/"
KERNEL_SOURCES = {
    "dl_step_kernel": ("dl_device.cuh", "dl_common.cuh", "dl_q8.cuh", "dl_step.cuh"),
    "dl_merge_kernel": ("dl_device.cuh", "dl_common.cuh", "dl_q8.cuh", "dl_merge.cuh"),
    "dl_merge_q8_kernel": ("dl_device.cuh", "dl_common.cuh", "dl_q8.cuh", "dl_tmem.cuh",
                           "dl_fold_tmem.cuh", "dl_merge.cuh"),
    "dl_eager_kernel": ("dl_device.cuh", "dl_common.cuh", "dl_eager.cuh"),
}


def kernel_hash(kernel: str = "dl_step_kernel") -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, _CSRC, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, **match):
    """The committed ncu traffic record of `kernel` for this workload (every
    key in `match` equal), taken from the current sources; None if there is
    none."""
    import glob
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*traffic*.json"))):
        try:
            with open(path) as f:
                t = json.load(f)
        except Exception:
            continue
        if not str(t.get("kernel", "")).startswith(kernel):
            continue
        if t.get("kernel_hash") != kernel_hash(kernel):
            continue
        if all(t.get(k, "f32" if k == "base" else None) == v for k, v in match.items()):
            return t
    return None


def mean_dram(t, key):
    """Mean per-launch DRAM bytes (`dram_read` or `dram_write`) of a record."""
    xs = [float(x[key]) for x in t.get("launches", [])]
    return sum(xs) / len(xs) if xs else None


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------ distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = os.environ.get("DL_BENCH_BACKEND", "nccl")
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def world_plan(gpus: int, env) -> str:
    """How this process takes part in a run of ``--gpus gpus``: "run" when it
    is one of the ranks (a launcher set WORLD_SIZE = gpus, or gpus is 1),
    "spawn" when --gpus N > 1 arrives without a launcher (this process then
    starts the N local ranks itself).  A WORLD_SIZE that disagrees with
    --gpus is an error."""
    if gpus < 1:
        raise SystemExit(f"bench.py: --gpus must be >= 1 (got {gpus})")
    ws = env.get("WORLD_SIZE")
    if ws is None:
        return "run" if gpus == 1 else "spawn"
    if int(ws) != gpus:
        raise SystemExit(f"bench.py: --gpus {gpus} but the launcher started WORLD_SIZE={ws} ranks")
    return "run"


def spawn_command(gpus: int, argv, port: int) -> list:
    """torch.distributed.run over ``gpus`` local ranks (one per GPU) re-running
    this script with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """Maximum of a host float over all ranks (the bench's timing rule)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(tokens_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / max_seconds


# ------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU during a region.

    NVML is read from a background thread every ~2 ms, plus once when the
    region opens and once when it closes, so even a region of a few
    milliseconds carries several samples (nvidia-smi's 100 ms loop is the
    fallback when NVML cannot be opened)."""

    REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
                   ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_s: float = 0.002):
        self.gpu = gpu_index
        self.period = period_s
        self.rows = []          # (sm_mhz, max_mhz, power_w, reason names)
        self.nvml = None
        self.handle = None
        self.thread = None
        self.stop = None
        self.proc = None
        self.path = None

    def _open_nvml(self):
        import pynvml
        pynvml.nvmlInit()
        h = None
        try:  # the CUDA device's own GPU, whatever CUDA_VISIBLE_DEVICES says
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            h = None
        if h is None:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        self.nvml, self.handle = pynvml, h

    def _sample(self):
        n, h = self.nvml, self.handle
        sm = float(n.nvmlDeviceGetClockInfo(h, n.NVML_CLOCK_SM))
        mx = float(n.nvmlDeviceGetMaxClockInfo(h, n.NVML_CLOCK_SM))
        try:
            pw = n.nvmlDeviceGetPowerUsage(h) / 1000.0
        except Exception:
            pw = None
        try:
            bits = int(n.nvmlDeviceGetCurrentClocksEventReasons(h))
        except Exception:
            bits = int(n.nvmlDeviceGetCurrentClocksThrottleReasons(h))
        self.rows.append((sm, mx, pw, [name for name, b in self.REASON_BITS if bits & b]))

    def _loop(self):
        while not self.stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            self.stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            self._open_nvml()
            self._sample()
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.nvml = None
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.nvml is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            try:
                self._sample()
            except Exception:
                pass
            return
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                        names = [nm for i, (nm, _) in enumerate(self.REASON_BITS)
                                 if parts[5 + i].lower() in ("active", "1")]
                        self.rows.append((float(parts[1]), float(parts[2]) if parts[2].replace(".", "").isdigit()
                                          else None, None, names))
            os.unlink(self.path)

    def summary(self):
        return summarize_clocks(self.rows, "nvml" if self.nvml is not None else
                                ("nvidia-smi" if self.proc is not None else None))


def summarize_clocks(rows, source):
    """The JSON line's `clocks` object from (sm_mhz, max_mhz, power_w, reasons) rows."""
    if source is None:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0,
                "source": source}
    sm = [r[0] for r in rows]
    mx = [r[1] for r in rows if r[1] is not None]
    pw = [r[2] for r in rows if r[2] is not None]
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
            "sm_mhz_min": min(sm), "reasons": sorted({n for r in rows for n in r[3]}),
            "samples": len(rows), "power_w_max": round(max(pw), 1) if pw else None, "source": source}


# ------------------------------------------------------------ byte model

def base_tile_bytes(cfg) -> int:
    """Bytes of one head's base: fp32 d_v x d_k, or int8 codes + fp32 row scales."""
    if getattr(cfg, "base", "f32") == "q8":
        return cfg.d_v * cfg.d_k + cfg.d_v * 4
    return cfg.d_v * cfg.d_k * 4


def step_bytes(cfg, fills: np.ndarray, fused: bool) -> tuple:
    """Algorithmic bytes one step-kernel launch must move (read, write).

    Per head with f log entries before the step (GDN, fp32 state):
      read : S_b (d_v*d_k*4) + q,k,v + decay,beta + fill + f log entries
      write: o (d_v*4) + fill + the appended entry, or (fused merge, f = L-1)
             the merged S_b instead of the entry.
    """
    ein = 2 if cfg.in_dtype == "bf16" else 4
    dk, dv, H = cfg.d_k, cfg.d_v, cfg.H
    gw = 1 if cfg.variant == "gdn" else dk
    uin = ein if cfg.variant == "rwkv6" else 4
    entry = dv * uin + dk * ein + gw * 4
    tile = base_tile_bytes(cfg)
    vec = (2 * dk + dv) * ein + (4 if cfg.variant == "gdn" else dk * 4)
    if cfg.variant == "gdn2":
        vec += dk * 4 + dv * 4            # erase gate b_t [d_k], write gate w_t [d_v]
    elif cfg.variant != "rwkv6":
        vec += 4                          # beta
    f = fills.astype(np.int64)
    merging = (f == cfg.L - 1) if fused else np.zeros_like(f, dtype=bool)
    rd = H * (tile + vec + 4 + f * entry)
    wr = H * (dv * 4 + 4 + np.where(merging, tile, entry))
    return int(rd.sum()), int(wr.sum())


def merge_bytes(cfg, fills_after_step: np.ndarray) -> tuple:
    """Algorithmic bytes of a separate merge launch (sequences with f == L)."""
    ein = 2 if cfg.in_dtype == "bf16" else 4
    dk, dv, H = cfg.d_k, cfg.d_v, cfg.H
    gw = 1 if cfg.variant == "gdn" else dk
    uin = ein if cfg.variant == "rwkv6" else 4
    entry = dv * uin + dk * ein + gw * 4
    tile = base_tile_bytes(cfg)
    n = int((fills_after_step == cfg.L).sum())
    allfill = fills_after_step.size * H * 4
    return allfill + n * H * (tile + cfg.L * entry), n * H * (tile + 4)


def eager_bytes(cfg) -> tuple:
    ein = 2 if cfg.in_dtype == "bf16" else 4
    dk, dv = cfg.d_k, cfg.d_v
    tile = dv * dk * 4
    vec = (2 * dk + dv) * ein + (4 if cfg.variant == "gdn" else dk * 4)
    if cfg.variant == "gdn2":
        vec += dk * 4 + dv * 4            # erase gate b_t [d_k], write gate w_t [d_v]
    elif cfg.variant != "rwkv6":
        vec += 4                          # beta
    return cfg.heads * (tile + vec), cfg.heads * (tile + dv * 4)


# ------------------------------------------------------------ our arm

def log_entry_bytes(cfg) -> int:
    ein = 2 if cfg.in_dtype == "bf16" else 4
    uin = ein if cfg.variant == "rwkv6" else 4
    gw = 1 if cfg.variant == "gdn" else cfg.d_k
    return cfg.d_v * uin + cfg.d_k * ein + gw * 4


def measure_merge_materialize(cfg, w, ring, bonus, S0, device, stream, peak, reps: int = 3):
    """Times dl_merge (every log full, all heads) and dl_materialize (logs
    half full) with CUDA events; algorithmic bytes per head: merge reads the
    tile and L entries and writes the tile; materialize reads the tile and f
    entries and writes the dense state to a separate buffer."""
    import dataclasses as dc

    from linear_attention_recurrent_deltalog_b200 import deltalog as dlb
    cm = dc.replace(cfg, fused_merge=False)
    st = dlb.DeltaLogState(cm, device=device)
    o = torch.empty(w.heads * w.d_v, dtype=torch.float32, device=device)
    tile = base_tile_bytes(cm)
    dense = w.d_v * w.d_k * 4
    entry = log_entry_bytes(cm)
    ms_merge = []
    for r in range(reps):
        st.reset(S0, [0] * w.B)
        for i in range(w.L):
            q, k, v, dec, beta, wg = ring[i % len(ring)]
            st.step(q, k, v, dec, beta, wg if wg is not None else bonus, o)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold_stream()
        a.record(stream)
        st.merge(dlb.DL_MERGE_FULL)
        b.record(stream)
        torch.cuda.synchronize(device)
        ms_merge.append(a.elapsed_time(b))
    mb = w.heads * (2 * tile + w.L * entry + 8)
    t_merge = sorted(ms_merge)[len(ms_merge) // 2] / 1e3
    st.reset(S0, [0] * w.B)
    half = w.L // 2
    for i in range(half):
        q, k, v, dec, beta, wg = ring[i % len(ring)]
        st.step(q, k, v, dec, beta, wg if wg is not None else bonus, o)
    out = torch.empty(w.heads * w.d_v * w.d_k, dtype=torch.float32, device=device)
    st.materialize(out)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hold_stream()
    a.record(stream)
    for _ in range(reps):
        st.materialize(out)
    b.record(stream)
    torch.cuda.synchronize(device)
    t_mat = a.elapsed_time(b) / reps / 1e3
    mtb = w.heads * (tile + dense + half * entry + 4)
    code, head = st.device_error()
    st.close()
    del out
    if code != 0:
        raise RuntimeError(f"device error {code} at head {head}")
    return ({"launch_ms": round(t_merge * 1e3, 4), "achieved_gbs": round(mb / t_merge / 1e9, 1),
             "frac": round(mb / t_merge / 1e9 / peak, 4), "heads": w.heads, "entries": w.L,
             "algorithmic_bytes": int(mb)},
            {"launch_ms": round(t_mat * 1e3, 4), "achieved_gbs": round(mtb / t_mat / 1e9, 1),
             "frac": round(mtb / t_mat / 1e9 / peak, 4), "heads": w.heads, "entries": half,
             "algorithmic_bytes": int(mtb)})


def workload_desc(w, merge: str, base: str = "f32") -> str:
    kla = f", KLA step size eps={w.kla_eps:g}" if w.kla_eps is not None else ""
    state = ("int8 base with fp32 row scales (requantized at each merge), fp32 log"
             if base == "q8" else "fp32 state")
    return (f"{w.variant.upper()} decode B={w.B} H={w.H} d_k={w.d_k} d_v={w.d_v} {state}, "
            f"{w.in_dtype} q/k/v, {'ragged fills, ' if w.ragged else ''}L={w.L}, merge={merge}{kla}")


def to_dev(s, device):
    def up(x):
        if x is None:
            return None
        if x.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device).view(torch.bfloat16).reshape(-1)
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device).reshape(-1)
    return (up(s.device_array("q")), up(s.device_array("k")), up(s.device_array("v")),
            up(s.decay), up(s.beta), up(s.wgate))


def run_ours(args, world, rank, local):
    from linear_attention_recurrent_deltalog_b200 import deltalog as dlb

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    fused = args.merge == "fused"
    w = wl.WORKLOADS[args.workload]
    w = w.replace(L=args.L or w.L, B=args.B or w.B,
                  kla_eps=args.kla_eps if args.kla_eps >= 0 else None)
    cfg = dlb.Config(w.variant, w.B, w.H, w.d_k, w.d_v, w.L, w.in_dtype, fused_merge=fused,
                     step_split=args.split, kla_eps=w.kla_eps,
                     base=args.base)
    stream = torch.cuda.current_stream(device)

    # inputs: a device ring of RING pre-drawn steps (the generator's recipe)
    workers = args.gen_workers
    if workers is None:  # share the host cores among the ranks of this node
        workers = max(0, min(16, ((os.cpu_count() or 1) - 1) // max(1, world)))
    host_steps = list(wl.StepStream(w, RING, workers=workers))
    ring = [to_dev(s, device) for s in host_steps]
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    S0 = (torch.randn(w.heads * w.d_v * w.d_k, generator=gen, device=device) * w.s0_std).contiguous()
    fill0 = wl.fill_offsets(w)

    bonus = (torch.from_numpy(wl.rwkv6_bonus(w)).to(device).reshape(-1)
             if w.variant == wl.RWKV6 else None)
    st = dlb.DeltaLogState(cfg, device=device)
    st.reset(S0, fill0.tolist())
    o = torch.empty(w.heads * w.d_v, dtype=torch.float32, device=device)

    def one_step(i, ev=None):
        q, k, v, dec, beta, wg = ring[i % RING]
        if ev is not None:
            ev[0].record(stream)
        st.step(q, k, v, dec, beta, wg if wg is not None else bonus, o)
        if ev is not None:
            ev[1].record(stream)
        if not fused:
            st.merge(dlb.DL_MERGE_FULL)

    for i in range(args.warmup):
        one_step(i)
    torch.cuda.synchronize(device)

    # algorithmic bytes of the timed steps, from the host fill mirror
    fills = np.array(st.fill(), dtype=np.int64)
    rd = wr = mrd = mwr = 0
    for i in range(args.steps):
        r_, w_ = step_bytes(cfg, fills, fused)
        rd, wr = rd + r_, wr + w_
        fills = fills + 1
        if not fused:
            a, b = merge_bytes(cfg, fills)
            mrd, mwr = mrd + a, mwr + b
        fills[fills == cfg.L] = 0

    # With the fused merge every launch in the timed region is the step
    # kernel, so the region's own events give its mean launch duration
    # (back-to-back launches; the gaps between them count against it).
    # Events around each launch would serialise the stream at every step and
    # cost 4-6 us per step on B200, so they are recorded only in the
    # separate mode, whose merge launches sit between the steps.
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)] if not fused else [None] * args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = dlb.dl_launch_count()
    dist_barrier(world)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clk:
        hold_stream()  # the host needs ~60 us to issue a step
        start.record(stream)
        for i in range(args.steps):
            one_step(args.warmup + i, evs[i])
        end.record(stream)
        torch.cuda.synchronize(device)
    dist_barrier(world)
    launches = dlb.dl_launch_count() - n0
    elapsed = start.elapsed_time(end) / 1e3
    step_kernel_s = (sum(a.elapsed_time(b) for a, b in evs) / 1e3) if not fused else elapsed
    code, head = st.device_error()
    if code != 0:
        raise RuntimeError(f"device error {code} at head {head}")
    max_elapsed = max_over_ranks(elapsed, world, device)
    state_mib = w.heads * base_tile_bytes(cfg) / 2**20
    tokens = w.B * args.steps
    value = aggregate_value(tokens, world, max_elapsed)

    peak, peak_kind = hbm_peak()
    step_avg = step_kernel_s / args.steps
    step_bytes_avg = (rd + wr) / args.steps
    achieved = step_bytes_avg / step_avg / 1e9
    rec = traffic_record("dl_step_kernel", workload=w.name, B=w.B, L=w.L, merge=args.merge,
                         base=args.base)
    traffic = rec.get("bytes_per_launch") if rec else None

    if args.only_step:
        st.close()
        return {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "only_step": True,
                "config": {"workload": w.name, "B": w.B, "L": w.L, "merge": args.merge, "split": args.split,
                           "base": args.base},
                "roofline": {"achieved": round(achieved, 1), "peak": peak,
                             "frac": round(achieved / peak, 4), "launch_ms": round(step_avg * 1e3, 5)}}

    # eager dense step on a separate 1 GiB state, same inputs
    S_e = S0.clone()
    for i in range(args.warmup):
        q, k, v, dec, beta, wg = ring[i % RING]
        dlb.dl_eager_step(cfg, S_e, q, k, v, dec, beta, wg if wg is not None else bonus, o)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hold_stream()
    e0.record(stream)
    for i in range(args.steps):
        q, k, v, dec, beta, wg = ring[i % RING]
        dlb.dl_eager_step(cfg, S_e, q, k, v, dec, beta, wg if wg is not None else bonus, o)
    e1.record(stream)
    torch.cuda.synchronize(device)
    eager_s = e0.elapsed_time(e1) / 1e3
    erd, ewr = eager_bytes(cfg)
    del S_e

    # The merge and materialize kernels on their own: a state whose sequences
    # all sit at the same phase, so that after L steps every log is full.
    merge_k, mat_k = measure_merge_materialize(cfg, w, ring, bonus, S0, device, stream, peak)

    # End to end through the public API: every step copies its inputs from
    # pinned host memory and its output o back to pinned host memory.  The
    # copies and the kernel run on three streams so step i's compute overlaps
    # step i+1's upload and step i-1's download (double-buffered device
    # inputs and outputs; a buffer is reused only after the step that last
    # used it has finished with it).
    # Each ring slot's inputs are packed into one pinned byte buffer (q, k, v,
    # decay, beta at 256-B aligned offsets) so a step uploads with one copy;
    # the typed views into the device buffers are built once.
    def _bytes(a):
        a = np.ascontiguousarray(a if a.dtype == np.uint16 else a.astype(np.float32))
        return a.view(np.uint8).reshape(-1)

    def _parts(s):
        ps = [s.device_array("q"), s.device_array("k"), s.device_array("v"), s.decay]
        if s.beta is not None:
            ps.append(s.beta)
        if s.wgate is not None:
            ps.append(s.wgate)
        return ps

    parts0 = [_bytes(x) for x in _parts(host_steps[0])]
    offs, total = [], 0
    for part in parts0:
        offs.append(total)
        total += (part.size + 255) // 256 * 256
    pinned = []
    for s in host_steps:
        buf = np.zeros(total, dtype=np.uint8)
        for off, part in zip(offs, _parts(s)):
            pb = _bytes(part)
            buf[off:off + pb.size] = pb
        pinned.append(torch.from_numpy(buf).pin_memory())
    NB = 2
    tin = cfg.torch_in_dtype
    dbufs, dviews = [], []
    for _ in range(NB):
        d = torch.empty(total, dtype=torch.uint8, device=device)
        dbufs.append(d)
        views = []
        for j, (off, part) in enumerate(zip(offs, parts0)):
            raw = d[off:off + part.size]
            views.append(raw.view(tin) if j < 3 else raw.view(torch.float32))
        while len(views) < 6:
            views.append(None)
        dviews.append(views)
    obufs = [torch.empty(o.numel(), dtype=torch.float32, device=device) for _ in range(NB)]
    o_hosts = [torch.empty(o.numel(), dtype=torch.float32).pin_memory() for _ in range(NB)]
    h2d = int(total)  # bytes of the one pinned buffer copied per step (incl. alignment padding)
    d2h = o_hosts[0].numel() * 4
    s_cmp = stream
    s_h2d = torch.cuda.Stream(device)
    s_d2h = torch.cuda.Stream(device)
    ev_h2d = [torch.cuda.Event() for _ in range(NB)]
    ev_cmp = [torch.cuda.Event() for _ in range(NB)]
    ev_d2h = [torch.cuda.Event() for _ in range(NB)]

    def e2e_step(i):
        b = i % NB
        s_h2d.wait_event(ev_cmp[b])          # step i-NB has finished reading dbufs[b]
        with torch.cuda.stream(s_h2d):
            dbufs[b].copy_(pinned[i % RING], non_blocking=True)
        ev_h2d[b].record(s_h2d)
        s_cmp.wait_event(ev_h2d[b])
        s_cmp.wait_event(ev_d2h[b])          # step i-NB's output has left obufs[b]
        q, k, v, dec, beta, wg = dviews[b]
        st.step(q, k, v, dec, beta, wg if wg is not None else bonus, obufs[b], stream=s_cmp)
        if not fused:
            st.merge(dlb.DL_MERGE_FULL, stream=s_cmp)
        ev_cmp[b].record(s_cmp)
        s_d2h.wait_event(ev_cmp[b])
        with torch.cuda.stream(s_d2h):
            o_hosts[b].copy_(obufs[b], non_blocking=True)
        ev_d2h[b].record(s_d2h)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize(device)
    dist_barrier(world)
    x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x0.record(s_cmp)
    s_h2d.wait_event(x0)
    s_d2h.wait_event(x0)
    for i in range(args.steps):
        e2e_step(i)
    for b in range(NB):
        s_cmp.wait_event(ev_d2h[b])
    x1.record(s_cmp)
    torch.cuda.synchronize(device)
    dist_barrier(world)
    e2e_s = max_over_ranks(x0.elapsed_time(x1) / 1e3, world, device)
    st.close()

    eager_gbs = (erd + ewr) / (eager_s / args.steps) / 1e9
    # The contract's peak is the measured copy bandwidth; in-repo
    # streaming kernels (eager, materialize) can beat that copy, so the line
    # also reports the fraction of the best of the three, and of nominal HBM.
    best_stream = max(peak, eager_gbs, mat_k["achieved_gbs"])
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(max_elapsed * 1e3 / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": workload_desc(w, args.merge, args.base), "name": w.name, "base": args.base,
                   "B": w.B, "H": w.H, "d_k": w.d_k, "d_v": w.d_v, "L": w.L, "merge": args.merge,
                   "step_split": args.split,
                   "global_batch": w.B * world,
                   "parallelism": f"replicas x{world} (dp, no collective)",
                   "l2": (f"base {state_mib:.0f} MiB > 126 MB L2 on every step: no flush needed"
                          if state_mib * 2**20 > L2_BYTES else f"state {state_mib:.0f} MiB fits L2: not a bench line"),
                   "input_ring_steps": RING},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs); "
                                  "the headline frac uses it",
                     "best_stream_gbs": round(best_stream, 1),
                     "frac_of_best_stream": round(achieved / best_stream, 4),
                     "frac_of_nominal_8tbs": round(achieved / 8000.0, 4),
                     "kernel": "dl_step_kernel", "algorithmic_bytes_per_launch": int(step_bytes_avg),
                     "launch_ms": round(step_avg * 1e3, 5)},
        "gpu_launches": int(launches),
        "e2e": {"value": round(aggregate_value(tokens, world, e2e_s), 1), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "clocks": clk.summary(),
        "hbm_gbs_step_plus_merge": round(((rd + wr + mrd + mwr) / args.steps) / (max_elapsed / args.steps) / 1e9, 1),
        "write_bytes_per_token": write_bytes_line(w, args, wr + mwr, ewr, rec),
        "merge_kernel": merge_k,
        "materialize_kernel": mat_k,
        "eager": {"value": round(aggregate_value(tokens, 1, eager_s), 1), "unit": UNIT,
                  "achieved_gbs": round(eager_gbs, 1),
                  "frac": round(eager_gbs / peak, 4),
                  "speedup_of_deltalog": round(eager_s / elapsed, 3)},
    }
    return line


def write_bytes_line(w, args, dl_write_total, eager_write, step_rec):
    """State write bytes per token: algorithmic (DeltaLog's timed steps and
    the eager step), and measured (DRAM writes per launch from the committed
    ncu records of the step and eager kernels at this batch, while both
    kernels' sources are unchanged)."""
    out = {"deltalog": round(dl_write_total / args.steps / w.B, 1),
           "eager": round(eager_write / w.B, 1),
           "reduction": round(eager_write / (dl_write_total / args.steps), 3)}
    eager_rec = traffic_record("dl_eager_kernel", workload=w.name, B=w.B)
    sw = mean_dram(step_rec, "dram_write") if step_rec and args.merge == "fused" else None
    ew = mean_dram(eager_rec, "dram_write") if eager_rec else None
    if sw and ew:
        out["measured"] = {"deltalog_dram_write_per_token": round(sw / w.B, 1),
                           "eager_dram_write_per_token": round(ew / w.B, 1),
                           "measured_reduction": round(ew / sw, 3),
                           "source": "profiles/ ncu records (dram__bytes_write.sum per launch)"}
    else:
        out["measured"] = None
    return out


# ------------------------------------------------------------ serving loop

def run_serving(args, world, rank, local):
    """A multi-layer decode loop with continuous batching: every token step
    runs the DeltaLog step of `layers` layers (fused merges), and every
    `admit_every` steps a fraction of the batch's slots take new sequences
    (dl_state_load_seqs with zero states, in every layer).  Reports decode
    tokens/s of the whole stack and the share of time spent on admission."""
    from linear_attention_recurrent_deltalog_b200 import deltalog as dlb

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = wl.WORKLOADS[args.workload]
    w = w.replace(L=args.L or w.L, B=args.B or w.B)
    cfg = dlb.Config(w.variant, w.B, w.H, w.d_k, w.d_v, w.L, w.in_dtype, fused_merge=True,
                     step_split=args.split)
    stream = torch.cuda.current_stream(device)
    host_steps = list(wl.StepStream(w, RING, workers=args.gen_workers))
    ring = [to_dev(s, device) for s in host_steps]
    bonus = (torch.from_numpy(wl.rwkv6_bonus(w)).to(device).reshape(-1)
             if w.variant == wl.RWKV6 else None)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    fills = wl.fill_offsets(w).tolist()
    layers = []
    for _ in range(args.layers):
        st = dlb.DeltaLogState(cfg, device=device)
        S0 = torch.randn(w.heads * w.d_v * w.d_k, generator=gen, device=device) * w.s0_std
        st.reset(S0, fills)
        del S0
        layers.append(st)
    o = torch.empty(w.heads * w.d_v, dtype=torch.float32, device=device)
    churn = max(1, w.B // 64)
    rng = np.random.default_rng(w.seed)

    def token_step(i):
        if args.admit_every > 0 and i % args.admit_every == args.admit_every - 1:
            seqs = rng.choice(w.B, size=churn, replace=False).tolist()
            for st in layers:
                st.load_seqs(seqs)
        q, k, v, dec, beta, wg = ring[i % RING]
        for st in layers:
            st.step(q, k, v, dec, beta, wg if wg is not None else bonus, o)

    for i in range(args.warmup):
        token_step(i)
    torch.cuda.synchronize(device)
    dist_barrier(world)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hold_stream()
    a.record(stream)
    for i in range(args.steps):
        token_step(args.warmup + i)
    b.record(stream)
    torch.cuda.synchronize(device)
    el = max_over_ranks(a.elapsed_time(b) / 1e3, world, device)
    for st in layers:
        code, head = st.device_error()
        if code != 0:
            raise RuntimeError(f"device error {code} at head {head}")
        st.close()
    return {"serving": True, "metric": "decode tokens/s through an N-layer state-update stack",
            "value": round(aggregate_value(w.B * args.steps, world, el), 1), "unit": UNIT,
            "layers": args.layers, "n_gpus": world, "steps": args.steps,
            "ms_per_token_step": round(el * 1e3 / args.steps, 4),
            "ms_per_layer_step": round(el * 1e3 / args.steps / args.layers, 4),
            "admission": {"every_steps": args.admit_every, "sequences": churn if args.admit_every else 0},
            "config": {"workload": workload_desc(w, "fused"), "B": w.B, "L": w.L}}


# ------------------------------------------------------------ CPU oracle

def oracle_tokens_per_s(w, target_s: float = 0.0, seqs: int = 2, steps: int = 0, warmup: int = 0):
    """The fp64 oracle as it stands on a bounded sample of the workload: the
    first ``seqs`` sequences (all H heads each), one decode step at a time.
    After ``warmup`` untimed steps it times either exactly ``steps`` steps or,
    when ``steps`` is 0, steps until ``target_s`` seconds of oracle time.
    Drawing the inputs is not timed.  Returns (tokens/s, steps, seconds,
    threads)."""
    import types

    import oracle
    seqs = min(seqs, w.B)
    heads = np.arange(seqs * w.H)
    shape = (heads.size, w.d_k, w.d_v) if w.variant == wl.RWKV6 else (heads.size, w.d_v, w.d_k)
    S = np.random.default_rng(w.seed).standard_normal(shape) * w.s0_std
    bonus = wl.rwkv6_bonus(w)[heads % w.H] if w.variant == wl.RWKV6 else None
    done, el, t = 0, 0.0, 0
    while (done < steps) if steps > 0 else (el < target_s):
        s = wl.step_inputs(w, t)
        sl = lambda x: None if x is None else x.reshape((w.heads,) + x.shape[2:])[heads][:, None]
        st = types.SimpleNamespace(q=sl(s.q), k=sl(s.k), v=sl(s.v), decay=sl(s.decay), beta=sl(s.beta),
                                   wgate=sl(s.wgate))
        a = time.perf_counter()
        S = oracle.run_eager(w.variant, S, [st], bonus=bonus, kla_eps=w.kla_eps).S
        dt = time.perf_counter() - a
        t += 1
        if t > warmup:
            el += dt
            done += 1
    threads = None
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        threads = max((i.get("num_threads", 1) for i in info), default=None)
    except Exception:
        threads = os.cpu_count()
    return seqs * done / el, done, el, threads


def host_cpu() -> dict:
    """The host's CPU model and logical core count (for the CPU baseline)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


def oracle_single_core(w, target_s: float):
    """oracle_tokens_per_s with the numerical libraries held to one thread."""
    try:
        import threadpoolctl
        with threadpoolctl.threadpool_limits(1):
            v, steps, el, _ = oracle_tokens_per_s(w, target_s=target_s, warmup=1)
    except Exception as e:  # a reported figure only: never fail the line for it
        return {"unavailable": f"{type(e).__name__}: {e}"}
    return {"value": round(v, 3), "cores": 1, "sample": cpu_sample_desc(w, steps, el)}


def cpu_sample_desc(w, steps, el, seqs=2):
    n = min(seqs, w.B)
    return (f"first {n} of {w.B} sequences ({n * w.H} heads), {steps} steps, "
            f"{el:.1f} s of fp64 eager oracle time")


def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = wl.WORKLOADS[args.workload]
    w = w.replace(L=args.L or w.L, B=args.B or w.B)
    # each step decodes the first 2 sequences (1 when K is large) of the batch
    seqs = 2 if args.steps + args.warmup <= 4000 else 1
    v, steps, el, threads = oracle_tokens_per_s(w, seqs=seqs, steps=args.steps, warmup=args.warmup)
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(v, 3), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(el * 1e3 / steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_desc(w, args.merge) + " (oracle: eager fp64)",
                   "name": w.name, "B": w.B, "H": w.H, "d_k": w.d_k, "d_v": w.d_v, "L": w.L},
        "cpu_baseline": {"value": round(v, 3), "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": cpu_sample_desc(w, steps, el, seqs), **host_cpu()},
        "e2e": {"value": round(v, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="gdn_serving", choices=sorted(wl.WORKLOADS),
                    help="synthetic workload (the headline line is gdn_serving)")
    ap.add_argument("--L", type=int, default=0, help="log length (0: the workload's)")
    ap.add_argument("--B", type=int, default=0, help="sequences (0: the workload's)")
    ap.add_argument("--kla-eps", type=float, default=-1.0,
                    help=">= 0: KLA step size beta = eta / (|k|^2 + eps) (GDN/KDA)")
    ap.add_argument("--split", type=int, default=0,
                    help="CTAs per head in the step kernel (0 = library default)")
    ap.add_argument("--only-step", action="store_true",
                    help="time the DeltaLog step only (profiling); not a bench line")
    ap.add_argument("--merge", choices=("fused", "separate"), default=None,
                    help="merge mode (default: fused for the fp32 base, separate for the int8 "
                         "base, the faster mode of each)")
    ap.add_argument("--base", choices=("f32", "q8"), default="f32",
                    help="base storage: fp32, or int8 codes + row scales requantized per window")
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gen-workers", type=int, default=None)
    ap.add_argument("--sweep", action="store_true", help="also print one line per L in 4..64")
    ap.add_argument("--serving", action="store_true",
                    help="multi-layer decode loop with slot admission instead of the headline line")
    ap.add_argument("--layers", type=int, default=8, help="layers of the --serving loop")
    ap.add_argument("--admit-every", type=int, default=8,
                    help="--serving: admit B/64 new sequences every this many steps (0: never)")
    args = ap.parse_args()
    if args.merge is None:
        args.merge = "separate" if args.base == "q8" else "fused"
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if world_plan(args.gpus, os.environ) == "spawn":
        if args.impl == "ours" and torch.cuda.device_count() < args.gpus:
            raise SystemExit(f"bench.py: --gpus {args.gpus} needs {args.gpus} CUDA devices, "
                             f"{torch.cuda.device_count()} visible")
        try:
            rc = subprocess.call(spawn_command(args.gpus, sys.argv[1:], free_port()), timeout=3600)
        except subprocess.TimeoutExpired:
            rc = 124
        sys.exit(rc)

    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            line = run_reference(args, world, rank)
            if line is not None:
                print(json.dumps(line), flush=True)
            return
        if args.serving:
            line = run_serving(args, world, rank, local)
            if rank == 0:
                print(json.dumps(line), flush=True)
            return
        line = run_ours(args, world, rank, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.only_step:
            w = wl.WORKLOADS[args.workload]
            w = w.replace(L=args.L or w.L, B=args.B or w.B)
            v, steps, el, threads = oracle_tokens_per_s(w, target_s=args.cpu_seconds, warmup=1)
            line["cpu_baseline"] = {"value": round(v, 3), "unit": UNIT, "cores": threads, "kind": "oracle",
                                    "sample": cpu_sample_desc(w, steps, el), **host_cpu(),
                                    "single_core": oracle_single_core(w, args.cpu_seconds / 2)}
        if rank == 0:
            print(json.dumps(line), flush=True)
        if args.sweep:
            for L in wl.SERVING_L_SWEEP:
                for merge in ("fused", "separate"):
                    a2 = argparse.Namespace(**vars(args))
                    a2.L, a2.merge = L, merge
                    a2.steps = min(args.steps, 500)
                    l2 = run_ours(a2, world, rank, local)
                    if rank == 0:
                        print(json.dumps({"sweep": True, "L": L, "merge": merge, "value": l2["value"],
                                          "roofline": l2["roofline"], "eager": l2["eager"],
                                          "write_bytes_per_token": l2["write_bytes_per_token"],
                                          "hbm_gbs_step_plus_merge": l2["hbm_gbs_step_plus_merge"]}),
                              flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
