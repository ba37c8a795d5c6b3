"""Benchmark of the sparse-convolution hot path on B200.

One step is one pass of every stage of the path over the LiDAR-shaped
SubmConv3d workload (batch 2 x 100k voxels in a 1440x1440x41 grid, fp16,
64 channels), all through the C ABI:

  stream 1: hash build -> submanifold kernel map (probe, pairs, mask sort,
            tile masks) -> SubmConv3d fwd 64->64 -> dgrad -> per-offset wgrad
  stream 2: strided support (k=2 s=2, with each voxel's coarse row)
            -> strided + transposed kernel maps from those parent rows
            -> strided Conv3d fwd 64->128 -> ConvTranspose3d fwd 128->64.

The two chains depend only on the step's inputs, so stream 2 is forked from
stream 1 when the step starts and joined back before it ends; the step's
events sit on stream 1 around both.

value = effective TFLOP/s of the step (sum over the five convolution passes
of 2 * pairs * Cin * Cout, divided by the step's device time); the kernel-map
rate (voxels / (hash + query time)) is reported beside it.  L2 is flushed
(256 MB write) before every timed step, outside the step's events.

--impl reference times the CPU oracle on the same workload (a bounded sample
of steps on the host cores).  Under torchrun every rank runs its own batch
(weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

WORKLOAD = "lidar_subm"
METRIC = "sparse-conv effective TFLOP/s + kmap Mvoxels/s at 1 B200, % of roofline"
CIN, CMID = 64, 128
RSV_RATIO = 4.0  # hash slots per voxel (hash_rsv_ratio)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# --------------------------------------------------------------------------- multi-rank helpers
def rank_seed(base_seed: int, rank: int) -> int:
    """Every rank draws its own batch (weak scaling: per-rank work is fixed)."""
    return base_seed + 1000 * rank


def max_over_ranks(x: float, dist, device) -> float:
    """The slowest rank's time: all ranks report, the max is the job's time."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank: float, world: int, steps: int, total_ms: float) -> float:
    """Whole-job effective TFLOP/s: the work of all ranks over the max-over-ranks time."""
    return flops_per_rank * world * steps / (total_ms * 1e-3) / 1e12


# --------------------------------------------------------------------------- inputs
def make_inputs(rank: int):
    wl = synthetic.WORKLOADS[WORKLOAD]
    seed = rank_seed(wl.seed, rank)
    coords = synthetic.lidar(seed=seed, **wl.gen_args)
    n = len(coords)
    x = torch.from_numpy(synthetic.features(n, CIN, seed)).half()
    g = torch.from_numpy(synthetic.features(n, CIN, seed, 1)).half()
    w = torch.from_numpy(synthetic.weights(27, CIN, CIN, seed)).half()
    wd = torch.from_numpy(synthetic.weights(8, CIN, CMID, seed, 1)).half()
    wu = torch.from_numpy(synthetic.weights(8, CMID, CIN, seed, 2)).half()
    return dict(coords=torch.from_numpy(coords), x=x, g=g, w=w, wd=wd, wu=wu)


# --------------------------------------------------------------------------- GPU pipeline
class Pipeline:
    """Preallocated buffers + the sequence of C-ABI calls of one step.

    The step is two chains of calls that share only their inputs: the
    submanifold layer (hash, kernel map, fwd, dgrad, wgrad) on the caller's
    stream, and the strided / transposed pair (coarse support, maps from
    parents, down conv, up conv) on a second stream forked from it at the start
    and joined back at the end.  Each chain has its own workspace.  Many of the
    kernels are short or latency-bound, so the two chains fill each other's
    gaps on the GPU.  The host enqueues the coarse support first, then the
    kernel map and the forward pass, then reads the coarse row count and
    enqueues the rest of both chains interleaved; the second chain's stream has
    the higher priority (it waits on the host for the count halfway through)."""

    MAIN_PHASES = ["hash", "kmap", "fwd", "dgrad", "wgrad"]
    SIDE_PHASES = ["downsample", "down_maps", "down_fwd", "up_fwd"]
    PHASES = MAIN_PHASES + SIDE_PHASES

    def __init__(self, host: dict, dev: torch.device):
        import sparse_convolution_voxel_b200 as scv
        self.scv = scv
        self.dev = dev
        self.d = {k: v.to(dev) for k, v in host.items()}
        n = self.n = host["coords"].shape[0]
        self.status = scv.new_status(dev)
        self.ws = scv.Workspace(dev)
        self.ws_side = scv.Workspace(dev)
        # the second chain waits on the host for the coarse row count halfway through,
        # so its kernels get the higher stream priority: its first half finishes
        # sooner and its second half is enqueued sooner
        self.side = torch.cuda.Stream(dev, priority=torch.cuda.Stream.priority_range()[1])
        self.forked, self.joined = torch.cuda.Event(), torch.cuda.Event()
        self.table = torch.empty(scv.lat_hash_bytes(n, RSV_RATIO) // 8, dtype=torch.int64, device=dev)
        self.km = scv.KernelMap(n, n, 27, dev)
        self.y = torch.empty((n, CIN), dtype=torch.half, device=dev)
        self.dx = torch.empty((n, CIN), dtype=torch.half, device=dev)
        self.dw = torch.empty((27, CIN, CIN), dtype=torch.float32, device=dev)
        self.coarse_buf = torch.empty((n, 4), dtype=torch.int32, device=dev)
        self.z = torch.empty((n, CIN), dtype=torch.half, device=dev)
        self.g_sub, self.g_down, self.g_up = scv.subm_geom(3), scv.strided_geom(2, 2, 0), scv.transposed_geom(2, 2, 0)
        # the coarse support size is fixed for a fixed input: size the coarse buffers once
        self.parent = torch.empty(n, dtype=torch.int32, device=dev)
        self.nc = scv.lat_downsample_coords(self.d["coords"], self.g_down, self.coarse_buf,
                                            self.ws.get(scv.lat_downsample_ws_bytes(n, self.g_down)), self.status,
                                            parent=self.parent)
        nc = self.nc
        self.km_down = scv.KernelMap(n, nc, 8, dev)
        self.km_up = scv.KernelMap(nc, n, 8, dev)
        self.yc = torch.empty((nc, CMID), dtype=torch.half, device=dev)
        self.wsb = self.ws.get(max(scv.lat_kmap_ws_bytes(n, 27),
                                   scv.lat_sconv_ws_bytes(2, CIN, CIN, self.km.c, torch.half),
                                   scv.lat_sconv_ws_bytes(0, CIN, CIN, self.km.c, torch.half),
                                   scv.lat_sconv_ws_bytes(1, CIN, CIN, self.km.c, torch.half)))
        self.wsb_side = self.ws_side.get(max(scv.lat_downsample_ws_bytes(n, self.g_down),
                                             scv.lat_kmap_from_parent_ws_bytes(n, nc, 8),
                                             scv.lat_sconv_ws_bytes(0, CIN, CMID, self.km_down.c, torch.half),
                                             scv.lat_sconv_ws_bytes(0, CMID, CIN, self.km_up.c, torch.half)))
        self.nc_host = torch.empty(1, dtype=torch.int64, pin_memory=True)
        self.nc_view = self.nc_host.numpy()  # read without building a tensor each step
        self.nc_ready = torch.cuda.Event()
        self.pairs = None

    def step(self, ev: dict | None = None):
        """Run one step.  `ev` maps a phase name to a (start, end) pair of timing
        events, recorded on the stream that phase runs on; any subset of PHASES."""
        scv, d, s = self.scv, self.d, self.status
        main, side = torch.cuda.current_stream(self.dev), self.side
        ev = ev or {}

        def rec(phase, i, stream):
            if phase in ev:
                ev[phase][i].record(stream)

        self.forked.record(main)
        side.wait_event(self.forked)
        rec("downsample", 0, side)
        scv.lat_downsample_coords_async(d["coords"], self.g_down, self.coarse_buf, self.wsb_side, self.nc_host, s,
                                        stream=side, parent=self.parent)
        self.nc_ready.record(side)
        rec("downsample", 1, side)
        rec("hash", 0, main)
        scv.lat_hash_build(d["coords"], self.table, s)
        rec("hash", 1, main)
        rec("kmap", 0, main)
        scv.lat_kmap_query(self.table, d["coords"], self.g_sub, self.km.c, self.wsb, s)
        rec("kmap", 1, main)
        rec("fwd", 0, main)
        scv.lat_sconv_fwd(d["x"], d["w"], self.km.c, self.y, self.wsb, s)
        rec("fwd", 1, main)
        self.nc_ready.synchronize()
        nc = int(self.nc_view[0])
        if nc < 0:  # coarse fields too wide for the bitmap: blocking radix-sort path
            nc = scv.lat_downsample_coords(d["coords"], self.g_down, self.coarse_buf, self.wsb_side, s,
                                           stream=side, parent=self.parent)
        assert nc == self.nc
        rec("down_maps", 0, side)
        scv.lat_kmap_from_parent(d["coords"], self.parent, self.g_down, self.km_down.c, self.km_up.c, self.wsb_side, s,
                                 stream=side)
        rec("down_maps", 1, side)
        rec("dgrad", 0, main)
        scv.lat_sconv_dgrad(d["g"], d["w"], self.km.c, True, self.dx, self.wsb, s)
        rec("dgrad", 1, main)
        rec("down_fwd", 0, side)
        scv.lat_sconv_fwd(d["x"], d["wd"], self.km_down.c, self.yc, self.wsb_side, s, stream=side)
        rec("down_fwd", 1, side)
        rec("wgrad", 0, main)
        scv.lat_sconv_wgrad(d["x"], d["g"], self.km.c, self.dw, self.wsb, s)
        rec("wgrad", 1, main)
        rec("up_fwd", 0, side)
        scv.lat_sconv_fwd(self.yc, d["wu"], self.km_up.c, self.z, self.wsb_side, s, stream=side)
        rec("up_fwd", 1, side)
        self.joined.record(side)
        main.wait_event(self.joined)

    def pair_count(self) -> int:
        if self.pairs is None:
            self.pairs = int(self.km.pair_off[27].item())
        return self.pairs

    def flops(self) -> float:
        p = self.pair_count()
        return 2.0 * (3 * p * CIN * CIN + self.n * CIN * CMID + self.n * CMID * CIN)

    def phase_bytes(self) -> dict:
        """Algorithmic bytes per phase (fp16 features, int32 indices)."""
        n, p, nc, e = self.n, self.pair_count(), self.nc, 2
        w = 27 * CIN * CIN * e
        return {
            "hash": n * 16 + n * 16,
            "kmap": n * 16 + n * 27 * 4 + n * 4 + 8 * p,
            "fwd": p * CIN * e + n * CIN * e + w + 8 * p,
            "dgrad": p * CIN * e + n * CIN * e + w + 8 * p,
            "wgrad": p * 2 * CIN * e + 27 * CIN * CIN * 4 + 8 * p,
            "down_fwd": n * CIN * e + nc * CMID * e + 8 * CIN * CMID * e + 8 * n,
            "up_fwd": n * CMID * e + n * CIN * e + 8 * CIN * CMID * e + 8 * n,
        }


# The kernel the roofline object reports: the path kernel with the largest
# share of the step's ncu launch list (serialised; the tcgen05 strided Conv3d
# 64 -> 128, 6.9% of the step's kernel time, the largest of the path's kernels).
DOMINANT_KERNEL = "down_fwd"

# DRAM bytes per launch from that ncu launch list of this workload (caches not
# flushed between kernels): the strided conv, and the submanifold kmap query's
# kernels summed; None where no capture matches the current kernels.
PHASE_TRAFFIC = {"down_fwd": 72.3e6, "kmap": 27.2e6}


def flush_l2(buf: torch.Tensor):
    buf.add_(1)


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML every ~0.5 ms while the
    timed region runs, plus one sample as it starts and one as it ends
    (read-only queries; nothing is changed on the GPU)."""

    NAMES = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
             "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
             "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
             "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, device: torch.device, period_s: float = 0.0005):
        import threading
        self.period = period_s
        self.samples = []
        self.stop = threading.Event()
        self.thread = None
        self.handle = None
        self.max_mhz = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            props = torch.cuda.get_device_properties(device)
            try:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self.handle = nv.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.handle = nv.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
        except Exception:
            self.handle = None

    def _sample(self):
        nv = self.nv
        try:
            self.samples.append((nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM),
                                 nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)))
        except Exception:
            pass

    def _run(self):
        while not self.stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        import threading
        if self.handle is not None:
            self._sample()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        return self

    def mark_end(self):
        """A last sample while the timed work may still be running on the GPU."""
        if self.handle is not None:
            self._sample()

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)

    def summary(self) -> dict:
        if self.handle is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        reasons = set()
        for _, r in self.samples:
            for name, attr in self.NAMES.items():
                if r & getattr(self.nv, attr):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(c for c, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples), "source": "nvml"}


def count_launches(pipe: Pipeline) -> int:
    """Kernels one step launches, counted with the CUDA profiler (outside timing)."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        pipe.step()
        torch.cuda.synchronize()
    n = 0
    for e in prof.events():
        if e.device_type == torch.autograd.DeviceType.CUDA and "memset" not in e.name.lower() \
                and "memcpy" not in e.name.lower():
            n += 1
    return n


# --------------------------------------------------------------------------- CPU oracle arm
def oracle_step(host: dict, nthreads: int = 0) -> float:
    """One step of the oracle on the same input; returns its effective flops."""
    import oracle
    c = host["coords"].numpy()
    x = host["x"].double().numpy()
    g = host["g"].double().numpy()
    w = host["w"].double().numpy()
    nbr = oracle.kmap(c, c, 3, 1, 1, oracle.SUBM, nthreads)
    oracle.conv_fwd(x, w, nbr, nthreads)
    oracle.conv_dgrad(g, w, nbr, len(c), nthreads)
    oracle.conv_wgrad(x, g, nbr, nthreads)
    coarse = oracle.downsample(c, 2, 2, 0)
    down = oracle.kmap(c, coarse, 2, 2, 0, oracle.STRIDED, nthreads)
    up = oracle.kmap(coarse, c, 2, 2, 0, oracle.TRANSPOSED, nthreads)
    yc = oracle.conv_fwd(x, host["wd"].double().numpy(), down, nthreads)
    oracle.conv_fwd(yc, host["wu"].double().numpy(), up, nthreads)
    p = int((nbr >= 0).sum())
    n = len(c)
    return 2.0 * (3 * p * CIN * CIN + n * CIN * CMID + n * CMID * CIN)


def cpu_baseline(host: dict, budget_s: float = 15.0) -> dict:
    import oracle
    cores = oracle.max_threads()
    times, flops = [], 0.0
    t_all = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        flops = oracle_step(host)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all > budget_s or len(times) >= 5:
            break
    t = statistics.median(times)
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(times)} full oracle steps of the {WORKLOAD} workload (median {t:.2f} s per step)"}


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return
    host = make_inputs(0)
    import oracle
    cores = oracle.max_threads()
    for _ in range(args.warmup):
        oracle_step(host)
    times, flops = [], 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        flops = oracle_step(host)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = flops * args.steps / total / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(host["coords"].shape[0], world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} full oracle steps of the {WORKLOAD} workload"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(n, world):
    return {"workload": f"{WORKLOAD}: LiDAR-shaped SubmConv3d k=3 (batch 2 x 100k voxels, 1440x1440x41 grid, fp16, "
                        f"64->64) + dgrad + wgrad + strided Conv3d k2s2 64->128 + ConvTranspose3d 128->64 on the "
                        f"same support",
            "voxels_per_gpu": int(n), "global_batch": 2 * world, "parallelism": f"replicas x{world}",
            "l2": "flushed (256 MB write) before every timed step"}


# --------------------------------------------------------------------------- single-op mode (profiling)
def run_only(args):
    """Run one op of the path repeatedly on a named workload (used for ncu captures)."""
    import sparse_convolution_voxel_b200 as scv
    from sparse_convolution_voxel_b200 import build as b
    if not os.path.exists(scv.LIB_PATH):
        b.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = synthetic.WORKLOADS[args.workload]
    dt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[wl.dtype]
    # even kernels (the down/up workload) have no submanifold form: its subm ops use 3x3x3
    ksize = wl.ksize if all(k % 2 for k in wl.ksize) else (3, 3, 3)
    k3 = int(np.prod(ksize))
    coords = torch.from_numpy(wl.coords()).to(dev)
    n = coords.shape[0]
    cin, cout = wl.cin, wl.cout
    x = torch.from_numpy(synthetic.features(n, cin, wl.seed)).to(dt).to(dev)
    g = torch.from_numpy(synthetic.features(n, cout, wl.seed, 1)).to(dt).to(dev)
    w = torch.from_numpy(synthetic.weights(k3, cin, cout, wl.seed)).to(dt).to(dev)
    st = scv.new_status(dev)
    ws = scv.Workspace(dev)
    geom = scv.subm_geom(ksize)
    table = scv.hash_table(coords, args.rsv_ratio, st)
    km = scv.kernel_map(table, n, coords, geom, ws, st)
    y = torch.empty((n, cout), dtype=dt, device=dev)
    dx = torch.empty((n, cin), dtype=dt, device=dev)
    dw = torch.empty((k3, cin, cout), dtype=torch.float32, device=dev)
    coarse = torch.empty((n * 8, 4), dtype=torch.int32, device=dev)
    parent = torch.empty(n, dtype=torch.int32, device=dev)
    g_up = scv.transposed_geom(2, 2, 0)
    wsb = ws.get(max(scv.lat_kmap_ws_bytes(n, k3), scv.lat_sconv_ws_bytes(2, cin, cout, km.c, dt),
                     scv.lat_sconv_ws_bytes(0, cin, cout, km.c, dt), scv.lat_sconv_ws_bytes(1, cin, cout, km.c, dt),
                     scv.lat_downsample_ws_bytes(n, scv.strided_geom(2, 2, 0)), scv.lat_upsample_ws_bytes(n, g_up)))
    # generative decoder step: the k2s2 transposed support of the coarse support
    coarse_c = scv.downsample(coords, scv.strided_geom(2, 2, 0), ws).contiguous() if args.only == "upsample" else coords
    fine_buf = torch.empty((coarse_c.shape[0] * 8, 4), dtype=torch.int32, device=dev)
    n_fine = scv.lat_upsample_coords(coarse_c, g_up, fine_buf, wsb, st) if args.only == "upsample" else 0
    torch.cuda.synchronize()
    P = int(km.pair_off[k3].item())
    e = dt.itemsize
    ops = {
        "hash": (lambda: scv.lat_hash_build(coords, table, st), n * 32),
        "kmap": (lambda: scv.lat_kmap_query(table, coords, geom, km.c, wsb, st), n * 16 + n * k3 * 4 + n * 4 + 8 * P),
        "fwd": (lambda: scv.lat_sconv_fwd(x, w, km.c, y, wsb, st), P * cin * e + n * cout * e + w.numel() * e + 8 * P),
        "dgrad": (lambda: scv.lat_sconv_dgrad(g, w, km.c, True, dx, wsb, st),
                  P * cout * e + n * cin * e + w.numel() * e + 8 * P),
        "wgrad": (lambda: scv.lat_sconv_wgrad(x, g, km.c, dw, wsb, st), P * (cin + cout) * e + dw.numel() * 4 + 8 * P),
        "downsample": (lambda: scv.lat_downsample_coords(coords, scv.strided_geom(2, 2, 0), coarse, wsb, st,
                                                         parent=parent),
                       n * 16 * 2),
        "upsample": (lambda: scv.lat_upsample_coords(coarse_c, g_up, fine_buf, wsb, st),
                     coarse_c.shape[0] * 16 + n_fine * 16),
        # pooling: x read once, y written once, the mask and every used neighbour index
        "pool_max": (lambda: scv.lat_sparse_pool(x, km.c, scv.LAT_POOL_MAX, dx, st), 2 * n * cin * e + 4 * n + 4 * P),
        "pool_avg": (lambda: scv.lat_sparse_pool(x, km.c, scv.LAT_POOL_AVG, dx, st), 2 * n * cin * e + 4 * n + 4 * P),
    }
    if args.only == "pool_down":
        # k2s2 max pooling onto the generated coarse support
        g_dn = scv.strided_geom(2, 2, 0)
        coarse_p = scv.downsample(coords, g_dn, ws).contiguous()
        km_dn = scv.kernel_map(table, n, coarse_p, g_dn, ws, st)
        y_dn = torch.empty((coarse_p.shape[0], cin), dtype=dt, device=dev)
        torch.cuda.synchronize()
        P = int(km_dn.pair_off[8].item())
        ops["pool_down"] = (lambda: scv.lat_sparse_pool(x, km_dn.c, scv.LAT_POOL_MAX, y_dn, st),
                            (n + coarse_p.shape[0]) * cin * e + 4 * coarse_p.shape[0] + 4 * P)
    if args.only == "down_fwd":
        # strided Conv3d k2s2 Cin -> 2 Cin onto the generated coarse support (maps from
        # parents): on lidar_subm the bench step's fp16 64 -> 128 down conv
        g_dn = scv.strided_geom(2, 2, 0)
        coarse_d, par = scv.downsample(coords, g_dn, ws, with_parent=True)
        ncd = coarse_d.shape[0]
        km_d, _ = scv.maps_from_parent(coords, par.contiguous(), ncd, g_dn, ws, st)
        cd = 2 * cin
        wd = torch.from_numpy(synthetic.weights(8, cin, cd, wl.seed)).to(dt).to(dev)
        yd = torch.empty((ncd, cd), dtype=dt, device=dev)
        wsd = torch.empty(max(1, scv.lat_sconv_ws_bytes(0, cin, cd, km_d.c, dt)), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()
        ops["down_fwd"] = (lambda: scv.lat_sconv_fwd(x, wd, km_d.c, yd, wsd, st),
                           n * cin * e + ncd * cd * e + 8 * cin * cd * e + 8 * n)
    if args.only == "dense":
        # dense grid over the coordinates' bounding box: the whole grid written once, rows read once
        lo, hi = coords.amin(0).tolist(), coords.amax(0).tolist()
        box = [hi[a + 1] - lo[a + 1] + 1 for a in range(3)]
        grid = torch.empty((hi[0] + 1, *box, cin), dtype=dt, device=dev)
        ops["dense"] = (lambda: scv.lat_to_dense(coords, x, lo[1:], box, hi[0] + 1, grid, st),
                        grid.numel() * e + n * 16 + n * cin * e)
    fn, nbytes = ops[args.only]
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    ms = []
    for _ in range(args.steps):
        flush_l2(flush)
        a, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        bb.record()
        torch.cuda.synchronize()
        ms.append(a.elapsed_time(bb))
    # host cost of one call, and the device time per call when calls are issued back to back
    torch.cuda.synchronize()
    reps = 20
    h0 = time.perf_counter()
    a, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    bb.record()
    host_us = (time.perf_counter() - h0) / reps * 1e6
    torch.cuda.synchronize()
    b2b_ms = a.elapsed_time(bb) / reps
    stv = scv.lat_status_fetch(st)
    t = statistics.median(ms)
    hbm, _, src = load_peaks()
    print(json.dumps({"only": args.only, "workload": args.workload, "rsv_ratio": args.rsv_ratio, "rows": n,
                      "pairs": P, "ms_median": t,
                      "ms_min": min(ms), "alg_bytes": nbytes, "achieved_gbs": nbytes / (t * 1e-3) / 1e9,
                      "frac_hbm": nbytes / (t * 1e-3) / 1e9 / hbm, "peak_source": src, "status": stv,
                      "host_us_per_call": host_us, "b2b_ms_per_call": b2b_ms}), flush=True)


# --------------------------------------------------------------------------- main GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", choices=["hash", "kmap", "fwd", "dgrad", "wgrad", "downsample", "upsample", "pool_max",
                                       "pool_avg", "pool_down", "dense", "down_fwd"],
                    help="time a single op of the path on --workload (for profiler captures)")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--rsv-ratio", type=float, default=RSV_RATIO, help="hash table slots per voxel (--only mode)")
    ap.add_argument("--lean", action="store_true",
                    help="skip launch counting, the end-to-end pass and the CPU baseline (for profiler runs)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args)
    if args.only:
        return run_only(args)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    import sparse_convolution_voxel_b200 as scv
    try:
        scv.load()
    except ImportError:
        from sparse_convolution_voxel_b200 import build as b
        b.build()
        scv.load()

    host = make_inputs(rank)
    pipe = Pipeline(host, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        pipe.step()
    torch.cuda.synchronize()
    st = scv.lat_status_fetch(pipe.status)
    if st:
        raise scv.LatticeError(st, "device status after warm-up")
    launches_per_step = None if args.lean else count_launches(pipe)

    # per-phase times from instrumented steps outside the timed region: a timing
    # event between two kernels holds back the next kernel's early launch, so the
    # timed steps carry events around the dominant kernel's call only
    pb = pipe.phase_bytes()
    inst = [{p: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for p in Pipeline.PHASES} for _ in range(min(args.steps, 10))]
    torch.cuda.synchronize()
    for ev in inst:
        flush_l2(flush)
        pipe.step(ev)
    torch.cuda.synchronize()
    phase_ms_inst = {p: statistics.mean(ev[p][0].elapsed_time(ev[p][1]) for ev in inst) for p in Pipeline.PHASES}
    dominant = DOMINANT_KERNEL

    steps = [{"step": (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)),
              dominant: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))}
             for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        for ev in steps:
            flush_l2(flush)
            ev["step"][0].record()
            pipe.step({dominant: ev[dominant]})
            ev["step"][1].record()
        clk.mark_end()
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    step_ms = [ev["step"][0].elapsed_time(ev["step"][1]) for ev in steps]
    dominant_ms = statistics.mean(ev[dominant][0].elapsed_time(ev[dominant][1]) for ev in steps)
    total_ms = sum(step_ms)
    if pg:
        total_ms = max_over_ranks(total_ms, pg, dev)
    flops = pipe.flops()
    value = job_throughput(flops, world, args.steps, total_ms)
    kmap_ms = phase_ms_inst["hash"] + phase_ms_inst["kmap"]

    # end to end through the public API: host inputs in, results back to the host
    e2e = None
    if rank == 0 and not args.lean:
        e2e = measure_e2e(host, dev, steps=max(3, min(args.steps, 20)))

    if rank == 0:
        hbm, tc, src = load_peaks()
        achieved = pb[dominant] / (dominant_ms * 1e-3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": config_dict(pipe.n, world),
            "kmap_mvoxels_per_s": pipe.n / (kmap_ms * 1e-3) / 1e6,
            "pairs": pipe.pair_count(), "coarse_voxels": pipe.nc,
            "phase_ms": {k: round(v, 4) for k, v in phase_ms_inst.items()},
            "phase_ms_note": "per-phase event times from instrumented steps outside the timed region "
                             "(the two chains overlap, so phases do not add up to the step)",
            "roofline": {"kernel": f"{dominant} (conv_tc_kernel, strided Conv3d 64->128 on tcgen05)", "bound": "hbm",
                         "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "traffic": PHASE_TRAFFIC.get(dominant),
                         "alg_bytes": pb[dominant], "ms": dominant_ms, "peak_source": f"{src} hbm_gbs",
                         "timing": "CUDA events around this phase on its stream in every timed step",
                         "traffic_per_phase": PHASE_TRAFFIC,
                         "per_phase_frac": {p: round(pb[p] / (phase_ms_inst[p] * 1e-3) / 1e9 / hbm, 4)
                                            for p in pb}},
            "gpu_launches": None if launches_per_step is None else launches_per_step * args.steps,
            "e2e": e2e,
            "clocks": clk.summary(),
        }
        if not args.no_cpu_baseline and not args.lean and world == 1:
            line["cpu_baseline"] = cpu_baseline(host)
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def measure_e2e(host: dict, dev: torch.device, steps: int) -> dict:
    """Same step through the public API with inputs copied from pinned host memory and
    the step's result (dW) copied back, copies inside the timed region.  Steps alternate between
    two device buffer sets: step i+1's inputs are copied in (two H2D streams) and step
    i-1's result copied out (D2H stream) while step i computes; the L2 is flushed before
    every step's compute.  Time = first copy-in start to last copy-out end."""
    pinned = {k: v.pin_memory() for k, v in host.items()}
    pipes = [Pipeline(host, dev), Pipeline(host, dev)]
    # the step's result read back every step: the weight gradient (what a training
    # step hands to the optimizer); the activations and dx stay on the device, as
    # they would between layers
    outs = [{"dw": torch.empty(p.dw.shape, dtype=torch.float32).pin_memory()} for p in pipes]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in outs[0].values())
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    comp, up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    # the inputs cross the host link on two copy streams (largest first, alternating):
    # consecutive copies on one stream reach ~38 GB/s, two streams the link's ~54 GB/s
    up2 = torch.cuda.Stream(dev)
    order = sorted(pinned, key=lambda k: -pinned[k].numel() * pinned[k].element_size())
    computed = [torch.cuda.Event() for _ in pipes]   # the buffer set's last step finished computing
    copied_out = [torch.cuda.Event() for _ in pipes]  # its results reached the host

    inputs_in = [[torch.cuda.Event(), torch.cuda.Event()] for _ in pipes]  # a set's inputs arrived (2 streams)

    def copy_in(i: int):
        """Enqueue step i's input copies into buffer set i % 2 (no host wait)."""
        b = i % 2
        p = pipes[b]
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(computed[b])  # the set's previous step has read its inputs
            began = torch.cuda.Event()
            began.record()
        up2.wait_event(began)
        for c, k in enumerate(order):
            with torch.cuda.stream(up if c % 2 == 0 else up2):
                p.d[k].copy_(pinned[k], non_blocking=True)
        inputs_in[b][0].record(up)
        inputs_in[b][1].record(up2)

    def run(n: int, start: torch.cuda.Event | None = None, end: torch.cuda.Event | None = None):
        # step i+1's copies are enqueued before step i runs: the step blocks the host
        # on its coarse row count, and the next copies must not wait behind that
        if start is not None:
            start.record(up)
        copy_in(0)
        for i in range(n):
            b = i % 2
            p, o = pipes[b], outs[b]
            if i + 1 < n:
                copy_in(i + 1)
            with torch.cuda.stream(comp):
                comp.wait_event(inputs_in[b][0])
                comp.wait_event(inputs_in[b][1])
                if i >= 2:
                    comp.wait_event(copied_out[b])  # its previous results have left
                flush_l2(flush)
                p.step()
                computed[b].record()
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                for k, v in o.items():
                    v.copy_(getattr(p, k), non_blocking=True)
                copied_out[b].record()
                if i == n - 1 and end is not None:
                    end.record()

    run(4)
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run(steps, a, e)
    torch.cuda.synchronize()
    t = a.elapsed_time(e) / steps
    return {"value": pipes[0].flops() / (t * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": t,
            "overlap": "copies of the next step's inputs (two H2D streams) and the previous step's result run "
                       "during each step; two buffer sets; L2 flushed before each step's compute",
            "result_read_back": "dW (fp32, 27 x 64 x 64) every step; y, dx and the up-conv output stay on the device"}


if __name__ == "__main__":
    main()
