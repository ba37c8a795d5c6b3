"""Benchmark of the sparse-convolution hot path on B200.

Headline step: one SubmConv3d k=3 training step of the LiDAR-shaped
workload `lidar_train` (batch 4 x 125k voxels in a 1440x1440x41 grid, bf16,
128 -> 128 channels), all through the C ABI on one stream:

    hash build -> submanifold kernel map (probe, pairs, mask sort, tile masks)
    -> forward -> data gradient -> per-offset weight gradient

with the upstream gradient N(0,1).  value = effective TFLOP/s of the step:
the three convolution passes' 2 * pairs * Cin * Cout each, divided by the
step's device time (hash and kernel map included).  The L2 is flushed
(256 MB write) before every timed step, outside the step's events.

Beside the headline, `configs` carries every workload with its own timing
(flushed L2, CUDA events, clocks sampled while it runs), its per-phase
roofline fractions and its error statistics against the CPU oracle:

    subm_small     2k uniform voxels, fp32 16 -> 16, training step
    lidar_subm     200k LiDAR voxels, fp16 64 -> 64, training step
    lidar_down_up  200k LiDAR voxels (its own scan), bf16: strided Conv3d
                   k2s2 64 -> 128 onto the generated coarse support, then
                   ConvTranspose3d k2s2 128 -> 64 back onto the fine support
    images_subm    256 sparse 512x512 images, fp32 8 -> 32, 3x3 training step
    lidar_train    the headline step

--impl reference times the CPU oracle on the headline workload (a bounded
sample of steps on the host cores).  Under torchrun every rank runs its own
batch (weak scaling, no collective on the data path).  --only OP times one op
on one workload (for profiler captures); --cpu-table times the oracle per pass
and workload, single-threaded and on all cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import platform
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402

WORKLOAD = "lidar_train"
CONFIG_ORDER = ["subm_small", "lidar_subm", "lidar_down_up", "images_subm", "lidar_train"]
METRIC = "sparse-conv effective TFLOP/s + kmap Mvoxels/s at 1 B200, % of roofline"
RSV_RATIO = 4.0  # hash slots per voxel (hash_rsv_ratio)
FLUSH_BYTES = 256 * 1024 * 1024
TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
# fp32 normwise 1e-5 relative, fp16 / bf16 max|err| <= 2e-2 max|ref|
REL_TOL = {torch.float32: 1e-5, torch.float16: 2e-2, torch.bfloat16: 2e-2}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


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
def make_host(name: str, rank: int = 0) -> dict:
    """Seeded host inputs of a workload (coordinates, features, upstream gradient, weights)."""
    wl = synthetic.WORKLOADS[name]
    seed = rank_seed(wl.seed, rank)
    coords = dataclasses.replace(wl, seed=seed).coords()
    n = len(coords)
    dt = TORCH_DT[wl.dtype]
    h = {"coords": torch.from_numpy(coords), "x": torch.from_numpy(synthetic.features(n, wl.cin, seed)).to(dt)}
    if name == "lidar_down_up":
        h["wd"] = torch.from_numpy(synthetic.weights(8, wl.cin, wl.cout, seed)).to(dt)
        h["wu"] = torch.from_numpy(synthetic.weights(8, wl.cout, wl.cin, seed, 1)).to(dt)
    else:
        k3 = int(np.prod(wl.ksize))
        h["g"] = torch.from_numpy(synthetic.features(n, wl.cout, seed, 1)).to(dt)
        h["w"] = torch.from_numpy(synthetic.weights(k3, wl.cin, wl.cout, seed)).to(dt)
    return h


def make_layer(name: str, host: dict, dev: torch.device):
    return DownUpLayer(name, host, dev) if name == "lidar_down_up" else SubmLayer(name, host, dev)


# --------------------------------------------------------------------------- GPU steps
class SubmLayer:
    """One SubmConv3d training step through the C ABI: hash build, kernel map
    and forward on the current stream, then the data gradient on a second
    (high-priority) stream beside the weight gradient -- both read only the
    inputs, the weights and the map -- joined back into the current stream."""

    PHASES = ["hash", "kmap", "fwd", "dgrad", "wgrad"]
    CONV = ["fwd", "dgrad", "wgrad"]
    SPANS = ["conv_span"]  # forward start to the join of the two gradient streams

    def __init__(self, name: str, host: dict, dev: torch.device):
        import sparse_convolution_voxel_b200 as scv
        self.scv, self.name, self.dev = scv, name, dev
        wl = synthetic.WORKLOADS[name]
        self.wl = wl
        self.dt = TORCH_DT[wl.dtype]
        self.cin, self.cout = wl.cin, wl.cout
        self.k3 = int(np.prod(wl.ksize))
        self.d = {k: v.to(dev) for k, v in host.items()}
        n = self.n = host["coords"].shape[0]
        self.status = scv.new_status(dev)
        self.ws = scv.Workspace(dev)
        self.table = torch.empty(scv.lat_hash_bytes(n, RSV_RATIO) // 8, dtype=torch.int64, device=dev)
        self.km = scv.KernelMap(n, n, self.k3, dev)
        self.y = torch.empty((n, self.cout), dtype=self.dt, device=dev)
        self.dx = torch.empty((n, self.cin), dtype=self.dt, device=dev)
        self.dw = torch.empty((self.k3, self.cin, self.cout), dtype=torch.float32, device=dev)
        self.geom = scv.subm_geom(wl.ksize)
        c = self.km.c
        self.wsb = self.ws.get(max(scv.lat_kmap_ws_bytes(n, self.k3),
                                   *(scv.lat_sconv_ws_bytes(op, self.cin, self.cout, c, self.dt) for op in range(3))))
        # the data gradient's own workspace (its tile counter) and stream
        self.ws_side = scv.Workspace(dev)
        self.wsb_side = self.ws_side.get(scv.lat_sconv_ws_bytes(1, self.cin, self.cout, c, self.dt))
        self.side = torch.cuda.Stream(device=dev, priority=torch.cuda.Stream.priority_range()[1])
        self.ev_fwd, self.ev_dgrad = torch.cuda.Event(), torch.cuda.Event()
        self.overlap = True  # False: the data gradient on the current stream too (per-pass timing)
        self.pairs = None

    def step(self, ev: dict | None = None):
        scv, d, s = self.scv, self.d, self.status
        ev = ev or {}
        cur = torch.cuda.current_stream(self.dev)

        def rec(p, i, stream=cur):
            if p in ev:
                ev[p][i].record(stream)

        rec("hash", 0)
        scv.lat_hash_build(d["coords"], self.table, s)
        rec("hash", 1)
        rec("kmap", 0)
        scv.lat_kmap_query(self.table, d["coords"], self.geom, self.km.c, self.wsb, s)
        rec("kmap", 1)
        rec("conv_span", 0)
        rec("fwd", 0)
        scv.lat_sconv_fwd(d["x"], d["w"], self.km.c, self.y, self.wsb, s)
        rec("fwd", 1)
        dstream = self.side if self.overlap else cur
        self.ev_fwd.record(cur)
        dstream.wait_event(self.ev_fwd)
        rec("dgrad", 0, dstream)
        scv.lat_sconv_dgrad(d["g"], d["w"], self.km.c, True, self.dx, self.wsb_side, s, stream=dstream)
        rec("dgrad", 1, dstream)
        self.ev_dgrad.record(dstream)
        rec("wgrad", 0)
        scv.lat_sconv_wgrad(d["x"], d["g"], self.km.c, self.dw, self.wsb, s)
        rec("wgrad", 1)
        cur.wait_event(self.ev_dgrad)
        rec("conv_span", 1)

    def outputs(self) -> dict:
        return {"y": self.y, "dx": self.dx, "dw": self.dw}

    def pair_count(self) -> int:
        if self.pairs is None:
            self.pairs = int(self.km.pair_off[self.k3].item())
        return self.pairs

    def phase_flops(self) -> dict:
        f = 2.0 * self.pair_count() * self.cin * self.cout
        return {"hash": 0.0, "kmap": 0.0, "fwd": f, "dgrad": f, "wgrad": f}

    def flops(self) -> float:
        return sum(self.phase_flops().values())

    def phase_bytes(self) -> dict:
        """Algorithmic bytes per phase: the gathered rows, each output written
        once, the weights, one int32 pair of indices per pair (and, for the
        kernel map, the coordinates read and the table, mask and pairs written)."""
        n, p, k3, e = self.n, self.pair_count(), self.k3, self.dt.itemsize
        ci, co = self.cin, self.cout
        return {
            "hash": n * 16 + n * 16,
            "kmap": n * 16 + n * k3 * 4 + n * 4 + 8 * p,
            "fwd": p * ci * e + n * co * e + k3 * ci * co * e + 8 * p,
            "dgrad": p * co * e + n * ci * e + k3 * ci * co * e + 8 * p,
            "wgrad": p * (ci + co) * e + k3 * ci * co * 4 + 8 * p,
        }

    def extra_bytes(self) -> dict:
        """Bytes a phase moves beyond its algorithmic ones that the API makes it
        move: the hash table's clearing fill."""
        return {"hash_table_fill": self.table.numel() * 8}

    def kmap_rows(self) -> int:
        return self.n

    def check(self, host: dict) -> dict:
        """Outputs of the last step against the oracle (full outputs; kernel map bit for bit)."""
        import oracle
        coords = host["coords"].numpy()
        pad = oracle.subm_pad(self.wl.ksize)
        nbr = oracle.kmap(coords, coords, self.wl.ksize, 1, pad, oracle.SUBM)
        got_nbr = self.km.nbr_table().cpu().numpy()
        x, g, w = (host[k].double().numpy() for k in ("x", "g", "w"))
        ax, ag, aw = np.abs(x), np.abs(g), np.abs(w)
        out = {"kmap_bit_exact": bool(np.array_equal(got_nbr, nbr))}
        refs = {"y": (oracle.conv_fwd(x, w, nbr), oracle.conv_fwd(ax, aw, nbr)),
                "dx": (oracle.conv_dgrad(g, w, nbr, self.n), oracle.conv_dgrad(ag, aw, nbr, self.n)),
                "dw": (oracle.conv_wgrad(x, g, nbr), oracle.conv_wgrad(ax, ag, nbr))}
        outs = self.outputs()
        for k, (ref, terms) in refs.items():
            out[k] = err_stats(outs[k].double().cpu().numpy(), ref, terms, self.dt)
        return out


class DownUpLayer:
    """Strided Conv3d k2s2 onto the support it generates, then ConvTranspose3d
    k2s2 back onto the fine support, on the current stream: coarse support with
    each fine row's coarse row (its count read by the host), strided and
    transposed maps from those parent rows, down conv, up conv."""

    PHASES = ["downsample", "maps", "down_fwd", "up_fwd"]
    CONV = ["down_fwd", "up_fwd"]

    def __init__(self, name: str, host: dict, dev: torch.device):
        import sparse_convolution_voxel_b200 as scv
        self.scv, self.name, self.dev = scv, name, dev
        wl = self.wl = synthetic.WORKLOADS[name]
        self.dt = TORCH_DT[wl.dtype]
        self.cin, self.cmid = wl.cin, wl.cout
        self.d = {k: v.to(dev) for k, v in host.items()}
        n = self.n = host["coords"].shape[0]
        self.status = scv.new_status(dev)
        self.ws = scv.Workspace(dev)
        self.g_down = scv.strided_geom(2, 2, 0)
        self.coarse = torch.empty((n, 4), dtype=torch.int32, device=dev)
        self.parent = torch.empty(n, dtype=torch.int32, device=dev)
        self.nc = scv.lat_downsample_coords(self.d["coords"], self.g_down, self.coarse,
                                            self.ws.get(scv.lat_downsample_ws_bytes(n, self.g_down)), self.status,
                                            parent=self.parent)
        nc = self.nc
        self.km_down = scv.KernelMap(n, nc, 8, dev)
        self.km_up = scv.KernelMap(nc, n, 8, dev)
        self.yc = torch.empty((nc, self.cmid), dtype=self.dt, device=dev)
        self.z = torch.empty((n, self.cin), dtype=self.dt, device=dev)
        self.wsb = self.ws.get(max(scv.lat_downsample_ws_bytes(n, self.g_down),
                                   scv.lat_kmap_from_parent_ws_bytes(n, nc, 8),
                                   scv.lat_sconv_ws_bytes(0, self.cin, self.cmid, self.km_down.c, self.dt),
                                   scv.lat_sconv_ws_bytes(0, self.cmid, self.cin, self.km_up.c, self.dt)))
        self.nc_host = torch.empty(1, dtype=torch.int64, pin_memory=True)
        self.nc_view = self.nc_host.numpy()
        self.nc_ready = torch.cuda.Event()

    def step(self, ev: dict | None = None):
        scv, d, s = self.scv, self.d, self.status
        ev = ev or {}
        cur = torch.cuda.current_stream(self.dev)

        def rec(p, i):
            if p in ev:
                ev[p][i].record(cur)

        rec("downsample", 0)
        scv.lat_downsample_coords_async(d["coords"], self.g_down, self.coarse, self.wsb, self.nc_host, s,
                                        parent=self.parent)
        self.nc_ready.record(cur)
        self.nc_ready.synchronize()
        nc = int(self.nc_view[0])
        if nc < 0:  # coarse fields too wide for the bitmap: the blocking radix-sort path
            nc = scv.lat_downsample_coords(d["coords"], self.g_down, self.coarse, self.wsb, s, parent=self.parent)
        rec("downsample", 1)
        if nc != self.nc:
            raise RuntimeError(f"coarse row count changed: {nc} != {self.nc}")
        rec("maps", 0)
        scv.lat_kmap_from_parent(d["coords"], self.parent, self.g_down, self.km_down.c, self.km_up.c, self.wsb, s)
        rec("maps", 1)
        rec("down_fwd", 0)
        scv.lat_sconv_fwd(d["x"], d["wd"], self.km_down.c, self.yc, self.wsb, s)
        rec("down_fwd", 1)
        rec("up_fwd", 0)
        scv.lat_sconv_fwd(self.yc, d["wu"], self.km_up.c, self.z, self.wsb, s)
        rec("up_fwd", 1)

    def outputs(self) -> dict:
        return {"y_coarse": self.yc, "z": self.z}

    def phase_flops(self) -> dict:
        f = 2.0 * self.n * self.cin * self.cmid  # k = s: one pair per fine row in both relations
        return {"downsample": 0.0, "maps": 0.0, "down_fwd": f, "up_fwd": f}

    def flops(self) -> float:
        return sum(self.phase_flops().values())

    def pair_count(self) -> int:
        return self.n

    def phase_bytes(self) -> dict:
        n, nc, e, ci, cm = self.n, self.nc, self.dt.itemsize, self.cin, self.cmid
        return {
            "downsample": n * 16 + nc * 16 + n * 4,
            "maps": n * 16 + n * 4 + (nc + n) * 8 * 4 + 2 * 8 * n,
            "down_fwd": n * ci * e + nc * cm * e + 8 * ci * cm * e + 8 * n,
            "up_fwd": n * cm * e + n * ci * e + 8 * ci * cm * e + 8 * n,
        }

    def extra_bytes(self) -> dict:
        return {}

    def kmap_rows(self) -> int:
        return self.n

    def check(self, host: dict) -> dict:
        import oracle
        coords = host["coords"].numpy()
        ref_coarse = oracle.downsample(coords, 2, 2, 0)
        got_coarse = self.coarse[:self.nc].cpu().numpy()
        down = oracle.kmap(coords, ref_coarse, 2, 2, 0, oracle.STRIDED)
        up = oracle.kmap(ref_coarse, coords, 2, 2, 0, oracle.TRANSPOSED)
        out = {"coarse_bit_exact": bool(np.array_equal(got_coarse, ref_coarse)),
               "kmap_bit_exact": bool(np.array_equal(self.km_down.nbr_table().cpu().numpy(), down)
                                      and np.array_equal(self.km_up.nbr_table().cpu().numpy(), up))}
        x, wd, wu = (host[k].double().numpy() for k in ("x", "wd", "wu"))
        yc = self.yc.double().cpu().numpy()  # the up pass consumes the GPU's rounded coarse features
        out["y_coarse"] = err_stats(yc, oracle.conv_fwd(x, wd, down), oracle.conv_fwd(np.abs(x), np.abs(wd), down),
                                    self.dt)
        out["z"] = err_stats(self.z.double().cpu().numpy(), oracle.conv_fwd(yc, wu, up),
                             oracle.conv_fwd(np.abs(yc), np.abs(wu), up), self.dt)
        return out


def err_stats(got: np.ndarray, ref: np.ndarray, terms: np.ndarray, dtype: torch.dtype) -> dict:
    """The tests' normwise check (max|err| / max|ref| against the dtype's
    tolerance) and the per-element error relative to the sum of the absolute
    values of the terms summed into that element (p50 / p99 / max over the
    elements that have any term)."""
    err = np.abs(got - ref)
    scale = max(float(np.abs(ref).max(initial=0.0)), 1e-300)
    norm = float(err.max(initial=0.0)) / scale
    sel = terms > 0
    rel = err[sel] / terms[sel]
    q = np.percentile(rel, [50, 99]) if rel.size else [0.0, 0.0]
    return {"max_err_over_max_ref": norm, "tol": REL_TOL[dtype], "pass": bool(norm <= REL_TOL[dtype]),
            "rel_terms_p50": float(q[0]), "rel_terms_p99": float(q[1]),
            "rel_terms_max": float(rel.max(initial=0.0)), "elements": int(err.size),
            "nonfinite": int((~np.isfinite(got)).sum())}


# --------------------------------------------------------------------------- timing helpers
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
                "sm_mhz_min": min(c for c, _ in self.samples), "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml"}


def new_events(names) -> dict:
    return {p: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for p in names}


def phase_times(layer, flush: torch.Tensor, reps: int, overlap: bool = False) -> dict:
    """Mean per-phase event time (ms) over `reps` instrumented steps, L2 flushed
    before each (events between phases; outside any timed region).  With
    overlap=False a layer that runs two passes side by side runs them one
    after the other, so each phase's time is its own."""
    names = layer.PHASES + getattr(layer, "SPANS", [])
    inst = [new_events(names) for _ in range(reps)]
    prev = getattr(layer, "overlap", None)
    if prev is not None:
        layer.overlap = overlap
    try:
        torch.cuda.synchronize()
        for ev in inst:
            flush_l2(flush)
            layer.step(ev)
        torch.cuda.synchronize()
    finally:
        if prev is not None:
            layer.overlap = prev
    return {p: statistics.mean(ev[p][0].elapsed_time(ev[p][1]) for ev in inst) for p in names}


def roofline_of(layer, phase_ms: dict, peaks: dict, fp32_tflops: float | None) -> dict:
    """Per-phase fraction of roofline: t_roofline = max(alg bytes / HBM, flops /
    compute peak) over the phase's measured time; the compute peak is the
    measured bf16 tensor rate for 16-bit inputs, the measured fp32 FMA rate
    otherwise."""
    pb, pf = layer.phase_bytes(), layer.phase_flops()
    comp = peaks["bf16_tflops"] if layer.dt != torch.float32 else (fp32_tflops or 74.4)
    out, t_roof_sum = {}, 0.0
    for p in layer.PHASES:
        t_mem = pb[p] / (peaks["hbm_gbs"] * 1e9)
        t_cmp = pf[p] / (comp * 1e12)
        t_roof = max(t_mem, t_cmp)
        t_roof_sum += t_roof
        t = phase_ms[p] * 1e-3
        out[p] = {"ms": round(phase_ms[p], 5), "alg_bytes": int(pb[p]),
                  "achieved_gbs": round(pb[p] / t / 1e9, 1) if t > 0 else None,
                  "bound": "hbm" if t_mem >= t_cmp else "compute",
                  "frac": round(t_roof / t, 4) if t > 0 else None}
    return {"phases": out, "t_roofline_ms": t_roof_sum * 1e3}


def time_steps(layer, flush: torch.Tensor, steps: int, dev, extra_ev: str | None = None):
    """`steps` steps, L2 flushed before each, CUDA events around each step on the
    current stream (and around phase `extra_ev`, if given), clocks sampled
    throughout.  Returns (step ms list, extra phase ms list, clock summary)."""
    evs = [{"step": (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))}
           for _ in range(steps)]
    if extra_ev:
        for ev in evs:
            ev.update(new_events([extra_ev]))
    cur = torch.cuda.current_stream(dev)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        for ev in evs:
            flush_l2(flush)
            ev["step"][0].record(cur)
            layer.step({extra_ev: ev[extra_ev]} if extra_ev else None)
            ev["step"][1].record(cur)
        clk.mark_end()
        torch.cuda.synchronize()
    step_ms = [ev["step"][0].elapsed_time(ev["step"][1]) for ev in evs]
    extra_ms = [ev[extra_ev][0].elapsed_time(ev[extra_ev][1]) for ev in evs] if extra_ev else []
    return step_ms, extra_ms, clk.summary()


def count_launches(layer) -> int:
    """Kernels one step launches, counted with the CUDA profiler (outside timing)."""
    from torch.profiler import ProfilerActivity, profile
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        layer.step()
        torch.cuda.synchronize()
    n = 0
    for e in prof.events():
        if e.device_type == torch.autograd.DeviceType.CUDA and "memset" not in e.name.lower() \
                and "memcpy" not in e.name.lower():
            n += 1
    return n


def config_entry(name: str, dev, flush, peaks, fp32_tflops, min_ms: float = 400.0) -> dict:
    """One workload's own measurement: warm-up, per-phase times, timed steps
    (at least 20, and about `min_ms` of device time), clocks, oracle errors."""
    host = make_host(name)
    layer = make_layer(name, host, dev)
    for _ in range(5):
        layer.step()
    torch.cuda.synchronize()
    st = layer.scv.lat_status_fetch(layer.status)
    if st:
        raise layer.scv.LatticeError(st, f"{name}: device status after warm-up")
    pms = phase_times(layer, flush, 10)
    spans = phase_times(layer, flush, 10, overlap=True) if getattr(layer, "SPANS", None) else {}
    est = sum(pms[p] for p in layer.PHASES)
    steps = int(min(2000, max(20, min_ms / max(est, 1e-3))))
    step_ms, _, clocks = time_steps(layer, flush, steps, dev)
    t = statistics.mean(step_ms)
    rl = roofline_of(layer, pms, peaks, fp32_tflops)
    kmap_phases = [p for p in ("hash", "kmap", "downsample", "maps") if p in pms]
    kmap_ms = sum(pms[p] for p in kmap_phases)
    # the passes' wall span in the timed schedule (two of them side by side), else their sum
    conv_ms = spans.get("conv_span", sum(pms[p] for p in layer.CONV))
    entry = {
        "workload": synthetic.WORKLOADS[name].description, "dtype": synthetic.WORKLOADS[name].dtype,
        "rows": layer.n, "pairs": layer.pair_count(), "steps": steps, "ms_per_step": t,
        "ms_per_step_median": statistics.median(step_ms),
        "tflops": layer.flops() / (t * 1e-3) / 1e12,
        "conv_tflops": layer.flops() / (conv_ms * 1e-3) / 1e12,
        "kmap_mvoxels_per_s": layer.kmap_rows() / (kmap_ms * 1e-3) / 1e6, "kmap_phases": kmap_phases,
        "frac_roofline_step": rl["t_roofline_ms"] / t, "phases": rl["phases"],
        "extra_bytes": layer.extra_bytes(), "clocks": clocks,
    }
    if isinstance(layer, DownUpLayer):
        entry["coarse_rows"] = layer.nc
    torch.cuda.synchronize()
    entry["errors"] = layer.check(host)
    del layer
    torch.cuda.empty_cache()
    return entry


# --------------------------------------------------------------------------- CPU oracle arm
def oracle_train_step(host: dict, ksize, nthreads: int = 0, rows: int | None = None) -> dict:
    """One oracle SubmConv3d training step (kernel map, fwd, dgrad, wgrad) over
    the first `rows` output rows (all by default); returns seconds per pass and
    the pair count processed."""
    import oracle
    c = host["coords"].numpy()
    q = c if rows is None else c[:rows]
    x = host["x"].double().numpy()
    g = host["g"].double().numpy()[:len(q)]
    w = host["w"].double().numpy()
    pad = oracle.subm_pad(ksize)
    t = {}
    t0 = time.perf_counter()
    nbr = oracle.kmap(c, q, ksize, 1, pad, oracle.SUBM, nthreads)
    t["kmap"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.conv_fwd(x, w, nbr, nthreads)
    t["fwd"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.conv_dgrad(g, w, nbr, len(c), nthreads)
    t["dgrad"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.conv_wgrad(x, g, nbr, nthreads)
    t["wgrad"] = time.perf_counter() - t0
    return {"s": t, "pairs": int((nbr >= 0).sum()), "rows": len(q)}


def cpu_baseline(host: dict, budget_s: float = 20.0) -> dict:
    """The oracle on the host cores: whole training steps of the headline
    workload until about `budget_s` has passed (at least 1 step)."""
    import oracle
    wl = synthetic.WORKLOADS[WORKLOAD]
    cores = oracle.max_threads()
    times, flops = [], 0.0
    t_all = time.perf_counter()
    while True:
        r = oracle_train_step(host, wl.ksize)
        times.append(sum(r["s"].values()))
        flops = 3 * 2.0 * r["pairs"] * wl.cin * wl.cout
        if time.perf_counter() - t_all > budget_s or len(times) >= 5:
            break
    t = statistics.median(times)
    return {"value": flops / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(times)} whole oracle training steps of {WORKLOAD} (kernel map + fwd + dgrad + wgrad, "
                      f"fp64; median {t:.2f} s per step)"}


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return
    import oracle
    wl = synthetic.WORKLOADS[WORKLOAD]
    host = make_host(WORKLOAD)
    cores = oracle.max_threads()
    # each step is a bounded sample: the kernel map and the three passes over
    # the first `rows` output rows (the whole workload at --sample-rows 0)
    rows = args.sample_rows if args.sample_rows > 0 else None
    for _ in range(args.warmup):
        oracle_train_step(host, wl.ksize, rows=rows)
    times, flops = [], 0.0
    for _ in range(args.steps):
        r = oracle_train_step(host, wl.ksize, rows=rows)
        times.append(sum(r["s"].values()))
        flops = 3 * 2.0 * r["pairs"] * wl.cin * wl.cout
    total = sum(times)
    value = flops * args.steps / total / 1e12
    sample = (f"oracle training step (kernel map + fwd + dgrad + wgrad, fp64) over the first {r['rows']} of "
              f"{host['coords'].shape[0]} output rows ({r['pairs']} pairs) of {WORKLOAD}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(host["coords"].shape[0], world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_cpu_table(args):
    """The oracle per workload and pass, single-threaded and on all cores, median
    of 3; single-threaded runs of the large workloads take the first rows only
    (the rate is per pair).  Prints one JSON line."""
    import oracle
    cores = oracle.max_threads()
    cpu = platform.processor() or ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                cpu = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    table = {}
    for name in CONFIG_ORDER:
        if name == "lidar_down_up":
            continue
        wl = synthetic.WORKLOADS[name]
        host = make_host(name)
        n = host["coords"].shape[0]
        row = {}
        for label, nt, rows in (("all_cores", 0, None), ("single_thread", 1, None if n <= 50_000 else n // 16)):
            runs = [oracle_train_step(host, wl.ksize, nt, rows) for _ in range(3)]
            med = {p: statistics.median(r["s"][p] for r in runs) for p in runs[0]["s"]}
            pairs = runs[0]["pairs"]
            f = 2.0 * pairs * wl.cin * wl.cout
            row[label] = {"threads": cores if nt == 0 else 1, "rows": runs[0]["rows"], "pairs": pairs,
                          "s": {p: round(v, 4) for p, v in med.items()},
                          "gflops": {p: round(f / med[p] / 1e9, 3) for p in ("fwd", "dgrad", "wgrad")},
                          "kmap_mvoxels_per_s": round(runs[0]["rows"] / med["kmap"] / 1e6, 3)}
        table[name] = row
    print(json.dumps({"cpu_table": table, "cpu": cpu, "cores": cores, "median_of": 3}), flush=True)


def config_dict(n, world):
    return {"workload": f"{WORKLOAD}: SubmConv3d k=3 training step (hash + kernel map + fwd + dgrad + wgrad), "
                        f"batch 4 x 125k LiDAR-shaped voxels in a 1440x1440x41 grid, bf16, 128->128, upstream grad "
                        f"N(0,1)",
            "voxels_per_gpu": int(n), "global_batch": 4 * world, "parallelism": f"replicas x{world}",
            "streams": "hash, kernel map, fwd, wgrad on one stream; dgrad on a second stream beside wgrad",
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
    dt = TORCH_DT[wl.dtype]
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
    if args.only in ("down_fwd", "up_fwd"):
        # strided Conv3d k2s2 Cin -> 2 Cin onto the generated coarse support (maps from
        # parents), and the ConvTranspose3d 2 Cin -> Cin back onto the fine support
        g_dn = scv.strided_geom(2, 2, 0)
        coarse_d, par = scv.downsample(coords, g_dn, ws, with_parent=True)
        ncd = coarse_d.shape[0]
        km_d, km_u = scv.maps_from_parent(coords, par.contiguous(), ncd, g_dn, ws, st)
        cd = 2 * cin
        wd = torch.from_numpy(synthetic.weights(8, cin, cd, wl.seed)).to(dt).to(dev)
        wu = torch.from_numpy(synthetic.weights(8, cd, cin, wl.seed, 1)).to(dt).to(dev)
        yd = torch.empty((ncd, cd), dtype=dt, device=dev)
        zd = torch.empty((n, cin), dtype=dt, device=dev)
        wsd = torch.empty(max(1, scv.lat_sconv_ws_bytes(0, cin, cd, km_d.c, dt),
                              scv.lat_sconv_ws_bytes(0, cd, cin, km_u.c, dt)), dtype=torch.uint8, device=dev)
        scv.lat_sconv_fwd(x, wd, km_d.c, yd, wsd, st)
        torch.cuda.synchronize()
        ops["down_fwd"] = (lambda: scv.lat_sconv_fwd(x, wd, km_d.c, yd, wsd, st),
                           n * cin * e + ncd * cd * e + 8 * cin * cd * e + 8 * n)
        ops["up_fwd"] = (lambda: scv.lat_sconv_fwd(yd, wu, km_u.c, zd, wsd, st),
                         n * cd * e + n * cin * e + 8 * cin * cd * e + 8 * n)
    if args.only == "dense":
        # dense grid over the coordinates' bounding box: the whole grid written once, rows read once
        lo, hi = coords.amin(0).tolist(), coords.amax(0).tolist()
        box = [hi[a + 1] - lo[a + 1] + 1 for a in range(3)]
        grid = torch.empty((hi[0] + 1, *box, cin), dtype=dt, device=dev)
        ops["dense"] = (lambda: scv.lat_to_dense(coords, x, lo[1:], box, hi[0] + 1, grid, st),
                        grid.numel() * e + n * 16 + n * cin * e)
    fn, nbytes = ops[args.only]
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    ms = []
    with ClockSampler(dev) as clk:
        for _ in range(args.steps):
            flush_l2(flush)
            a, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            bb.record()
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(bb))
        clk.mark_end()
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
    hbm = load_peaks()
    print(json.dumps({"only": args.only, "workload": args.workload, "rsv_ratio": args.rsv_ratio, "rows": n,
                      "pairs": P, "ms_median": t, "ms_min": min(ms), "alg_bytes": nbytes,
                      "achieved_gbs": nbytes / (t * 1e-3) / 1e9,
                      "frac_hbm": nbytes / (t * 1e-3) / 1e9 / hbm["hbm_gbs"], "peak_source": hbm["source"],
                      "status": stv, "host_us_per_call": host_us, "b2b_ms_per_call": b2b_ms,
                      "clocks": clk.summary()}), flush=True)


# --------------------------------------------------------------------------- end to end
def measure_e2e(host: dict, dev: torch.device, steps: int) -> dict:
    """The headline step through the public API with HOST buffers: every step's
    inputs (coordinates, features, upstream gradient, weights) are copied in
    from pinned host memory and all of its results (y, dx, dW) copied back,
    copies inside the timed region.  Steps alternate between two device buffer
    sets: step i+1's inputs are copied in (two H2D streams) and step i-1's
    results copied out (D2H stream) while step i computes; the L2 is flushed
    before every step's compute.  Time = first copy-in start to last copy-out end."""
    pinned = {k: v.pin_memory() for k, v in host.items()}
    layers = [SubmLayer(WORKLOAD, host, dev), SubmLayer(WORKLOAD, host, dev)]
    outs = [{k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in L.outputs().items()} for L in layers]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in outs[0].values())
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    comp, up, up2, down = (torch.cuda.Stream(dev) for _ in range(4))
    order = sorted(pinned, key=lambda k: -pinned[k].numel() * pinned[k].element_size())
    computed = [torch.cuda.Event() for _ in layers]    # the set's last step finished computing
    copied_out = [torch.cuda.Event() for _ in layers]  # its results reached the host
    inputs_in = [[torch.cuda.Event(), torch.cuda.Event()] for _ in layers]

    def copy_in(i: int):
        b = i % 2
        L = layers[b]
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(computed[b])  # the set's previous step has read its inputs
            began = torch.cuda.Event()
            began.record()
        up2.wait_event(began)
        for c, k in enumerate(order):
            with torch.cuda.stream(up if c % 2 == 0 else up2):
                L.d[k].copy_(pinned[k], non_blocking=True)
        inputs_in[b][0].record(up)
        inputs_in[b][1].record(up2)

    def run(n: int, start=None, end=None):
        if start is not None:
            start.record(up)
        copy_in(0)
        for i in range(n):
            b = i % 2
            L, o = layers[b], outs[b]
            if i + 1 < n:
                copy_in(i + 1)
            with torch.cuda.stream(comp):
                comp.wait_event(inputs_in[b][0])
                comp.wait_event(inputs_in[b][1])
                if i >= 2:
                    comp.wait_event(copied_out[b])  # its previous results have left
                flush_l2(flush)
                L.step()
                computed[b].record()
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                for k, v in L.outputs().items():
                    o[k].copy_(v, non_blocking=True)
                copied_out[b].record()
                if i == n - 1 and end is not None:
                    end.record()

    run(4)
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev) as clk:
        run(steps, a, e)
        clk.mark_end()
        torch.cuda.synchronize()
    t = a.elapsed_time(e) / steps
    return {"value": layers[0].flops() / (t * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": t, "steps": steps,
            "overlap": "copies of the next step's inputs (two H2D streams) and the previous step's results run "
                       "during each step; two buffer sets; L2 flushed before each step's compute",
            "result_read_back": "y (bf16), dx (bf16) and dW (fp32) of every step", "clocks": clk.summary()}


# --------------------------------------------------------------------------- main GPU arm
# The kernel the roofline object reports: the path kernel with the largest
# share of the headline step's ncu launch list.
DOMINANT = "fwd"
DOMINANT_KERNEL = "conv_tc_kernel<bf16, 128, 128>, forward: gathered x times W[k] on tcgen05"
# DRAM bytes (read + write) per launch of that phase's kernel from an ncu
# capture of the current kernel on the same workload (None: no capture
# matches the kernel as it is).
PHASE_TRAFFIC = {"fwd": 168_960_000 + 83_851_264}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload entries")
    ap.add_argument("--only", choices=["hash", "kmap", "fwd", "dgrad", "wgrad", "downsample", "upsample", "pool_max",
                                       "pool_avg", "pool_down", "dense", "down_fwd", "up_fwd"],
                    help="time a single op of the path on --workload (for profiler captures)")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--rsv-ratio", type=float, default=RSV_RATIO, help="hash table slots per voxel (--only mode)")
    ap.add_argument("--sample-rows", type=int, default=250_000,
                    help="--impl reference: output rows per oracle step (0 = all)")
    ap.add_argument("--cpu-table", action="store_true", help="time the oracle per workload and pass")
    ap.add_argument("--lean", action="store_true",
                    help="skip launch counting, the end-to-end pass, the per-workload entries and the CPU baseline "
                         "(for profiler runs)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    world, rank, local = dist_env()
    if args.impl == "reference":
        return run_reference(args)
    if args.cpu_table:
        return run_cpu_table(args)
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
    peaks = load_peaks()

    host = make_host(WORKLOAD, rank)
    layer = SubmLayer(WORKLOAD, host, dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        layer.step()
    torch.cuda.synchronize()
    st = scv.lat_status_fetch(layer.status)
    if st:
        raise scv.LatticeError(st, "device status after warm-up")
    launches_per_step = None if args.lean else count_launches(layer)
    pms = phase_times(layer, flush, 10)

    if pg:
        pg.barrier()
    step_ms, dom_ms, clocks = time_steps(layer, flush, args.steps, dev, DOMINANT)
    if pg:
        pg.barrier()
    total_ms = sum(step_ms)
    if pg:
        total_ms = max_over_ranks(total_ms, pg, dev)
    flops = layer.flops()
    value = job_throughput(flops, world, args.steps, total_ms)

    if rank == 0:
        fp32 = {"skipped": "--lean"}
        rowcopy = {"skipped": "--lean"}
        if not args.lean:
            try:
                from sparse_convolution_voxel_b200 import measure
                fp32 = measure.ffma_peak(dev)
                rowcopy = measure.gather_peak(dev, n=layer.n, row_bytes=layer.cin * layer.dt.itemsize)
            except Exception as exc:  # the probe library is optional for the headline
                fp32 = rowcopy = {"error": str(exc)}
        fp32_tflops = fp32.get("tflops")
        rl = roofline_of(layer, pms, peaks, fp32_tflops)
        pb = layer.phase_bytes()
        dominant_ms = statistics.mean(dom_ms)
        achieved = pb[DOMINANT] / (dominant_ms * 1e-3) / 1e9
        kmap_ms = pms["hash"] + pms["kmap"]
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(layer.n, world),
            "kmap_mvoxels_per_s": layer.n / (kmap_ms * 1e-3) / 1e6,
            "pairs": layer.pair_count(),
            "phases": rl["phases"],
            "frac_roofline_step": rl["t_roofline_ms"] / (total_ms / args.steps),
            "phase_note": "per-phase event times from 10 instrumented steps outside the timed region, L2 flushed "
                          "before each, the passes one after another (the timed steps run dgrad on a second stream "
                          "beside wgrad); frac = t_roofline / t per phase",
            "roofline": {"kernel": f"{DOMINANT} ({DOMINANT_KERNEL})", "bound": "hbm", "achieved": achieved,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": PHASE_TRAFFIC.get(DOMINANT), "alg_bytes": pb[DOMINANT], "ms": dominant_ms,
                         "peak_source": f"{peaks['source']} hbm_gbs (burst copy; the kernel is timed inside the step)",
                         "timing": "CUDA events around this phase on its stream in every timed step",
                         "frac_of_random_row_copy": (achieved / rowcopy["gbs"]) if "gbs" in rowcopy else None},
            "gpu_launches": None if launches_per_step is None else launches_per_step * args.steps,
            "launches_per_step": launches_per_step,
            "clocks": clocks,
            "peaks": {**peaks, "fp32_ffma": fp32, "random_row_copy": rowcopy},
        }
        del layer
        torch.cuda.empty_cache()
        if not args.lean and world == 1:
            line["e2e"] = measure_e2e(host, dev, steps=max(3, min(args.steps, 10)))
            torch.cuda.empty_cache()
        if not args.lean and not args.no_configs and world == 1:
            line["configs"] = {name: config_entry(name, dev, flush, peaks, fp32_tflops) for name in CONFIG_ORDER}
            line["errors"] = line["configs"][WORKLOAD]["errors"]
        if not args.no_cpu_baseline and not args.lean and world == 1:
            line["cpu_baseline"] = cpu_baseline(host)
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
