#!/usr/bin/env python
"""Throughput of the W8A8 selective-scan hot path on B200.

One step = one Mamba-130M-shaped W8A8 layer pass (b 8, L 2048, d 1536, N 16,
G 1, z gate): group-quantize binary16 x (8 sorted-and-clustered channel
groups), B and C (one scale per 4 states) with static calibrated scales, then
the Mamba-1 selective scan.  Metric: Gtokens*ch/s = b L d / step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank scans its own independent layer batch
(weak scaling, no data-path collective); only the timing is reduced (max over
ranks).  --impl reference times the CPU oracle (double precision, all host
cores) on a bounded sample of the same workload.
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 scan Gtokens·ch/s and HBM GB/s (frac of roofline) on 1 B200"
UNIT = "Gtokens·ch/s"
WORKLOAD = "m130m"
SMS = 148
MUFU_PER_CLK = 16  # ex2 results per clock per SM (SFU)


def measured_traffic(kernel):
    """DRAM bytes per launch of `kernel` from one ncu capture
    (profiles/traffic.json: dram__bytes_read.sum + dram__bytes_write.sum),
    or None once any of its source files has changed since that capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            e = json.load(f)["kernels"][kernel]
        h = hashlib.sha256()
        for rel in e["sources"]:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        return e["bytes_per_launch"] if h.hexdigest() == e["sha256"] else None
    except (OSError, KeyError, ValueError):
        return None


def peaks():
    p = {"hbm_gbs": 6531.0, "bf16_tflops": 1602.0, "sm_max_mhz": 1965.0, "source": "measured"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        p.update({k: float(m[k]) for k in ("hbm_gbs", "bf16_tflops", "sm_max_mhz") if k in m})
        p["bf16_tflops_sustained"] = float(m.get("bf16_tflops_sustained", p["bf16_tflops"]))
    except (OSError, ValueError, KeyError):
        p.update({"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"})
    return p


def config_dict(dm):
    return {"workload": "m130m: Mamba-130M-shaped W8A8 layer (quantize x/B/C + selective scan)",
            "batch": dm["batch"], "seqlen": dm["seqlen"], "d_inner": dm["dim"],
            "d_state": dm["dstate"], "ngroups": dm["ngroups"], "x_clusters": dm["x_clusters"],
            "bc_state_group": dm["state_group_size"], "gate": "silu(z)",
            "operands": "int8 x/B/C with fp32 scales, f16 dt/z/y, f32 state",
            "l2": "inputs exceed L2 (f16 x, dt, z, y = 201 MB per step)"}


# ---- clocks ------------------------------------------------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    """Samples the SM clock and clock-event reasons with NVML in a thread."""

    def __init__(self, torch_dev, period=0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period
        self.ok = False
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            props = __import__("torch").cuda.get_device_properties(torch_dev)
            bus = "%08X:%02X:%02X.0" % (getattr(props, "pci_domain_id", 0), props.pci_bus_id,
                                        props.pci_device_id)
            try:
                self.h = nv.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = nv.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.reason_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.ok = True
        except Exception as e:  # no NVML: report that, do not fail the bench
            self.err = str(e)

    def _run(self):
        while not self.stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.reason_fn(self.h)
                for bit, name in _REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.stop = threading.Event()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---- the workload ------------------------------------------------------------

class Layer:
    """Inputs (resident in HBM), static calibration and outputs of one step."""

    def __init__(self, dev, seed, fused=False):
        import torch

        from quantized_state_space_b200 import calibrate, synth
        self.dm, raw = synth.workload_inputs(WORKLOAD, seed=seed)
        dm = self.dm
        self.b, self.L, self.d = dm["batch"], dm["seqlen"], dm["dim"]
        self.N, self.G, self.gs, self.k = dm["dstate"], dm["ngroups"], dm["state_group_size"], \
            dm["x_clusters"]
        # offline calibration (untimed)
        grp, xs = calibrate.m1_x_clusters(raw["x"], self.k)
        bs = calibrate.state_group_absmax_scales(raw["B"], self.G, self.N, self.gs, "gnl")
        cs = calibrate.state_group_absmax_scales(raw["C"], self.G, self.N, self.gs, "gnl")
        smap = calibrate.state_group_map(self.G, self.N, self.gs)
        self.raw = raw
        T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
        self.host = {k: torch.from_numpy(raw[k]).pin_memory() for k in ("x", "dt", "z", "B", "C")
                     if raw.get(k) is not None}
        self.x, self.dt, self.z, self.B, self.C = (None if raw.get(k) is None else T(raw[k])
                                                   for k in ("x", "dt", "z", "B", "C"))
        self.A, self.D = T(raw["A"]), T(raw["D"])
        self.grp, self.xs, self.bs, self.cs, self.smap = T(grp), T(xs), T(bs), T(cs), T(smap)
        self.xq = torch.empty(self.x.shape, dtype=torch.int8, device=dev)
        self.Bq = torch.empty(self.B.shape, dtype=torch.int8, device=dev)
        self.Cq = torch.empty(self.C.shape, dtype=torch.int8, device=dev)
        self.y = torch.empty(self.x.shape, dtype=torch.float16, device=dev)
        self.hf = torch.empty((self.b, self.d, self.N), dtype=torch.float32, device=dev)
        self.units = self.b * self.L * self.d
        # fused: the scan reads binary16 x and quantizes it itself (the result
        # is byte-identical to quantizing x first); else x is quantized with
        # B and C and the scan reads the int8 codes
        self.fused = fused
        # x, B and C are quantized by one batched launch (B and C alone in
        # the fused form), then the scan
        self.launches_per_step = 2

    def quantize(self):
        from quantized_state_space_b200 import api
        b, L, d, G, N, gs = self.b, self.L, self.d, self.G, self.N, self.gs
        jobs = [(self.B, b, G * N, L, self.smap, G * N // gs, self.bs, self.Bq),
                (self.C, b, G * N, L, self.smap, G * N // gs, self.cs, self.Cq)]
        if not self.fused:
            jobs.insert(0, (self.x, b, d, L, self.grp, self.k, self.xs, self.xq))
        api.quantize_groups_batch(jobs)

    def scan(self, time_segments=1):
        from quantized_state_space_b200 import api
        api.selective_scan(self.x if self.fused else self.xq, self.dt, self.A, self.Bq, self.Cq,
                           self.bs, self.cs, self.gs, x_group=self.grp, x_scale=self.xs, D=self.D,
                           z=self.z, y=self.y, h_final=self.hf, time_segments=time_segments)

    def scan_bytes(self):
        """Algorithmic HBM bytes of one scan launch."""
        b, L, d, N, G = self.b, self.L, self.d, self.N, self.G
        xb = 2 if self.fused else 1                   # binary16 x or int8 codes
        return (b * d * L * (xb + 2 + 2 + 2)          # x, dt, z, y f16
                + 2 * b * G * N * L                   # B, C int8
                + d * N * 4 + d * 4 + b * d * N * 4)  # A, D, h_final

    def step_bytes(self):
        b, L, d, N, G = self.b, self.L, self.d, self.N, self.G
        xq = 0 if self.fused else b * d * L * 3
        return self.scan_bytes() + xq + 2 * 3 * b * G * N * L


def sfu_peak(ex2, mhz):
    """Scan roof in G state updates/s (one exponential each): the probe's
    measured rate, else the CUDA guide's 16 results per clock per SM."""
    if ex2 and ex2.get("gex2_per_s"):
        return ex2["gex2_per_s"], ("measured: ssmq_probe_ex2 in this run, %.1f G ex2/s "
                                   "(%s per SM per clock at %s MHz); one exp per state update"
                                   % (ex2["gex2_per_s"], ex2.get("per_sm_per_clock"),
                                      ex2.get("sm_mhz")))
    return SMS * MUFU_PER_CLK * mhz * 1e6 / 1e9, ("%d SMs x %d ex2/clk (SFU, CUDA guide "
                                                  "figure) x %.0f MHz" % (SMS, MUFU_PER_CLK, mhz))


def cuda_events(torch):
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def measure_ex2(torch, dev, reps=5):
    """Rate of the special-function unit's base-2 exponential on this GPU,
    measured with the library's own probe kernel (independent ex2 chains on
    every SM, CUDA events, the SM clock sampled meanwhile): the compute roof
    of the Mamba-1 scan, one exponential per state update."""
    from quantized_state_space_b200 import _native as N
    sink = torch.zeros(4, dtype=torch.float32, device=dev)
    iters = 2048
    for _ in range(3):
        N.ssmq_probe_ex2(iters, sink)
    torch.cuda.synchronize()
    times = []
    with ClockSampler(dev.index or 0, period=0.001) as clk:
        for _ in range(reps):
            a, b = cuda_events(torch)
            a.record()
            n = N.ssmq_probe_ex2(iters, sink)
            b.record()
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b) / 1e3)
    t = statistics.median(times)
    c = clk.summary()
    mhz = c.get("sm_mhz") or None
    rate = n / t / 1e9
    return {"gex2_per_s": round(rate, 1), "ms_per_launch": round(t * 1e3, 4), "n_ex2": n,
            "per_sm_per_clock": round(rate * 1e3 / (SMS * mhz), 3) if mhz else None,
            "sm_mhz": mhz, "sm_max_mhz": c.get("sm_max_mhz"), "reasons": c.get("reasons"),
            "method": "ssmq_probe_ex2: %d SMs x 8 CTAs x 256 threads x 8 independent ex2 "
                      "chains, median of %d launches (CUDA events)" % (SMS, reps)}


def cpu_baseline(layer, threads=None, max_units=None):
    """The oracle, as it stands, on the host cores: quantize + scan of a
    bounded sample of (batch, channel) rows of the same workload."""
    from oracle import oracle as O
    raw = layer.raw
    b, L, d, N, G, gs, k = layer.b, layer.L, layer.d, layer.N, layer.G, layer.gs, layer.k
    threads = threads or O.default_threads()
    n_units = max_units or b * d
    bb = max(1, n_units // d)
    units = np.arange(min(n_units, b * d))
    t0 = time.perf_counter()
    og, oxs = O.cluster_by_absmax(O.absmax_per_mid(raw["x"], b, d, L), k)
    smap = np.arange(G * N) // gs
    _, obs, _ = O.quantize_groups(raw["B"], b, G * N, L, smap, G * N // gs, O.SCALE_ABSMAX)
    _, ocs, _ = O.quantize_groups(raw["C"], b, G * N, L, smap, G * N // gs, O.SCALE_ABSMAX)
    t_cal = time.perf_counter() - t0
    t1 = time.perf_counter()
    xs = raw["x"][:bb]
    ox, _, _ = O.quantize_groups(xs, bb, d, L, og, k, O.SCALE_STATIC, oxs)
    oB, _, _ = O.quantize_groups(raw["B"][:bb], bb, G * N, L, smap, G * N // gs, O.SCALE_STATIC, obs)
    oC, _, _ = O.quantize_groups(raw["C"][:bb], bb, G * N, L, smap, G * N // gs, O.SCALE_STATIC, ocs)
    yo, ho = O.m1_scan(ox, raw["dt"][:bb], raw["A"], oB, oC, obs, ocs, gs, x_group=og,
                       x_scale=oxs, D=raw["D"], z=raw["z"][:bb], units=units[:bb * d],
                       threads=threads)
    dt = time.perf_counter() - t1
    units_done = bb * d * L
    layer.oracle_out = (bb, yo, ho)  # for the in-run parity check
    return {"value": units_done / dt / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": "%d of %d batch rows (%d channel rows x L %d): static quantize of "
                      "x/B/C + double-precision scan; calibration (%.1f s) untimed"
                      % (bb, b, bb * d, L, t_cal),
            "seconds": dt}


Y_TOL, STATE_TOL = 2e-3, 1e-4  # max |y - y_ref| / max |y_ref|; final-state relative L2


def parity(y_gpu, y_ref, h_gpu=None, h_ref=None, what=""):
    """Errors of the GPU result against the oracle on the same inputs, with
    the stated tolerances."""
    y, r = np.asarray(y_gpu, np.float64), np.asarray(y_ref, np.float64)
    out = {"y_max_err_rel": float(np.max(np.abs(y - r)) / max(np.max(np.abs(r)), 1e-30)),
           "y_tol": Y_TOL, "sample": what}
    if h_gpu is not None:
        h, hr = np.asarray(h_gpu, np.float64), np.asarray(h_ref, np.float64)
        out["state_rel_l2"] = float(np.linalg.norm(h - hr) / max(np.linalg.norm(hr), 1e-30))
        out["state_tol"] = STATE_TOL
    out["ok"] = out["y_max_err_rel"] <= Y_TOL and out.get("state_rel_l2", 0.0) <= STATE_TOL
    return out


# ---- ranks -----------------------------------------------------------------
# One process per GPU; every rank scans its own independent layer batch (the
# path has no exchange step), so the only cross-rank traffic is the reduction
# of the measured time.

def rank_env():
    """(world, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(rank):
    """Each rank draws an independent batch of the workload."""
    return rank


def max_over_ranks(value, dist=None, device=None):
    """The slowest rank's time (max over the process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world, units_per_rank, steps, ms_max):
    """Whole-job throughput: units of all ranks over the slowest rank's time,
    in giga-units per second."""
    return world * units_per_rank * steps / (ms_max / 1e3) / 1e9


# ---- our arm ----------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    from quantized_state_space_b200 import build_native
    if rank == 0:
        build_native.build()
    if world > 1:
        dist.barrier()
    pk = peaks()
    layer = Layer(dev, seed=rank_seed(rank), fused=args.fused)
    stream = torch.cuda.current_stream()

    def step():
        layer.quantize()
        layer.scan()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    K = args.steps
    scan_ev = [cuda_events(torch) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        e0, e1 = cuda_events(torch)
        e0.record(stream)
        for i in range(K):
            layer.quantize()
            scan_ev[i][0].record(stream)
            layer.scan()
            scan_ev[i][1].record(stream)
        e1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
    scan_ms = [a.elapsed_time(b) for a, b in scan_ev]
    ms_step = ms / K
    value = weak_scaling_value(world, layer.units, K, ms)

    # end to end through the public API from pinned host buffers: every step
    # uploads its inputs, quantizes and scans, and reads y back; steps are
    # pipelined over an upload, a compute and a download stream with two
    # device copies of the inputs and of y (step i + 1 uploads while step i
    # computes and step i - 1 downloads)
    Ke = max(1, min(K, args.e2e_steps))
    h2d = sum(layer.host[k].numel() * layer.host[k].element_size() for k in layer.host)
    d2h = layer.y.numel() * 2
    e2e_ms = e2e_pipelined(torch, layer, Ke)
    ems = max_over_ranks(e2e_ms, dist if world > 1 else None, dev)
    e2e_value = weak_scaling_value(world, layer.units, Ke, ems)
    floor_ms = e2e_copy_floor(torch, layer, Ke) / Ke

    out = None
    ex2 = None
    if rank == 0:
        try:  # the SFU roof, measured on this GPU after the timed region
            ex2 = measure_ex2(torch, dev)
        except Exception as e:
            ex2 = {"error": "%s: %s" % (type(e).__name__, e)}
    if rank == 0:
        scan_avg_s = statistics.mean(scan_ms) / 1e3
        clocks = clk.summary()
        mhz_max = float(clocks.get("sm_max_mhz") or pk["sm_max_mhz"])
        updates = layer.b * layer.L * layer.d * layer.N
        peak_upd, peak_basis = sfu_peak(ex2, mhz_max)
        achieved_upd = updates / scan_avg_s / 1e9
        scan_gbs = layer.scan_bytes() / scan_avg_s / 1e9
        out = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": max(args.warmup, 3), "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded numpy draws shaped like the workload; no dataset)",
            "config": dict(config_dict(layer.dm), parallelism="dp%d (independent replicas)" % world),
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": Ke,
                    "ms_per_step": round(ems / Ke, 5),
                    "copy_floor_ms_per_step": round(floor_ms, 5),
                    "frac_of_copy_floor": round(floor_ms / (ems / Ke), 4),
                    "copy_floor": "the same host<->device copies without kernels, "
                                  "uploads and the download on two streams"},
            "gpu_launches": layer.launches_per_step * K,
            "x_path": ("binary16 x quantized inside the scan (byte-identical to a separate "
                       "quantize launch followed by the int8 scan)" if layer.fused else
                       "x, B and C quantized by one batched launch; the scan reads int8 codes"),
            "roofline": {"bound": "alu", "kernel": "m1_scan_kernel (selective scan)",
                         "achieved": round(achieved_upd, 2), "peak": round(peak_upd, 1),
                         "unit": "Gupdates/s", "frac": round(achieved_upd / peak_upd, 4),
                         "traffic": measured_traffic("m1_scan_kernel" if not layer.fused
                                                     else "m1_scan_kernel_f16x"),
                         "peak_basis": peak_basis, "sfu_probe": ex2,
                         "hbm_achieved_gbs": round(scan_gbs, 1), "hbm_peak_gbs": pk["hbm_gbs"],
                         "hbm_frac": round(scan_gbs / pk["hbm_gbs"], 4),
                         "algorithmic_bytes_per_launch": layer.scan_bytes(),
                         "scan_ms_per_launch": round(scan_avg_s * 1e3, 5),
                         "peaks_source": pk["source"]},
            "step_hbm_gbs": round(layer.step_bytes() / (ms_step / 1e3) / 1e9, 1),
            "quantize_leg": {"kernel": "quant_batch_kernel (x, B, C in one launch)",
                             "algorithmic_bytes_per_launch": layer.step_bytes() - layer.scan_bytes(),
                             "ms_per_launch": round(ms_step - scan_avg_s * 1e3, 5),
                             "hbm_frac": round((layer.step_bytes() - layer.scan_bytes()) /
                                               ((ms_step - scan_avg_s * 1e3) / 1e3) / 1e9 /
                                               pk["hbm_gbs"], 4),
                             "traffic": measured_traffic("quant_batch_kernel"),
                             "note": "time = step minus the scan's CUDA-event time"},
            "clocks": clocks,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            try:
                out["cpu_baseline"] = cpu_baseline(layer)
                # the y / h_final of the last timed step against the oracle on
                # the baseline's sample (the same inputs every step)
                bb, yo, ho = layer.oracle_out
                out["parity"] = parity(
                    layer.y[:bb].float().cpu().numpy().reshape(bb * layer.d, layer.L), yo,
                    layer.hf[:bb].cpu().numpy().reshape(bb * layer.d, layer.N), ho,
                    "%d (batch, channel) rows of the last timed step" % (bb * layer.d))
            except Exception as e:  # report, keep the measured line
                out["cpu_baseline"] = {"error": "%s: %s" % (type(e).__name__, e)}
        if world == 1 and not args.no_forms:
            only = args.forms.split(",") if args.forms else None
            out["forms"] = {}
            if not only or "m130m_other_x_path" in only:
                out["forms"]["m130m_other_x_path"] = form_other_x_path(torch, layer)
            if not only or "m130m_int8_y" in only:
                out["forms"]["m130m_int8_y"] = form_int8_y(torch, layer)
            out["forms"].update(run_forms(dev, pk, out["clocks"].get("sm_max_mhz") or
                                          pk["sm_max_mhz"], only=only, layer=layer, ex2=ex2))
        print(json.dumps(out), flush=True)


# ---- the other forms, device-timed (information beside the headline) -------

def _timed(torch, fn, reps):
    fn()
    torch.cuda.synchronize()
    a, b = cuda_events(torch)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps / 1e3


def setup_decode(torch, dev, steps=None):
    """decode8b inputs for `steps` chained single-token updates (b 64, H 128,
    P 64, N 128, G 8), int8 inputs quantized ahead of the chain; returns the
    dims and step(t)."""
    from quantized_state_space_b200 import api, calibrate, synth
    dm, raw = synth.workload_inputs("decode8b", **({"steps": steps} if steps else {}))
    b, H, P, N, G, gs, S, k = (dm["batch"], dm["nheads"], dm["headdim"], dm["dstate"],
                               dm["ngroups"], dm["state_group_size"], dm["steps"], dm["x_clusters"])
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    grp, xs = calibrate.ssd_x_clusters(raw["x"], k)
    bs = calibrate.state_group_absmax_scales(raw["B"], G, N, gs, "gn")
    cs = calibrate.state_group_absmax_scales(raw["C"], G, N, gs, "gn")
    smap = T(calibrate.state_group_map(G, N, gs))
    xq, _ = api.quantize_groups(T(raw["x"]), S * b, H * P, 1, T(grp), k, scales=T(xs))
    Bq, _ = api.quantize_groups(T(raw["B"]), S * b, G * N, 1, smap, G * N // gs, scales=T(bs))
    Cq, _ = api.quantize_groups(T(raw["C"]), S * b, G * N, 1, smap, G * N // gs, scales=T(cs))
    dt, A, D, grp_t, xs_t, bs_t, cs_t = (T(raw["dt"]), T(raw["A"]), T(raw["D"]), T(grp), T(xs),
                                        T(bs), T(cs))
    state = T(raw["state"])
    y = torch.empty((b, H, P), dtype=torch.float16, device=dev)

    def step(t):
        api.state_update(state, xq[t], dt[t], A, Bq[t], Cq[t], bs_t, cs_t, gs, x_group=grp_t,
                         x_scale=xs_t, D=D, y=y)

    return dict(b=b, H=H, P=P, N=N, G=G, S=S, gs=gs, k=k, step=step, raw=raw, state=state, y=y)


def e2e_pipelined(torch, layer, steps):
    """Milliseconds for `steps` end-to-end steps of the layer (upload of x,
    dt, z, B, C from pinned host memory, quantize + scan, download of y into
    pinned host memory), pipelined over three streams."""
    from quantized_state_space_b200 import api
    names = ("x", "dt", "z", "B", "C")
    sets = [{k: getattr(layer, k) for k in names},
            {k: torch.empty_like(getattr(layer, k)) for k in names}]
    ys = [layer.y, torch.empty_like(layer.y)]
    y_host = [torch.empty(layer.y.shape, dtype=torch.float16).pin_memory() for _ in range(2)]
    up, comp, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event(enable_timing=False)
    in_ready = [ev(), ev()]
    in_free = [ev(), ev()]
    y_ready = [ev(), ev()]
    y_free = [ev(), ev()]
    b, L, d, G, N, gs = layer.b, layer.L, layer.d, layer.G, layer.N, layer.gs

    def run(n):
        for i in range(n):
            j = i % 2
            S = sets[j]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(in_free[j])
                for k in names:
                    S[k].copy_(layer.host[k], non_blocking=True)
                in_ready[j].record(up)
            with torch.cuda.stream(comp):
                comp.wait_event(in_ready[j])
                if i >= 2:
                    comp.wait_event(y_free[j])
                api.quantize_groups_batch(
                    [(S["x"], b, d, L, layer.grp, layer.k, layer.xs, layer.xq),
                     (S["B"], b, G * N, L, layer.smap, G * N // gs, layer.bs, layer.Bq),
                     (S["C"], b, G * N, L, layer.smap, G * N // gs, layer.cs, layer.Cq)])
                api.selective_scan(layer.xq, S["dt"], layer.A, layer.Bq, layer.Cq, layer.bs,
                                   layer.cs, gs, x_group=layer.grp, x_scale=layer.xs, D=layer.D,
                                   z=S["z"], y=ys[j], h_final=layer.hf)
                in_free[j].record(comp)  # the scan read dt and z of this set
                y_ready[j].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(y_ready[j])
                y_host[j].copy_(ys[j], non_blocking=True)
                y_free[j].record(down)

    run(2)  # warm-up
    torch.cuda.synchronize()
    a0, a1 = cuda_events(torch)
    a0.record(up)
    run(steps)
    for s_ in (up, comp):
        down.wait_stream(s_)
    a1.record(down)
    torch.cuda.synchronize()
    # every step has the same inputs: each downloaded y equals a plain step's
    layer.quantize()
    layer.scan()
    torch.cuda.synchronize()
    ref = layer.y.cpu()
    for yh in y_host[:min(steps, 2)]:
        if not torch.equal(yh.view(torch.int16), ref.view(torch.int16)):
            raise RuntimeError("pipelined end-to-end step: downloaded y differs")
    return a0.elapsed_time(a1)


def e2e_copy_floor(torch, layer, steps):
    """Milliseconds for `steps` steps of the end-to-end copies alone (every
    input up, y down, on two streams as in the pipelined run, no kernels):
    the host-link floor of an end-to-end step."""
    names = ("x", "dt", "z", "B", "C")
    dst = {k: torch.empty_like(getattr(layer, k)) for k in names}
    y_host = torch.empty(layer.y.shape, dtype=torch.float16).pin_memory()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def run(n):
        for _ in range(n):
            with torch.cuda.stream(up):
                for k in names:
                    dst[k].copy_(layer.host[k], non_blocking=True)
            with torch.cuda.stream(down):
                y_host.copy_(layer.y, non_blocking=True)

    run(1)
    torch.cuda.synchronize()
    a0, a1 = cuda_events(torch)
    a0.record(up)
    down.wait_stream(up)
    run(steps)
    down.wait_stream(up)
    a1.record(down)
    torch.cuda.synchronize()
    return a0.elapsed_time(a1)


def form_other_x_path(torch, layer):
    """The headline step with the other x path on the same inputs: binary16 x
    encoded inside the scan vs x quantized with B and C (byte-identical
    results; the GPU parity tests check that)."""
    layer.fused = not layer.fused
    try:
        def step():
            layer.quantize()
            layer.scan()
        t = _timed(torch, step, 50)
        t_scan = _timed(torch, layer.scan, 20)
        return {"workload": "m130m step, " + ("binary16 x encoded inside the scan" if layer.fused
                                               else "x quantized in the batched launch"),
                "value": round(layer.units / t / 1e9, 3), "unit": UNIT,
                "ms_per_step": round(t * 1e3, 4), "scan_ms": round(t_scan * 1e3, 4),
                "launches_per_step": layer.launches_per_step}
    finally:
        layer.fused = not layer.fused


def form_int8_y(torch, layer):
    """The headline step with the persistent-INT8 epilogue: the scan writes int8
    y (static per-cluster output scales calibrated on this layer's binary16 y)
    instead of binary16 y; beside it the binary16 step followed by a separate
    quantize of y, which produces the same bytes."""
    from quantized_state_space_b200 import api, calibrate
    b, d, L, k = layer.b, layer.d, layer.L, layer.k
    layer.quantize()
    layer.scan()
    torch.cuda.synchronize()
    ygrp, ysc = calibrate.m1_x_clusters(layer.y.cpu().numpy(), k)
    yg = torch.from_numpy(ygrp).to(layer.y.device)
    ys = torch.from_numpy(ysc).to(layer.y.device)
    yq = torch.empty(layer.y.shape, dtype=torch.int8, device=layer.y.device)

    def step_q():
        layer.quantize()
        api.selective_scan(layer.x if layer.fused else layer.xq, layer.dt, layer.A, layer.Bq,
                           layer.Cq, layer.bs, layer.cs, layer.gs, x_group=layer.grp,
                           x_scale=layer.xs, D=layer.D, z=layer.z, h_final=layer.hf, y_group=yg,
                           y_scale=ys, y_q=yq, want_y=False)

    def step_sep():
        layer.quantize()
        layer.scan()
        api.quantize_groups(layer.y, b, d, L, yg, k, scales=ys, out=yq)

    t_q = _timed(torch, step_q, 50)
    t_s = _timed(torch, step_sep, 50)
    return {"workload": "m130m step with int8 y (persistent-INT8 epilogue, no binary16 y)",
            "value": round(layer.units / t_q / 1e9, 3), "unit": UNIT,
            "ms_per_step": round(t_q * 1e3, 4),
            "separate_quantize_of_y": {"value": round(layer.units / t_s / 1e9, 3),
                                       "ms_per_step": round(t_s * 1e3, 4)}}


def _units_value(units_tokens_ch, seconds):
    return round(units_tokens_ch / seconds / 1e9, 6)


def oracle_timing(run, single, allc, threads, what):
    """The oracle, as it stands, timed twice on bounded samples of a form's
    workload: `single` (n_units, tokens*channels) on one thread, `allc` on
    all host cores.  run(n_units, threads) computes the sample and returns
    its outputs (those of the all-core run are returned for the parity check)."""
    t = time.perf_counter()
    run(single[0], 1)
    t1 = time.perf_counter() - t
    t = time.perf_counter()
    out = run(allc[0], threads)
    ta = time.perf_counter() - t
    return {"kind": "oracle", "unit": UNIT,
            "single_thread": {"value": _units_value(single[1], t1), "seconds": round(t1, 3),
                              "cores": 1, "sample": "%d %s" % (single[0], what)},
            "all_cores": {"value": _units_value(allc[1], ta), "seconds": round(ta, 3),
                          "cores": threads, "sample": "%d %s" % (allc[0], what)},
            "value": _units_value(allc[1], ta), "cores": threads,
            "sample": "%d %s on %d threads" % (allc[0], what, threads)}, out


def _threaded_units(fn, units, threads):
    """fn(units_slice) over `threads` Python threads (the oracle's C calls run
    without the interpreter lock); returns the per-slice results in order."""
    import concurrent.futures as cf
    parts = [p for p in np.array_split(np.asarray(units), max(1, threads)) if p.size]
    with cf.ThreadPoolExecutor(max_workers=len(parts)) as ex:
        return list(ex.map(fn, parts))


def form_decode(torch, dev, pk):
    """decode8b: 1000 chained single-token state updates."""
    c = setup_decode(torch, dev)
    b, H, P, N, G, S = c["b"], c["H"], c["P"], c["N"], c["G"], c["S"]

    def chain():
        for t in range(S):
            c["step"](t)

    # parity: the first step from the initial state, then restore it
    from oracle import oracle as O
    raw = c["raw"]
    st0 = c["state"].clone()
    c["step"](0)
    torch.cuda.synchronize()
    y_gpu = c["y"].float().cpu().numpy().reshape(b * H, P)
    st1 = c["state"].cpu().numpy().reshape(b * H, P, N)
    c["state"].copy_(st0)
    del st0
    gs, k = c["gs"], c["k"]
    head_abs = np.abs(raw["x"].astype(np.float32)).max(axis=(0, 1, 3))
    ohc, oxs = O.cluster_by_absmax(head_abs.astype(np.float64), k)
    ogrp = np.repeat(ohc, P).astype(np.int32)
    omap = np.arange(G * N) // gs
    Bf = raw["B"].reshape(S * b, G * N)
    Cf = raw["C"].reshape(S * b, G * N)
    _, obs, _ = O.quantize_groups(Bf, S * b, G * N, 1, omap, G * N // gs, O.SCALE_ABSMAX)
    _, ocs, _ = O.quantize_groups(Cf, S * b, G * N, 1, omap, G * N // gs, O.SCALE_ABSMAX)
    nst = 8  # steps in the timed oracle sample
    ox, _, _ = O.quantize_groups(raw["x"][:nst].reshape(nst * b, H * P), nst * b, H * P, 1, ogrp,
                                 k, O.SCALE_STATIC, oxs)
    oB, _, _ = O.quantize_groups(Bf[:nst * b], nst * b, G * N, 1, omap, G * N // gs,
                                 O.SCALE_STATIC, obs)
    oC, _, _ = O.quantize_groups(Cf[:nst * b], nst * b, G * N, 1, omap, G * N // gs,
                                 O.SCALE_STATIC, ocs)
    ox, oB, oC = ox.reshape(nst, b, H, P), oB.reshape(nst, b, G, N), oC.reshape(nst, b, G, N)

    def run(n_steps, threads):
        units = np.arange(b * H)
        state = raw["state"].reshape(b * H, P, N).astype(np.float64)

        def part(us):
            stp = np.ascontiguousarray(state[us])
            ys = []
            for t in range(n_steps):
                ys.append(O.decode_step(stp, ox[t], raw["dt"][t], raw["A"], oB[t], oC[t], obs, ocs,
                                        gs, x_group=ogrp, x_scale=oxs, D=raw["D"], units=us))
            return ys[0], stp if n_steps == 1 else None

        return _threaded_units(part, units, threads)

    threads = O.default_threads()
    base, _ = oracle_timing(run, (1, b * H * P), (nst, nst * b * H * P), threads,
                            "chained steps over all %d (batch, head) states" % (b * H))
    base["sample"] += " (of the 1000-step chain; the full chain would take ~%.0f s)" % (
        1000 * base["all_cores"]["seconds"] / nst)
    one = run(1, threads)
    par = parity(y_gpu, np.concatenate([r[0] for r in one]), st1,
                 np.concatenate([r[1] for r in one]),
                 "step 1 of the chain, every (batch, head): y and the updated state")
    del one
    sec = _timed(torch, chain, 2) / S
    byts = 2 * b * H * P * N * 4 + b * H * P * (1 + 2) + b * H * 2 + 2 * b * G * N
    return {"workload": "decode8b: b 64, H 128, P 64, N 128, G 8, 1000 chained steps",
            "cpu_baseline": base, "parity": par,
            "value": round(b * H * P / sec / 1e9, 3), "unit": "Gtokens·ch/s",
            "us_per_step": round(sec * 1e6, 2),
            "roofline": {"bound": "hbm", "achieved": round(byts / sec / 1e9, 1),
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(byts / sec / 1e9 / pk["hbm_gbs"], 4),
                         "algorithmic_bytes_per_launch": byts,
                         "traffic": measured_traffic("decode_kernel")},
            "l2": "state 268 MB exceeds L2"}


def setup_softedge(torch, dev):
    """softedge inputs (b 16, L 8192, d 1536, N 16, z gate); returns the dims
    and enc (binary16 x -> soft-edge codes), quant_bc, scan."""
    from quantized_state_space_b200 import api, calibrate, synth
    dm, raw = synth.workload_inputs("softedge")
    b, L, d, N, G, gs = (dm["batch"], dm["seqlen"], dm["dim"], dm["dstate"], dm["ngroups"],
                         dm["state_group_size"])
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    s, lo, hi = calibrate.softedge_params(raw["x"])
    bs = calibrate.state_group_absmax_scales(raw["B"], G, N, gs, "gnl")
    cs = calibrate.state_group_absmax_scales(raw["C"], G, N, gs, "gnl")
    smap = T(calibrate.state_group_map(G, N, gs))
    x, dt, z, B, C = (T(raw[k]) for k in ("x", "dt", "z", "B", "C"))
    A, D, bs_t, cs_t = T(raw["A"]), T(raw["D"]), T(bs), T(cs)
    codes = torch.empty(x.shape, dtype=torch.uint8, device=dev)
    Bq = torch.empty(B.shape, dtype=torch.int8, device=dev)
    Cq = torch.empty(C.shape, dtype=torch.int8, device=dev)
    y = torch.empty(x.shape, dtype=torch.float16, device=dev)
    hf = torch.empty((b, d, N), dtype=torch.float32, device=dev)

    def enc():
        api.softedge_encode(x, s, lo, hi, 2, out=codes)

    def quant_bc():  # B and C in one batched launch
        api.quantize_groups_batch([(B, b, G * N, L, smap, G * N // gs, bs_t, Bq),
                                   (C, b, G * N, L, smap, G * N // gs, cs_t, Cq)])

    def scan():
        api.selective_scan(codes, dt, A, Bq, Cq, bs_t, cs_t, gs, se_scale=s, D=D, z=z, y=y,
                           h_final=hf)

    def scan_fused():  # binary16 x encoded inside the scan
        api.selective_scan(x, dt, A, Bq, Cq, bs_t, cs_t, gs, se_scale=s, se_lo=lo, se_hi=hi, D=D,
                           z=z, y=y, h_final=hf)

    return dict(b=b, L=L, d=d, N=N, G=G, gs=gs, enc=enc, quant_bc=quant_bc, scan=scan,
                scan_fused=scan_fused, raw=raw, y=y, hf=hf)


def softedge_oracle_check(torch, c):
    """The oracle on sampled channel rows of the softedge workload: its own
    thresholds (percentiles of |x| over the whole tensor) and encoder, its own
    B / C quantizer (untimed), then the double-precision scan, timed on one
    thread (8 rows) and on all cores (one batch row, 1536 rows); the all-core
    sample against the GPU's y and h_final of the last scan."""
    from oracle import oracle as O
    raw = c["raw"]
    b, L, d, N, G, gs = c["b"], c["L"], c["d"], c["N"], c["G"], c["gs"]
    olo = np.float32(O.percentile_abs(raw["x"], 5.0))
    ohi = np.float32(O.percentile_abs(raw["x"], 99.9))
    osc = np.float32(np.float64(ohi) / 63.0)
    ox, _ = O.softedge_encode(raw["x"][:1], osc, olo, ohi, 2)
    gmap = np.arange(G * N) // gs
    _, obs, _ = O.quantize_groups(raw["B"], b, G * N, L, gmap, G * N // gs, O.SCALE_ABSMAX)
    _, ocs, _ = O.quantize_groups(raw["C"], b, G * N, L, gmap, G * N // gs, O.SCALE_ABSMAX)
    oB, _, _ = O.quantize_groups(raw["B"][:1], 1, G * N, L, gmap, G * N // gs, O.SCALE_STATIC, obs)
    oC, _, _ = O.quantize_groups(raw["C"][:1], 1, G * N, L, gmap, G * N // gs, O.SCALE_STATIC, ocs)
    threads = O.default_threads()

    def run(n, th):
        return O.m1_scan(ox.reshape(1, d, L), raw["dt"][:1], raw["A"], oB.reshape(1, G, N, L),
                         oC.reshape(1, G, N, L), obs, ocs, gs, se_scale=float(osc), D=raw["D"],
                         z=raw["z"][:1], units=np.arange(n), threads=th)

    base, (yo, ho) = oracle_timing(run, (8, 8 * L), (d, d * L), threads,
                                   "channel rows of L %d" % L)
    yg = c["y"][0].float().cpu().numpy()
    hg = c["hf"][0].cpu().numpy()
    return base, parity(yg, yo, hg, ho, "batch row 0: %d channel rows" % d)


def form_softedge(torch, dev, pk, mhz, ex2=None):
    """softedge: encode binary16 x to soft-edge codes, quantize B/C, scan."""
    c = setup_softedge(torch, dev)
    b, L, d, N = c["b"], c["L"], c["d"], c["N"]
    enc, quant_bc, scan = c["enc"], c["quant_bc"], c["scan"]
    t_enc = _timed(torch, enc, 5)
    t_bc = _timed(torch, quant_bc, 5)
    t_fused = _timed(torch, c["scan_fused"], 3)
    t_scan = _timed(torch, scan, 3)  # last: its y is the one checked
    base, par = softedge_oracle_check(torch, c)
    t = t_enc + t_bc + t_scan
    t_f = t_bc + t_fused
    n = b * L * d
    enc_bytes = n * 3
    upd = n * N
    peak_upd, _ = sfu_peak(ex2, mhz)
    return {"workload": "softedge: b 16, L 8192, d 1536, N 16; encode + scan",
            "value": round(n / t / 1e9, 3), "unit": "Gtokens·ch/s",
            "ms_per_step": round(t * 1e3, 4), "cpu_baseline": base, "parity": par,
            "x_path": "encode launch, then the scan reads the codes",
            "fused_path": {"x_path": "binary16 x soft-edge encoded inside the scan "
                                     "(byte-identical result)",
                           "value": round(n / t_f / 1e9, 3), "ms_per_step": round(t_f * 1e3, 4),
                           "scan_ms": round(t_fused * 1e3, 4)},
            "encode": {"ms": round(t_enc * 1e3, 4), "bound": "hbm",
                       "achieved": round(enc_bytes / t_enc / 1e9, 1), "peak": pk["hbm_gbs"],
                       "unit": "GB/s", "frac": round(enc_bytes / t_enc / 1e9 / pk["hbm_gbs"], 4),
                       "kernel": "se_encode_lut_kernel", "algorithmic_bytes_per_launch": enc_bytes,
                       "traffic": measured_traffic("se_encode_lut_kernel")},
            "scan": {"ms": round(t_scan * 1e3, 4), "bound": "alu",
                     "achieved": round(upd / t_scan / 1e9, 1), "peak": round(peak_upd, 1),
                     "unit": "Gupdates/s", "frac": round(upd / t_scan / 1e9 / peak_upd, 4)}}


def setup_ssd(torch, dev):
    """ssd27b inputs (b 4, L 4096, H 80, P 64, N 128, G 1, chunk 256); returns
    the dims and quant (x / B / C), ssd."""
    from quantized_state_space_b200 import api, calibrate, synth
    dm, raw = synth.workload_inputs("ssd27b")
    b, L, H, P, N, G, gs, k = (dm["batch"], dm["seqlen"], dm["nheads"], dm["headdim"],
                               dm["dstate"], dm["ngroups"], dm["state_group_size"],
                               dm["x_clusters"])
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    grp, xs = calibrate.ssd_x_clusters(raw["x"], k)
    smap = T(calibrate.state_group_map(G, N, gs))
    bs = calibrate.state_group_absmax_scales(raw["B"], G, N, gs, "lgn")
    cs = calibrate.state_group_absmax_scales(raw["C"], G, N, gs, "lgn")
    x, dt, B, C = T(raw["x"]), T(raw["dt"]), T(raw["B"]), T(raw["C"])
    A, D, grp_t, xs_t, bs_t, cs_t = T(raw["A"]), T(raw["D"]), T(grp), T(xs), T(bs), T(cs)
    xq = torch.empty(x.shape, dtype=torch.int8, device=dev)
    Bq = torch.empty(B.shape, dtype=torch.int8, device=dev)
    Cq = torch.empty(C.shape, dtype=torch.int8, device=dev)
    y = torch.empty(x.shape, dtype=torch.float16, device=dev)
    hf = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)

    def quant():  # x, then B and C in one batched launch (with x: slower, 135 us)
        api.quantize_groups_batch([(x, b * L, H * P, 1, grp_t, k, xs_t, xq)])
        api.quantize_groups_batch([(B, b * L, G * N, 1, smap, G * N // gs, bs_t, Bq),
                                   (C, b * L, G * N, 1, smap, G * N // gs, cs_t, Cq)])

    def ssd():
        api.ssd_chunk_scan(xq, dt, A, Bq, Cq, bs_t, cs_t, gs, chunk=dm["chunk"], x_group=grp_t,
                           x_scale=xs_t, D=D, y=y, h_final=hf)

    return dict(b=b, L=L, H=H, P=P, N=N, G=G, gs=gs, k=k, quant=quant, ssd=ssd, raw=raw, y=y,
                hf=hf)


def ssd_oracle_check(torch, c):
    """The oracle on sampled (batch, head) sequences of ssd27b: its own
    calibration and quantizers from the raw arrays (untimed), then the
    sequential double-precision scan, timed on one thread (one sequence) and
    on all cores (one sequence per core); the all-core sample against the GPU's
    y and h_final of the last timed call."""
    from oracle import oracle as O
    raw = c["raw"]
    b, L, H, P, N, G, gs, k = c["b"], c["L"], c["H"], c["P"], c["N"], c["G"], c["gs"], c["k"]
    y_gpu, hf_gpu = c["y"], c["hf"]
    head_abs = np.abs(raw["x"].astype(np.float32)).max(axis=(0, 1, 3))
    ohc, oxs = O.cluster_by_absmax(head_abs.astype(np.float64), k)
    ogrp = np.repeat(ohc, P).astype(np.int32)
    omap = np.arange(G * N) // gs
    _, obs, _ = O.quantize_groups(raw["B"], b * L, G * N, 1, omap, G * N // gs, O.SCALE_ABSMAX)
    _, ocs, _ = O.quantize_groups(raw["C"], b * L, G * N, 1, omap, G * N // gs, O.SCALE_ABSMAX)
    ox, _, _ = O.quantize_groups(raw["x"], b * L, H * P, 1, ogrp, k, O.SCALE_STATIC, oxs)
    oB, _, _ = O.quantize_groups(raw["B"], b * L, G * N, 1, omap, G * N // gs, O.SCALE_STATIC, obs)
    oC, _, _ = O.quantize_groups(raw["C"], b * L, G * N, 1, omap, G * N // gs, O.SCALE_STATIC, ocs)
    ox = ox.reshape(b, L, H, P)
    oB, oC = oB.reshape(b, L, G, N), oC.reshape(b, L, G, N)
    rng = np.random.default_rng(3)
    threads = O.default_threads()
    units = np.sort(rng.choice(b * H, size=min(b * H, threads), replace=False))

    def run(n, th):
        return O.ssd_scan(ox, raw["dt"], raw["A"], oB, oC, obs, ocs, gs, x_group=ogrp,
                          x_scale=oxs, D=raw["D"], units=units[:n], threads=th)

    base, (yo, ho) = oracle_timing(run, (1, L * P), (len(units), len(units) * L * P), threads,
                                   "(batch, head) sequences of L %d x P %d" % (L, P))
    yg = np.stack([y_gpu[u // H, :, u % H, :].float().cpu().numpy() for u in units])
    hg = hf_gpu.reshape(b * H, P, N)[torch.as_tensor(units, device=hf_gpu.device)].cpu().numpy()
    return base, parity(yg, yo, hg, ho, "%d sampled (batch, head) sequences" % len(units))


def form_ssd(torch, dev, pk):
    """ssd27b: quantize x / B / C and run the SSD chunked scan on tcgen05."""
    c = setup_ssd(torch, dev)
    b, L, H, P, N, G = c["b"], c["L"], c["H"], c["P"], c["N"], c["G"]
    quant, ssd = c["quant"], c["ssd"]
    t_q = _timed(torch, quant, 5)
    t_s = _timed(torch, ssd, 5)
    base, par = ssd_oracle_check(torch, c)
    q = 256  # the chunk length the algorithmic count refers to
    nch = L // q
    useful = (2 * q * (q + 1) // 2 * N * b * nch * G          # C B^T, causal half
              + 2 * q * (q + 1) // 2 * P * b * nch * H        # diagonal blocks
              + 2 * 2 * q * N * P * b * nch * H)              # carried state in and out
    executed = 2 * b * H * (L // 128) * (128 ** 3 + 128 * 128 * 64 * 4)  # CB, Y_diag, Y_off, 2 x state
    byts = b * L * H * P * (1 + 2) + b * L * H * 2 + 2 * b * L * G * N + b * H * P * N * 4
    tf = useful / t_s / 1e12
    return {"workload": "ssd27b: b 4, L 4096, H 80, P 64, N 128, G 1, chunk 256; quantize + SSD",
            "value": round(b * L * H * P / (t_q + t_s) / 1e9, 3), "unit": "Gtokens·ch/s",
            "ms_per_step": round((t_q + t_s) * 1e3, 4), "ssd_ms": round(t_s * 1e3, 4),
            "quantize_ms": round(t_q * 1e3, 4), "cpu_baseline": base, "parity": par,
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tf / pk["bf16_tflops"], 4),
                         "algorithmic_flops_per_launch": useful,
                         "executed_mma_flops_per_launch": executed,
                         "hbm_achieved_gbs": round(byts / t_s / 1e9, 1),
                         "hbm_frac": round(byts / t_s / 1e9 / pk["hbm_gbs"], 4),
                         "traffic": measured_traffic("ssd_kernel")}}


def form_calibrate(torch, dev, pk, layer):
    """Device calibration: per-channel maxima of the m130m x and their
    sort-and-cluster (the offline step, on the GPU), and the soft-edge
    thresholds (5th / 99.9th percentiles of |x|) of the softedge x."""
    from quantized_state_space_b200 import api, synth
    b, d, L, k = layer.b, layer.d, layer.L, layer.k
    ident = torch.arange(d, dtype=torch.int32, device=dev)
    amax = torch.empty(d, dtype=torch.float32, device=dev)
    t_max = _timed(torch, lambda: api.group_absmax(layer.x, b, d, L, ident, d, out=amax), 10)
    t_cl = _timed(torch, lambda: api.cluster_by_absmax(amax, k), 10)
    dm, raw = synth.workload_inputs("softedge")
    x = torch.from_numpy(raw["x"]).to(dev)
    del raw
    nb = api.N.ssmq_percentile_workspace_size()
    ws = torch.empty(nb + 256, dtype=torch.uint8, device=dev)
    thr = torch.zeros(3, dtype=torch.float32, device=dev)
    t_pct = _timed(torch, lambda: api.softedge_calibrate(x, thr, workspace=ws), 5)
    bx = layer.x.numel() * 2
    bs = x.numel() * 2
    return {"workload": "m130m x channel maxima + sort-and-cluster (k %d); softedge x "
                        "thresholds (%d M binary16 elements)" % (k, x.numel() // 10**6),
            "absmax_ms": round(t_max * 1e3, 4),
            "absmax_hbm": {"achieved": round(bx / t_max / 1e9, 1), "peak": pk["hbm_gbs"],
                           "unit": "GB/s", "frac": round(bx / t_max / 1e9 / pk["hbm_gbs"], 4)},
            "cluster_ms": round(t_cl * 1e3, 4),
            "thresholds_ms": round(t_pct * 1e3, 4),
            "thresholds_hbm": {"achieved": round(bs / t_pct / 1e9, 1), "peak": pk["hbm_gbs"],
                               "unit": "GB/s", "frac": round(bs / t_pct / 1e9 / pk["hbm_gbs"], 4)}}


def form_tiny(torch, dev, reps=50):
    """tiny (b 1, L 256, d 64, N 16, per-tensor absmax scales): latency of
    one call, CUDA events around each call, median of `reps`.  The step is
    the device-side per-tensor absmax quantize of x, B and C (scales computed
    on the device) followed by the scan; the scan is also timed alone.  The
    whole workload is checked against the oracle and timed on it."""
    from oracle import oracle as O
    from quantized_state_space_b200 import api, synth
    dm, raw = synth.workload_inputs("tiny")
    b, L, d, N, G, gs = (dm["batch"], dm["seqlen"], dm["dim"], dm["dstate"], dm["ngroups"],
                         dm["state_group_size"])
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    x, dt, B, C, A, D = (T(raw[k]) for k in ("x", "dt", "B", "C", "A", "D"))
    g0 = torch.zeros(d, dtype=torch.int32, device=dev)
    s0 = torch.zeros(G * N, dtype=torch.int32, device=dev)
    xq = torch.empty(x.shape, dtype=torch.int8, device=dev)
    Bq = torch.empty(B.shape, dtype=torch.int8, device=dev)
    Cq = torch.empty(C.shape, dtype=torch.int8, device=dev)
    y = torch.empty(x.shape, dtype=torch.float16, device=dev)
    hf = torch.empty((b, d, N), dtype=torch.float32, device=dev)
    sc = {}

    def quant():
        _, sc["x"] = api.quantize_groups(x, b, d, L, g0, 1, absmax=True, out=xq)
        _, sc["B"] = api.quantize_groups(B, b, G * N, L, s0, 1, absmax=True, out=Bq)
        _, sc["C"] = api.quantize_groups(C, b, G * N, L, s0, 1, absmax=True, out=Cq)

    def scan():
        api.selective_scan(xq, dt, A, Bq, Cq, sc["B"], sc["C"], gs, x_group=g0, x_scale=sc["x"],
                           D=D, y=y, h_final=hf)

    def step():
        quant()
        scan()

    def lat(fn):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, e = cuda_events(torch)
            a.record()
            fn()
            e.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(e) * 1e3)
        return round(statistics.median(ts), 2)

    t_step, t_scan = lat(step), lat(scan)
    # the same step captured once in a CUDA graph and replayed: the device-side
    # latency without the host's per-launch cost
    try:
        g = torch.cuda.CUDAGraph()
        s_ = torch.cuda.Stream()
        s_.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s_):
            step()
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s_):
                step()
        torch.cuda.current_stream().wait_stream(s_)
        t_graph = lat(g.replay)
    except Exception as e:  # report, keep the eager numbers
        t_graph = "%s: %s" % (type(e).__name__, e)
    ox, oxs, _ = O.quantize_groups(raw["x"], b, d, L, np.zeros(d, np.int32), 1, O.SCALE_ABSMAX)
    gm = np.zeros(G * N, np.int32)
    oB, obs, _ = O.quantize_groups(raw["B"], b, G * N, L, gm, 1, O.SCALE_ABSMAX)
    oC, ocs, _ = O.quantize_groups(raw["C"], b, G * N, L, gm, 1, O.SCALE_ABSMAX)

    def run(n, th):
        return O.m1_scan(ox, raw["dt"], raw["A"], oB, oC, obs, ocs, gs,
                         x_group=np.zeros(d, np.int32), x_scale=oxs, D=raw["D"],
                         units=np.arange(n), threads=th)

    base, (yo, ho) = oracle_timing(run, (b * d, b * d * L), (b * d, b * d * L),
                                   O.default_threads(), "channel rows of L %d (the whole "
                                   "workload)" % L)
    par = parity(y.float().cpu().numpy().reshape(b * d, L), yo,
                 hf.cpu().numpy().reshape(b * d, N), ho, "the whole workload")
    return {"workload": "tiny: b 1, L 256, d 64, N 16, per-tensor absmax scales; latency",
            "step_us": t_step, "scan_us": t_scan, "step_graph_replay_us": t_graph,
            "step": "device absmax quantize of x, B, C (3 calls, 12 launches incl. memsets) "
                    "+ scan", "statistic": "median of %d calls, CUDA events per call" % reps,
            "value": round(b * L * d / (t_step / 1e6) / 1e9, 4), "unit": UNIT,
            "roofline": "launch-latency bound (98.6 KB, 262 k state updates): not meaningful",
            "cpu_baseline": base, "parity": par}


def form_conv(torch, dev, pk, layer):
    """Producer-side fusion: causal depthwise conv (W 4) + SiLU + the group
    quantizer on the m130m-shaped conv input (binary16, 8 x 1536 x 2048, the
    layer's x standing in for the in_proj output), int8 codes straight out.
    Algorithmic bytes: 2 in + 1 out per element (weights negligible)."""
    from quantized_state_space_b200 import api
    b, d, L = layer.b, layer.d, layer.L
    rng = np.random.default_rng(12)
    w = torch.from_numpy(rng.uniform(-0.5, 0.5, size=(d, 4)).astype(np.float32)).to(dev)
    bs = torch.from_numpy(rng.uniform(-0.2, 0.2, size=d).astype(np.float32)).to(dev)
    codes = torch.empty((b, d, L), dtype=torch.int8, device=dev)

    def conv():
        api.conv_silu_quantize(layer.x, w, bias=bs, x_group=layer.grp, x_scale=layer.xs,
                               codes=codes)

    t = _timed(torch, conv, 20)
    byts = b * d * L * 3 + d * 4 * 5
    return {"workload": "m130m conv input (8 x 1536 x 2048 binary16) -> causal conv W 4 + "
                        "SiLU + int8 group codes (8 clusters), one launch",
            "ms": round(t * 1e3, 4), "value": round(b * d * L / t / 1e9, 3), "unit": UNIT,
            "roofline": {"bound": "hbm", "achieved": round(byts / t / 1e9, 1),
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(byts / t / 1e9 / pk["hbm_gbs"], 4),
                         "algorithmic_bytes_per_launch": byts,
                         "traffic": measured_traffic("conv_vec_kernel")}}


def run_forms(dev, pk, mhz, only=None, layer=None, ex2=None):
    import torch
    out = {}
    if layer is not None and (not only or "conv" in only):
        try:
            out["conv"] = form_conv(torch, dev, pk, layer)
        except Exception as e:
            out["conv"] = {"error": "%s: %s" % (type(e).__name__, e)}
    if layer is not None and (not only or "calibrate" in only):
        try:
            out["calibrate"] = form_calibrate(torch, dev, pk, layer)
        except Exception as e:
            out["calibrate"] = {"error": "%s: %s" % (type(e).__name__, e)}
        torch.cuda.empty_cache()
    for name, fn in (("ssd27b", lambda: form_ssd(torch, dev, pk)),
                     ("decode8b", lambda: form_decode(torch, dev, pk)),
                     ("softedge", lambda: form_softedge(torch, dev, pk, mhz, ex2)),
                     ("tiny", lambda: form_tiny(torch, dev))):
        if only and name not in only:
            continue
        try:
            out[name] = fn()
        except Exception as e:  # a failing form is reported, the headline stands
            out[name] = {"error": "%s: %s" % (type(e).__name__, e)}
        torch.cuda.empty_cache()
    return out


# ---- reference arm: the CPU oracle ------------------------------------------

def run_reference(args):
    world, rank, _ = rank_env()
    if rank != 0:
        return
    from oracle import oracle as O
    from quantized_state_space_b200 import calibrate, synth

    class Dummy:
        pass

    lay = Dummy()
    lay.dm, lay.raw = synth.workload_inputs(WORKLOAD, seed=0)
    dm = lay.dm
    lay.b, lay.L, lay.d, lay.N, lay.G, lay.gs, lay.k = (dm["batch"], dm["seqlen"], dm["dim"],
                                                       dm["dstate"], dm["ngroups"],
                                                       dm["state_group_size"], dm["x_clusters"])
    threads = O.default_threads()
    # each step: one batch row (d x L channel rows), sized for a few minutes total
    per = []
    for i in range(max(args.warmup, 3) + args.steps):
        r = cpu_baseline(lay, threads=threads, max_units=lay.d)
        if i >= max(args.warmup, 3):
            per.append(r["seconds"])
    s = sum(per)
    units = lay.d * lay.L * len(per)
    v = units / s / 1e9
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 5), "unit": UNIT,
           "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
           "ms_per_step": round(1e3 * s / len(per), 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded numpy draws shaped like the workload; no dataset)",
           "config": dict(config_dict(dm), parallelism="host cores"),
           "cpu_baseline": {"value": round(v, 5), "unit": UNIT, "cores": threads, "kind": "oracle",
                            "sample": "per step: 1 of %d batch rows (%d channel rows x L %d), "
                                      "static quantize + double-precision scan" %
                                      (lay.b, lay.d, lay.L)},
           "e2e": {"value": round(v, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_kernel(args):
    """Profiling aid: one kernel on its workload, `--warmup` untimed then
    `--steps` timed launches (no benchmark line)."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from quantized_state_space_b200 import api
    name = args.kernel
    if name == "ex2":
        print(json.dumps(dict(kernel="ex2_rate_kernel (SFU exp2 throughput probe)",
                              **measure_ex2(torch, dev))), flush=True)
        return
    if name == "conv":
        lay = Layer(dev, 0)
        rng = np.random.default_rng(12)
        w = torch.from_numpy(rng.uniform(-0.5, 0.5, size=(lay.d, 4)).astype(np.float32)).to(dev)
        bs = torch.from_numpy(rng.uniform(-0.2, 0.2, size=lay.d).astype(np.float32)).to(dev)
        fn = (lambda: api.conv_silu_quantize(lay.x, w, bias=bs, x_group=lay.grp,
                                             x_scale=lay.xs, codes=lay.xq))
        label = "m130m conv input: causal conv + SiLU + int8 group codes"
    elif name in ("scan", "scan-int8", "quantize", "quantize-batch"):
        global WORKLOAD
        WORKLOAD = args.workload
        lay = Layer(dev, 0, fused=name == "scan")
        lay.quantize()
        k = args.time_segments
        fn = {"scan": lambda: lay.scan(k), "scan-int8": lambda: lay.scan(k),
              "quantize-batch": lay.quantize,
              "quantize": (lambda: api.quantize_groups(lay.x, lay.b, lay.d, lay.L, lay.grp, lay.k,
                                                       scales=lay.xs, out=lay.xq))}[name]
        label = args.workload + " " + {"scan": "selective scan, binary16 x encoded in the scan",
                            "scan-int8": "selective scan of int8 x codes",
                            "quantize": "x quantize (static scales)",
                            "quantize-batch": "x, B, C quantize in one launch"}[name]
    elif name == "ssd":
        c = setup_ssd(torch, dev)
        c["quant"]()
        fn, label = c["ssd"], "ssd27b SSD chunk scan"
    elif name in ("encode", "softedge-scan"):
        c = setup_softedge(torch, dev)
        c["enc"]()
        c["quant_bc"]()
        fn = c["enc"] if name == "encode" else c["scan"]
        label = "softedge " + ("encode" if name == "encode" else "scan of soft-edge codes")
    else:  # decode
        c = setup_decode(torch, dev, steps=args.warmup + args.steps + 1)
        it = iter(range(args.warmup + args.steps + 1))
        fn, label = (lambda: c["step"](next(it))), "decode8b single-token update"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    if args.steps > 1:
        ms = _timed(torch, fn, args.steps - 1) * 1e3  # first timed-region launch included
    else:
        fn()
        torch.cuda.synchronize()
        ms = None
    print(json.dumps({"kernel": label, "ms_per_launch": ms, "launches": args.warmup + args.steps}),
          flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-forms", action="store_true")
    ap.add_argument("--forms", default="", help="comma list of m130m_other_x_path,m130m_int8_y,conv,calibrate,ssd27b,"
                         "decode8b,softedge,tiny")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fused", action="store_true",
                    help="headline step with binary16 x encoded inside the scan (byte-identical "
                         "result; default: x quantized by its own launch, the faster path here)")
    ap.add_argument("--kernel", choices=["scan", "scan-int8", "quantize", "quantize-batch",
                                         "ssd", "encode", "softedge-scan", "decode", "ex2",
                                         "conv"],
                    help="profiling aid: run only this kernel on its workload")
    ap.add_argument("--workload", choices=["m130m", "tiny", "softedge"], default="m130m",
                    help="with --kernel scan / scan-int8 / quantize / quantize-batch: the "
                         "Mamba-1 workload")
    ap.add_argument("--time-segments", type=int, default=1,
                    help="with --kernel scan / scan-int8: time segments of the scan call")
    args = ap.parse_args()
    if args.kernel:
        run_kernel(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
