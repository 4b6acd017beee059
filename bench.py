#!/usr/bin/env python
"""Benchmark of the selective-SSM mixer core on B200.

One step = one pass of the whole hot path over one batch of the Mamba-130M
layer workload (8 sequences x 2048 tokens, d_inner 1536, N 16, conv width 4,
bf16 activations, fp32 state): causal conv1d + SiLU with conv-state output,
the selective scan with final-state output, then one decode step of the 8
rows from those states. The headline is tokens x channels per second of
the step (Gtoken*ch/s). The scan's throughput is also given as a share of
its special-function-unit roofline (d_inner * N exponentials per token).

Each step reads a different one of 4 input sets (about 600 MB together),
so no step finds its inputs in the 126 MB L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --scan-sweep [NPT,SCHED ...]   # scan alone per kernel variant

With N > 1 (torchrun) every rank runs the same workload on its own GPU (the
path shards with no exchange: replicas), and the value counts every rank's
tokens over the slowest rank's time. `--impl reference` times the fp64 CPU
oracle on a bounded channel sample instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "scan Gtoken·ch/s and % of HBM/MUFU roofline; decode steps/s at B=256"
UNIT = "Gtoken*ch/s"
HEADLINE = "mamba130m_layer_b8_l2048"
N_STATE = 16
SMS = 148
MUFU_PER_CLK_PER_SM = 16  # ex2 results per clock per SM (special-function unit)
FALLBACK_HBM_GBS = 6650.0
# kernel that each scan schedule launches (ssm_set_scan_variant numbering)
SCAN_KERNELS = {1: "scan_kernel", 2: "scan_tma_kernel", 3: "scan_ts_kernel", 4: "scan_tma_kernel",
                5: "scan_tma_kernel", 6: "scan_ws_kernel", 7: "scan_warp_kernel",
                8: "scan_staged_kernel"}


# ---------------------------------------------------------------------------
# environment
# ---------------------------------------------------------------------------

def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the packed, long-context and decode workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--replay-windows", type=int, nargs="+", default=[3], metavar="W",
                    help="checkpoint intervals of the replay decode measurement")
    ap.add_argument("--profile-scan-bwd", nargs="?", const="packed", default=None,
                    choices=["packed", "layer"],
                    help="instead of the step: run 3 backward scans, untimed, for ncu captures: "
                         "over 16384 packed tokens of 5120 channels (packed, about 2.2 GB) or "
                         "over the Mamba-130M layer's 8 x 2048 x 1536 (layer)")
    ap.add_argument("--profile-decode", type=int, default=None, metavar="W",
                    help="instead of the step: run 3 windows of replay decode steps (checkpoint "
                         "every W tokens, bf16 copy) and 3 eager decode steps at 256 x 8192 from "
                         "random states, untimed, as a small case for ncu captures")
    ap.add_argument("--scan-sweep", nargs="*", metavar="NPT,SCHED", default=None,
                    help="instead of the step: time the scan alone for each variant "
                         "(states per lane, schedule; default: a standard list) on the "
                         "four prefill shapes and print one JSON line per measurement")
    return ap.parse_args()


def dist_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "sm_max_mhz": float(pk.get("sm_max_mhz", 1965.0)),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0, "source": "fallback"}


def mufu_peak_gexp(sm_mhz: float) -> float:
    return SMS * MUFU_PER_CLK_PER_SM * sm_mhz * 1e6 / 1e9


def source_sha(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "selective_state_space_causal_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, sha: str):
    """DRAM bytes per launch from profiles/ncu_traffic.txt, if taken on this source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    try:
        for line in open(path):
            f = line.split()
            if len(f) >= 4 and not line.startswith("#") and f[0] == kernel and f[1] == sha:
                return float(f[3])
    except OSError:
        pass
    return None


class ClockSampler(threading.Thread):
    """Polls SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period: float = 0.01):
        super().__init__(daemon=True)
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._halt = threading.Event()
        self.ok = False

    def run(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            hd = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(hd, pynvml.NVML_CLOCK_SM)
            self.ok = True
            while not self._halt.is_set():
                self.samples.append(pynvml.nvmlDeviceGetClockInfo(hd, pynvml.NVML_CLOCK_SM))
                mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(hd)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
                time.sleep(self.period)
        except Exception as e:  # NVML missing: report no clocks rather than fail
            self.error = str(e)

    def stop(self):
        self._halt.set()
        self.join(timeout=2)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons - {"gpu_idle"})}


# ---------------------------------------------------------------------------
# workloads on the device
# ---------------------------------------------------------------------------

class Layer:
    def __init__(self, D, seed=0):
        import torch

        from selective_state_space_causal_b200 import synth

        prm = synth.make_params(seed, D)
        dev = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
        self.w, self.b, self.A = dev(prm.conv_w), dev(prm.conv_b), dev(prm.A)
        self.Dskip, self.dt_bias = dev(prm.Dskip), dev(prm.dt_bias)
        self.D = D


def _events(n):
    import torch

    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def _barrier_sync(world):
    import torch
    import torch.distributed as dist

    if world > 1:
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def _max_over_ranks(x: float, world: int) -> float:
    """Slowest rank's value (timings are taken per rank on the device)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Units all ranks processed per second, in G/s, over the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3) / 1e9


class HeadlineStep:
    """conv -> scan -> one decode step on the Mamba-130M layer shape."""

    SETS = 4

    def __init__(self, seed=0):
        import torch

        from selective_state_space_causal_b200 import synth

        import selective_state_space_causal_b200 as ssm

        self.ssm = ssm
        w = synth.WORKLOADS[HEADLINE]
        self.Bn, self.L, self.D, self.K = w["batch"], w["seqlen"], w["D"], w["K"]
        self.tok = self.Bn * self.L
        self.layer = Layer(self.D, seed)
        self.sets = [synth.device_activations(seed + i, self.tok, self.D) for i in range(self.SETS)]
        self.dec = [synth.device_activations(seed + 100 + i, self.Bn, self.D)
                    for i in range(self.SETS)]
        bf = torch.bfloat16
        self.xc = torch.empty((self.tok, self.D), dtype=bf, device="cuda")
        self.y = torch.empty_like(self.xc)
        self.cs = torch.empty((self.Bn, self.D, self.K - 1), dtype=bf, device="cuda")
        self.h = torch.empty((self.Bn, self.D, N_STATE), device="cuda")
        self.yd = torch.empty((self.Bn, self.D), dtype=bf, device="cuda")

    def units(self):
        return self.tok * self.D

    def scan_exps(self):
        return self.tok * self.D * N_STATE

    def run(self, i, ev=None, inputs=None, dec_inputs=None, y=None, yd=None):
        ssm, ly = self.ssm, self.layer
        a = inputs if inputs is not None else self.sets[i % self.SETS]
        d = dec_inputs if dec_inputs is not None else self.dec[i % self.SETS]
        y = self.y if y is None else y
        yd = self.yd if yd is None else yd
        ssm.ssm_causal_conv1d(a["x"], self.xc, ly.w, bias=ly.b, S=self.Bn,
                              conv_state_out=self.cs)
        if ev is not None:
            ev[0].record()
        ssm.ssm_selective_scan_fwd(self.xc, a["dt"], ly.A, a["B"], a["C"], y, Dskip=ly.Dskip,
                                   z=a["z"], dt_bias=ly.dt_bias, h_final=self.h, S=self.Bn)
        if ev is not None:
            ev[1].record()
        ssm.ssm_selective_state_update(self.cs, self.h, d["x"], d["dt"], d["B"], d["C"], yd,
                                       ly.w, ly.A, z=d["z"], conv_b=ly.b, Dskip=ly.Dskip,
                                       dt_bias=ly.dt_bias)


def bench_headline(args, world, peaks, rank_dev):
    import torch

    st = HeadlineStep()
    for i in range(args.warmup):
        st.run(i)
    K = args.steps
    evs = [_events(2) for _ in range(K)]
    start, stop = _events(2)
    launches0 = st.ssm.ssm_launch_count()
    clocks = ClockSampler(rank_dev)
    clocks.start()
    time.sleep(0.05)
    _barrier_sync(world)
    start.record()
    for i in range(K):
        st.run(i, ev=evs[i])
    stop.record()
    _barrier_sync(world)
    clk = clocks.stop()
    launches = st.ssm.ssm_launch_count() - launches0
    ms = start.elapsed_time(stop) / K
    scan_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    ms_max = _max_over_ranks(ms, world)
    value = whole_job_rate(st.units(), world, ms_max)

    mufu = mufu_peak_gexp(peaks["sm_max_mhz"])
    achieved = st.scan_exps() / (scan_ms * 1e-3) / 1e9
    sha = source_sha("scan.cu", "scan_parts.cuh", "common.cuh")
    npt, sched = st.ssm.ssm_scan_variant_for(st.Bn, st.D)
    kernel = SCAN_KERNELS.get(sched, "scan_tma_kernel")
    traffic = recorded_traffic(kernel, sha)
    roofline = {"kernel": kernel, "variant": {"states_per_lane": npt, "schedule": sched},
                "bound": "alu", "unit": "Gexp/s",
                "achieved": round(achieved, 1), "peak": round(mufu, 1),
                "frac": round(achieved / mufu, 4), "traffic": traffic,
                "kernel_ms": round(scan_ms, 5),
                "algorithmic_bytes_per_launch": st.tok * st.D * 8 + st.tok * 64 + st.Bn * st.D * 64,
                "peak_basis": f"{SMS} SMs x {MUFU_PER_CLK_PER_SM} ex2/clk x {peaks['sm_max_mhz']:.0f} MHz",
                "hbm_peak_gbs": peaks["hbm_gbs"], "hbm_peak_source": peaks["source"]}
    roofline["hbm_frac"] = round(roofline["algorithmic_bytes_per_launch"] / (scan_ms * 1e-3)
                                 / 1e9 / peaks["hbm_gbs"], 4)
    res = {"value": value, "ms_per_step": ms_max, "roofline": roofline, "clocks": clk,
           "gpu_launches": int(launches), "step_ms_this_rank": ms}

    # the same step with the fused conv -> scan kernel
    def fused_step(i, ev=None):
        ssm_, ly = st.ssm, st.layer
        a = st.sets[i % st.SETS]
        d = st.dec[i % st.SETS]
        if ev is not None:
            ev[0].record()
        ssm_.ssm_conv_scan_fwd(a["x"], ly.w, a["dt"], ly.A, a["B"], a["C"], st.y, conv_b=ly.b,
                               conv_state_out=st.cs, Dskip=ly.Dskip, z=a["z"],
                               dt_bias=ly.dt_bias, h_final=st.h, S=st.Bn)
        if ev is not None:
            ev[1].record()
        ssm_.ssm_selective_state_update(st.cs, st.h, d["x"], d["dt"], d["B"], d["C"], st.yd, ly.w,
                                        ly.A, z=d["z"], conv_b=ly.b, Dskip=ly.Dskip,
                                        dt_bias=ly.dt_bias)

    for i in range(args.warmup):
        fused_step(i)
    Kf = max(10, K // 4)
    fevs = [_events(2) for _ in range(Kf)]
    _barrier_sync(world)
    start.record()
    for i in range(Kf):
        fused_step(i, fevs[i])
    stop.record()
    _barrier_sync(world)
    fms = _max_over_ranks(start.elapsed_time(stop) / Kf, world)
    f_kernel_ms = sum(e[0].elapsed_time(e[1]) for e in fevs) / Kf
    res["fused_step"] = {
        "value": whole_job_rate(st.units(), world, fms), "unit": UNIT, "ms_per_step": fms,
        "conv_scan_kernel_ms": round(f_kernel_ms, 5),
        "mufu_frac": round(st.scan_exps() / (f_kernel_ms * 1e-3) / 1e9 / mufu, 4),
        "step": "ssm_conv_scan_fwd (fused conv1d+silu -> selective_scan) -> 1 decode step"}

    # end to end through the public API with pinned host buffers
    host_in = {k: v.cpu().pin_memory() for k, v in st.sets[0].items()}
    host_dec = {k: v.cpu().pin_memory() for k, v in st.dec[0].items()}
    dev_in = {k: torch.empty_like(v) for k, v in st.sets[0].items()}
    dev_dec = {k: torch.empty_like(v) for k, v in st.dec[0].items()}
    y_host = torch.empty(st.y.shape, dtype=st.y.dtype).pin_memory()
    yd_host = torch.empty(st.yd.shape, dtype=st.yd.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host_in.values()) + sum(
        v.numel() * v.element_size() for v in host_dec.values())
    d2h = y_host.numel() * y_host.element_size() + yd_host.numel() * yd_host.element_size()

    def e2e_step(i):
        for k in dev_in:
            dev_in[k].copy_(host_in[k], non_blocking=True)
        for k in dev_dec:
            dev_dec[k].copy_(host_dec[k], non_blocking=True)
        st.run(i, inputs=dev_in, dec_inputs=dev_dec)
        y_host.copy_(st.y, non_blocking=True)
        yd_host.copy_(st.yd, non_blocking=True)

    for i in range(max(3, args.warmup // 4)):
        e2e_step(i)
    Ke = max(10, K // 4)
    _barrier_sync(world)
    start.record()
    for i in range(Ke):
        e2e_step(i)
    stop.record()
    _barrier_sync(world)
    ems_serial = _max_over_ranks(start.elapsed_time(stop) / Ke, world)

    # The same steps pipelined the way a serving loop runs them: step i+1's
    # inputs are copied in (one stream) while step i computes (a second) and
    # step i-1's outputs are copied out (a third), with double-buffered device
    # inputs and outputs; every step still copies its own inputs in and its
    # own outputs out inside the timed region.
    s_in, s_cmp, s_out = (torch.cuda.Stream() for _ in range(3))
    dev_in2 = [dev_in, {k: torch.empty_like(v) for k, v in dev_in.items()}]
    dev_dec2 = [dev_dec, {k: torch.empty_like(v) for k, v in dev_dec.items()}]
    y2 = [st.y, torch.empty_like(st.y)]
    yd2 = [st.yd, torch.empty_like(st.yd)]
    y_host2 = [y_host, torch.empty_like(y_host).pin_memory()]
    yd_host2 = [yd_host, torch.empty_like(yd_host).pin_memory()]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def pipelined(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[b])  # step i-2 has read these inputs
                for k in dev_in2[b]:
                    dev_in2[b][k].copy_(host_in[k], non_blocking=True)
                for k in dev_dec2[b]:
                    dev_dec2[b][k].copy_(host_dec[k], non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[b])
                if i >= 2:
                    s_cmp.wait_event(ev_out[b])  # step i-2's outputs are copied out
                st.run(i, inputs=dev_in2[b], dec_inputs=dev_dec2[b], y=y2[b], yd=yd2[b])
                ev_cmp[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[b])
                y_host2[b].copy_(y2[b], non_blocking=True)
                yd_host2[b].copy_(yd2[b], non_blocking=True)
                ev_out[b].record(s_out)

    torch.cuda.synchronize()
    pipelined(max(3, args.warmup // 4))
    torch.cuda.synchronize()
    _barrier_sync(world)
    start.record(s_in)
    pipelined(Ke)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    stop.record(s_out)
    torch.cuda.synchronize()
    _barrier_sync(world)
    ems = _max_over_ranks(start.elapsed_time(stop) / Ke, world)
    res["e2e"] = {"value": whole_job_rate(st.units(), world, ems), "unit": UNIT,
                  "ms_per_step": ems, "h2d_bytes_per_step": int(h2d),
                  "d2h_bytes_per_step": int(d2h),
                  "how": "pipelined: copy-in, compute and copy-out streams, double-buffered"}
    res["e2e_serial"] = {"value": whole_job_rate(st.units(), world, ems_serial), "unit": UNIT,
                         "ms_per_step": ems_serial,
                         "how": "copy in, compute, copy out, one step after another"}
    del st
    torch.cuda.empty_cache()
    return res


def bench_secondary(peaks, world, steps_scale=1.0, replay_windows=(3,)):
    """Packed varlen prefill, chunked long-context prefill and batch-256 decode."""
    import torch

    import selective_state_space_causal_b200 as ssm
    from selective_state_space_causal_b200 import synth

    out = {}
    mufu = mufu_peak_gexp(peaks["sm_max_mhz"])
    bf = torch.bfloat16

    # -- packed variable-length prefill ------------------------------------
    w = synth.WORKLOADS["packmamba_2p8b_varlen_65536"]
    D, tot = w["D"], w["total"]
    lens = synth.sample_lengths(0, tot, w["len_lo"], w["len_hi"])
    cu = torch.from_numpy(synth.cu_from_lengths(lens)).cuda()
    S = len(lens)
    ly = Layer(D)
    a = synth.device_activations(0, tot, D)
    xc = torch.empty_like(a["x"])
    y = torch.empty_like(a["x"])
    cs = torch.empty((S, D, 3), dtype=bf, device="cuda")
    h = torch.empty((S, D, N_STATE), device="cuda")
    ws = torch.empty(max(1, ssm.ssm_scan_workspace_size(tot, D, N_STATE, S)), dtype=torch.uint8,
                     device="cuda")

    def step(ev=None):
        ssm.ssm_causal_conv1d(a["x"], xc, ly.w, bias=ly.b, cu_seqlens=cu, conv_state_out=cs)
        if ev:
            ev[0].record()
        ssm.ssm_selective_scan_fwd(xc, a["dt"], ly.A, a["B"], a["C"], y, Dskip=ly.Dskip, z=a["z"],
                                   dt_bias=ly.dt_bias, h_final=h, cu_seqlens=cu, workspace=ws)
        if ev:
            ev[1].record()

    for _ in range(3):
        step()
    n = max(3, int(20 * steps_scale))
    evs = [_events(2) for _ in range(n)]
    s0, s1 = _events(2)
    _barrier_sync(world)
    s0.record()
    for i in range(n):
        step(evs[i])
    s1.record()
    _barrier_sync(world)
    ms = _max_over_ranks(s0.elapsed_time(s1) / n, world)
    scan_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / n
    out["packmamba_2p8b_varlen_65536"] = {
        "gtoken_ch_per_s": tot * D * world / (ms * 1e-3) / 1e9, "ms_per_step": ms,
        "scan_ms": scan_ms, "scan_mufu_frac": round(tot * D * N_STATE / (scan_ms * 1e-3) / 1e9 / mufu, 4),
        "sequences": S, "step": "conv1d+selective_scan (packed, longest-first schedule)"}
    del xc, y, cs, h, ws
    torch.cuda.empty_cache()

    # -- backward of the packed prefill's scan (PackMamba training) ---------
    out["packmamba_2p8b_varlen_65536_scan_bwd"] = bench_scan_bwd(peaks, world, ly, a, cu, S,
                                                                steps_scale)
    del a
    torch.cuda.empty_cache()

    # -- backward at the Mamba-130M layer shape (8 dense rows of 2048) -------
    wl = synth.WORKLOADS["mamba130m_layer_b8_l2048"]
    lyl = Layer(wl["D"])
    al = synth.device_activations(0, wl["batch"] * wl["seqlen"], wl["D"])
    out["mamba130m_layer_b8_l2048_scan_bwd"] = bench_scan_bwd(
        peaks, world, lyl, al, None, wl["batch"], steps_scale, label="8 x 2048 x 1536 (dense rows)")
    del al
    torch.cuda.empty_cache()

    # -- long-context chunked prefill --------------------------------------
    w = synth.WORKLOADS["falcon_mamba7b_longctx_131072"]
    D, L, chunk = w["D"], w["seqlen"], w["chunk"]
    ly = Layer(D)
    a = synth.device_activations(1, L, D)
    xc = torch.empty((chunk, D), dtype=bf, device="cuda")
    y = torch.empty((L, D), dtype=bf, device="cuda")
    cs = torch.zeros((1, D, 3), dtype=bf, device="cuda")
    h = torch.zeros((1, D, N_STATE), device="cuda")

    def prefill(evs=None):
        cs.zero_()
        h.zero_()
        for j, c0 in enumerate(range(0, L, chunk)):
            sl = slice(c0, c0 + chunk)
            ssm.ssm_causal_conv1d(a["x"][sl], xc, ly.w, bias=ly.b, conv_state_in=cs,
                                  conv_state_out=cs)
            if evs:
                evs[j][0].record()
            ssm.ssm_selective_scan_fwd(xc, a["dt"][sl], ly.A, a["B"][sl], a["C"][sl], y[sl],
                                       Dskip=ly.Dskip, z=a["z"][sl], dt_bias=ly.dt_bias, h0=h,
                                       h_final=h)
            if evs:
                evs[j][1].record()

    prefill()
    n = max(2, int(3 * steps_scale))
    nch = L // chunk
    evs = [[_events(2) for _ in range(nch)] for _ in range(n)]
    _barrier_sync(world)
    s0.record()
    for i in range(n):
        prefill(evs[i])
    s1.record()
    _barrier_sync(world)
    ms = _max_over_ranks(s0.elapsed_time(s1) / n, world)
    scan_ms = sum(e[0].elapsed_time(e[1]) for row in evs for e in row) / n
    out["falcon_mamba7b_longctx_131072"] = {
        "gtoken_ch_per_s": L * D * world / (ms * 1e-3) / 1e9, "ms_per_prefill": ms,
        "scan_ms_per_prefill": scan_ms,
        "scan_mufu_frac": round(L * D * N_STATE / (scan_ms * 1e-3) / 1e9 / mufu, 4),
        "step": "16 x (conv1d + selective_scan) of 8192 tokens, states carried"}
    del a, xc, y
    torch.cuda.empty_cache()

    # -- batch-256 decode ----------------------------------------------------
    w = synth.WORKLOADS["decode_b256_d8192"]
    Bt, D, L0, steps = w["batch"], w["D"], w["prefill_len"], w["steps"]
    ly = Layer(D)
    a = synth.device_activations(2, Bt * L0, D)
    xc = torch.empty_like(a["x"])
    yp = torch.empty_like(a["x"])
    cs = torch.empty((Bt, D, 3), dtype=bf, device="cuda")
    h = torch.empty((Bt, D, N_STATE), device="cuda")
    ssm.ssm_causal_conv1d(a["x"], xc, ly.w, bias=ly.b, S=Bt, conv_state_out=cs)
    ssm.ssm_selective_scan_fwd(xc, a["dt"], ly.A, a["B"], a["C"], yp, Dskip=ly.Dskip, z=a["z"],
                               dt_bias=ly.dt_bias, h_final=h, S=Bt)
    del a, xc, yp
    torch.cuda.empty_cache()
    block = 100
    yd = torch.empty((Bt, D), dtype=bf, device="cuda")
    total_ms = 0.0
    done = 0
    for b0 in range(0, steps, block):
        blk = [synth.device_activations(5000 + b0 + i, Bt, D) for i in range(block)]
        _barrier_sync(world)
        s0.record()
        for s in blk:
            ssm.ssm_selective_state_update(cs, h, s["x"], s["dt"], s["B"], s["C"], yd, ly.w, ly.A,
                                           z=s["z"], conv_b=ly.b, Dskip=ly.Dskip,
                                           dt_bias=ly.dt_bias)
        s1.record()
        _barrier_sync(world)
        total_ms += _max_over_ranks(s0.elapsed_time(s1), world)
        done += block
        del blk
    per = total_ms / done
    bytes_step = (Bt * D * N_STATE * 4 * 2 + Bt * D * 3 * 2 * 2 + Bt * D * 2 * 4
                  + Bt * N_STATE * 2 * 2 + D * (4 * 4 + 3 * 4 + N_STATE * 4))
    out["decode_b256_d8192"] = {
        "steps_per_s": 1e3 / per * world, "ms_per_step": per, "steps": done,
        "algorithmic_bytes_per_step": bytes_step,
        "hbm_frac": round(bytes_step / (per * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        "step": "ssm_selective_state_update, 256 rows x 8192 channels, fresh inputs per step"}
    for W in replay_windows:
        out[f"decode_b256_d8192_replay_w{W}"] = bench_replay(peaks, world, ly, cs, h, W, steps,
                                                             mufu)
    del cs, h
    torch.cuda.empty_cache()
    return out


def bench_scan_bwd(peaks, world, ly, a, cu, S, steps_scale=1.0, label="packed 65536 x 5120"):
    """Backward of the selective scan on a prefill's inputs (bf16 activations,
    upstream gradient dy drawn like x; packed when cu is given, else S dense
    rows). Algorithmic work per
    (token, channel): 2 x 16 exponentials (the decays of one forward pass to
    produce the states and of the reverse pass; the kernel executes 3 x 16, as
    it recomputes the states chunk by chunk from checkpoints instead of storing
    them) and 14 bytes (u, dt, z, dy in; du, ddelta, dz out)."""
    import torch

    import selective_state_space_causal_b200 as ssm
    from selective_state_space_causal_b200 import synth

    tok, D = a["x"].shape
    dy = synth.device_activations(77, tok, D)["x"]
    f32 = dict(device="cuda", dtype=torch.float32)
    g = {"du": torch.empty_like(a["x"]), "ddelta": torch.empty_like(a["x"]),
         "dz": torch.empty_like(a["x"]), "dB": torch.empty((tok, N_STATE), **f32),
         "dC": torch.empty((tok, N_STATE), **f32), "dA": torch.empty((D, N_STATE), **f32),
         "dDskip": torch.empty((D,), **f32), "ddt_bias": torch.empty((D,), **f32),
         "dh0": torch.empty((S, D, N_STATE), **f32)}
    ws = torch.empty(ssm.ssm_scan_bwd_workspace_size(tok, D, N_STATE, S), dtype=torch.uint8,
                     device="cuda")

    def call():
        ssm.ssm_selective_scan_bwd(a["x"], a["dt"], ly.A, a["B"], a["C"], dy, g, Dskip=ly.Dskip,
                                   z=a["z"], dt_bias=ly.dt_bias, cu_seqlens=cu, S=S,
                                   workspace=ws)

    def timed(variant):
        ssm.ssm_set_scan_bwd_variant(variant)
        for _ in range(2):
            call()
        n = max(3, int(10 * steps_scale))
        s0, s1 = _events(2)
        _barrier_sync(world)
        s0.record()
        for _ in range(n):
            call()
        s1.record()
        _barrier_sync(world)
        return _max_over_ranks(s0.elapsed_time(s1) / n, world)

    # both kernels (4 lanes per channel; one thread per channel), then the
    # library's own choice, which is the reported figure
    per_variant = {str(v): round(timed(v), 4) for v in (1, 2)}
    ms = timed(0)
    mufu = mufu_peak_gexp(peaks["sm_max_mhz"])
    units = tok * D
    res = {"gtoken_ch_per_s": units * world / (ms * 1e-3) / 1e9, "ms_per_call": ms,
           "mufu_frac": round(units * 2 * N_STATE / (ms * 1e-3) / 1e9 / mufu, 4),
           "executed_exp_frac": round(units * 3 * N_STATE / (ms * 1e-3) / 1e9 / mufu, 4),
           "hbm_frac": round(units * 14 / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
           "variant": ssm.ssm_scan_bwd_variant_for(S, D), "ms_per_variant": per_variant,
           "workspace_bytes": ws.numel(), "sequences": S,
           "step": f"ssm_selective_scan_bwd over the {label} prefill, all gradients"}
    del g, ws, dy
    return res


def replay_bytes_per_step(Bt, D, W, keep_lo=True):
    """Algorithmic HBM bytes of one replay decode step, averaged over a window of
    W steps taken in lockstep by every row (buffer lengths 0, 1, ..., W-1).

    Per (row, channel): conv state 6 B in and out, x, dt, z in and y out (2 B
    each); a step with j buffered tokens reads the checkpoint copy (32 B bf16,
    or 64 B fp32 without the copy), j buffered (delta, delta*xc) pairs (8 B
    each) and writes its own pair (8 B); the checkpoint step (j = W-1) instead
    reads the fp32 checkpoint (64 B), the W-1 pairs, and writes the checkpoint
    (64 B) and its copy (32 B). Per row: B and C (bf16, 32 B each), buffered B
    rows (64 B each), the new B row (64 B). Per channel: A, conv weight and
    biases, Dskip (92 B)."""
    per_ch = 0
    per_row = 0
    for j in range(W):
        per_ch += 12 + 8
        per_row += 2 * N_STATE * 2 + 64 * j
        if j == W - 1:
            per_ch += 64 + 8 * j + 64 + (32 if keep_lo else 0)
        else:
            per_ch += (32 if keep_lo else 64) + 8 * j + 8
            per_row += 64
    total = Bt * D * per_ch + Bt * per_row + W * D * (4 * 4 + 3 * 4 + N_STATE * 4)
    return total / W


def bench_replay(peaks, world, ly, cs, h, W, steps, mufu):
    """Batch-256 decode through the replay kernels (checkpoint + input buffer,
    bf16 checkpoint copy), on the same prefill states and the same kind of
    fresh per-step inputs as the eager decode measurement."""
    import torch

    import selective_state_space_causal_b200 as ssm
    from selective_state_space_causal_b200 import synth

    Bt, D = h.shape[0], h.shape[1]
    rep = ssm.replay_buffers(Bt, D, W, "cuda", keep_lo=True)
    rep["ckpt"].copy_(h)
    csr = cs.clone()
    ssm.ssm_replay_reset(rep)
    yd = torch.empty((Bt, D), dtype=torch.bfloat16, device="cuda")
    s0, s1 = _events(2)
    block = 100
    total_ms = 0.0
    done = 0
    l0 = ssm.ssm_launch_count()
    for b0 in range(0, steps, block):
        blk = [synth.device_activations(5000 + b0 + i, Bt, D) for i in range(block)]
        _barrier_sync(world)
        s0.record()
        for s in blk:
            ssm.ssm_replay_state_update(csr, rep, s["x"], s["dt"], s["B"], s["C"], yd, ly.w, ly.A,
                                        z=s["z"], conv_b=ly.b, Dskip=ly.Dskip,
                                        dt_bias=ly.dt_bias)
        s1.record()
        _barrier_sync(world)
        total_ms += _max_over_ranks(s0.elapsed_time(s1), world)
        done += block
        del blk
    launches = ssm.ssm_launch_count() - l0
    per = total_ms / done
    bytes_step = replay_bytes_per_step(Bt, D, W)
    exps_step = Bt * D * N_STATE * (W + 1) / 2
    res = {
        "steps_per_s": 1e3 / per * world, "ms_per_step": per, "steps": done, "window": W,
        "algorithmic_bytes_per_step": int(bytes_step),
        "hbm_frac": round(bytes_step / (per * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        "mufu_frac": round(exps_step / (per * 1e-3) / 1e9 / mufu, 4),
        "gpu_launches_per_step": launches / done,
        "step": f"ssm_replay_state_update (checkpoint every {W} tokens, bf16 copy for outputs), "
                "256 rows x 8192 channels, fresh inputs per step"}
    del rep, csr
    return res


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def oracle_sample_step(orc, n_ch, seed=0):
    """Returns a callable running the oracle on `n_ch` channels of the headline
    workload (conv, scan, one decode step) and the units it covers."""
    import numpy as np

    from selective_state_space_causal_b200 import synth

    w = synth.WORKLOADS[HEADLINE]
    Bn, L, D = w["batch"], w["seqlen"], w["D"]
    tok = Bn * L
    prm = synth.make_params(seed, D)
    rng = np.random.default_rng(seed)
    ch = np.sort(rng.choice(D, n_ch, replace=False))
    act = synth.make_activations(seed, tok, n_ch, bf16=True)
    dec = synth.make_activations(seed + 1, Bn, n_ch, bf16=True)
    cw, cb, A, Dk, dtb = (prm.conv_w[ch], prm.conv_b[ch], prm.A[ch], prm.Dskip[ch],
                          prm.dt_bias[ch])

    def run():
        xc, cs = orc.causal_conv1d(act["x"], cw, cb, S=Bn, want_state=True)
        _, h = orc.selective_scan(xc, act["dt"], A, act["B"], act["C"], Dskip=Dk, z=act["z"],
                                  dt_bias=dtb, S=Bn, want_state=True)
        orc.state_update(cs, h, dec["x"], dec["dt"], dec["B"], dec["C"], dec["z"], cw, cb, A, Dk,
                         dtb)

    return run, tok * n_ch


def cpu_baseline(n_ch=192):
    import oracle

    orc = oracle.load()
    run, units = oracle_sample_step(orc, n_ch)
    run()  # warm
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        if time.perf_counter() - t0 > 3.0:
            break
    dt = (time.perf_counter() - t0) / reps
    return {"value": units / dt / 1e9, "unit": UNIT, "cores": orc.num_threads(), "kind": "oracle",
            "sample": f"{HEADLINE}: all 8x2048 tokens of {n_ch} of 1536 channels "
                      f"(conv, scan and one decode step), {reps} repetitions, fp64"}


def bench_reference(args):
    rank, _, world = dist_info()
    if rank != 0:
        return 0
    import oracle

    orc = oracle.load()
    n_ch = 32
    run, units = oracle_sample_step(orc, n_ch)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t0
    ms = el / args.steps * 1e3
    value = units / (el / args.steps) / 1e9
    sample = (f"{HEADLINE}: all 8x2048 tokens of {n_ch} of 1536 channels per step "
              "(conv, scan and one decode step), fp64 oracle on the host cores")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": HEADLINE, "batch": 8, "seq_len": 2048,
                                            "d_inner": 1536, "d_state": 16, "d_conv": 4,
                                            "channels_sampled": n_ch},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------

SWEEP_VARIANTS = [(0, 0), (2, 8), (4, 8), (8, 2), (4, 1), (8, 7), (8, 6), (2, 3)]


def scan_sweep(variants, peaks):
    """Scan alone per variant on the prefill shapes; one JSON line each."""
    import torch

    import selective_state_space_causal_b200 as ssm
    from selective_state_space_causal_b200 import synth

    mufu = mufu_peak_gexp(peaks["sm_max_mhz"])
    lens = synth.sample_lengths(0, 65536)
    shapes = [("mamba130m_layer_b8_l2048", 16384, 1536, None, 8),
              ("packmamba_2p8b_varlen_65536", 65536, 5120, synth.cu_from_lengths(lens), len(lens)),
              ("falcon_mamba7b_longctx_131072 (one 8192-token call)", 8192, 8192, None, 1),
              ("uniform_32x2048_d5120", 65536, 5120, synth.cu_from_lengths([2048] * 32), 32)]
    for name, tok, D, cu, S in shapes:
        prm = synth.make_params(0, D)
        A, Dk, dtb = (torch.from_numpy(v).cuda() for v in (prm.A, prm.Dskip, prm.dt_bias))
        cu_d = torch.from_numpy(cu).cuda() if cu is not None else None
        sets = [synth.device_activations(i, tok, D) for i in range(3)]
        y = torch.empty((tok, D), dtype=torch.bfloat16, device="cuda")
        h = torch.empty((S, D, N_STATE), device="cuda")
        ws = torch.empty(max(1, ssm.ssm_scan_workspace_size(tok, D, N_STATE, S)),
                         dtype=torch.uint8, device="cuda")
        for npt, sched in variants:
            ssm.ssm_set_scan_variant(npt, sched)
            picked = ssm.ssm_scan_variant_for(S, D)

            def call(a):
                ssm.ssm_selective_scan_fwd(a["x"], a["dt"], A, a["B"], a["C"], y, Dskip=Dk,
                                           z=a["z"], dt_bias=dtb, h_final=h, cu_seqlens=cu_d,
                                           S=S, workspace=ws if cu_d is not None else None)

            for i in range(3):
                call(sets[i % 3])
            torch.cuda.synchronize()
            n = 30 if tok * D < 1e9 else 10
            e0, e1 = _events(2)
            e0.record()
            for i in range(n):
                call(sets[i % 3])
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / n
            gexp = tok * D * N_STATE / (ms * 1e-3) / 1e9
            print(json.dumps({"workload": name, "states_per_lane": picked[0], "schedule": picked[1],
                              "auto": npt == 0 and sched == 0, "scan_ms": round(ms, 4),
                              "gexp_per_s": round(gexp, 1), "mufu_frac": round(gexp / mufu, 4)}),
                  flush=True)
        ssm.ssm_set_scan_variant(0, 0)
        del sets
        torch.cuda.empty_cache()
    if ssm.ssm_device_status() != 0:
        raise RuntimeError("a bounded device wait timed out during the sweep")
    return 0


def profile_scan_bwd(shape="packed"):
    """Three backward scans, for profiler captures: on a quarter of the packed
    workload, or on the Mamba-130M layer shape (8 dense rows)."""
    import torch

    import selective_state_space_causal_b200 as ssm
    from selective_state_space_causal_b200 import synth

    if shape == "layer":
        D, tot = 1536, 8 * 2048
        lens = [2048] * 8
    else:
        D, tot = 5120, 16384
        lens = synth.sample_lengths(0, tot, 128, 8192)
    cu = torch.from_numpy(synth.cu_from_lengths(lens)).cuda()
    ly = Layer(D)
    a = synth.device_activations(0, tot, D)
    dy = synth.device_activations(1, tot, D)["x"]
    f32 = dict(device="cuda", dtype=torch.float32)
    g = {"du": torch.empty_like(a["x"]), "ddelta": torch.empty_like(a["x"]),
         "dz": torch.empty_like(a["x"]), "dB": torch.empty((tot, N_STATE), **f32),
         "dC": torch.empty((tot, N_STATE), **f32), "dA": torch.empty((D, N_STATE), **f32),
         "dDskip": torch.empty((D,), **f32), "ddt_bias": torch.empty((D,), **f32),
         "dh0": torch.empty((len(lens), D, N_STATE), **f32)}
    ws = torch.empty(ssm.ssm_scan_bwd_workspace_size(tot, D, N_STATE, len(lens)),
                     dtype=torch.uint8, device="cuda")
    for _ in range(3):
        ssm.ssm_selective_scan_bwd(a["x"], a["dt"], ly.A, a["B"], a["C"], dy, g, Dskip=ly.Dskip,
                                   z=a["z"], dt_bias=ly.dt_bias, cu_seqlens=cu, workspace=ws)
    torch.cuda.synchronize()
    assert ssm.ssm_device_status() == 0
    print(json.dumps({"profile_scan_bwd": {"tokens": tot, "d_inner": D, "sequences": len(lens),
                                           "variant": ssm.ssm_scan_bwd_variant_for(len(lens), D)}}))


def profile_decode(W):
    """A few replay and eager decode steps at 256 x 8192 from random states
    (about 0.5 GB on the device), for profiler captures; prints nothing timed."""
    import torch

    import selective_state_space_causal_b200 as ssm
    from selective_state_space_causal_b200 import synth

    Bt, D = 256, 8192
    ly = Layer(D)
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    h = 0.3 * torch.randn((Bt, D, N_STATE), device="cuda", generator=g)
    cs = torch.randn((Bt, D, 3), device="cuda", generator=g).to(torch.bfloat16)
    rep = ssm.replay_buffers(Bt, D, W, "cuda", keep_lo=True)
    rep["ckpt"].copy_(h)
    ssm.ssm_replay_reset(rep)
    ins = [synth.device_activations(10 + i, Bt, D) for i in range(4)]
    y = torch.empty((Bt, D), dtype=torch.bfloat16, device="cuda")
    for i in range(3 * W):
        s = ins[i % 4]
        ssm.ssm_replay_state_update(cs, rep, s["x"], s["dt"], s["B"], s["C"], y, ly.w, ly.A,
                                    z=s["z"], conv_b=ly.b, Dskip=ly.Dskip, dt_bias=ly.dt_bias)
    for i in range(3):
        s = ins[i % 4]
        ssm.ssm_selective_state_update(cs, h, s["x"], s["dt"], s["B"], s["C"], y, ly.w, ly.A,
                                       z=s["z"], conv_b=ly.b, Dskip=ly.Dskip, dt_bias=ly.dt_bias)
    torch.cuda.synchronize()
    assert ssm.ssm_device_status() == 0
    print(json.dumps({"profile_decode": {"window": W, "replay_steps": 3 * W, "eager_steps": 3}}))


def main():
    args = parse_args()
    if args.profile_decode is not None:
        profile_decode(args.profile_decode)
        return
    if args.profile_scan_bwd:
        profile_scan_bwd(args.profile_scan_bwd)
        return
    if args.impl == "reference":
        return bench_reference(args)
    if args.scan_sweep is not None:
        import torch

        torch.cuda.set_device(0)
        variants = ([tuple(int(x) for x in v.split(",")) for v in args.scan_sweep]
                    if args.scan_sweep else SWEEP_VARIANTS)
        return scan_sweep(variants, load_peaks())
    rank, local, world = dist_info()
    import torch

    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    peaks = load_peaks()
    res = bench_headline(args, world, peaks, local)
    secondary = None if args.no_secondary else bench_secondary(peaks, world, replay_windows=tuple(args.replay_windows))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()
    if rank == 0:
        line = {
            "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "io_dtype": "bf16", "data": "synthetic",
            "config": {"workload": HEADLINE, "batch": 8, "seq_len": 2048, "d_inner": 1536,
                       "d_state": 16, "d_conv": 4,
                       "step": "causal_conv1d+silu -> selective_scan (h_final) -> 1 decode step",
                       "l2": "4 rotating input sets (~600 MB) larger than L2",
                       "parallelism": f"replicas x{world}"},
            "roofline": res["roofline"], "clocks": res["clocks"], "e2e": res["e2e"],
            "e2e_serial": res["e2e_serial"], "fused_step": res["fused_step"],
            "gpu_launches": res["gpu_launches"], "cpu_baseline": cpu, "workloads": secondary,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
