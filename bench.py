#!/usr/bin/env python
"""Benchmark of the selective-SSM mixer core on B200.

Headline step: one long-context prefill at the Falcon-Mamba-7B layer shape,
then one decode token. The 131072-token sequence (d_inner 8192, N 16, conv
width 4, bf16 activations, fp32 state) is processed in 16 calls of 8192
tokens, each a causal conv1d + SiLU and a selective scan, with the SSM state
carried in place and the conv state between two buffers; the conv of chunk
j+1 runs on a second stream beside the scan of chunk j (it needs only the conv
state); the row then takes one decode step from the final states. The step is
captured once as a CUDA graph and replayed (--no-graph: plain launches). The
headline value is tokens x channels per second of the whole step
(Gtoken*ch/s), with the inputs resident in HBM (6.4 GB of inputs, far larger
than the 126 MB L2, so no step finds them in L2).

The scan, which dominates the step, is bound by the special-function unit (16
ex2 per token and channel); its roofline is exps per second against the
special-function unit's peak, measured in the same run with an ex2 throughput
probe (the unit-count figure 148 SMs x 16 ex2/clk x clock is given beside it).

Also reported: the same step end to end through the C ABI with the inputs in
pinned host memory (copies inside the timed region), the fp64 CPU oracle on a
channel sample of the same workload, and the other workloads (the Mamba-130M
layer, the packed PackMamba prefill, batch-256 decode, replay decode and the
backward scan), each with its own roofline, e2e and oracle figures.

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
import importlib.util
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
HEADLINE = "falcon_mamba7b_longctx_131072"
LAYER = "mamba130m_layer_b8_l2048"
PACKED = "packmamba_2p8b_varlen_65536"
DECODE = "decode_b256_d8192"
N_STATE = 16
SMS = 148
MUFU_PER_CLK_PER_SM = 16  # ex2 results per clock per SM (special-function unit)
FALLBACK_HBM_GBS = 6650.0
ORACLE_CHANNELS = 256     # channel sample of the CPU baseline on the large workloads
# kernel that each scan schedule launches (ssm_set_scan_variant numbering)
SCAN_KERNELS = {1: "scan_kernel", 2: "scan_tma_kernel", 3: "scan_ts_kernel", 4: "scan_tma_kernel",
                5: "scan_tma_kernel", 6: "scan_ws_kernel", 7: "scan_warp_kernel",
                8: "scan_staged_kernel", 9: "scan_pipe_kernel", 10: "scan_pipe_kernel",
                11: "scan_pipe_kernel", 12: "scan_wide_kernel"}
SCAN_SOURCES = ("scan.cu", "scan_pipe.cu", "scan_pipe.cuh", "scan_parts.cuh", "common.cuh", "tma.cuh")


# ---------------------------------------------------------------------------
# environment
# ---------------------------------------------------------------------------

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the Mamba-130M layer, packed, decode and backward workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the headline step as plain launches instead of a CUDA graph")
    ap.add_argument("--replay-windows", type=int, nargs="+", default=[2, 3], metavar="W",
                    help="checkpoint intervals of the replay decode measurement")
    ap.add_argument("--replay-copy", choices=["both", "bf16", "none"], default="both",
                    help="replay decode with the bf16 checkpoint copy for outputs (bf16), "
                         "with outputs from the fp32 checkpoint (none), or both")
    ap.add_argument("--profile-scan-bwd", nargs="?", const="packed", default=None,
                    choices=["packed", "layer"],
                    help="instead of the step: run 3 backward scans, untimed, for ncu captures: "
                         "over 16384 packed tokens of 5120 channels (packed, about 2.2 GB) or "
                         "over the Mamba-130M layer's 8 x 2048 x 1536 (layer)")
    ap.add_argument("--profile-decode", type=int, default=None, metavar="W",
                    help="instead of the step: run 3 windows of replay decode steps (checkpoint "
                         "every W tokens, bf16 copy) and 3 eager decode steps at 256 x 8192 from "
                         "random states, untimed, as a small case for ncu captures")
    ap.add_argument("--profile-scan", default=None,
                    choices=["layer", "long", "packed", "packed_fused", "conv_long",
                             "decode_fresh"],
                    help="instead of the step: 3 untimed calls of one kernel's workload for ncu "
                         "captures (the Mamba-130M layer scan, one 8192 x 8192 long-context scan "
                         "call, a 16384-token slice of the packed scan, the same slice through "
                         "the fused conv -> scan, one 8192 x 8192 conv call, or 3 eager decode "
                         "steps at 256 x 8192 on fresh inputs)")
    ap.add_argument("--scan-sweep", nargs="*", metavar="NPT,SCHED", default=None,
                    help="instead of the step: time the scan alone for each variant "
                         "(states per lane, schedule; default: a standard list) on the "
                         "four prefill shapes and print one JSON line per measurement")
    return ap.parse_args(argv)


def dist_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def load_synth():
    """The seeded input generator, loaded by file path: it holds no method
    arithmetic and needs neither the CUDA library nor the package."""
    path = os.path.join(ROOT, "selective_state_space_causal_b200", "synth.py")
    spec = importlib.util.spec_from_file_location("ssm_synth_inputs", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


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
    """Unit-count figure: SMs x 16 ex2 per clock x clock."""
    return SMS * MUFU_PER_CLK_PER_SM * sm_mhz * 1e6 / 1e9


def source_sha(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "selective_state_space_causal_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, sha: str):
    """DRAM bytes per launch of `kernel` on `workload` from profiles/ncu_traffic.txt,
    if they were taken on the current source (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    try:
        for line in open(path):
            f = line.split()
            if (len(f) >= 5 and not line.startswith("#") and f[0] == kernel and f[1] == workload
                    and f[2] == sha):
                return float(f[4])
    except OSError:
        pass
    return None


class ClockSampler(threading.Thread):
    """Polls SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period: float = 0.005):
        super().__init__(daemon=True)
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._halt = threading.Event()

    def run(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            hd = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(hd, pynvml.NVML_CLOCK_SM)
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
# timing helpers
# ---------------------------------------------------------------------------

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


def measure_mufu_peak(rank_dev: int):
    """ex2 throughput of the device (probe kernel over every SM, best of 5)."""
    import torch

    import selective_state_space_causal_b200 as ssm

    sink = torch.empty(ssm.ssm_probe_sink_floats(), device="cuda")
    iters = 20000
    ssm.ssm_probe_rate(0, iters // 10, sink)
    torch.cuda.synchronize()
    clocks = ClockSampler(rank_dev, 0.002)
    clocks.start()
    e0, e1 = _events(2)
    best, ops = None, 0.0
    for _ in range(5):
        e0.record()
        ops = ssm.ssm_probe_rate(0, iters, sink)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    clk = clocks.stop()
    gexp = ops / (best * 1e-3) / 1e9
    mhz = clk["sm_mhz"]
    return {"gexp_per_s": round(gexp, 1), "probe_ms": round(best, 4), "sm_mhz": mhz,
            "ex2_per_clk_per_sm": round(gexp * 1e9 / (SMS * mhz * 1e6), 3) if mhz else None,
            "how": "ex2.approx.ftz.f32, 8 independent chains per thread, 2048 threads per SM, "
                   "every SM; best of 5 launches (ssm_probe_rate kind 0)"}


class Layer:
    """Per-channel parameters of one mixer layer, on the device."""

    def __init__(self, D, seed=0):
        import torch

        synth = load_synth()
        prm = synth.make_params(seed, D)
        dev = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
        self.w, self.b, self.A = dev(prm.conv_w), dev(prm.conv_b), dev(prm.A)
        self.Dskip, self.dt_bias = dev(prm.Dskip), dev(prm.dt_bias)
        self.D = D


def scan_roofline(kernel, variant, exps, bytes_, kernel_ms, mufu, peaks, workload, sha):
    """The roofline block of a scan kernel: bound by the special-function unit."""
    achieved = exps / (kernel_ms * 1e-3) / 1e9
    return {"kernel": kernel, "variant": {"states_per_lane": variant[0], "schedule": variant[1]},
            "bound": "alu", "unit": "Gexp/s", "achieved": round(achieved, 1),
            "peak": mufu["gexp_per_s"], "frac": round(achieved / mufu["gexp_per_s"], 4),
            "peak_source": "measured in this run (ex2 throughput probe)",
            "peak_unit_count": round(mufu_peak_gexp(peaks["sm_max_mhz"]), 1),
            "frac_of_unit_count": round(achieved / mufu_peak_gexp(peaks["sm_max_mhz"]), 4),
            "traffic": recorded_traffic(kernel, workload, sha),
            "kernel_ms": round(kernel_ms, 5), "exps_per_launch": int(exps),
            "algorithmic_bytes_per_launch": int(bytes_),
            "hbm_frac": round(bytes_ / (kernel_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "hbm_peak_gbs": peaks["hbm_gbs"], "hbm_peak_source": peaks["source"]}


def conv_bytes(tok, D, S, state_in):
    """Algorithmic bytes of one bf16 conv call: x in and xc out (2 B each per
    token and channel), the conv state out (and in), 3 bf16 per sequence and
    channel, and the fp32 weights and bias."""
    return tok * D * 4 + S * D * 6 * (2 if state_in else 1) + D * 20


def conv_roofline(bytes_, kernel_ms, peaks, workload, two_launches=False):
    """The roofline block of a conv call: bound by HBM. With the state updated
    in place the state output is a second, small launch, timed with it."""
    achieved = bytes_ / (kernel_ms * 1e-3) / 1e9
    kernel = "conv1d_tma_kernel" + (" + conv_state_out_kernel" if two_launches else "")
    return {"kernel": kernel, "bound": "hbm", "unit": "GB/s", "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "frac": round(achieved / peaks["hbm_gbs"], 4),
            "peak_source": peaks["source"],
            "traffic": recorded_traffic("conv1d_tma_kernel", workload,
                                        source_sha("conv1d.cu", "common.cuh", "tma.cuh")),
            "kernel_ms": round(kernel_ms, 5), "algorithmic_bytes_per_launch": int(bytes_)}


def scan_bytes(tok, D, S):
    """Algorithmic bytes of one bf16 scan call: u, dt, z in and y out (2 B each
    per token and channel), B and C (64 B per token), the final state (64 B
    per sequence and channel, plus h0 when carried)."""
    return tok * D * 8 + tok * 64 + S * D * 64


# ---------------------------------------------------------------------------
# headline: long-context prefill (16 chunked calls) + one decode step
# ---------------------------------------------------------------------------

class LongCtxStep:
    def __init__(self, seed=0):
        import torch

        import selective_state_space_causal_b200 as ssm

        synth = load_synth()
        self.ssm = ssm
        w = synth.WORKLOADS[HEADLINE]
        self.L, self.D, self.chunk, self.K = w["seqlen"], w["D"], w["chunk"], w["K"]
        self.nch = self.L // self.chunk
        self.layer = Layer(self.D, seed)
        self.a = synth.device_activations(seed + 1, self.L, self.D)
        self.dec = synth.device_activations(seed + 101, 1, self.D)
        bf = torch.bfloat16
        # chunk j's conv output goes to xcs[j % 2]: the conv of chunk j + 1 runs
        # on a second stream while the scan of chunk j runs (it needs only the
        # conv state, not h), on the SMs the scan's grid leaves half empty
        self.xcs = [torch.empty((self.chunk, self.D), dtype=bf, device="cuda") for _ in range(2)]
        self.xc = self.xcs[0]
        self.s_conv = torch.cuda.Stream()
        self.ev_conv = [torch.cuda.Event() for _ in range(self.nch)]
        self.ev_scan = [torch.cuda.Event() for _ in range(self.nch)]
        self.y = torch.empty((self.L, self.D), dtype=bf, device="cuda")
        # the conv state alternates between two buffers (chunk j reads cs[j % 2]
        # and writes cs[(j + 1) % 2]), so the state output rides along with the
        # conv kernel instead of a second launch after it
        self.cs = [torch.zeros((1, self.D, self.K - 1), dtype=bf, device="cuda") for _ in range(2)]
        self.h = torch.zeros((1, self.D, N_STATE), device="cuda")
        self.yd = torch.empty((1, self.D), dtype=bf, device="cuda")

    def units(self):
        return self.L * self.D

    def conv_only(self):
        """The step's 16 conv calls alone, one after another."""
        ssm, ly, a = self.ssm, self.layer, self.a
        for j in range(self.nch):
            sl = slice(j * self.chunk, (j + 1) * self.chunk)
            ssm.ssm_causal_conv1d(a["x"][sl], self.xcs[j % 2], ly.w, bias=ly.b,
                                  conv_state_in=self.cs[j % 2],
                                  conv_state_out=self.cs[(j + 1) % 2])

    def run(self, ev=None):
        """One step; ev[j] (4 events per chunk) brackets chunk j's conv (on the
        conv stream) and scan (on the current stream)."""
        import torch

        ssm, ly, a = self.ssm, self.layer, self.a
        main, sc = torch.cuda.current_stream(), self.s_conv
        self.cs[0].zero_()
        self.h.zero_()
        sc.wait_stream(main)
        for j in range(self.nch):
            sl = slice(j * self.chunk, (j + 1) * self.chunk)
            with torch.cuda.stream(sc):
                if j >= 2:
                    sc.wait_event(self.ev_scan[j - 2])  # the scan two back has read xcs[j % 2]
                if ev is not None:
                    ev[j][0].record(sc)
                ssm.ssm_causal_conv1d(a["x"][sl], self.xcs[j % 2], ly.w, bias=ly.b,
                                      conv_state_in=self.cs[j % 2],
                                      conv_state_out=self.cs[(j + 1) % 2])
                if ev is not None:
                    ev[j][1].record(sc)
                self.ev_conv[j].record(sc)
            main.wait_event(self.ev_conv[j])
            if ev is not None:
                ev[j][2].record(main)
            ssm.ssm_selective_scan_fwd(self.xcs[j % 2], a["dt"][sl], ly.A, a["B"][sl], a["C"][sl],
                                       self.y[sl], Dskip=ly.Dskip, z=a["z"][sl],
                                       dt_bias=ly.dt_bias, h0=self.h, h_final=self.h)
            if ev is not None:
                ev[j][3].record(main)
            self.ev_scan[j].record(main)
        main.wait_stream(sc)
        d = self.dec
        ssm.ssm_selective_state_update(self.cs[self.nch % 2], self.h, d["x"], d["dt"], d["B"],
                                       d["C"], self.yd, ly.w, ly.A, z=d["z"], conv_b=ly.b,
                                       Dskip=ly.Dskip, dt_bias=ly.dt_bias)


def bench_headline(args, world, peaks, rank_dev, mufu):
    import torch

    st = LongCtxStep()
    for _ in range(args.warmup):
        st.run()
    K = args.steps
    # kernel times: the step with an event pair around every conv and scan call
    evs = [[_events(4) for _ in range(st.nch)] for _ in range(K)]
    launches0 = st.ssm.ssm_launch_count()
    p0, p1 = _events(2)
    _barrier_sync(world)
    p0.record()
    for i in range(K):
        st.run(ev=evs[i])
    p1.record()
    _barrier_sync(world)
    launches_per_step = (st.ssm.ssm_launch_count() - launches0) / K
    plain_ms = p0.elapsed_time(p1) / K
    conv_in_step_ms = sum(e[0].elapsed_time(e[1]) for row in evs for e in row) / (K * st.nch)
    scan_ms = sum(e[2].elapsed_time(e[3]) for row in evs for e in row) / (K * st.nch)
    # the conv calls alone (in the step they run beside the scans, so their
    # event times there measure waiting for room, not the kernel)
    cevs = [_events(2) for _ in range(K)]
    for i in range(K):
        cevs[i][0].record()
        st.conv_only()
        cevs[i][1].record()
    torch.cuda.synchronize()
    conv_ms = sum(e[0].elapsed_time(e[1]) for e in cevs) / (K * st.nch)
    # the timed steps: the step captured once as a CUDA graph (its 33 library
    # launches and 2 fills) and replayed, which removes the host's launch gaps
    graph = None
    if not args.no_graph:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            st.run()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            st.run()
        for _ in range(2):
            graph.replay()
    step = graph.replay if graph is not None else st.run
    launches0 = st.ssm.ssm_launch_count()
    start, stop = _events(2)
    clocks = ClockSampler(rank_dev)
    clocks.start()
    time.sleep(0.05)
    _barrier_sync(world)
    start.record()
    for _ in range(K):
        step()
    stop.record()
    _barrier_sync(world)
    clk = clocks.stop()
    # a replayed graph launches the captured kernels without calling the library
    launches = launches_per_step * K if graph is not None else (st.ssm.ssm_launch_count()
                                                                 - launches0)
    if st.ssm.ssm_device_status() != 0:
        raise RuntimeError("a bounded device wait timed out during the timed region")
    ms = start.elapsed_time(stop) / K
    ms_max = _max_over_ranks(ms, world)
    value = whole_job_rate(st.units(), world, ms_max)
    sha = source_sha(*SCAN_SOURCES)
    variant = st.ssm.ssm_scan_variant_for(1, st.D)
    kernel = SCAN_KERNELS.get(variant[1], "scan_kernel")
    roofline = scan_roofline(kernel, variant, st.chunk * st.D * N_STATE,
                             scan_bytes(st.chunk, st.D, 2), scan_ms, mufu, peaks,
                             "longctx_call_8192x8192", sha)
    res = {"value": value, "ms_per_step": ms_max, "step_ms_this_rank": ms, "roofline": roofline,
           "clocks": clk, "gpu_launches": int(launches), "cuda_graph": graph is not None,
           "step_ms_without_graph": round(plain_ms, 4),
           "scan_ms_per_step": round(scan_ms * st.nch, 4),
           "conv_roofline": dict(conv_roofline(conv_bytes(st.chunk, st.D, 1, True), conv_ms,
                                               peaks, "longctx_call_8192x8192"),
                                 measured="the 16 conv calls alone; in the step each runs "
                                          "beside a scan",
                                 in_step_event_ms=round(conv_in_step_ms, 5)),
           "launches_per_step": launches_per_step}
    del graph
    if not args.no_e2e:
        res["e2e"] = e2e_longctx(st, world, max(3, K // 4))
    del st
    torch.cuda.empty_cache()
    return res


def e2e_longctx(st, world, steps):
    """The headline step through the C ABI with its inputs in pinned host
    memory: every step copies all 16 chunks' inputs in and the whole y out.
    Pipelined by chunk on three streams: chunk j+1's inputs are copied in while
    chunk j computes and chunk j-1's output is copied out; the device staging
    buffers are double-buffered."""
    import torch

    bf = torch.bfloat16
    names = ("x", "dt", "z", "B", "C")
    host = {k: torch.empty(st.a[k].shape, dtype=bf, pin_memory=True) for k in names}
    for k in names:
        host[k].copy_(st.a[k])
    host_dec = {k: torch.empty(st.dec[k].shape, dtype=bf, pin_memory=True) for k in names}
    for k in names:
        host_dec[k].copy_(st.dec[k])
    y_host = torch.empty((st.L, st.D), dtype=bf, pin_memory=True)
    yd_host = torch.empty((1, st.D), dtype=bf, pin_memory=True)
    st.a = None  # the resident inputs are not used here
    torch.cuda.empty_cache()
    c, ssm, ly = st.chunk, st.ssm, st.layer
    stage = [{k: torch.empty((c,) + tuple(host[k].shape[1:]), dtype=bf, device="cuda")
              for k in names} for _ in range(2)]
    ystage = [torch.empty((c, st.D), dtype=bf, device="cuda") for _ in range(2)]
    dec_dev = {k: torch.empty(v.shape, dtype=bf, device="cuda") for k, v in host_dec.items()}
    s_in, s_cmp, s_out = (torch.cuda.Stream() for _ in range(3))
    ev_in, ev_used, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    ev_dec, ev_decdone = torch.cuda.Event(), torch.cuda.Event()
    h2d = sum(v.numel() * v.element_size() for v in host.values()) + sum(
        v.numel() * v.element_size() for v in host_dec.values())
    d2h = y_host.numel() * y_host.element_size() + yd_host.numel() * yd_host.element_size()
    g = [0]  # chunks issued so far, over all steps (picks the staging buffer)

    def step():
        with torch.cuda.stream(s_in):
            for k in names:
                dec_dev[k].copy_(host_dec[k], non_blocking=True)
            ev_dec.record(s_in)
        with torch.cuda.stream(s_cmp):
            st.cs[0].zero_()
            st.h.zero_()
        for j in range(st.nch):
            b, n = g[0] % 2, g[0]
            g[0] += 1
            with torch.cuda.stream(s_in):
                if n >= 2:
                    s_in.wait_event(ev_used[b])  # the chunk two back has read this stage
                for k in names:
                    stage[b][k].copy_(host[k][j * c:(j + 1) * c], non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[b])
                if n >= 2:
                    s_cmp.wait_event(ev_out[b])  # its output has been copied out
                a = stage[b]
                ssm.ssm_causal_conv1d(a["x"], st.xc, ly.w, bias=ly.b, conv_state_in=st.cs[j % 2],
                                      conv_state_out=st.cs[(j + 1) % 2])
                ssm.ssm_selective_scan_fwd(st.xc, a["dt"], ly.A, a["B"], a["C"], ystage[b],
                                           Dskip=ly.Dskip, z=a["z"], dt_bias=ly.dt_bias,
                                           h0=st.h, h_final=st.h)
                ev_used[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_used[b])
                y_host[j * c:(j + 1) * c].copy_(ystage[b], non_blocking=True)
                ev_out[b].record(s_out)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_dec)
            d = dec_dev
            ssm.ssm_selective_state_update(st.cs[st.nch % 2], st.h, d["x"], d["dt"], d["B"],
                                           d["C"], st.yd, ly.w, ly.A, z=d["z"], conv_b=ly.b,
                                           Dskip=ly.Dskip, dt_bias=ly.dt_bias)
            ev_decdone.record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_decdone)
            yd_host.copy_(st.yd, non_blocking=True)

    torch.cuda.synchronize()
    step()
    torch.cuda.synchronize()
    e0, e1 = _events(2)
    _barrier_sync(world)
    e0.record(s_in)
    for _ in range(steps):
        step()
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    e1.record(s_out)
    torch.cuda.synchronize()
    _barrier_sync(world)
    ms = _max_over_ranks(e0.elapsed_time(e1) / steps, world)
    out = {"value": whole_job_rate(st.units(), world, ms), "unit": UNIT, "ms_per_step": ms,
           "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "h2d_gb_per_s": round(h2d / (ms * 1e-3) / 1e9, 2),
           "how": "pinned host inputs copied in and y copied out every step, pipelined by "
                  "8192-token chunk on three streams (copy-in, compute, copy-out)"}
    del host, y_host, stage, ystage
    return out


# ---------------------------------------------------------------------------
# other workloads
# ---------------------------------------------------------------------------

class LayerStep:
    """conv -> scan -> one decode step on the Mamba-130M layer shape (8 x 2048 x 1536)."""

    SETS = 4

    def __init__(self, seed=0):
        import torch

        import selective_state_space_causal_b200 as ssm

        synth = load_synth()
        self.ssm = ssm
        w = synth.WORKLOADS[LAYER]
        self.Bn, self.L, self.D, self.K = w["batch"], w["seqlen"], w["D"], w["K"]
        self.tok = self.Bn * self.L
        self.layer = Layer(self.D, seed)
        self.sets = [synth.device_activations(seed + i, self.tok, self.D) for i in range(self.SETS)]
        self.dec = [synth.device_activations(seed + 100 + i, self.Bn, self.D)
                    for i in range(self.SETS)]
        bf = torch.bfloat16
        self.xc = torch.empty((self.tok, self.D), dtype=bf, device="cuda")
        self.y = torch.empty((self.tok, self.D), dtype=bf, device="cuda")
        self.cs = torch.empty((self.Bn, self.D, self.K - 1), dtype=bf, device="cuda")
        self.h = torch.empty((self.Bn, self.D, N_STATE), device="cuda")
        self.yd = torch.empty((self.Bn, self.D), dtype=bf, device="cuda")

    def units(self):
        return self.tok * self.D

    def run(self, i, ev=None, inputs=None, dec_inputs=None, y=None, yd=None):
        ssm, ly = self.ssm, self.layer
        a = inputs if inputs is not None else self.sets[i % self.SETS]
        d = dec_inputs if dec_inputs is not None else self.dec[i % self.SETS]
        y = self.y if y is None else y
        yd = self.yd if yd is None else yd
        if ev is not None:
            ev[0].record()
        ssm.ssm_causal_conv1d(a["x"], self.xc, ly.w, bias=ly.b, S=self.Bn,
                              conv_state_out=self.cs)
        if ev is not None:
            ev[1].record()
        ssm.ssm_selective_scan_fwd(self.xc, a["dt"], ly.A, a["B"], a["C"], y, Dskip=ly.Dskip,
                                   z=a["z"], dt_bias=ly.dt_bias, h_final=self.h, S=self.Bn)
        if ev is not None:
            ev[2].record()
        ssm.ssm_selective_state_update(self.cs, self.h, d["x"], d["dt"], d["B"], d["C"], yd,
                                       ly.w, ly.A, z=d["z"], conv_b=ly.b, Dskip=ly.Dskip,
                                       dt_bias=ly.dt_bias)


def _pipelined_e2e(run_compute, host_in, dev_shapes, y_dev_pair, y_host_pair, world, steps):
    """Step i+1's inputs copied in (one stream) while step i computes (a second)
    and step i-1's outputs are copied out (a third), double-buffered."""
    import torch

    s_in, s_cmp, s_out = (torch.cuda.Stream() for _ in range(3))
    dev_in = [{k: torch.empty_like(v, device="cuda") for k, v in host_in.items()}
              for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[b])
                for k in host_in:
                    dev_in[b][k].copy_(host_in[k], non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[b])
                if i >= 2:
                    s_cmp.wait_event(ev_out[b])
                run_compute(i, dev_in[b], b)
                ev_cmp[b].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[b])
                for yd, yh in zip(y_dev_pair[b], y_host_pair[b]):
                    yh.copy_(yd, non_blocking=True)
                ev_out[b].record(s_out)

    torch.cuda.synchronize()
    run(3)
    torch.cuda.synchronize()
    e0, e1 = _events(2)
    _barrier_sync(world)
    e0.record(s_in)
    run(steps)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    e1.record(s_out)
    torch.cuda.synchronize()
    _barrier_sync(world)
    return _max_over_ranks(e0.elapsed_time(e1) / steps, world)


def bench_layer(args, world, peaks, mufu):
    import torch

    st = LayerStep()
    for i in range(args.warmup):
        st.run(i)
    K = max(args.steps, 50)
    # kernel times: event pairs around the conv and the scan of every step
    evs = [_events(3) for _ in range(K)]
    l0 = st.ssm.ssm_launch_count()
    for i in range(K):
        st.run(i, ev=evs[i])
    torch.cuda.synchronize()
    launches_per_step = (st.ssm.ssm_launch_count() - l0) / K
    conv_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    scan_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / K
    # the timed steps: each input set's step captured once as a CUDA graph
    graphs = []
    if not args.no_graph:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for i in range(st.SETS):
                st.run(i)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        for i in range(st.SETS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                st.run(i)
            graphs.append(g)
        for g in graphs:
            g.replay()
    step = (lambda i: graphs[i % st.SETS].replay()) if graphs else st.run
    s0, s1 = _events(2)
    _barrier_sync(world)
    s0.record()
    for i in range(K):
        step(i)
    s1.record()
    _barrier_sync(world)
    ms = _max_over_ranks(s0.elapsed_time(s1) / K, world)
    del graphs
    variant = st.ssm.ssm_scan_variant_for(st.Bn, st.D)
    res = {"value": whole_job_rate(st.units(), world, ms), "unit": UNIT, "ms_per_step": ms,
           "gpu_launches_per_step": launches_per_step, "cuda_graph": not args.no_graph,
           "roofline": scan_roofline(SCAN_KERNELS.get(variant[1], "scan_kernel"), variant,
                                     st.tok * st.D * N_STATE, scan_bytes(st.tok, st.D, st.Bn),
                                     scan_ms, mufu, peaks, LAYER, source_sha(*SCAN_SOURCES)),
           "conv_roofline": conv_roofline(conv_bytes(st.tok, st.D, st.Bn, False), conv_ms, peaks,
                                          LAYER),
           "step": "causal_conv1d+silu -> selective_scan (h_final) -> 1 decode step; "
                   "4 rotating input sets (~600 MB) larger than L2; each set's step "
                   "replayed as a CUDA graph"}

    res["scan_bwd"] = bench_scan_bwd(world, st.layer, st.sets[0], None, st.Bn, mufu, peaks,
                                     label="Mamba-130M layer 8 x 2048 x 1536", n=10)

    # the same step with the fused conv -> scan kernel
    def fused(i, ev=None):
        ly, a, d = st.layer, st.sets[i % st.SETS], st.dec[i % st.SETS]
        if ev is not None:
            ev[0].record()
        st.ssm.ssm_conv_scan_fwd(a["x"], ly.w, a["dt"], ly.A, a["B"], a["C"], st.y, conv_b=ly.b,
                                 conv_state_out=st.cs, Dskip=ly.Dskip, z=a["z"],
                                 dt_bias=ly.dt_bias, h_final=st.h, S=st.Bn)
        if ev is not None:
            ev[1].record()
        st.ssm.ssm_selective_state_update(st.cs, st.h, d["x"], d["dt"], d["B"], d["C"], st.yd,
                                          ly.w, ly.A, z=d["z"], conv_b=ly.b, Dskip=ly.Dskip,
                                          dt_bias=ly.dt_bias)

    for i in range(args.warmup):
        fused(i)
    fevs = [_events(2) for _ in range(K)]
    _barrier_sync(world)
    s0.record()
    for i in range(K):
        fused(i, fevs[i])
    s1.record()
    _barrier_sync(world)
    fms = _max_over_ranks(s0.elapsed_time(s1) / K, world)
    fk = sum(e[0].elapsed_time(e[1]) for e in fevs) / K
    res["fused_step"] = {"value": whole_job_rate(st.units(), world, fms), "ms_per_step": fms,
                         "conv_scan_kernel_ms": round(fk, 5),
                         "mufu_frac": round(st.tok * st.D * N_STATE / (fk * 1e-3) / 1e9
                                            / mufu["gexp_per_s"], 4)}
    if not args.no_e2e:
        host_in = {k: v.cpu().pin_memory() for k, v in st.sets[0].items()}
        host_in.update({"d_" + k: v.cpu().pin_memory() for k, v in st.dec[0].items()})
        ys = [(st.y, st.yd), (torch.empty_like(st.y), torch.empty_like(st.yd))]
        yh = [tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in p) for p in ys]

        def compute(i, dev, b):
            a = {k: dev[k] for k in ("x", "dt", "z", "B", "C")}
            d = {k: dev["d_" + k] for k in ("x", "dt", "z", "B", "C")}
            st.run(i, inputs=a, dec_inputs=d, y=ys[b][0], yd=ys[b][1])

        ems = _pipelined_e2e(compute, host_in, None, ys, yh, world, max(10, K // 4))
        res["e2e"] = {"value": whole_job_rate(st.units(), world, ems), "unit": UNIT,
                      "ms_per_step": ems,
                      "h2d_bytes_per_step": sum(v.numel() * v.element_size()
                                                for v in host_in.values()),
                      "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in yh[0]),
                      "how": "pipelined: copy-in, compute and copy-out streams, double-buffered"}
    del st
    torch.cuda.empty_cache()
    return res


def bench_packed(args, world, peaks, mufu):
    import torch

    import selective_state_space_causal_b200 as ssm

    synth = load_synth()
    w = synth.WORKLOADS[PACKED]
    D, tot = w["D"], w["total"]
    lens = synth.sample_lengths(0, tot, w["len_lo"], w["len_hi"])
    cu = torch.from_numpy(synth.cu_from_lengths(lens)).cuda()
    S = len(lens)
    ly = Layer(D)
    a = synth.device_activations(0, tot, D)
    bf = torch.bfloat16
    xc = torch.empty_like(a["x"])
    y = torch.empty_like(a["x"])
    cs = torch.empty((S, D, 3), dtype=bf, device="cuda")
    h = torch.empty((S, D, N_STATE), device="cuda")
    ws = torch.empty(max(1, ssm.ssm_scan_workspace_size(tot, D, N_STATE, S)), dtype=torch.uint8,
                     device="cuda")

    def step(ev=None, src=a, yy=y):
        if ev:
            ev[0].record()
        ssm.ssm_causal_conv1d(src["x"], xc, ly.w, bias=ly.b, cu_seqlens=cu, conv_state_out=cs)
        if ev:
            ev[1].record()
        ssm.ssm_selective_scan_fwd(xc, src["dt"], ly.A, src["B"], src["C"], yy, Dskip=ly.Dskip,
                                   z=src["z"], dt_bias=ly.dt_bias, h_final=h, cu_seqlens=cu,
                                   workspace=ws)
        if ev:
            ev[2].record()

    def fused(ev=None):
        if ev:
            ev[0].record()
        ssm.ssm_conv_scan_fwd(a["x"], ly.w, a["dt"], ly.A, a["B"], a["C"], y, conv_b=ly.b,
                              conv_state_out=cs, Dskip=ly.Dskip, z=a["z"], dt_bias=ly.dt_bias,
                              h_final=h, cu_seqlens=cu)
        if ev:
            ev[1].record()

    def timed(fn, n, marks):
        """Step time and the mean time between consecutive marks."""
        for _ in range(3):
            fn()
        evs = [_events(marks) for _ in range(n)]
        s0, s1 = _events(2)
        _barrier_sync(world)
        s0.record()
        for i in range(n):
            fn(evs[i])
        s1.record()
        _barrier_sync(world)
        return (_max_over_ranks(s0.elapsed_time(s1) / n, world),
                [sum(e[m].elapsed_time(e[m + 1]) for e in evs) / n for m in range(marks - 1)])

    n = max(5, args.steps)
    ms, (conv_ms, scan_ms) = timed(step, n, 3)
    fms, (fk,) = timed(fused, n, 2)
    variant = ssm.ssm_scan_variant_for(S, D)
    res = {"value": whole_job_rate(tot * D, world, ms), "unit": UNIT, "ms_per_step": ms,
           "sequences": S,
           "roofline": scan_roofline(SCAN_KERNELS.get(variant[1], "scan_kernel"), variant,
                                     tot * D * N_STATE, scan_bytes(tot, D, S), scan_ms, mufu,
                                     peaks, PACKED, source_sha(*SCAN_SOURCES)),
           "conv_roofline": conv_roofline(conv_bytes(tot, D, S, False), conv_ms, peaks, PACKED),
           "fused_step": {"value": whole_job_rate(tot * D, world, fms), "ms_per_step": fms,
                          "conv_scan_kernel_ms": round(fk, 5)},
           "step": "conv1d+silu -> selective_scan over 43 packed sequences (longest first)"}
    if not args.no_e2e:
        host_in = {k: v.cpu().pin_memory() for k, v in a.items()}
        ys = [(y,), (torch.empty_like(y),)]
        yh = [(torch.empty(y.shape, dtype=y.dtype).pin_memory(),) for _ in range(2)]

        def compute(i, dev, b):
            step(src=dev, yy=ys[b][0])

        ems = _pipelined_e2e(compute, host_in, None, ys, yh, world, 5)
        res["e2e"] = {"value": whole_job_rate(tot * D, world, ems), "unit": UNIT,
                      "ms_per_step": ems,
                      "h2d_bytes_per_step": sum(v.numel() * v.element_size()
                                                for v in host_in.values()),
                      "d2h_bytes_per_step": y.numel() * y.element_size(),
                      "how": "pipelined: copy-in, compute and copy-out streams, double-buffered"}
    res["scan_bwd"] = bench_scan_bwd(world, ly, a, cu, S, mufu, peaks)
    del a, xc, y, cs, h, ws
    torch.cuda.empty_cache()
    return res


def decode_bytes_per_step(Bt, D):
    """Eager decode: SSM state in and out (64 + 64 B), conv state in and out
    (6 + 6 B), x, dt, z in and y out (2 B each) per (row, channel); B and C
    per row; A, conv weight and bias, Dskip and dt_bias per channel."""
    return (Bt * D * N_STATE * 4 * 2 + Bt * D * 3 * 2 * 2 + Bt * D * 2 * 4
            + Bt * N_STATE * 2 * 2 + D * (4 * 4 + 3 * 4 + N_STATE * 4))


def _time_block(world, steps, use_graph):
    """Device time (ms, max over ranks) of a block of step callables run back
    to back: captured as one CUDA graph outside the timed region and replayed
    inside it, or as plain launches."""
    import torch

    g = None
    if use_graph:
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):  # recorded, not run
            for f in steps:
                f()
    s0, s1 = _events(2)
    _barrier_sync(world)
    s0.record()
    if g is not None:
        g.replay()
    else:
        for f in steps:
            f()
    s1.record()
    _barrier_sync(world)
    ms = _max_over_ranks(s0.elapsed_time(s1), world)
    del g
    return ms


def bench_decode(args, world, peaks, mufu):
    import torch

    import selective_state_space_causal_b200 as ssm

    synth = load_synth()
    w = synth.WORKLOADS[DECODE]
    Bt, D, L0, steps = w["batch"], w["D"], w["prefill_len"], w["steps"]
    ly = Layer(D)
    a = synth.device_activations(2, Bt * L0, D)
    bf = torch.bfloat16
    xc = torch.empty_like(a["x"])
    yp = torch.empty_like(a["x"])
    cs = torch.empty((Bt, D, 3), dtype=bf, device="cuda")
    h = torch.empty((Bt, D, N_STATE), device="cuda")
    ssm.ssm_causal_conv1d(a["x"], xc, ly.w, bias=ly.b, S=Bt, conv_state_out=cs)
    ssm.ssm_selective_scan_fwd(xc, a["dt"], ly.A, a["B"], a["C"], yp, Dskip=ly.Dskip, z=a["z"],
                               dt_bias=ly.dt_bias, h_final=h, S=Bt)
    del a, xc, yp
    torch.cuda.empty_cache()
    cs0, h0 = cs.clone(), h.clone()
    block = 100
    yd = torch.empty((Bt, D), dtype=bf, device="cuda")
    total_ms, done, kernel_ms = 0.0, 0, []

    def one(s):
        ssm.ssm_selective_state_update(cs, h, s["x"], s["dt"], s["B"], s["C"], yd, ly.w, ly.A,
                                       z=s["z"], conv_b=ly.b, Dskip=ly.Dskip, dt_bias=ly.dt_bias)

    for b0 in range(0, steps, block):
        blk = [synth.device_activations(5000 + b0 + i, Bt, D) for i in range(block)]
        # the steps/s value: the block back to back (one CUDA graph), no events
        # between steps
        total_ms += _time_block(world, [lambda s=s: one(s) for s in blk], not args.no_graph)
        # the kernel time: the same block again, an event pair around each step
        evs = [_events(2) for _ in range(block)]
        for s, ev in zip(blk, evs):
            ev[0].record()
            one(s)
            ev[1].record()
        torch.cuda.synchronize()
        kernel_ms += [e[0].elapsed_time(e[1]) for e in evs]
        done += block
        del blk
    per = total_ms / done
    kms = sum(kernel_ms) / len(kernel_ms)
    bytes_step = decode_bytes_per_step(Bt, D)
    res = {"value": 1e3 / per * world, "unit": "steps/s", "ms_per_step": per, "steps": done,
           "roofline": {"kernel": "decode_bulk_kernel", "bound": "hbm", "unit": "GB/s",
                        "achieved": round(bytes_step / (kms * 1e-3) / 1e9, 1),
                        "peak": peaks["hbm_gbs"], "peak_source": peaks["source"],
                        "frac": round(bytes_step / (kms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                        "kernel_ms": round(kms, 5), "algorithmic_bytes_per_launch": bytes_step,
                        "traffic": recorded_traffic("decode_bulk_kernel", DECODE,
                                                    source_sha("decode.cu", "common.cuh",
                                                               "tma.cuh"))},
           "step": "ssm_selective_state_update, 256 rows x 8192 channels, fresh inputs per "
                   "step; blocks of 100 steps replayed as CUDA graphs"}
    if not args.no_e2e:
        one = synth.device_activations(6000, Bt, D)
        host_in = {k: v.cpu().pin_memory() for k, v in one.items()}
        ys = [(yd,), (torch.empty_like(yd),)]
        yh = [(torch.empty(yd.shape, dtype=yd.dtype).pin_memory(),) for _ in range(2)]
        csx, hx = cs0.clone(), h0.clone()

        def compute(i, dev, b):
            ssm.ssm_selective_state_update(csx, hx, dev["x"], dev["dt"], dev["B"], dev["C"],
                                           ys[b][0], ly.w, ly.A, z=dev["z"], conv_b=ly.b,
                                           Dskip=ly.Dskip, dt_bias=ly.dt_bias)

        ems = _pipelined_e2e(compute, host_in, None, ys, yh, world, 200)
        res["e2e"] = {"value": 1e3 / ems * world, "unit": "steps/s", "ms_per_step": ems,
                      "h2d_bytes_per_step": sum(v.numel() * v.element_size()
                                                for v in host_in.values()),
                      "d2h_bytes_per_step": yd.numel() * yd.element_size(),
                      "how": "per step: x, dt, z, B, C copied in from pinned host memory, y "
                             "copied out; states stay on the device; pipelined"}
        del csx, hx
    for W in args.replay_windows:
        if args.replay_copy != "none":
            res[f"replay_w{W}"] = bench_replay(peaks, world, ly, cs0, h0, W, steps, mufu,
                                               not args.no_graph)
        if args.replay_copy != "bf16":
            res[f"replay_w{W}_fp32_ckpt"] = bench_replay(peaks, world, ly, cs0, h0, W, steps, mufu,
                                                         not args.no_graph, keep_lo=False)
    del cs, h, cs0, h0
    torch.cuda.empty_cache()
    return res


def bench_scan_bwd(world, ly, a, cu, S, mufu, peaks, label="packed 65536 x 5120", n=5):
    """Backward of the selective scan on a prefill's inputs (bf16 activations,
    upstream gradient dy drawn like x). Algorithmic work per (token, channel):
    2 x 16 exponentials (the decays of one forward pass to produce the states
    and of the reverse pass; the kernels execute 3 x 16, recomputing the
    states chunk by chunk from checkpoints instead of storing them) and 14
    bytes (u, dt, z, dy in; du, ddelta, dz out)."""
    import torch

    import selective_state_space_causal_b200 as ssm

    synth = load_synth()
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

    for _ in range(2):
        call()
    s0, s1 = _events(2)
    _barrier_sync(world)
    s0.record()
    for _ in range(n):
        call()
    s1.record()
    _barrier_sync(world)
    ms = _max_over_ranks(s0.elapsed_time(s1) / n, world)
    units = tok * D
    res = {"value": units * world / (ms * 1e-3) / 1e9, "unit": UNIT, "ms_per_call": ms,
           "mufu_frac": round(units * 2 * N_STATE / (ms * 1e-3) / 1e9 / mufu["gexp_per_s"], 4),
           "executed_exp_frac": round(units * 3 * N_STATE / (ms * 1e-3) / 1e9
                                      / mufu["gexp_per_s"], 4),
           "hbm_frac": round(units * 14 / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
           "variant": ssm.ssm_scan_bwd_variant_for(S, D), "sequences": S,
           "step": f"ssm_selective_scan_bwd over the {label} prefill, all gradients"}

    # the training pair: the forward leaves its checkpoints in the workspace,
    # the backward reads them instead of running its own forward pass
    y = torch.empty_like(a["x"])
    fws = torch.empty(max(1, ssm.ssm_scan_workspace_size(tok, D, N_STATE, S)),
                      dtype=torch.uint8, device="cuda")
    fkw = dict(Dskip=ly.Dskip, z=a["z"], dt_bias=ly.dt_bias, cu_seqlens=cu, S=S, workspace=fws)

    def fwd():
        ssm.ssm_selective_scan_fwd(a["x"], a["dt"], ly.A, a["B"], a["C"], y, **fkw)

    def fwd_ck():
        ssm.ssm_selective_scan_fwd_ckpt(a["x"], a["dt"], ly.A, a["B"], a["C"], y, ws, **fkw)

    def bwd_ck():
        ssm.ssm_selective_scan_bwd(a["x"], a["dt"], ly.A, a["B"], a["C"], dy, g, Dskip=ly.Dskip,
                                   z=a["z"], dt_bias=ly.dt_bias, cu_seqlens=cu, S=S,
                                   workspace=ws, from_fwd_ckpt=True)

    def timed(fns):
        for _ in range(2):
            for f in fns:
                f()
        evs = [_events(len(fns) + 1) for _ in range(n)]
        _barrier_sync(world)
        for i in range(n):
            evs[i][0].record()
            for j, f in enumerate(fns):
                f()
                evs[i][j + 1].record()
        _barrier_sync(world)
        return [_max_over_ranks(sum(e[j].elapsed_time(e[j + 1]) for e in evs) / n, world)
                for j in range(len(fns))]

    f_ms, fck_ms, bck_ms = timed([fwd, fwd_ck, bwd_ck])
    res["from_forward_checkpoints"] = {
        "bwd_ms": round(bck_ms, 4), "fwd_ckpt_ms": round(fck_ms, 4), "fwd_ms": round(f_ms, 4),
        "value": units * world / (bck_ms * 1e-3) / 1e9, "unit": UNIT,
        "mufu_frac": round(units * N_STATE / (bck_ms * 1e-3) / 1e9 / mufu["gexp_per_s"], 4),
        "train_pair_ms": round(fck_ms + bck_ms, 4), "separate_pair_ms": round(f_ms + ms, 4),
        "step": "ssm_selective_scan_fwd_ckpt (the forward writes the state before every 8th "
                "token) then ssm_selective_scan_bwd_ckpt (no checkpointing pass); mufu_frac "
                "counts the 16 exponentials per (token, channel) the backward needs once the "
                "forward states are given"}
    del g, ws, dy, y, fws
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


def bench_replay(peaks, world, ly, cs, h, W, steps, mufu, use_graph=True, keep_lo=True):
    """Batch-256 decode through the replay kernels (checkpoint + input buffer,
    with or without the bf16 checkpoint copy), on the same prefill states and
    the same kind of fresh per-step inputs as the eager decode measurement."""
    import torch

    import selective_state_space_causal_b200 as ssm

    synth = load_synth()
    Bt, D = h.shape[0], h.shape[1]
    rep = ssm.replay_buffers(Bt, D, W, "cuda", keep_lo=keep_lo)
    rep["ckpt"].copy_(h)
    csr = cs.clone()
    ssm.ssm_replay_reset(rep)
    yd = torch.empty((Bt, D), dtype=torch.bfloat16, device="cuda")
    block = 100
    total_ms = 0.0
    done = 0
    l0 = ssm.ssm_launch_count()

    def one(s):
        ssm.ssm_replay_state_update(csr, rep, s["x"], s["dt"], s["B"], s["C"], yd, ly.w, ly.A,
                                    z=s["z"], conv_b=ly.b, Dskip=ly.Dskip, dt_bias=ly.dt_bias)

    for b0 in range(0, steps, block):
        blk = [synth.device_activations(5000 + b0 + i, Bt, D) for i in range(block)]
        total_ms += _time_block(world, [lambda s=s: one(s) for s in blk], use_graph)
        done += block
        del blk
    launches = ssm.ssm_launch_count() - l0
    per = total_ms / done
    bytes_step = replay_bytes_per_step(Bt, D, W, keep_lo)
    exps_step = Bt * D * N_STATE * (W + 1) / 2
    res = {
        "value": 1e3 / per * world, "unit": "steps/s", "ms_per_step": per, "steps": done,
        "window": W, "algorithmic_bytes_per_step": int(bytes_step),
        "hbm_frac": round(bytes_step / (per * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
        "mufu_frac": round(exps_step / (per * 1e-3) / 1e9 / mufu["gexp_per_s"], 4),
        "gpu_launches_per_step": launches / done,
        "step": f"ssm_replay_state_update (checkpoint every {W} tokens, "
                f"{'bf16 copy' if keep_lo else 'the fp32 checkpoint'} for outputs), "
                "256 rows x 8192 channels, fresh inputs per step; blocks of 100 steps "
                "replayed as CUDA graphs"}
    del rep, csr
    return res


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------

def oracle_longctx(orc, n_ch, seed=0):
    """A callable running the oracle on `n_ch` seeded channels of the headline
    step (all 131072 tokens: conv and scan with the states carried, then the
    decode token) and the (token, channel) units it covers. The oracle keeps
    the state in registers across the whole sequence, which is what the 16
    chunked calls with carried states compute."""
    import numpy as np

    synth = load_synth()
    w = synth.WORKLOADS[HEADLINE]
    L, D = w["seqlen"], w["D"]
    prm = synth.make_params(seed, D)
    rng = np.random.default_rng(seed)
    ch = np.sort(rng.choice(D, n_ch, replace=False))
    act = synth.make_activations(seed, L, n_ch, bf16=True)
    dec = synth.make_activations(seed + 1, 1, n_ch, bf16=True)
    cw, cb, A, Dk, dtb = (prm.conv_w[ch], prm.conv_b[ch], prm.A[ch], prm.Dskip[ch],
                          prm.dt_bias[ch])

    def run():
        xc, cs = orc.causal_conv1d(act["x"], cw, cb, S=1, want_state=True)
        _, h = orc.selective_scan(xc, act["dt"], A, act["B"], act["C"], Dskip=Dk, z=act["z"],
                                  dt_bias=dtb, S=1, want_state=True)
        orc.state_update(cs, h, dec["x"], dec["dt"], dec["B"], dec["C"], dec["z"], cw, cb, A, Dk,
                         dtb)

    return run, L * n_ch


def _time_oracle(run, min_s=2.0):
    run()
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        if time.perf_counter() - t0 > min_s:
            break
    return (time.perf_counter() - t0) / reps, reps


def cpu_baseline(n_ch=ORACLE_CHANNELS):
    """The fp64 oracle on the host cores, on a seeded channel sample of the
    headline workload; the rate on the sample is the rate on the whole
    workload (channels are independent), and the whole step's time is the
    sample's scaled by D / n_ch (extrapolated, not measured)."""
    import oracle

    orc = oracle.load()
    run, units = oracle_longctx(orc, n_ch)
    cores = orc.num_threads()
    dt, reps = _time_oracle(run)
    orc.set_num_threads(1)
    run1, units1 = oracle_longctx(orc, 32)
    dt1, _ = _time_oracle(run1, 1.0)
    orc.set_num_threads(cores)
    D = load_synth().WORKLOADS[HEADLINE]["D"]
    return {"value": units / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{HEADLINE}: all 131072 tokens (conv, scan, decode token) of {n_ch} "
                      f"seeded channels of {D}, fp64, {reps} repetitions on {cores} threads",
            "extrapolated_step_s": round(dt * D / n_ch, 3),
            "extrapolated_note": f"the whole step's time, scaled from the sample by {D}/{n_ch} "
                                 "(extrapolated, not measured)",
            "one_thread": {"value": units1 / dt1 / 1e9, "unit": UNIT, "cores": 1,
                           "sample": "the same on 32 channels, one thread"}}


def bench_reference(args):
    """The reference arm: the fp64 oracle as it stands, on the host cores, on a
    bounded channel sample of the headline workload per step."""
    rank, _, world = dist_info()
    if rank != 0:
        return 0
    import oracle

    orc = oracle.load()
    n_ch = 16
    run, units = oracle_longctx(orc, n_ch)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t0
    ms = el / args.steps * 1e3
    value = units / (el / args.steps) / 1e9
    sample = (f"{HEADLINE}: all 131072 tokens of {n_ch} of 8192 channels per step "
              "(conv, scan and the decode token), fp64 oracle on the host cores")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": HEADLINE, "batch": 1, "seq_len": 131072,
                                            "chunk": 8192, "d_inner": 8192, "d_state": 16,
                                            "d_conv": 4, "channels_sampled": n_ch},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# sweeps and profiler cases
# ---------------------------------------------------------------------------

SWEEP_VARIANTS = [(0, 0), (4, 10), (4, 11), (4, 9), (8, 9), (16, 12), (2, 9), (2, 8), (4, 1), (8, 2)]


def scan_sweep(variants, peaks):
    """Scan alone per variant on the prefill shapes; one JSON line each."""
    import torch

    import selective_state_space_causal_b200 as ssm

    synth = load_synth()
    mufu = mufu_peak_gexp(peaks["sm_max_mhz"])
    lens = synth.sample_lengths(0, 65536)
    shapes = [(LAYER, 16384, 1536, None, 8),
              (PACKED, 65536, 5120, synth.cu_from_lengths(lens), len(lens)),
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


def profile_scan(kind):
    """Three untimed calls of one kernel's workload, for ncu captures (a few GB
    on the device at most)."""
    import torch

    import selective_state_space_causal_b200 as ssm

    synth = load_synth()
    bf = torch.bfloat16
    if kind == "decode_fresh":
        Bt, D = 256, 8192
        ly = Layer(D)
        g = torch.Generator(device="cuda")
        g.manual_seed(3)
        h = 0.3 * torch.randn((Bt, D, N_STATE), device="cuda", generator=g)
        cs = torch.randn((Bt, D, 3), device="cuda", generator=g).to(bf)
        y = torch.empty((Bt, D), dtype=bf, device="cuda")
        ins = [synth.device_activations(20 + i, Bt, D) for i in range(3)]
        for s in ins:
            ssm.ssm_selective_state_update(cs, h, s["x"], s["dt"], s["B"], s["C"], y, ly.w, ly.A,
                                           z=s["z"], conv_b=ly.b, Dskip=ly.Dskip,
                                           dt_bias=ly.dt_bias)
        torch.cuda.synchronize()
        assert ssm.ssm_device_status() == 0
        print(json.dumps({"profile_scan": kind}))
        return
    if kind == "layer":
        tok, D, cu, S = 16384, 1536, None, 8
    elif kind in ("long", "conv_long"):
        tok, D, cu, S = 8192, 8192, None, 1
    else:  # a 16384-token slice of the packed workload's length mix, in the
        # variant the library picks for the whole packed workload
        lens = synth.sample_lengths(0, 16384)
        tok, D, cu, S = 16384, 5120, synth.cu_from_lengths(lens), len(lens)
        w = synth.WORKLOADS[PACKED]
        full = len(synth.sample_lengths(0, w["total"], w["len_lo"], w["len_hi"]))
        ssm.ssm_set_scan_variant(*ssm.ssm_scan_variant_for(full, D))
    ly = Layer(D)
    cu_d = torch.from_numpy(cu).cuda() if cu is not None else None
    a = synth.device_activations(0, tok, D)
    y = torch.empty((tok, D), dtype=bf, device="cuda")
    h = torch.zeros((S, D, N_STATE), device="cuda")
    cs = torch.zeros((S, D, 3), dtype=bf, device="cuda")
    ws = torch.empty(max(1, ssm.ssm_scan_workspace_size(tok, D, N_STATE, S)), dtype=torch.uint8,
                     device="cuda")
    for _ in range(3):
        if kind == "conv_long":
            ssm.ssm_causal_conv1d(a["x"], y, ly.w, bias=ly.b, conv_state_in=cs,
                                  conv_state_out=cs)
        elif kind == "packed_fused":
            ssm.ssm_conv_scan_fwd(a["x"], ly.w, a["dt"], ly.A, a["B"], a["C"], y, conv_b=ly.b,
                                  conv_state_in=cs, conv_state_out=cs, Dskip=ly.Dskip, z=a["z"],
                                  dt_bias=ly.dt_bias, h0=h, h_final=h, cu_seqlens=cu_d, S=S)
        else:
            ssm.ssm_selective_scan_fwd(a["x"], a["dt"], ly.A, a["B"], a["C"], y, Dskip=ly.Dskip,
                                       z=a["z"], dt_bias=ly.dt_bias, h0=h, h_final=h,
                                       cu_seqlens=cu_d, S=S,
                                       workspace=ws if cu_d is not None else None)
    torch.cuda.synchronize()
    assert ssm.ssm_device_status() == 0
    print(json.dumps({"profile_scan": kind, "tokens": tok, "d_inner": D, "sequences": S,
                      "variant": ssm.ssm_scan_variant_for(S, D)}))


def profile_scan_bwd(shape="packed"):
    """Three backward scans, for profiler captures: on a quarter of the packed
    workload, or on the Mamba-130M layer shape (8 dense rows)."""
    import torch

    import selective_state_space_causal_b200 as ssm

    synth = load_synth()
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

    synth = load_synth()
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
        return 0
    if args.profile_scan_bwd:
        profile_scan_bwd(args.profile_scan_bwd)
        return 0
    if args.profile_scan:
        profile_scan(args.profile_scan)
        return 0
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
    mufu = measure_mufu_peak(local)
    res = bench_headline(args, world, peaks, local, mufu)
    workloads = None
    if not args.no_secondary:
        workloads = {LAYER: bench_layer(args, world, peaks, mufu),
                     PACKED: bench_packed(args, world, peaks, mufu),
                     DECODE: bench_decode(args, world, peaks, mufu)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()
    if rank == 0:
        line = {
            "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "io_dtype": "bf16", "data": "synthetic",
            "config": {"workload": HEADLINE, "batch": 1, "seq_len": 131072, "chunk": 8192,
                       "d_inner": 8192, "d_state": 16, "d_conv": 4,
                       "step": "16 x (causal_conv1d+silu -> selective_scan) over 8192-token "
                               "chunks, h carried in place and the conv state between two "
                               "buffers, chunk j+1's conv on a second stream beside chunk j's "
                               "scan, then 1 decode step; replayed as one CUDA graph",
                       "l2": "inputs (6.4 GB) far larger than L2; no rotation needed",
                       "parallelism": f"replicas x{world}"},
            "roofline": res["roofline"], "mufu_peak": mufu, "clocks": res["clocks"],
            "e2e": res.get("e2e"), "gpu_launches": res["gpu_launches"],
            "launches_per_step": res["launches_per_step"], "conv_roofline": res["conv_roofline"],
            "scan_ms_per_step": res["scan_ms_per_step"], "cuda_graph": res["cuda_graph"],
            "step_ms_without_graph": res["step_ms_without_graph"],
            "cpu_baseline": cpu, "workloads": workloads,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
