#!/usr/bin/env python
"""Benchmark of the Gated DeltaNet core on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl gdn|reference]

One step = one pass of the whole prefill path over one batch: the chunked prefill
with the gate prologue fused in (gdn_chunk_prefill_gated: raw a, b -> gates ->
chunked gated delta rule) over the long-context workload B=1, T=32768, 16 q/k
heads, 32 value heads, d=128, bf16, BT=64 (synthetic, seeded).  The JSON line's ``value`` is prefill tokens/s over all
ranks.  The decode step (B=64, H=32, d=128, fp32 state, 1024 consecutive steps)
is measured in the same run and reported under ``decode`` with its HBM roofline.

Under torchrun every rank runs its own independent replica of the workload (the
path needs no exchange between GPUs); the step time is the max over ranks.

``--impl reference`` times the CPU fp64 oracle instead, on the host cores, on a
bounded prefix of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDN prefill tokens/s @32K,H32,d128; decode-step HBM GB/s vs peak"
PREFILL = dict(B=1, T=32768, HK=16, HV=32, D=128, BT=64)
DECODE = dict(B=64, H=32, D=128, steps=1024)
E2E_PIECE = 4096   # tokens per piece of the host-buffer pipeline (8 pieces at T = 32768)
WORKLOAD = "long prefill: B=1 T=32768 HK=16 HV=32 Dk=Dv=128 bf16 BT=64, fp32 state, zero initial state"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


class RankOps:
    """The cross-rank steps of a run: a barrier and the max over ranks of a time.  With
    ``dist`` None (one process) both are local.  With a process group they are
    collectives (NCCL between GPUs; gloo in the CPU tests), and every rank takes them in
    the same order.  No data of the path itself crosses ranks: each rank runs an
    independent replica of the workload (seed ``replica_seed``)."""

    def __init__(self, dist=None, device=None):
        self.dist = dist
        self.device = device

    def _sync(self):
        if self.device is not None and getattr(self.device, "type", "cpu") == "cuda":
            import torch
            torch.cuda.synchronize()

    def barrier(self):
        self._sync()
        if self.dist is not None:
            self.dist.barrier()
        self._sync()

    def max(self, x: float) -> float:
        if self.dist is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())


def replica_seed(base: int, rank: int) -> int:
    """Seed of rank ``rank``'s replica of a workload whose single-GPU seed is ``base``."""
    return base + 1000 * rank


def whole_job_rate(world: int, units_per_rank: int, ms_max: float) -> float:
    """Units per second over all ranks, timed by the slowest rank."""
    return world * units_per_rank / (ms_max * 1e-3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def prefill_flops_per_token(HK, HV, D, C):
    """Contraction FLOPs of the chunked form per token (a formula, not a count of
    what a kernel executes): per value head 6 C d (W, U, P Delta) + 6 d^2
    (W H, Q H, K^T Delta) + C^2 / 3 (triangular solve); per q/k head 4 C d
    (K K^T and Q K^T)."""
    return HV * (6 * C * D + 6 * D * D + C * C / 3.0) + HK * (4 * C * D)


def prefill_bytes_per_token(HK, HV, D, io_bytes=2):
    """Algorithmic HBM bytes per token: read q, k, v, g, beta; write o."""
    return 2 * HK * D * io_bytes + HV * D * io_bytes + 2 * HV * 4 + HV * D * io_bytes


def decode_bytes_per_step(B, HK, HV, Dk, Dv, io_bytes=2):
    """State read + write (fp32), q, k, v read, o written, g and beta read."""
    return (2 * B * HV * Dk * Dv * 4 + 2 * B * HK * Dk * io_bytes + 2 * B * HV * Dv * io_bytes
            + 2 * B * HV * 4)


# ---------------------------------------------------------------------------
class Clocks:
    """SM clock, power and clock-event (throttle) reasons sampled every 2 ms through NVML
    from a background thread; only samples inside the timed regions (host wall-clock
    windows added with ``window``) are summarised.  Reads settings only."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80))

    def __init__(self, device_index: int):
        self.dev = device_index
        self.windows = []
        self.samples = []
        self.thread = None
        self.stop_flag = False
        self.err = None

    def window(self, t0: float, t1: float):
        self.windows.append((t0, t1))

    def _handle(self, nv):
        try:
            import torch
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
        except Exception as e:  # pragma: no cover
            self.err = f"NVML unavailable: {e}"
            return

        def loop():
            while not self.stop_flag:
                try:
                    self.samples.append((time.time(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                         int(get_reasons(h)), nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except Exception as e:  # pragma: no cover
                    self.err = str(e)
                    return
                time.sleep(0.002)

        self.nv = nv
        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "not sampled"]}
        self.stop_flag = True
        self.thread.join(2)
        inside = [x for x in self.samples if any(a <= x[0] <= b for a, b in self.windows)]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.smax, "samples": 0,
                    "reasons": ["no samples inside the timed regions"]}
        reasons = set()
        for _, _, bits, _ in inside:
            for name, attr, default in self.REASONS:
                if bits & getattr(self.nv, attr, default):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": self.smax,
                "reasons": sorted(reasons), "samples": len(inside),
                "power_w_max": max(x[3] for x in inside), "sampled": "NVML every 2 ms, timed regions only"}


# ---------------------------------------------------------------------------
def cpu_oracle_sample(target_s: float, T_max: int):
    """Time the oracle (gates + recurrence, fp64, all host cores) on a prefix of
    the long workload sized to about ``target_s`` seconds.  Returns
    (tokens/s, tokens, seconds, threads)."""
    import numpy as np
    import oracle
    from gated_deltanet_sequence_delta_b200 import inputs as I
    probe_T = 64
    inp = I.make_prefill(1, probe_T, PREFILL["HK"], PREFILL["HV"], PREFILL["D"], PREFILL["D"],
                         io_dtype=I.BF16, seed=2)

    def run(inp):
        q, k, v = inp.q.f64(), inp.k.f64(), inp.v.f64()
        t0 = time.perf_counter()
        g, beta = oracle.gates(inp.a.astype(np.float64), inp.b.astype(np.float64),
                               inp.A_log.astype(np.float64), inp.dt_bias.astype(np.float64))
        oracle.recurrence(q, k, v, g, beta, scale=1.0, l2norm=True)
        return time.perf_counter() - t0

    run(inp)
    t = run(inp)
    T_s = int(min(T_max, max(probe_T, probe_T * target_s / max(t, 1e-6))))
    T_s = max(64, (T_s // 64) * 64)
    inp = I.make_prefill(1, T_s, PREFILL["HK"], PREFILL["HV"], PREFILL["D"], PREFILL["D"],
                         io_dtype=I.BF16, seed=2)
    t = run(inp)
    return T_s / t, T_s, t, oracle.max_threads()


def run_reference(args, rank, world):
    if rank != 0:
        return
    # size each step so that warmup + steps stay within about two minutes
    per_step = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_sample(per_step, PREFILL["T"])
    vals, toks, secs = [], [], []
    threads = None
    for _ in range(args.steps):
        v, T_s, t, threads = cpu_oracle_sample(per_step, PREFILL["T"])
        vals.append(v)
        toks.append(T_s)
        secs.append(t)
    value = sum(toks) / sum(secs)
    sample = (f"first {toks[0]} tokens of the T=32768 workload per step (all 32 value heads), "
              f"gates + fp64 recurrence")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(secs) / len(secs),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_step": toks[0], "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def run_gdn(args, rank, world, dist):
    import numpy as np
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    from gated_deltanet_sequence_delta_b200 import binding
    from gated_deltanet_sequence_delta_b200 import inputs as I

    binding.lib()  # fails loudly if the CUDA library is not built
    dev = torch.device("cuda", torch.cuda.current_device())
    P, pk = peaks()

    def dev_t(t):
        if isinstance(t, I.Tensor):
            if t.dtype == I.BF16:
                return torch.from_numpy(t.data.view(np.int16)).view(torch.bfloat16).to(dev)
            return torch.from_numpy(t.data).to(dev)
        return torch.from_numpy(np.ascontiguousarray(t)).to(dev)

    def pinned(t):
        if isinstance(t, I.Tensor):
            if t.dtype == I.BF16:
                return torch.from_numpy(t.data.view(np.int16)).view(torch.bfloat16).pin_memory()
            return torch.from_numpy(t.data).pin_memory()
        return torch.from_numpy(np.ascontiguousarray(t)).pin_memory()

    ops = RankOps(dist, dev)
    barrier, max_over_ranks = ops.barrier, ops.max

    T, HK, HV, D, BT = PREFILL["T"], PREFILL["HK"], PREFILL["HV"], PREFILL["D"], PREFILL["BT"]
    do_prefill = args.only in ("all", "prefill")
    do_decode = args.only in ("all", "decode")
    clocks = Clocks(torch.cuda.current_device())
    line = {"metric": METRIC, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic"}
    if do_prefill:
        clocks.start()
        line.update(bench_prefill(args, rank, world, dev, P, pk, dev_t, pinned, barrier, max_over_ranks,
                                  clocks))
    if do_decode:
        if not do_prefill:
            clocks.start()
        line["decode"] = bench_decode(args, rank, world, dev, P, pk, dev_t, barrier, max_over_ranks, clocks)
    line["clocks"] = clocks.stop()
    if do_prefill and rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, T_s, t, th = cpu_oracle_sample(args.cpu_seconds, T)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": th, "kind": "oracle",
                                "sample": f"first {T_s} tokens of the workload, all 32 value heads, "
                                          f"gates + fp64 recurrence, {t:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def _traffic():
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(prof):
        return json.load(open(prof))
    return {}


def bench_prefill(args, rank, world, dev, P, pk, dev_t, pinned, barrier, max_over_ranks, clocks):
    import numpy as np
    import statistics
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    from gated_deltanet_sequence_delta_b200 import inputs as I
    T, HK, HV, D, BT = PREFILL["T"], PREFILL["HK"], PREFILL["HV"], PREFILL["D"], PREFILL["BT"]
    inp = I.make_prefill(1, T, HK, HV, D, D, io_dtype=I.BF16, seed=replica_seed(2, rank), BT=BT, name="long")
    q, k, v = dev_t(inp.q), dev_t(inp.k), dev_t(inp.v)
    a, b = dev_t(inp.a), dev_t(inp.b)
    A_log, dt_bias = dev_t(inp.A_log), dev_t(inp.dt_bias)
    g = torch.empty((1, T, HV), dtype=torch.float32, device=dev)
    beta = torch.empty_like(g)
    o = torch.empty((1, T, HV, D), dtype=torch.bfloat16, device=dev)
    hT = torch.empty((1, HV, D, D), dtype=torch.float32, device=dev)
    ws = torch.empty(G.prefill_workspace_bytes(T, 1, HK, HV, D, D, BT, 1), dtype=torch.uint8, device=dev)

    G.gdn_gates(a, b, A_log, dt_bias, g=g, beta=beta)   # for the output-epilogue leg below

    def prefill_step(evs=None):
        if evs is not None:
            evs[0].record()
        G.gdn_chunk_prefill_gated(q, k, v, a, b, A_log, dt_bias, BT=BT, o=o, final_state=hT, workspace=ws)
        if evs is not None:
            evs[1].record()

    for _ in range(max(3, args.warmup)):
        prefill_step()
    barrier()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    n0 = G.kernel_launches()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    t0.record()
    for i in range(args.steps):
        prefill_step(kev[i])
    t1.record()
    barrier()
    clocks.window(w0, time.time())
    launches = G.kernel_launches() - n0
    ms_local = t0.elapsed_time(t1) / args.steps
    kernel_ms_local = statistics.mean(e0.elapsed_time(e1) for e0, e1 in kev)
    ms = max_over_ranks(ms_local)
    kernel_ms = max_over_ranks(kernel_ms_local)

    # ---------------- e2e through host buffers ----------------
    # gdn_chunk_prefill_host: host q, k, v, a, b (and the two per-head gate parameters) in,
    # host o and final state out; the library streams the sequence through the GPU in
    # pieces so that the copies in both directions overlap the kernels.
    hq, hk_, hv = pinned(inp.q), pinned(inp.k), pinned(inp.v)
    ha, hb = pinned(inp.a).view(1, T, HV), pinned(inp.b).view(1, T, HV)
    hAl, hdtb = pinned(inp.A_log), pinned(inp.dt_bias)
    ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    hh = torch.empty(hT.shape, dtype=hT.dtype).pin_memory()
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk_, hv, ha, hb, hAl, hdtb))
    d2h = ho.numel() * ho.element_size() + hh.numel() * hh.element_size()
    hws = torch.empty(G.prefill_host_workspace_bytes(1, T, HK, HV, D, D, BT, 1, 0, E2E_PIECE),
                      dtype=torch.uint8, device=dev)

    def e2e_step():
        G.gdn_chunk_prefill_host(hq, hk_, hv, ha, hb, hAl, hdtb, BT=BT, piece_tokens=E2E_PIECE, o=ho,
                                 final_state=hh, workspace=hws)

    for _ in range(2):
        e2e_step()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = max(1, min(args.steps, 5))
    e0.record()
    for _ in range(e2e_steps):
        e2e_step()
    e1.record()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    del hq, hk_, hv, ha, hb, hAl, hdtb, ho, hh, hws

    # ---------------- the same prefill with the output epilogue fused ----------------
    # out = o rsqrt(mean(o^2) + eps) (1 + w) sigmoid(z) per (token, value head), inside the
    # state-carry kernel (gdn_chunk_prefill_outgate); reported beside the core path
    z, w = I.outgate_inputs(T, HV, D, I.BF16, replica_seed(87, rank))
    zd, wd = dev_t(z).view(1, T, HV, D), dev_t(w)

    def gated_step():
        G.gdn_chunk_prefill_outgate(q, k, v, g, beta, zd, wd, 1e-6, BT=BT, o=o, final_state=hT, workspace=ws)

    for _ in range(3):
        gated_step()
    barrier()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record()
    for _ in range(args.steps):
        gated_step()
    g1.record()
    barrier()
    gated_ms = max_over_ranks(g0.elapsed_time(g1) / args.steps)
    del zd, wd

    # ---------------- the convolution prologue: raw q | k | v projections -> q, k, v ----------------
    C = 2 * HK * D + HV * D
    xr, cw, cst = I.conv_prefill_inputs(T, 1, HK, HV, D, I.BF16, replica_seed(88, rank), True)
    xd, cwd = dev_t(xr).view(1, T, C), dev_t(cw)
    csd = dev_t(np.ascontiguousarray(cst.transpose(0, 2, 1)))
    cq, ck, cv, cso = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(csd)
    del xr

    def conv_step():
        G.gdn_conv_prefill(xd, cwd, HK, HV, D, D, conv_state_in=csd, conv_act=1, q=cq, k=ck, v=cv,
                           conv_state_out=cso)

    for _ in range(3):
        conv_step()
    barrier()
    c0 = torch.cuda.Event(enable_timing=True)
    c1 = torch.cuda.Event(enable_timing=True)
    c0.record()
    for _ in range(args.steps):
        conv_step()
    c1.record()
    barrier()
    conv_ms = max_over_ranks(c0.elapsed_time(c1) / args.steps)
    conv_bytes = 2 * T * C * 2 + C * 16 + 2 * 3 * C * 4   # x in, q | k | v out, weights, states
    del xd, cwd, csd, cq, ck, cv, cso
    flops = prefill_flops_per_token(HK, HV, D, BT) * T
    pbytes = prefill_bytes_per_token(HK, HV, D) * T + HV * D * D * 4
    tflops = flops / (kernel_ms * 1e-3) / 1e12
    peak_tf = P["bf16_tflops"]
    return {
        "value": whole_job_rate(world, T, ms), "ms_per_step": ms,
        "config": {"workload": WORKLOAD, "tokens_per_step_per_gpu": T,
                   "l2": "no flush: each step reads/writes ~0.8 GB, over 6x the 126 MB L2",
                   "parallelism": f"replicas x{world} (independent problems, no collective)"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": tflops / peak_tf, "traffic": _traffic().get("prefill_bytes_per_launch"),
                     "peak_kind": f"{pk} bf16 dense (burst)",
                     "flops_per_launch": flops, "kernel_ms": kernel_ms,
                     "hbm_view": {"achieved_gbs": pbytes / (kernel_ms * 1e-3) / 1e9,
                                  "peak_gbs": P["hbm_gbs"],
                                  "frac": pbytes / (kernel_ms * 1e-3) / 1e9 / P["hbm_gbs"],
                                  "bytes_per_launch": pbytes}},
        "e2e": {"value": whole_job_rate(world, T, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": f"gdn_chunk_prefill_host, pinned host buffers, {E2E_PIECE}-token pieces"},
        "gpu_launches": launches,
        "gated_output": {"what": "gdn_chunk_prefill_outgate: the same prefill with the gated RMSNorm output "
                                 "epilogue (eps 1e-6) fused into the state carry; gates precomputed",
                         "ms_per_call": gated_ms, "tokens_per_s": whole_job_rate(world, T, gated_ms),
                         "core_prefill_ms_per_call": kernel_ms},
        "conv_prologue": {"what": "gdn_conv_prefill: kernel-4 causal convolution (SiLU) from the raw q|k|v "
                                  "projections [T, 8192] bf16 to the prefill's q, k, v, state carried in and out",
                          "ms_per_call": conv_ms, "bytes_per_call": conv_bytes,
                          "achieved_gbs": conv_bytes / (conv_ms * 1e-3) / 1e9,
                          "frac": conv_bytes / (conv_ms * 1e-3) / 1e9 / P["hbm_gbs"],
                          "traffic": _traffic().get("conv_prefill_bytes_per_launch"),
                          "peak_kind": f"{pk} copy bandwidth"},
    }


def bench_decode(args, rank, world, dev, P, pk, dev_t, barrier, max_over_ranks, clocks):
    import numpy as np
    import torch
    import gated_deltanet_sequence_delta_b200 as G
    from gated_deltanet_sequence_delta_b200 import inputs as I
    ds = I.decode(B=DECODE["B"], H=DECODE["H"], D=DECODE["D"], seed=replica_seed(1, rank))
    ring = []
    for s in range(8):
        dq, dk, dv, da, db = ds.step(s)
        ring.append((dev_t(dq), dev_t(dk), dev_t(dv), dev_t(da), dev_t(db)))
    state = dev_t(ds.state0)
    dA, dbias = dev_t(ds.A_log), dev_t(ds.dt_bias)
    dg = torch.empty((ds.B, ds.HV), dtype=torch.float32, device=dev)
    dbeta = torch.empty_like(dg)
    do = torch.empty((ds.B, ds.HV, ds.Dv), dtype=torch.bfloat16, device=dev)

    def decode_step(i):
        dq, dk, dv, da, db = ring[i % len(ring)]
        G.gdn_gates(da, db, dA, dbias, g=dg, beta=dbeta)
        G.gdn_decode_step(dq, dk, dv, dg, dbeta, state, o=do)

    for i in range(5):
        decode_step(i)
    barrier()
    n_dec = args.decode_steps
    d0 = torch.cuda.Event(enable_timing=True)
    d1 = torch.cuda.Event(enable_timing=True)
    nd0 = G.kernel_launches()
    w0 = time.time()
    d0.record()
    for i in range(n_dec):
        decode_step(i)
    d1.record()
    barrier()
    clocks.window(w0, time.time())
    dec_launches = G.kernel_launches() - nd0
    dec_ms = max_over_ranks(d0.elapsed_time(d1) / n_dec)
    # the decode kernel alone, same inputs, back to back
    dq, dk, dv, _, _ = ring[0]
    k0 = torch.cuda.Event(enable_timing=True)
    k1 = torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    k0.record()
    torch.cuda.nvtx.range_push("decode_b64")   # (lets a profiler pick a launch from the middle of this run)
    for i in range(n_dec):
        G.gdn_decode_step(dq, dk, dv, dg, dbeta, state, o=do)
    torch.cuda.nvtx.range_pop()
    k1.record()
    barrier()
    clocks.window(w0, time.time())
    dec_kernel_ms = max_over_ranks(k0.elapsed_time(k1) / n_dec)
    # the step with the gates formed inside the kernel (one launch per step)
    nf0 = G.kernel_launches()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    f0.record()
    for i in range(n_dec):
        dq, dk, dv, da, db = ring[i % len(ring)]
        G.gdn_decode_step_gated(dq, dk, dv, da, db, dA, dbias, state, o=do)
    f1.record()
    barrier()
    clocks.window(w0, time.time())
    gated_launches = G.kernel_launches() - nf0
    gated_ms = max_over_ranks(f0.elapsed_time(f1) / n_dec)
    # the step from raw projections: convolution (SiLU), gates and update in one launch
    fs = I.decode_fused(B=DECODE["B"], H=DECODE["H"], D=DECODE["D"], seed=replica_seed(1, rank))
    fring = [(dev_t(x), dev_t(a_), dev_t(b_)) for x, a_, b_ in (fs.step(s) for s in range(8))]
    cw = dev_t(fs.conv_w)
    cst = [dev_t(np.ascontiguousarray(fs.conv_state0.transpose(0, 2, 1))),   # tap-major [B, 3, C]
           torch.empty((ds.B, 3, fs.C), dtype=torch.float32, device=dev)]

    def fused_step(i):
        x, a_, b_ = fring[i % len(fring)]
        G.gdn_decode_step_fused(x, cw, cst[i % 2], a_, b_, dA, dbias, state, HK=ds.HK, conv_act=1, o=do,
                                conv_state_out=cst[(i + 1) % 2])

    for i in range(3):
        fused_step(i)
    barrier()
    nc0 = G.kernel_launches()
    c0 = torch.cuda.Event(enable_timing=True)
    c1 = torch.cuda.Event(enable_timing=True)
    w0 = time.time()
    c0.record()
    for i in range(n_dec):
        fused_step(i)
    c1.record()
    barrier()
    clocks.window(w0, time.time())
    fused_launches = G.kernel_launches() - nc0
    fused_ms = max_over_ranks(c0.elapsed_time(c1) / n_dec)
    # the same step with the output epilogue (zero-centred RMSNorm times 1 + w, sigmoid(z)) before
    # the store: gdn_decode_step_fused_outgate
    zring = [dev_t(fs.out_z(s_)).view(ds.B, ds.HV, ds.Dv) for s_ in range(8)]
    nwd = dev_t(fs.out_w())

    def fused_outgate_step(i):
        x, a_, b_ = fring[i % len(fring)]
        G.gdn_decode_step_fused(x, cw, cst[i % 2], a_, b_, dA, dbias, state, HK=ds.HK, conv_act=1, o=do,
                                conv_state_out=cst[(i + 1) % 2], outgate=(zring[i % len(zring)], nwd, 1e-6))

    for i in range(3):
        fused_outgate_step(i)
    barrier()
    c0.record()
    for i in range(n_dec):
        fused_outgate_step(i)
    c1.record()
    barrier()
    fused_og_ms = max_over_ranks(c0.elapsed_time(c1) / n_dec)
    del zring
    # a state twice the size of L2: B = 128 (256 MiB), the step alone (gates precomputed), so
    # that the HBM figure cannot rest on a state that stays in the 126 MB L2
    big = I.decode(B=2 * DECODE["B"], H=DECODE["H"], D=DECODE["D"], seed=replica_seed(5, rank))
    bstate = dev_t(big.state0)
    bq, bk, bv, ba_, bb_ = big.step(0)
    bq, bk, bv = dev_t(bq), dev_t(bk), dev_t(bv)
    bg, bbeta = G.gdn_gates(dev_t(ba_), dev_t(bb_), dev_t(big.A_log), dev_t(big.dt_bias))
    bo = torch.empty((big.B, big.HV, big.Dv), dtype=torch.bfloat16, device=dev)
    n_big = 256
    for _ in range(3):
        G.gdn_decode_step(bq, bk, bv, bg, bbeta, bstate, o=bo)
    barrier()
    c0.record()
    torch.cuda.nvtx.range_push("decode_b128")
    for _ in range(n_big):
        G.gdn_decode_step(bq, bk, bv, bg, bbeta, bstate, o=bo)
    torch.cuda.nvtx.range_pop()
    c1.record()
    barrier()
    big_ms = max_over_ranks(c0.elapsed_time(c1) / n_big)
    big_bytes = decode_bytes_per_step(big.B, big.HK, big.HV, big.Dk, big.Dv)
    big_gbs = big_bytes / (big_ms * 1e-3) / 1e9
    del bstate
    fbytes = (2 * ds.B * ds.HV * ds.Dk * ds.Dv * 4          # state in and out
              + ds.B * fs.C * 2 + 2 * ds.B * fs.C * 3 * 4   # x (bf16), convolution state in and out
              + fs.C * 16 + ds.B * ds.HV * (2 * 4 + ds.Dv * 2) + 2 * ds.HV * 4)   # weights, a, b, o, A_log, dt_bias
    fgbs = fbytes / (fused_ms * 1e-3) / 1e9
    dbytes = decode_bytes_per_step(ds.B, ds.HK, ds.HV, ds.Dk, ds.Dv)
    dgbs = dbytes / (dec_kernel_ms * 1e-3) / 1e9
    ggbs = dbytes / (gated_ms * 1e-3) / 1e9
    return {"workload": "decode: B=64 HK=HV=32 Dk=Dv=128 bf16 q/k/v, fp32 state 128 MiB, "
                        f"{n_dec} consecutive steps (gates + step), inputs cycled from 8 resident steps",
            "ms_per_step": dec_ms, "steps_per_s": world * 1e3 / dec_ms,
            "tokens_per_s": world * ds.B * 1e3 / dec_ms,
            "gpu_launches": dec_launches,
            "fused_step": {"what": "gdn_decode_step_fused: raw q|k|v projections, kernel-4 convolution (SiLU), "
                                   "gates and update in one launch per step",
                           "ms_per_step": fused_ms, "steps_per_s": world * 1e3 / fused_ms, "bytes_per_step": fbytes,
                           "achieved_gbs": fgbs, "frac": fgbs / P["hbm_gbs"], "gpu_launches": fused_launches},
            "fused_outgate_step": {"what": "gdn_decode_step_fused_outgate: the step from raw projections with the "
                                           "output epilogue (zero-centred RMSNorm x (1 + w), sigmoid(z), eps 1e-6) "
                                           "before the store",
                                   "ms_per_step": fused_og_ms, "steps_per_s": world * 1e3 / fused_og_ms,
                                   "vs_fused_step_us": (fused_og_ms - fused_ms) * 1e3},
            "state_2x_l2": {"what": "gdn_decode_step alone on B=128 (state 256 MiB, twice the L2), 256 steps",
                            "ms_per_step": big_ms, "bytes_per_step": big_bytes, "achieved_gbs": big_gbs,
                            "frac": big_gbs / P["hbm_gbs"]},
            "gated_step": {"what": "gdn_decode_step_gated: gates formed in the decode kernel, one launch per step",
                           "ms_per_step": gated_ms, "steps_per_s": world * 1e3 / gated_ms,
                           "achieved_gbs": ggbs, "frac": ggbs / P["hbm_gbs"], "gpu_launches": gated_launches},
            "roofline": {"bound": "hbm", "achieved": dgbs, "peak": P["hbm_gbs"], "unit": "GB/s",
                         "frac": dgbs / P["hbm_gbs"],
                         "traffic": _traffic().get("decode_bytes_per_launch"),
                         "peak_kind": f"{pk} copy bandwidth", "bytes_per_launch": dbytes,
                         "kernel_ms": dec_kernel_ms}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["gdn", "reference"], default="gdn")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--only", choices=["all", "prefill", "decode"], default="all")
    ap.add_argument("--decode-steps", type=int, default=DECODE["steps"])
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_gdn(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
