#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200.

One step = one kda_chunk_fwd over the B=4, H=32, T=8192, d=128 bf16 prefill
workload (strong decay), inputs resident in HBM. The same run also times the
decode step (N=256 sequences, H=32, d=128, 1000 chained in-place steps) and
reports it under "decode". Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs as one process per GPU under torch.distributed.run: every rank
processes its own copy of the workload (independent sequences: weak scaling,
no data-path collective); times are the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA chunk-fwd tokens/s (H=32,d=128,T=8K,bf16) and % of roofline; decode GB/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Algorithmic bytes per token-head for the prefill: q, k, v, log_alpha (bf16,
# d=128 each: 4 * 256 B), beta (2 B) and o (256 B). States are added per head.
BYTES_PER_TOKEN_HEAD = 4 * 256 + 2 + 256
# Dense chunkwise flop count per token-head at C=64, d=128: A and P (2*2*C*d),
# W and U (2*C*2d), P.D (2*C*d), W S, Ktilde^T D and Qtilde S (3*2*d*d).
FLOPS_PER_TOKEN_HEAD = 2 * 2 * 64 * 128 + 2 * 64 * 256 + 2 * 64 * 128 + 3 * 2 * 128 * 128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of one GPU
    while the timed region runs: NVML polled every ~1 ms from a thread
    (nvidia-smi as a fallback). Only reads state; changes nothing."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4}

    def __init__(self, torch_device_index: int):
        self.index = torch_device_index
        self.samples = []
        self.max_mhz = None
        self.err = None
        self._stop = threading.Event()

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            p = torch.cuda.get_device_properties(self.index)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _open(self):
        """NVML handle and maximum clock, opened before the timed region starts."""
        try:
            nv, h = self._handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            return lambda: (float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)), int(get_reasons(h)))
        except Exception as e:
            self.err = repr(e)
            return None

    def _smi(self):  # no NVML: one nvidia-smi reading
        try:
            out = subprocess.run(["nvidia-smi", "-i", str(self.index), "--query-gpu=clocks.sm,clocks.max.sm",
                                  "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                 timeout=10).stdout.strip().split(",")
            self.samples.append((float(out[0]), 0))
            self.max_mhz = float(out[1])
        except Exception:
            pass

    def _run(self):
        try:
            while True:
                self.samples.append(self._read())
                if self._stop.wait(0.001):
                    break
        except Exception as e:
            self.err = repr(e)

    def __enter__(self):
        self._read = self._open()
        if self._read is None:
            self._smi()
            self._t = None
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no clock samples: " + str(self.err)]}
        sm = sorted(x for x, _ in self.samples)
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = sorted(k for k, bit in self.REASONS.items() if mask & bit)
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "source": "nvml" if self.err is None else "nvidia-smi"}


# Source files each profiled kernel is built from: a recorded ncu traffic
# figure is reported only while these files are unchanged.
KERNEL_SOURCES = {
    "decode": ["kda_decode.cu", "kda_common.cuh"],
    "simt": ["kda_chunk_simt.cu", "kda_common.cuh"],
    "tc": ["kda_chunk_tc.cu", "kda_common.cuh", "kda_sm100.cuh"],
    "bwd": ["kda_chunk_bwd.cu", "kda_common.cuh"],
}
WIDENED = ("varlen", "variants", "b2_h16_t4k", "exact_path", "long_context", "backward")


def kernel_source_digest(kind: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        p = os.path.join(ROOT, "gated_delta_rule_134_b200", "csrc", name)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, algo: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d.get(f"{workload}/{algo}")
        if e and e.get("source_digest") == kernel_source_digest(algo):
            return e.get("dram_bytes_per_launch")
    except Exception:
        return None
    return None


def oracle_sample(cfg, n_heads, nthreads=0):
    """Times the fp64 oracle on n_heads full-length heads of cfg. Returns
    (seconds, equivalent tokens, threads used, sample description)."""
    import oracle
    from gated_delta_rule_134_b200 import inputs as I
    heads = [(i // cfg.H % cfg.B, i % cfg.H) for i in range(n_heads)]
    xs = I.prefill_inputs(cfg, heads=heads)
    arrs = [xs[k] for k in ("q", "k", "v", "log_alpha", "beta")]
    arrs = [a.double().numpy() for a in arrs]
    S0 = None if xs["S0"] is None else xs["S0"].double().numpy()
    cores = nthreads or os.cpu_count()
    t0 = time.perf_counter()
    oracle.recurrent(*arrs, S0, nthreads=cores)
    dt = time.perf_counter() - t0
    tokens = n_heads * cfg.T / cfg.H
    return dt, tokens, min(cores, n_heads), f"{n_heads} of {cfg.B * cfg.H} heads x T={cfg.T}, fp64 recurrence"


def run_reference(args):
    """Reference arm: the fp64 CPU oracle, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from gated_delta_rule_134_b200 import inputs as I
    cfg = I.B4_H32_T8K
    cores = os.cpu_count()
    n_heads = max(1, min(cores, cfg.B * cfg.H))
    for _ in range(args.warmup):
        oracle_sample(cfg, n_heads)
    total_t, total_tok = 0.0, 0.0
    for _ in range(args.steps):
        dt, tok, used, sample = oracle_sample(cfg, n_heads)
        total_t += dt
        total_tok += tok
    value = total_tok / total_t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "T": cfg.T, "dk": cfg.dk, "dv": cfg.dv,
                       "chunk": cfg.C, "parallelism": "host threads over heads"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                             "sample": f"per step: {sample}"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


class Ctx:
    """Per-process distributed context (one rank per GPU). The path shards by
    replicas: ranks exchange nothing on the data path, only the barrier and
    the max-over-ranks of the timings. backend="gloo" runs the same host logic
    on CPU (tests)."""

    def __init__(self, backend: str = "nccl", timeout_s: float = 120.0):
        import torch
        import torch.distributed as dist
        self.torch, self.dist = torch, dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        cuda = backend == "nccl"
        if cuda:
            torch.cuda.set_device(self.local)
        if self.world > 1:
            import datetime
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
        self.dev = torch.device("cuda", self.local) if cuda else torch.device("cpu")
        self.stream = torch.cuda.current_stream(self.dev) if cuda else None

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, x: float) -> float:
        if self.world == 1:
            return x
        t = self.torch.tensor([x], dtype=self.torch.float64, device=self.dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def replica_seed(base_seed: int, rank: int) -> int:
    """Each replica draws its own inputs of the same workload."""
    return base_seed + 1000 * rank


def whole_job_rate(world: int, units_per_rank: float, ms_max: float) -> float:
    """Units per second of the whole job: every rank processed units_per_rank
    in at most ms_max milliseconds (the max over ranks)."""
    return world * units_per_rank / (ms_max * 1e-3)


class Prefill:
    """The B=4, H=32, T=8192 bf16 prefill workload resident on this rank's GPU."""

    def __init__(self, ctx, kda, I, algo, profile_T=None):
        torch = ctx.torch
        self.kda, self.ctx, self.algo = kda, ctx, algo
        base = I.B4_H32_T8K
        self.cfg = cfg = base.replace(seed=replica_seed(base.seed, ctx.rank), T=profile_T or base.T)
        self.name = base.name if not profile_T else f"{base.name}_profile_T{profile_T}"
        self.x = {k: (None if v is None else v.to(ctx.dev)) for k, v in I.prefill_inputs(cfg).items()}
        B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv
        self.o = torch.empty(B, T, H, dv, dtype=torch.bfloat16, device=ctx.dev)
        self.ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device=ctx.dev)
        self.ws_bytes = kda.workspace_size(B, T, H, dk, dv, cfg.C, "bf16", algo)
        self.ws = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=ctx.dev)
        self.use_tc = algo == "tc" or (algo == "auto" and self.ws_bytes > 0)
        self.algo_name = "tc" if self.use_tc else "simt"
        self.launches_per_step = 1
        self.tokens_per_step = B * T

    def run(self, x=None):
        x = x or self.x
        self.kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], chunk=self.cfg.C,
                           algo=self.algo, o=self.o, S_T=self.ST, workspace=self.ws if self.ws_bytes else None,
                           stream=self.ctx.stream)

    def algorithmic_bytes(self):
        cfg = self.cfg
        state = self.ST.numel() * 4 * (2 if self.x["S0"] is not None else 1)
        return BYTES_PER_TOKEN_HEAD * cfg.B * cfg.T * cfg.H + state

    def algorithmic_flops(self):
        cfg = self.cfg
        return FLOPS_PER_TOKEN_HEAD * cfg.B * cfg.T * cfg.H


def time_prefill(args, ctx, pf, peaks, peak_kind):
    torch = ctx.torch
    for _ in range(args.warmup):
        pf.run()
    torch.cuda.synchronize()
    ctx.barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
    with ClockSampler(ctx.local) as clk:
        for i in range(args.steps):
            ev[2 * i].record(ctx.stream)
            pf.run()
            ev[2 * i + 1].record(ctx.stream)
        torch.cuda.synchronize()
    ctx.barrier()
    total_ms = ctx.max_over_ranks(ev[0].elapsed_time(ev[-1]))
    per_launch = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps)]
    avg_launch_ms = ctx.max_over_ranks(sum(per_launch) / len(per_launch))
    if pf.use_tc and pf.kda.workspace_status(pf.ws, ctx.stream) != 0:
        raise RuntimeError("device-side timeout reported by the prefill kernel")
    ms_per_step = total_ms / args.steps
    alg_bytes = pf.algorithmic_bytes()
    achieved = alg_bytes / (avg_launch_ms * 1e-3) / 1e9
    tflops = pf.algorithmic_flops() / (avg_launch_ms * 1e-3) / 1e12
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": recorded_traffic(pf.name, pf.algo_name),
                "peak_source": ("of measured (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                                else "of fallback"),
                "kernel": "kda_chunk_tc_kernel" if pf.use_tc else "chunk_simt_kernel",
                "algorithmic_bytes_per_launch": alg_bytes, "avg_launch_ms": avg_launch_ms,
                "tensor": {"achieved_tflops": tflops, "peak_tflops": peaks["bf16_tflops"],
                           "frac": tflops / peaks["bf16_tflops"],
                           "algorithmic_flops_per_launch": pf.algorithmic_flops()}}
    return ms_per_step, roofline, clk.summary()


def time_e2e(args, ctx, pf, pieces_per_seq: int = 4):
    """Same metric through the C ABI with host buffers: every step copies all
    of its inputs host->device from pinned memory and reads o and S_T back.
    The batch is cut into pieces of whole chunks along T (each sequence in
    order, its state passed from piece to piece through S0 / S_T), and three
    streams overlap the copy of piece p+1, the prefill of piece p and the
    read-back of piece p-1; the copy engines then set the pace."""
    torch = ctx.torch
    cfg = pf.cfg
    B, T = cfg.B, cfg.T
    pin = {k: (None if v is None else v.cpu().pin_memory()) for k, v in pf.x.items()}
    dbuf = {k: (None if v is None else torch.empty_like(v)) for k, v in pf.x.items()}
    o_host = torch.empty(pf.o.shape, dtype=pf.o.dtype, pin_memory=True)
    ST_host = torch.empty(pf.ST.shape, dtype=pf.ST.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pin.values() if v is not None)
    d2h = o_host.numel() * o_host.element_size() + ST_host.numel() * ST_host.element_size()
    LT = max(cfg.C, (T // pieces_per_seq + cfg.C - 1) // cfg.C * cfg.C)  # tokens per piece, whole chunks
    cuts = [(b, t0, min(t0 + LT, T)) for b in range(B) for t0 in range(0, T, LT)]
    s_in, s_run, s_out = torch.cuda.Stream(ctx.dev), torch.cuda.Stream(ctx.dev), torch.cuda.Stream(ctx.dev)
    dts = "bf16" if pf.x["q"].dtype == torch.bfloat16 else "f32"
    ws_piece = max(pf.kda.workspace_size(1, t1 - t0, cfg.H, cfg.dk, cfg.dv, cfg.C, dts, pf.algo)
                   for _, t0, t1 in cuts)
    ws = torch.empty(max(ws_piece, 256), dtype=torch.uint8, device=ctx.dev)

    def step():
        start = torch.cuda.Event()
        start.record(ctx.stream)
        for st in (s_in, s_run, s_out):
            st.wait_event(start)
        for b, t0, t1 in cuts:
            with torch.cuda.stream(s_in):
                for k in ("q", "k", "v", "log_alpha", "beta"):
                    dbuf[k][b, t0:t1].copy_(pin[k][b, t0:t1], non_blocking=True)
                if t0 == 0 and pin["S0"] is not None:
                    dbuf["S0"][b].copy_(pin["S0"][b], non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
            s_run.wait_event(landed)
            sl = lambda key: dbuf[key][b:b + 1, t0:t1]
            S0 = (dbuf["S0"][b:b + 1] if pin["S0"] is not None else None) if t0 == 0 else pf.ST[b:b + 1]
            pf.kda.chunk_fwd(sl("q"), sl("k"), sl("v"), sl("log_alpha"), sl("beta"), S0, chunk=cfg.C,
                             algo=pf.algo, o=pf.o[b:b + 1, t0:t1], S_T=pf.ST[b:b + 1], workspace=ws,
                             stream=s_run)
            done = torch.cuda.Event()
            done.record(s_run)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                o_host[b, t0:t1].copy_(pf.o[b, t0:t1], non_blocking=True)
                if t1 == T:
                    ST_host[b].copy_(pf.ST[b], non_blocking=True)
        fin = torch.cuda.Event()
        fin.record(s_out)
        ctx.stream.wait_event(fin)

    n = max(3, min(args.steps, 10))
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ctx.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(ctx.stream)
    for _ in range(n):
        step()
    e1.record(ctx.stream)
    torch.cuda.synchronize()
    ms = ctx.max_over_ranks(e0.elapsed_time(e1) / n)
    if pf.use_tc and pf.kda.workspace_status(ws, s_run) != 0:
        raise RuntimeError("device-side timeout reported by the prefill kernel")
    # the pieces must reproduce one call over the whole batch (up to rounding)
    o_one, S_one = pf.o.clone(), pf.ST.clone()
    pf.run()
    torch.cuda.synchronize()
    den_o, den_s = pf.o.float().abs().max().item(), pf.ST.abs().max().item()
    diff = max((o_host.to(ctx.dev).float() - pf.o.float()).abs().max().item() / max(den_o, 1e-30),
               (ST_host.to(ctx.dev) - pf.ST).abs().max().item() / max(den_s, 1e-30))
    del o_one, S_one
    if not diff < 2e-2:
        raise RuntimeError(f"pipelined end-to-end result differs from one call: {diff}")
    return {"value": whole_job_rate(ctx.world, pf.tokens_per_step, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": n,
            "pieces": len(cuts), "tokens_per_piece": LT, "max_rel_diff_vs_one_call": diff,
            "path": "pinned host -> device copies, kda_chunk_fwd per piece (state chained through S0/S_T), "
                    "device -> pinned host copies of o and S_T; copy, compute and read-back on three streams"}


def time_decode(args, ctx, kda, I, peaks, peak_kind):
    """N=256 x H=32, d=128 decode: chained in-place steps with fresh inputs
    each step (pre-generated on the device by torch's seeded generator)."""
    torch = ctx.torch
    dcfg = I.DECODE_N256_H32
    nd = args.decode_steps
    g = torch.Generator(device=ctx.dev)
    g.manual_seed(dcfg.seed + 1000 * ctx.rank)
    S = dcfg.s_std * torch.randn(dcfg.N, dcfg.H, dcfg.dk, dcfg.dv, device=ctx.dev, generator=g)

    def unit(z):
        return z / z.norm(dim=-1, keepdim=True)

    shp = (nd, dcfg.N, dcfg.H)
    dq = unit(torch.randn(*shp, dcfg.dk, device=ctx.dev, generator=g)).bfloat16()
    dk = unit(torch.randn(*shp, dcfg.dk, device=ctx.dev, generator=g)).bfloat16()
    dv = torch.randn(*shp, dcfg.dv, device=ctx.dev, generator=g).bfloat16()
    dla = (-(dcfg.la_lo + (dcfg.la_hi - dcfg.la_lo) * torch.rand(*shp, dcfg.dk, device=ctx.dev,
                                                                   generator=g))).bfloat16()
    db = torch.sigmoid(torch.randn(*shp, device=ctx.dev, generator=g)).bfloat16()
    do = torch.empty(dcfg.N, dcfg.H, dcfg.dv, dtype=torch.bfloat16, device=ctx.dev)
    for i in range(min(3, nd)):
        kda.decode_step(dq[i], dk[i], dv[i], dla[i], db[i], S, o=do, stream=ctx.stream)
    torch.cuda.synchronize()
    ctx.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(ctx.local) as clk:
        e0.record(ctx.stream)
        for i in range(nd):
            kda.decode_step(dq[i], dk[i], dv[i], dla[i], db[i], S, o=do, stream=ctx.stream)
        e1.record(ctx.stream)
        torch.cuda.synchronize()
    ms = ctx.max_over_ranks(e0.elapsed_time(e1))
    us = ms * 1e3 / nd
    nbytes = 2 * S.numel() * 4 + (3 * dq[0].numel() + dv[0].numel() + db[0].numel() + do.numel()) * 2
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"workload": dcfg.name, "value": ctx.world * gbs, "unit": "GB/s", "us_per_step": us, "steps": nd,
            "algorithmic_bytes_per_step": nbytes, "gpu_launches": nd,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "kernel": "decode_step_kernel",
                         "peak_source": "of measured" if peak_kind == "measured" else "of fallback",
                         "traffic": recorded_traffic(dcfg.name, "decode")},
            "clocks": clk.summary(), "inputs": "pre-generated on the device, fresh each step"}


def _time_calls(ctx, fn, warmup, steps):
    """Average device time (ms) of fn() over `steps` launches on ctx.stream,
    after `warmup` untimed ones; max over ranks."""
    torch = ctx.torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ctx.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(ctx.stream)
    for _ in range(steps):
        fn()
    e1.record(ctx.stream)
    torch.cuda.synchronize()
    return ctx.max_over_ranks(e0.elapsed_time(e1) / steps)


def time_widened(args, ctx, kda, I, pf, peaks):
    """The widened rows, each on a workload of the headline's size:
    packed variable-length sequences (about 32K tokens in 32 sequences of
    mixed lengths, H32 d128, strong decay), the four variants on the
    B4 H32 T8192 inputs, the B1 H32 T131072 long-context prefill with
    and without the chunk-parallel segment scan, and the backward pass on
    the B4 H32 T8192 inputs. Tokens/s and the HBM roofline fraction of each
    (algorithmic bytes: q, k, v, the gate as the variant reads it, beta, o,
    and the states)."""
    steps = max(3, min(args.steps, 10))
    hbm = peaks["hbm_gbs"]
    out = {}
    if "varlen" in args.parts:
        out["varlen"] = _time_varlen(args, ctx, kda, I, steps, hbm)
    if "variants" in args.parts:
        out["variants"] = _time_variants(args, ctx, kda, pf, steps, hbm)
    if "b2_h16_t4k" in args.parts:
        out["b2_h16_t4k"] = _time_b2_h16(ctx, kda, I, hbm)
    if "exact_path" in args.parts:
        out["exact_path"] = _time_exact_path(args, ctx, kda, pf, steps, hbm)
    if "long_context" in args.parts:
        out["long_context"] = _time_long_context(ctx, kda, I, hbm, args.long_T)
    if "backward" in args.parts:
        out["backward"] = _time_backward(ctx, kda, pf, hbm)
    if pf.use_tc and kda.workspace_status(pf.ws, ctx.stream) != 0:
        raise RuntimeError("device-side timeout reported by the prefill kernel")
    return out


def _time_varlen(args, ctx, kda, I, steps, hbm):
    torch = ctx.torch
    lengths = I.varlen_lengths(32, 1024, seed=48 + ctx.rank)
    vcfg = I.B4_H32_T8K.replace(seed=48 + ctx.rank)
    xv = {k: (None if v is None else v.to(ctx.dev)) for k, v in I.varlen_inputs(vcfg, lengths).items()}
    TT, N, H = sum(lengths), len(lengths), vcfg.H
    ov = torch.empty(TT, H, vcfg.dv, dtype=torch.bfloat16, device=ctx.dev)
    Sv = torch.empty(N, H, vcfg.dk, vcfg.dv, dtype=torch.float32, device=ctx.dev)
    wsv = torch.empty(256, dtype=torch.uint8, device=ctx.dev)

    def run_v():
        kda.chunk_fwd_varlen(xv["q"], xv["k"], xv["v"], xv["log_alpha"], xv["beta"], xv["cu_seqlens"], xv["S0"],
                             o=ov, S_T=Sv, workspace=wsv, stream=ctx.stream)
    ms = _time_calls(ctx, run_v, args.warmup, steps)
    nbytes = BYTES_PER_TOKEN_HEAD * TT * H + Sv.numel() * 4 + 4 * (N + 1)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"packed_n{N}_total{TT}_h32_d128_bf16_strong_decay", "lengths": "U(1, 2047)",
            "value": ctx.world * TT / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "algorithmic_bytes_per_launch": nbytes}}


def _time_variants(args, ctx, kda, pf, steps, hbm):
    x = pf.x
    cfg = pf.cfg
    la_tok = x["log_alpha"][..., 0].contiguous()
    per_gate = {"channel": 256, "scalar": 2, "none": 0}
    variants = {"kda": (True, "channel"), "scalar_gated_delta": (True, "scalar"), "delta_rule": (True, "none"),
                "gated_linear_attention": (False, "channel"), "linear_attention": (False, "none")}
    res = {}
    for name, (erase, gate) in variants.items():
        la = {"channel": x["log_alpha"], "scalar": la_tok, "none": None}[gate]

        def run_x():
            kda.chunk_fwd(x["q"], x["k"], x["v"], la, x["beta"], x["S0"], chunk=cfg.C, algo=pf.algo, o=pf.o,
                          S_T=pf.ST, workspace=pf.ws if pf.ws_bytes else None, stream=ctx.stream, erase=erase,
                          gate=gate)
        ms = _time_calls(ctx, run_x, args.warmup, steps)
        ntok = cfg.B * cfg.T
        nbytes = (3 * 256 + per_gate[gate] + 2 + 256) * ntok * cfg.H + pf.ST.numel() * 4
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"erase": erase, "gate": gate, "value": ctx.world * ntok / (ms * 1e-3), "unit": "tokens/s",
                     "ms_per_step": ms, "roofline_frac": gbs / hbm, "achieved_gbs": gbs}
    return {"workload": cfg.name, "steps": steps, **res}


def _time_b2_h16(ctx, kda, I, hbm):
    """B2 H16 T4096 (few heads: 32 (batch, head) units on the GPU): AUTO, the
    one-pass tensor-core kernel and the segment scan, with the algorithm AUTO
    picked (it adds the scan when the workspace it asks for holds segment
    maps)."""
    torch = ctx.torch
    cfg = I.B2_H16_T4K.replace(seed=I.B2_H16_T4K.seed + 1000 * ctx.rank)
    x = {k: (None if v is None else v.to(ctx.dev)) for k, v in I.prefill_inputs(cfg).items()}
    o = torch.empty(cfg.B, cfg.T, cfg.H, cfg.dv, dtype=torch.bfloat16, device=ctx.dev)
    S = torch.empty(cfg.B, cfg.H, cfg.dk, cfg.dv, dtype=torch.float32, device=ctx.dev)
    ntok = cfg.B * cfg.T
    nbytes = BYTES_PER_TOKEN_HEAD * ntok * cfg.H + 2 * S.numel() * 4  # S0 read, S_T written
    res = {"workload": cfg.name, "units": cfg.B * cfg.H}
    for algo in ("auto", "tc", "tc_scan"):
        wsb = kda.workspace_size(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, cfg.C, "bf16", algo)
        ws = torch.empty(max(wsb, 256), dtype=torch.uint8, device=ctx.dev)

        def run_b():
            kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], chunk=cfg.C, algo=algo, o=o,
                          S_T=S, workspace=ws, stream=ctx.stream)
        ms = _time_calls(ctx, run_b, 5, 20)
        if kda.workspace_status(ws, ctx.stream) != 0:
            raise RuntimeError("device-side timeout reported by the prefill kernel")
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[algo] = {"value": ctx.world * ntok / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": 20,
                     "roofline_frac": gbs / hbm, "achieved_gbs": gbs, "workspace_bytes": wsb}
    res["auto_picked"] = "tc_scan" if res["auto"]["workspace_bytes"] > 256 else "tc"
    del x, o, S
    return res


def _time_exact_path(args, ctx, kda, pf, steps, hbm):
    """The B4 H32 T8192 shapes with decays too strong for the chunk-start
    reference point (|G| > 80 within a chunk): -U(1.5, 3) per token and
    channel (about 144 per chunk, the G_last / 2 reference takes the chunks)
    and -U(3, 6) (about 288 per chunk, the exact per-pair path)."""
    torch = ctx.torch
    x, cfg = pf.x, pf.cfg
    ntok = cfg.B * cfg.T
    nbytes = BYTES_PER_TOKEN_HEAD * ntok * cfg.H + pf.ST.numel() * 4
    out = {}
    for key, lo, hi, path in (("mid_reference", 1.5, 3.0, "reference point G_last / 2"),
                              ("exact", 3.0, 6.0, "exact per-pair exponentials")):
        g = torch.Generator(device=ctx.dev)
        g.manual_seed(cfg.seed + 555 + 1000 * ctx.rank)
        la = (-(lo + (hi - lo) * torch.rand(cfg.B, cfg.T, cfg.H, cfg.dk, device=ctx.dev, generator=g))).bfloat16()

        def run_e():
            kda.chunk_fwd(x["q"], x["k"], x["v"], la, x["beta"], x["S0"], chunk=cfg.C, algo=pf.algo, o=pf.o,
                          S_T=pf.ST, workspace=pf.ws if pf.ws_bytes else None, stream=ctx.stream)
        ms = _time_calls(ctx, run_e, 3, 3)
        gbs = nbytes / (ms * 1e-3) / 1e9
        del la
        out[key] = {"workload": f"{cfg.name}_decay_U{lo:g}_{hi:g}", "path": path,
                    "value": ctx.world * ntok / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": 3,
                    "roofline_frac": gbs / hbm, "achieved_gbs": gbs}
    return out


def _time_long_context(ctx, kda, I, hbm, T=None):
    """B1 H32 T131072: one pass per sequence against the segment scan. T
    shortens the sequence for profiler captures (the same grid and segment
    count for T >= 16384)."""
    torch = ctx.torch
    lc = I.B1_H32_T128K if not T else I.B1_H32_T128K.replace(T=T, name=f"{I.B1_H32_T128K.name}_profile_T{T}")
    g = torch.Generator(device=ctx.dev)
    g.manual_seed(lc.seed + 1000 * ctx.rank)
    shp = (lc.B, lc.T, lc.H)

    def unit(z):
        return (z / z.norm(dim=-1, keepdim=True)).bfloat16()
    xl = {"q": unit(torch.randn(*shp, lc.dk, device=ctx.dev, generator=g)),
          "k": unit(torch.randn(*shp, lc.dk, device=ctx.dev, generator=g)),
          "v": torch.randn(*shp, lc.dv, device=ctx.dev, generator=g).bfloat16(),
          "log_alpha": (-(lc.la_lo + (lc.la_hi - lc.la_lo) * torch.rand(*shp, lc.dk, device=ctx.dev,
                                                                          generator=g))).bfloat16(),
          "beta": torch.sigmoid(torch.randn(*shp, device=ctx.dev, generator=g)).bfloat16()}
    ol = torch.empty(*shp, lc.dv, dtype=torch.bfloat16, device=ctx.dev)
    Sl = torch.empty(lc.B, lc.H, lc.dk, lc.dv, dtype=torch.float32, device=ctx.dev)
    ntok = lc.B * lc.T
    nbytes = BYTES_PER_TOKEN_HEAD * ntok * lc.H + Sl.numel() * 4
    long_ctx = {"workload": lc.name, "inputs": "drawn on the device (same distributions)"}
    for algo in ("tc", "tc_scan"):
        wsb = kda.workspace_size(lc.B, lc.T, lc.H, lc.dk, lc.dv, lc.C, "bf16", algo)
        wsl = torch.empty(wsb, dtype=torch.uint8, device=ctx.dev)

        def run_l():
            kda.chunk_fwd(xl["q"], xl["k"], xl["v"], xl["log_alpha"], xl["beta"], None, chunk=lc.C, algo=algo,
                          o=ol, S_T=Sl, workspace=wsl, stream=ctx.stream)
        ms = _time_calls(ctx, run_l, 3, 3)
        if kda.workspace_status(wsl, ctx.stream) != 0:
            raise RuntimeError("device-side timeout reported by the prefill kernel")
        gbs = nbytes / (ms * 1e-3) / 1e9
        long_ctx[algo] = {"value": ctx.world * ntok / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
                          "steps": 3, "roofline_frac": gbs / hbm, "achieved_gbs": gbs, "workspace_bytes": wsb}
    del xl, ol, Sl
    return long_ctx


def _time_backward(ctx, kda, pf, hbm):
    """Gradients of o and S_T on the prefill inputs (kda_chunk_bwd)."""
    torch = ctx.torch
    x, cfg = pf.x, pf.cfg
    gb = torch.Generator(device=ctx.dev)
    gb.manual_seed(cfg.seed + 77 + 1000 * ctx.rank)
    dO = torch.randn(cfg.B, cfg.T, cfg.H, cfg.dv, device=ctx.dev, generator=gb).bfloat16()
    dST = torch.randn(cfg.B, cfg.H, cfg.dk, cfg.dv, device=ctx.dev, generator=gb)
    wbb = int(kda.load().kda_chunk_bwd_workspace_size(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv))
    wsb = torch.empty(wbb, dtype=torch.uint8, device=ctx.dev)

    def run_b():
        kda.chunk_bwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], dO, dST, workspace=wsb,
                      stream=ctx.stream)
    ms = _time_calls(ctx, run_b, 3, 3)
    ntok = cfg.B * cfg.T
    # read q, k, v, log_alpha, beta, dO; write dq, dk, dv, dlog_alpha, dbeta; dS_T read, dS0 written
    nbytes = (5 * 256 + 2 + 4 * 256 + 2) * ntok * cfg.H + 2 * pf.ST.numel() * 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    del dO, dST, wsb
    return {"workload": pf.name, "kernel": "chunk_bwd_kernel", "value": ctx.world * ntok / (ms * 1e-3),
            "unit": "tokens/s", "ms_per_step": ms, "steps": 3, "workspace_bytes": wbb,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "algorithmic_bytes_per_launch": nbytes, "traffic": recorded_traffic(pf.name, "bwd")},
            "note": "fp32 (tf32x3 warp MMAs for the products), one CTA per (batch, head): barrier and latency bound"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kda", choices=["kda", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-T", type=int, default=None,
                    help="shorter sequence for profiler captures (the printed line is then not a bench value)")
    ap.add_argument("--e2e-pieces", type=int, default=4,
                    help="pieces per sequence in the end-to-end pipeline (whole chunks each)")
    ap.add_argument("--long-T", type=int, default=None,
                    help="shorter sequence for the long-context leg (profiler captures; not a bench value)")
    ap.add_argument("--parts", default="prefill,e2e,decode,widened",
                    help="comma list of prefill, e2e, decode, widened (= varlen, variants, b2_h16_t4k, exact_path, long_context, "
                         "backward) (profiling runs select one)")
    args = ap.parse_args()
    args.parts = set(args.parts.split(","))
    if "widened" in args.parts:
        args.parts |= set(WIDENED)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import gated_delta_rule_134_b200 as kda
    from gated_delta_rule_134_b200 import inputs as I

    ctx = Ctx()
    kda.load()
    peaks, peak_kind = load_peaks()
    line = {"metric": METRIC, "value": None, "unit": "tokens/s", "n_gpus": ctx.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": None, "data": "synthetic", "config": None, "roofline": None,
            "cpu_baseline": None, "e2e": None, "gpu_launches": None, "clocks": None, "decode": None,
            "widened": None}
    if args.parts & ({"prefill", "e2e"} | set(WIDENED)):
        pf = Prefill(ctx, kda, I, args.algo, args.profile_T)
        line["config"] = {"workload": pf.name, "B": pf.cfg.B, "H": pf.cfg.H, "T": pf.cfg.T, "dk": pf.cfg.dk,
                          "dv": pf.cfg.dv, "chunk": pf.cfg.C, "algo": pf.algo_name,
                          "parallelism": f"replicas x{ctx.world}",
                          "l2": "inputs larger than L2 (1.07 GB read per step, L2 126 MB)"}
        line["dtype"] = "bf16" if pf.use_tc else "f32"
        if "prefill" in args.parts:
            ms, roof, clocks = time_prefill(args, ctx, pf, peaks, peak_kind)
            line.update(value=whole_job_rate(ctx.world, pf.tokens_per_step, ms), ms_per_step=ms, roofline=roof,
                        clocks=clocks, gpu_launches=pf.launches_per_step * args.steps)
        if "e2e" in args.parts:
            line["e2e"] = time_e2e(args, ctx, pf, args.e2e_pieces)
        if args.parts & set(WIDENED):
            line["widened"] = time_widened(args, ctx, kda, I, pf, peaks)
        del pf
    if "decode" in args.parts:
        line["decode"] = time_decode(args, ctx, kda, I, peaks, peak_kind)
    if ctx.rank == 0 and ctx.world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count()
        n_heads = max(1, min(cores, 128))
        dt, tok, used, sample = oracle_sample(I.B4_H32_T8K, n_heads)
        line["cpu_baseline"] = {"value": tok / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
                                "sample": sample, "seconds": dt}
    if ctx.rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
