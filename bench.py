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
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except FileNotFoundError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = sorted(float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit())
        mx = max((float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(self.rows)}


def kernel_source_digest():
    import glob
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "gated_delta_rule_134_b200", "csrc", "*"))):
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
        if e and e.get("source_digest") == kernel_source_digest():
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kda", choices=["kda", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import gated_delta_rule_134_b200 as kda
    from gated_delta_rule_134_b200 import inputs as I

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    kda.load()
    peaks, peak_kind = load_peaks()
    cfg = I.B4_H32_T8K.replace(seed=I.B4_H32_T8K.seed + 1000 * rank)
    x = {k: (None if v is None else v.to(dev)) for k, v in I.prefill_inputs(cfg).items()}
    B, T, H, dk, dv = cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv
    o = torch.empty(B, T, H, dv, dtype=torch.bfloat16, device=dev)
    ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    ws_bytes = kda.workspace_size(B, T, H, dk, dv, cfg.C, "bf16", args.algo)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    use_tc = args.algo == "tc" or (args.algo == "auto" and ws_bytes > 0)
    algo_name = "tc" if use_tc else "simt"
    launches_per_step = 1

    def step():
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["beta"], x["S0"], chunk=cfg.C, algo=args.algo,
                      o=o, S_T=ST, workspace=ws if ws_bytes else None, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * args.steps)]
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            ev[2 * i].record(stream)
            step()
            ev[2 * i + 1].record(stream)
        torch.cuda.synchronize()
    barrier()
    per_launch_ms = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(args.steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    total_ms = max_over_ranks(total_ms)
    avg_launch_ms = max_over_ranks(sum(per_launch_ms) / len(per_launch_ms))
    ms_per_step = total_ms / args.steps
    tokens_per_step = B * T
    value = world * tokens_per_step / (ms_per_step * 1e-3)
    if use_tc and kda.workspace_status(ws, stream) != 0:
        raise RuntimeError("device-side timeout reported by the prefill kernel")

    alg_bytes = BYTES_PER_TOKEN_HEAD * B * T * H + ST.numel() * 4 + (0 if x["S0"] is None else ST.numel() * 4)
    achieved_gbs = alg_bytes / (avg_launch_ms * 1e-3) / 1e9
    alg_flops = FLOPS_PER_TOKEN_HEAD * B * T * H
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": recorded_traffic(cfg.name.split("_seed")[0],
                                                                                     algo_name),
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                else "fallback",
                "algorithmic_bytes_per_launch": alg_bytes, "avg_launch_ms": avg_launch_ms,
                "kernel": "kda_chunk_tc_kernel" if use_tc else "chunk_simt_kernel",
                "tensor": {"achieved_tflops": alg_flops / (avg_launch_ms * 1e-3) / 1e12,
                           "peak_tflops": peaks["bf16_tflops"],
                           "frac": alg_flops / (avg_launch_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}}

    # ---- end to end through the C ABI with host buffers
    pin = {k: (None if v is None else v.cpu().pin_memory()) for k, v in x.items()}
    dbuf = {k: (None if v is None else torch.empty_like(v)) for k, v in x.items()}
    o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    ST_host = torch.empty(ST.shape, dtype=ST.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in pin.values() if v is not None)
    d2h = o_host.numel() * o_host.element_size() + ST_host.numel() * 4

    def e2e_step():
        for k_ in pin:
            if pin[k_] is not None:
                dbuf[k_].copy_(pin[k_], non_blocking=True)
        kda.chunk_fwd(dbuf["q"], dbuf["k"], dbuf["v"], dbuf["log_alpha"], dbuf["beta"], dbuf["S0"], chunk=cfg.C,
                      algo=args.algo, o=o, S_T=ST, workspace=ws if ws_bytes else None, stream=stream)
        o_host.copy_(o, non_blocking=True)
        ST_host.copy_(ST, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps)
    e2e = {"value": world * tokens_per_step / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps}
    del pin, dbuf

    # ---- decode step: N=256 sequences x 32 heads, 1000 chained in-place steps
    dcfg = I.DECODE_N256_H32
    nd = args.decode_steps
    g = torch.Generator(device=dev)
    g.manual_seed(dcfg.seed + 1000 * rank)
    S = dcfg.s_std * torch.randn(dcfg.N, dcfg.H, dcfg.dk, dcfg.dv, device=dev, generator=g)

    def unit(z):
        return z / z.norm(dim=-1, keepdim=True)

    shp = (nd, dcfg.N, dcfg.H)
    dq = unit(torch.randn(*shp, dcfg.dk, device=dev, generator=g)).bfloat16()
    dk_ = unit(torch.randn(*shp, dcfg.dk, device=dev, generator=g)).bfloat16()
    dv_ = torch.randn(*shp, dcfg.dv, device=dev, generator=g).bfloat16()
    dla = (-(dcfg.la_lo + (dcfg.la_hi - dcfg.la_lo) * torch.rand(*shp, dcfg.dk, device=dev, generator=g))).bfloat16()
    db = torch.sigmoid(torch.randn(*shp, device=dev, generator=g)).bfloat16()
    do = torch.empty(dcfg.N, dcfg.H, dcfg.dv, dtype=torch.bfloat16, device=dev)
    for i in range(3):
        kda.decode_step(dq[i], dk_[i], dv_[i], dla[i], db[i], S, o=do, stream=stream)
    torch.cuda.synchronize()
    barrier()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as dclk:
        d0.record(stream)
        for i in range(nd):
            kda.decode_step(dq[i], dk_[i], dv_[i], dla[i], db[i], S, o=do, stream=stream)
        d1.record(stream)
        torch.cuda.synchronize()
    dec_ms = max_over_ranks(d0.elapsed_time(d1))
    us_step = dec_ms * 1e3 / nd
    dec_bytes = 2 * S.numel() * 4 + (dq[0].numel() * 3 + dv_[0].numel() + db[0].numel() + do.numel()) * 2
    dec_gbs = dec_bytes / (us_step * 1e-6) / 1e9
    decode = {"workload": dcfg.name, "value": world * dec_gbs, "unit": "GB/s", "us_per_step": us_step,
              "steps": nd, "algorithmic_bytes_per_step": dec_bytes,
              "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": dec_gbs / peaks["hbm_gbs"], "kernel": "decode_step_kernel",
                           "traffic": recorded_traffic(dcfg.name, "decode")},
              "clocks": dclk.summary(), "inputs": "pre-generated on the device, fresh each step"}
    del dq, dk_, dv_, dla, db, S

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_heads = max(1, min(os.cpu_count(), cfg.B * cfg.H))
        dt, tok, used, sample = oracle_sample(I.B4_H32_T8K, n_heads)
        cpu = {"value": tok / dt, "unit": "tokens/s", "cores": used, "kind": "oracle", "sample": sample,
               "seconds": dt}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if use_tc else "f32", "data": "synthetic",
                "config": {"workload": I.B4_H32_T8K.name, "B": B, "H": H, "T": T, "dk": dk, "dv": dv,
                           "chunk": cfg.C, "algo": algo_name, "parallelism": f"replicas x{world}",
                           "l2": "inputs larger than L2 (1.07 GB read per step)"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clk.summary(), "decode": decode}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
