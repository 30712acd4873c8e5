"""Benchmark of the gated delta-rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-decode]

One step = one dn_chunk_fwd over the GDN prefill workload (B=8, H=16, T=4096,
d_k=d_v=128, bf16 q/k/v, scalar fp32 gates, chunk 64) with inputs resident in
HBM. The same run also times the decode workload (1024 sequences x 32 heads,
d=128, fp32 state of 2 GiB updated in place, 100 consecutive steps) and reports
its HBM throughput. Prints ONE JSON line on rank 0.

Multi-GPU (torchrun): heads are independent, so every rank runs its own full
workload with no collective on the data path (weak scaling); the time is the
max over ranks.

--impl reference times the fp64 CPU oracle on the host cores over a bounded
sample of the same workload (there is no upstream code to run).
"""
from __future__ import annotations

import argparse
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

import dn_inputs as di  # noqa: E402

METRIC = "tokens/s gated-delta chunk fwd (H=16,d=128,T=4096); decode GB/s; % roofline"
WORKLOAD = "gdn_prefill"
DECODE = "decode"
L2_BYTES = 126 * 1024 * 1024


def algorithmic_bytes(w: di.Workload) -> int:
    """HBM bytes one dn_chunk_fwd must move: read q, k, v, gates, S0; write o, S_T."""
    es = 2 if w.io == "bf16" else 4
    ntok = w.B * w.T * w.H
    b = ntok * (2 * w.dk + w.dv) * es + ntok * w.dv * es
    for mode, width in ((w.alpha, w.dk), (w.beta_k, w.dk), (w.beta_v, w.dv), (w.key_scale, w.dk)):
        if mode == di.GATE_SCALAR:
            b += ntok * 4
        elif mode == di.GATE_CHANNEL:
            b += ntok * width * 4
    sbytes = w.B * w.H * w.dk * w.dv * 4
    b += sbytes * (2 if w.s0_std > 0 else 1)
    return b


def chunk_flops(w: di.Workload, C: int = 64) -> int:
    """Executed flops of one dn_chunk_fwd in chunk form (2 per multiply-add), per head-token:
    2 C (3 d_k + 2 d_v) for the Gram, scores and WY products, 6 d_k d_v for the three state products
    (Wk S, Q S, W^T U) and C^2 / 3 for the triangular inverse."""
    return w.B * w.T * w.H * (2 * C * (3 * w.dk + 2 * w.dv) + 6 * w.dk * w.dv + C * C // 3)


def seq_flops(w: di.Workload) -> int:
    """Flops of the sequential evaluation (fp32 io): per head-token the decay, the two reductions S^T k and
    S^T q and the rank-1 update, 2 flops each over d_k d_v."""
    return w.B * w.T * w.H * 8 * w.dk * w.dv


def decode_bytes(w: di.Workload) -> int:
    """HBM bytes of one decode step: S read + written once, plus the token's vectors and o."""
    nh = w.B * w.H
    b = 2 * nh * w.dk * w.dv * 4
    b += nh * (2 * w.dk + w.dv) * 2 + nh * w.dv * 2
    b += nh * (w.dk + w.dk + w.dv) * 4  # alpha, beta_k, beta_v (channel)
    return b


def osdn_bytes(w: di.Workload) -> int:
    """HBM bytes the OSDN preconditioner scan must move: read k, beta, retention; write d and d_T."""
    es = 2 if w.io == "bf16" else 4
    ntok = w.B * w.T * w.H
    return ntok * w.dk * es + 2 * ntok * 4 + ntok * w.dk * 4 + w.B * w.H * w.dk * 4


def bwd_flops(w: di.Workload, C: int = 64) -> int:
    """Flops of one dn_chunk_bwd as its chunk algorithm states them (2 per multiply-add, every product
    counted in full, triangular ones included), per chunk of C tokens:
      9 C dk dv  (K+ S_m, W-^T U, W- dX, Q+^T dO, K+^T dV~, dO S_m^T, dV~ S_m^T, U dX^T, W-^T U for X)
      6 C^2 dk   (K+ W-^T, Q+ W-^T, dP W-, dL W-, dP^T Q+, dL^T K+)
      5 C^2 dv   (T R, P^T dO, T^T dU, dO U^T, dV~ U^T)
      C^3 / 6    (the unit-lower inverse)."""
    nc = (w.T + C - 1) // C
    per = 9 * C * w.dk * w.dv + 6 * C * C * w.dk + 5 * C * C * w.dv + C ** 3 // 6
    return 2 * per * nc * w.B * w.H


def reduce_max(value: float, world: int, device: str = "cuda") -> float:
    """Max over ranks of a per-rank time: the slowest rank sets a multi-rank step's time."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput when every rank processes `units_per_rank` in (max-over-ranks) `ms`."""
    return units_per_rank * world / (ms * 1e-3)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# sources each timed kernel is built from (its recorded DRAM traffic is void once any changes)
KERNEL_SOURCES = {
    "chunk_fwd": ["dn_split_sc.cu", "dn_sc_factors.cuh", "dn_ut_inverse.cuh", "dn_tc_ptx.cuh", "dn_tma.cu",
                  "dn_common.cuh"],
    "chunk_sc": ["dn_chunk_sc.cu", "dn_sc_factors.cuh", "dn_ut_inverse.cuh", "dn_tc_ptx.cuh", "dn_tma.cu",
                 "dn_common.cuh"],
    "chunk_tc": ["dn_chunk_tc.cu", "dn_ut_inverse.cuh", "dn_tc_ptx.cuh", "dn_tma.cu", "dn_common.cuh"],
    "decode": ["dn_decode.cu", "dn_common.cuh"],
    "osdn": ["dn_osdn.cu", "dn_tc_ptx.cuh", "dn_common.cuh"],
    "chunk_bwd": ["dn_bwd.cu", "dn_bwd.cuh", "dn_ut_inverse.cuh", "dn_tc_ptx.cuh", "dn_common.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_linear_attention_dn_b200", "csrc")
    for fn in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, entry: str = ""):
    """DRAM bytes per launch from the committed ncu summary (entry `entry`, default the kernel's own
    name), if taken on the current sources of `kernel`."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(entry or kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, interval_ms: int = 100):
        self.index = index
        self.interval_ms = interval_ms
        self.proc = None
        self.lines = []
        self.t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", str(self.interval_ms)],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample(w: di.Workload, x: dict, budget_s: float, nthreads: int, heads_cap: int = 10 ** 9):
    """Run the fp64 oracle over whole heads of `w` until ~budget_s of CPU work; returns
    (head_tokens, seconds, heads)."""
    import oracle
    allh = [(b, h) for b in range(w.B) for h in range(w.H)]
    done, t_total = 0, 0.0
    step = max(1, nthreads)
    while done < min(len(allh), heads_cap) and t_total < budget_s:
        batch = allh[done:done + step]
        t0 = time.perf_counter()
        oracle.fwd(**x, heads=batch, nthreads=nthreads)
        t_total += time.perf_counter() - t0
        done += len(batch)
    return done * w.T, t_total, done


def bench_config(world: int) -> dict:
    """The workload description both arms print (the reference arm times the oracle on it)."""
    w = di.WORKLOADS[WORKLOAD]
    alg = algorithmic_bytes(w)
    return {"workload": "gdn_prefill B=8 H=16 T=4096 d_k=d_v=128 bf16 q/k/v, scalar fp32 gates, chunk 64, S0=0",
            "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"dp{world}",
            "l2": f"inputs {alg / 1e6:.0f} MB per step > {L2_BYTES / 1e6:.0f} MB L2 (no flush)"}


def run_reference(args, rank: int, world: int):
    """CPU oracle arm: each step times the oracle on a bounded sample of the workload."""
    if rank != 0:
        return
    import oracle
    w = di.WORKLOADS[WORKLOAD]
    oracle.build()
    nthreads = oracle.max_threads()
    # a sample of whole heads: sequences are independent, so per-head cost is exact
    ws = w.scaled(B=1)
    x = di.make_inputs(ws)
    per_step_heads = max(1, nthreads)
    for _ in range(args.warmup):
        oracle.fwd(**x, heads=[(0, h % ws.H) for h in range(min(per_step_heads, ws.H))], nthreads=nthreads)
    times = []
    for s in range(args.steps):
        hs = [(0, h % ws.H) for h in range(min(per_step_heads, ws.H))]
        t0 = time.perf_counter()
        oracle.fwd(**x, heads=hs, nthreads=nthreads)
        times.append(time.perf_counter() - t0)
    nheads = min(per_step_heads, ws.H)
    tok_per_s = nheads * w.T / statistics.mean(times) / w.H  # sequence tokens (all H heads) per second
    line = {
        "impl": "reference", "metric": METRIC, "value": tok_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(world),
        "cpu_baseline": {"value": tok_per_s, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"{nheads} whole heads of T={w.T} per step (all heads are independent); "
                                   "tokens/s = head-tokens/s / H"},
        "e2e": {"value": tok_per_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_single_kernel(args):
    """Profiling mode: warm-up + timed launches of one kernel on a (smaller) batch of a workload.

    Used for the ncu captures summarised in profiles/: the same code path as the bench, with a
    batch that keeps the capture small while the inputs stay larger than L2."""
    import torch

    import gated_linear_attention_dn_b200 as dn
    from gated_linear_attention_dn_b200 import build as dnbuild

    if not os.path.exists(dnbuild.LIB):
        dnbuild.build()
    name = {"chunk": WORKLOAD, "decode": DECODE, "osdn": "osdn_phase1", "bwd": WORKLOAD, "kda": "kda",
            "fg2": "fg2_osdn_long", "mc": WORKLOAD}[args.only]
    w = di.WORKLOADS[name]
    if args.batch:
        w = w.scaled(B=args.batch)
    if args.seq:
        w = w.scaled(T=args.seq)
    x = di.make_osdn_inputs(w) if args.only == "osdn" else di.make_inputs(w)
    eta = x.pop("eta", None)

    def to_dev(a):
        if a is None:
            return None
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.cuda()

    xd = {n: to_dev(a) for n, a in x.items()}
    S = xd["S0"].clone() if xd.get("S0") is not None else None
    if args.only == "bwd":
        gb = {n: to_dev(a) for n, a in di.make_bwd_inputs(w).items()}
        desc = dn.make_desc(xd["q"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"])
        wsb = torch.empty(dn.dn_chunk_bwd_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
        gout = dn.dn_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                               xd["S0"], dO=gb["dO"], dS_T=gb["dS_T"], workspace=wsb)

    if args.only == "mc":
        # the Memory Caching read-out of the bench's leg: segments of 1024 tokens, their memories (the
        # chunked pass's S_T of each segment, computed once here), residual gates
        L = 1024
        nseg = w.T // L
        seg = lambda t: None if t is None else t.reshape(w.B * nseg, L, *t.shape[2:])
        Mc = torch.empty((w.B * nseg, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
        o_mc = torch.empty((w.B, w.T, w.H, w.dv), dtype=xd["q"].dtype, device="cuda")
        dn.dn_chunk_fwd(seg(xd["q"]), seg(xd["k"]), seg(xd["v"]), seg(xd["alpha"]), seg(xd["beta_k"]),
                        seg(xd["beta_v"]), seg(xd["key_scale"]), None, o=o_mc.view(w.B * nseg, L, w.H, w.dv), S_T=Mc)

    def launch():
        if args.only == "mc":
            dn.dn_mc_readout(xd["q"], Mc.view(w.B, nseg, w.H, w.dk, w.dv), None, o_mc, seg_len=L)
        elif args.only == "bwd":
            dn.dn_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"], dO=gb["dO"], dS_T=gb["dS_T"], workspace=wsb, out=gout)
        elif args.only == "osdn":
            dn.dn_osdn_precond(xd["k"], xd["beta"], xd["retention"], None, eta=eta)
        elif args.only in ("chunk", "kda", "fg2"):
            dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"])
        else:
            dn.dn_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"],
                              xd["key_scale"], S=S)

    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        launch()
    e1.record()
    torch.cuda.synchronize()
    if dn.dn_stream_status() != dn.DN_OK:
        raise RuntimeError("device status")
    print(json.dumps({"only": args.only, "workload": name, "batch": w.B, "seq": w.T, "steps": args.steps,
                      "ms_per_launch": e0.elapsed_time(e1) / max(1, args.steps)}))


# kernels per dn_chunk_fwd call of each configuration on a 148-SM B200: the chunk form in fp32 (three);
# kda's 128 sequences fill the GPU, so the fused per-channel kernel (one); fg2_osdn_long's 32 leave SMs
# idle, so the split evaluation (the chunk-parallel prep, then the chains: two)
CONFIG_KERNELS = {"gdn_fp32_small": 3, "kda": 1, "fg2_osdn_long": 2}

CONFIG_LEGS = {
    "gdn_fp32_small": "B=1 H=2 T=256 d_k=d_v=64 fp32 q/k/v, alpha~U(0.9,1) and beta per token, S0=0 "
                      "(chunk form in fp32: three kernels on split-TF32 warp tensor cores)",
    "kda": "B=4 H=32 T=8192 d_k=d_v=128 bf16 q/k/v, channel alpha, beta per token, S0~N(0,0.02^2) "
           "(fused per-channel kernel, one CTA per head)",
    "fg2_osdn_long": "B=2 H=16 T=32768 d_k=d_v=128 bf16 q/k/v, channel alpha, beta^k, beta^v, OSDN d, "
                     "S0~N(0,0.02^2) (split evaluation: chunk-parallel prep, then 64 chains of 64 columns)",
}


def time_chunk_lengths(w, xd, o, ST, stream, world, chunks, reps, flush=None):
    """ms per dn_chunk_fwd call for each chunk length in `chunks` on the same device inputs (each with
    its own workspace): 64 is the tensor-core kernels' tile; 16 and 32 run the chunk form in fp32."""
    import torch

    import gated_linear_attention_dn_b200 as dn
    out = {}
    for C in chunks:
        desc = dn.make_desc(xd["q"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], chunk=C)
        ws = torch.empty(max(dn.dn_chunk_fwd_workspace_bytes(desc), 16), dtype=torch.uint8, device="cuda")

        def call():
            dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"], o=o, S_T=ST, stream=stream, chunk=C, workspace=ws)

        for _ in range(3):
            call()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(reps):
            if flush is not None:
                flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        if dn.dn_stream_status(stream) != dn.DN_OK:
            raise RuntimeError(f"device status after chunk = {C}")
        out[str(C)] = reduce_max(tot / reps, world)
        del ws
    return out


def run_config_leg(name, peaks, stream, world, barrier, to_dev, want_cpu, reps):
    """One dn_chunk_fwd workload of the pages' configurations: ms per call, tokens/s, the HBM and tensor
    roofline fractions, and (rank 0, one GPU) the fp64 oracle on whole heads of the same workload."""
    import torch

    import gated_linear_attention_dn_b200 as dn
    w = di.WORKLOADS[name]
    x = di.make_inputs(w)
    xd = {n: to_dev(a) for n, a in x.items()}
    o = torch.empty((w.B, w.T, w.H, w.dv), dtype=xd["q"].dtype, device="cuda")
    ST = torch.empty((w.B, w.H, w.dk, w.dv), dtype=torch.float32, device="cuda")
    alg = algorithmic_bytes(w)
    # inputs smaller than L2 are timed one launch at a time with an L2 flush in between
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda") if alg < 2 * L2_BYTES else None

    def step():
        dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                        xd["S0"], o=o, S_T=ST, stream=stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    barrier()
    for e0, e1 in evs:
        if flush is not None:
            flush.zero_()
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    if dn.dn_stream_status(stream) != dn.DN_OK:
        raise RuntimeError(f"device status after the {name} leg")
    ms = reduce_max(statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs), world)
    gbs = alg / (ms * 1e-3) / 1e9
    leg = {"workload": f"{name}: {CONFIG_LEGS[name]}", "ms_per_call": ms, "kernels_per_call": CONFIG_KERNELS[name],
           "tokens_per_s": weak_scaling_rate(w.B * w.T, world, ms),
           "l2": "flushed (2 x L2 written) before every timed launch" if flush is not None
                 else f"inputs {alg / 1e6:.0f} MB per call > L2 (no flush)",
           "hbm": {"achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                   "algorithmic_bytes_per_launch": alg}}
    if w.io == "bf16":
        fl = chunk_flops(w)
        tf = fl / (ms * 1e-3) / 1e12
        leg["tensor"] = {"achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tf / peaks["bf16_tflops"], "executed_flops_per_launch": fl,
                         "peak_source": f"{peaks['source']} bf16 burst"}
        leg["roofline_time_us"] = 1e6 * max(alg / (peaks["hbm_gbs"] * 1e9), fl / (peaks["bf16_tflops"] * 1e12))
        leg["traffic"] = recorded_traffic("chunk_tc", f"chunk_tc:{name}")
    else:
        fl = seq_flops(w)
        tf = fl / (ms * 1e-3) / 1e12
        fp32_peak = 148 * 4 * 32 * 2 * 1.965e9 / 1e12
        leg["alu"] = {"achieved": tf, "peak": fp32_peak, "unit": "TFLOP/s", "frac": tf / fp32_peak,
                      "flops_per_launch": fl, "peak_source": "fp32 FFMA: 148 SMs x 128 lanes x 2 flops x 1.965 GHz",
                      "note": "4 chunks per head in sequence over 3 kernels: launch and latency bound at this size"}
    # the other chunk lengths: 16 and 32 in the chunk form in fp32 (all three for fp32 io)
    by_chunk = time_chunk_lengths(w, xd, o, ST, stream, world, (16, 32) if w.io == "f32" else (32,),
                                  reps=reps if w.io == "f32" else 2, flush=flush)
    by_chunk["64"] = ms
    leg["chunk_lengths"] = {"ms_per_call": by_chunk, "best": int(min(by_chunk, key=by_chunk.get)),
                            "note": "64: the default evaluation above; 16 and 32: the chunk form in fp32 "
                                    "(split-TF32 warp tensor cores) with that chunk length"}
    if want_cpu:
        import oracle
        oracle.build()
        nthreads = oracle.max_threads()
        head_tokens, secs, nheads = oracle_sample(w, x, budget_s=4.0, nthreads=nthreads)
        leg["cpu_baseline"] = {"value": head_tokens / secs / w.H, "unit": "tokens/s", "cores": nthreads,
                               "kind": "oracle",
                               "sample": f"{nheads} of {w.B * w.H} heads, whole T={w.T} each ({secs:.1f} s); "
                                         "tokens/s = head-tokens/s / H"}
    del xd, o, ST, flush
    return leg


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-osdn", action="store_true", help="skip the OSDN preconditioner scan leg")
    ap.add_argument("--no-mc", action="store_true", help="skip the Memory Caching leg")
    ap.add_argument("--no-bwd", action="store_true", help="skip the chunked backward leg")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the gdn_fp32_small, kda and fg2_osdn_long workload legs")
    ap.add_argument("--decode-steps", type=int, default=100)
    ap.add_argument("--only", choices=["chunk", "decode", "osdn", "bwd", "kda", "fg2", "mc"], default=None,
                    help="profiling mode: run just one kernel on the workload with batch --batch")
    ap.add_argument("--batch", type=int, default=0, help="with --only: batch size of the scaled workload")
    ap.add_argument("--seq", type=int, default=0, help="with --only: sequence length of the scaled workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.only:
        run_single_kernel(args)
        return

    import torch
    import torch.distributed as dist

    import gated_linear_attention_dn_b200 as dn
    from gated_linear_attention_dn_b200 import build as dnbuild

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    if not os.path.exists(dnbuild.LIB):
        dnbuild.build()
    dn.load()
    peaks = measured_peaks()

    w = di.WORKLOADS[WORKLOAD]
    x = di.make_inputs(w)

    def to_dev(a):
        if a is None:
            return None
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.cuda()

    xd = {n: to_dev(a) for n, a in x.items()}
    B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device="cuda")
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    # the split evaluation: transform kernel + state-chain kernel through a workspace allocated once
    desc_f = dn.make_desc(xd["q"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"])
    ws_f = torch.empty(max(1, dn.dn_chunk_fwd_workspace_bytes(desc_f)), dtype=torch.uint8, device="cuda")
    kernels_per_step = 2 if dn.dn_chunk_fwd_workspace_bytes(desc_f) else 1

    def step(workspace=ws_f):
        dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                        xd["S0"], o=o, S_T=ST, stream=stream, workspace=workspace)

    def barrier():
        if world > 1:
            dist.barrier()

    # clocks are sampled from before the warm-up to the end of the decode timing: the timed regions
    # alone are often shorter than one nvidia-smi sampling interval
    clocks = ClockSampler(local)
    clocks.__enter__()
    time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dn.dn_stream_status(stream) != dn.DN_OK:
        raise RuntimeError("device status after warm-up")

    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier()
    torch.cuda.synchronize()
    evs[0].record(stream)
    for i in range(args.steps):
        step()
        evs[i + 1].record(stream)
    torch.cuda.synchronize()
    barrier()
    per_launch_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    total_ms = evs[0].elapsed_time(evs[-1])
    if dn.dn_stream_status(stream) != dn.DN_OK:
        raise RuntimeError("device status after timed region")
    total_ms = reduce_max(total_ms, world)
    ms_per_step = total_ms / args.steps
    value = weak_scaling_rate(B * T * args.steps, world, total_ms)
    kern_ms = statistics.mean(per_launch_ms)
    alg = algorithmic_bytes(w)
    achieved = alg / (kern_ms * 1e-3) / 1e9
    fl = chunk_flops(w)
    tf = fl / (kern_ms * 1e-3) / 1e12
    # the fused evaluation (no workspace, one kernel per head) on the same inputs, for comparison
    for _ in range(3):
        step(False)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        step(False)
    f1.record(stream)
    torch.cuda.synchronize()
    if dn.dn_stream_status(stream) != dn.DN_OK:
        raise RuntimeError("device status after the fused evaluation")
    fused_ms = reduce_max(f0.elapsed_time(f1) / args.steps, world)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": recorded_traffic("chunk_fwd"),
                "peak_source": peaks["source"], "algorithmic_bytes_per_launch": alg,
                "kernel_ms": kern_ms,
                "tensor": {"achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                           "frac": tf / peaks["bf16_tflops"], "executed_flops_per_launch": fl},
                "roofline_time_us": 1e6 * max(alg / (peaks["hbm_gbs"] * 1e9), fl / (peaks["bf16_tflops"] * 1e12)),
                "scope": f"the whole dn_chunk_fwd call ({kernels_per_step} kernels: chunk-parallel transform, then "
                         "the state chain), CUDA events on the launching stream",
                "fused_ms": fused_ms, "fused_frac": alg / (fused_ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    # 32-token chunks on the same inputs (the chunk form in fp32; the tensor-core kernels' tile is 64)
    by_chunk = time_chunk_lengths(w, xd, o, ST, stream, world, (32,), reps=2)
    by_chunk["64"] = kern_ms
    roofline["chunk_lengths"] = {"ms_per_call": by_chunk, "best": int(min(by_chunk, key=by_chunk.get))}

    # ---- end to end: pinned host buffers, H2D of the step's inputs, D2H of o and S_T
    pin = {n: (None if t is None else t.cpu().pin_memory()) for n, t in xd.items()}
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    S_h = torch.empty(ST.shape, dtype=ST.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pin.values() if t is not None)
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size()

    # steps are pipelined as a serving loop would run them: step i's input copies (copy stream) overlap
    # step i - 1's kernels (compute stream) and step i - 2's read-back (read-back stream), through two
    # sets of device inputs and outputs; every step still copies its own inputs in and its o and S_T
    # out inside the timed region
    sets = [(xd, o, ST), ({n: (None if t is None else torch.empty_like(t)) for n, t in xd.items()},
                          torch.empty_like(o), torch.empty_like(ST))]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run_e2e(nsteps, e_start=None, e_end=None):
        done_k = [None, None]   # per set: kernels finished (its inputs may be overwritten)
        done_out = [None, None]  # per set: read-back finished (its outputs may be overwritten)
        if e_start is not None:
            e_start.record(s_in)
        for i in range(nsteps):
            xin, oo, SS = sets[i % 2]
            if done_k[i % 2] is not None:
                s_in.wait_event(done_k[i % 2])
            with torch.cuda.stream(s_in):
                for n, t in pin.items():
                    if t is not None:
                        xin[n].copy_(t, non_blocking=True)
            copied = torch.cuda.Event()
            copied.record(s_in)
            stream.wait_event(copied)
            if done_out[i % 2] is not None:
                stream.wait_event(done_out[i % 2])
            dn.dn_chunk_fwd(xin["q"], xin["k"], xin["v"], xin["alpha"], xin["beta_k"], xin["beta_v"],
                            xin["key_scale"], xin["S0"], o=oo, S_T=SS, stream=stream, workspace=ws_f)
            kdone = torch.cuda.Event()
            kdone.record(stream)
            done_k[i % 2] = kdone
            s_out.wait_event(kdone)
            with torch.cuda.stream(s_out):
                o_h.copy_(oo, non_blocking=True)
                S_h.copy_(SS, non_blocking=True)
            odone = torch.cuda.Event()
            odone.record(s_out)
            done_out[i % 2] = odone
        if e_end is not None:
            e_end.record(s_out)

    run_e2e(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_steps = max(3, min(args.steps, 10))
    barrier()
    torch.cuda.synchronize()
    run_e2e(e_steps, e0, e1)
    torch.cuda.synchronize()
    if dn.dn_stream_status(stream) != dn.DN_OK:
        raise RuntimeError("device status after the end-to-end leg")
    e_ms = reduce_max(e0.elapsed_time(e1), world)
    e2e = {"value": weak_scaling_rate(B * T * e_steps, world, e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "pipelining": "step i's input copies overlap step i-1's kernels and step i-2's read-back "
                         "(two device buffer sets, copy, compute and read-back streams)"}
    del pin, sets

    # ---- decode workload
    decode = None
    launches = kernels_per_step * args.steps
    launches += 2 * 3  # the two timed calls with 32-token chunks (three kernels each)
    if not args.no_decode:
        wd = di.WORKLOADS[DECODE]
        nd = args.decode_steps
        xs = [di.make_inputs(wd, step=s) for s in range(nd)]
        S = to_dev(xs[0]["S0"])
        steps_dev = [{n: to_dev(a) for n, a in xx.items() if n != "S0"} for xx in xs]
        del xs
        od = torch.empty((wd.B, 1, wd.H, wd.dv), dtype=torch.bfloat16, device="cuda")

        def dstep(s):
            z = steps_dev[s]
            dn.dn_decode_step(z["q"], z["k"], z["v"], z["alpha"], z["beta_k"], z["beta_v"], z["key_scale"],
                              S=S, o=od, stream=stream)

        for s in range(3):
            dstep(s)
        torch.cuda.synchronize()
        devs = [torch.cuda.Event(enable_timing=True) for _ in range(nd + 1)]
        barrier()
        devs[0].record(stream)
        for s in range(nd):
            dstep(s)
            devs[s + 1].record(stream)
        torch.cuda.synchronize()
        if dn.dn_stream_status(stream) != dn.DN_OK:
            raise RuntimeError("device status after decode")
        dms = [devs[i].elapsed_time(devs[i + 1]) for i in range(nd)]
        d_ms = reduce_max(statistics.mean(dms), world)
        db = decode_bytes(wd)
        gbs = db / (d_ms * 1e-3) / 1e9
        decode = {"workload": "decode 1024 seq x 32 heads, d=128, fp32 state 2 GiB in place, channel gates",
                  "steps": nd, "ms_per_step": d_ms, "tokens_per_s": weak_scaling_rate(wd.B, world, d_ms),
                  "GB/s": gbs * world,
                  "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": gbs / peaks["hbm_gbs"], "traffic": recorded_traffic("decode"),
                               "algorithmic_bytes_per_launch": db}}
        launches += nd
        del steps_dev, S

    # ---- OSDN phase 1 (the preconditioner scan), next to the chunked pass it feeds
    osdn = None
    if not args.no_osdn:
        wo = di.WORKLOADS["osdn_phase1"]
        xo = di.make_osdn_inputs(wo)
        ko, bo, ro = to_dev(xo["k"]), to_dev(xo["beta"]), to_dev(xo["retention"])
        do = torch.empty((wo.B, wo.T, wo.H, wo.dk), dtype=torch.float32, device="cuda")
        dTo = torch.empty((wo.B, wo.H, wo.dk), dtype=torch.float32, device="cuda")
        desc = dn.DnOsdnDesc(wo.B, wo.T, wo.H, wo.dk, dn.DN_BF16, xo["eta"])
        wso = torch.empty(dn.dn_osdn_precond_workspace_bytes(desc), dtype=torch.uint8, device="cuda")

        def ostep():
            dn.dn_osdn_precond(ko, bo, ro, None, eta=xo["eta"], d=do, d_T=dTo, workspace=wso, stream=stream)

        # the chunked pass over the same keys (fg2_osdn_long), with the scan's d as its key scale
        wf = di.WORKLOADS["fg2_osdn_long"]
        xf = {n: to_dev(a) for n, a in di.make_inputs(wf).items()}
        Sf = torch.empty((wf.B, wf.H, wf.dk, wf.dv), dtype=torch.float32, device="cuda")
        of = torch.empty((wf.B, wf.T, wf.H, wf.dv), dtype=torch.bfloat16, device="cuda")

        def fstep():
            dn.dn_chunk_fwd(xf["q"], xf["k"], xf["v"], xf["alpha"], xf["beta_k"], xf["beta_v"], do, xf["S0"],
                            o=of, S_T=Sf, stream=stream)

        def timed(fn, n):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            a0.record(stream)
            for _ in range(n):
                fn()
            a1.record(stream)
            torch.cuda.synchronize()
            return reduce_max(a0.elapsed_time(a1) / n, world)

        o_ms = timed(ostep, 10)
        f_ms = timed(fstep, 3)
        if dn.dn_stream_status(stream) != dn.DN_OK:
            raise RuntimeError("device status after the OSDN scan")
        ob = osdn_bytes(wo)
        ogbs = ob / (o_ms * 1e-3) / 1e9
        osdn = {"workload": "OSDN preconditioner scan, B=2 H=16 T=32768 d_k=128 (fg2_osdn_long's keys), "
                            "scalar beta, retention, eta=0.5",
                "ms_per_call": o_ms, "tokens_per_s": weak_scaling_rate(wo.B * wo.T, world, o_ms),
                "chunk_fwd_ms_same_keys": f_ms, "scan_over_chunk_fwd": o_ms / f_ms,
                "roofline": {"bound": "hbm", "achieved": ogbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": ogbs / peaks["hbm_gbs"], "traffic": recorded_traffic("osdn"),
                             "algorithmic_bytes_per_launch": ob}}
        launches += 2 * 10 + 3  # timed: 10 scans of two kernels, 3 chunked passes
        del ko, bo, ro, do, dTo, wso, xf, Sf, of

    # ---- the pages' other configurations, one dn_chunk_fwd workload each
    configs = None
    if not args.no_configs:
        configs = {}
        for name, reps in (("gdn_fp32_small", 20), ("kda", 10), ("fg2_osdn_long", 5)):
            configs[name] = run_config_leg(name, peaks, stream, world, barrier, to_dev,
                                           want_cpu=(rank == 0 and world == 1 and not args.no_cpu_baseline),
                                           reps=reps)
            launches += reps * CONFIG_KERNELS[name]
            # the timed calls with other chunk lengths (three kernels each)
            launches += 3 * (2 * reps if di.WORKLOADS[name].io == "f32" else 2)

    # ---- Memory Caching on the prefill workload: 4 segments of 1024 tokens, residual memory
    mc = None
    if not args.no_mc:
        L = 1024
        nseg = T // L
        Mc = torch.empty((B * nseg, H, dk, dv), dtype=torch.float32, device="cuda")

        def seg(t):
            return None if t is None else t.view(B * nseg, L, *t.shape[2:])

        def mc_online():
            dn.dn_chunk_fwd(seg(xd["q"]), seg(xd["k"]), seg(xd["v"]), seg(xd["alpha"]), seg(xd["beta_k"]),
                            seg(xd["beta_v"]), seg(xd["key_scale"]), None, o=o.view(B * nseg, L, H, dv),
                            S_T=Mc, stream=stream)

        def mc_read():
            dn.dn_mc_readout(xd["q"], Mc.view(B, nseg, H, dk, dv), None, o, seg_len=L, stream=stream)

        def timed2(fn, n):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            a0.record(stream)
            for _ in range(n):
                fn()
            a1.record(stream)
            torch.cuda.synchronize()
            return reduce_max(a0.elapsed_time(a1) / n, world)

        on_ms = timed2(mc_online, 10)
        rd_ms = timed2(mc_read, 10)
        if dn.dn_stream_status(stream) != dn.DN_OK:
            raise RuntimeError("device status after Memory Caching")
        # the read-out (tensor cores, bf16 io): the rows of the tokens past the first segment read q
        # once and read and write o once, and the memories 0 .. N-2 are read once; for the residual
        # memory each 128-token tile multiplies by the sum of the memories it reads, split bf16 hi +
        # lo: two M 128 x N d_v x K d_k products per tile
        later = B * H * (T - L)
        rd_bytes = later * (dk * 2 + 2 * dv * 2) + B * (nseg - 1) * H * dk * dv * 4
        flops = later * 2 * dk * dv * 2
        gbs = rd_bytes / (rd_ms * 1e-3) / 1e9
        tf = flops / (rd_ms * 1e-3) / 1e12
        mc = {"workload": "Memory Caching on gdn_prefill: 4 segments of 1024 tokens, residual memory",
              "online_ms": on_ms, "readout_ms": rd_ms, "total_ms": on_ms + rd_ms,
              "tokens_per_s": weak_scaling_rate(B * T, world, on_ms + rd_ms),
              "readout_roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                   "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                                   "peak_source": peaks["source"], "algorithmic_bytes_per_launch": rd_bytes,
                                   "tensor": {"achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                              "frac": tf / peaks["bf16_tflops"], "executed_flops_per_launch": flops}}}
        launches += 10 + 10
        del Mc

    # ---- chunked backward on the prefill workload (the training pass of the same recurrence)
    bwd = None
    if not args.no_bwd:
        gb = {n: to_dev(a) for n, a in di.make_bwd_inputs(w).items()}
        desc_b = dn.make_desc(xd["q"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"])
        wsb = torch.empty(dn.dn_chunk_bwd_workspace_bytes(desc_b), dtype=torch.uint8, device="cuda")
        gout = dn.dn_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                               xd["S0"], dO=gb["dO"], dS_T=gb["dS_T"], workspace=wsb, stream=stream)

        def bstep():
            dn.dn_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"], dO=gb["dO"], dS_T=gb["dS_T"], workspace=wsb, out=gout, stream=stream)

        for _ in range(3):
            bstep()
        torch.cuda.synchronize()
        nb = 5
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        b0.record(stream)
        for _ in range(nb):
            bstep()
        b1.record(stream)
        torch.cuda.synchronize()
        if dn.dn_stream_status(stream) != dn.DN_OK:
            raise RuntimeError("device status after the backward")
        b_ms = reduce_max(b0.elapsed_time(b1) / nb, world)
        fl = bwd_flops(w)
        tf32_peak = peaks["bf16_tflops"] * 1.1 / 2.25  # nominal dense tf32 : bf16 ratio
        btf = fl / (b_ms * 1e-3) / 1e12
        bwd = {"workload": "chunked backward of gdn_prefill (B=8 H=16 T=4096 d=128 bf16, scalar gates); "
                           "dO ~ N(0,1) bf16, dS_T ~ N(0,0.1^2)",
               "ms_per_call": b_ms, "tokens_per_s": weak_scaling_rate(B * T, world, b_ms),
               "fwd_ms": kern_ms, "bwd_over_fwd": b_ms / kern_ms, "kernels_per_call": 4,
               "roofline": {"bound": "tensor", "achieved": btf, "peak": tf32_peak, "unit": "TFLOP/s",
                            "frac": btf / tf32_peak, "traffic": recorded_traffic("chunk_bwd"),
                            "peak_source": f"{peaks['source']} bf16 x 1.1/2.25 (dense tf32 : bf16)",
                            "scope": "the whole call (4 kernels); flops as bwd_flops counts them",
                            "algorithmic_flops_per_launch": fl}}
        launches += 4 * nb
        del gb, wsb, gout

    clocks.__exit__(None, None, None)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        nthreads = oracle.max_threads()
        head_tokens, secs, nheads = oracle_sample(w, x, budget_s=12.0, nthreads=nthreads)
        cpu = {"value": head_tokens / secs / w.H, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
               "sample": f"{nheads} of {w.B * w.H} heads of the same workload, whole T={w.T} each "
                         f"({secs:.1f} s); tokens/s = head-tokens/s / H"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(world),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "clocks": clocks.summary(), "gpu_launches": launches, "decode": decode, "osdn_phase1": osdn,
            "memory_caching": mc, "chunk_bwd": bwd, "configs": configs,
            "kernel_source": {k: kernel_source_hash(k) for k in KERNEL_SOURCES},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
