#!/usr/bin/env python
"""Benchmark of the Gated Delta Rule chunked forward on B200.

One step = one forward pass (chunk table, intra-chunk, state pass, output)
over the one-layer prefill workload: B = 1, T = 32768 tokens,
Nqk = 16, Nv = 32, Dk = Dv = 128, L = 128, bf16 q/k/v/beta, fp32 g, inputs
already resident in HBM.  Every rank of a multi-GPU run processes its own
batch (independent problems, weak scaling, no collective on the data path).

FLOPs per token (dense tensor-core work, counted once per qk-head where the
product is shared by the v-heads of a group):
    F = Nv (4 L Dv + 2 L Dk + 6 Dk Dv) + Nqk (4 L Dk)    (= 7,340,032 at this size)
i.e. per chunk and v-head: U = T (beta V), W = T (beta e^gamma K), W S, Q S,
P U', K^T U'; per chunk and qk-head: K K^T and Q K^T.  The triangular solve
and the masked halves are not counted.

Two HBM-bound side workloads are timed in the same run (skipped with
--no-short) and reported in the same line: ``short_seq`` (256 sequences of
1..8 tokens from an fp32 state pool, gdn_chunk_fwd's fused short path) and
``spec_decode`` (256 sequences of 4 draft tokens, a pool slot per token,
gdn_recurrent_fwd updating the pool in place) and ``decode_bf16`` /
``decode_bf16_dk64_dv512`` (one token per sequence on a bf16 pool with the
key-dimension gate, at Dk = Dv = 128 and at the decode page's Dk = 64, Dv = 512).

Prints ONE JSON line (rank 0).  ``--impl reference`` times the fp64 CPU
oracle (the reference arm) on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_linear_17_b200 import dist as gdist  # noqa: E402
from gated_deltanet_linear_17_b200 import inputs  # noqa: E402

METRIC = "GDN fwd tokens/s @Nv32 D128 S32K; % bf16 TC roofline; short-seq HBM GB/s"
WORKLOAD = "prefill_s32k"
L = D = 128


def flops_per_token(Nqk, Nv):
    return Nv * (4 * L * D + 2 * L * D + 6 * D * D) + Nqk * (4 * L * D)


def stage_work(T, Nqk, Nv, NC, B, B_init=0):
    """Algorithmic work of one launch of each kernel: {kernel: (FLOP, HBM bytes)}.

    Both follow the operator's own counts, not this implementation's data flow.
    FLOP: the kernel's share of the dense products of the chunked form (the
    per-token formula above, split by the kernel that computes each product):
      intra  U = T (beta V), W = T (beta e^gamma K) per v-head, K K^T per qk-head
      state  W S and K~^T U' per v-head
      output Q S and P U' per v-head, Q K^T per qk-head
    Bytes: the operator inputs and outputs the kernel reads or writes (q, k, v,
    g, beta, out, initial and final state), each once; the per-chunk tiles this
    implementation passes between its kernels (U, W, Mk, S_c and the factor
    records) are not algorithmic and are not counted:
      intra  k, v, g, beta;  state  k, g, the initial and the final states;
      output q, k, g, out."""
    qk, v, g, beta = T * Nqk * D * 2, T * Nv * D * 2, T * Nv * 4, T * Nv * 2
    states = (B_init + B) * Nv * D * D * 4
    return {
        "chunk_map": (0.0, 4.0 * (B + 1)),
        "intra": (T * (Nv * (2 * L * D + 2 * L * D) + Nqk * 2 * L * D), qk + v + g + beta),
        "state": (T * Nv * 4 * D * D, qk + g + states),
        "output": (T * (Nv * (2 * D * D + 2 * L * D) + Nqk * 2 * L * D), 2 * qk + g + v),
    }


def step_bytes(T, Nqk, Nv, B, B_init=0):
    """Algorithmic HBM bytes of one whole forward pass: every input read once, every output written once."""
    return T * (2 * Nqk * D * 2 + Nv * D * 2 + Nv * 4 + Nv * 2 + Nv * D * 2) + (B_init + B) * Nv * D * D * 4


def roofline_of(flop, nbytes, sec, peaks):
    """The roofline that binds (the larger time at peak) and the fraction achieved on it; the other
    side's fraction is reported beside it."""
    t_tc = flop / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    tc = {"achieved": flop / sec / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
          "frac": flop / sec / 1e12 / peaks["bf16_tflops"], "per_launch": f"{flop:.4g} FLOP per launch"}
    hbm = {"achieved": nbytes / sec / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
           "frac": nbytes / sec / 1e9 / peaks["hbm_gbs"], "per_launch": f"{nbytes:.4g} bytes per launch"}
    if t_hbm >= t_tc:
        return {"bound": "hbm", **hbm, "other": {"bound": "tensor", "frac": tc["frac"]}}
    return {"bound": "tensor", **tc, "other": {"bound": "hbm", "frac": hbm["frac"]}}


def measured_traffic(kernel, units):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, scaled from the
    captured workload to `units` (chunk, v-head) pairs; None when there is no capture or
    the kernel's source has changed since it was taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, "gated_deltanet_linear_17_b200", "csrc", rec["source"])
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
            return None
    return rec["dram_bytes_per_launch"] * units / rec["units"]


def short_bytes(inp):
    """HBM bytes of the short-sequence pass: state read + write plus per-token I/O."""
    per_tok = 2 * inp.Nqk * D * 2 + inp.Nv * D * 2 + inp.Nv * 4 + inp.Nv * 2 + inp.Nv * D * 2
    return 2 * inp.B * inp.Nv * D * D * 4 + inp.T * per_tok


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            uuid = str(device_index)
        self.target = uuid

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="gdn_clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.target, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx = float(parts[1])
                except ValueError:
                    continue
                for n, v in zip(names, parts[3:7]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def cpu_oracle_sample(inp, tokens):
    """Time the fp64 oracle on the first `tokens` tokens of a one-sequence batch (all v-heads)."""
    import oracle
    n = min(tokens, inp.T)
    t0 = time.perf_counter()
    _, _, threads = oracle.recurrent(inp.q[:n], inp.k[:n], inp.v[:n], inp.g[:n], inp.beta[:n],
                                     torch.tensor([0, n], dtype=torch.int32), None, None,
                                     scale=inp.scale, eps=inp.eps, return_threads=True)
    dt = time.perf_counter() - t0
    return n / dt, threads, dt, n


def run_reference(args, rank, world):
    """The reference arm: the fp64 CPU oracle, timed as it stands on the host cores."""
    if rank != 0:
        return 0
    inp = inputs.config(WORKLOAD)
    tok = args.ref_tokens
    for _ in range(args.warmup):
        cpu_oracle_sample(inp, min(tok, 256))
    t0 = time.perf_counter()
    threads = 0
    for _ in range(args.steps):
        _, threads, _, n = cpu_oracle_sample(inp, tok)
    dt = time.perf_counter() - t0
    value = args.steps * n / dt
    sample = f"first {n} tokens of the {inp.T}-token sequence, all {inp.Nv} v-heads, per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(inp),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(inp):
    return {"workload": f"{WORKLOAD}: one-layer prefill, B={inp.B} T={inp.T} Nqk={inp.Nqk} Nv={inp.Nv} "
                        f"D=128 L=128", "B": inp.B, "T": inp.T, "Nqk": inp.Nqk, "Nv": inp.Nv, "D": 128, "L": 128,
            "flop_per_token": flops_per_token(inp.Nqk, inp.Nv),
            "l2": "inputs larger than L2 (q, k, v, out = 805 MB per step; no flush)",
            "parallelism": "independent batch per GPU (weak scaling, no data-path collective)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=8192, help="tokens of the CPU-oracle baseline sample")
    ap.add_argument("--ref-tokens", type=int, default=2048, help="tokens per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-short", action="store_true")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override the prefill length (profiling on a smaller case; not a bench line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        rank, _, world = gdist.env_rank()
        return run_reference(args, rank, world)

    import gated_deltanet_linear_17_b200 as gdn
    rank, local, world = gdist.init("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()

    if args.seq_len:
        rec = dict(inputs.CONFIGS[WORKLOAD])
        rec["lens"] = [args.seq_len]
        rec["seed"] += rank
        host = inputs.make(name=f"{WORKLOAD}@{args.seq_len}", **rec)
    else:
        host = inputs.config(WORKLOAD, seed=inputs.CONFIGS[WORKLOAD]["seed"] + rank)
    inp = host.to(dev)
    T, B, Nqk, Nv = inp.T, inp.B, inp.Nqk, inp.Nv
    st = gdn.Stages(T, B, Nqk, Nv, dev)
    out = torch.empty(T, Nv, D, dtype=torch.bfloat16, device=dev)
    fin = torch.empty(B, Nv, D, D, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    names = ["chunk_map", "intra", "state", "output"]

    ws = torch.empty(gdn.workspace_bytes(T, B, Nqk, Nv), dtype=torch.uint8, device=dev)

    def step():  # the public call: chunk ranges pipelined over the library's streams
        gdn.chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.state_pool, inp.state_indices,
                      scale=inp.scale, eps=inp.eps, out=out, final_state=fin, workspace=ws)

    def staged(evs=None):  # the same kernels one after another, timed one by one
        calls = [lambda: st.chunk_map(inp.cu_seqlens),
                 lambda: st.intra(inp.k, inp.v, inp.g, inp.beta, inp.eps),
                 lambda: st.state(inp.k, inp.state_pool, inp.state_indices, fin),
                 lambda: st.output(inp.q, inp.k, inp.g, out, inp.scale, inp.eps)]
        for i, c in enumerate(calls):
            if evs is not None:
                evs[i].record(stream)
            c()
        if evs is not None:
            evs[len(calls)].record(stream)

    for _ in range(args.warmup):
        step()
        staged()
    torch.cuda.synchronize()

    # timed region 1: the forward pass through the public call (the metric)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local) if rank == 0 else None
    if clk:
        clk.start()
    gdist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    gdist.barrier()
    clocks = clk.stop() if clk else None
    total_ms = t0.elapsed_time(t1)

    # timed region 2: the same kernels staged one by one, each between events (per-kernel roofline)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    gdist.barrier()
    torch.cuda.synchronize()
    for k in range(args.steps):
        staged(evs[k])
    torch.cuda.synchronize()
    gdist.barrier()
    stage_ms = {n: sum(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps)) / args.steps
                for i, n in enumerate(names)}
    staged_ms = sum(stage_ms.values())
    ms = gdist.max_over_ranks(total_ms / args.steps, device=dev)
    value = world * T / (ms / 1e3)
    F = flops_per_token(Nqk, Nv)
    tc_frac = F * T / (ms / 1e3) / (peaks["bf16_tflops"] * 1e12)

    nchunks = sum((n + L - 1) // L for n in inp.seqlens)
    b_init = inp.B if inp.state_pool is not None else 0
    work = stage_work(T, Nqk, Nv, nchunks, inp.B, b_init)
    dom = max(names, key=lambda n: stage_ms[n])
    units = nchunks * Nv  # (chunk, v-head) pairs, the CTAs of the intra and output kernels
    traffic = measured_traffic(f"{dom}_kernel", units)
    roofline = {"kernel": dom, **roofline_of(*work[dom], stage_ms[dom] / 1e3, peaks), "traffic": traffic,
                "traffic_over_algorithmic": None if traffic is None else traffic / work[dom][1],
                "peak_source": f"{peaks['source']} (burst bf16 / STREAM copy)",
                "work": "FLOP and bytes of the operator's chunked form (see stage_work), no intermediate tiles"}
    stage_roofline = {n: {"bound": r["bound"], "frac": round(r["frac"], 4), "other_frac": round(r["other"]["frac"], 4)}
                      for n in names if n != "chunk_map"
                      for r in [roofline_of(*work[n], stage_ms[n] / 1e3, peaks)]}
    # the whole forward pass: the headline fraction of the tensor roofline, and the HBM side
    sbytes = step_bytes(T, Nqk, Nv, inp.B, b_init)
    step_traffic = [measured_traffic(f"{n}_kernel", units) for n in ("intra", "state", "output")]
    step_roofline = {"tc_frac": tc_frac, "flop": F * T, "bytes": sbytes,
                     "hbm_frac": sbytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "floor_ms": 1e3 * max(F * T / (peaks["bf16_tflops"] * 1e12), sbytes / (peaks["hbm_gbs"] * 1e9)),
                     "dram_traffic": None if None in step_traffic else sum(step_traffic),
                     "traffic_over_algorithmic": None if None in step_traffic else sum(step_traffic) / sbytes}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; see inputs.CONFIGS)",
            "config": workload_config(inp), "tc_frac": tc_frac, "step_roofline": step_roofline,
            "stages_ms": {n: round(v, 5) for n, v in stage_ms.items()}, "roofline": roofline,
            "stage_roofline": stage_roofline,
            "staged_ms_per_step": staged_ms, "pipeline_ranges": gdn.pipeline_ranges(T, B),
            "gpu_launches": (1 + 3 * gdn.pipeline_ranges(T, B)) * args.steps, "clocks": clocks}

    # ---- the same prefill under the LinearAttention page's other update rules (gdn_chunk_fwd_rule)
    rule_lines = {}
    for rule in ("delta", "gated", "linear"):
        def rstep():
            gdn.chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.cu_seqlens, inp.state_pool, inp.state_indices,
                          scale=inp.scale, eps=inp.eps, out=out, final_state=fin, workspace=ws, update_rule=rule)
        for _ in range(args.warmup):
            rstep()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            rstep()
        e1.record(stream)
        torch.cuda.synchronize()
        rms_ = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device=dev)
        rule_lines[rule] = {"ms_per_step": rms_, "tokens/s": world * T / (rms_ / 1e3)}
        line["gpu_launches"] += (1 + 3 * gdn.pipeline_ranges(T, B, inp.Nqk, inp.Nv)) * args.steps
    line["prefill_update_rules"] = rule_lines

    # ---- short-sequence state-pool pass (HBM-bound)
    if not args.no_short:
        sh = inputs.config("short_pool_b256", seed=inputs.CONFIGS["short_pool_b256"]["seed"] + rank).to(dev)
        so = torch.empty(sh.T, sh.Nv, D, dtype=torch.bfloat16, device=dev)
        sf = torch.empty(sh.B, sh.Nv, D, D, dtype=torch.float32, device=dev)
        ms_len = sh.max_seqlen

        def sstep():
            gdn.chunk_fwd(sh.q, sh.k, sh.v, sh.g, sh.beta, sh.cu_seqlens, sh.state_pool, sh.state_indices,
                          scale=sh.scale, eps=sh.eps, max_seqlen=ms_len, out=so, final_state=sf)
        for _ in range(args.warmup):
            sstep()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            sstep()
        e1.record(stream)
        torch.cuda.synchronize()
        sms = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device=dev)
        nb = short_bytes(sh)
        gbs = nb / (sms / 1e3) / 1e9
        line["short_seq"] = {"workload": f"short_pool_b256: B={sh.B} lens 1..8 (T={sh.T}), Nqk={sh.Nqk}, "
                                         f"Nv={sh.Nv}, fp32 pool [512,{sh.Nv},128,128]",
                             "ms": sms, "bytes": nb, "GB/s": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
                             "tokens/s": world * sh.T / (sms / 1e3), "kernel": "short_kernel",
                             "l2": "state traffic 1.07 GB per step > L2"}
        line["gpu_launches"] += args.steps
        del sh, so, sf

        # speculative decoding on a pool updated in place (one slot per token; HBM-bound)
        cfg = inputs.CONFIGS["spec_decode_b256x4"]
        sp = inputs.config("spec_decode_b256x4", seed=cfg["seed"] + rank)
        slots, acc = inputs.spec_slots(sp, seed=cfg["seed"] + 100 + rank)
        sp, slots, acc = sp.to(dev), slots.to(dev), acc.to(dev)
        spo = torch.empty(sp.T, sp.Nv, D, dtype=torch.bfloat16, device=dev)

        def pstep():
            gdn.recurrent_fwd(sp.q, sp.k, sp.v, sp.g, sp.beta, sp.cu_seqlens, sp.state_pool, slots,
                              num_accepted=acc, scale=sp.scale, eps=sp.eps, max_seqlen=sp.max_seqlen, out=spo)
        for _ in range(args.warmup):
            pstep()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            pstep()
        e1.record(stream)
        torch.cuda.synchronize()
        pms = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device=dev)
        sbytes = sp.Nv * D * D * 4
        pb = sp.B * sbytes + sp.T * sbytes + (short_bytes(sp) - 2 * sp.B * sbytes)  # starts, per-token states, I/O
        line["spec_decode"] = {"workload": f"spec_decode_b256x4: B={sp.B} x 4 draft tokens (T={sp.T}), Nqk={sp.Nqk}, "
                                           f"Nv={sp.Nv}, a pool slot per token, accepted counts uniform 1..4, "
                                           f"fp32 pool [{sp.state_pool.shape[0]},{sp.Nv},128,128] updated in place",
                               "ms": pms, "bytes": pb, "GB/s": pb / (pms / 1e3) / 1e9,
                               "hbm_frac": pb / (pms / 1e3) / 1e9 / peaks["hbm_gbs"],
                               "tokens/s": world * sp.T / (pms / 1e3), "kernel": "short_kernel (per-token slots)",
                               "call": "gdn_recurrent_fwd"}
        # the same workload under each update rule of the LinearAttention page (GB/s counts the same bytes)
        rules = {}
        for rule in ("gated_delta", "delta", "gated", "linear"):
            decay, delta = rule in ("gated_delta", "gated"), rule in ("gated_delta", "delta")

            def rstep():
                gdn.recurrent_fwd(sp.q, sp.k, sp.v, sp.g if decay else None, sp.beta if delta else None,
                                  sp.cu_seqlens, sp.state_pool, slots, num_accepted=acc, scale=sp.scale, eps=sp.eps,
                                  update_rule=rule, max_seqlen=sp.max_seqlen, out=spo)
            for _ in range(args.warmup):
                rstep()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                rstep()
            e1.record(stream)
            torch.cuda.synchronize()
            rms_ = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device=dev)
            rules[rule] = {"ms": rms_, "hbm_frac": pb / (rms_ / 1e3) / 1e9 / peaks["hbm_gbs"]}
            line["gpu_launches"] += args.steps
        line["spec_decode"]["update_rules"] = rules
        line["gpu_launches"] += args.steps
        del sp, slots, acc, spo

        # one decode step on a bf16 pool with the key-dimension gate (the decode page's operator), at the
        # bench's head size and at the page's example shape
        def decode_line(name):
            cfg = inputs.CONFIGS[name]
            dc = inputs.config(name, seed=cfg["seed"] + rank)
            dgk = inputs.key_gate(dc, seed=cfg["seed"] + 200 + rank).to(dev)
            dslots = dc.state_indices.clone().to(dev)  # one token per sequence: its slot is the sequence's
            dc = dc.to(dev)
            dpool = dc.state_pool.to(torch.bfloat16)
            Dk, Dv = dc.q.shape[2], dc.v.shape[2]
            dco = torch.empty(dc.T, dc.Nv, Dv, dtype=torch.bfloat16, device=dev)

            def dstep():
                gdn.recurrent_fwd(dc.q, dc.k, dc.v, dc.g, dc.beta, dc.cu_seqlens, dpool, dslots, scale=dc.scale,
                                  eps=dc.eps, gk=dgk, max_seqlen=1, out=dco)
            for _ in range(args.warmup):
                dstep()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                dstep()
            e1.record(stream)
            torch.cuda.synchronize()
            dms = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device=dev)
            per_tok = 2 * dc.Nqk * Dk * 2 + dc.Nv * Dv * 2 + dc.Nv * 4 + dc.Nv * 2 + dc.Nv * Dv * 2 + dc.Nv * Dk * 4
            db = 2 * dc.B * dc.Nv * Dk * Dv * 2 + dc.T * per_tok  # bf16 states in and out, token I/O with gk
            line["gpu_launches"] += args.steps
            return {"workload": f"{name}: B={dc.B} x 1 token, Nqk={dc.Nqk}, Nv={dc.Nv}, Dk={Dk}, Dv={Dv}, bf16 pool "
                                f"[{dpool.shape[0]},{dc.Nv},{Dk},{Dv}] updated in place, key gate gk",
                    "ms": dms, "bytes": db, "GB/s": db / (dms / 1e3) / 1e9,
                    "hbm_frac": db / (dms / 1e3) / 1e9 / peaks["hbm_gbs"], "tokens/s": world * dc.T / (dms / 1e3),
                    "kernel": "short_kernel (slots, gk, bf16 pool)", "call": "gdn_recurrent_fwd"}
        line["decode_bf16"] = decode_line("decode_b256_bf16")
        line["decode_bf16_dk64_dv512"] = decode_line("decode_dk64_dv512")

        # a state window of the LinearAttention page (gdn_recurrent_window_fwd): 256 sequences of 2 tokens, W = 4
        W = 4
        wc = inputs.make([2] * 256, Nqk=16, Nv=32, g=("uniform_neg", 1.0, 0.01), seed=8 + rank, name="window")
        wgen = torch.Generator(device=dev).manual_seed(9 + rank)
        win = torch.randn(W, wc.B, wc.Nv, D, D, device=dev, generator=wgen) * 0.02
        wc = wc.to(dev)
        wo = torch.empty(wc.T, wc.Nv, D, dtype=torch.bfloat16, device=dev)

        def wstep():
            gdn.recurrent_window_fwd(wc.q, wc.k, wc.v, wc.g, wc.beta, wc.cu_seqlens, win, W, scale=wc.scale,
                                     eps=wc.eps, max_seqlen=2, out=wo)
        for _ in range(args.warmup):
            wstep()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            wstep()
        e1.record(stream)
        torch.cuda.synchronize()
        wms = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device=dev)
        sb = wc.Nv * D * D * 4
        # per sequence: the shift reads entries 2, 3 and writes 0, 1; the recurrence reads entry 3 and writes 2, 3
        wb = wc.B * 7 * sb + (short_bytes(wc) - 2 * wc.B * sb)
        line["state_window"] = {"workload": f"window_b256_w{W}: B={wc.B} x 2 tokens, Nqk={wc.Nqk}, Nv={wc.Nv}, "
                                            f"fp32 window [{W},{wc.B},{wc.Nv},128,128] updated in place",
                                "ms": wms, "bytes": wb, "GB/s": wb / (wms / 1e3) / 1e9,
                                "hbm_frac": wb / (wms / 1e3) / 1e9 / peaks["hbm_gbs"],
                                "tokens/s": world * wc.T / (wms / 1e3),
                                "kernel": "window_shift_kernel + short_kernel (window slots)",
                                "call": "gdn_recurrent_window_fwd"}
        line["gpu_launches"] += 2 * args.steps
        del win, wc, wo

    # ---- end to end from pinned host buffers through the public call
    if not args.no_e2e:
        pin = lambda t: None if t is None else t.pin_memory()
        hq, hk, hv, hg, hb, hc = (pin(getattr(host, n)) for n in ("q", "k", "v", "g", "beta", "cu_seqlens"))
        oh = torch.empty(T, Nv, D, dtype=torch.bfloat16, pin_memory=True)
        fh = torch.empty(B, Nv, D, D, dtype=torch.float32, pin_memory=True)
        del st, ws  # the host entry brings its own device buffer
        dbuf = torch.empty(gdn.host_buffer_bytes(hc, Nqk, Nv, False), dtype=torch.uint8, device=dev)
        plan = gdn.host_plan(hc)
        for _ in range(max(1, args.warmup // 2)):
            gdn.chunk_fwd_host(hq, hk, hv, hg, hb, hc, scale=host.scale, eps=host.eps, device=dev,
                               out_host=oh, final_host=fh, device_buffer=dbuf)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        gdist.barrier()
        e0.record(stream)
        h2d = d2h = 0
        for _ in range(args.steps):
            _, _, h2d, d2h = gdn.chunk_fwd_host(hq, hk, hv, hg, hb, hc, scale=host.scale, eps=host.eps, device=dev,
                                                out_host=oh, final_host=fh, device_buffer=dbuf)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = gdist.max_over_ranks(e0.elapsed_time(e1) / args.steps, device=dev)
        line["e2e"] = {"value": world * T / (ems / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": ems,
                       "call": f"gdn_chunk_fwd_host from pinned host buffers, {len(plan)} pieces, uploads and "
                               f"downloads overlapped with the compute",
                       "h2d_GB/s": h2d / (ems / 1e3) / 1e9, "d2h_GB/s": d2h / (ems / 1e3) / 1e9}
        # per piece: the cu kernel, one chunk table, the pipelined kernels and the status fold
        line["gpu_launches"] += args.steps * sum(3 + 3 * gdn.pipeline_ranges(r[4] - r[3], r[2], Nqk, Nv)
                                                 for r in plan)

    # ---- CPU oracle baseline (rank 0, one GPU only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, threads, dt, n = cpu_oracle_sample(host, args.cpu_tokens)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": f"first {n} of {T} tokens, all {Nv} v-heads ({dt:.1f} s wall)"}

    if rank == 0:
        print(json.dumps(line), flush=True)
    if torch.distributed.is_initialized():
        gdist.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
