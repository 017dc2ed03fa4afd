#!/usr/bin/env python
"""Benchmark of the B200 Gated Delta Rule-2 mixer.

One step = gdr2_chunk_fwd_train + gdr2_chunk_bwd_saved (forward keeping its per-chunk intermediates,
then the backward reading them) over one batch of the training-shaped workload
(B=8, H=16, dk=dv=128, T=4096, C=64, bf16 operands, fp32 state), inputs resident in HBM. The
decode step (256 sequences x 16 heads, fp32 state, 100 consecutive tokens) is timed after it and
reported in the same JSON line under "decode".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun). Every rank runs its own batch (independent sequences:
the mixer has no cross-sequence term), so per-GPU work is fixed ("weak" scaling) and there is no
collective on the data path; the only collectives are the barriers and the max-over-ranks timing.
`--impl reference` times the fp64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import glob
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GDR-2 fwd+bwd tokens/s @H=16,d=128,T=4K; % of roofline; decode tok/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}

# Algorithmic work per token-head (d = dk = dv = 128, C = 64, bf16 operands, fp32 log-decay/state):
# forward reads q,k,v,b,w (5 x 256 B) + log_alpha (512 B), writes o (256 B), plus the amortised
# initial/final state; backward reads the same plus dO and writes dq,dk,dv,db,dw (bf16) + dlog_alpha
# (fp32). Lower-triangular C x C products counted at half.
FWD_BYTES_PER_TH = 2080
BWD_BYTES_PER_TH = 3888
FWD_FLOP_PER_TH = 5 * 64 * 128 + 6 * 128 * 128 + 64 * 64 // 3
BWD_FLOP_PER_TH = 16 * 128 * 128 + 14 * 64 * 128 + 4 * 64 * 64 // 3 + 64 * 64 // 3
DECODE_BYTES_PER_SEQHEAD = 2 * 128 * 128 * 4 + 2048


def reduce_max(x, device="cuda"):
    """Max of a float over all ranks of the default process group (the value itself when single-rank)."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(base_seed, rank):
    """Each rank draws its own independent batch (weak scaling: no data shared between ranks)."""
    return base_seed + 7919 * rank


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


# Source files each kernel family is compiled from (its .cu file and the headers it includes). A DRAM traffic
# record in profiles/traffic.json holds for a kernel while the digest of these files matches the one stored
# with the capture.
KERNEL_SOURCES = {
    "chain_": ["chain_tc.cu", "common.cuh", "kernels.h", "tc.cuh", "tma_host.h", "status.cuh"],
    "tc_": ["chunk_tc.cu", "common.cuh", "kernels.h", "tc.cuh", "tma_host.h", "status.cuh"],
}


def source_digest(kernel=None):
    """Digest of the sources of `kernel` (by name prefix), or of every library source when none is given or
    the kernel has no entry in KERNEL_SOURCES."""
    csrc = os.path.join(ROOT, "gated_delta_rule_65_b200", "csrc")
    files = None
    for prefix, names in KERNEL_SOURCES.items():
        if kernel is not None and kernel.startswith(prefix):
            files = [os.path.join(csrc, n) for n in names]
    if files is None:
        files = sorted(f for f in glob.glob(os.path.join(csrc, "**", "*"), recursive=True) if os.path.isfile(f))
    h = hashlib.sha256()
    for f in files:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------------------------------------------
# per-kernel compulsory traffic (bytes per launch), keyed by the kernel names the library reports.
# Each entry counts every tensor the kernel must read or write once at its stored width.
def kernel_bytes(name, B, T, H, dk, dv, eb):
    C = 64
    NT = (T + C - 1) // C
    nch = B * H * NT
    tok = B * T * H
    KB = 1024
    ck, cv, cc, ss = C * dk * 4, C * dv * 4, C * C * 4, dk * dv * 4
    if name == "decode":
        return B * H * (2 * dk * dv * 4 + (3 * dk + 3 * dv) * eb + dk * 4)
    # tensor-core path (dk = dv = 128): bytes per chunk read + written once. Operand images are hi + lo
    # bf16 pairs (the same bytes as fp32).
    inputs = 5 * 16 * KB + 32 * KB                       # q, k, b, v, w (bf16) + log_alpha (fp32)
    fwd_ws = 3 * 32 * KB + 16 * KB + 32 * KB + 512       # Y, Q_gamma, K_tail, A_qk images; U; gamma_C
    state_rd = 3 * 32 * KB + 16 * KB + 32 * KB + 512     # Y, Q_gamma, K_tail, A_qk; U; gamma_C
    tc = {
        "tc_local": inputs + fwd_ws,
        "tc_local_train": inputs + fwd_ws + 16 * KB,                      # + A image
        "tc_state_fwd": state_rd + 16 * KB,                               # + o
        "tc_state_fwd_train": state_rd + 16 * KB + 64 * KB + 32 * KB,     # + S_0^T, R^T images
        "tc_state_fwd_store": 2 * 32 * KB + 32 * KB + 512 + 64 * KB + 32 * KB,
        "tc_state_rev": 16 * KB + 16 * KB + 3 * 32 * KB + 512 + 64 * KB + 32 * KB,
        "tc_bwd_chunk": (32 + 64 + 64 + 32 + 16 + 16) * KB + inputs + 5 * 16 * KB + 32 * KB,
    }
    # per-chain fused kernels: raw inputs read once; the training forward writes o and the per-chunk record
    # (S_0^T fp16 image 32 KB, A and A_qk fp16 images 8 KB each), the backward reads inputs, dO and the record
    # and writes the six gradients (dq, dk, db, dv, dw bf16, dlog_alpha fp32)
    rec = 48 * KB
    chain = {
        "chain_fwd": inputs + 16 * KB,
        "chain_fwd_train": inputs + 16 * KB + rec,
        "chain_fwd_record": inputs + rec,
        "chain_bwd": inputs + 16 * KB + rec + 5 * 16 * KB + 32 * KB,
    }
    if name in chain:
        return nch * chain[name] + 2 * B * H * ss
    if name in tc:
        extra = 0
        if name in ("tc_state_fwd", "tc_state_fwd_train"):
            extra = 2 * B * H * ss
        elif name == "tc_state_rev":
            extra = 2 * B * H * ss
        elif name == "tc_state_fwd_store":
            extra = B * H * ss
        return nch * tc[name] + extra
    if name == "simt_prep":
        return tok * (dk * (3 * eb + 4) + dv * 2 * eb) + nch * (6 * ck + 2 * cv + 2 * cc)
    if name == "simt_state_fwd":
        return nch * (4 * ck + cv + cc + dk * 4) + tok * dv * eb + 2 * B * H * ss
    if name == "simt_state_fwd_store":
        return nch * (2 * ck + cv + dk * 4 + ss) + B * H * ss
    if name == "simt_state_bwd":
        return nch * (3 * ck + cc + dk * 4 + ss + cv) + tok * dv * eb + 2 * B * H * ss
    if name == "simt_chunk_bwd":
        return (tok * (2 * dk * eb + 3 * dv * eb) + nch * (6 * ck + 3 * cv + cc + 2 * ss)
                + nch * 2 * (cv + 5 * ck) + tok * (3 * dk * eb + dk * 4 + 2 * dv * eb))
    return None


def algorithmic_bytes(name, B, T, H):
    """The method's minimum I/O per launch (bytes each launch must read and write once at the operand widths):
    2,080 B per token-head for a forward (q, k, v, b, w, log_alpha in, o out, states amortised) and 3,888 B
    for a backward (inputs, dO and dS_T in; dq, dk, dv, db, dw, dlog_alpha and dS0 out). A kernel that does
    only part of a pass is given that whole pass's bytes, which understates nothing about the pass."""
    th = B * T * H
    if name.startswith("chain_fwd") or name.startswith("tc_local") or name.startswith("tc_state_fwd") or \
            name.startswith("simt_prep") or name.startswith("simt_state_fwd"):
        return th * FWD_BYTES_PER_TH
    if name in ("chain_bwd", "tc_bwd_chunk", "tc_state_rev", "simt_state_bwd", "simt_chunk_bwd"):
        return th * BWD_BYTES_PER_TH
    return None


# ------------------------------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="gdr2_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------------------
def cpu_oracle_sample(inputs_cpu_chains, T, H, target_s=10.0):
    """Time the fp64 oracle (fwd + bwd) on (b, h) chains; repeat rounds until ~target_s of work."""
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    rounds, elapsed, chains = 0, 0.0, 0
    while True:
        t0 = time.perf_counter()
        oracle.fwd(*(inputs_cpu_chains[n] for n in ("q", "k", "v", "log_alpha", "b", "w")),
                   inputs_cpu_chains.get("initial_state"))
        oracle.bwd(*(inputs_cpu_chains[n] for n in ("q", "k", "v", "log_alpha", "b", "w")),
                   inputs_cpu_chains.get("initial_state"), inputs_cpu_chains["d_o"], inputs_cpu_chains["d_final_state"])
        elapsed += time.perf_counter() - t0
        rounds += 1
        chains += inputs_cpu_chains["q"].shape[0]
        if elapsed >= target_s or rounds >= 20:
            break
    tokens = chains * T / H
    return {"value": tokens / elapsed, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{chains} (batch, head) chains x T={T} fwd+bwd in fp64 ({rounds} rounds of "
                      f"{inputs_cpu_chains['q'].shape[0]} chains, {elapsed:.1f} s), = {tokens:.0f} token-equivalents "
                      f"at H={H}"}


def chain_sample(inp, n, T):
    """n (b, h) chains of the workload as CPU tensors shaped [n, T, 1, d]."""
    import torch
    B, _, H, _ = inp["q"].shape
    picks = [(i % B, (i * 7) % H) for i in range(n)]
    out = {}
    for key, t in inp.items():
        if t is None:
            out[key] = None
        elif key in ("initial_state", "d_final_state"):
            out[key] = torch.stack([t[b, h] for b, h in picks])[:, None].cpu()
        else:
            out[key] = torch.stack([t[b, :T, h] for b, h in picks])[:, :, None].cpu()
    return out


# ------------------------------------------------------------------------------------------------
def train_config(B, T, H, dk, dv, world):
    """The training workload's `config` object, shared by both arms of the benchmark."""
    return {"workload": f"train_fwd_bwd: GDR-2 chunk fwd+bwd, B={B}, H={H}, dk={dk}, dv={dv}, T={T}, C=64, "
                        "bf16 operands, fp32 log-decay and state",
            "global_batch": world * B, "seq_len": T, "heads": H, "dk": dk, "dv": dv,
            "parallelism": f"replicas x{world} (independent batches, no collective)",
            "l2": "inputs larger than L2 (0.94 GB of inputs read per step vs 126 MB L2)"}


def run_reference(args, rank):
    """--impl reference: the fp64 oracle on host cores, rank 0 only."""
    if rank != 0:
        return 0
    import torch
    from gated_delta_rule_65_b200 import workloads
    import oracle
    oracle.build()
    wl = workloads.WORKLOADS["train_fwd_bwd"]
    cores = os.cpu_count() or 1
    nchains = max(1, min(cores, 64))
    inp = workloads.chunk_inputs(wl, B=1, T=wl.T, seed=wl.seed)
    # cut nchains chains out of a one-sequence draw (heads are independent chains)
    chains = chain_sample({k: v for k, v in inp.items()}, min(nchains, wl.H), wl.T)
    reps = max(1, nchains // wl.H)
    chains = {k: (None if v is None else v.repeat(*([reps] + [1] * (v.dim() - 1)))) for k, v in chains.items()}
    ncha = chains["q"].shape[0]
    names = ("q", "k", "v", "log_alpha", "b", "w")

    def step():
        oracle.fwd(*(chains[n] for n in names), chains.get("initial_state"))
        oracle.bwd(*(chains[n] for n in names), chains.get("initial_state"), chains["d_o"], chains["d_final_state"])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    tokens = ncha * wl.T / wl.H
    value = tokens * args.steps / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": train_config(wl.B, wl.T, wl.H, wl.dk, wl.dv, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: {ncha} (batch, head) chains x T={wl.T} fwd+bwd in fp64 = "
                                       f"{tokens:.0f} token-equivalents"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-runs", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="override B of the training workload (profiling only)")
    ap.add_argument("--chunk-path", choices=["auto", "chain", "split"], default="auto",
                    help="kernel layout of the training step: automatic, per-chain or chunk-parallel (profiling only)")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode measurement (profiling only)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer measurement (profiling only)")
    ap.add_argument("--no-long", action="store_true", help="skip the long-context measurement (profiling only)")
    ap.add_argument("--long-steps", type=int, default=5)
    ap.add_argument("--no-varlen", action="store_true", help="skip the packed-batch measurement (profiling only)")
    ap.add_argument("--no-prologue", action="store_true", help="skip the gate-prologue measurement (profiling only)")
    ap.add_argument("--no-gva", action="store_true", help="skip the grouped-value-head measurement (profiling only)")
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of replaying the step as a CUDA graph")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank)
    args.warmup = max(args.warmup, 3)

    import torch
    from gated_delta_rule_65_b200 import gdr2, workloads

    torch.cuda.set_device(local)
    dist = world > 1
    if dist:
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                 device_id=torch.device("cuda", local))

    def barrier():
        if dist:
            torch.distributed.barrier()

    def max_over_ranks(x):
        return reduce_max(x, "cuda")

    peaks = load_peaks()
    gdr2.lib()
    gdr2.set_chunk_path({"auto": gdr2.PATH_AUTO, "chain": gdr2.PATH_CHAIN, "split": gdr2.PATH_SPLIT}[args.chunk_path])
    wl = workloads.WORKLOADS["train_fwd_bwd"]
    if args.batch:
        import dataclasses
        wl = dataclasses.replace(wl, B=args.batch)
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    eb = 2
    inp = workloads.chunk_inputs(wl, seed=shard_seed(wl.seed, rank), gen_device="cuda")
    names_in = ("q", "k", "v", "log_alpha", "b", "w")
    g = inp
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device="cuda")
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    grads = {n: torch.empty_like(g["q"]) for n in ("dq", "dk", "db")}
    grads.update({n: torch.empty_like(g["v"]) for n in ("dv", "dw")})
    grads["dlog_alpha"] = torch.empty_like(g["log_alpha"])
    grads["dS0"] = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    ws = gdr2.alloc_workspace(B, T, H, dk, dv, 1, 1)

    def step(src):  # training step: forward keeping its intermediates, then the backward reading them
        gdr2.chunk_fwd(*(src[n] for n in names_in), src["initial_state"], o=o, final_state=ST, workspace=ws,
                       train=True)
        gdr2.chunk_bwd(*(src[n] for n in names_in), src["initial_state"], src["d_o"], src["d_final_state"],
                       out=grads, workspace=ws, saved=True)

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step(g)
    torch.cuda.synchronize()
    gdr2.profile_collect()

    # ---- per-kernel device times (eager launches, events recorded by the library on the stream) -----
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gdr2.profile_enable(True)
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step(g)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    gdr2.profile_enable(False)
    prof = gdr2.profile_collect()
    # eager launches again without the library's per-kernel events: the host-launched step as a user runs it
    barrier()
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(args.steps):
        step(g)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    eager_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps)

    # ---- device-resident timed region: the step replayed as one CUDA graph (no host launch gaps) ----
    graph = None
    if not args.eager:
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            step(g)  # warm the capture stream
        stream.wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step(g)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                step(g)
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
    clocks = clk.summary()
    ms_step = max_over_ranks(ev0.elapsed_time(ev1) / args.steps)
    tokens_step = B * T
    value = world * tokens_step / (ms_step / 1000.0)
    launches = sum(v[0] for k, v in prof.items() if not k.startswith("<"))

    # ---- roofline of the dominant kernel -----------------------------------------------------
    dom = max((k for k in prof if not k.startswith("<")), key=lambda k: prof[k][1])
    nl, tot = prof[dom]
    avg_s = tot / nl / 1000.0
    kb = algorithmic_bytes(dom, B, T, H)
    modelled = kernel_bytes(dom, B, T, H, dk, dv, eb)
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        rec = json.load(open(tpath)).get(dom)
        if rec and rec.get("source_digest") == source_digest(dom):
            traffic = rec.get("dram_bytes_per_launch")
    roofline = {"bound": "hbm", "kernel": dom, "achieved": (kb / avg_s / 1e9) if kb else None,
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": (kb / avg_s / 1e9 / peaks["hbm_gbs"]) if kb else None, "traffic": traffic,
                "bytes_per_launch": kb, "bytes_basis": "algorithmic (minimum I/O of the pass per token-head)",
                "modelled_bytes_per_launch": modelled, "avg_launch_ms": tot / nl, "launches": nl,
                "peak_source": peaks["source"] + " (hbm_gbs, copy read+write)"}
    th = B * T * H
    step_bytes = th * (FWD_BYTES_PER_TH + BWD_BYTES_PER_TH)
    step_flop = th * (FWD_FLOP_PER_TH + BWD_FLOP_PER_TH)
    t_roof = max(step_bytes / (peaks["hbm_gbs"] * 1e9), step_flop / (peaks["bf16_tflops_sustained"] * 1e12))
    step_roofline = {"bound": "hbm" if step_bytes / peaks["hbm_gbs"] / 1e9 >= step_flop / peaks["bf16_tflops_sustained"] / 1e12 else "tensor",
                     "roofline_ms": 1000 * t_roof, "measured_ms": ms_step, "frac": 1000 * t_roof / ms_step,
                     "bytes": step_bytes, "flop": step_flop,
                     "achieved_gbs": step_bytes / (ms_step / 1000) / 1e9,
                     "achieved_tflops": step_flop / (ms_step / 1000) / 1e12}
    kernels = {k: {"launches": v[0], "ms_per_step": v[1] / args.steps, "share": v[1] / sum(x[1] for x in prof.values())}
               for k, v in prof.items() if not k.startswith("<")}

    # ---- end to end through the C ABI with host buffers --------------------------------------
    e2e = None
    if not args.no_e2e:
        e2e = e2e_measure(g, ws, names_in, args, stream, barrier, max_over_ranks, world, tokens_step)

    gdr2.set_chunk_path(gdr2.PATH_AUTO)  # the other workloads take the automatic layout
    decode = None
    if not args.no_decode:
        decode = decode_measure(args, rank, world, names_in, stream, barrier, max_over_ranks, peaks, dk, dv)

    long_ctx = None
    if not args.no_long:
        long_ctx = long_context_measure(args, rank, world, names_in, stream, barrier, max_over_ranks, peaks)

    varlen = None
    if not args.no_varlen:
        varlen = varlen_measure(args, rank, world, names_in, stream, barrier, max_over_ranks, peaks)

    gva = None
    if not args.no_gva:
        gva = gva_measure(args, rank, world, names_in, stream, barrier, max_over_ranks, peaks)

    prologue = None
    if not args.no_prologue:
        prologue = prologue_measure(args, rank, world, stream, barrier, max_over_ranks, peaks)

    # ---- oracle on the host cores (rank 0, single GPU only) ---------------------------------
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        sample = chain_sample({k: v for k, v in g.items()}, max(1, min(cores, 64)), T)
        cpu_baseline = cpu_oracle_sample(sample, T, H)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": train_config(B, T, H, dk, dv, world), "decode": decode,
                "timing": "CUDA graph replay of the step" if graph is not None else "eager launches",
                "eager_ms_per_step": eager_ms,
                "roofline": roofline, "step_roofline": step_roofline, "kernels": kernels,
                "long_context": long_ctx, "varlen": varlen, "grouped_value_heads": gva,
                "gate_prologue": prologue,
                "cpu_baseline": cpu_baseline, "e2e": e2e, "gpu_launches": launches, "clocks": clocks}
        print(json.dumps(line))
    if dist:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def e2e_measure(g, ws, names_in, args, stream, barrier, max_over_ranks, world, tokens_step):
    """The training step through the C ABI with host buffers: every step copies its inputs in from pinned
    host memory and reads every result (o, final state, all gradients) back. As in a training input
    pipeline, the copies of neighbouring steps overlap the compute: step i+1's inputs go in on one stream
    and step i-1's results come out on another while step i runs (two device buffer sets, ordered by
    events), so PCIe carries both directions at once. All copies lie inside the timed region."""
    import torch
    from gated_delta_rule_65_b200 import gdr2
    host_in = {n: (None if t is None else t.cpu().pin_memory()) for n, t in g.items()}
    dev_in = [{n: (None if t is None else torch.empty_like(t)) for n, t in g.items()} for _ in range(2)]
    B, T, H, dk = g["q"].shape
    dv = g["v"].shape[-1]

    def out_set():
        o = {"o": torch.empty_like(g["v"]), "ST": torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")}
        gr = {n: torch.empty_like(g["q"]) for n in ("dq", "dk", "db")}
        gr.update({n: torch.empty_like(g["v"]) for n in ("dv", "dw")})
        gr["dlog_alpha"] = torch.empty_like(g["log_alpha"])
        gr["dS0"] = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
        o["grads"] = gr
        return o

    outs = [out_set(), out_set()]
    flat = lambda o: [o["o"], o["ST"], *o["grads"].values()]  # noqa: E731
    host_out = [t.cpu().pin_memory() for t in flat(outs[0])]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values() if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    s_comp, s_in, s_out = stream, torch.cuda.Stream(), torch.cuda.Stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]
    for e in done + read:
        e.record(s_comp)

    def pipeline(n):
        for i in range(n):
            b = i % 2
            d, o = dev_in[b], outs[b]
            s_in.wait_event(done[b])  # step i-2 has finished with this input set
            with torch.cuda.stream(s_in):
                for name, t in host_in.items():
                    if t is not None:
                        d[name].copy_(t, non_blocking=True)
                in_ready[b].record(s_in)
            s_comp.wait_event(in_ready[b])
            s_comp.wait_event(read[b])  # step i-2's results have been read out of this output set
            args_in = [d[x] for x in names_in]
            gdr2.chunk_fwd(*args_in, d["initial_state"], o=o["o"], final_state=o["ST"], workspace=ws, train=True,
                           stream=s_comp)
            gdr2.chunk_bwd(*args_in, d["initial_state"], d["d_o"], d["d_final_state"], out=o["grads"], workspace=ws,
                           saved=True, stream=s_comp)
            done[b].record(s_comp)
            s_out.wait_event(done[b])
            with torch.cuda.stream(s_out):
                for hbuf, t in zip(host_out, flat(o)):
                    hbuf.copy_(t, non_blocking=True)
                read[b].record(s_out)
        s_comp.wait_event(read[(n - 1) % 2])

    pipeline(2)
    torch.cuda.synchronize()
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(s_comp)
    s_in.wait_event(ev0)
    s_out.wait_event(ev0)
    pipeline(args.steps)
    ev1.record(s_comp)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps)
    return {"value": world * tokens_step / (e2e_ms / 1000.0), "unit": "tokens/s", "ms_per_step": e2e_ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "overlap": "step i+1 inputs in and step i-1 results out during step i (3 streams, 2 device buffer sets)"}


def decode_measure(args, rank, world, names_in, stream, barrier, max_over_ranks, peaks, dk, dv):
    """Decode: 256 sequences x 16 heads, 100 consecutive tokens, timed with CUDA events."""
    import torch
    from gated_delta_rule_65_b200 import gdr2, workloads
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dwl = workloads.DECODE_WORKLOADS["decode_256x16"]
    dinp = decode_inputs_cuda(dwl, rank)  # seeded per rank as well
    S = dinp["state"]
    od = torch.empty((dwl.B, dwl.H, dwl.dv), dtype=torch.bfloat16, device="cuda")
    steps_in = [{n: dinp[n][t] for n in names_in} for t in range(dwl.steps)]

    def decode_run():
        for t in range(dwl.steps):
            s = steps_in[t]
            gdr2.decode_step(s["q"], s["k"], s["v"], s["log_alpha"], s["b"], s["w"], S, o=od)

    decode_run()
    torch.cuda.synchronize()
    gdr2.profile_collect()
    gdr2.profile_enable(True)
    barrier()
    ev0.record(stream)
    for _ in range(args.decode_runs):
        decode_run()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    gdr2.profile_enable(False)
    dprof = gdr2.profile_collect()
    dec_us = max_over_ranks(1000.0 * ev0.elapsed_time(ev1) / (args.decode_runs * dwl.steps))
    dn, dtot = dprof.get("decode", (1, float("nan")))
    dbytes = dwl.B * dwl.H * DECODE_BYTES_PER_SEQHEAD
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = decode_cpu_baseline(dwl)
    return {"metric": "decode tokens/s (one token per sequence per step)",
            "value": world * dwl.B / (dec_us / 1e6), "unit": "tokens/s", "us_per_step": dec_us,
            "config": {"workload": "decode_256x16: 256 sequences x H=16, dk=dv=128, fp32 state, bf16 operands, "
                                   "100 consecutive steps", "state_bytes": dwl.B * dwl.H * dk * dv * 4},
            "roofline": {"bound": "hbm", "kernel": "decode", "achieved": dbytes / (dtot / dn / 1000) / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": dbytes / (dtot / dn / 1000) / 1e9 / peaks["hbm_gbs"],
                         "bytes_per_launch": dbytes, "avg_launch_us": 1000 * dtot / dn, "launches": dn},
            "cpu_baseline": cpu}


def decode_cpu_baseline(dwl, target_s=8.0):
    """The oracle's decode step (fp64, one token per (sequence, head)) on the host cores, on a bounded sample of
    the workload's sequences with all 16 heads, stepped repeatedly; tokens/s = sequences x steps / time."""
    import oracle
    from gated_delta_rule_65_b200 import workloads
    oracle.build()
    n = 16
    inp = workloads.decode_inputs(dwl, B=n, steps=8)
    S = inp["state"]
    steps, elapsed = 0, 0.0
    while elapsed < target_s and steps < 400:
        t = steps % 8
        t0 = time.perf_counter()
        _, S = oracle.decode(inp["q"][t], inp["k"][t], inp["v"][t], inp["log_alpha"][t], inp["b"][t], inp["w"][t], S)
        elapsed += time.perf_counter() - t0
        steps += 1
    return {"value": n * steps / elapsed, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} sequences x H=16 x {steps} decode steps in fp64 ({elapsed:.1f} s; the oracle's decode "
                      f"loop runs on one thread)"}


def long_context_measure(args, rank, world, names_in, stream, barrier, max_over_ranks, peaks):
    """Long context: the training pair on B=1, H=16, T=65536 (16 chains of 1024 chunks). With so few
    chains the serial passes run as a chunk-level scan; timed with CUDA events over eager launches."""
    import torch
    from gated_delta_rule_65_b200 import gdr2, workloads
    wl = workloads.WORKLOADS["long_neg_eig"]
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv
    g = workloads.chunk_inputs(wl, seed=shard_seed(wl.seed, rank), gen_device="cuda")
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device="cuda")
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    grads = {n: torch.empty_like(g["q"]) for n in ("dq", "dk", "db")}
    grads.update({n: torch.empty_like(g["v"]) for n in ("dv", "dw")})
    grads["dlog_alpha"] = torch.empty_like(g["log_alpha"])
    grads["dS0"] = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    ws = gdr2.alloc_workspace(B, T, H, dk, dv, 1, 1)

    def step():
        gdr2.chunk_fwd(*(g[n] for n in names_in), g["initial_state"], o=o, final_state=ST, workspace=ws, train=True)
        gdr2.chunk_bwd(*(g[n] for n in names_in), g["initial_state"], g["d_o"], g["d_final_state"], out=grads,
                       workspace=ws, saved=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    gdr2.profile_collect()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gdr2.profile_enable(True)
    barrier()
    ev0.record(stream)
    for _ in range(args.long_steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    gdr2.profile_enable(False)
    prof = gdr2.profile_collect()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.long_steps)
    th = B * T * H
    step_bytes = th * (FWD_BYTES_PER_TH + BWD_BYTES_PER_TH)
    step_flop = th * (FWD_FLOP_PER_TH + BWD_FLOP_PER_TH)
    t_roof = max(step_bytes / (peaks["hbm_gbs"] * 1e9), step_flop / (peaks["bf16_tflops_sustained"] * 1e12))
    total = sum(x[1] for x in prof.values()) or 1.0
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        sample = chain_sample({k: v for k, v in g.items()}, max(1, min(cores, H)), 4096)
        cpu = cpu_oracle_sample(sample, 4096, H, target_s=8.0)
        cpu["sample"] = "first 4096 tokens of " + cpu["sample"]
    return {"metric": "GDR-2 fwd+bwd tokens/s, long context", "value": world * B * T / (ms / 1000.0),
            "cpu_baseline": cpu,
            "unit": "tokens/s", "ms_per_step": ms,
            "config": {"workload": "long_neg_eig: B=1, H=16, dk=dv=128, T=65536, C=64, b in [0, 2], bf16 operands",
                       "timing": "eager launches, CUDA events"},
            "step_roofline": {"roofline_ms": 1000 * t_roof, "frac": 1000 * t_roof / ms},
            "kernels": {k: {"launches": v[0], "ms_per_step": v[1] / args.long_steps, "share": v[1] / total}
                        for k, v in prof.items() if not k.startswith("<")}}


def varlen_measure(args, rank, world, names_in, stream, barrier, max_over_ranks, peaks):
    """Packed variable-length batch: 16 sequences of 358..5986 tokens (32,768 in all, the token count of
    the 8 x 4096 training batch), H = 16, training pair; timed with CUDA events over eager launches."""
    import torch
    from gated_delta_rule_65_b200 import gdr2, workloads
    wl = workloads.VARLEN_WORKLOADS["varlen_mix"]
    g = workloads.varlen_inputs(wl, gen_device="cuda")
    T, H, N = wl.T, wl.H, wl.N
    cu = g["cu_seqlens"]
    o = torch.empty_like(g["v"])
    ST = torch.empty((N, H, 128, 128), dtype=torch.float32, device="cuda")
    grads = {n: torch.empty_like(g["q"]) for n in ("dq", "dk", "db")}
    grads.update({n: torch.empty_like(g["v"]) for n in ("dv", "dw")})
    grads["dlog_alpha"] = torch.empty_like(g["log_alpha"])
    grads["dS0"] = torch.empty((N, H, 128, 128), dtype=torch.float32, device="cuda")
    ws = gdr2.alloc_workspace_varlen(N, T, H, 128, 128, 1, 1)

    def step():
        gdr2.chunk_fwd_varlen(*(g[n] for n in names_in), cu, g["initial_state"], o=o, final_state=ST, workspace=ws,
                              train=True)
        gdr2.chunk_bwd_varlen(*(g[n] for n in names_in), cu, g["initial_state"], g["d_o"], g["d_final_state"],
                              out=grads, workspace=ws, saved=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    gdr2.profile_collect()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gdr2.profile_enable(True)
    barrier()
    ev0.record(stream)
    for _ in range(args.long_steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    gdr2.profile_enable(False)
    prof = gdr2.profile_collect()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.long_steps)
    th = T * H
    step_bytes = th * (FWD_BYTES_PER_TH + BWD_BYTES_PER_TH)
    step_flop = th * (FWD_FLOP_PER_TH + BWD_FLOP_PER_TH)
    t_roof = max(step_bytes / (peaks["hbm_gbs"] * 1e9), step_flop / (peaks["bf16_tflops_sustained"] * 1e12))
    total = sum(x[1] for x in prof.values()) or 1.0
    return {"metric": "GDR-2 fwd+bwd tokens/s, packed variable-length batch", "value": world * T / (ms / 1000.0),
            "unit": "tokens/s", "ms_per_step": ms,
            "config": {"workload": f"varlen_mix: N={N} sequences, lengths {min(workloads.varlen_lengths(wl))}.."
                                   f"{max(workloads.varlen_lengths(wl))} (log-uniform, seeded), T={T} packed, "
                                   "H=16, dk=dv=128, bf16 operands",
                       "timing": "eager launches, CUDA events"},
            "step_roofline": {"roofline_ms": 1000 * t_roof, "frac": 1000 * t_roof / ms},
            "kernels": {k: {"launches": v[0], "ms_per_step": v[1] / args.long_steps, "share": v[1] / total}
                        for k, v in prof.items() if not k.startswith("<")}}


def gva_measure(args, rank, world, names_in, stream, barrier, max_over_ranks, peaks):
    """Grouped value heads: the training pair on B=8, T=4096 with 8 key heads shared by 16 value heads
    (the state and value traffic of the 16-head training batch, half its key side); CUDA events."""
    import torch
    from gated_delta_rule_65_b200 import gdr2, workloads
    wl = workloads.GVA_WORKLOADS["gva_train"]
    H, Hv = 8, wl.H
    import dataclasses
    g = workloads.gva_inputs(dataclasses.replace(wl, seed=shard_seed(wl.seed, rank)), H, gen_device="cuda")
    B, T = wl.B, wl.T
    o = torch.empty_like(g["v"])
    ST = torch.empty((B, Hv, 128, 128), dtype=torch.float32, device="cuda")
    grads = {n: torch.empty_like(g["q"]) for n in ("dq", "dk", "db")}
    grads.update({n: torch.empty_like(g["v"]) for n in ("dv", "dw")})
    grads["dlog_alpha"] = torch.empty_like(g["log_alpha"])
    grads["dS0"] = torch.empty((B, Hv, 128, 128), dtype=torch.float32, device="cuda")
    ws = gdr2.alloc_workspace_gva(B, T, H, Hv, 128, 128, 1, 1)

    def step():
        gdr2.chunk_fwd_gva(*(g[n] for n in names_in), g["initial_state"], o=o, final_state=ST, workspace=ws,
                           train=True)
        gdr2.chunk_bwd_gva(*(g[n] for n in names_in), g["initial_state"], g["d_o"], g["d_final_state"], out=grads,
                           workspace=ws, saved=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    gdr2.profile_collect()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gdr2.profile_enable(True)
    barrier()
    ev0.record(stream)
    for _ in range(args.long_steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    gdr2.profile_enable(False)
    prof = gdr2.profile_collect()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.long_steps)
    total = sum(x[1] for x in prof.values()) or 1.0
    return {"metric": "GDR-2 fwd+bwd tokens/s, grouped value heads", "value": world * B * T / (ms / 1000.0),
            "unit": "tokens/s", "ms_per_step": ms,
            "config": {"workload": "gva_train: B=8, T=4096, H=8 key heads, Hv=16 value heads, dk=dv=128, bf16",
                       "timing": "eager launches, CUDA events"},
            "kernels": {k: {"launches": v[0], "ms_per_step": v[1] / args.long_steps, "share": v[1] / total}
                        for k, v in prof.items() if not k.startswith("<")}}


# Gate prologue bytes per token-head (bf16, dk = dv = 128): forward reads x_q, x_k, x_f, x_b, x_w and
# writes q, k, b, w (bf16) and log_alpha (fp32); backward reads the five pre-activations, dq, dk, db, dw
# and dlog_alpha (fp32) and writes the five pre-activation gradients.
PRO_FWD_BYTES_PER_TH = 5 * 256 + 4 * 256 + 512
PRO_BWD_BYTES_PER_TH = 5 * 256 + 4 * 256 + 512 + 5 * 256


def prologue_measure(args, rank, world, stream, barrier, max_over_ranks, peaks):
    """The gate and normalisation prologue of the training batch (B=8, T=4096, H=16, d=128, bf16):
    forward and backward launches timed with CUDA events (inputs 1.3-2.1 GB per launch, beyond L2)."""
    import torch
    from gated_delta_rule_65_b200 import gdr2, workloads
    wl = workloads.PROLOGUE_WORKLOADS["prologue_train"]
    g = workloads.prologue_inputs(dataclasses_replace_seed(wl, rank), gen_device="cuda")
    X = ("xq", "xk", "xf", "xb", "xw", "a", "delta")
    fo = gdr2.gate_prologue_fwd(*(g[n] for n in X))
    bo = gdr2.gate_prologue_bwd(*(g[n] for n in X), g["dq"], g["dk"], g["dlog_alpha"], g["db"], g["dw"])
    n_ws = int(gdr2.lib().gdr2_gate_prologue_workspace_bytes(wl.B, wl.T, wl.H, wl.dk, wl.dv, 1))
    ws = torch.empty(max(n_ws, 16), dtype=torch.uint8, device="cuda")
    res = {}
    for name, call in (("fwd", lambda: gdr2.gate_prologue_fwd(*(g[n] for n in X), out=fo)),
                       ("bwd", lambda: gdr2.gate_prologue_bwd(*(g[n] for n in X), g["dq"], g["dk"], g["dlog_alpha"],
                                                              g["db"], g["dw"], out=bo, workspace=ws))):
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(args.steps, 5)
        gdr2.profile_collect()
        gdr2.profile_enable(True)
        barrier()
        ev0.record(stream)
        for _ in range(n):
            call()
        ev1.record(stream)
        torch.cuda.synchronize()
        gdr2.profile_enable(False)
        prof = gdr2.profile_collect()
        ms = max_over_ranks(ev0.elapsed_time(ev1) / n)
        per_th = PRO_FWD_BYTES_PER_TH if name == "fwd" else PRO_BWD_BYTES_PER_TH
        nbytes = wl.B * wl.T * wl.H * per_th
        main = prof.get("prologue_" + name)
        kms = main[1] / main[0] if main else None
        res[name] = {"ms": ms, "bytes": nbytes, "achieved_gbs": nbytes / (ms / 1000) / 1e9,
                     "frac": nbytes / (ms / 1000) / 1e9 / peaks["hbm_gbs"],
                     "kernel_ms": kms, "kernel_frac": (nbytes / (kms / 1000) / 1e9 / peaks["hbm_gbs"]) if kms else None,
                     "kernels": {k: v[1] / v[0] for k, v in prof.items() if not k.startswith("<")}}
    return {"metric": "gate prologue, HBM GB/s", "unit": "GB/s", "bound": "hbm", "peak": peaks["hbm_gbs"],
            "config": {"workload": "prologue_train: B=8, T=4096, H=16, dk=dv=128, bf16 (fp32 log-decay)",
                       "timing": "CUDA events, back-to-back launches"},
            **res}


def dataclasses_replace_seed(wl, rank):
    import dataclasses
    return dataclasses.replace(wl, seed=shard_seed(wl.seed, rank))


def decode_inputs_cuda(dwl, rank):
    """Decode inputs drawn directly on the GPU (same distributions as workloads.decode_inputs)."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(shard_seed(dwl.seed, rank))
    n = lambda *s: torch.randn(*s, generator=g, device="cuda")  # noqa: E731
    l2n = lambda x: x / x.norm(dim=-1, keepdim=True)  # noqa: E731
    st = dwl.steps
    return {
        "state": dwl.s0_std * n(dwl.B, dwl.H, dwl.dk, dwl.dv),
        "q": l2n(n(st, dwl.B, dwl.H, dwl.dk)).bfloat16(), "k": l2n(n(st, dwl.B, dwl.H, dwl.dk)).bfloat16(),
        "v": n(st, dwl.B, dwl.H, dwl.dv).bfloat16(),
        "log_alpha": (-0.1 * torch.nn.functional.softplus(n(st, dwl.B, dwl.H, dwl.dk))).bfloat16().float(),
        "b": torch.sigmoid(n(st, dwl.B, dwl.H, dwl.dk)).bfloat16(),
        "w": torch.sigmoid(n(st, dwl.B, dwl.H, dwl.dv)).bfloat16(),
    }


if __name__ == "__main__":
    sys.exit(main())
