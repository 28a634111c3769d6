#!/usr/bin/env python
"""Benchmark of the RLT recurrent decoder transition on B200; prints one JSON line.

A step is one full decoder sweep of the workload: starting from H_0 = (s*, empty), all
B sequences take T lockstep transitions H_{t-1}, e_t -> H_t with the log-probability of
the next token gathered at every step.  The encoder outputs e and M are produced once,
before timing, and stay resident in HBM (the decoder's inputs).  Metric: decoder
tokens/s = (ranks x B x T) / device time of the sweep, max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun every rank runs its own replica on its own sequences (weak scaling, no
collective on the data path; the only collective is the max over ranks of the timing).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from workloads import WORKLOADS, RLT_300M, make_tokens, make_weights, decoder_param_count  # noqa: E402

METRIC = "RLT decoder tokens/s (seqs×steps) on 1 B200; % of per-step roofline"
DEFAULT_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        d["source"] = "measured"
        return d
    return dict(DEFAULT_PEAKS)


# ----------------------------------------------------------------------------- cost model

def step_cost(m, B: int, t: int, m_once: bool = False) -> tuple[float, float]:
    """Algorithmic bytes and FLOPs of one decoder step at position t (1-based) for B sequences:
    the decoder weights once, the SWA window of every layer, M_{<=t} once per reading layer,
    the current k/v writes and e_t.  m_once: the stricter bound for a memory shared by all
    layers (G = 1) that counts M_{<=t} once per step, as if it stayed on chip across layers."""
    bw = 2 if m.dtype == "bf16" else 4
    d, W, L = m.d, m.W, m.L_D
    P = decoder_param_count(m)
    win = min(t, W)
    m_reads = 1 if (m_once and m.G == 1) else L
    nbytes = P * bw + B * L * ((win - 1) * 2 * d * bw + 2 * d * bw) + B * m_reads * t * 2 * d * bw + B * d * bw
    flops = B * (2 * P + L * 4 * d * (win + t))
    return float(nbytes), float(flops)


def kind_cost(kind: str, m, B: int, T: int) -> tuple[str, float]:
    """('hbm', bytes) or ('tensor', flops) summed over a sweep of T steps for one kernel kind."""
    bw = 2 if m.dtype == "bf16" else 4
    d, L, F, V, W = m.d, m.L_D, m.F, m.V, m.W
    ts = np.arange(1, T + 1, dtype=np.float64)
    if kind == "xattn":
        return "hbm", float(L * np.sum(B * ts * 2 * d * bw + B * d * 4 + B * d * bw))
    if kind == "swa":
        win = np.minimum(ts, W)
        return "hbm", float(L * np.sum(B * ((win - 1) * 2 * d * bw + 2 * d * bw + 3 * d * 4 + d * bw)))
    gemm = {"qkv": (3 * d, d, L), "o_proj": (d, d, L), "qc_proj": (d, d, L), "oc_proj": (d, d, L),
            "ffn_up": (2 * F, d, L), "ffn_down": (d, F, L), "merge": (2 * d, 2 * d, 1), "head": (V, d, 1)}
    if kind in gemm:
        N, K, n = gemm[kind]
        steps = T - 1 if kind == "head" else T
        return "tensor", float(2.0 * B * N * K * n * steps)
    if kind in ("norm", "final_norm"):
        n = 3 * L if kind == "norm" else 1
        return "hbm", float(T * n * B * d * (4 + bw))
    if kind == "lse":
        return "hbm", float((T - 1) * B * V * 4)
    if kind == "small_step":
        # one launch per step: the step's algorithmic bytes (weights, window, memory, e_t)
        return "hbm", float(sum(step_cost(m, B, int(t))[0] for t in ts))
    return "hbm", 0.0


def encode_flops(m, B: int, T: int) -> float:
    """FLOPs of one rlt_encode over B sequences of T tokens: 2 per weight and token for the
    encoder layers (q/k/v/o 4d^2, SwiGLU 3dF) and the G memory projections (2d^2 each), plus the
    causal attention (q k^T and p v: 4 * hd FLOPs per (query, key <= query) pair and head)."""
    lin = 2.0 * B * T * (m.L_E * (4 * m.d * m.d + 3 * m.d * m.F) + m.G * 2 * m.d * m.d)
    att = 4.0 * m.L_E * B * m.n_heads * m.head_dim * T * (T + 1) / 2
    return lin + att


def run_roofline_s(m, B: int, T: int, peaks: dict, m_once: bool = False) -> float:
    bw = peaks["hbm_gbs"] * 1e9
    fl = peaks["bf16_tflops"] * 1e12
    tot = 0.0
    for t in range(1, T + 1):
        b, f = step_cost(m, B, t, m_once)
        tot += max(b / bw, f / fl)
    return tot


# ----------------------------------------------------------------------------- ranks

def rank_sequences(rank: int, B: int) -> range:
    """Sequences of the seeded batch stream that rank `rank` decodes (B per rank, disjoint)."""
    return range(rank * B, (rank + 1) * B)


def max_over_ranks(value: float, device=None) -> float:
    """Slowest rank's time: the job's time.  Identity without a process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = Path(tempfile.gettempdir()) / f"rlt_bench_clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            self.out.parent.mkdir(exist_ok=True)
            self.f = open(self.out, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if self.proc is None or not self.out.exists():
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.read_text().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_id_for(dev) -> str:
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


# ----------------------------------------------------------------------------- CPU oracle baseline

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(wl, steps: int, seqs=(0,)) -> tuple[float, str]:
    """Time the CPU oracle (float32) on `seqs` x the first `steps` tokens: encode + decoder
    steps.  Returns (tokens per second, description)."""
    from oracle import RLTOracle
    m = wl.model
    w = make_weights(m, wl.weight_seed)
    tok = make_tokens(wl, seqs)[:, :steps]
    ora = RLTOracle(m, w, np.float32)
    del w
    t0 = time.perf_counter()
    e, M = ora.encode(tok)
    st = ora.init_state(len(seqs))
    for t in range(1, steps + 1):
        st, _ = ora.step(st, e[:, t - 1], M, wl.tau)
    dt = time.perf_counter() - t0
    return len(seqs) * steps / dt, (f"{len(seqs)} sequence(s) x first {steps} tokens of {wl.name}: encode + "
                                    f"{steps} decoder steps, numpy float32 oracle")


def oracle_steps_for(wl) -> int:
    return {"tiny-f32": 64, "small-bf16": 128, "300m-12+12-b512": 48}.get(wl.name, 12)


# ----------------------------------------------------------------------------- reference arm

def arm_config(wl, B: int, T: int, world: int) -> dict:
    """The workload description both arms print (the reference arm adds its sample)."""
    return {"workload": wl.name, "B_per_gpu": B, "T": T, "global_batch": world * B, "seq_len": T,
            "parallelism": f"replicas x{world} (sequences sharded, no data-path collective)",
            "l2": "inputs larger than L2 (M, SWA cache and weights stream from HBM every step)",
            "step": "one full decoder sweep of T lockstep transitions with next-token log-prob gather"}


def run_reference(args, wl, rank: int, world: int) -> None:
    if rank != 0:
        return
    steps = oracle_steps_for(wl)
    vals = []
    for i in range(args.warmup + args.steps):
        v, desc = oracle_sample(wl, steps)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * steps / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {**arm_config(wl, wl.B, wl.T, world), "sample": desc},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- traffic from ncu

def traffic_per_unit(kind: str) -> float | None:
    """DRAM bytes per algorithmic byte of `kind` from the committed ncu summary, if that summary
    was taken from the current kernel source (its recorded hash matches); else None."""
    f = ROOT / "profiles" / f"{kind}_traffic.txt"
    if not f.exists():
        return None
    kv = dict(line.split("=", 1) for line in f.read_text().splitlines() if "=" in line and not line.startswith("#"))
    src = ROOT / "cross_token_latent_b200" / "csrc" / kv.get("source", "").strip()
    if not src.exists():
        return None
    if hashlib.sha256(src.read_bytes()).hexdigest()[:16] != kv.get("source_sha256_16", "").strip():
        return None
    try:
        return float(kv["dram_bytes_per_algorithmic_byte"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- main

def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=RLT_300M.name, choices=sorted(WORKLOADS))
    ap.add_argument("--T", type=int, default=None, help="override the sweep length (profiling runs only)")
    ap.add_argument("--B", type=int, default=None, help="override the batch (profiling runs only)")
    ap.add_argument("--option", action="append", default=[], metavar="NAME=VALUE",
                    help="scheduling option of the model handle (rlt_set_option), repeatable")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-replay", action="store_true")
    ap.add_argument("--no-generate", action="store_true")
    ap.add_argument("--nvtx-sample", type=int, default=0,
                    help="profiling runs: wrap this many evenly spaced steps of the first timed sweep in an NVTX "
                         "range 'sample' (for ncu --nvtx-include sample/); skips the breakdown sweep")
    args = ap.parse_args()
    if args.warmup < 3 and not args.nvtx_sample:
        ap.error("--warmup must be >= 3")

    wl = WORKLOADS[args.workload]
    if args.T or args.B:
        wl = wl.with_batch(args.B or wl.B, args.T or wl.T)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return 0

    import torch
    import torch.distributed as dist
    from cross_token_latent_b200 import RLTModel

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=900),
                                device_id=dev)
    peaks = load_peaks()
    m, B, T = wl.model, wl.B, wl.T

    model = RLTModel(m, max_pos=T)
    for opt in args.option:
        name, value = opt.split("=", 1)
        model.set_option(name, int(value))
    w = make_weights(m, wl.weight_seed)
    model.load_weights(w)
    del w
    tokens = make_tokens(wl, rank_sequences(rank, B))
    tok = torch.from_numpy(tokens).to(dev)
    tok_tb = tok.t().contiguous()                        # row t = x_{t+1} of every sequence
    e, M = model.encode(tok)
    torch.cuda.synchronize()
    model.release_workspaces()
    state = model.new_state(B)
    lp_tb = torch.zeros((T, B), dtype=torch.float32, device=dev)

    sample_steps = set()
    if args.nvtx_sample:
        sample_steps = {int(round(i * (T - 1) / max(1, args.nvtx_sample - 1))) for i in range(args.nvtx_sample)}

    def sweep(mark=False):
        model.reset_state(state)
        for t in range(T):
            nxt = t + 1 < T
            tag = mark and t in sample_steps
            if tag:
                torch.cuda.nvtx.range_push("sample")
            model.decode_step(state, e, M, next_tok=tok_tb[t + 1] if nxt else None, tau=wl.tau,
                              logp_tok=lp_tb[t] if nxt else None)
            if tag:
                torch.cuda.nvtx.range_pop()

    for _ in range(args.warmup):
        sweep()
    torch.cuda.synchronize()
    model.check_device_errors()

    # one untimed sweep with every kernel kind bracketed: the breakdown and the dominant kernel
    if args.nvtx_sample:
        breakdown = {"xattn": (1.0, 1)}
    else:
        model.profile_start()
        sweep()
        breakdown = model.profile_stop()
    dominant = max((k for k in breakdown if k != "encoder"), key=lambda k: breakdown[k][0])

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = model.launch_count
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_id_for(local)) as clk:
        model.profile_start([dominant])
        torch.cuda.nvtx.range_push("timed")
        ev0.record()
        for i in range(args.steps):
            sweep(mark=i == 0)
        ev1.record()
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        dom = model.profile_stop()
    launches = model.launch_count - launches0
    ms = ev0.elapsed_time(ev1)
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ms, dev)
    ms_per_step = ms / args.steps
    value = world * B * T / (ms_per_step / 1e3)

    # roofline of the dominant kernel, timed live inside the timed region
    bound, alg = kind_cost(dominant, m, B, T)
    dom_ms, dom_n = dom.get(dominant, (0.0, 0))
    per_launch = alg / max(1, breakdown[dominant][1])
    if bound == "hbm":
        achieved = alg * args.steps / (dom_ms / 1e3) / 1e9 if dom_ms else None
        peak, unit = peaks["hbm_gbs"], "GB/s"
    else:
        achieved = alg * args.steps / (dom_ms / 1e3) / 1e12 if dom_ms else None
        peak, unit = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]), "TFLOP/s"
    tpu = traffic_per_unit(dominant)
    roofline = {"kernel": dominant, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": (achieved / peak) if achieved else None,
                "traffic": (tpu * per_launch) if tpu is not None else None,
                "algorithmic_per_launch": per_launch, "launches_timed": dom_n,
                "avg_launch_us": 1e3 * dom_ms / max(1, dom_n), "peak_source": peaks.get("source")}
    rr = run_roofline_s(m, B, T, peaks)
    rr1 = run_roofline_s(m, B, T, peaks, m_once=True)
    step_roofline = {"run_roofline_ms": 1e3 * rr, "measured_ms": ms_per_step,
                     "frac": 1e3 * rr / ms_per_step,
                     "note": "sum over t of max(bytes(t)/HBM, flops(t)/bf16 burst peak)",
                     "m_once_run_roofline_ms": 1e3 * rr1, "m_once_frac": 1e3 * rr1 / ms_per_step,
                     "m_once_note": "stricter bound for G=1: M_{<=t} read once per step instead of once per layer"}
    clocks = clk.summary()

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        tok_host = torch.from_numpy(tokens).pin_memory()
        lp_host = torch.empty((T, B), dtype=torch.float32).pin_memory()

        def e2e_once():
            td = tok_host.to(dev, non_blocking=True)
            ee, MM = model.encode(td, out=(e, M))
            ttb = td.t().contiguous()
            model.reset_state(state)
            for t in range(T):
                nxt = t + 1 < T
                model.decode_step(state, ee, MM, next_tok=ttb[t + 1] if nxt else None, tau=wl.tau,
                                  logp_tok=lp_tb[t] if nxt else None)
            lp_host.copy_(lp_tb, non_blocking=True)

        e2e_once()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        e2e_once()
        b.record()
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), dev)
        e2e = {"value": world * B * T / (e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": tokens.nbytes,
               "d2h_bytes_per_step": int(lp_host.numel() * 4), "ms_per_step": e_ms,
               "includes": "H2D tokens, rlt_encode, T rlt_decode_step calls, D2H log-probs"}

    # the encoder on its own (the rlt_encode call of the e2e path), tensor-bound
    enc = None
    if not args.no_e2e:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        model.encode(tok, out=(e, M))
        a.record()
        model.encode(tok, out=(e, M))
        b.record()
        torch.cuda.synchronize()
        enc_ms = max_over_ranks(a.elapsed_time(b), dev)
        ef = encode_flops(m, B, T)
        enc_roof_ms = 1e3 * ef / (peaks["bf16_tflops"] * 1e12)
        # one more encode with its launches bracketed by kind (brackets cost a few us each)
        model.profile_start(["enc_gemm", "enc_attn", "enc_other"])
        model.encode(tok, out=(e, M))
        enc_kinds = {k: round(v[0], 2) for k, v in model.profile_stop().items()}
        enc = {"ms": enc_ms, "tflop": ef / 1e12, "achieved_tflops": ef / (enc_ms / 1e3) / 1e12,
               "peak_tflops": peaks["bf16_tflops"], "roofline_ms": enc_roof_ms, "frac": enc_roof_ms / enc_ms,
               "breakdown_ms": enc_kinds,
               "note": "one rlt_encode of the whole batch; FLOPs of the linear maps and the causal attention"}

    replay = None
    if not args.no_replay:
        P = torch.full((B,), wl.prompt_len, dtype=torch.int32, device=dev)
        model.replay(tok, P, wl.tau)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        model.replay(tok, P, wl.tau)
        b.record()
        torch.cuda.synchronize()
        r_ms = max_over_ranks(a.elapsed_time(b), dev)
        r_roof_ms = 1e3 * rr + 1e3 * encode_flops(m, B, T) / (peaks["bf16_tflops"] * 1e12)
        replay = {"value": world * B * T / (r_ms / 1e3), "unit": "tokens/s", "ms": r_ms,
                  "roofline_ms": r_roof_ms, "frac": r_roof_ms / r_ms,
                  "includes": "rlt_replay: encode + T steps + response scoring",
                  "roofline_note": "decoder run roofline + encoder FLOPs at the bf16 burst peak"}
    # the generation loop: prompt of T/2 tokens, then T/2 sampled ones (prefill with an encoder
    # cache, decoder steps over the prompt, then [decode with the full row, sample, encode the
    # draw incrementally] per new token); tokens/s counts the sampled tokens of all sequences
    gen = None
    if not args.no_generate and T >= 4:
        P = T // 2
        n_new = T - P
        g = torch.Generator(device=dev).manual_seed(1234)
        u = torch.rand((n_new, B), generator=g, device=dev)
        prompt = tok[:, :P].contiguous()
        model.generate(prompt, n_new, u, tau=wl.tau, top_k=50, top_p=0.95)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        model.generate(prompt, n_new, u, tau=wl.tau, top_k=50, top_p=0.95)
        b.record()
        torch.cuda.synchronize()
        g_ms = max_over_ranks(a.elapsed_time(b), dev)
        gen = {"value": world * B * n_new / (g_ms / 1e3), "unit": "generated tokens/s", "ms": g_ms,
               "prompt": P, "new_tokens": n_new, "top_k": 50, "top_p": 0.95,
               "includes": "rlt_encode_prefill, P decoder steps, then per new token: rlt_decode_step with the "
                           "full log-prob row, rlt_sample, rlt_encode_append"}
        model.release_workspaces()
    model.check_device_errors()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc = oracle_sample(wl, oracle_steps_for(wl))
        cpu = {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": m.dtype, "data": "synthetic",
            "config": {**arm_config(wl, B, T, world), **({"options": args.option} if args.option else {})},
            "roofline": roofline, "step_roofline": step_roofline, "cpu_baseline": cpu, "e2e": e2e,
            "replay": replay, "encode": enc, "generate": gen, "gpu_launches": launches, "clocks": clocks,
            "kernel_breakdown_ms_per_sweep": {k: round(v[0], 3) for k, v in sorted(breakdown.items())},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
