"""Benchmark of the RLT decoder hot path on B200 GPUs.

Default workload (one GPU): current-policy replay of the reference-width model
at L_E = L_D = 24 (d=2048, 16x128 heads, W=256, G=1, F=5632, V=32000), B = 256
sequences of S = 1024 tokens.  One step = one rlt_replay_logprobs call:
token-parallel encoder + memory projection over [B, S], then S-1 lock-step
decoder transitions with the readout of every next-token log-prob.  The
metric is decoder tokens/s = B x (S-1) x steps / time.  (The 48+48 model at
B=128 with 2048+2048 tokens needs about 229 GB of state and does not fit one
GPU; this is the largest of the benchmarked configurations that does.)

Multi-GPU (torchrun): sequences shard across ranks with no data-path
collective (weak scaling, B sequences per rank); timing is the max over ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

BENCH_WORKLOADS = {
    # name: (synth workload, overrides, kind)
    "replay": ("replay", {}, "replay"),
    "layerwise": ("layerwise", {}, "replay"),
    "small": ("small", {}, "generate"),
    "refdepth-b64": ("refdepth", {"batch": 64}, "generate"),
    "refdepth-b128-t3072": ("refdepth", {"gen": 1024}, "generate"),
    # full-BPTT forward + backward (rlt_replay_backward) of the small model
    "bptt-small": ("small", {"prompt": 256, "gen": 0}, "backward"),
}
BPTT_METRIC = "RLT full-BPTT tokens/s (replay forward + backward through the whole history) on 1 B200"
BPTT_SEGMENT = 32

METRIC = "RLT decoder tokens/s (B seqs, 48+48 tied) on 1 B200; % of step roofline"


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- roofline model
def step_roofline(w: dict, kind: str, peaks: dict) -> dict:
    """Analytic lower bound of one step: per decoder transition the slower of
    (weights + KV bytes)/HBM and FLOPs/tensor peak, plus the token-parallel
    encoder at tensor peak."""
    d, L, F, V, G, W, B = w["d"], w["n_layers"], w["ffn"], w["vocab"], w["groups"], w["window"], w["batch"]
    eb = 2 if w["dtype"] == 1 else 4
    merge = 3 * d * d if w.get("merge_kind", 0) == 0 else 2 * d * d
    p_dec = L * (4 * d * d + 2 * d * d + 3 * d * F) + merge + V * d
    p_enc = L * (4 * d * d + 3 * d * F) + 2 * d * d * G
    hbm = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops_sustained"] * 1e12
    T = w["prompt"]
    n_gen = w.get("gen", 0) if kind == "generate" else 0
    total = 0.0
    dec_steps = (T - 1 if kind == "replay" else T + n_gen - 1)
    for t in range(1, dec_steps + 1):
        kv = B * eb * 2 * d * (L * (min(t, W) - 1) + L + L * t)
        wbytes = eb * p_dec
        flops = 2 * B * p_dec + 4 * B * d * (L * min(t, W) + L * t)
        if kind == "generate" and t > T:
            kv += B * eb * 2 * d * (L * t + L + G)
            wbytes += eb * p_enc
            flops += 2 * B * p_enc + 4 * B * d * L * t
        total += max((kv + wbytes) / hbm, flops / tc)
    S = T
    enc_flops = 2 * B * S * p_enc + 4 * B * L * d * S * S / 2
    total += enc_flops / tc
    return {"bound_ms": total * 1e3, "decoder_transitions": dec_steps}


# ---------------------------------------------------------------- sharding
def shard_tokens(w: dict, rank: int, world: int) -> np.ndarray:
    """Rank `rank`'s share of the global batch: the global batch holds
    world * B sequences drawn from the workload's seed; rank r owns rows
    [r*B, (r+1)*B).  Sequences are independent (report §4.1), so no data
    moves between ranks."""
    B = w["batch"]
    length = w["prompt"]
    g = synth.tokens(w, batch=world * B, length=length)
    return np.ascontiguousarray(g[rank * B:(rank + 1) * B])


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """Step time of the job = the slowest rank's."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.rows.append(parts)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ---------------------------------------------------------------- CPU oracle leg
def oracle_sample(w: dict, n_tokens: int, seed_seq: int = 0) -> tuple[float, int, str]:
    """Times the fp64 oracle on one sequence truncated to n_tokens of the
    workload (encoder + n_tokens-1 decoder transitions with readouts).
    Returns (decoder tokens/s, threads, description)."""
    import oracle
    om = oracle.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)
    tok = synth.tokens(w, batch=1, length=n_tokens, seed=w["data_seed"] + seed_seq)[0]
    t0 = time.perf_counter()
    om.replay_logprobs(tok)
    dt = time.perf_counter() - t0
    return (n_tokens - 1) / dt, oracle.num_threads(), f"1 sequence x {n_tokens} tokens (teacher-forced replay), fp64"


def oracle_bptt_sample(w: dict, n_tokens: int, seed_seq: int = 0) -> tuple[float, int, str]:
    """Times the gradient oracle (fp64 autograd, full BPTT) on one sequence
    truncated to n_tokens.  Returns (scored tokens/s, threads, description)."""
    import torch

    import oracle
    from oracle import bptt
    om = oracle.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)
    tok = synth.tokens(w, batch=1, length=n_tokens, seed=w["data_seed"] + seed_seq)[0]
    t0 = time.perf_counter()
    bptt.loss_and_grads(om, tok, bptt.target_weights("pretrain", n_tokens))
    dt = time.perf_counter() - t0
    return ((n_tokens - 1) / dt, torch.get_num_threads(),
            f"1 sequence x {n_tokens} tokens, forward + full-BPTT backward, fp64 autograd")


def oracle_tokens_for(w: dict) -> int:
    d, L = w["d"], w["n_layers"]
    per_tok = L * (10 * d * d + 6 * d * w["ffn"]) + w["vocab"] * d  # weights streamed per token (enc + dec)
    scale = max(1.0, per_tok / 4e8)
    return int(max(16, min(w["prompt"], 256 / scale)))


# ---------------------------------------------------------------- GPU leg
def run_gpu(args, w: dict, kind: str, peaks: dict, rank: int, world: int) -> dict | None:
    import torch
    import torch.distributed as dist
    import stateful_decoder_b200 as rlt

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    cfg = synth.model_config(w)
    B = w["batch"]
    model = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    stream = torch.cuda.current_stream()

    if kind == "replay":
        S = w["prompt"]
        tok_host = torch.from_numpy(shard_tokens(w, rank, world)).pin_memory()
        tok = tok_host.cuda()
        logp = torch.empty(B, S - 1, device=dev)
        logp_host = torch.empty(B, S - 1).pin_memory()
        tokens_per_step = B * (S - 1)

        def step():
            rlt.rlt_replay_logprobs(model, tok, logp)

        def step_e2e():
            tok.copy_(tok_host, non_blocking=True)
            rlt.rlt_replay_logprobs(model, tok, logp)
            logp_host.copy_(logp, non_blocking=True)

        h2d, d2h = tok_host.numel() * 4, logp_host.numel() * 4
    else:
        T, n_gen = w["prompt"], w["gen"]
        state = rlt.rlt_state_create(model, B, T + n_gen, rlt.STATE_ENCODER_CACHE)
        tok_host = torch.from_numpy(shard_tokens(w, rank, world)).pin_memory()
        tok = tok_host.cuda()
        ids = torch.zeros(n_gen, B, dtype=torch.int32, device=dev)
        lmu = torch.zeros(n_gen, B, device=dev)
        lps = torch.zeros(n_gen, B, device=dev)
        ids_host = torch.zeros(n_gen, B, dtype=torch.int32).pin_memory()
        samp = {"temperature": synth.TEMPERATURE, "top_k": synth.TOP_K, "seed": synth.SAMPLER_SEED}
        tokens_per_step = B * (T + n_gen - 1)

        def step():
            rlt.rlt_state_reset(state)
            rlt.rlt_prefill(model, state, tok)
            rlt.rlt_readout(model, state, sampling=samp, sampled=ids[0], logp_sampled=lps[0], logmu=lmu[0])
            for i in range(1, n_gen):
                rlt.rlt_decoder_step(model, state, tokens=ids[i - 1], sampling=samp, sampled=ids[i],
                                     logp_sampled=lps[i], logmu=lmu[i])

        def step_e2e():
            tok.copy_(tok_host, non_blocking=True)
            step()
            ids_host.copy_(ids, non_blocking=True)

        h2d, d2h = tok_host.numel() * 4, ids_host.numel() * 4

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, k, profile=False):
        barrier()
        torch.cuda.synchronize()
        if profile:
            rlt.rlt_profile_enable(model, True)
        n0 = rlt.rlt_kernel_launches()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.nvtx.range_push("timed" if profile else "timed_e2e")  # lets ncu select the timed launches
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        launches = rlt.rlt_kernel_launches() - n0
        ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        barrier()
        return ms, launches

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rlt.rlt_check_device()

    clocks = ClockSampler(dev.index)
    clocks.start()
    ms, launches = timed(step, args.steps, profile=True)
    clk = clocks.stop()
    a_ms, a_n, a_bytes = rlt.rlt_profile_read(model, 0)
    s_ms, s_n, s_bytes = rlt.rlt_profile_read(model, 1)
    rlt.rlt_profile_enable(model, False)
    ms_e2e, _ = timed(step_e2e, args.steps)
    rlt.rlt_check_device()

    # the library times the attention launches of every 4th position; scale
    # the sampled time up to all launches of the timed steps for the share
    L = w["n_layers"]
    if kind == "replay":
        n_prefix = n_swa = L * (w["prompt"] - 1) * args.steps
    else:
        n_dec = w["prompt"] + w["gen"] - 1
        n_prefix = (L * n_dec + L * (w["gen"] - 1)) * args.steps
        n_swa = L * n_dec * args.steps
    value = world * tokens_per_step * args.steps / (ms / 1e3)
    e2e = world * tokens_per_step * args.steps / (ms_e2e / 1e3)
    roof = step_roofline(w, kind, peaks)
    ms_step = ms / args.steps
    achieved = (a_bytes / a_n) / ((a_ms / a_n) / 1e3) / 1e9 if a_n else None
    return {
        "value": value, "ms_per_step": ms_step, "e2e": e2e, "h2d": h2d, "d2h": d2h, "launches": launches,
        "clocks": clk, "attn": {"ms": a_ms, "n": a_n, "bytes": a_bytes, "gbs": achieved,
                                "ms_all": a_ms * n_prefix / a_n if a_n else None},
        "swa": {"ms": s_ms, "n": s_n, "bytes": s_bytes,
                "gbs": (s_bytes / s_n) / ((s_ms / s_n) / 1e3) / 1e9 if s_n else None,
                "ms_all": s_ms * n_swa / s_n if s_n else None},
        "step_roofline": {"bound_ms": roof["bound_ms"], "frac": roof["bound_ms"] / ms_step},
        "tokens_per_step": tokens_per_step,
    }


def run_backward(args, w: dict, rank: int, world: int) -> dict:
    """Times rlt_replay_backward (eq. 5.1 weights) over the workload's token
    ids, already resident on the device: K calls after W warm-up calls."""
    import torch
    import stateful_decoder_b200 as rlt

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    model = rlt.rlt_init_weights(synth.model_config(w), synth.WEIGHT_SEED)
    tok = torch.from_numpy(shard_tokens(w, rank, world)).cuda()
    B, S = tok.shape
    wts = torch.full((B, S - 1), 1.0 / (B * (S - 1)), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        rlt.rlt_replay_backward(model, tok, wts, segment=BPTT_SEGMENT)
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    clocks = ClockSampler(dev.index)
    clocks.start()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    n0 = rlt.rlt_kernel_launches()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        rlt.rlt_replay_backward(model, tok, wts, segment=BPTT_SEGMENT)
    e1.record(stream)
    torch.cuda.synchronize()
    launches = rlt.rlt_kernel_launches() - n0
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    clk = clocks.stop()
    rlt.rlt_check_device()
    return {"value": world * B * (S - 1) * args.steps / (ms / 1e3), "ms_per_step": ms / args.steps,
            "launches": launches, "clocks": clk, "B": B, "S": S}


def read_traffic_ratio() -> tuple[float | None, str]:
    """DRAM bytes per algorithmic byte of the prefix-attention kernel from the
    committed ncu summary, with a note.  The summary records the SHA-1 of the
    kernel's source file at capture time; if the source has changed since,
    the counters no longer describe the kernel and the ratio is None."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "prefix_attn_replay.md")
    if not os.path.exists(p):
        return None, "no ncu summary"
    ratio, sha = None, None
    for line in open(p):
        if line.startswith("traffic_per_algorithmic_byte:"):
            v = line.split(":", 1)[1].strip()
            ratio = None if v in ("", "null") else float(v)
        elif line.startswith("kernel_source_sha1:"):
            sha = line.split(":", 1)[1].strip()
    src = os.path.join(ROOT, "stateful_decoder_b200", "csrc", "attn_decode.cu")
    now = hashlib.sha1(open(src, "rb").read()).hexdigest()
    if sha != now:
        return None, "kernel source changed since the ncu capture in profiles/prefix_attn_replay.md"
    return ratio, "from profiles/prefix_attn_replay.md, scaled to the mean timed launch"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="replay", choices=sorted(BENCH_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    wname, over, kind = BENCH_WORKLOADS[args.workload]
    w = synth.workload(wname, **over)
    peaks = load_peaks()
    cfg_desc = {"workload": args.workload, "d": w["d"], "n_heads": w["n_heads"], "layers": f"{w['n_layers']}+{w['n_layers']}",
                "window": w["window"], "groups": w["groups"], "ffn": w["ffn"], "vocab": w["vocab"],
                "batch_per_gpu": w["batch"], "global_batch": w["batch"] * world,
                "tokens": w["prompt"] if kind == "replay" else f"{w['prompt']}+{w['gen']}",
                "schedule": "replay (teacher-forced)" if kind == "replay" else "prefill + sampled generation",
                "merge": "paper eqs. 2.9-2.11", "l2": "inputs larger than L2 (KV state of several GB per step)",
                "parallelism": f"dp{world} (independent sequences, no collective)"}

    if args.impl == "reference":
        # the reference arm is the fp64 oracle on the host cores (rank 0 only)
        if rank != 0:
            return
        n_tok = oracle_tokens_for(w)
        sample = oracle_sample
        if kind == "backward":
            n_tok, sample = min(n_tok, 16), oracle_bptt_sample
        for _ in range(args.warmup):
            sample(w, n_tok)
        vals = []
        t0 = time.perf_counter()
        for i in range(args.steps):
            v, cores, desc = sample(w, n_tok, seed_seq=i)
            vals.append(v)
        dt = time.perf_counter() - t0
        value = statistics.mean(vals)
        print(json.dumps({
            "impl": "reference", "metric": BPTT_METRIC if kind == "backward" else METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg_desc,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }), flush=True)
        return

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=timedelta(seconds=600))

    if kind == "backward":
        r = run_backward(args, w, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({
                "metric": BPTT_METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic (seeded Zipf(1.1) token ids, random-init weights)",
                "config": dict(cfg_desc, tokens=r["S"], schedule=f"full BPTT, segments of {BPTT_SEGMENT}",
                               objective="eq. 5.1 weights"),
                "roofline": None, "note": "first backward engine (CUDA-core functor kernels), not yet characterised",
                "gpu_launches": r["launches"], "clocks": r["clocks"]}), flush=True)
        return

    r = run_gpu(args, w, kind, peaks, rank, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_tok = oracle_tokens_for(w)
        v, cores, desc = oracle_sample(w, n_tok)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    ratio, traffic_note = read_traffic_ratio()
    a = r["attn"]
    traffic = ratio * (a["bytes"] / a["n"]) if (ratio is not None and a["n"]) else None
    line = {
        "metric": METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Zipf(1.1) token ids, random-init weights)",
        "config": cfg_desc,
        "roofline": {"bound": "hbm", "kernel": "prefix_attn (cross-attention over M_<=t)",
                     "achieved": a["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": (a["gbs"] / peaks["hbm_gbs"]) if a["gbs"] else None, "traffic": traffic,
                     "traffic_note": traffic_note,
                     "peak_source": peaks["source"] + " (copy bandwidth)",
                     "timed_launches": a["n"], "sampling": "launches at every 4th position, CUDA events",
                     "share_of_step": a["ms_all"] / (r["ms_per_step"] * args.steps) if a["ms_all"] else None},
        "swa_attn": {"achieved_gbs": r["swa"]["gbs"],
                     "share_of_step": r["swa"]["ms_all"] / (r["ms_per_step"] * args.steps) if r["swa"]["ms_all"] else None},
        "step_roofline": r["step_roofline"],
        "cpu_baseline": cpu,
        "e2e": {"value": r["e2e"], "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
