"""Benchmark of the RLT decoder hot path on B200 GPUs.

Default workload (one GPU): the reference-depth model, L_E = L_D = 48 tied
(d=2048, 16x128 heads, W=256, G=1, F=5632, V=32000, bf16), B = 128 sequences
per GPU.  A 2048-token prompt is prefilled (token-parallel encoder, memory
projection and 2048 decoder transitions) before the timed region; one step is
then a block of 32 sampled generation transitions continuing from the state:
for every sequence, the encoder step over the cache C^E (eq. 2.8), the memory
append, the merge, the 48 decoder blocks and the readout with the behaviour
sampler (temperature 0.8, top-k 50).  The metric is decoder tokens/s =
B x 32 x steps / time.  The warm-up blocks come first, so the timed positions
follow them (t = 2048 + 32*warmup + 1 ...).  The full 2048 + 2048 schedule at
B = 128 needs about 229 GB of state and does not fit one GPU; the positions
reached here stay well inside it.

Other workloads (--workload): `replay` (the reference width at L = 24,
B = 256 x 1024 tokens, one rlt_replay_logprobs call per step), `layerwise`,
`small`, `refdepth-b64` (one whole prefill + generation per step) and
`bptt-small` and `bptt-replay` (full-BPTT backward).

Multi-GPU (torchrun): sequences shard across ranks with no data-path
collective during the timed steps (weak scaling, B sequences per rank);
timing is the max over ranks, and the shards' results are all-gathered once
at the end of the run.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

BENCH_WORKLOADS = {
    # name: (synth workload, overrides, kind)
    "refdepth": ("refdepth", {"block": 32}, "block"),
    "replay": ("replay", {}, "replay"),
    "layerwise": ("layerwise", {}, "replay"),
    "small": ("small", {}, "generate"),
    "refdepth-b64": ("refdepth", {"batch": 64}, "generate"),
    # full-BPTT forward + backward (rlt_replay_backward) of the small model
    "bptt-small": ("small", {"prompt": 256, "gen": 0}, "backward"),
    # the same at the reference width (d=2048, 24+24 layers), 16 sequences
    "bptt-replay": ("replay", {"batch": 16, "prompt": 256, "gen": 0}, "backward"),
}
DEFAULT_WORKLOAD = "refdepth"
BPTT_METRIC = "RLT full-BPTT tokens/s (replay forward + backward through the whole history) on 1 B200"
BPTT_SEGMENT = 32
# decode-attention launches recorded with CUDA events by the library in the
# profiling pass (every 4th position), then scaled to all launches
PROFILE_STRIDE = 4
# profiling blocks that follow the timed ones (block workloads)
PROFILE_BLOCKS = 2
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def metric_name(w: dict, kind: str) -> str:
    """The metric string names the model actually run: a line never claims
    48+48 unless the 48-layer model ran."""
    L = w["n_layers"]
    tie = "tied" if w.get("tied", 1) else "untied"
    extra = ", teacher-forced replay" if kind == "replay" else ""
    return f"RLT decoder tokens/s (B seqs, {L}+{L} {tie}{extra}) on 1 B200; % of step roofline"


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- roofline model
def params(w: dict) -> tuple[int, int]:
    """Weights streamed by one decoder transition (with its readout) and by one
    encoder step (with the memory projection)."""
    d, L, F, V, G = w["d"], w["n_layers"], w["ffn"], w["vocab"], w["groups"]
    merge = 3 * d * d if w.get("merge_kind", 0) == 0 else 2 * d * d
    p_dec = L * (4 * d * d + 2 * d * d + 3 * d * F) + merge + V * d
    p_enc = L * (4 * d * d + 3 * d * F) + 2 * d * d * G
    return p_dec, p_enc


def transition_bound_s(w: dict, t: int, gen: bool, peaks: dict) -> float:
    """Analytic lower bound of one decoder transition at position t for B
    sequences: the slower of (weights + KV bytes)/HBM and FLOPs/tensor peak.
    KV bytes: SWA ring read (min(t,W)-1 entries) and insert, memory M_<=t
    read; with the encoder step (gen) also the C^E_<=t read, its insert and
    the memory append."""
    d, L, G, W, B = w["d"], w["n_layers"], w["groups"], w["window"], w["batch"]
    eb = 2 if w["dtype"] == 1 else 4
    p_dec, p_enc = params(w)
    kv = B * eb * 2 * d * (L * (min(t, W) - 1) + L + L * t)
    wbytes = eb * p_dec
    flops = 2 * B * p_dec + 4 * B * d * (L * min(t, W) + L * t)
    if gen:
        kv += B * eb * 2 * d * (L * t + L + G)
        wbytes += eb * p_enc
        flops += 2 * B * p_enc + 4 * B * d * L * t
    return max((kv + wbytes) / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops_sustained"] * 1e12))


def encoder_bound_s(w: dict, T: int, peaks: dict) -> float:
    """Token-parallel encoder + memory projection over T tokens at tensor peak."""
    _, p_enc = params(w)
    flops = 2 * w["batch"] * T * p_enc + 4 * w["batch"] * w["n_layers"] * w["d"] * T * T / 2
    return flops / (peaks["bf16_tflops_sustained"] * 1e12)


def step_roofline(w: dict, kind: str, peaks: dict, t_range: tuple[int, int] | None = None) -> dict:
    """Analytic bound of one step, in ms (see transition_bound_s).
    replay: encoder over S tokens + transitions 1..S-1; generate: encoder over
    the prompt + transitions 1..T (prefill) and T+1..T+n_gen-1 (with encoder
    steps); block: the generation transitions t_range[0]..t_range[1]
    inclusive, averaged per block of w['block']."""
    if kind == "replay":
        S = w["prompt"]
        total = encoder_bound_s(w, S, peaks) + sum(transition_bound_s(w, t, False, peaks) for t in range(1, S))
        return {"bound_ms": total * 1e3, "decoder_transitions": S - 1}
    if kind == "generate":
        T, n_gen = w["prompt"], w["gen"]
        total = encoder_bound_s(w, T, peaks)
        total += sum(transition_bound_s(w, t, t > T, peaks) for t in range(1, T + n_gen))
        return {"bound_ms": total * 1e3, "decoder_transitions": T + n_gen - 1}
    a, b = t_range
    total = sum(transition_bound_s(w, t, True, peaks) for t in range(a, b + 1))
    n_blocks = (b - a + 1) / w["block"]
    return {"bound_ms": total * 1e3 / n_blocks, "decoder_transitions": w["block"]}


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


def gather_rows(x, world: int):
    """The optional end-of-run collective of the sharded path: every rank's
    per-sequence results (rows, dim 0) gathered, in rank order, into one
    [world * rows, ...] tensor on every rank (NCCL on GPUs, gloo on CPU).
    Nothing is exchanged during the timed steps."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    x = x.contiguous()
    parts = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(parts, x)
    return torch.cat(parts)


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


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ---------------------------------------------------------------- CPU oracle leg
# Every oracle sample is bounded: the fp64 oracle streams the whole model per
# token (about 13 GFLOP per token at the reference depth), so a sample is a
# few short sequences, not the benchmarked batch.
ORACLE_SAMPLE = {
    # kind: (sequences, prompt tokens, generated tokens); replay/generate use (sequences, tokens)
    "block": (2, 6, 6),
}


def oracle_model(w: dict):
    import oracle
    return oracle.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)


def oracle_sample(w: dict, kind: str, om, seed_seq: int = 0) -> tuple[float, int, str]:
    """Times the fp64 oracle on a bounded sample of the workload and returns
    (decoder transitions/s, threads, description).  block: a few sequences
    with a short prompt and sampled generation (prefill, then encoder step +
    transition + sampler per token, as the timed GPU step does); otherwise a
    teacher-forced replay of one sequence truncated to a prefix."""
    import oracle
    if kind == "block":
        n_seq, n_prompt, n_new = ORACLE_SAMPLE["block"]
        tok = synth.tokens(w, batch=n_seq, length=n_prompt, seed=w["data_seed"] + 17 * seed_seq)
        t0 = time.perf_counter()
        for b in range(n_seq):
            om.generate(tok[b], n_new, synth.TEMPERATURE, synth.TOP_K, synth.SAMPLER_SEED, b)
        dt = time.perf_counter() - t0
        n = n_seq * (n_prompt + n_new - 1)
        return (n / dt, oracle.num_threads(),
                f"{n_seq} sequences x ({n_prompt}-token prompt + {n_new} sampled tokens) from BOS = {n} transitions, "
                f"fp64; positions t <= {n_prompt + n_new - 1}, so its attention work per token is lower than at the "
                f"benched positions")
    n_tok = oracle_tokens_for(w)
    tok = synth.tokens(w, batch=1, length=n_tok, seed=w["data_seed"] + seed_seq)[0]
    t0 = time.perf_counter()
    om.replay_logprobs(tok)
    dt = time.perf_counter() - t0
    return (n_tok - 1) / dt, oracle.num_threads(), f"1 sequence x {n_tok} tokens (teacher-forced replay), fp64"


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
def run_gpu(args, w: dict, kind: str, peaks: dict, rank: int, world: int) -> dict:
    import torch
    import torch.distributed as dist
    import stateful_decoder_b200 as rlt

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    cfg = synth.model_config(w)
    B = w["batch"]
    model = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    stream = torch.cuda.current_stream()
    samp = {"temperature": synth.TEMPERATURE, "top_k": synth.TOP_K, "seed": synth.SAMPLER_SEED}
    setup = None  # untimed preparation before a pass (block workloads: the prompt prefill)
    after_warmup = None  # untimed hook between the warm-up and the timed e2e steps
    t_range = None

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
        n_prof = 1
        result = lambda: (logp, "teacher-forced log-probs [B, S-1] fp32")  # noqa: E731
        # decode-attention launches of one step: prefix (memory), SWA
        launches_per_step = (w["n_layers"] * (S - 1), w["n_layers"] * (S - 1))
    elif kind == "generate":
        T, n_gen = w["prompt"], w["gen"]
        state = rlt.rlt_state_create(model, B, T + n_gen, rlt.STATE_ENCODER_CACHE | rlt.STATE_GRAPHS)
        tok_host = torch.from_numpy(shard_tokens(w, rank, world)).pin_memory()
        tok = tok_host.cuda()
        ids = torch.zeros(n_gen, B, dtype=torch.int32, device=dev)
        lmu = torch.zeros(n_gen, B, device=dev)
        lps = torch.zeros(n_gen, B, device=dev)
        ids_host = torch.zeros(n_gen, B, dtype=torch.int32).pin_memory()
        tokens_per_step = B * (T + n_gen - 1)

        def step():
            rlt.rlt_state_reset(state)
            rlt.rlt_prefill(model, state, tok)
            rlt.rlt_readout(model, state, sampling=samp, sampled=ids[0], logp_sampled=lps[0], logmu=lmu[0])
            for i in range(1, n_gen):
                # consumes the token the previous readout sampled (pending in
                # the state), so every position shares one token source and
                # the step graphs differ only by the attention chunk count
                rlt.rlt_decoder_step(model, state, sampling=samp, sampled=ids[i], logp_sampled=lps[i], logmu=lmu[i])

        def step_e2e():
            tok.copy_(tok_host, non_blocking=True)
            step()
            ids_host.copy_(ids, non_blocking=True)

        h2d, d2h = tok_host.numel() * 4, ids_host.numel() * 4
        n_prof = 1
        result = lambda: (ids.t(), "sampled token ids [B, generated] int32")  # noqa: E731
        n_dec = T + n_gen - 1
        launches_per_step = (w["n_layers"] * n_dec + w["n_layers"] * (n_gen - 1), w["n_layers"] * n_dec)
    else:  # block: prompt prefilled untimed, then blocks of sampled transitions
        T, blk = w["prompt"], w["block"]
        n_blocks = args.warmup + args.steps + PROFILE_BLOCKS
        max_len = T + blk * n_blocks
        # decoder steps replay one CUDA graph per step shape (bit-identical to
        # plain launches)
        state = rlt.rlt_state_create(model, B, max_len, rlt.STATE_ENCODER_CACHE | rlt.STATE_GRAPHS)
        tok = torch.from_numpy(shard_tokens(w, rank, world)).cuda()
        ids = torch.zeros(blk, B, dtype=torch.int32, device=dev)
        lmu = torch.zeros(blk, B, device=dev)
        lps = torch.zeros(blk, B, device=dev)
        ids_host = torch.zeros(blk, B, dtype=torch.int32).pin_memory()
        lmu_host = torch.zeros(blk, B).pin_memory()
        first = torch.zeros(B, dtype=torch.int32, device=dev)
        tokens_per_step = B * blk
        t_range = (T + blk * args.warmup + 1, T + blk * (args.warmup + args.steps))

        def setup():
            # H_T after the prompt (App. A.1) and the first sampled token,
            # which stays pending in the state and is copied to the host
            rlt.rlt_state_reset(state)
            rlt.rlt_prefill(model, state, tok)
            rlt.rlt_readout(model, state, sampling=samp, sampled=ids[blk - 1], logp_sampled=lps[blk - 1],
                            logmu=lmu[blk - 1])
            ids_host.copy_(ids)

        def step():
            # each transition consumes the token the previous readout sampled
            for i in range(blk):
                rlt.rlt_decoder_step(model, state, sampling=samp, sampled=ids[i], logp_sampled=lps[i], logmu=lmu[i])

        def step_e2e():
            # the block's first tokens come from the host (what a serving
            # loop holds after reading back the previous block), the block's
            # sampled ids and behaviour log-probs go back to the host
            first.copy_(ids_host[blk - 1], non_blocking=True)
            rlt.rlt_decoder_step(model, state, tokens=first, sampling=samp, sampled=ids[0], logp_sampled=lps[0],
                                 logmu=lmu[0])
            for i in range(1, blk):
                rlt.rlt_decoder_step(model, state, sampling=samp, sampled=ids[i], logp_sampled=lps[i], logmu=lmu[i])
            ids_host.copy_(ids, non_blocking=True)
            lmu_host.copy_(lmu, non_blocking=True)

        def after_warmup():
            ids_host.copy_(ids)  # the host holds the last block's ids, as a serving loop would

        h2d, d2h = first.numel() * 4, ids_host.numel() * 4 + lmu_host.numel() * 4
        n_prof = PROFILE_BLOCKS
        result = lambda: (ids.t(), "last block's sampled token ids [B, 32] int32")  # noqa: E731
        # prefix attention: encoder step over C^E and cross-attention over M; SWA
        launches_per_step = (2 * w["n_layers"] * blk, w["n_layers"] * blk)

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(fn, k):
        barrier()
        torch.cuda.synchronize()
        n0 = rlt.rlt_kernel_launches()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        launches = rlt.rlt_kernel_launches() - n0
        ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        barrier()
        return ms, launches

    if setup:
        setup()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    rlt.rlt_check_device()

    # timed pass: instrumentation off
    clocks = ClockSampler(dev.index)
    clocks.start()
    ms, launches = timed(step, args.steps)
    clk = clocks.stop()

    # profiling pass (not timed): the library records CUDA events around the
    # decode-attention launches of every 4th position
    rlt.rlt_profile_enable(model, True)
    for _ in range(n_prof):
        step()
    torch.cuda.synchronize()
    a_ms, a_n, a_bytes = rlt.rlt_profile_read(model, 0)
    s_ms, s_n, s_bytes = rlt.rlt_profile_read(model, 1)
    rlt.rlt_profile_enable(model, False)
    rlt.rlt_check_device()

    # end-to-end pass through the public API with host copies in the timed region
    if setup:
        setup()
        for _ in range(args.warmup):
            step()
        after_warmup()
    ms_e2e, _ = timed(step_e2e, args.steps)
    rlt.rlt_check_device()

    # untimed: the shards' results gathered once at the end of the run
    res, what = result()
    gathered = gather_rows(res, world)
    collective = None if world <= 1 else {
        "end_of_run_all_gather": what, "rows": int(gathered.shape[0]),
        "bytes": int(gathered.numel() * gathered.element_size())}

    value = world * tokens_per_step * args.steps / (ms / 1e3)
    e2e = world * tokens_per_step * args.steps / (ms_e2e / 1e3)
    roof = step_roofline(w, kind, peaks, t_range)
    free_b, total_b = torch.cuda.mem_get_info(dev)  # the state, weights and workspaces are all still held
    ms_step = ms / args.steps

    def share(ms_sampled, n_sampled, per_step, scale=1.0):
        # mean sampled launch time x launches of one step / step time
        return (ms_sampled / n_sampled) * per_step / ms_step * scale if n_sampled else None

    # The block workload profiles the blocks after the timed ones, where every
    # prefix-attention launch reads more keys (t of them: C^E_<=t and
    # M_<=t); its share is scaled to the timed positions by the ratio of mean
    # key counts.  The SWA ring is full at both, and the other workloads
    # profile the same schedule they time.
    key_scale, share_note = 1.0, "profiled and timed positions are the same schedule"
    if kind == "block":
        key_scale, share_note = block_share_scale(t_range, w["block"], n_prof)

    def gbs(nbytes, ms_sampled, n_sampled):
        return (nbytes / n_sampled) / ((ms_sampled / n_sampled) / 1e3) / 1e9 if n_sampled else None

    return {
        "value": value, "ms_per_step": ms_step, "e2e": e2e, "h2d": h2d, "d2h": d2h, "launches": launches,
        "clocks": clk, "t_range": t_range,
        "attn": {"ms": a_ms, "n": a_n, "bytes": a_bytes, "gbs": gbs(a_bytes, a_ms, a_n),
                 "share": share(a_ms, a_n, launches_per_step[0], key_scale), "share_note": share_note},
        "swa": {"gbs": gbs(s_bytes, s_ms, s_n), "share": share(s_ms, s_n, launches_per_step[1])},
        "step_roofline": {"bound_ms": roof["bound_ms"], "frac": roof["bound_ms"] / ms_step},
        "tokens_per_step": tokens_per_step,
        "memory": {"device_used_gib": (total_b - free_b) / 2**30, "device_total_gib": total_b / 2**30},
        "collective": collective,
    }


def block_share_scale(t_range: tuple[int, int], blk: int, n_prof: int) -> tuple[float, str]:
    """Factor from the profiled to the timed positions of the block workload
    for the prefix-attention share: the profiling pass runs the n_prof blocks
    after the timed positions t_range, sampling every PROFILE_STRIDE-th
    position, and a launch at position t reads t keys (C^E_<=t, M_<=t)."""
    t_hi = t_range[1]
    prof_t = [t for t in range(t_hi + 1, t_hi + blk * n_prof + 1) if t % PROFILE_STRIDE == 0]
    scale = ((t_range[0] + t_range[1]) / 2) / (sum(prof_t) / len(prof_t))
    note = (f"profiled launches at t={prof_t[0]}..{prof_t[-1]} (every {PROFILE_STRIDE}th), scaled by "
            f"{scale:.4f} = mean attended keys at the timed t={t_range[0]}..{t_range[1]} / at the profiled t")
    return scale, note


def backward_flops(w: dict, B: int, S: int) -> float:
    """Contraction FLOPs of one full-BPTT call (rlt_replay_backward) over B
    sequences of S tokens: the encoder and memory projection forward once and
    backward once (dX and dW: twice the forward), the S-1 decoder transitions
    forward twice (the sweep and the segment recompute) and backward once
    (dX and dW)."""
    p_dec, p_enc = params(w)
    n = B * S
    return 2.0 * n * p_enc * 3 + 2.0 * B * (S - 1) * p_dec * 4


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
    free_b, total_b = torch.cuda.mem_get_info(dev)  # the kept backward buffers are still held
    return {"value": world * B * (S - 1) * args.steps / (ms / 1e3), "ms_per_step": ms / args.steps,
            "launches": launches, "clocks": clk, "B": B, "S": S,
            "memory": {"device_used_gib": (total_b - free_b) / 2**30, "device_total_gib": total_b / 2**30}}


def read_traffic_ratio() -> tuple[float | None, str]:
    """DRAM bytes per algorithmic byte of the prefix-attention kernel, from the
    machine-readable record of the committed ncu capture.  The record holds
    the SHA-1 of the kernel's source file at capture time; if the source has
    changed since, the counters no longer describe the kernel and the ratio
    is None."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, "no ncu traffic record"
    rec = json.load(open(TRAFFIC_FILE)).get("prefix_attn")
    if not rec:
        return None, "no ncu traffic record for prefix_attn"
    src = os.path.join(ROOT, rec["source"])
    now = hashlib.sha1(open(src, "rb").read()).hexdigest()
    if rec["source_sha1"] != now:
        return None, "kernel source changed since the ncu capture"
    return rec["traffic_per_algorithmic_byte"], (f"ncu capture ({rec['case']}): DRAM bytes / algorithmic bytes, "
                                                 f"scaled to the mean profiled launch")


def config_desc(args, w: dict, kind: str, world: int) -> dict:
    if kind in ("replay", "backward"):
        tokens, schedule = w["prompt"], "replay (teacher-forced)"
    elif kind == "generate":
        tokens, schedule = f"{w['prompt']}+{w['gen']}", "prefill + sampled generation"
    else:
        a = w["prompt"] + w["block"] * args.warmup + 1
        b = w["prompt"] + w["block"] * (args.warmup + args.steps)
        tokens = f"prompt {w['prompt']} prefilled untimed; step = {w['block']} sampled transitions; timed t={a}..{b}"
        schedule = "sampled generation (encoder step + memory append + transition + readout/sampler per token)"
    return {"workload": args.workload, "d": w["d"], "n_heads": w["n_heads"],
            "layers": f"{w['n_layers']}+{w['n_layers']}", "window": w["window"], "groups": w["groups"],
            "ffn": w["ffn"], "vocab": w["vocab"], "batch_per_gpu": w["batch"], "global_batch": w["batch"] * world,
            "tokens": tokens, "schedule": schedule, "merge": "paper eqs. 2.9-2.11",
            "sampler": f"temperature {synth.TEMPERATURE}, top-k {synth.TOP_K}" if kind != "replay" else None,
            "l2": "inputs larger than L2 (KV state of tens of GB read per transition)",
            "parallelism": f"dp{world} (independent sequences, no collective)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(BENCH_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    wname, over, kind = BENCH_WORKLOADS[args.workload]
    w = synth.workload(wname, **over)
    peaks = load_peaks()
    cfg_desc = config_desc(args, w, kind, world)
    metric = BPTT_METRIC if kind == "backward" else metric_name(w, kind)

    if args.impl == "reference":
        # the reference arm is the fp64 oracle on the host cores (rank 0 only)
        if rank != 0:
            return
        vals = []
        if kind == "backward":
            n_tok = min(oracle_tokens_for(w), 16)
            for _ in range(args.warmup):
                oracle_bptt_sample(w, n_tok)
            t0 = time.perf_counter()
            for i in range(args.steps):
                v, cores, desc = oracle_bptt_sample(w, n_tok, seed_seq=i)
                vals.append(v)
        else:
            om = oracle_model(w)
            for _ in range(args.warmup):
                oracle_sample(w, kind, om)
            t0 = time.perf_counter()
            for i in range(args.steps):
                v, cores, desc = oracle_sample(w, kind, om, seed_seq=i)
                vals.append(v)
        dt = time.perf_counter() - t0
        value = statistics.mean(vals)
        print(json.dumps({
            "impl": "reference", "metric": metric, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg_desc,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc,
                             "cpu": cpu_model()},
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
        fl = backward_flops(w, r["B"], r["S"])
        tf = fl / (r["ms_per_step"] / 1e3) / 1e12
        pk = peaks["bf16_tflops_sustained"]
        roof = {"bound": "tensor", "kernel": "whole backward: contraction FLOPs at the bf16 tensor peak",
                "flops_per_step": fl, "achieved": tf, "peak": pk, "unit": "TFLOP/s", "frac": tf / pk,
                "traffic": None, "peak_source": peaks["source"] + " (sustained bf16 GEMM)"}
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({
                "metric": BPTT_METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded Zipf(1.1) token ids, random-init weights)",
                "config": dict(cfg_desc, tokens=r["S"], schedule=f"full BPTT, segments of {BPTT_SEGMENT}",
                               objective="eq. 5.1 weights",
                               arithmetic="contractions on tcgen05 with bf16 operands, fp32 accumulation; "
                                          "attention, norms and elementwise adjoints on CUDA cores in fp32"),
                "roofline": roof, "gpu_launches": r["launches"], "clocks": r["clocks"],
                "memory": r["memory"]}), flush=True)
        return

    r = run_gpu(args, w, kind, peaks, rank, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        om = oracle_model(w)
        v, cores, desc = oracle_sample(w, kind, om)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc, "cpu": cpu_model()}

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
        "metric": metric, "value": r["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Zipf(1.1) token ids, random-init weights)",
        "config": cfg_desc,
        "roofline": {"bound": "hbm",
                     "kernel": "prefix_attn (encoder step over C^E and cross-attention over M_<=t)",
                     "achieved": a["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": (a["gbs"] / peaks["hbm_gbs"]) if a["gbs"] else None, "traffic": traffic,
                     "traffic_note": traffic_note,
                     "peak_source": peaks["source"] + " (copy bandwidth)",
                     "profiled_launches": a["n"],
                     "sampling": f"separate untimed pass: launches at every {PROFILE_STRIDE}th position, CUDA events",
                     "share_of_step": a["share"], "share_note": a["share_note"]},
        "swa_attn": {"achieved_gbs": r["swa"]["gbs"], "share_of_step": r["swa"]["share"]},
        "step_roofline": r["step_roofline"],
        "cpu_baseline": cpu,
        "e2e": {"value": r["e2e"], "unit": "tokens/s", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
        "memory": r["memory"],
        "collective": r["collective"],
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
