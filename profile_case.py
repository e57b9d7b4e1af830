"""Profiling helpers for librlt (a benchmark companion, not part of the
library), used to make the ncu summaries in profiles/.  Each case runs the
launches to be captured between cudaProfilerStart/Stop, so that
`ncu --profile-from-start off --clock-control none -k <kernel> -c 1` captures
one launch of a chosen kernel on a small case.  --layers keeps every kernel
shape of the workload's model but holds fewer layers' state.

  python profile_case.py step --workload replay --batch 64 --len 640 --t 601 [--layers 2]
      Encodes `len` tokens of `batch` sequences, applies t-1 decoder
      transitions, then profiles transition t (no encoder step).

  python profile_case.py gen --workload refdepth --batch 64 --len 1200 --t 1203 [--layers 2]
      Prefills `len` tokens, samples up to position t-1 through the
      generation path, then profiles the generation step at t: the encoder
      step over the cache C^E, the memory append, the transition and the
      readout with the sampler.

  python profile_case.py encoder --workload refdepth --batch 4 --len 2048 [--layers 1]
      Profiles the token-parallel encoder and memory projection over `len`
      tokens of `batch` sequences (GEMMs with B*len activation rows, causal
      attention on the tensor cores).

  python profile_case.py bptt --workload small --batch 16 --len 64 [--layers 2] [--eager]
      Profiles one full-BPTT backward (rlt_replay_backward, eq. 5.1 weights,
      segments of 32) of `batch` sequences of `len` tokens: the second call
      of its size (the replay of the captured graph), or with --eager a
      first call again (direct launches; the NVTX range "rlt_weight_grads"
      then marks each segment's weight-gradient contractions).

  python profile_case.py summarize launches.csv [S]
      Per-kernel summary of an ncu launch list (gpu__time_duration.sum, --csv)
      captured with `--nvtx --nvtx-include "rlt_sample]"` on a replay of S
      tokens: the library wraps the token-parallel encoder and every position
      t = 64 (mod 128) in that range while profiling is enabled, so the list
      holds the encoder once and a stratified sample of positions; each sampled
      position stands for the positions of its 128-wide stratum.
"""
from __future__ import annotations

import argparse
import collections
import csv
import os
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def step(args) -> None:
    import torch

    import stateful_decoder_b200 as rlt
    import synth
    over = dict(batch=args.batch, prompt=args.len)
    if args.layers:
        over["n_layers"] = args.layers  # same kernel shapes, fewer layers' state on the device
    w = synth.workload(args.workload, **over)
    m = rlt.rlt_init_weights(synth.model_config(w), synth.WEIGHT_SEED)
    tok = torch.from_numpy(synth.tokens(w)).cuda()
    st = rlt.rlt_state_create(m, args.batch, args.len, 0)
    rlt.rlt_encode_prefix(m, st, tok)
    for _ in range(1, args.t):
        rlt.rlt_decoder_step(m, st)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStart()
    rlt.rlt_decoder_step(m, st)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStop()
    rlt.rlt_check_device()
    print("profiled transition", st.info()["n_dec"])


def _model(args):
    import stateful_decoder_b200 as rlt
    import synth
    over = dict(batch=args.batch, prompt=args.len)
    if args.layers:
        over["n_layers"] = args.layers
    w = synth.workload(args.workload, **over)
    return rlt, w, rlt.rlt_init_weights(synth.model_config(w), synth.WEIGHT_SEED)


def gen(args) -> None:
    import torch

    import synth
    rlt, w, m = _model(args)
    tok = torch.from_numpy(synth.tokens(w)).cuda()
    st = rlt.rlt_state_create(m, args.batch, args.t, rlt.STATE_ENCODER_CACHE)
    samp = {"temperature": synth.TEMPERATURE, "top_k": synth.TOP_K, "seed": synth.SAMPLER_SEED}
    ids = torch.zeros(args.batch, dtype=torch.int32, device="cuda")
    rlt.rlt_prefill(m, st, tok)
    rlt.rlt_readout(m, st, sampling=samp, sampled=ids)
    for _ in range(args.len + 1, args.t):
        rlt.rlt_decoder_step(m, st, sampling=samp, sampled=ids)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStart()
    rlt.rlt_decoder_step(m, st, sampling=samp, sampled=ids)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStop()
    rlt.rlt_check_device()
    print("profiled generation step", st.info()["n_dec"])


def encoder(args) -> None:
    import torch

    import synth
    rlt, w, m = _model(args)
    tok = torch.from_numpy(synth.tokens(w)).cuda()
    st = rlt.rlt_state_create(m, args.batch, args.len, 0)
    rlt.rlt_encode_prefix(m, st, tok)  # first pass allocates the encoder workspace
    rlt.rlt_state_reset(st)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStart()
    rlt.rlt_encode_prefix(m, st, tok)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStop()
    rlt.rlt_check_device()
    print("profiled encoder over", args.batch, "x", args.len, "tokens")


def bptt(args) -> None:
    import torch

    import synth
    rlt, w, m = _model(args)
    tok = torch.from_numpy(synth.tokens(w)).cuda()
    B, S = tok.shape
    wts = torch.full((B, S - 1), 1.0 / (B * (S - 1)), device="cuda")
    rlt.rlt_replay_backward(m, tok, wts, segment=32)  # warm-up
    torch.cuda.synchronize()
    if args.eager:
        # the profiled call then launches its kernels one by one (a first call
        # of its size), so NVTX ranges around a phase select its launches
        rlt.rlt_backward_release(m)
    torch.cuda.cudart().cudaProfilerStart()
    rlt.rlt_replay_backward(m, tok, wts, segment=32)
    torch.cuda.synchronize()
    torch.cuda.cudart().cudaProfilerStop()
    rlt.rlt_check_device()
    print("profiled backward over", B, "x", S, "tokens")


def summarize(path: str, S: int) -> str:
    rows = list(csv.reader(open(path)))
    hdr_i = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    hdr, data = rows[hdr_i], rows[hdr_i + 1:]
    ki, vi, ii = hdr.index("Kernel Name"), hdr.index("Metric Value"), hdr.index("ID")
    seq = sorted((int(r[ii]), r[ki].split("(")[0].replace("void ", ""), float(r[vi].replace(",", ""))) for r in data)
    segs: list[list[tuple[str, float]]] = []
    for _, name, v in seq:  # a new segment starts at the encoder's first kernel and at every merge
        if not segs or "merge_prep_kernel" in name:
            segs.append([])
        segs[-1].append((name, v))
    n_dec = S - 1
    samples = [64 + 128 * i for i in range(len(segs) - 1)]
    weights = [1.0] + [min(n_dec, t + 63) - max(1, t - 64) + 1 for t in samples]
    agg = collections.defaultdict(lambda: [0.0, 0.0])
    for wgt, seg in zip(weights, segs):
        for name, v in seg:
            agg[name][0] += wgt
            agg[name][1] += wgt * v
    tot = sum(v[1] for v in agg.values())
    out = [f"captured launches: {len(seq)} in {len(segs)} segments (encoder + positions {samples})",
           f"stratum weights: {weights}",
           f"estimated serialised step time: {tot / 1e6:.1f} ms",
           "| share | est. time ms | launches | kernel |", "|---:|---:|---:|---|"]
    for k, (n, t) in sorted(agg.items(), key=lambda x: -x[1][1]):
        out.append(f"| {100 * t / tot:.2f}% | {t / 1e6:.1f} | {n:.0f} | `{k}` |")
    return "\n".join(out)


def main() -> None:
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="cmd", required=True)
    a = sub.add_parser("step")
    a.add_argument("--workload", default="replay")
    a.add_argument("--batch", type=int, default=64)
    a.add_argument("--len", type=int, default=640)
    a.add_argument("--t", type=int, default=601)
    a.add_argument("--layers", type=int, default=0, help="override the workload's layer count (0: keep)")
    g = sub.add_parser("gen")
    g.add_argument("--workload", default="refdepth")
    g.add_argument("--batch", type=int, default=64)
    g.add_argument("--len", type=int, default=1200)
    g.add_argument("--t", type=int, default=1203)
    g.add_argument("--layers", type=int, default=0)
    e = sub.add_parser("encoder")
    e.add_argument("--workload", default="refdepth")
    e.add_argument("--batch", type=int, default=4)
    e.add_argument("--len", type=int, default=2048)
    e.add_argument("--layers", type=int, default=0)
    p = sub.add_parser("bptt")
    p.add_argument("--workload", default="small")
    p.add_argument("--batch", type=int, default=16)
    p.add_argument("--len", type=int, default=64)
    p.add_argument("--layers", type=int, default=0)
    p.add_argument("--eager", action="store_true",
                   help="profile a first call of its size (direct launches) instead of the graph replay")
    b = sub.add_parser("summarize")
    b.add_argument("csv")
    b.add_argument("S", type=int, nargs="?", default=1024)
    args = ap.parse_args()
    if args.cmd == "step":
        step(args)
    elif args.cmd == "gen":
        gen(args)
    elif args.cmd == "encoder":
        encoder(args)
    elif args.cmd == "bptt":
        bptt(args)
    else:
        print(summarize(args.csv, args.S))


if __name__ == "__main__":
    main()
