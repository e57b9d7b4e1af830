"""Writes the stored expected log-probs of the full-size parity tests.

Every value here comes from the fp64 oracle (``oracle/``) on token ids from
the seeded generator (``synth``); nothing reads the CUDA library.  Each golden
is one ``.npz`` file in this directory holding

* ``logp``    float64 [len(rows), length-1]: log p(x_{t+1} | x_1..t) of each
              selected sequence, t = 1..length-1 (report §2.3 eq. 2.6, with
              the eq. 5.1 indexing of targets);
* ``rows``    int32, the batch rows of ``synth.tokens(workload, batch,
              length)`` the sequences are (the GPU test runs the whole batch
              and compares these rows);
* ``meta``    a JSON string: workload name, batch, length, and ``prompt``,
              the number of tokens the GPU test prefills before it switches to
              teacher-forced generation steps (0: the replay schedule).

By Prop. 3.1 of the report (prefill and incremental schedules compute the
same distributions), the oracle's replay of the whole sequence is the
expected output of either GPU schedule.

A second kind of golden (``bptt_hd128_long``) holds the full-BPTT gradient
of the oracle on a long sequence (see GRAD_GOLDEN below).

    python tests/golden/make_goldens.py [name ...]     # default: all
"""
from __future__ import annotations

import json
import os
import sys
import time

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

# name: (workload, batch, length, rows, prompt)
GOLDENS = {
    # the "small" configuration: prompt 512, then 512 positions through the
    # generation path (encoder step + transition), teacher-forced
    "small_gen": ("small", 16, 1024, (0, 15), 512),
    # layer-specific memory (G = L = 24, d = 1024, hd 64), teacher-forced T = 2048
    "layerwise_replay": ("layerwise", 64, 2048, (0, 63), 0),
    # RL exact replay: reference width at L = 24, B = 256, S = 1024, every position
    "replay_full": ("replay", 256, 1024, (0, 255), 0),
    # reference depth 48+48, B = 128: prompt 2048 prefilled, then 64 positions
    # through the generation path
    "refdepth_gen": ("refdepth", 128, 2048 + 64, (0, 127), 2048),
}


# Gradient golden of the full-BPTT backward (report §5.4): a bf16 model at
# hd 128 over S = 600 tokens (the forward's decode attention spans three
# 256-key chunks), weights of eq. 5.1, gradients of the oracle's autograd
# (oracle/bptt.py).  Only the tensors in GRAD_NAMES are stored (float32).
GRAD_GOLDEN = "bptt_hd128_long"
GRAD_MODEL = dict(d=256, n_heads=2, n_layers=1, window=8, ffn=384, vocab=128, dtype=1, prompt=600, gen=0)
GRAD_NAMES = ("s_star", "b_gate", "g_merge", "g_out", "w_gate", "w_state", "w_out", "wq.0", "wk.0", "w2.0",
              "wq_mem.0", "wk_mem.0", "g_dsa.0", "g_ea.0")


def grad_workload() -> dict:
    return synth.workload("tiny", **GRAD_MODEL)


def make_grad() -> None:
    import oracle
    from oracle import bptt
    w = grad_workload()
    tok = synth.tokens(w, batch=1)
    S = tok.shape[1]
    om = oracle.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)
    wts = np.full(S - 1, 1.0 / (S - 1))  # eq. 5.1
    t0 = time.time()
    loss, g = bptt.loss_and_grads(om, tok[0], wts)
    print(f"{GRAD_GOLDEN}: {S} tokens in {time.time() - t0:.0f} s", flush=True)
    lp = om.replay_logprobs(tok[0])
    arrays = {"grad_" + n.replace(".", "_"): np.asarray(g[n], dtype=np.float32) for n in GRAD_NAMES}
    tmp = path(GRAD_GOLDEN) + ".tmp.npz"
    np.savez_compressed(tmp, logp=lp, loss=np.float64(loss), names=np.asarray(GRAD_NAMES), **arrays)
    os.replace(tmp, path(GRAD_GOLDEN))


def load_grad() -> dict:
    z = np.load(path(GRAD_GOLDEN))
    return {"logp": z["logp"], "loss": float(z["loss"]),
            "grads": {n: z["grad_" + n.replace(".", "_")] for n in GRAD_NAMES}}


def path(name: str) -> str:
    return os.path.join(HERE, name + ".npz")


def load(name: str) -> dict:
    z = np.load(path(name))
    meta = json.loads(str(z["meta"]))
    return {"logp": z["logp"], "rows": z["rows"], **meta}


def make(name: str) -> None:
    import oracle
    wname, batch, length, rows, prompt = GOLDENS[name]
    w = synth.workload(wname)
    tok = synth.tokens(w, batch=batch, length=length)
    om = oracle.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)
    out = []
    for r in rows:
        t0 = time.time()
        out.append(om.replay_logprobs(tok[r]))
        print(f"{name}: row {r} ({length} tokens) in {time.time() - t0:.0f} s", flush=True)
    meta = json.dumps({"workload": wname, "batch": batch, "length": length, "prompt": prompt})
    tmp = path(name) + ".tmp.npz"
    np.savez(tmp, logp=np.stack(out), rows=np.asarray(rows, dtype=np.int32), meta=np.asarray(meta))
    os.replace(tmp, path(name))


if __name__ == "__main__":
    for n in (sys.argv[1:] or list(GOLDENS) + [GRAD_GOLDEN]):
        if n == GRAD_GOLDEN:
            make_grad()
        else:
            make(n)
