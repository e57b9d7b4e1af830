"""Full-BPTT backward on the GPU through the C ABI (rlt_replay_backward),
against the gradient oracle (``oracle.bptt``: autograd over the fp64
forward, itself pinned by finite differences).

fp32 models: the engine differentiates fp32 copies of the stored weights on
CUDA cores, so the bar is fp32 accumulation error: per tensor, the largest
deviation within 1e-4 of the tensor's largest gradient entry, plus 1e-6, and
log-probs within 1e-4.

bf16 models: the contractions run on the tensor cores with bf16 operands
(activations and adjoints rounded to bf16, relative error 2^-9 each, fp32
accumulation), the precision of the model's forward.  Log-probs meet the
bf16 bar of the forward (5e-2); per tensor the largest gradient deviation
must stay within 5e-2 of the tensor's largest entry (the same relative
budget as the log-probs: a handful of bf16 roundings compounded through the
layers and the recurrence).  With RLT_GRAD_REPORT set to a file name, each
case appends its relative errors there.

The host build of the same engine meets the oracle to 1e-10 in fp64
(``test_bptt_host.py``).
"""
import json
import os

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def rlt():
    import torch
    torch.cuda.init()
    import stateful_decoder_b200 as m
    return m


VARIANTS = [
    (dict(d=32, n_heads=2, ffn=48, vocab=40, prompt=12), 4),
    (dict(d=32, n_heads=2, ffn=48, vocab=40, prompt=12, tied=0, merge_kind=1, groups=2, window=3), 3),
    (dict(d=128, n_heads=2, ffn=192, vocab=256, prompt=10, dtype=1, window=3), 9),
    # every contraction on the tensor cores (d, F and V multiples of 128), hd 128
    (dict(d=256, n_heads=2, n_layers=2, ffn=384, vocab=256, prompt=40, dtype=1, window=8), 8),
]


@pytest.mark.parametrize("kw,seg", VARIANTS, ids=["f32_tied", "f32_untied_convex_GL", "bf16_hd64", "bf16_tc_hd128"])
def test_backward_matches_gradient_oracle(rlt, oracle_lib, kw, seg):
    import torch

    from oracle import bptt
    w = synth.workload("tiny", **kw)
    cfg = synth.model_config(w)
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
    tok = synth.tokens(w, batch=2)
    B, S = tok.shape
    wts = np.random.default_rng(7).uniform(-1.0, 1.0, (B, S - 1)).astype(np.float32)
    lp = torch.zeros((B, S - 1), dtype=torch.float32, device="cuda")
    rlt.rlt_replay_backward(m, torch.from_numpy(tok).cuda(), torch.from_numpy(wts).cuda(), segment=seg, logp=lp)
    bf16 = cfg["dtype"] == 1
    lp_tol, g_rel = (5e-2, 5e-2) if bf16 else (1e-4, 1e-4)
    want = None
    lp_err = 0.0
    for b in range(B):
        lp_err = max(lp_err, float(np.max(np.abs(lp[b].cpu().numpy() - om.replay_logprobs(tok[b])))))
        _, g = bptt.loss_and_grads(om, tok[b], wts[b].astype(np.float64))
        want = g if want is None else {k: want[k] + g[k] for k in want}
    rel = {}
    for name, ref in want.items():
        got = m.grad(name)
        scale = float(np.max(np.abs(ref)))
        rel[name] = float(np.max(np.abs(got - ref))) / max(scale, 1e-30)
    report = os.environ.get("RLT_GRAD_REPORT")
    if report:
        worst = sorted(rel.items(), key=lambda x: -x[1])[:5]
        with open(report, "a") as f:
            f.write(json.dumps({"case": kw, "logp_err": lp_err, "worst_rel": worst}) + "\n")
    assert lp_err <= lp_tol
    for name, ref in want.items():
        scale = float(np.max(np.abs(ref)))
        assert rel[name] * scale <= g_rel * scale + 1e-6, (name, rel[name])
    rlt.rlt_check_device()


def test_backward_accumulates_and_zeroes(rlt):
    import torch
    w = synth.workload("tiny", d=32, n_heads=2, ffn=48, vocab=40, prompt=8)
    cfg = synth.model_config(w)
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    tok = torch.from_numpy(synth.tokens(w, batch=2)).cuda()
    wts = torch.full((2, 7), 1.0 / 7, dtype=torch.float32, device="cuda")
    assert not np.any(m.grad("w_out"))
    rlt.rlt_replay_backward(m, tok, wts, segment=2)
    one = {n: m.grad(n) for n in ("emb", "s_star", "w_gate", "wq.0", "g_dffn.1")}
    rlt.rlt_replay_backward(m, tok, wts, segment=7)  # a different segment length gives the same gradient
    for n, g in one.items():
        assert np.allclose(m.grad(n), 2 * g, rtol=1e-5, atol=1e-7), n
    rlt.rlt_grad_zero(m)
    torch.cuda.synchronize()
    assert not np.any(m.grad("emb"))
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_replay_backward(m, tok, wts, segment=0)
    assert e.value.code == rlt.RLT_E_INVAL
    bad = tok.clone()
    bad[1, 3] = cfg["vocab"]  # rejected on the host before any launch
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_replay_backward(m, bad, wts, segment=2)
    assert e.value.code == rlt.RLT_E_INVAL and "out of range" in str(e.value)
    rlt.rlt_check_device()


def test_backward_on_a_side_stream(rlt, oracle_lib):
    """The first backward of a model zeroes the fresh gradient buffers on the
    caller's stream: run on a non-blocking side stream, its gradients still
    equal the oracle's."""
    import torch

    from oracle import bptt
    w = synth.workload("tiny", d=32, n_heads=2, ffn=48, vocab=40, prompt=9)
    cfg = synth.model_config(w)
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    tok = synth.tokens(w, batch=2)
    wts = np.full((2, 8), 0.125, dtype=np.float32)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        t = torch.from_numpy(tok).cuda(non_blocking=False)
        wd = torch.from_numpy(wts).cuda(non_blocking=False)
        side.synchronize()
        rlt.rlt_replay_backward(m, t, wd, segment=3, stream=side)
    side.synchronize()
    om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
    want = None
    for b in range(2):
        _, g = bptt.loss_and_grads(om, tok[b], wts[b].astype(np.float64))
        want = g if want is None else {k: want[k] + g[k] for k in want}
    for name in ("emb", "s_star", "w_gate", "wq.0", "w2.1", "w_out"):
        ref = want[name]
        assert np.max(np.abs(m.grad(name) - ref)) <= 1e-4 * float(np.max(np.abs(ref))) + 1e-6, name
    rlt.rlt_check_device()


def test_backward_long_sequence_hd128():
    """A bf16 model at hd 128 over 600 tokens (the forward's decode attention
    spans three 256-key chunks; the SWA window wraps 75 times; 19 segments
    of 32): the log-probs and the gradients of the stored tensors against
    the oracle's, kept as a golden (tests/golden/make_goldens.py, the
    gradient oracle's autograd in fp64), at the bf16 bars above."""
    import torch

    import stateful_decoder_b200 as rlt
    from tests.golden import make_goldens as goldens
    g = goldens.load_grad()
    w = goldens.grad_workload()
    cfg = synth.model_config(w)
    tok = synth.tokens(w, batch=1)
    S = tok.shape[1]
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    wts = torch.full((1, S - 1), 1.0 / (S - 1), device="cuda")
    lp = torch.zeros(1, S - 1, device="cuda")
    rlt.rlt_replay_backward(m, torch.from_numpy(tok).cuda(), wts, segment=32, logp=lp)
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    assert np.max(np.abs(lp.cpu().numpy()[0] - g["logp"])) <= 5e-2
    for name, ref in g["grads"].items():
        ref = ref.astype(np.float64)
        scale = float(np.max(np.abs(ref)))
        err = float(np.max(np.abs(m.grad(name) - ref)))
        assert err <= 5e-2 * scale + 1e-6, (name, err / scale)


def test_backward_kept_between_calls_and_replayed(rlt, oracle_lib):
    """The model keeps the backward's buffers between calls of one size: the
    first call launches its kernels, the second captures the whole pass as a
    CUDA graph, later ones replay it.  Every call below starts from zeroed
    gradients and meets the oracle at the bf16 bars: four calls of one size
    on different tokens and target weights, with a weight loaded between the
    second and the third (the graph's prologue refreshes the fp32 weight
    copies); then a call of another batch size (the kept buffers are
    rebuilt); then one after rlt_backward_release."""
    import torch

    from oracle import bptt
    w = synth.workload("tiny", d=128, n_heads=2, ffn=192, vocab=256, prompt=10, dtype=1, window=3)
    cfg = synth.model_config(w)
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
    rng = np.random.default_rng(11)

    def check(tok, seg=4):
        B, S = tok.shape
        wts = rng.uniform(-1.0, 1.0, (B, S - 1)).astype(np.float32)
        rlt.rlt_grad_zero(m)
        lp = torch.zeros((B, S - 1), dtype=torch.float32, device="cuda")
        rlt.rlt_replay_backward(m, torch.from_numpy(tok).cuda(), torch.from_numpy(wts).cuda(), segment=seg, logp=lp)
        want = None
        lp_err = 0.0
        for b in range(B):
            lp_err = max(lp_err, float(np.max(np.abs(lp[b].cpu().numpy() - om.replay_logprobs(tok[b])))))
            _, g = bptt.loss_and_grads(om, tok[b], wts[b].astype(np.float64))
            want = g if want is None else {k: want[k] + g[k] for k in want}
        assert lp_err <= 5e-2
        for name, ref in want.items():
            scale = float(np.max(np.abs(ref)))
            assert float(np.max(np.abs(m.grad(name) - ref))) <= 5e-2 * scale + 1e-6, name

    base = synth.tokens(w, batch=2)
    for i in range(4):
        tok = base.copy() if i == 0 else rng.integers(0, cfg["vocab"], size=base.shape).astype(np.int32)
        tok[:, 0] = base[:, 0]  # BOS
        if i == 2:
            ws = m.get_weights("w_state")[::-1].copy()
            m.load_weights("w_state", ws)
            om.set("w_state", ws)
        check(tok)
    check(synth.tokens(w, batch=3))
    rlt.rlt_backward_release(m)
    check(base)
    rlt.rlt_check_device()
