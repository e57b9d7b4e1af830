"""Pins of the full-BPTT gradient oracle (``oracle.bptt``).

The gradient oracle is tied to things other than itself:

* its forward log-probabilities equal the C oracle's replay (itself pinned in
  ``test_oracle_pins.py``);
* every gradient entry of two small models (tied/untied stacks, both merge
  forms, one or L memory groups) equals a central finite difference of the C
  oracle's weighted replay loss, which involves no differentiation code;
* the gradients of the readout matrix and of its norm gain equal their closed
  forms, built from the C oracle's recurrent outputs s_t;
* App. C's statement that cutting s_t or the decoder KV at a step boundary
  keeps every forward value but changes the gradient.  The truncated
  gradients differ from the finite differences far beyond the tolerance,
  which also shows that the finite-difference pin would catch a dropped
  path.

A hand-derived reverse-time schedule (``tests/manual_backward.py``: segment
recompute from checkpoints, SWA adjoints owed across segment boundaries,
deferred memory-key/value adjoints, one weight product per segment) gives
the autograd gradient to 1e-11.  This holds for segment lengths from 1 to the
whole sequence.
"""
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")

# a model small enough to difference every entry: d=8 (2 heads of 4), L=2,
# W=2 (the window evicts), F=12, V=11, 8 tokens; larger weights than the
# workloads' 0.02 so that every path carries a gradient well above the
# finite-difference error
MICRO = dict(d=8, n_heads=2, n_layers=2, window=2, groups=1, ffn=12, vocab=11, dtype=0,
             batch=1, prompt=8, gen=0, dist="uniform", data_seed=77, init_std=0.35)

MICRO_VARIANTS = [dict(), dict(tied=0, merge_kind=1, groups=2, window=3)]


def _micro(oracle_lib, **kw):
    w = synth.workload("tiny", **dict(MICRO, **kw))
    cfg = synth.model_config(w)
    m = oracle_lib.Model(cfg, seed=9)
    rng = np.random.default_rng(5)
    # gains and the gate bias away from their initial 1 and 0, so that a
    # dropped gain or bias changes the result
    from oracle import bptt
    for name, shp in bptt.tensor_shapes(cfg).items():
        if name.startswith("g_") or name == "b_gate":
            m.set(name, 1.0 * (name != "b_gate") + 0.3 * rng.standard_normal(shp))
    return w, cfg, m


def _loss_c(m, tok, wts):
    return -float(np.dot(wts, m.replay_logprobs(tok)))


def _fd_grad(m, name, shape, tok, wts, h=1e-4):
    """Central differences of the C oracle's L_w over every entry of one
    tensor; the step is the one fp32 storage actually takes."""
    base = m.get(name, shape).astype(np.float32)
    g = np.zeros(shape)
    for idx in np.ndindex(*shape):
        w0 = float(base[idx])
        plus, minus = base.copy(), base.copy()
        plus[idx] = np.float32(w0 + h)
        minus[idx] = np.float32(w0 - h)
        m.set(name, plus)
        lp = _loss_c(m, tok, wts)
        m.set(name, minus)
        lm = _loss_c(m, tok, wts)
        g[idx] = (lp - lm) / (float(plus[idx]) - float(minus[idx]))
    m.set(name, base)
    return g


@pytest.mark.parametrize("kw", [dict(), dict(window=32, groups=2, merge_kind=1), dict(window=1),
                                dict(tied=0, window=3), dict(dtype=1, window=5, alpha=0.5)],
                         ids=["tiny", "fullwin_G2_convex", "W1", "untied", "bf16"])
def test_bptt_forward_equals_c_oracle(oracle_lib, kw):
    from oracle import bptt
    w = synth.workload("tiny", **kw)
    cfg = synth.model_config(w)
    m = oracle_lib.Model(cfg, seed=42)
    tok = synth.tokens(w, batch=2)
    P = bptt.parameters(m)
    for b in range(2):
        got = bptt.logprobs(P, cfg, tok[b]).detach().numpy()
        assert np.max(np.abs(got - m.replay_logprobs(tok[b]))) < 1e-11


@pytest.mark.parametrize("kw", MICRO_VARIANTS, ids=["tied_paper_merge", "untied_convex_GL"])
def test_bptt_gradient_equals_finite_differences_everywhere(oracle_lib, kw):
    from oracle import bptt
    w, cfg, m = _micro(oracle_lib, **kw)
    tok = synth.tokens(w)[0]
    wts = np.random.default_rng(3).uniform(-1.0, 1.0, tok.size - 1)  # a generic L_w
    loss, grads = bptt.loss_and_grads(m, tok, wts)
    assert abs(loss - _loss_c(m, tok, wts)) < 1e-12
    shapes = bptt.tensor_shapes(cfg)
    assert set(grads) == set(shapes)
    for name, shp in shapes.items():
        fd = _fd_grad(m, name, shp, tok, wts)
        err = np.max(np.abs(grads[name] - fd))
        assert err < 1e-7 + 1e-5 * np.max(np.abs(fd)), (name, err)
    if cfg["merge_kind"] == 1:
        assert np.all(grads["b_gate"] == 0.0)  # the convex gate has no bias
    # the initial state reaches the loss only through the recurrence
    assert np.linalg.norm(grads["s_star"]) > 1e-3


def test_truncation_keeps_values_and_changes_gradients(oracle_lib):
    """App. C / eq. C.1: detaching s_t or the decoder KV at every step
    boundary leaves the log-probabilities as they are and removes gradient
    paths; full BPTT is the one that matches the finite differences."""
    from oracle import bptt
    w, cfg, m = _micro(oracle_lib)
    tok = synth.tokens(w)[0]
    wts = bptt.target_weights("pretrain", tok.size)
    P = bptt.parameters(m)
    full = bptt.logprobs(P, cfg, tok).detach().numpy()
    _, g_full = bptt.loss_and_grads(m, tok, wts)
    for cut, name in ((("s",), "w_state"), (("swa",), "wk.1"), (("s", "swa"), "s_star")):
        assert np.array_equal(bptt.logprobs(P, cfg, tok, cut).detach().numpy(), full)
        _, g_cut = bptt.loss_and_grads(m, tok, wts, cut)
        fd = _fd_grad(m, name, bptt.tensor_shapes(cfg)[name], tok, wts)
        assert np.max(np.abs(g_full[name] - fd)) < 1e-7 + 1e-5 * np.max(np.abs(fd))
        assert np.max(np.abs(g_cut[name] - fd)) > 1e-4, cut


def test_readout_gradients_closed_form(oracle_lib):
    """dL_w/dW_o = sum_t w_t (softmax(l_t) - onehot(x_{t+1})) n_t^T and
    dL_w/dgamma_o = sum_t w_t (W_o^T (p_t - y_t)) * s_t / rms(s_t), with
    l_t = W_o n_t, n_t = RMSNorm(s_t; gamma_o) (eq. 2.6), from the C
    oracle's step-by-step states."""
    from oracle import bptt
    w = synth.workload("tiny")
    cfg = synth.model_config(w)
    m = oracle_lib.Model(cfg, seed=42)
    d, V = cfg["d"], cfg["vocab"]
    m.set("g_out", 1.0 + 0.2 * np.random.default_rng(1).standard_normal((1, d)))
    tok = synth.tokens(w, batch=1)[0]
    S = tok.size
    mask = (np.arange(S - 1) % 3 != 0).astype(np.float64)
    wts = bptt.target_weights("sft", S, mask=mask)
    W_o = m.get("w_out", (V, d)).astype(np.float64)
    g_o = m.get("g_out", (1, d)).astype(np.float64)[0]
    q = m.seq(S)
    q.encode_prefill(tok)
    gW, gg = np.zeros((V, d)), np.zeros(d)
    for t in range(S - 1):
        logits = q.decoder_step()
        s = q.s()
        shat = s / np.sqrt(np.mean(s * s) + cfg["rms_eps"])
        assert np.allclose(logits, W_o @ (shat * g_o), rtol=0, atol=1e-12)
        p = np.exp(logits - logits.max())
        p /= p.sum()
        p[tok[t + 1]] -= 1.0
        gW += wts[t] * np.outer(p, shat * g_o)
        gg += wts[t] * (W_o.T @ p) * shat
    _, grads = bptt.loss_and_grads(m, tok, wts)
    assert np.max(np.abs(grads["w_out"] - gW)) < 1e-12
    assert np.max(np.abs(grads["g_out"][0] - gg)) < 1e-12


def test_objective_weights_and_masked_targets(oracle_lib):
    """Eqs. 5.1/5.2/5.4 as weights; a target with w_t = 0 adds nothing, and
    the gradient is linear in w (so the per-objective gradients are weighted
    sums of per-target ones)."""
    from oracle import bptt
    S = 9
    assert np.allclose(bptt.target_weights("pretrain", S), 1 / 8)
    m5 = np.array([0, 0, 1, 1, 0, 1, 1, 1], dtype=float)
    assert np.allclose(bptt.target_weights("sft", S, mask=m5), m5 / 5)
    sc = bptt.target_weights("score", S, reward=2.0, baseline=0.5, prompt_len=4)
    assert np.allclose(sc, [0, 0, 0, 1.5, 1.5, 1.5, 1.5, 1.5])
    with pytest.raises(ValueError):
        bptt.target_weights("sft", S, mask=np.zeros(8))
    with pytest.raises(ValueError):
        bptt.target_weights("score", S, prompt_len=0)

    w, cfg, m = _micro(oracle_lib)
    tok = synth.tokens(w)[0]
    wa = np.random.default_rng(8).uniform(size=tok.size - 1)
    wb = np.random.default_rng(9).uniform(size=tok.size - 1)
    _, ga = bptt.loss_and_grads(m, tok, wa)
    _, gb = bptt.loss_and_grads(m, tok, wb)
    _, gab = bptt.loss_and_grads(m, tok, 2.0 * wa - wb)
    for k in ga:
        assert np.allclose(gab[k], 2.0 * ga[k] - gb[k], rtol=0, atol=1e-12)
    # the last target only: the embedding row of a token that appears only
    # after position t has no gradient from targets up to t (causality)
    last = np.zeros(tok.size - 1)
    last[2] = 1.0  # target x_4 given x_1..x_3
    _, g3 = bptt.loss_and_grads(m, tok, last)
    later = set(tok[4:].tolist()) - set(tok[:4].tolist())
    for v in later:
        assert np.all(g3["emb"][v] == 0.0)


# --------------------------------------------------------------------------
# the hand-derived, segment-checkpointed reverse-time schedule
# --------------------------------------------------------------------------

@pytest.mark.parametrize("kw,seg", [(dict(), 1), (dict(), 3), (dict(window=1), 4),
                                    (dict(tied=0, merge_kind=1, groups=2, window=3), 2),
                                    (dict(window=32, alpha=0.5), 5), (dict(dtype=1, window=5), 31)],
                         ids=["seg1", "seg3", "W1_seg4", "untied_convex_GL_seg2", "fullwin_seg5", "bf16_oneseg"])
def test_manual_reverse_time_schedule_equals_autograd(oracle_lib, kw, seg):
    """The reverse-time schedule (segment recompute from checkpoints,
    deferred memory adjoints, per-segment weight products) gives the
    autograd gradient of full BPTT; checkpointing changes no value (§4.3,
    §5.4, App. C)."""
    from oracle import bptt
    from tests.manual_backward import ManualBPTT
    w = synth.workload("tiny", **kw)
    cfg = synth.model_config(w)
    m = oracle_lib.Model(cfg, seed=42)
    rng = np.random.default_rng(4)
    for name, shp in bptt.tensor_shapes(cfg).items():
        if cfg["dtype"] == 0 and (name.startswith("g_") or name == "b_gate"):
            m.set(name, 1.0 * (name != "b_gate") + 0.2 * rng.standard_normal(shp))
    tok = synth.tokens(w, batch=1)[0]
    wts = rng.uniform(-1.0, 1.0, tok.size - 1)
    loss, g_auto = bptt.loss_and_grads(m, tok, wts)
    P = {k: v.detach().numpy() for k, v in bptt.parameters(m).items()}
    mloss, mlogp, g_man = ManualBPTT(P, cfg).loss_and_grads(tok, wts, seg)
    assert np.max(np.abs(mlogp - m.replay_logprobs(tok))) < 1e-11
    assert abs(mloss - loss) < 1e-11
    for k in g_auto:
        scale = max(1.0, np.max(np.abs(g_auto[k])))
        assert np.max(np.abs(g_man[k] - g_auto[k])) < 1e-11 * scale, k
