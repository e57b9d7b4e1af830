"""Pins of the fp64 oracle to things other than itself.

Each test ties an oracle function to a published value, a closed form, a
library routine, an independent formulation, or an invariant that "Recurrent
Looped Transformer" states (Prop. 3.1 split invariance, Prop. B.1 causality,
§2.1/§2.5 cache bound), chosen so that a dropped term, a wrong sign or index,
or a transposed operand fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.special as sps
import scipy.stats as st

import synth

torch = pytest.importorskip("torch")


def _tiny(**kw):
    w = synth.workload("tiny", **kw)
    return w, synth.model_config(w)


# --------------------------------------------------------------------------
# counter-based generator
# --------------------------------------------------------------------------

def test_philox_known_answers(oracle_lib):
    """Random123 known-answer vectors for Philox4x32-10 (Salmon et al., SC'11;
    tests/golden/philox4x32_10_kat.txt)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        vals = [int(x, 16) for x in r]
        ctr, key, want = vals[0:4], vals[4:6], vals[6:10]
        assert list(oracle_lib.philox4x32_10(ctr, key)) == want


def test_normal_ih12_moments(oracle_lib):
    """Irwin-Hall(12) - 6: mean 0, variance 1, support [-6, 6], excess
    kurtosis -1/10 (sum of 12 uniforms: -6/(5*12))."""
    z = np.array([oracle_lib.normal_ih12(5, 3, i) for i in range(40000)])
    assert abs(z.mean()) < 0.02
    assert abs(z.var() - 1.0) < 0.03
    assert z.min() >= -6 and z.max() < 6
    assert abs(st.kurtosis(z) - (-0.1)) < 0.06


def test_weight_init_statistics(oracle_lib):
    w, cfg = _tiny()
    m = oracle_lib.Model(cfg, seed=42)
    emb = m.get("emb", (256, 64)).astype(np.float64)
    assert abs(emb.std() - 0.02) < 0.001 and abs(emb.mean()) < 0.001
    assert np.all(m.get("g_ea.0", (64,)) == 1.0)
    assert np.all(m.get("b_gate", (64,)) == 0.0)
    # distinct tensors draw from distinct streams
    assert not np.array_equal(m.get("wq.0", (64, 64)), m.get("wk.0", (64, 64)))
    # bf16 storage holds the round-to-nearest-even image of the fp32 draw
    wb, cfgb = _tiny(dtype=1)
    mb = oracle_lib.Model(cfgb, seed=42)
    assert np.array_equal(mb.get("wq.1", (64, 64)), synth.bf16_bits(m.get("wq.1", (64, 64))))


# --------------------------------------------------------------------------
# building blocks
# --------------------------------------------------------------------------

def test_rmsnorm_closed_forms(oracle_lib):
    rng = np.random.default_rng(0)
    x = rng.standard_normal(96)
    g = rng.standard_normal(96)
    y = oracle_lib.rmsnorm(x, np.ones(96), 0.0)
    assert math.isclose(np.sqrt(np.mean(y * y)), 1.0, rel_tol=1e-13)       # unit RMS
    assert np.allclose(oracle_lib.rmsnorm(7.5 * x, g, 0.0), oracle_lib.rmsnorm(x, g, 0.0), atol=1e-13)
    c = oracle_lib.rmsnorm(np.full(8, 3.0), np.arange(8.0), 1e-6)           # constant vector
    assert np.allclose(c, np.arange(8.0) * 3.0 / np.sqrt(9.0 + 1e-6), atol=1e-15)
    t = torch.nn.functional.rms_norm(torch.tensor(x), (96,), weight=torch.tensor(g), eps=1e-6)
    assert np.allclose(oracle_lib.rmsnorm(x, g, 1e-6), t.numpy(), atol=1e-13)


def test_rope_is_complex_rotation(oracle_lib):
    rng = np.random.default_rng(1)
    hd = 16
    x = rng.standard_normal(hd)
    for p in (0.0, 1.0, 37.0, 4095.0):
        y = oracle_lib.rope(x, p, 10000.0)
        z = (x[:8] + 1j * x[8:]) * np.exp(1j * p * 10000.0 ** (-np.arange(8) * 2.0 / hd))
        assert np.allclose(y, np.concatenate([z.real, z.imag]), atol=1e-12)
    # dot products depend only on the position difference
    q, k = rng.standard_normal(hd), rng.standard_normal(hd)
    a = oracle_lib.rope(q, 10, 1e4) @ oracle_lib.rope(k, 3, 1e4)
    b = oracle_lib.rope(q, 107, 1e4) @ oracle_lib.rope(k, 100, 1e4)
    assert math.isclose(a, b, rel_tol=1e-10, abs_tol=1e-12)
    assert np.allclose(oracle_lib.rope(x, 0.0), x)


def test_attention_closed_forms(oracle_lib):
    rng = np.random.default_rng(2)
    hd = 8
    q, K, V = rng.standard_normal(hd), rng.standard_normal((5, hd)), rng.standard_normal((5, hd))
    assert np.allclose(oracle_lib.attend(q, K[:1], V[:1]), V[0])             # one key -> its value
    assert np.allclose(oracle_lib.attend(np.zeros(hd), K, V), V.mean(0))     # zero query -> mean
    s = K[:2] @ q / np.sqrt(hd)                                              # two keys -> sigmoid
    w0 = sps.expit(s[0] - s[1])
    assert np.allclose(oracle_lib.attend(q, K[:2], V[:2]), w0 * V[0] + (1 - w0) * V[1], atol=1e-14)
    p = sps.softmax(K @ q / np.sqrt(hd))
    assert np.allclose(oracle_lib.attend(q, K, V), p @ V, atol=1e-14)


def test_log_softmax_library(oracle_lib):
    x = np.random.default_rng(3).standard_normal(1000) * 5
    y = oracle_lib.log_softmax(x)
    assert np.allclose(y, sps.log_softmax(x), atol=1e-12)
    assert math.isclose(np.exp(y).sum(), 1.0, rel_tol=1e-12)


def test_merge_special_cases(oracle_lib):
    w, cfg = _tiny()
    d = cfg["d"]
    rng = np.random.default_rng(4)
    e, s = rng.standard_normal(d), rng.standard_normal(d)
    # alpha = 0: the merge passes e through (eq. 2.11)
    m0 = oracle_lib.Model(dict(cfg, alpha=0.0), seed=42)
    assert np.array_equal(m0.merge(e, s), e)
    # W_g = 0, b_g = 0 -> g = 1/2; W_s = I -> u = e + alpha/2 * RMSNorm_s(s)
    m = oracle_lib.Model(dict(cfg, alpha=0.7), seed=42)
    m.set("w_gate", np.zeros((d, 2 * d), np.float32))
    m.set("w_state", np.eye(d, dtype=np.float32))
    r = s / np.sqrt(np.mean(s * s) + cfg["rms_eps"])
    assert np.allclose(m.merge(e, s), e + 0.35 * r, atol=1e-13)
    # gate bias only: sigmoid(b) scales the state term
    b = rng.standard_normal(d).astype(np.float32)
    m.set("b_gate", b)
    assert np.allclose(m.merge(e, s), e + 0.7 * sps.expit(b.astype(np.float64)) * r, atol=1e-13)
    # convex gate: W_g = 0 -> u = (e + s)/2; gate from e only (right half 0)
    mc = oracle_lib.Model(dict(cfg, merge_kind=1), seed=42)
    mc.set("w_gate", np.zeros((d, 2 * d), np.float32))
    assert np.allclose(mc.merge(e, s), 0.5 * (e + s), atol=1e-15)
    Wg = np.zeros((d, 2 * d), np.float32)
    Wg[:, :d] = np.eye(d, dtype=np.float32)
    mc.set("w_gate", Wg)
    gg = sps.expit(e)
    assert np.allclose(mc.merge(e, s), gg * e + (1 - gg) * s, atol=1e-14)


# --------------------------------------------------------------------------
# whole forward: independent formulation and invariants
# --------------------------------------------------------------------------

VARIANTS = [
    dict(),                                              # tiny as specified: W=4 wraps 8 times over T=32
    dict(window=32, groups=2, merge_kind=1),             # W >= T: full causal decoder attention; G = L_D
    dict(window=1),                                      # empty SWA cache
    dict(tied=0, window=3),                              # untied stacks
    dict(dtype=1, window=5, alpha=0.5),                  # bf16 storage
]


@pytest.mark.parametrize("kw", VARIANTS, ids=["tiny", "fullwin_G2_convex", "W1", "untied", "bf16"])
def test_oracle_matches_torch_formulation(oracle_lib, kw):
    from tests.torch_model import forward_logprobs
    w, cfg = _tiny(**kw)
    m = oracle_lib.Model(cfg, seed=42)
    tok = synth.tokens(w, batch=2)
    for b in range(2):
        got = m.replay_logprobs(tok[b])
        want = forward_logprobs(m, cfg, tok[b])
        assert np.max(np.abs(got - want)) < 1e-10


def test_prefill_equals_step_encoder_and_split_invariance(oracle_lib):
    """Prop. 3.1: batched encoder prefill + decoder updates equals the
    incremental schedule, whatever the prompt/response split."""
    w, cfg = _tiny()
    m = oracle_lib.Model(cfg, seed=42)
    tok = synth.tokens(w)[1]
    a = m.replay_logprobs(tok, schedule=0)
    b = m.replay_logprobs(tok, schedule=1)
    assert np.max(np.abs(a - b)) <= 1e-12
    for T in (1, 7, 20, 31):
        q = m.seq(32)
        q.encode_prefill(tok[:T])
        got = []
        for t in range(1, 32):
            if t > T:
                q.encode_step(tok[t - 1])
            got.append(oracle_lib.log_softmax(q.decoder_step())[tok[t]])
        assert np.max(np.abs(np.array(got) - a)) <= 1e-12


def test_causality(oracle_lib):
    """Prop. B.1: outputs at t depend only on x_{1:t}."""
    w, cfg = _tiny()
    m = oracle_lib.Model(cfg, seed=42)
    tok = synth.tokens(w)[0].copy()
    a = m.replay_logprobs(tok)
    tok2 = tok.copy()
    tok2[20:] = (tok2[20:] + 17) % cfg["vocab"]
    b = m.replay_logprobs(tok2)
    # log p(x_{t+1}|x_{1:t}) for t+1 < 20 uses only unchanged tokens
    assert np.array_equal(a[:18], b[:18])
    assert not np.array_equal(a[19:], b[19:])


def test_cache_bound_and_retained_positions(oracle_lib):
    """§2.1/§2.5: after update t the cache holds positions max(1,t-W+2)..t,
    at most W-1 entries, none for W=1."""
    for W in (1, 2, 4, 9):
        w, cfg = _tiny(window=W)
        m = oracle_lib.Model(cfg, seed=42)
        tok = synth.tokens(w)[0]
        q = m.seq(32)
        q.encode_prefill(tok)
        for t in range(1, 33):
            q.decoder_step(logits=False)
            for l in range(cfg["n_layers"]):
                pos, _, _ = q.window(l)
                assert list(pos) == list(range(max(1, t - W + 2), t + 1)) if W > 1 else len(pos) == 0
                assert len(pos) <= W - 1


def test_window_only_reaches_output_through_swa(oracle_lib):
    """The window W enters only through the decoder SWA sublayer (eq. 2.14):
    with the decoder's SWA output projection zeroed, W = 1 and W = 6 agree;
    with it present they differ."""
    w, cu = _tiny(window=1, tied=0)
    tok = synth.tokens(w)[0]
    a = oracle_lib.Model(cu, seed=42)
    b = oracle_lib.Model(dict(cu, window=6), seed=42)
    assert np.max(np.abs(a.replay_logprobs(tok) - b.replay_logprobs(tok))) > 1e-9
    for mm in (a, b):
        for l in range(cu["n_layers"]):
            mm.set(f"dwo.{l}", np.zeros((64, 64), np.float32))
    assert np.max(np.abs(a.replay_logprobs(tok) - b.replay_logprobs(tok))) < 1e-13


def test_groups_equal_weights_equal_shared_memory(oracle_lib):
    """G = L_D with every group's projections equal to the shared ones gives
    the G = 1 model (eq. 2.2: only g(l) differs)."""
    w, cfg = _tiny()
    m1 = oracle_lib.Model(cfg, seed=42)
    mL = oracle_lib.Model(dict(cfg, groups=cfg["n_layers"]), seed=42)
    for g in range(cfg["n_layers"]):
        mL.set(f"wk_mem.{g}", m1.get("wk_mem.0", (64, 64)))
        mL.set(f"wv_mem.{g}", m1.get("wv_mem.0", (64, 64)))
    tok = synth.tokens(w)[0]
    assert np.array_equal(m1.replay_logprobs(tok), mL.replay_logprobs(tok))


def test_alpha_zero_cuts_state_feedback(oracle_lib):
    """alpha = 0: u_t = e_t, so s_star and s_{t-1} never reach the output."""
    w, cfg = _tiny(alpha=0.0)
    a = oracle_lib.Model(cfg, seed=42)
    b = oracle_lib.Model(cfg, seed=42)
    b.set("s_star", np.full(64, 3.0, np.float32))
    tok = synth.tokens(w)[0]
    assert np.array_equal(a.replay_logprobs(tok), b.replay_logprobs(tok))
    c = oracle_lib.Model(dict(cfg, alpha=1.0), seed=42)
    c.set("s_star", np.full(64, 3.0, np.float32))
    assert not np.array_equal(a.replay_logprobs(tok), c.replay_logprobs(tok))


# --------------------------------------------------------------------------
# sampler
# --------------------------------------------------------------------------

def test_sampler_top_k_order_and_ties(oracle_lib):
    """Candidates ordered by (value desc, id asc); a sharp temperature puts
    all mass on the first candidate, which must be the smallest tied id."""
    lg = np.zeros(20, np.float32)
    lg[[3, 7, 11]] = 5.0
    for t in range(50):
        tok, lmu, lp, _ = oracle_lib.sample(lg, 1e-3, 2, seed=9, t=t, b=0)
        assert tok in (3, 7)
        assert math.isclose(lmu, math.log(0.5), abs_tol=1e-12)
    tok, lmu, _, _ = oracle_lib.sample(lg, 1.0, 1, seed=9, t=0, b=0)
    assert tok == 3 and lmu == 0.0


def test_sampler_distribution_chi2(oracle_lib):
    """Empirical frequencies over many counters match the tempered,
    truncated, renormalised distribution (brute force on V=12)."""
    rng = np.random.default_rng(5)
    lg = rng.standard_normal(12).astype(np.float32)
    tau, k = float(np.float32(0.8)), 5  # the sampler takes its temperature in fp32
    order = sorted(range(12), key=lambda i: (-lg[i], i))[:k]
    p = np.exp(lg[order].astype(np.float64) / tau)
    p /= p.sum()
    n = 20000
    counts = np.zeros(k)
    for t in range(n):
        tok, lmu, lp, _ = oracle_lib.sample(lg, tau, k, seed=123, t=t, b=3)
        j = order.index(tok)
        counts[j] += 1
        if t < 50:
            assert math.isclose(lmu, math.log(p[j]), rel_tol=1e-9)
            assert math.isclose(lp, sps.log_softmax(lg.astype(np.float64))[tok], rel_tol=1e-9)
    chi2 = ((counts - n * p) ** 2 / (n * p)).sum()
    assert chi2 < st.chi2.ppf(0.999, k - 1)


def test_replay_ratios_pins(oracle_lib):
    """Eq. 5.5 replay ratios.  Pinned by: (a) an untempered, untruncated
    sampler (tau = 1, top_k = V) records log mu equal to the raw model log-prob,
    so the replay of its own rollout gives ratio 1 at every action (this ties
    the sampler's generation schedule to the replay schedule, Prop. 3.1);
    (b) tokens outside the action mask get no factor; (c) the trajectory
    log-ratio is the log of the product of the action ratios; (d) shifting
    log mu by c on k actions shifts the trajectory log-ratio by -k c."""
    w = synth.workload("tiny")
    cfg = synth.model_config(w)
    m = oracle_lib.Model(cfg, seed=42)
    prompt = synth.tokens(w)[0, :10]
    V = cfg["vocab"]
    g = m.generate(prompt, 8, 1.0, V, 11, 0)
    hist = np.concatenate([prompt, g["tokens"]])
    n = hist.size - 1
    logmu = np.zeros(n)
    mask = np.zeros(n, np.uint8)
    logmu[prompt.size - 1:] = g["logmu"]
    mask[prompt.size - 1:] = 1  # the sampled response tokens are the actions
    r = m.replay_ratios(hist, logmu, mask)
    assert np.allclose(r["ratio"][mask == 1], 1.0, atol=1e-6)
    assert abs(r["seq_logratio"]) <= 1e-5
    assert np.all(r["ratio"][mask == 0] == 1.0)
    assert np.allclose(r["logp"], m.replay_logprobs(hist), atol=0, rtol=0)
    rng = np.random.default_rng(3)
    lmu2 = r["logp"] + rng.normal(0, 0.3, n)
    mask2 = (rng.random(n) < 0.5).astype(np.uint8)
    r2 = m.replay_ratios(hist, lmu2, mask2)
    assert np.all(r2["ratio"][mask2 == 0] == 1.0)
    assert math.isclose(np.prod(r2["ratio"]), math.exp(r2["seq_logratio"]), rel_tol=1e-12)
    r3 = m.replay_ratios(hist, lmu2 + 0.25 * mask2, mask2)
    assert math.isclose(r3["seq_logratio"], r2["seq_logratio"] - 0.25 * int(mask2.sum()), abs_tol=1e-12)
