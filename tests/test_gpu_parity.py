"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerances: per-token log-prob max abs error <= 1e-4 for fp32 models and
<= 5e-2 for bf16 models (teacher-forced tokens); bit-exact for weights,
token ids of the sampler on identical fp32 logits, cache positions and ring
indices.  Inputs come from the seeded generator in ``synth``; the oracle
never sees a value produced by the CUDA path.
"""
import math

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 5e-2


@pytest.fixture(scope="module")
def rlt():
    import torch
    torch.cuda.init()
    import stateful_decoder_b200 as m
    return m


@pytest.fixture(scope="module")
def torch_mod():
    import torch
    return torch


def _tiny(**kw):
    w = synth.workload("tiny", **kw)
    return w, synth.model_config(w)


def _bf16_small(**kw):
    """A small bf16 model that still spans several 128-row GEMM tiles, two
    256-key attention chunks and a ragged tail."""
    base = dict(d=256, n_heads=2, n_layers=2, window=16, groups=1, ffn=512, vocab=1024, dtype=1, batch=3,
                prompt=300, gen=0, dist="zipf", data_seed=1101)
    base.update(kw)
    w = synth.workload("small", **base)
    return w, synth.model_config(w)


def _gpu_replay(rlt, torch, cfg, tok, seed=synth.WEIGHT_SEED, model=None):
    m = model if model is not None else rlt.rlt_init_weights(cfg, seed)
    t = torch.from_numpy(tok).cuda()
    out = torch.zeros(tok.shape[0], tok.shape[1] - 1, dtype=torch.float32, device="cuda")
    rlt.rlt_replay_logprobs(m, t, out)
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    return out.cpu().numpy().astype(np.float64), m


def _oracle_replay(oracle_lib, cfg, tok, seed=synth.WEIGHT_SEED, model=None):
    om = model if model is not None else oracle_lib.Model(cfg, seed=seed)
    return np.stack([om.replay_logprobs(tok[b]) for b in range(tok.shape[0])]), om


# ------------------------------------------------------------------ kernels
@pytest.mark.parametrize("M,N,K", [(128, 1, 64), (256, 37, 192), (2048, 256, 2048), (384, 700, 512),
                                   (32000, 16, 512), (11264, 64, 2048), (2048, 200, 5632)])
def test_tensor_core_linear(rlt, torch_mod, M, N, K):
    torch = torch_mod
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    w = (torch.randn(M, K, generator=g) * 0.05).to(torch.bfloat16).cuda()
    x = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    want = (x.float() @ w.float().T)
    y_tc = torch.zeros(N, M, device="cuda")
    y_simt = torch.zeros(N, M, device="cuda")
    rlt.rlt_op_linear(w, x, y_tc, use_tensor_cores=True)
    rlt.rlt_op_linear(w, x, y_simt, use_tensor_cores=False)
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    scale = want.abs().max().item()
    assert (y_simt - want).abs().max().item() <= 1e-4 * scale
    assert (y_tc - want).abs().max().item() <= 1e-4 * scale


def test_weights_match_oracle_generator(rlt, oracle_lib):
    for cfg in (_tiny()[1], _tiny(tied=0, groups=2)[1], _bf16_small()[1], _bf16_small(groups=2)[1]):
        m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
        om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
        names = ["emb", "s_star", "g_mem", "w_gate", "b_gate", "w_state", "w_out", "wk_mem.0", "wv_mem.0"]
        for l in range(cfg["n_layers"]):
            names += [f"{k}.{l}" for k in ("wq", "wk", "wv", "wo", "w1", "w2", "w3", "g_ea", "g_dsa", "wq_mem",
                                           "wo_mem")]
            if not cfg["tied"]:
                names += [f"d{k}.{l}" for k in ("wq", "wk", "wv", "wo", "w1", "w2", "w3")]
        for n in names:
            r, c, _ = m.tensor_info(n)
            assert np.array_equal(m.get_weights(n), om.get(n, (r, c)).reshape(r, c)), n


# ------------------------------------------------------------------ teacher-forced parity
# W160_hd64: a ring of 159 entries takes the streamed SWA kernel (chunks of
# 64 keys at hd 64 in fp32: 64 + 64 + 31) and wraps twice over 400 positions.
TINY_VARIANTS = [dict(), dict(window=1), dict(window=32), dict(groups=2, merge_kind=1), dict(tied=0, window=3),
                 dict(alpha=0.5, window=2), dict(window=160, n_heads=1, prompt=400)]


@pytest.mark.parametrize("kw", TINY_VARIANTS, ids=["tiny", "W1", "Wfull", "G2_convex", "untied", "W2", "W160_hd64"])
def test_replay_parity_fp32(rlt, torch_mod, oracle_lib, kw):
    w, cfg = _tiny(**kw)
    tok = synth.tokens(w)
    got, _ = _gpu_replay(rlt, torch_mod, cfg, tok)
    want, _ = _oracle_replay(oracle_lib, cfg, tok)
    assert np.max(np.abs(got - want)) <= TOL_F32


@pytest.mark.parametrize("kw", [dict(), dict(n_heads=4), dict(groups=2, merge_kind=1), dict(window=1),
                                dict(window=200, prompt=420)],
                         ids=["hd128", "hd64", "G2_convex", "W1", "W200_wrap"])
def test_replay_parity_bf16(rlt, torch_mod, oracle_lib, kw):
    w, cfg = _bf16_small(**kw)
    tok = synth.tokens(w)
    got, _ = _gpu_replay(rlt, torch_mod, cfg, tok)
    want, _ = _oracle_replay(oracle_lib, cfg, tok)
    err = np.max(np.abs(got - want))
    assert err <= TOL_BF16, err


def test_replay_parity_bf16_many_rows(rlt, torch_mod, oracle_lib):
    """A token-parallel encoder pass with more than 4096 rows (16 x 300) takes
    the warp-per-row RMSNorm; the GPU replays all 16 sequences and the oracle
    checks three of them, including the last."""
    w, cfg = _bf16_small(batch=16, data_seed=1202)
    tok = synth.tokens(w)
    assert tok.shape[0] * tok.shape[1] >= 4096
    got, _ = _gpu_replay(rlt, torch_mod, cfg, tok)
    pick = [0, 7, 15]
    want, _ = _oracle_replay(oracle_lib, cfg, tok[pick])
    err = np.max(np.abs(got[pick] - want))
    assert err <= TOL_BF16, err


def test_generation_path_teacher_forced(rlt, torch_mod, oracle_lib):
    """Prompt prefill then incremental encoder steps (eq. 2.8) and decoder
    transitions, scored on teacher tokens, equal the oracle's replay
    (Prop. 3.1: the split does not change the distribution)."""
    torch = torch_mod
    for w, cfg, tol in ((*_tiny(), TOL_F32), (*_bf16_small(prompt=80), TOL_BF16)):
        tok = synth.tokens(w)
        B, S = tok.shape
        T0 = 20
        m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
        tdev = torch.from_numpy(tok).cuda()
        pre = torch.zeros(B, T0 - 1, device="cuda")
        st2 = rlt.rlt_state_create(m, B, S, rlt.STATE_ENCODER_CACHE)
        rlt.rlt_prefill(m, st2, tdev[:, :T0].contiguous(), pre)
        got = [pre.cpu().numpy()]
        col = torch.zeros(B, device="cuda")
        rlt.rlt_readout(m, st2, next_tokens=tdev[:, T0].contiguous(), logp=col)
        got.append(col.cpu().numpy()[:, None])
        for t in range(T0 + 1, S):
            rlt.rlt_decoder_step(m, st2, tokens=tdev[:, t - 1].contiguous(), next_tokens=tdev[:, t].contiguous(),
                                 logp=col)
            got.append(col.cpu().numpy()[:, None])
        torch.cuda.synchronize()
        rlt.rlt_check_device()
        got = np.concatenate(got, axis=1).astype(np.float64)
        want, _ = _oracle_replay(oracle_lib, cfg, tok)
        assert np.max(np.abs(got - want)) <= tol
        info = st2.info()
        assert info["n_enc"] == S - 1 and info["n_dec"] == S - 1


def test_batched_equals_single(rlt, torch_mod):
    """§4.1: a sequence's result does not depend on the other sequences of
    the batch (no batch-size-dependent reduction order)."""
    for w, cfg in (_tiny(), _bf16_small(prompt=90)):
        tok = synth.tokens(w, batch=3)
        m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
        full, _ = _gpu_replay(rlt, torch_mod, cfg, tok, model=m)
        for b in range(3):
            one, _ = _gpu_replay(rlt, torch_mod, cfg, tok[b:b + 1].copy(), model=m)
            assert np.array_equal(one[0], full[b]), (b, np.max(np.abs(one[0] - full[b])))


def test_causality_gpu(rlt, torch_mod):
    """Prop. B.1 on the device: changing tokens after position 20 leaves every
    earlier log-prob bit-identical."""
    for w, cfg in (_tiny(), _bf16_small(prompt=64)):
        tok = synth.tokens(w)
        m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
        a, _ = _gpu_replay(rlt, torch_mod, cfg, tok, model=m)
        tok2 = tok.copy()
        tok2[:, 20:] = (tok2[:, 20:] + 5) % cfg["vocab"]
        b, _ = _gpu_replay(rlt, torch_mod, cfg, tok2, model=m)
        assert np.array_equal(a[:, :18], b[:, :18])


def test_ring_bookkeeping_and_contents(rlt, torch_mod, oracle_lib):
    """§2.1/§2.5: the ring keeps min(t, W-1) entries, position j in slot
    (j-1) mod (W-1); contents equal the oracle's retained keys/values."""
    torch = torch_mod
    for W in (1, 2, 4, 7):
        w, cfg = _tiny(window=W)
        tok = synth.tokens(w)
        B, S = tok.shape
        m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
        om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
        for T in (1, 3, 17, 32):
            st = rlt.rlt_state_create(m, B, S)
            rlt.rlt_prefill(m, st, torch.from_numpy(tok[:, :T].copy()).cuda())
            torch.cuda.synchronize()
            info = st.info()
            assert info["n_dec"] == T and info["ring_valid"] == min(T, W - 1)
            assert info["ring_head"] == (T % (W - 1) if W > 1 else 0)
            if W == 1:
                continue
            H, hd = cfg["n_heads"], cfg["d"] // cfg["n_heads"]
            for layer in range(cfg["n_layers"]):
                rk = st.read(rlt.READ_RING_K, layer)
                rv = st.read(rlt.READ_RING_V, layer)
                for b in range(B):
                    q = om.seq(S, keep_enc_cache=False)
                    q.encode_prefill(tok[b])
                    for _ in range(T):
                        q.decoder_step(logits=False)
                    pos, k, v = q.window(layer)
                    assert list(pos) == list(range(max(1, T - W + 2), T + 1))
                    for j, kk, vv in zip(pos, k, v):
                        slot = (j - 1) % (W - 1)
                        gk = rk[b, :, slot, :].reshape(H * hd)
                        gv = rv[b, :, slot, :].reshape(H * hd)
                        assert np.max(np.abs(gk - kk)) < 1e-4 and np.max(np.abs(gv - vv)) < 1e-4


# ------------------------------------------------------------------ sampler
def test_sampler_decisions_match_oracle(rlt, torch_mod, oracle_lib):
    """Identical fp32 logits in, identical token ids out (the decision is
    taken in fp32 on both sides); log mu and log p within fp32 rounding."""
    torch = torch_mod
    B, V = 16, 32000
    for seed, tau, k in ((11, 0.8, 50), (12, 1.0, 1), (13, 0.5, 256), (14, 2.0, 7)):
        lg = synth.logits(B, V, seed=seed, scale=2.0)
        dev = torch.from_numpy(lg).cuda()
        tok = torch.zeros(B, dtype=torch.int32, device="cuda")
        lp = torch.zeros(B, device="cuda")
        lmu = torch.zeros(B, device="cuda")
        samp = {"temperature": tau, "top_k": k, "seed": 1234 + seed}
        for t in (0, 5, 1000):
            rlt.rlt_op_sample(dev, samp, t, tok, lp, lmu)
            torch.cuda.synchronize()
            g_tok, g_lp, g_lmu = tok.cpu().numpy(), lp.cpu().numpy(), lmu.cpu().numpy()
            for b in range(B):
                o_tok, o_lmu, o_lp, margin = oracle_lib.sample(lg[b], tau, k, samp["seed"], t, b)
                if margin > 1e-5:
                    assert g_tok[b] == o_tok, (seed, t, b)
                if g_tok[b] == o_tok:
                    assert abs(g_lmu[b] - o_lmu) < 2e-5 and abs(g_lp[b] - o_lp) < 2e-5


def test_sampled_generation_against_oracle(rlt, torch_mod, oracle_lib):
    """App. A.2: prompt prefill, then sample/consume.  Sampled ids equal the
    oracle's while every decision is clear of the numerical band; raw and
    behaviour log-probs agree within tolerance on the common prefix."""
    torch = torch_mod
    for (w, cfg), tol, band in ((_tiny(), TOL_F32, 1e-4), (_bf16_small(prompt=24), TOL_BF16, 5e-2)):
        tok = synth.tokens(w, batch=2)
        B, T = tok.shape[0], 16
        n_new = 12
        m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
        st = rlt.rlt_state_create(m, B, T + n_new, rlt.STATE_ENCODER_CACHE)
        samp = {"temperature": synth.TEMPERATURE, "top_k": synth.TOP_K, "seed": synth.SAMPLER_SEED}
        tdev = torch.from_numpy(tok[:, :T].copy()).cuda()
        rlt.rlt_prefill(m, st, tdev)
        ids = torch.zeros(n_new, B, dtype=torch.int32, device="cuda")
        lps = torch.zeros(n_new, B, device="cuda")
        lmus = torch.zeros(n_new, B, device="cuda")
        rlt.rlt_readout(m, st, sampling=samp, sampled=ids[0], logp_sampled=lps[0], logmu=lmus[0])
        for i in range(1, n_new):
            rlt.rlt_decoder_step(m, st, tokens=ids[i - 1], sampling=samp, sampled=ids[i], logp_sampled=lps[i],
                                 logmu=lmus[i])
        torch.cuda.synchronize()
        rlt.rlt_check_device()
        ids, lps, lmus = ids.cpu().numpy().T, lps.cpu().numpy().T, lmus.cpu().numpy().T
        om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
        for b in range(B):
            o = om.generate(tok[b, :T], n_new, synth.TEMPERATURE, synth.TOP_K, synth.SAMPLER_SEED, b)
            for i in range(n_new):
                if ids[b, i] == o["tokens"][i]:
                    assert abs(lps[b, i] - o["logp"][i]) <= tol
                    assert abs(lmus[b, i] - o["logmu"][i]) <= 2 * tol
                if o["margin"][i] <= band:
                    break  # decision inside the numerical band: later ids may legitimately differ
                assert ids[b, i] == o["tokens"][i], (b, i)


# ------------------------------------------------------------------ error paths
def test_error_paths(rlt, torch_mod):
    torch = torch_mod
    w, cfg = _tiny()
    tok = torch.from_numpy(synth.tokens(w)).cuda()
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    st = rlt.rlt_state_create(m, 2, 8)
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_prefill(m, st, tok)  # 32 tokens > max_len 8
    assert e.value.code == rlt.RLT_E_CAPACITY
    rlt.rlt_prefill(m, st, tok[:, :8].contiguous())
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_decoder_step(m, st, tokens=tok[:, 8].contiguous())
    assert e.value.code == rlt.RLT_E_CAPACITY
    st2 = rlt.rlt_state_create(m, 2, 16)
    rlt.rlt_prefill(m, st2, tok[:, :8].contiguous())
    with pytest.raises(rlt.RltError) as e:  # no encoder cache: x_9 cannot be encoded
        rlt.rlt_decoder_step(m, st2, tokens=tok[:, 8].contiguous())
    assert e.value.code == rlt.RLT_E_STATE
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_encode_prefix(m, st2, tok[:, :4].contiguous())
    assert e.value.code == rlt.RLT_E_STATE
    m.load_weights("s_star", np.zeros((1, cfg["d"]), np.float32))
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_readout(m, st2, next_tokens=tok[:, 8].contiguous(), logp=torch.zeros(2, device="cuda"))
    assert e.value.code == rlt.RLT_E_STALE
    rlt.rlt_state_reset(st2)
    rlt.rlt_prefill(m, st2, tok[:, :8].contiguous())
    torch.cuda.synchronize()
    rlt.rlt_check_device()


# ------------------------------------------------------------------ full size, sampled
def test_replay_full_size_sampled(rlt, torch_mod, oracle_lib):
    """The benchmark workload (reference model at L=24, B=256, S=1024, in the
    launch configuration the benchmark times): sampled sequences checked
    against the oracle on their first 40 positions (causality lets the oracle
    stop there)."""
    torch = torch_mod
    w = synth.workload("replay")
    cfg = synth.model_config(w)
    tok = synth.tokens(w)
    got, m = _gpu_replay(rlt, torch, cfg, tok)
    assert np.all(np.isfinite(got)) and np.all(got <= 0)
    om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
    for b in (0, 255):
        want = om.replay_logprobs(tok[b, :40])
        assert np.max(np.abs(got[b, :39] - want)) <= TOL_BF16


def test_batched_equals_single_wide_tiles(rlt, torch_mod):
    """At the reference width the decode GEMMs pick wider activation tiles for
    B=256 than for B=100 or B=1 (and the LM head differs too); a sequence's
    log-probs must still be bit-identical (no batch-dependent reduction
    order)."""
    w = synth.workload("replay", n_layers=1, batch=256, prompt=24)
    cfg = synth.model_config(w)
    tok = synth.tokens(w)
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    full, _ = _gpu_replay(rlt, torch_mod, cfg, tok, model=m)
    for b in (0, 131, 255):
        one, _ = _gpu_replay(rlt, torch_mod, cfg, tok[b:b + 1].copy(), model=m)
        assert np.array_equal(one[0], full[b]), (b, np.max(np.abs(one[0] - full[b])))
    # 65..128 rows take two 64-wide tiles where the plan has 128-wide ones
    mid, _ = _gpu_replay(rlt, torch_mod, cfg, tok[:100].copy(), model=m)
    assert np.array_equal(mid, full[:100])


# ------------------------------------------------------------------ RL replay ratios
def test_replay_ratios_match_oracle(rlt, torch_mod, oracle_lib):
    """Eq. 5.5 through rlt_replay_ratios: current-policy log-probs as
    rlt_replay_logprobs gives them, ratios exp(log p - log mu) on the action
    tokens and 1 elsewhere, and the trajectory log-ratio; against the
    oracle's replay on the same rollout, recorded log mu and action mask."""
    torch = torch_mod
    for (w, cfg), tol in ((_tiny(), TOL_F32), (_bf16_small(prompt=120), TOL_BF16)):
        tok = synth.tokens(w)
        B, S = tok.shape
        rng = np.random.default_rng(5150)
        logmu = rng.normal(-4.0, 1.0, (B, S - 1)).astype(np.float32)
        mask = (rng.random((B, S - 1)) < 0.6).astype(np.uint8)
        m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
        tdev = torch.from_numpy(tok).cuda()
        lp = torch.zeros(B, S - 1, device="cuda")
        ratio = torch.zeros(B, S - 1, device="cuda")
        seq = torch.zeros(B, device="cuda")
        rlt.rlt_replay_ratios(m, tdev, torch.from_numpy(logmu).cuda(), torch.from_numpy(mask).cuda(), lp, ratio, seq)
        ref = torch.zeros(B, S - 1, device="cuda")
        rlt.rlt_replay_logprobs(m, tdev, ref)
        torch.cuda.synchronize()
        rlt.rlt_check_device()
        lp, ratio, seq, ref = (x.cpu().numpy().astype(np.float64) for x in (lp, ratio, seq, ref))
        assert np.array_equal(lp, ref)
        assert np.all(ratio[mask == 0] == 1.0)
        # the kernel's arithmetic on its own log-probs (fp32 exp, fp64 sum)
        mine = np.where(mask == 1, np.exp(lp - logmu), 1.0)
        assert np.allclose(ratio, mine, rtol=1e-6, atol=0)
        assert np.allclose(seq, ((lp - logmu) * mask).sum(1), rtol=1e-6, atol=1e-4)
        om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
        for b in range(B):
            o = om.replay_ratios(tok[b], logmu[b], mask[b])
            assert np.max(np.abs(lp[b] - o["logp"])) <= tol
            assert np.all(np.abs(ratio[b] - o["ratio"]) <= o["ratio"] * math.expm1(tol) + 1e-6)
            assert abs(seq[b] - o["seq_logratio"]) <= tol * int(mask[b].sum()) + 1e-4
