"""Multi-turn cache semantics of "Recurrent Looped Transformer" §6 and App. A
through the C ABI: the chunked encoder schedule (an appended span encoded in
one pass over the cached prefix), exact prefix snapshots (export, import,
continue) and the pending sampled token.

The chunked schedule computes every row exactly as the one-pass schedule
does (rows of the contraction are independent and the attention visits key
tiles in the same order), so the comparisons between the two GPU schedules
are bit-exact.  A restored snapshot continues bit-identically.  The appended
multi-turn history is also scored against the fp64 oracle on the same
synthetic tokens, at the usual tolerances.
"""
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
    base = dict(d=256, n_heads=2, n_layers=2, window=16, groups=1, ffn=512, vocab=1024, dtype=1, batch=3,
                prompt=300, gen=0, dist="zipf", data_seed=1101)
    base.update(kw)
    w = synth.workload("small", **base)
    return w, synth.model_config(w)


CASES = [
    pytest.param(lambda: _tiny(prompt=48), TOL_F32, 17, id="fp32-tiny"),
    pytest.param(lambda: _tiny(prompt=48, groups=2, merge_kind=1), TOL_F32, 30, id="fp32-G2-convex"),
    pytest.param(lambda: _bf16_small(prompt=300), TOL_BF16, 137, id="bf16-hd128"),
    pytest.param(lambda: _bf16_small(prompt=200, n_heads=4, groups=2), TOL_BF16, 129, id="bf16-hd64-G2"),
]


def _read_all(rlt, st, cfg, n):
    """Encoder outputs, memory and encoder cache rows 0..n-1 of every sequence."""
    out = {"e": st.read(rlt.READ_E)[:, :n]}
    for g in range(cfg["groups"]):
        out[f"mk{g}"] = st.read(rlt.READ_MEM_K, g)[:, :, :n]
        out[f"mv{g}"] = st.read(rlt.READ_MEM_V, g)[:, :, :n]
    for l in range(cfg["n_layers"]):
        out[f"ck{l}"] = st.read(rlt.READ_ENC_K, l)[:, :, :n]
        out[f"cv{l}"] = st.read(rlt.READ_ENC_V, l)[:, :, :n]
    return out


def _teacher_steps(rlt, torch, m, st, tdev, t0, t1):
    """Transitions t0+1..t1 on teacher tokens (already encoded), returning the
    log-prob of each next token."""
    col = torch.zeros(tdev.shape[0], device="cuda")
    got = []
    for t in range(t0 + 1, t1 + 1):
        rlt.rlt_decoder_step(m, st, next_tokens=tdev[:, t].contiguous() if t < tdev.shape[1] else None,
                             logp=col if t < tdev.shape[1] else None)
        if t < tdev.shape[1]:
            got.append(col.cpu().numpy().copy())
    return np.stack(got, axis=1) if got else np.zeros((tdev.shape[0], 0))


@pytest.mark.parametrize("make,tol,T1", CASES)
def test_chunked_encoder_equals_one_pass(rlt, torch_mod, make, tol, T1):
    """Encoding x_1..x_T1 and then x_T1+1..x_T in a second pass over the cached
    prefix leaves exactly the encoder outputs, memory and encoder cache of one
    pass over x_1..x_T, and the decoder then scores identically."""
    torch = torch_mod
    w, cfg = make()
    tok = synth.tokens(w)
    B, T = tok.shape
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    tdev = torch.from_numpy(tok).cuda()
    one = rlt.rlt_state_create(m, B, T, rlt.STATE_ENCODER_CACHE)
    two = rlt.rlt_state_create(m, B, T + 5, rlt.STATE_ENCODER_CACHE)
    rlt.rlt_encode_prefix(m, one, tdev)
    rlt.rlt_encode_prefix(m, two, tdev[:, :T1].contiguous())
    assert two.info()["n_enc"] == T1 and two.info()["n_dec"] == 0
    rlt.rlt_encode_prefix(m, two, tdev[:, T1:].contiguous())
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    assert two.info()["n_enc"] == T
    a, b = _read_all(rlt, one, cfg, T), _read_all(rlt, two, cfg, T)
    for k in a:
        assert np.array_equal(a[k].view(np.uint8), b[k].view(np.uint8)), k
    la = _teacher_steps(rlt, torch, m, one, tdev, 0, T - 1)
    lb = _teacher_steps(rlt, torch, m, two, tdev, 0, T - 1)
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    assert np.array_equal(la, lb)


@pytest.mark.parametrize("make,tol,T1", CASES)
def test_multi_turn_append_matches_oracle(rlt, torch_mod, oracle_lib, make, tol, T1):
    """Report §6 and App. A.2: a prompt prefill, a response consumed token by
    token (encoder steps), then an external span appended with the chunked
    encoder and stepped through the decoder: the log-probs of every scored
    token equal the oracle's replay of the whole history."""
    torch = torch_mod
    w, cfg = make()
    tok = synth.tokens(w)
    B, S = tok.shape
    T0, R = T1 // 2 + 1, 6  # prompt length, response tokens consumed one at a time
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    tdev = torch.from_numpy(tok).cuda()
    st = rlt.rlt_state_create(m, B, S, rlt.STATE_ENCODER_CACHE)
    pre = torch.zeros(B, T0 - 1, device="cuda")
    rlt.rlt_prefill(m, st, tdev[:, :T0].contiguous(), pre)
    got = [pre.cpu().numpy()]
    col = torch.zeros(B, device="cuda")
    rlt.rlt_readout(m, st, next_tokens=tdev[:, T0].contiguous(), logp=col)
    got.append(col.cpu().numpy()[:, None].copy())
    for t in range(T0 + 1, T0 + R + 1):  # response: encoder step + transition per token
        rlt.rlt_decoder_step(m, st, tokens=tdev[:, t - 1].contiguous(), next_tokens=tdev[:, t].contiguous(), logp=col)
        got.append(col.cpu().numpy()[:, None].copy())
    n = T0 + R
    assert st.info()["n_enc"] == n and st.info()["n_dec"] == n
    rlt.rlt_encode_prefix(m, st, tdev[:, n:].contiguous())  # the appended span, one pass
    got.append(_teacher_steps(rlt, torch, m, st, tdev, n, S - 1))
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    got = np.concatenate(got, axis=1).astype(np.float64)
    om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
    want = np.stack([om.replay_logprobs(tok[b]) for b in range(B)])
    assert got.shape == want.shape
    assert np.max(np.abs(got - want)) <= tol


@pytest.mark.parametrize("make,tol,T1", CASES[::2])
def test_snapshot_restores_bit_exact(rlt, torch_mod, make, tol, T1):
    """An exact prefix snapshot taken mid-generation (ring wrapped, a sampled
    token pending) restores into a fresh state with a larger max_len, and both
    states continue identically: sampled ids, log-probs and s_t."""
    torch = torch_mod
    w, cfg = make()
    tok = synth.tokens(w)
    B = tok.shape[0]
    T0 = min(T1, 40)
    n_new = 10
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    samp = {"temperature": synth.TEMPERATURE, "top_k": synth.TOP_K, "seed": synth.SAMPLER_SEED}
    a = rlt.rlt_state_create(m, B, T0 + 2 * n_new, rlt.STATE_ENCODER_CACHE)
    tdev = torch.from_numpy(tok[:, :T0].copy()).cuda()
    rlt.rlt_prefill(m, a, tdev)
    ids = torch.zeros(B, dtype=torch.int32, device="cuda")
    rlt.rlt_readout(m, a, sampling=samp, sampled=ids)
    for _ in range(3):  # consume pending tokens, sampling the next each time
        rlt.rlt_decoder_step(m, a, sampling=samp, sampled=ids)
    assert a.info()["has_pending"] == 1
    snap = rlt.rlt_state_export(a)
    b = rlt.rlt_state_create(m, B, T0 + 3 * n_new, rlt.STATE_ENCODER_CACHE)
    rlt.rlt_state_import(b, snap)
    ia, ib = a.info(), b.info()
    for k in ("n_enc", "n_dec", "ring_valid", "ring_head", "has_pending"):
        assert ia[k] == ib[k], k
    assert np.array_equal(a.read(rlt.READ_S), b.read(rlt.READ_S))

    def cont(st):
        out_ids, out_lp = [], []
        sid = torch.zeros(B, dtype=torch.int32, device="cuda")
        lp = torch.zeros(B, device="cuda")
        for _ in range(n_new):
            rlt.rlt_decoder_step(m, st, sampling=samp, sampled=sid, logp_sampled=lp)
            out_ids.append(sid.cpu().numpy().copy())
            out_lp.append(lp.cpu().numpy().copy())
        return np.stack(out_ids), np.stack(out_lp), st.read(rlt.READ_S)

    ca, cb = cont(a), cont(b)
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    for x, y in zip(ca, cb):
        assert np.array_equal(x, y)
    # the two continued states export byte for byte the same snapshot
    assert np.array_equal(rlt.rlt_state_export(b), rlt.rlt_state_export(a))


def test_pending_token_is_consumed_once(rlt, torch_mod):
    """App. A: the state represents the consumed prefix; a sampled token is
    recorded as pending, the next transition consumes it (tokens=None), and
    consuming it equals passing the sampled ids explicitly."""
    torch = torch_mod
    w, cfg = _tiny()
    tok = synth.tokens(w)
    B = tok.shape[0]
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    samp = {"temperature": synth.TEMPERATURE, "top_k": synth.TOP_K, "seed": synth.SAMPLER_SEED}
    tdev = torch.from_numpy(tok[:, :12].copy()).cuda()
    sts = [rlt.rlt_state_create(m, B, 24, rlt.STATE_ENCODER_CACHE) for _ in range(2)]
    ids = torch.zeros(B, dtype=torch.int32, device="cuda")
    for st in sts:
        rlt.rlt_prefill(m, st, tdev)
        assert st.info()["has_pending"] == 0
        with pytest.raises(rlt.RltError) as e:  # nothing sampled yet: x_13 must be given
            rlt.rlt_decoder_step(m, st)
        assert e.value.code == rlt.RLT_E_STATE
        rlt.rlt_readout(m, st, sampling=samp, sampled=ids)
        assert st.info()["has_pending"] == 1
    rlt.rlt_decoder_step(m, sts[0])
    rlt.rlt_decoder_step(m, sts[1], tokens=ids)
    for st in sts:
        assert st.info()["has_pending"] == 0 and st.info()["n_dec"] == 13
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    assert np.array_equal(sts[0].read(rlt.READ_S), sts[1].read(rlt.READ_S))
    with pytest.raises(rlt.RltError) as e:  # the pending token was consumed
        rlt.rlt_decoder_step(m, sts[0])
    assert e.value.code == rlt.RLT_E_STATE


def test_snapshot_errors(rlt, torch_mod):
    torch = torch_mod
    w, cfg = _tiny()
    tok = torch.from_numpy(synth.tokens(w)[:, :10].copy()).cuda()
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    a = rlt.rlt_state_create(m, 2, 16, rlt.STATE_ENCODER_CACHE)
    rlt.rlt_prefill(m, a, tok)
    snap = rlt.rlt_state_export(a)

    def code_of(fn):
        with pytest.raises(rlt.RltError) as e:
            fn()
        return e.value.code

    assert code_of(lambda: rlt.rlt_state_import(rlt.rlt_state_create(m, 3, 16, rlt.STATE_ENCODER_CACHE), snap)) \
        == rlt.RLT_E_INVAL  # batch
    assert code_of(lambda: rlt.rlt_state_import(rlt.rlt_state_create(m, 2, 8, rlt.STATE_ENCODER_CACHE), snap)) \
        == rlt.RLT_E_CAPACITY  # positions beyond max_len
    bad = snap.copy()
    bad[0] ^= 1
    assert code_of(lambda: rlt.rlt_state_import(a, bad)) == rlt.RLT_E_INVAL  # magic
    assert code_of(lambda: rlt.rlt_state_import(a, snap[:-4])) == rlt.RLT_E_INVAL  # truncated
    other = rlt.rlt_init_weights(dict(cfg, window=5), synth.WEIGHT_SEED)
    assert code_of(lambda: rlt.rlt_state_import(rlt.rlt_state_create(other, 2, 16), snap)) == rlt.RLT_E_INVAL
    reseeded = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED + 1)
    assert code_of(lambda: rlt.rlt_state_import(rlt.rlt_state_create(reseeded, 2, 16), snap)) == rlt.RLT_E_STALE
    nocache = rlt.rlt_state_create(m, 2, 16)
    rlt.rlt_prefill(m, nocache, tok)
    assert code_of(lambda: rlt.rlt_state_import(a, rlt.rlt_state_export(nocache))) == rlt.RLT_E_STATE
    rlt.rlt_state_import(rlt.rlt_state_create(m, 2, 16), snap)  # a state without the cache may drop it
    m.load_weights("s_star", np.zeros((1, cfg["d"]), np.float32))  # weight update: old snapshots are stale
    assert code_of(lambda: rlt.rlt_state_import(rlt.rlt_state_create(m, 2, 16, rlt.STATE_ENCODER_CACHE), snap)) \
        == rlt.RLT_E_STALE
    torch.cuda.synchronize()
    rlt.rlt_check_device()


def test_model_free_refuses_live_states(rlt, torch_mod):
    """A model is not freed under a live state (its handle stays valid); once
    the state is gone it frees normally.  The model-owned replay state does
    not count."""
    w, cfg = _tiny()
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    tok = torch_mod.from_numpy(synth.tokens(w)[:, :6].copy()).cuda()
    lp = torch_mod.zeros((tok.shape[0], 5), dtype=torch_mod.float32, device="cuda")
    rlt.rlt_replay_logprobs(m, tok, lp)
    st = rlt.rlt_state_create(m, 2, 8)
    assert m.free() == rlt.RLT_E_STATE
    assert rlt.rlt_last_error()[0] == rlt.RLT_E_STATE
    rlt.rlt_prefill(m, st, tok)  # the model still works
    st.free()
    assert m.free() == rlt.RLT_OK
    assert m.free() == rlt.RLT_OK  # idempotent
