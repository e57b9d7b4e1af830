"""Sequences at different positions in one batch (report §4.1: the batch
gathers ready transitions of independent sequences, each with its own
memory, cache, s and position).

Schedule, per sequence b of a batch of four:
  1. prompts of different lengths, appended to a fresh state with
     rlt_append_spans (a ragged prefill);
  2. teacher-forced generation steps: every sequence advances by one per
     rlt_decoder_step, each at its own position (encoder step over C^E,
     memory append, transition);
  3. appended spans of different lengths, one of them empty (report §6,
     multi-turn: the span is encoded over the cached prefix, then every span
     token gets its transition; a sequence whose span is over sits out);
  4. more generation steps.
Checks: every log-prob the schedule produces equals the oracle's replay of
that sequence's history (1e-4 fp32, 5e-2 bf16); every output is
bit-identical to running the sequence alone (B = 1) through the same calls;
the per-sequence positions, ring fill and ring head are exact; a snapshot of
the ragged state restores and continues bit-identically; the calls that
need equal positions refuse a ragged state.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

PROMPTS = [37, 5, 100, 64]
SPANS = [3, 0, 17, 9]
GEN1, GEN2 = 6, 4
# bf16_wide: a window of 160 (the streamed SWA kernel); two of the rings wrap
# during the prompt, one during the steps, one never
PROMPTS_WIDE = [190, 5, 230, 157]


@pytest.fixture(scope="module")
def rlt():
    import torch
    torch.cuda.init()
    import stateful_decoder_b200 as m
    return m


def _model(kind):
    if kind == "f32":
        w = synth.workload("tiny", window=4, prompt=8, batch=4)
        tol = 1e-4
    else:
        w = synth.workload("small", d=256, n_heads=2, n_layers=2, window=160 if kind == "bf16_wide" else 16,
                           groups=1, ffn=512, vocab=1024, dtype=1, batch=4, prompt=8, gen=0, dist="zipf",
                           data_seed=1201)
        tol = 5e-2
    return w, synth.model_config(w), tol, PROMPTS_WIDE if kind == "bf16_wide" else PROMPTS


def _histories(w, rows, prompts):
    n = max(prompts) + GEN1 + max(SPANS) + GEN2 + 2
    tok = synth.tokens(w, batch=4, length=n)
    return tok[rows]


def _run(rlt, torch, m, hist, prompts, spans, snapshot_at_end=False):
    """The schedule of the module docstring on the sequences `hist` [B, n].
    Returns {(b, t): log p(hist[b][t] | hist[b][:t])} for every scored
    position, the per-phase positions, and (optionally) the state."""
    B = hist.shape[0]
    n = hist.shape[1]
    st = rlt.rlt_state_create(m, B, n, rlt.STATE_ENCODER_CACHE)
    out = {}
    phases = []
    cols = torch.from_numpy(hist).cuda()

    def span_call(lens, start):
        L = max(lens)
        if L == 0:
            return
        toks = np.zeros((B, L), np.int32)
        for b in range(B):
            toks[b, :lens[b]] = hist[b, start[b]:start[b] + lens[b]]
        lp = torch.full((B, max(L - 1, 1)), 7.0, device="cuda")
        rlt.rlt_append_spans(m, st, torch.from_numpy(toks).cuda(), lens, lp)
        lp = lp.cpu().numpy()
        for b in range(B):
            for i in range(lens[b] - 1):
                out[(b, start[b] + i + 1)] = lp[b, i]

    def readout():
        pos = st.positions()["n_dec"]
        nxt = torch.from_numpy(np.array([hist[b, pos[b]] for b in range(B)], np.int32)).cuda()
        lp = torch.zeros(B, device="cuda")
        rlt.rlt_readout(m, st, next_tokens=nxt, logp=lp)
        lp = lp.cpu().numpy()
        for b in range(B):
            out[(b, int(pos[b]))] = lp[b]

    def steps(k):
        for _ in range(k):
            pos = st.positions()["n_dec"]
            x = torch.from_numpy(np.array([hist[b, pos[b]] for b in range(B)], np.int32)).cuda()
            nxt = torch.from_numpy(np.array([hist[b, pos[b] + 1] for b in range(B)], np.int32)).cuda()
            lp = torch.zeros(B, device="cuda")
            rlt.rlt_decoder_step(m, st, tokens=x, next_tokens=nxt, logp=lp)
            lp = lp.cpu().numpy()
            for b in range(B):
                out[(b, int(pos[b]) + 1)] = lp[b]

    span_call(prompts, [0] * B)
    phases.append(st.positions())
    readout()
    steps(GEN1)
    phases.append(st.positions())
    pos = st.positions()["n_dec"]
    span_call(spans, [int(p) for p in pos])
    phases.append(st.positions())
    readout()
    steps(GEN2)
    phases.append(st.positions())
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    del cols
    return out, phases, st


@pytest.mark.parametrize("kind", ["f32", "bf16", "bf16_wide"])
def test_ragged_batch(rlt, oracle_lib, kind):
    import torch
    w, cfg, tol, prompts = _model(kind)
    hist = _histories(w, [0, 1, 2, 3], prompts)
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    got, phases, st = _run(rlt, torch, m, hist, prompts, SPANS)

    # per-sequence positions and ring bookkeeping, exact
    Wm1 = cfg["window"] - 1
    want_dec = [np.array(prompts), np.array(prompts) + GEN1, np.array(prompts) + GEN1 + np.array(SPANS),
                np.array(prompts) + GEN1 + np.array(SPANS) + GEN2]
    for ph, dec in zip(phases, want_dec):
        assert np.array_equal(ph["n_dec"], dec) and np.array_equal(ph["n_enc"], dec)
        assert np.array_equal(ph["ring_valid"], np.minimum(dec, Wm1))
        assert np.array_equal(ph["ring_head"], dec % Wm1)
    info = st.info()
    assert info["uniform"] == 0 and info["n_dec"] == int(want_dec[-1].max())

    # every log-prob against the oracle's replay of the sequence's history
    om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
    for b in range(4):
        n_b = int(want_dec[-1][b])  # positions scored: 1..n_b
        ref = om.replay_logprobs(hist[b, :n_b + 1])  # ref[t-1] = log p(hist[t] | hist[:t])
        ts = sorted(t for (bb, t) in got if bb == b)
        assert ts == list(range(1, n_b + 1)), (b, ts[:5], ts[-5:])
        err = max(abs(got[(b, t)] - ref[t - 1]) for t in ts)
        assert err <= tol, (kind, b, err)

    # bit-identical to each sequence alone
    for b in range(4):
        one, ph1, st1 = _run(rlt, torch, m, hist[b:b + 1], [prompts[b]], [SPANS[b]])
        for (bb, t), v in one.items():
            assert got[(b, t)] == v, (kind, b, t, got[(b, t)], v)
        assert int(ph1[-1]["n_dec"][0]) == int(want_dec[-1][b])
        st1.free()

    # a snapshot of the ragged state restores and continues bit-identically
    snap = rlt.rlt_state_export(st)
    st2 = rlt.rlt_state_create(m, 4, st.max_len, rlt.STATE_ENCODER_CACHE)
    rlt.rlt_state_import(st2, snap)
    for k in ("n_enc", "n_dec"):
        assert np.array_equal(st2.positions()[k], st.positions()[k])
    pos = st.positions()["n_dec"]
    x = torch.from_numpy(np.array([hist[b, pos[b]] for b in range(4)], np.int32)).cuda()
    nxt = torch.from_numpy(np.array([hist[b, pos[b] + 1] for b in range(4)], np.int32)).cuda()
    a, c = torch.zeros(4, device="cuda"), torch.zeros(4, device="cuda")
    rlt.rlt_decoder_step(m, st, tokens=x, next_tokens=nxt, logp=a)
    rlt.rlt_decoder_step(m, st2, tokens=x, next_tokens=nxt, logp=c)
    assert torch.equal(a, c)
    assert np.array_equal(rlt.rlt_state_export(st), rlt.rlt_state_export(st2))

    # calls that need every sequence at one position refuse a ragged state
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_encode_prefix(m, st, torch.zeros(4, 2, dtype=torch.int32, device="cuda"))
    assert e.value.code == rlt.RLT_E_STATE
    with pytest.raises(rlt.RltError) as e:  # a span beyond max_len
        rlt.rlt_append_spans(m, st, torch.zeros(4, 4, dtype=torch.int32, device="cuda"), [0, 0, st.max_len, 0])
    assert e.value.code in (rlt.RLT_E_CAPACITY, rlt.RLT_E_INVAL)
    ids = torch.zeros(4, dtype=torch.int32, device="cuda")
    rlt.rlt_readout(m, st, sampling={"temperature": 0.8, "top_k": 5, "seed": 3}, sampled=ids)
    with pytest.raises(rlt.RltError) as e:  # the pending sampled token comes first
        rlt.rlt_append_spans(m, st, torch.zeros(4, 1, dtype=torch.int32, device="cuda"), [1, 1, 1, 1])
    assert e.value.code == rlt.RLT_E_STATE
    torch.cuda.synchronize()
    rlt.rlt_check_device()
