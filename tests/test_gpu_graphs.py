"""CUDA-graph replay of decoder steps (RLT_STATE_GRAPHS) equals plain
launches bit for bit.

The same schedule runs on two states of one model, one made with the flag:
a ragged prefill (sequences at different positions, so the step's attention
grid covers the furthest one), then sampled generation steps that cross a
256-key chunk boundary (a new step shape, so a new graph) and consume the
pending sampled token, then teacher-forced steps with explicit tokens (another
token source, another graph).  Sampled ids, behaviour log-probs, teacher
log-probs, per-sequence positions and the final snapshots must be identical.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _run(rlt, torch, m, cfg, hist, prompts, n_samp, n_teach, flags):
    B = hist.shape[0]
    st = rlt.rlt_state_create(m, B, hist.shape[1] + n_samp + 2, flags)
    toks = torch.from_numpy(hist).cuda()
    L = max(prompts)
    rlt.rlt_append_spans(m, st, toks[:, :L].contiguous(), prompts)
    samp = {"temperature": 0.8, "top_k": 50, "seed": 7}
    ids = torch.zeros(n_samp + 1, B, dtype=torch.int32, device="cuda")
    lmu = torch.zeros(n_samp + 1, B, device="cuda")
    rlt.rlt_readout(m, st, sampling=samp, sampled=ids[0], logmu=lmu[0])
    for i in range(1, n_samp + 1):
        rlt.rlt_decoder_step(m, st, sampling=samp, sampled=ids[i], logmu=lmu[i])
    lp = torch.zeros(n_teach, B, device="cuda")
    for i in range(n_teach):
        x = ids[n_samp].contiguous() if i == 0 else toks[:, i].contiguous()
        rlt.rlt_decoder_step(m, st, tokens=x, next_tokens=toks[:, i + 1].contiguous(), logp=lp[i])
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    return ids.cpu().numpy(), lmu.cpu().numpy(), lp.cpu().numpy(), st.positions(), rlt.rlt_state_export(st)


@pytest.mark.parametrize("kind", ["f32", "bf16"])
def test_graph_replay_equals_plain_launches(kind):
    import torch
    import stateful_decoder_b200 as rlt
    if kind == "f32":
        w = synth.workload("tiny", window=4, prompt=8, batch=3)
    else:
        w = synth.workload("small", d=256, n_heads=2, n_layers=2, window=16, groups=1, ffn=512, vocab=1024, dtype=1,
                           batch=3, prompt=8, gen=0, dist="zipf", data_seed=1301)
    cfg = synth.model_config(w)
    prompts = [250, 100, 17]  # the furthest sequence crosses 256 keys during sampling
    hist = synth.tokens(w, batch=3, length=max(prompts) + 8)
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    plain = _run(rlt, torch, m, cfg, hist, prompts, 12, 4, rlt.STATE_ENCODER_CACHE)
    graph = _run(rlt, torch, m, cfg, hist, prompts, 12, 4, rlt.STATE_ENCODER_CACHE | rlt.STATE_GRAPHS)
    for a, b in zip(plain[:3], graph[:3]):
        assert np.array_equal(a, b)
    for k in ("n_enc", "n_dec"):
        assert np.array_equal(plain[3][k], graph[3][k])
    assert np.array_equal(plain[4], graph[4])
    assert int(graph[3]["n_dec"][0]) > 256
