"""Failure detection of the bounded device waits, made to run out on purpose
without faulting the GPU.

Every mbarrier wait of the tensor-core kernels is bounded by %globaltimer;
when a wait runs out the kernel raises a device error word and returns
instead of spinning, and rlt_check_device() reports RLT_E_CUDA.  The probe
entry point waits on a barrier that no thread ever arrives at, with a 1 ms
limit: the kernel must come back, the error must be reported once and
cleared, and the context must still compute correct results afterwards.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_context_stays_usable(oracle_lib):
    import torch
    import stateful_decoder_b200 as rlt
    rlt.rlt_check_device()  # nothing pending from earlier tests
    waited = rlt.rlt_test_bounded_wait(1000)  # 1 ms limit
    assert 1_000_000 <= waited < 1_000_000_000, waited
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_check_device()
    assert e.value.code == rlt.RLT_E_CUDA and "bounded device wait ran out" in str(e.value)
    rlt.rlt_check_device()  # the word was cleared
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_test_bounded_wait(0)
    assert e.value.code == rlt.RLT_E_INVAL
    # a following replay (tensor-core GEMMs and attention, whose waits now
    # complete) still matches the oracle
    w = synth.workload("small", d=256, n_heads=2, n_layers=2, window=16, ffn=512, vocab=1024, batch=2, prompt=40)
    cfg = synth.model_config(w)
    tok = synth.tokens(w)
    m = rlt.rlt_init_weights(cfg, synth.WEIGHT_SEED)
    out = torch.zeros(2, 39, device="cuda")
    rlt.rlt_replay_logprobs(m, torch.from_numpy(tok).cuda(), out)
    torch.cuda.synchronize()
    rlt.rlt_check_device()
    om = oracle_lib.Model(cfg, seed=synth.WEIGHT_SEED)
    want = np.stack([om.replay_logprobs(tok[b]) for b in range(2)])
    assert np.max(np.abs(out.cpu().numpy() - want)) <= 5e-2
