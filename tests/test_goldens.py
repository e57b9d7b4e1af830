"""The stored goldens of the full-size parity tests are the oracle's output.

``tests/golden/make_goldens.py`` writes them from the fp64 oracle alone.
These CPU checks recompute the first positions of every stored sequence with
the oracle as it stands and require agreement to 1e-12: by causality (report
Prop. B.1) the log-probs of a prefix do not depend on later tokens, so a
short replay reproduces the stored values exactly.  They also check that the
stored files match the table of the script (workload, batch, length, rows)
and that the values are log-probabilities.
"""
import numpy as np
import pytest

import synth
from tests.golden import make_goldens as goldens

N_CHECK = 6


@pytest.mark.parametrize("name", list(goldens.GOLDENS))
def test_golden_is_the_oracle_output(oracle_lib, name):
    g = goldens.load(name)
    wname, batch, length, rows, prompt = goldens.GOLDENS[name]
    assert (g["workload"], g["batch"], g["length"], g["prompt"]) == (wname, batch, length, prompt)
    assert tuple(g["rows"]) == rows
    lp = g["logp"]
    assert lp.shape == (len(rows), length - 1)
    assert np.all(np.isfinite(lp)) and np.all(lp < 0)
    w = synth.workload(wname)
    tok = synth.tokens(w, batch=batch, length=length)
    om = oracle_lib.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)
    for i, r in enumerate(rows):
        want = om.replay_logprobs(tok[r, :N_CHECK + 1])
        assert np.max(np.abs(lp[i, :N_CHECK] - want)) <= 1e-12, (name, r)


def test_gradient_golden_is_the_oracle_output(oracle_lib):
    """The stored full-BPTT gradients (float32) equal a fresh run of the
    gradient oracle on the same model, tokens and eq. 5.1 weights."""
    from oracle import bptt
    g = goldens.load_grad()
    w = goldens.grad_workload()
    tok = synth.tokens(w, batch=1)
    S = tok.shape[1]
    om = oracle_lib.Model(synth.model_config(w), seed=synth.WEIGHT_SEED)
    loss, want = bptt.loss_and_grads(om, tok[0], np.full(S - 1, 1.0 / (S - 1)))
    assert abs(loss - g["loss"]) <= 1e-12 * max(1.0, abs(loss))
    assert np.max(np.abs(om.replay_logprobs(tok[0]) - g["logp"])) <= 1e-12
    for name, stored in g["grads"].items():
        ref = want[name]
        assert stored.shape == ref.shape, name
        assert np.max(np.abs(stored.astype(np.float64) - ref)) <= 1e-6 * max(1.0, float(np.max(np.abs(ref)))), name
