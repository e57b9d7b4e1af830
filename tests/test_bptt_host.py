"""The library's full-BPTT engine, run on the CPU.

``stateful_decoder_b200/csrc/bptt_core.h`` holds the reverse-time schedule
and every operation of the backward pass as functors.  The CUDA backend runs
them as kernels.  Here ``tests/bptt_host/bptt_host.cpp`` runs the same
functors in a host loop, in fp64, built with AddressSanitizer and
UBSanitizer.  Every gradient entry must equal the gradient oracle
(``oracle.bptt``, autograd over the fp64 forward); a single out-of-bounds
index or bad stride fails the sanitizers.  The variants cover tied and
untied stacks, both merge forms, G = 1 and G = L (up to three layers), one
head and several, W = 1, W wrapping, W >= S, another RoPE base, and segment
lengths from 1 to the whole sequence.
"""
import os
import shutil
import struct
import subprocess

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "bptt_host", "bptt_host.cpp")
CORE = os.path.join(ROOT, "stateful_decoder_b200", "csrc", "bptt_core.h")
EXE = os.path.join(ROOT, "tests", "_build", "bptt_host")


@pytest.fixture(scope="module")
def host_exe():
    if shutil.which("g++") is None:
        pytest.skip("no g++")
    os.makedirs(os.path.dirname(EXE), exist_ok=True)
    if not os.path.exists(EXE) or os.path.getmtime(EXE) < max(os.path.getmtime(SRC), os.path.getmtime(CORE)):
        base = ["g++", "-std=c++17", "-O1", "-g", "-Wall", "-Wextra", "-Werror", "-I", os.path.dirname(CORE), SRC,
                "-o", EXE]
        san = ["-fsanitize=address,undefined", "-fno-omit-frame-pointer", "-fno-sanitize-recover=undefined"]
        r = subprocess.run(base + san, capture_output=True, text=True)
        if r.returncode != 0:  # a toolchain without the sanitizer runtimes: check the arithmetic alone
            subprocess.run(base, check=True, capture_output=True, text=True)
    return EXE


def _dims(cfg, B, S):
    return [B, S, cfg["d"], cfg["n_heads"], cfg["n_layers"], cfg["window"], cfg["groups"], cfg["ffn"],
            cfg["vocab"], cfg.get("tied", 1), cfg.get("merge_kind", 0)]


def _names(exe, cfg, B, S):
    out = subprocess.run([exe, "names"] + [str(v) for v in _dims(cfg, B, S)], check=True, capture_output=True,
                         text=True).stdout
    return [(ln.split()[1], int(ln.split()[2]), int(ln.split()[3])) for ln in out.strip().splitlines()]


def _run_host(exe, tmp_path, cfg, P, tok, wts, seg, passes=1):
    B, S = tok.shape
    names = _names(exe, cfg, B, S)
    inp, outp = str(tmp_path / "in.bin"), str(tmp_path / "out.bin")
    with open(inp, "wb") as f:
        f.write(struct.pack("<12i", *_dims(cfg, B, S), seg))
        f.write(struct.pack("<3d", cfg["alpha"], cfg["rms_eps"], cfg["rope_base"]))
        f.write(np.ascontiguousarray(tok, dtype=np.int32).tobytes())
        f.write(np.ascontiguousarray(wts, dtype=np.float64).tobytes())
        for name, r, c in names:
            a = P[name]
            assert a.shape == (r, c), name
            f.write(np.ascontiguousarray(a, dtype=np.float64).tobytes())
    env = dict(os.environ, ASAN_OPTIONS="detect_leaks=1:abort_on_error=0", UBSAN_OPTIONS="halt_on_error=1")
    r = subprocess.run([exe, "run", inp, outp, str(passes)], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-4000:]
    raw = np.fromfile(outp, dtype=np.float64)
    n_lp = B * (S - 1)
    logp, off, grads = raw[:n_lp].reshape(B, S - 1), n_lp, {}
    for name, rr, cc in names:
        grads[name] = raw[off:off + rr * cc].reshape(rr, cc)
        off += rr * cc
    assert off == raw.size
    return logp, grads


VARIANTS = [
    (dict(), 1),
    (dict(), 5),
    (dict(window=1), 3),
    (dict(tied=0, merge_kind=1, groups=2, window=3), 2),
    (dict(window=32, alpha=0.5), 31),
    (dict(dtype=1, window=5), 4),
    (dict(n_layers=3, groups=3, window=2, n_heads=1, rope_base=500.0), 6),
]


@pytest.mark.parametrize("kw,seg", VARIANTS,
                         ids=["seg1", "seg5", "W1_seg3", "untied_convex_GL_seg2", "fullwin_oneseg", "bf16_seg4",
                              "L3_GL_one_head_base500_seg6"])
def test_host_engine_equals_gradient_oracle(oracle_lib, host_exe, tmp_path, kw, seg):
    from oracle import bptt
    w = synth.workload("tiny", **dict(dict(d=32, n_heads=4, ffn=48, vocab=40, prompt=12), **kw))
    cfg = synth.model_config(w)
    m = oracle_lib.Model(cfg, seed=42)
    rng = np.random.default_rng(11)
    for name, shp in bptt.tensor_shapes(cfg).items():  # gains and the gate bias away from 1 and 0
        if cfg["dtype"] == 0 and (name.startswith("g_") or name == "b_gate"):
            m.set(name, 1.0 * (name != "b_gate") + 0.2 * rng.standard_normal(shp))
    tok = synth.tokens(w, batch=2)
    B, S = tok.shape
    wts = rng.uniform(-1.0, 1.0, (B, S - 1))
    P = {k: v.detach().numpy() for k, v in bptt.parameters(m).items()}
    logp, grads = _run_host(host_exe, tmp_path, cfg, P, tok, wts, seg)
    want = {k: np.zeros_like(v) for k, v in P.items()}
    for b in range(B):
        assert np.max(np.abs(logp[b] - m.replay_logprobs(tok[b]))) < 1e-11
        _, g = bptt.loss_and_grads(m, tok[b], wts[b])
        for k in want:
            want[k] += g[k]
    assert set(grads) == set(want)
    for k in want:
        scale = max(1.0, np.max(np.abs(want[k])))
        assert np.max(np.abs(grads[k] - want[k])) < 1e-10 * scale, k


def test_host_engine_reused_for_more_passes(oracle_lib, host_exe, tmp_path):
    """One engine running three passes (as the library keeps it between calls
    of one size): every pass starts from zeroed buffers, so the gradients are
    exactly three times one pass's and the log-probs the oracle's."""
    from oracle import bptt
    w = synth.workload("tiny", d=32, n_heads=4, ffn=48, vocab=40, prompt=12, window=3)
    cfg = synth.model_config(w)
    m = oracle_lib.Model(cfg, seed=42)
    rng = np.random.default_rng(13)
    tok = synth.tokens(w, batch=2)
    B, S = tok.shape
    wts = rng.uniform(-1.0, 1.0, (B, S - 1))
    P = {k: v.detach().numpy() for k, v in bptt.parameters(m).items()}
    logp1, g1 = _run_host(host_exe, tmp_path, cfg, P, tok, wts, 4)
    logp3, g3 = _run_host(host_exe, tmp_path, cfg, P, tok, wts, 4, passes=3)
    assert np.array_equal(logp1, logp3)
    for b in range(B):
        assert np.max(np.abs(logp3[b] - m.replay_logprobs(tok[b]))) < 1e-11
    for k in g1:
        scale = max(1.0, np.max(np.abs(g1[k])))
        assert np.max(np.abs(g3[k] - 3.0 * g1[k])) < 1e-12 * scale, k
