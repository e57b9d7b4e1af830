"""The C-ABI library loads and exports every entry point include/rlt.h
declares; argument validation runs on the host without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "rlt.h")).read()
    return sorted(set(re.findall(r"^int32_t\s+(rlt_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for need in ("rlt_init_weights", "rlt_encode_prefix", "rlt_decoder_step", "rlt_prefill", "rlt_replay_logprobs"):
        assert need in names


def test_library_exports_every_declared_symbol():
    import stateful_decoder_b200 as rlt
    lib = ctypes.CDLL(rlt.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(rlt.EXPORTED)


def test_invalid_config_rejected_on_host():
    import stateful_decoder_b200 as rlt
    import synth
    bad = synth.model_config(synth.workload("tiny"))
    bad["n_heads"] = 3  # 64 % 3 != 0
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_init_weights(bad, 42)
    assert e.value.code == rlt.RLT_E_INVAL
    bad = synth.model_config(synth.workload("small"))
    bad["d"] = 520  # bf16 models need d % 128 == 0
    bad["n_heads"] = 8
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_init_weights(bad, 42)
    assert e.value.code == rlt.RLT_E_INVAL
    code, msg = rlt.rlt_last_error()
    assert code == rlt.RLT_E_INVAL and "128" in msg
    for g in (0, 3):
        c = synth.model_config(synth.workload("tiny"))
        c["groups"] = g
        with pytest.raises(rlt.RltError):
            rlt.rlt_init_weights(c, 42)


def test_op_arguments_validated_on_host():
    import stateful_decoder_b200 as rlt
    lib = rlt._lib
    assert lib.rlt_op_linear(None, None, None, 128, 1, 64, 1, 1, None) == rlt.RLT_E_INVAL
    s = rlt.Sampling(temperature=0.0, top_k=50, seed=1)
    assert lib.rlt_op_sample(ctypes.c_void_p(16), 1, 10, ctypes.byref(s), 0, ctypes.c_void_p(16), None, None,
                             None) == rlt.RLT_E_INVAL
    s = rlt.Sampling(temperature=0.8, top_k=257, seed=1)
    assert lib.rlt_op_sample(ctypes.c_void_p(16), 1, 10, ctypes.byref(s), 0, ctypes.c_void_p(16), None, None,
                             None) == rlt.RLT_E_INVAL


def test_state_and_replay_arguments_validated_on_host():
    """Snapshot, replay and step entry points reject missing handles and
    buffers before touching a device."""
    import stateful_decoder_b200 as rlt
    lib = rlt._lib
    used = ctypes.c_size_t(0)
    assert lib.rlt_state_export(None, None, 0, ctypes.byref(used), None) == rlt.RLT_E_INVAL
    assert lib.rlt_state_import(None, None, 0, None) == rlt.RLT_E_INVAL
    assert lib.rlt_replay_logprobs(None, None, 1, 2, None, None) == rlt.RLT_E_INVAL
    assert lib.rlt_replay_ratios(None, None, 1, 2, None, None, None, None, None, None) == rlt.RLT_E_INVAL
    assert lib.rlt_decoder_step(None, None, None, None, None, None, None) == rlt.RLT_E_INVAL
    assert lib.rlt_encode_prefix(None, None, None, 0, None) == rlt.RLT_E_INVAL
    buf = ctypes.create_string_buffer(256)
    assert lib.rlt_last_error(buf, 256) == rlt.RLT_E_INVAL
    assert buf.value  # the last failure's text


def test_backward_arguments_validated_on_host():
    """The backward entry points reject missing handles and buffers, and
    a gradient of an unknown tensor, before touching a device."""
    import stateful_decoder_b200 as rlt
    lib = rlt._lib
    assert lib.rlt_replay_backward(None, None, 1, 2, None, 4, None, None) == rlt.RLT_E_INVAL
    assert lib.rlt_grad_zero(None, None) == rlt.RLT_E_INVAL
    assert lib.rlt_backward_release(None) == rlt.RLT_E_INVAL
    buf = (ctypes.c_float * 4)()
    assert lib.rlt_grad_read(None, b"emb", buf, 16) == rlt.RLT_E_INVAL


class _FakeCuda:
    """A CPU tensor that passes the binding's device checks and hands the
    library a null pointer, so that only the binding's size checks can
    refuse a call (and a call that got through would be rejected by the
    library's own null checks, never reach a device)."""

    def __init__(self, t):
        self.t = t
        self.is_cuda = True
        self.shape = t.shape
        self.dtype = t.dtype

    def numel(self):
        return self.t.numel()

    def dim(self):
        return self.t.dim()

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return 0


def test_binding_refuses_short_buffers():
    """The C ABI receives bare pointers, so the binding checks every buffer
    the library writes or reads against the size the call implies."""
    import types

    import torch

    import stateful_decoder_b200 as rlt

    def z(*shape, dtype=torch.float32):
        return _FakeCuda(torch.zeros(*shape, dtype=dtype))

    i32 = torch.int32
    model = types.SimpleNamespace(h=None, cfg={"vocab": 40})
    state = types.SimpleNamespace(h=None, batch=2)
    tok = z(2, 9, dtype=i32)
    samp = {"temperature": 1.0, "top_k": 4, "seed": 1}
    cases = [
        (lambda: rlt.rlt_replay_logprobs(model, tok, z(2, 7)), "elements"),
        (lambda: rlt.rlt_replay_backward(model, tok, z(2, 7)), "elements"),
        (lambda: rlt.rlt_replay_backward(model, tok, z(2, 8), logp=z(2, 7)), "elements"),
        (lambda: rlt.rlt_replay_ratios(model, tok, z(2, 8), z(2, 8, dtype=torch.uint8), z(2, 8),
                                       seq_logratio=z(1)), "elements"),
        (lambda: rlt.rlt_prefill(model, state, tok, logp=z(2, 7)), "elements"),
        (lambda: rlt.rlt_prefill(model, state, z(3, 9, dtype=i32)), "shape"),
        (lambda: rlt.rlt_encode_prefix(model, state, z(9, dtype=i32)), "shape"),
        (lambda: rlt.rlt_readout(model, state, logits=z(2, 39)), "elements"),
        (lambda: rlt.rlt_decoder_step(model, state, tokens=z(1, dtype=i32)), "elements"),
        (lambda: rlt.rlt_op_sample(z(3, 40), samp, 0, z(2, dtype=i32)), "elements"),
        (lambda: rlt.rlt_op_linear(z(4, 8), z(3, 8), z(3, 3)), "elements"),
        (lambda: rlt.rlt_op_linear(z(4, 8), z(3, 7), z(3, 4)), "x must be"),
        (lambda: rlt.rlt_op_prefix_attention(z(2, 32), z(2, 2, 8, 16), z(2, 2, 8, 16), 4, z(2, 31)), "elements"),
        (lambda: rlt.rlt_op_prefix_attention(z(2, 32), z(2, 2, 8, 16), z(2, 2, 8, 16), 4, z(2, 32),
                                             rope_cs=z(4, 8, 2), qpos=4), "elements"),
        (lambda: rlt.rlt_op_prefix_attention(z(2, 32), z(2, 2, 8, 16), z(2, 2, 7, 16), 4, z(2, 32)), "match"),
    ]
    for i, (call, msg) in enumerate(cases):
        with pytest.raises(ValueError, match=msg):
            call()
    # a correctly sized call gets through the binding to the library, whose
    # own checks then refuse the null handle
    with pytest.raises(rlt.RltError):
        rlt.rlt_replay_logprobs(model, tok, z(2, 8), stream=0)
