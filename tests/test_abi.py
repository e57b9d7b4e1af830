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
