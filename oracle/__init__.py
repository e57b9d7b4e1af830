"""fp64 CPU oracle of the Recurrent Looped Transformer hot path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``stateful_decoder_b200``) never imports, links or calls it; the two share no
code, and neither imports the other.  The only common dependency is the seeded
input generator in ``synth``.

The arithmetic lives in ``rlt_oracle.c`` (plain C, fp64, OpenMP over the rows
of each matrix-vector product).  This module is a ctypes binding to it: it
marshals arguments and nothing else.  The module header of the C file lists
which passage of "Recurrent Looped Transformer" each function follows.

``bptt.py`` adds the full-BPTT gradient of the replay loss (plain PyTorch
fp64 with autograd, no code shared with the C file or the library).

Functions that no test pins to anything but themselves: none.  The pins are in
``tests/test_oracle_pins.py`` and ``tests/test_oracle_bptt.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rlt_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

_c_double_p = ctypes.POINTER(ctypes.c_double)
_c_float_p = ctypes.POINTER(ctypes.c_float)
_c_int32_p = ctypes.POINTER(ctypes.c_int32)
_c_uint32_p = ctypes.POINTER(ctypes.c_uint32)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE semantics, no FMA contraction)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp.%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _SO)
    return _SO


class _Config(ctypes.Structure):
    _fields_ = [
        ("d", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("n_layers", ctypes.c_int32),
        ("window", ctypes.c_int32), ("groups", ctypes.c_int32), ("ffn", ctypes.c_int32),
        ("vocab", ctypes.c_int32), ("tied", ctypes.c_int32), ("merge_kind", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("alpha", ctypes.c_double), ("rms_eps", ctypes.c_double),
        ("rope_base", ctypes.c_double), ("init_std", ctypes.c_double), ("bos_id", ctypes.c_int32),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        L.orc_philox4x32_10.argtypes = [_c_uint32_p, _c_uint32_p, _c_uint32_p]
        L.orc_normal_ih12.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64]
        L.orc_normal_ih12.restype = ctypes.c_double
        L.orc_model_new.argtypes = [ctypes.POINTER(_Config)]
        L.orc_model_new.restype = ctypes.c_void_p
        L.orc_model_free.argtypes = [ctypes.c_void_p]
        L.orc_model_init.argtypes = [ctypes.c_void_p, ctypes.c_uint64]
        L.orc_tensor_set.argtypes = [ctypes.c_void_p, ctypes.c_char_p, ctypes.c_void_p, ctypes.c_int64]
        L.orc_tensor_get.argtypes = [ctypes.c_void_p, ctypes.c_char_p, ctypes.c_void_p, ctypes.c_int64]
        L.orc_rmsnorm.argtypes = [_c_double_p, _c_double_p, ctypes.c_int, ctypes.c_double, _c_double_p]
        L.orc_rope.argtypes = [_c_double_p, ctypes.c_int, ctypes.c_double, ctypes.c_double]
        L.orc_attend.argtypes = [_c_double_p, ctypes.POINTER(_c_double_p), ctypes.POINTER(_c_double_p),
                                 ctypes.c_int, ctypes.c_int, _c_double_p]
        L.orc_log_softmax.argtypes = [_c_double_p, ctypes.c_int, _c_double_p]
        L.orc_merge.argtypes = [ctypes.c_void_p, _c_double_p, _c_double_p, _c_double_p]
        L.orc_seq_new.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32]
        L.orc_seq_new.restype = ctypes.c_void_p
        L.orc_seq_free.argtypes = [ctypes.c_void_p]
        L.orc_encode_prefill.argtypes = [ctypes.c_void_p, _c_int32_p, ctypes.c_int32]
        L.orc_encode_step.argtypes = [ctypes.c_void_p, ctypes.c_int32]
        L.orc_decoder_step.argtypes = [ctypes.c_void_p, _c_double_p]
        L.orc_sample.argtypes = [_c_float_p, _c_double_p, ctypes.c_int32, ctypes.c_float, ctypes.c_int32,
                                 ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, _c_int32_p, _c_double_p,
                                 _c_double_p, _c_double_p]
        L.orc_replay_logprobs.argtypes = [ctypes.c_void_p, _c_int32_p, ctypes.c_int32, ctypes.c_int32, _c_double_p]
        L.orc_replay_ratios.argtypes = [ctypes.c_void_p, _c_int32_p, ctypes.c_int32, _c_double_p,
                                        ctypes.POINTER(ctypes.c_uint8), _c_double_p, _c_double_p, _c_double_p]
        L.orc_generate.argtypes = [ctypes.c_void_p, _c_int32_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                   ctypes.c_int32, ctypes.c_uint64, ctypes.c_uint32, _c_int32_p, _c_double_p,
                                   _c_double_p, _c_double_p]
        L.orc_seq_pos.argtypes = [ctypes.c_void_p, ctypes.c_int32]
        L.orc_seq_pos.restype = ctypes.c_int32
        L.orc_seq_get_s.argtypes = [ctypes.c_void_p, _c_double_p]
        L.orc_seq_set_s.argtypes = [ctypes.c_void_p, _c_double_p]
        L.orc_seq_get_e.argtypes = [ctypes.c_void_p, ctypes.c_int32, _c_double_p]
        L.orc_seq_get_mem.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _c_double_p]
        L.orc_seq_window.argtypes = [ctypes.c_void_p, ctypes.c_int32, _c_int32_p, _c_double_p, _c_double_p]
        L.orc_seq_window.restype = ctypes.c_int32
        L.orc_num_threads.restype = ctypes.c_int32
        _lib = L
    return _lib


def _dp(a: np.ndarray):
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(_c_double_p)


def _ip(a: np.ndarray):
    assert a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data_as(_c_int32_p)


# --------------------------------------------------------------------------
# building blocks (exposed for the pin tests)
# --------------------------------------------------------------------------

def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    o = np.zeros(4, dtype=np.uint32)
    lib().orc_philox4x32_10(c.ctypes.data_as(_c_uint32_p), k.ctypes.data_as(_c_uint32_p),
                            o.ctypes.data_as(_c_uint32_p))
    return o


def normal_ih12(seed: int, tensor_id: int, idx: int) -> float:
    return lib().orc_normal_ih12(seed, tensor_id, idx)


def rmsnorm(x, gamma, eps: float) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    g = np.ascontiguousarray(gamma, dtype=np.float64)
    out = np.zeros_like(x)
    lib().orc_rmsnorm(_dp(x), _dp(g), x.size, eps, _dp(out))
    return out


def rope(x, p: float, base: float = 10000.0) -> np.ndarray:
    y = np.ascontiguousarray(x, dtype=np.float64).copy()
    lib().orc_rope(_dp(y), y.size, float(p), float(base))
    return y


def attend(q, K, V) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    n, hd = K.shape
    kp = (_c_double_p * max(n, 1))(*[K[j].ctypes.data_as(_c_double_p) for j in range(n)])
    vp = (_c_double_p * max(n, 1))(*[V[j].ctypes.data_as(_c_double_p) for j in range(n)])
    out = np.zeros(hd)
    lib().orc_attend(_dp(q), kp, vp, n, hd, _dp(out))
    return out


def log_softmax(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    lib().orc_log_softmax(_dp(x), x.size, _dp(out))
    return out


def sample(logits_f32, temperature: float, top_k: int, seed: int, t: int, b: int, logits64=None):
    """Returns (token, log_mu, log_p, margin)."""
    lf = np.ascontiguousarray(logits_f32, dtype=np.float32)
    l64 = None if logits64 is None else np.ascontiguousarray(logits64, dtype=np.float64)
    tok = ctypes.c_int32()
    lmu, lp, mg = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    rc = lib().orc_sample(lf.ctypes.data_as(_c_float_p), None if l64 is None else _dp(l64), lf.size,
                          float(temperature), int(top_k), int(seed), int(t), int(b), ctypes.byref(tok),
                          ctypes.byref(lmu), ctypes.byref(lp), ctypes.byref(mg))
    if rc:
        raise ValueError("orc_sample rejected its arguments")
    return tok.value, lmu.value, lp.value, mg.value


def num_threads() -> int:
    return lib().orc_num_threads()


# --------------------------------------------------------------------------
# model and sequences
# --------------------------------------------------------------------------

def _cfg_struct(cfg: dict) -> _Config:
    return _Config(
        d=cfg["d"], n_heads=cfg["n_heads"], n_layers=cfg["n_layers"], window=cfg["window"],
        groups=cfg["groups"], ffn=cfg["ffn"], vocab=cfg["vocab"], tied=cfg.get("tied", 1),
        merge_kind=cfg.get("merge_kind", 0), dtype=cfg["dtype"], alpha=cfg.get("alpha", 1.0),
        rms_eps=cfg.get("rms_eps", 1e-6), rope_base=cfg.get("rope_base", 10000.0),
        init_std=cfg.get("init_std", 0.02), bos_id=cfg.get("bos_id", 0))


class Model:
    """Oracle model: weights in the configured storage precision."""

    def __init__(self, cfg: dict, seed: int | None = None):
        self.cfg = dict(cfg)
        self._c = _cfg_struct(cfg)
        self._lib = lib()  # kept for __del__, which may run after module teardown
        self.h = self._lib.orc_model_new(ctypes.byref(self._c))
        if not self.h:
            raise ValueError("oracle rejected the configuration")
        if seed is not None:
            lib().orc_model_init(self.h, seed)

    def __del__(self):
        if getattr(self, "h", None):
            self._lib.orc_model_free(self.h)
            self.h = None

    @property
    def storage_dtype(self):
        return np.float32 if self.cfg["dtype"] == 0 else np.uint16

    def set(self, name: str, raw: np.ndarray) -> None:
        raw = np.ascontiguousarray(raw, dtype=self.storage_dtype)
        if lib().orc_tensor_set(self.h, name.encode(), raw.ctypes.data, raw.nbytes):
            raise KeyError(name)

    def get(self, name: str, shape) -> np.ndarray:
        out = np.zeros(shape, dtype=self.storage_dtype)
        if lib().orc_tensor_get(self.h, name.encode(), out.ctypes.data, out.nbytes):
            raise KeyError(name)
        return out

    def merge(self, e, s) -> np.ndarray:
        e = np.ascontiguousarray(e, dtype=np.float64)
        s = np.ascontiguousarray(s, dtype=np.float64)
        u = np.zeros_like(e)
        lib().orc_merge(self.h, _dp(e), _dp(s), _dp(u))
        return u

    def replay_logprobs(self, tokens, schedule: int = 0) -> np.ndarray:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        out = np.zeros(tok.size - 1)
        if lib().orc_replay_logprobs(self.h, _ip(tok), tok.size, schedule, _dp(out)):
            raise ValueError("orc_replay_logprobs failed")
        return out

    def replay_ratios(self, tokens, logmu, mask) -> dict:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        lmu = np.ascontiguousarray(logmu, dtype=np.float64)
        msk = np.ascontiguousarray(mask, dtype=np.uint8)
        if lmu.size != tok.size - 1 or msk.size != tok.size - 1:
            raise ValueError("logmu and mask need S-1 entries")
        lp, r, tot = np.zeros(tok.size - 1), np.zeros(tok.size - 1), ctypes.c_double()
        if lib().orc_replay_ratios(self.h, _ip(tok), tok.size, _dp(lmu),
                                   msk.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), _dp(lp), _dp(r),
                                   ctypes.byref(tot)):
            raise ValueError("orc_replay_ratios failed")
        return {"logp": lp, "ratio": r, "seq_logratio": tot.value}

    def generate(self, prompt, n_new: int, temperature: float, top_k: int, seed: int, b: int) -> dict:
        p = np.ascontiguousarray(prompt, dtype=np.int32)
        tok = np.zeros(n_new, dtype=np.int32)
        lp, lmu, mg = np.zeros(n_new), np.zeros(n_new), np.zeros(n_new)
        if lib().orc_generate(self.h, _ip(p), p.size, n_new, float(temperature), int(top_k), int(seed), int(b),
                              _ip(tok), _dp(lp), _dp(lmu), _dp(mg)):
            raise ValueError("orc_generate failed")
        return {"tokens": tok, "logp": lp, "logmu": lmu, "margin": mg}

    def seq(self, max_len: int, keep_enc_cache: bool = True) -> "Seq":
        return Seq(self, max_len, keep_enc_cache)


class Seq:
    """One independent sequence's complete state (encoder cache, memory, H_t)."""

    def __init__(self, model: Model, max_len: int, keep_enc_cache: bool):
        self.model = model
        self.d = model.cfg["d"]
        self._lib = lib()
        self.h = self._lib.orc_seq_new(model.h, max_len, int(keep_enc_cache))
        if not self.h:
            raise ValueError("bad max_len")

    def __del__(self):
        if getattr(self, "h", None):
            self._lib.orc_seq_free(self.h)
            self.h = None

    def encode_prefill(self, tokens) -> None:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        if lib().orc_encode_prefill(self.h, _ip(tok), tok.size):
            raise ValueError("encode_prefill failed")

    def encode_step(self, token: int) -> None:
        if lib().orc_encode_step(self.h, int(token)):
            raise ValueError("encode_step failed")

    def decoder_step(self, logits: bool = True):
        out = np.zeros(self.model.cfg["vocab"]) if logits else None
        if lib().orc_decoder_step(self.h, None if out is None else _dp(out)):
            raise ValueError("decoder_step failed")
        return out

    @property
    def n_enc(self) -> int:
        return lib().orc_seq_pos(self.h, 0)

    @property
    def n_dec(self) -> int:
        return lib().orc_seq_pos(self.h, 1)

    def s(self) -> np.ndarray:
        out = np.zeros(self.d)
        lib().orc_seq_get_s(self.h, _dp(out))
        return out

    def set_s(self, s) -> None:
        s = np.ascontiguousarray(s, dtype=np.float64)
        lib().orc_seq_set_s(self.h, _dp(s))

    def e(self, pos1: int) -> np.ndarray:
        out = np.zeros(self.d)
        lib().orc_seq_get_e(self.h, pos1, _dp(out))
        return out

    def mem(self, g: int, pos1: int, which: int) -> np.ndarray:
        out = np.zeros(self.d)
        lib().orc_seq_get_mem(self.h, g, pos1, which, _dp(out))
        return out

    def window(self, layer: int):
        W = self.model.cfg["window"]
        n_max = max(W - 1, 1)
        pos = np.zeros(n_max, dtype=np.int32)
        k = np.zeros((n_max, self.d))
        v = np.zeros((n_max, self.d))
        n = lib().orc_seq_window(self.h, layer, _ip(pos), _dp(k), _dp(v))
        return pos[:n].copy(), k[:n].copy(), v[:n].copy()
