"""Python binding of librlt.so, the sm_100a implementation of the Recurrent
Looped Transformer hot path (C ABI in include/rlt.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the library.  Device arrays are torch CUDA tensors (their
``data_ptr()`` is handed to the library); host arrays are numpy arrays.  The
library must have been built (``stateful_decoder_b200.build.build()``); if it
is missing this module raises at import -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librlt.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python stateful_decoder_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

RLT_OK = 0
RLT_E_INVAL = -1
RLT_E_CAPACITY = -2
RLT_E_OOM = -3
RLT_E_CUDA = -4
RLT_E_STALE = -5
RLT_E_STATE = -6

MERGE_PAPER = 0
MERGE_CONVEX = 1
DTYPE_F32 = 0
DTYPE_BF16 = 1
STATE_ENCODER_CACHE = 1
STATE_GRAPHS = 2

READ_S, READ_E, READ_RING_K, READ_RING_V, READ_MEM_K, READ_MEM_V, READ_ENC_K, READ_ENC_V = range(8)

EXPORTED = (
    "rlt_init_weights", "rlt_load_weights", "rlt_get_weights", "rlt_tensor_info", "rlt_model_free",
    "rlt_state_create", "rlt_state_free", "rlt_state_reset", "rlt_state_info_get", "rlt_state_read",
    "rlt_encode_prefix", "rlt_readout", "rlt_decoder_step", "rlt_prefill", "rlt_replay_logprobs",
    "rlt_last_error", "rlt_check_device", "rlt_profile_enable", "rlt_profile_read", "rlt_op_linear",
    "rlt_op_sample", "rlt_kernel_launches", "rlt_op_prefix_attention", "rlt_op_prefix_attention_noalloc",
    "rlt_state_export", "rlt_state_import", "rlt_replay_ratios", "rlt_replay_backward", "rlt_grad_read",
    "rlt_grad_zero", "rlt_test_bounded_wait", "rlt_state_positions", "rlt_append_spans", "rlt_backward_release",
)


class RltError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"rlt error {code}: {msg}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("n_layers", ctypes.c_int32),
        ("window", ctypes.c_int32), ("groups", ctypes.c_int32), ("ffn", ctypes.c_int32), ("vocab", ctypes.c_int32),
        ("tied", ctypes.c_int32), ("merge_kind", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("alpha", ctypes.c_float), ("rms_eps", ctypes.c_float), ("rope_base", ctypes.c_float),
        ("init_std", ctypes.c_float), ("bos_id", ctypes.c_int32),
    ]


class Sampling(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("top_k", ctypes.c_int32), ("seed", ctypes.c_uint64)]


class ReadoutOut(ctypes.Structure):
    _fields_ = [("logp", ctypes.c_void_p), ("sampled", ctypes.c_void_p), ("logp_sampled", ctypes.c_void_p),
                ("logmu", ctypes.c_void_p), ("logits", ctypes.c_void_p)]


class StateInfo(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("max_len", ctypes.c_int32), ("n_enc", ctypes.c_int32),
                ("n_dec", ctypes.c_int32), ("ring_valid", ctypes.c_int32), ("ring_head", ctypes.c_int32),
                ("has_encoder_cache", ctypes.c_int32), ("model_version", ctypes.c_uint64),
                ("has_pending", ctypes.c_int32), ("uniform", ctypes.c_int32)]


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_sig = {
    "rlt_init_weights": [ctypes.POINTER(Config), ctypes.c_uint64, ctypes.POINTER(_vp)],
    "rlt_load_weights": [_vp, ctypes.c_char_p, _vp, ctypes.c_size_t],
    "rlt_get_weights": [_vp, ctypes.c_char_p, _vp, ctypes.c_size_t],
    "rlt_tensor_info": [_vp, ctypes.c_char_p, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                        ctypes.POINTER(_i32)],
    "rlt_model_free": [_vp],
    "rlt_state_create": [_vp, _i32, _i32, _i32, ctypes.POINTER(_vp)],
    "rlt_state_free": [_vp],
    "rlt_state_reset": [_vp, _vp],
    "rlt_state_info_get": [_vp, ctypes.POINTER(StateInfo)],
    "rlt_state_read": [_vp, _i32, _i32, _vp, ctypes.c_size_t],
    "rlt_state_export": [_vp, _vp, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t), _vp],
    "rlt_state_import": [_vp, _vp, ctypes.c_size_t, _vp],
    "rlt_encode_prefix": [_vp, _vp, _vp, _i32, _vp],
    "rlt_readout": [_vp, _vp, _vp, ctypes.POINTER(Sampling), ctypes.POINTER(ReadoutOut), _vp],
    "rlt_decoder_step": [_vp, _vp, _vp, _vp, ctypes.POINTER(Sampling), ctypes.POINTER(ReadoutOut), _vp],
    "rlt_prefill": [_vp, _vp, _vp, _i32, _vp, _vp],
    "rlt_replay_logprobs": [_vp, _vp, _i32, _i32, _vp, _vp],
    "rlt_replay_ratios": [_vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp],
    "rlt_replay_backward": [_vp, _vp, _i32, _i32, _vp, _i32, _vp, _vp],
    "rlt_grad_read": [_vp, ctypes.c_char_p, _vp, ctypes.c_size_t],
    "rlt_grad_zero": [_vp, _vp],
    "rlt_backward_release": [_vp],
    "rlt_op_linear": [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp],
    "rlt_op_prefix_attention": [_vp, _vp, _vp, ctypes.c_int64, _i32, _i32, _i32, _i32, _i32, _vp, _i32, _vp, _vp],
    "rlt_op_prefix_attention_noalloc": [_vp, _vp, _vp, ctypes.c_int64, _i32, _i32, _i32, _i32, _i32, _vp, _i32, _vp,
                                        _vp],
    "rlt_op_sample": [_vp, _i32, _i32, ctypes.POINTER(Sampling), ctypes.c_uint32, _vp, _vp, _vp, _vp],
    "rlt_last_error": [ctypes.c_char_p, ctypes.c_size_t],
    "rlt_check_device": [],
    "rlt_kernel_launches": [ctypes.POINTER(ctypes.c_int64)],
    "rlt_test_bounded_wait": [ctypes.c_uint32, ctypes.POINTER(ctypes.c_uint64), _vp],
    "rlt_state_positions": [_vp, _vp, _vp, _vp, _vp],
    "rlt_append_spans": [_vp, _vp, _vp, ctypes.c_int64, _vp, _vp, ctypes.c_int64, _vp],
    "rlt_profile_enable": [_vp, _i32],
    "rlt_profile_read": [_vp, _i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64),
                         ctypes.POINTER(ctypes.c_double)],
}
for _name, _args in _sig.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = ctypes.c_int32


def rlt_last_error() -> tuple[int, str]:
    buf = ctypes.create_string_buffer(1024)
    code = _lib.rlt_last_error(buf, 1024)
    return code, buf.value.decode(errors="replace")


def _check(code: int) -> None:
    if code != RLT_OK:
        _, msg = rlt_last_error()
        raise RltError(code, msg)


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, dtype_name: str | None = None, numel: int | None = None):
    """Device pointer of a contiguous CUDA tensor (or None).  The library
    reads or writes `numel` elements through it: a smaller tensor is refused
    here, since the C ABI receives a bare pointer and cannot check."""
    if t is None:
        return None
    if numel is not None and t.numel() < numel:
        raise ValueError(f"tensor of {t.numel()} elements where {numel} are needed")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("expected a contiguous CUDA tensor")
    if dtype_name is not None and str(t.dtype) != dtype_name:
        raise ValueError(f"expected {dtype_name}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def make_config(**kw) -> Config:
    return Config(d_model=kw["d"], n_heads=kw["n_heads"], n_layers=kw["n_layers"], window=kw["window"],
                  groups=kw["groups"], ffn=kw["ffn"], vocab=kw["vocab"], tied=kw.get("tied", 1),
                  merge_kind=kw.get("merge_kind", 0), dtype=kw["dtype"], alpha=kw.get("alpha", 1.0),
                  rms_eps=kw.get("rms_eps", 1e-6), rope_base=kw.get("rope_base", 10000.0),
                  init_std=kw.get("init_std", 0.02), bos_id=kw.get("bos_id", 0))


class Model:
    """Owner of an ``rlt_model*``."""

    def __init__(self, handle: ctypes.c_void_p, cfg: dict):
        self.h = handle
        self.cfg = dict(cfg)
        self._lib = _lib  # kept for __del__, which may run after module teardown

    def __del__(self):
        self.free()

    def free(self) -> int:
        """Frees the model; returns RLT_E_STATE (and keeps the model) while
        states made on it are alive."""
        if getattr(self, "h", None):
            code = self._lib.rlt_model_free(self.h)
            if code != RLT_OK:
                return code
            self.h = None
        return RLT_OK

    @property
    def storage_dtype(self):
        return np.float32 if self.cfg["dtype"] == DTYPE_F32 else np.uint16

    def tensor_info(self, name: str):
        r, c, s = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
        _check(_lib.rlt_tensor_info(self.h, name.encode(), ctypes.byref(r), ctypes.byref(c), ctypes.byref(s)))
        return r.value, c.value, s.value

    def load_weights(self, name: str, raw: np.ndarray) -> None:
        raw = np.ascontiguousarray(raw, dtype=self.storage_dtype)
        _check(_lib.rlt_load_weights(self.h, name.encode(), raw.ctypes.data, raw.nbytes))

    def get_weights(self, name: str) -> np.ndarray:
        r, c, _ = self.tensor_info(name)
        out = np.zeros((r, c), dtype=self.storage_dtype)
        _check(_lib.rlt_get_weights(self.h, name.encode(), out.ctypes.data, out.nbytes))
        return out

    def grad(self, name: str) -> np.ndarray:
        """Accumulated fp32 gradient of a stored tensor (rlt_replay_backward)."""
        r, c, _ = self.tensor_info(name)
        out = np.zeros((r, c), dtype=np.float32)
        _check(_lib.rlt_grad_read(self.h, name.encode(), out.ctypes.data, out.nbytes))
        return out


class State:
    """Owner of an ``rlt_state*``."""

    def __init__(self, handle: ctypes.c_void_p, model: Model, batch: int, max_len: int):
        self.h = handle
        self.model = model
        self.batch = batch
        self.max_len = max_len
        self._lib = _lib  # kept for __del__, which may run after module teardown

    def __del__(self):
        self.free()

    def free(self):
        if getattr(self, "h", None):
            self._lib.rlt_state_free(self.h)
            self.h = None

    def info(self) -> dict:
        i = StateInfo()
        _check(_lib.rlt_state_info_get(self.h, ctypes.byref(i)))
        return {f: getattr(i, f) for f, _ in StateInfo._fields_}

    def positions(self) -> dict:
        """Per-sequence n_enc, n_dec, ring_valid and ring_head (int32 [B])."""
        out = {k: np.zeros(self.batch, np.int32) for k in ("n_enc", "n_dec", "ring_valid", "ring_head")}
        _check(_lib.rlt_state_positions(self.h, *(out[k].ctypes.data for k in ("n_enc", "n_dec", "ring_valid",
                                                                                 "ring_head"))))
        return out

    def read(self, what: int, index: int = 0) -> np.ndarray:
        c = self.model.cfg
        d, B, L = c["d"], self.batch, self.max_len
        H = c["n_heads"]
        hd = d // H
        sd = self.model.storage_dtype
        if what == READ_S:
            out = np.zeros((B, d), np.float32)
        elif what == READ_E:
            out = np.zeros((B, L, d), np.float32)
        elif what in (READ_RING_K, READ_RING_V):
            out = np.zeros((B, H, c["window"] - 1, hd), sd)
        else:
            out = np.zeros((B, H, L, hd), sd)
        _check(_lib.rlt_state_read(self.h, what, index, out.ctypes.data, out.nbytes))
        return out


# ------------------------------------------------------------------ entry points
def rlt_init_weights(cfg: dict, seed: int) -> Model:
    c = make_config(**cfg)
    h = ctypes.c_void_p()
    _check(_lib.rlt_init_weights(ctypes.byref(c), seed, ctypes.byref(h)))
    return Model(h, cfg)


def rlt_state_create(model: Model, batch: int, max_len: int, flags: int = 0) -> State:
    h = ctypes.c_void_p()
    _check(_lib.rlt_state_create(model.h, batch, max_len, flags, ctypes.byref(h)))
    return State(h, model, batch, max_len)


def rlt_state_reset(state: State, stream=None) -> None:
    _check(_lib.rlt_state_reset(state.h, _stream(stream)))


def rlt_state_export(state: State, stream=None) -> np.ndarray:
    """Exact prefix snapshot of the state as a uint8 array (host memory)."""
    n = ctypes.c_size_t()
    _check(_lib.rlt_state_export(state.h, None, 0, ctypes.byref(n), _stream(stream)))
    buf = np.zeros(n.value, np.uint8)
    _check(_lib.rlt_state_export(state.h, buf.ctypes.data, buf.nbytes, ctypes.byref(n), _stream(stream)))
    return buf


def rlt_state_import(state: State, snapshot: np.ndarray, stream=None) -> None:
    snap = np.ascontiguousarray(snapshot, dtype=np.uint8)
    _check(_lib.rlt_state_import(state.h, snap.ctypes.data, snap.nbytes, _stream(stream)))


def _rows(tokens, batch: int) -> int:
    """T of a [batch, T] token tensor."""
    if tokens.dim() != 2 or tokens.shape[0] != batch:
        raise ValueError(f"expected tokens of shape [{batch}, T], got {tuple(tokens.shape)}")
    return tokens.shape[1]


def rlt_encode_prefix(model: Model, state: State, tokens, stream=None) -> None:
    """tokens: int32 CUDA tensor [B, T], placed at positions n_enc+1..n_enc+T."""
    T = _rows(tokens, state.batch)
    _check(_lib.rlt_encode_prefix(model.h, state.h, _dev(tokens, "torch.int32"), T, _stream(stream)))


def _readout_out(B: int, V: int, logp=None, sampled=None, logp_sampled=None, logmu=None, logits=None):
    return ReadoutOut(logp=_dev(logp, "torch.float32", B), sampled=_dev(sampled, "torch.int32", B),
                      logp_sampled=_dev(logp_sampled, "torch.float32", B), logmu=_dev(logmu, "torch.float32", B),
                      logits=_dev(logits, "torch.float32", B * V))


def _sampling(sampling):
    if sampling is None:
        return None
    return ctypes.byref(Sampling(temperature=sampling["temperature"], top_k=sampling["top_k"], seed=sampling["seed"]))


def rlt_append_spans(model: Model, state: State, tokens, lens, logp=None, stream=None) -> None:
    """Appends span b = tokens[b, :lens[b]] to every sequence b: tokens int32
    CUDA tensor [B, L] (L >= max(lens)), lens host ints; logp (optional)
    float32 CUDA tensor [B, L-1] receives log p(span_b[i+1] | history) for
    i < lens[b]-1."""
    B = state.batch
    if tokens.dim() != 2 or tokens.shape[0] != B:
        raise ValueError(f"expected tokens of shape [{B}, L]")
    ln = np.ascontiguousarray(np.asarray(lens, dtype=np.int32))
    if ln.shape != (B,):
        raise ValueError(f"expected {B} span lengths")
    ld = tokens.shape[1]
    if logp is not None and (logp.dim() != 2 or logp.shape[0] != B):
        raise ValueError(f"expected logp of shape [{B}, L-1]")
    ld_lp = logp.shape[1] if logp is not None else 0
    _check(_lib.rlt_append_spans(model.h, state.h, _dev(tokens, "torch.int32"), ld, ln.ctypes.data,
                                 _dev(logp, "torch.float32", B * ld_lp) if logp is not None else None, ld_lp,
                                 _stream(stream)))


def rlt_readout(model: Model, state: State, next_tokens=None, sampling: dict | None = None, stream=None,
                **outs) -> None:
    o = _readout_out(state.batch, model.cfg["vocab"], **outs)
    _check(_lib.rlt_readout(model.h, state.h, _dev(next_tokens, "torch.int32", state.batch), _sampling(sampling),
                            ctypes.byref(o), _stream(stream)))


def rlt_decoder_step(model: Model, state: State, tokens=None, next_tokens=None, sampling: dict | None = None,
                     stream=None, **outs) -> None:
    o = _readout_out(state.batch, model.cfg["vocab"], **outs)
    _check(_lib.rlt_decoder_step(model.h, state.h, _dev(tokens, "torch.int32", state.batch),
                                 _dev(next_tokens, "torch.int32", state.batch), _sampling(sampling), ctypes.byref(o),
                                 _stream(stream)))


def rlt_prefill(model: Model, state: State, tokens, logp=None, stream=None) -> None:
    """tokens int32 [B, T]; logp (optional) float32 [B, T-1] (CUDA tensors)."""
    T = _rows(tokens, state.batch)
    _check(_lib.rlt_prefill(model.h, state.h, _dev(tokens, "torch.int32"), T,
                            _dev(logp, "torch.float32", state.batch * (T - 1)), _stream(stream)))


def rlt_replay_logprobs(model: Model, tokens, logp, stream=None) -> None:
    """tokens int32 [B, S] and logp float32 [B, S-1], both CUDA tensors."""
    B, S = tokens.shape
    _check(_lib.rlt_replay_logprobs(model.h, _dev(tokens, "torch.int32"), B, S,
                                    _dev(logp, "torch.float32", B * (S - 1)), _stream(stream)))


def rlt_replay_ratios(model: Model, tokens, logmu, action_mask, logp, ratio=None, seq_logratio=None,
                      stream=None) -> None:
    """tokens int32 [B, S]; logmu float32 and action_mask uint8 [B, S-1]; outputs
    logp and ratio float32 [B, S-1], seq_logratio float32 [B] (CUDA tensors)."""
    B, S = tokens.shape
    n = B * (S - 1)
    _check(_lib.rlt_replay_ratios(model.h, _dev(tokens, "torch.int32"), B, S, _dev(logmu, "torch.float32", n),
                                  _dev(action_mask, "torch.uint8", n), _dev(logp, "torch.float32", n),
                                  _dev(ratio, "torch.float32", n), _dev(seq_logratio, "torch.float32", B),
                                  _stream(stream)))


def rlt_replay_backward(model: Model, tokens, weights, segment: int = 32, logp=None, stream=None) -> None:
    """Full-BPTT gradient of -sum w[b][t] log p(x_{t+1} | x_1..t): tokens int32
    [B, S], weights float32 [B, S-1], optional logp float32 [B, S-1] (CUDA
    tensors).  Gradients accumulate in the model (Model.grad, rlt_grad_zero).
    The model keeps the pass's buffers (and, from the second call of a size,
    a CUDA graph of the pass) until rlt_backward_release or another size."""
    B, S = tokens.shape
    _check(_lib.rlt_replay_backward(model.h, _dev(tokens, "torch.int32"), B, S,
                                    _dev(weights, "torch.float32", B * (S - 1)), segment,
                                    _dev(logp, "torch.float32", B * (S - 1)), _stream(stream)))


def rlt_grad_zero(model: Model, stream=None) -> None:
    _check(_lib.rlt_grad_zero(model.h, _stream(stream)))


def rlt_backward_release(model: Model) -> None:
    """Frees what rlt_replay_backward keeps between calls."""
    _check(_lib.rlt_backward_release(model.h))


def rlt_op_linear(w, x, y, use_tensor_cores: bool = True, stream=None) -> None:
    """y [N, M] fp32 = x [N, K] @ w [M, K]^T (CUDA tensors, bf16 or fp32)."""
    M, K = w.shape
    N = x.shape[0]
    if x.dim() != 2 or x.shape[1] != K or x.dtype != w.dtype:
        raise ValueError("x must be [N, K] in the dtype of w")
    dt = DTYPE_BF16 if str(w.dtype) == "torch.bfloat16" else DTYPE_F32
    _check(_lib.rlt_op_linear(_dev(w), _dev(x), _dev(y, "torch.float32", N * M), M, N, K, dt, int(use_tensor_cores),
                              _stream(stream)))


def _prefix_attention_args(q, k, v, n, out, rope_cs, qpos, stream):
    B, H, ld_t, hd = k.shape
    if tuple(v.shape) != tuple(k.shape) or v.dtype != k.dtype or out.dtype != k.dtype:
        raise ValueError("v and out must match k's shape and dtype")
    dt = DTYPE_BF16 if str(k.dtype) == "torch.bfloat16" else DTYPE_F32
    return (_dev(q, "torch.float32", B * H * hd), _dev(k), _dev(v), ld_t, B, H, hd, n, dt,
            _dev(rope_cs, "torch.float32", (qpos + 1) * hd), qpos, _dev(out, None, B * H * hd), _stream(stream))


def rlt_op_prefix_attention(q, k, v, n: int, out, rope_cs=None, qpos: int = 0, stream=None) -> None:
    """out [B, H*hd] = attention of q [B, H*hd] (fp32) over rows 0..n-1 of
    k, v [B, H, ld_t, hd] (bf16 or fp32); rope_cs [pos, hd/2, 2] rotates q at qpos."""
    _check(_lib.rlt_op_prefix_attention(*_prefix_attention_args(q, k, v, n, out, rope_cs, qpos, stream)))


def rlt_op_prefix_attention_noalloc(q, k, v, n: int, out, rope_cs=None, qpos: int = 0, stream=None) -> None:
    """Same as rlt_op_prefix_attention, but its scratch is the library's static
    16 MiB device array instead of a per-call allocation (for callers that
    cannot allocate device memory); calls that overlap on the GPU race on it."""
    _check(_lib.rlt_op_prefix_attention_noalloc(*_prefix_attention_args(q, k, v, n, out, rope_cs, qpos, stream)))


def rlt_op_sample(logits, sampling: dict, t: int, token, logp=None, logmu=None, stream=None) -> None:
    """Sample from fp32 logits [B, V] (CUDA) as position t."""
    B, V = logits.shape
    _check(_lib.rlt_op_sample(_dev(logits, "torch.float32"), B, V, _sampling(sampling), t,
                              _dev(token, "torch.int32", B), _dev(logp, "torch.float32", B),
                              _dev(logmu, "torch.float32", B), _stream(stream)))


def rlt_check_device() -> None:
    _check(_lib.rlt_check_device())


def rlt_test_bounded_wait(limit_us: int, stream=None) -> int:
    """Runs the failure-detection probe (a bounded wait that cannot complete)
    and returns how long it waited, in ns; the device error word is left set
    for rlt_check_device to report."""
    n = ctypes.c_uint64()
    _check(_lib.rlt_test_bounded_wait(limit_us, ctypes.byref(n), _stream(stream)))
    return n.value


def rlt_kernel_launches() -> int:
    n = ctypes.c_int64()
    _check(_lib.rlt_kernel_launches(ctypes.byref(n)))
    return n.value


def rlt_profile_enable(model: Model, on: bool) -> None:
    _check(_lib.rlt_profile_enable(model.h, int(on)))


def rlt_profile_read(model: Model, kind: int) -> tuple[float, int, float]:
    ms, n, by = ctypes.c_double(), ctypes.c_int64(), ctypes.c_double()
    _check(_lib.rlt_profile_read(model.h, kind, ctypes.byref(ms), ctypes.byref(n), ctypes.byref(by)))
    return ms.value, n.value, by.value
