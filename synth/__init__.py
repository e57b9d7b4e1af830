"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds workload sizes and random inputs only: no step of the
model's arithmetic lives here.  Both the CUDA library (through its Python
binding) and the fp64 oracle consume what it produces; neither side imports
the other.

Workloads (sizes follow the five configurations the hot path is measured on):

* ``tiny``      fp32, d=64, 4 heads, L=2, W=4, G=1, V=256, B=2, T=32, uniform ids
* ``small``     bf16, d=512, 8x64, L=8, W=64, G=1, F=1536, V=32000, B=16,
                prompt 512 + 512 sampled tokens, Zipf(1.1) ids
* ``layerwise`` bf16, d=1024, 16 heads, L=24, W=128, G=L, F=2816, V=32000, B=64,
                T=2048 teacher-forced, Zipf(1.1) ids
* ``refdepth``  bf16, d=2048, 16x128, L=48, W=256, G=1, F=5632, V=32000, B=128,
                prompt 2048 + 2048 sampled tokens (temperature 0.8, top-k 50)
* ``replay``    bf16, the ``refdepth`` model at L=24, B=256, S=1024, with a
                prompt/response split uniform in [64, 960] per sequence

Token ids: x_1 = BOS = 0 ("Recurrent Looped Transformer", §2.1: every sequence
starts with BOS); the rest are uniform over the vocabulary (tiny) or follow a
Zipf(1.1) law truncated to the vocabulary, P(id = r-1) proportional to
r^-1.1, standing in for natural-language token frequencies.  No public
dataset is involved.
"""
from __future__ import annotations

import numpy as np

BOS = 0

_COMMON = dict(tied=1, merge_kind=0, alpha=1.0, rms_eps=1e-6, rope_base=10000.0, init_std=0.02, bos_id=BOS)

WORKLOADS = {
    "tiny": dict(_COMMON, d=64, n_heads=4, n_layers=2, window=4, groups=1, ffn=192, vocab=256, dtype=0,
                 batch=2, prompt=32, gen=0, dist="uniform", data_seed=1000),
    "small": dict(_COMMON, d=512, n_heads=8, n_layers=8, window=64, groups=1, ffn=1536, vocab=32000, dtype=1,
                  batch=16, prompt=512, gen=512, dist="zipf", data_seed=1001),
    "layerwise": dict(_COMMON, d=1024, n_heads=16, n_layers=24, window=128, groups=24, ffn=2816, vocab=32000,
                      dtype=1, batch=64, prompt=2048, gen=0, dist="zipf", data_seed=1002),
    "refdepth": dict(_COMMON, d=2048, n_heads=16, n_layers=48, window=256, groups=1, ffn=5632, vocab=32000,
                     dtype=1, batch=128, prompt=2048, gen=2048, dist="zipf", data_seed=1003),
    "replay": dict(_COMMON, d=2048, n_heads=16, n_layers=24, window=256, groups=1, ffn=5632, vocab=32000,
                   dtype=1, batch=256, prompt=1024, gen=0, dist="zipf", data_seed=1004,
                   split_lo=64, split_hi=960),
}

WEIGHT_SEED = 42
SAMPLER_SEED = 7
TEMPERATURE = 0.8
TOP_K = 50

MODEL_KEYS = ("d", "n_heads", "n_layers", "window", "groups", "ffn", "vocab", "tied", "merge_kind", "dtype",
              "alpha", "rms_eps", "rope_base", "init_std", "bos_id")


def workload(name: str, **overrides) -> dict:
    w = dict(WORKLOADS[name])
    w.update(overrides)
    return w


def model_config(w: dict) -> dict:
    """The model hyper-parameters of a workload (no batch/length keys)."""
    return {k: w[k] for k in MODEL_KEYS}


def _zipf_cdf(vocab: int, a: float = 1.1) -> np.ndarray:
    r = np.arange(1, vocab + 1, dtype=np.float64)
    p = r ** (-a)
    c = np.cumsum(p)
    return c / c[-1]


def tokens(w: dict, batch: int | None = None, length: int | None = None, seed: int | None = None) -> np.ndarray:
    """int32 [batch, length] token ids with column 0 = BOS."""
    B = w["batch"] if batch is None else batch
    T = (w["prompt"] if length is None else length)
    rng = np.random.Generator(np.random.PCG64(w["data_seed"] if seed is None else seed))
    V = w["vocab"]
    if w["dist"] == "uniform":
        x = rng.integers(0, V, size=(B, T), dtype=np.int64)
    else:
        u = rng.random(size=(B, T))
        x = np.searchsorted(_zipf_cdf(V), u, side="right")
        x = np.minimum(x, V - 1)
    x[:, 0] = BOS
    return np.ascontiguousarray(x.astype(np.int32))


def splits(w: dict, batch: int | None = None, seed: int | None = None) -> np.ndarray:
    """Prompt/response split T_b ~ U[split_lo, split_hi] per sequence."""
    B = w["batch"] if batch is None else batch
    rng = np.random.Generator(np.random.PCG64((w["data_seed"] if seed is None else seed) + 500))
    return rng.integers(w.get("split_lo", 1), w.get("split_hi", 1) + 1, size=B).astype(np.int32)


def logits(batch: int, vocab: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """fp32 [batch, vocab] random logits for sampler tests (normal, with a few
    exact ties planted so the (value desc, id asc) order is exercised)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = (rng.standard_normal((batch, vocab)) * scale).astype(np.float32)
    for b in range(batch):
        j = rng.integers(0, vocab, size=4)
        x[b, j] = x[b].max()
    return np.ascontiguousarray(x)


def random_state(shape, seed: int, scale: float = 1.0, dtype=np.float32) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.ascontiguousarray((rng.standard_normal(shape) * scale).astype(dtype))


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 bit patterns (storage format used
    when a test loads explicit weights into a bf16 model)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
