"""Full back-propagation through time for the Recurrent Looped Transformer,
in fp64 on the CPU.

TEST INFRASTRUCTURE ONLY.  The rules of the rest of ``oracle`` hold here too:
only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this module, and the product path never does.

What it computes ("Recurrent Looped Transformer", §5.1-§5.4 and App. C): the
gradient of a weighted replay log-likelihood

    L_w(Theta) = - sum_{t=1}^{S-1} w_t log p_Theta(x_{t+1} | x_{1:t})

with respect to every stored tensor of the model.  The gradient runs through
the whole computation: the causal encoder, the memory projections, the merge,
every decoder sliding-window key/value and the recurrent output s_t, over all
positions.  Nothing is detached.  That is full BPTT in the sense of §5.4, and
App. C adds that evicting an entry from the SWA window is not a stop-gradient:
the steps that read the entry before its eviction still carry its gradient.

The objectives of §5 are choices of the weights w (``target_weights``):

    eq. 5.1 pretraining      w_t = 1/(S-1) on every target
    eq. 5.2 SFT              w_t = m_{t+1} / sum m over the selected targets
    eq. 5.4 score function   w_t = R - b on the response targets, 0 on the
                             prompt; minimising L_w follows the per-sample
                             term of eq. 5.4 (the prompt's computation still
                             carries gradient, §5.2)

The forward pass is the recurrence of §2 (eqs. 2.1-2.16) written with
elementary PyTorch fp64 tensor operations; the backward pass is
``torch.autograd`` over that graph.  The readings are the ones the C oracle
states in its header: SwiGLU FFN, rotate-half RoPE at 0-based position t-1
(base from the configuration), one pre-norm RMSNorm per sublayer, no final
encoder norm, multi-head attention scaled by 1/sqrt(hd), no biases but b_g,
and the merge of eqs. 2.9-2.11 (kind 0) or the convex gate (kind 1, which has
no bias, so b_g gets a zero gradient there).

Pins (``tests/test_oracle_bptt.py``): the forward log-probabilities equal the
C oracle's replay; every gradient entry of small models equals a central
finite difference of the C oracle's L_w; the gradients of the readout matrix
and its norm gain equal their closed forms built from the C oracle's states.
"""
from __future__ import annotations

import math

import numpy as np
import torch

_LAYER_SLOTS = ("wq", "wk", "wv", "wo", "w1", "w2", "w3", "g_ea", "g_ef", "g_dsa", "g_dmem", "g_dffn",
                "wq_mem", "wo_mem")
_UNTIED_SLOTS = ("dwq", "dwk", "dwv", "dwo", "dw1", "dw2", "dw3")


def tensor_shapes(cfg: dict) -> dict[str, tuple[int, int]]:
    """Name -> (rows, cols) of every tensor the model stores, in the storage
    layout: a matrix [out, in] maps x to W x; a gain or bias is [1, d]."""
    d, F, V = cfg["d"], cfg["ffn"], cfg["vocab"]
    shp = {"emb": (V, d), "s_star": (1, d), "g_mem": (1, d), "g_merge": (1, d), "w_gate": (d, 2 * d),
           "b_gate": (1, d), "w_state": (d, d), "g_out": (1, d), "w_out": (V, d)}
    for g in range(cfg["groups"]):
        shp[f"wk_mem.{g}"] = (d, d)
        shp[f"wv_mem.{g}"] = (d, d)
    slots = _LAYER_SLOTS + (() if cfg.get("tied", 1) else _UNTIED_SLOTS)
    for l in range(cfg["n_layers"]):
        for s in slots:
            if s in ("w1", "w3", "dw1", "dw3"):
                shp[f"{s}.{l}"] = (F, d)
            elif s in ("w2", "dw2"):
                shp[f"{s}.{l}"] = (d, F)
            elif s.startswith("g_"):
                shp[f"{s}.{l}"] = (1, d)
            else:
                shp[f"{s}.{l}"] = (d, d)
    return shp


def parameters(model) -> dict[str, torch.Tensor]:
    """Every stored tensor of an oracle ``Model`` as an fp64 leaf that
    requires grad.  bf16 bit patterns are widened exactly."""
    out = {}
    for name, shape in tensor_shapes(model.cfg).items():
        raw = model.get(name, shape)
        if model.cfg["dtype"] == 1:
            raw = (raw.astype(np.uint32) << 16).view(np.float32)
        out[name] = torch.tensor(np.asarray(raw, dtype=np.float64), requires_grad=True)
    return out


def _rms(x, gain, eps):
    """RMSNorm over the last axis with gain (§2.5)."""
    return x / torch.sqrt((x * x).mean(-1, keepdim=True) + eps) * gain


def _rope(x, pos, n_heads, base):
    """Rotate-half RoPE of rows x [T, d] at 0-based positions pos [T]: within
    each head, the pair (x_i, x_{i+hd/2}) turns by pos * base^(-2i/hd)."""
    T, d = x.shape
    hd = d // n_heads
    h = hd // 2
    inv = base ** (-2.0 * torch.arange(h, dtype=torch.float64) / hd)
    ang = pos.to(torch.float64)[:, None] * inv[None, :]
    c, s = torch.cos(ang)[:, None, :], torch.sin(ang)[:, None, :]
    xh = x.reshape(T, n_heads, hd)
    x1, x2 = xh[..., :h], xh[..., h:]
    return torch.cat([x1 * c - x2 * s, x1 * s + x2 * c], dim=-1).reshape(T, d)


def _attend(q, K, V, n_heads, allowed=None):
    """Multi-head softmax attention of queries q [Tq, d] over K, V [Tk, d];
    allowed [Tq, Tk] (bool) restricts the keys each query may see."""
    Tq, d = q.shape
    Tk = K.shape[0]
    hd = d // n_heads
    qh = q.reshape(Tq, n_heads, hd).transpose(0, 1)
    kh = K.reshape(Tk, n_heads, hd).transpose(0, 1)
    vh = V.reshape(Tk, n_heads, hd).transpose(0, 1)
    sc = qh @ kh.transpose(1, 2) / math.sqrt(hd)
    if allowed is not None:
        sc = sc.masked_fill(~allowed[None], float("-inf"))
    a = torch.softmax(sc, dim=-1)
    return (a @ vh).transpose(0, 1).reshape(Tq, d)


def _swiglu(y, w1, w3, w2):
    u = y @ w1.T
    return (u * torch.sigmoid(u) * (y @ w3.T)) @ w2.T


def logprobs(P: dict[str, torch.Tensor], cfg: dict, tokens, detach: tuple[str, ...] = ()) -> torch.Tensor:
    """log p(x_{t+1} | x_{1:t}) for t = 1..S-1 of one sequence, as a
    differentiable fp64 tensor [S-1] (§5.3, replay from H_0 = (s_star, empty)).

    ``detach`` names the decoder-state tensors cut at every step boundary, the
    truncation of eq. C.1: "s" stops the gradient of s_t where step t+1 reads
    it, "swa" stops it on the window keys/values of earlier positions.  The
    values, and so the log-probabilities, do not change.  The default, no
    detach, is full BPTT."""
    if not set(detach) <= {"s", "swa"}:
        raise ValueError(f"unknown detach {detach}")
    d, H, L, W = cfg["d"], cfg["n_heads"], cfg["n_layers"], cfg["window"]
    eps, base, alpha = cfg["rms_eps"], cfg["rope_base"], cfg["alpha"]
    tied = cfg.get("tied", 1)
    tok = torch.as_tensor(np.asarray(tokens, dtype=np.int64))
    S = tok.numel()
    pos = torch.arange(S)

    def dec(name, l):
        return P[f"{name}.{l}"] if tied else P[f"d{name}.{l}"]

    # eq. 2.1: token-parallel causal encoder over the whole sequence
    h = P["emb"][tok]
    causal = torch.ones(S, S, dtype=torch.bool).tril()
    for l in range(L):
        x = _rms(h, P[f"g_ea.{l}"][0], eps)
        q = _rope(x @ P[f"wq.{l}"].T, pos, H, base)
        k = _rope(x @ P[f"wk.{l}"].T, pos, H, base)
        v = x @ P[f"wv.{l}"].T
        h = h + _attend(q, k, v, H, causal) @ P[f"wo.{l}"].T
        h = h + _swiglu(_rms(h, P[f"g_ef.{l}"][0], eps), P[f"w1.{l}"], P[f"w3.{l}"], P[f"w2.{l}"])
    e = h
    # eq. 2.2: memory keys/values of every group from the normed features
    n = _rms(e, P["g_mem"][0], eps)
    mem = [(_rope(n @ P[f"wk_mem.{g}"].T, pos, H, base), n @ P[f"wv_mem.{g}"].T) for g in range(cfg["groups"])]

    s = P["s_star"][0]
    keys = [[] for _ in range(L)]
    vals = [[] for _ in range(L)]
    out = []
    for t in range(S - 1):  # consumes token t+1 (1-based), position t (0-based)
        et = e[t]
        if t > 0 and "s" in detach:
            s = s.detach()
        if cfg.get("merge_kind", 0) == 0:  # eqs. 2.9-2.11
            r = _rms(s, P["g_merge"][0], eps)
            gate = torch.sigmoid(P["w_gate"] @ torch.cat([et, r]) + P["b_gate"][0])
            z = et + alpha * gate * (P["w_state"] @ r)
        else:  # convex gate
            gate = torch.sigmoid(P["w_gate"] @ torch.cat([et, s]))
            z = gate * et + (1.0 - gate) * s
        pt = pos[t:t + 1]
        for l in range(L):
            # eqs. 2.12-2.13: SWA over the window of the last W positions
            x = _rms(z, P[f"g_dsa.{l}"][0], eps)[None]
            q = _rope(x @ dec("wq", l).T, pt, H, base)
            keys[l].append(_rope(x @ dec("wk", l).T, pt, H, base))
            vals[l].append(x @ dec("wv", l).T)
            lo = max(0, t - W + 1)
            if "swa" in detach:
                Kw = torch.cat([kk.detach() for kk in keys[l][lo:-1]] + keys[l][-1:])
                Vw = torch.cat([vv.detach() for vv in vals[l][lo:-1]] + vals[l][-1:])
            else:
                Kw, Vw = torch.cat(keys[l][lo:]), torch.cat(vals[l][lo:])
            o = _attend(q, Kw, Vw, H)
            b = z + (o @ dec("wo", l).T)[0]
            # eq. 2.14: cross-attention over the memory of tokens 1..t+1
            g = 0 if cfg["groups"] == 1 else l
            xm = _rms(b, P[f"g_dmem.{l}"][0], eps)[None]
            qm = _rope(xm @ P[f"wq_mem.{l}"].T, pt, H, base)
            om = _attend(qm, mem[g][0][:t + 1], mem[g][1][:t + 1], H)
            a = b + (om @ P[f"wo_mem.{l}"].T)[0]
            # eqs. 2.15-2.16: FFN
            z = a + _swiglu(_rms(a, P[f"g_dffn.{l}"][0], eps)[None], dec("w1", l), dec("w3", l), dec("w2", l))[0]
        s = z
        logits = P["w_out"] @ _rms(s, P["g_out"][0], eps)  # eq. 2.6
        out.append(logits[tok[t + 1]] - torch.logsumexp(logits, dim=0))
    return torch.stack(out) if out else torch.zeros(0, dtype=torch.float64)


def target_weights(kind: str, S: int, mask=None, reward: float = 0.0, baseline: float = 0.0,
                   prompt_len: int | None = None) -> np.ndarray:
    """The w_t of L_w for the objectives of §5, one per target t = 1..S-1.

    kind "pretrain": eq. 5.1.  kind "sft": eq. 5.2 with mask[t-1] = m_{t+1}.
    kind "score": eq. 5.4 for a response that starts at token prompt_len+1.
    """
    n = S - 1
    if kind == "pretrain":
        return np.full(n, 1.0 / n)
    if kind == "sft":
        m = np.asarray(mask, dtype=np.float64)
        if m.shape != (n,) or m.sum() == 0:
            raise ValueError("SFT needs S-1 mask entries with at least one selected target")
        return m / m.sum()
    if kind == "score":
        if prompt_len is None or not 1 <= prompt_len <= n:
            raise ValueError("score needs 1 <= prompt_len <= S-1")
        w = np.zeros(n)
        w[prompt_len - 1:] = reward - baseline
        return w
    raise ValueError(kind)


def loss_and_grads(model, tokens, weights, detach: tuple[str, ...] = ()) -> tuple[float, dict[str, np.ndarray]]:
    """L_w of one sequence and its gradient with respect to every stored
    tensor (name -> array in the storage shape), by full BPTT unless
    ``detach`` asks for the truncation of eq. C.1."""
    P = parameters(model)
    lp = logprobs(P, model.cfg, tokens, detach)
    w = torch.as_tensor(np.asarray(weights, dtype=np.float64))
    if w.shape != lp.shape:
        raise ValueError("need one weight per target")
    loss = -(w * lp).sum()
    grads = torch.autograd.grad(loss, list(P.values()), allow_unused=True)
    return float(loss.detach()), {k: (np.zeros(tuple(v.shape)) if g is None else g.numpy())
                         for (k, v), g in zip(P.items(), grads)}
