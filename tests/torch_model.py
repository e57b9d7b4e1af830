"""An independent fp64 formulation of the RLT forward pass, written with
PyTorch library routines (``F.rms_norm``, ``F.scaled_dot_product_attention``,
``F.silu``, ``F.log_softmax``) and complex-number rotations.  It exists only to
pin the oracle: it shares no code with it and uses different data structures
(the decoder keeps its whole key/value history and slices the window out of it
by position; rotary maps are complex multiplications).

Definitions follow "Recurrent Looped Transformer" §2.1-§2.6 (eqs. 2.1-2.16)
with the readings stated in the oracle's header.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

import synth


def _weights(model, cfg):
    d, Fd, V, L, G = cfg["d"], cfg["ffn"], cfg["vocab"], cfg["n_layers"], cfg["groups"]

    def g(name, shape):
        raw = model.get(name, shape)
        if cfg["dtype"] == 1:
            raw = synth.bf16_to_f32(raw).reshape(shape)
        return torch.from_numpy(np.asarray(raw, dtype=np.float64).copy())

    W = {"emb": g("emb", (V, d)), "s_star": g("s_star", (1, d))[0], "g_mem": g("g_mem", (1, d))[0],
         "g_merge": g("g_merge", (1, d))[0], "w_gate": g("w_gate", (d, 2 * d)), "b_gate": g("b_gate", (1, d))[0],
         "w_state": g("w_state", (d, d)), "g_out": g("g_out", (1, d))[0], "w_out": g("w_out", (V, d))}
    W["mem"] = [(g(f"wk_mem.{j}", (d, d)), g(f"wv_mem.{j}", (d, d))) for j in range(G)]
    W["layers"] = []
    for l in range(L):
        lay = {k: g(f"{k}.{l}", (d, d)) for k in ("wq", "wk", "wv", "wo", "wq_mem", "wo_mem")}
        lay["w1"] = g(f"w1.{l}", (Fd, d))
        lay["w3"] = g(f"w3.{l}", (Fd, d))
        lay["w2"] = g(f"w2.{l}", (d, Fd))
        for k in ("g_ea", "g_ef", "g_dsa", "g_dmem", "g_dffn"):
            lay[k] = g(f"{k}.{l}", (1, d))[0]
        if cfg.get("tied", 1):
            for k in ("wq", "wk", "wv", "wo", "w1", "w2", "w3"):
                lay["d" + k] = lay[k]
        else:
            for k in ("wq", "wk", "wv", "wo"):
                lay["d" + k] = g(f"d{k}.{l}", (d, d))
            lay["dw1"] = g(f"dw1.{l}", (Fd, d))
            lay["dw3"] = g(f"dw3.{l}", (Fd, d))
            lay["dw2"] = g(f"dw2.{l}", (d, Fd))
        W["layers"].append(lay)
    return W


def _rot(x, pos, H, base):
    """x [..., T, d] rotated per head at integer positions pos [T] with the
    complex form z_i * exp(i * pos * base^(-2i/hd)), z_i = x_i + i x_{i+hd/2}."""
    T, d = x.shape[-2], x.shape[-1]
    hd = d // H
    h = hd // 2
    xh = x.reshape(*x.shape[:-1], H, hd)
    z = torch.complex(xh[..., :h], xh[..., h:])
    freq = base ** (-torch.arange(0, h, dtype=torch.float64) * 2.0 / hd)
    ang = torch.as_tensor(pos, dtype=torch.float64)[:, None] * freq[None, :]
    z = z * torch.polar(torch.ones_like(ang), ang)[:, None, :]
    return torch.cat([z.real, z.imag], dim=-1).reshape(x.shape)


def _heads(x, H):
    T, d = x.shape
    return x.reshape(T, H, d // H).transpose(0, 1)  # [H, T, hd]


def forward_logprobs(model, cfg, tokens) -> np.ndarray:
    """log p(x_{t+1} | x_{1:t}) for t = 1..S-1 of one sequence."""
    W = _weights(model, cfg)
    d, H, L, Wn = cfg["d"], cfg["n_heads"], cfg["n_layers"], cfg["window"]
    eps, base, alpha = cfg["rms_eps"], cfg["rope_base"], cfg["alpha"]
    tok = torch.as_tensor(np.asarray(tokens, dtype=np.int64))
    S = tok.numel()
    pos = torch.arange(S, dtype=torch.float64)  # p = t-1

    def rms(x, gm):
        return F.rms_norm(x, (d,), weight=gm, eps=eps)

    # encoder: token-parallel causal stack
    h = W["emb"][tok].clone()
    for lay in W["layers"]:
        x = rms(h, lay["g_ea"])
        q = _rot(x @ lay["wq"].T, pos, H, base)
        k = _rot(x @ lay["wk"].T, pos, H, base)
        v = x @ lay["wv"].T
        o = F.scaled_dot_product_attention(_heads(q, H), _heads(k, H), _heads(v, H), is_causal=True)
        h = h + o.transpose(0, 1).reshape(S, d) @ lay["wo"].T
        y = rms(h, lay["g_ef"])
        h = h + (F.silu(y @ lay["w1"].T) * (y @ lay["w3"].T)) @ lay["w2"].T
    e = h
    n = rms(e, W["g_mem"])
    mem = [(_rot(n @ wk.T, pos, H, base), n @ wv.T) for (wk, wv) in W["mem"]]

    # decoder recurrence: the history of every layer's current k/v is kept
    # and the window is sliced out of it by position
    hist_k = [[] for _ in range(L)]
    hist_v = [[] for _ in range(L)]
    s = W["s_star"].clone()
    out = []
    for t in range(S - 1):  # 0-based position of token t+1
        et = e[t]
        if cfg.get("merge_kind", 0) == 0:
            r = rms(s, W["g_merge"])
            gate = torch.sigmoid(W["w_gate"] @ torch.cat([et, r]) + W["b_gate"])
            z = et + alpha * gate * (W["w_state"] @ r)
        else:
            gate = torch.sigmoid(W["w_gate"] @ torch.cat([et, s]))
            z = gate * et + (1 - gate) * s
        p1 = torch.tensor([float(t)])
        for l, lay in enumerate(W["layers"]):
            x = rms(z, lay["g_dsa"])
            q = _rot((lay["dwq"] @ x)[None], p1, H, base)
            k = _rot((lay["dwk"] @ x)[None], p1, H, base)
            v = (lay["dwv"] @ x)[None]
            hist_k[l].append(k)
            hist_v[l].append(v)
            lo = max(0, t - Wn + 1)
            K = torch.cat(hist_k[l][lo:t + 1])
            Vv = torch.cat(hist_v[l][lo:t + 1])
            o = F.scaled_dot_product_attention(_heads(q, H), _heads(K, H), _heads(Vv, H))
            b = z + lay["dwo"] @ o.transpose(0, 1).reshape(d)
            qm = _rot((lay["wq_mem"] @ rms(b, lay["g_dmem"]))[None], p1, H, base)
            g = 0 if cfg["groups"] == 1 else l
            Km, Vm = mem[g][0][: t + 1], mem[g][1][: t + 1]
            om = F.scaled_dot_product_attention(_heads(qm, H), _heads(Km, H), _heads(Vm, H))
            a = b + lay["wo_mem"] @ om.transpose(0, 1).reshape(d)
            y = rms(a, lay["g_dffn"])
            z = a + lay["dw2"] @ (F.silu(lay["dw1"] @ y) * (lay["dw3"] @ y))
        s = z
        logp = F.log_softmax(W["w_out"] @ rms(s, W["g_out"]), dim=-1)
        out.append(logp[tok[t + 1]].item())
    return np.array(out)
