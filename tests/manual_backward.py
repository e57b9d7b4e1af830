"""Reverse-time BPTT of the Recurrent Looped Transformer, derived by hand and
written out in numpy fp64, with segment checkpointing.

Test-side only.  It is a second, independent derivation of the gradient that
``oracle.bptt`` obtains from autograd, and it fixes the schedule that a
backward kernel set follows:

* The forward pass keeps only checkpoints at segment starts: the recurrent
  output entering the segment, and the SWA keys/values of the W-1 positions
  before it.  The encoder activations, the memory and the per-token merge
  inputs e_t are kept whole; they are token-parallel.
* Segments run in reverse order.  Each one is recomputed from its checkpoint
  with the same parameters, as "Recurrent Looped Transformer" §4.3 and §5.4
  ask.  Its steps are then reversed one at a time:
  - the readout adjoint enters s_t;
  - each layer's FFN, memory cross-attention and SWA sublayers are reversed,
    then the merge;
  - the adjoint leaves through s_{t-1} (the sequential chain) and through
    e_t (to the encoder).
* SWA keys/values of position j get adjoints from the later steps
  j+1..j+W-1, whose reversal comes first.  So when step j is reversed, the
  adjoints of its own key and value are complete.  They are kept in a
  pending table across segment boundaries (App. C: eviction is not a
  stop-gradient).
* The memory cross-attention needs dq per step, on the chain.  The
  adjoints of the memory keys/values are deferred: each segment gathers its
  queries, output adjoints and log-sum-exps, then makes one token-parallel,
  causally masked pass over the memory.  This is the flash-attention
  backward form.
* The decoder's weight gradients are one matrix product per weight and
  segment, dW += dY^T X over the segment's steps.  They are not a rank-1
  update per step.
* The encoder backward runs token-parallel at the end.  It takes the memory
  adjoints and the per-token e_t adjoints of the merges.

Loss: L_w = -sum_t w_t log p(x_{t+1} | x_{1:t}) (eqs. 5.1, 5.2, 5.4 as
choices of w).
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------------------
# primitives with their adjoints (rows are vectors)
# ---------------------------------------------------------------------------

def rms_f(x, g, eps):
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)
    return x * r[..., None] * g, r


def rms_b(dy, x, r, g):
    """Adjoint of y = g * x / rms(x): returns (dx, dg)."""
    xh = x * r[..., None]
    dxh = dy * g
    dx = r[..., None] * (dxh - xh * np.mean(dxh * xh, axis=-1, keepdims=True))
    return dx, np.sum(dy * xh, axis=tuple(range(dy.ndim - 1)))


def rot(x, pos, H, base, sign=1.0):
    """Rotate-half RoPE of rows x [n, d] at positions pos [n]; sign=-1 applies
    the inverse (= transposed) rotation, which is the adjoint."""
    n, d = x.shape
    hd = d // H
    h = hd // 2
    inv = base ** (-2.0 * np.arange(h) / hd)
    ang = sign * np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    xh = x.reshape(n, H, hd)
    x1, x2 = xh[..., :h], xh[..., h:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1).reshape(n, d)


def _split(x, H):
    n, d = x.shape
    return x.reshape(n, H, d // H).transpose(1, 0, 2)  # [H, n, hd]


def _merge_heads(x):
    H, n, hd = x.shape
    return x.transpose(1, 0, 2).reshape(n, H * hd)


def attn_f(q, K, V, H, allowed=None):
    """Softmax attention; returns (o [n, d], P [H, n, m], lse [H, n])."""
    hd = q.shape[1] // H
    sc = _split(q, H) @ _split(K, H).transpose(0, 2, 1) / np.sqrt(hd)
    if allowed is not None:
        sc = np.where(allowed[None], sc, -np.inf)
    mx = sc.max(axis=-1, keepdims=True)
    ex = np.exp(sc - mx)
    den = ex.sum(axis=-1, keepdims=True)
    P = ex / den
    return _merge_heads(P @ _split(V, H)), P, (mx + np.log(den))[..., 0]


def attn_b(do, q, K, V, P, H):
    """Adjoint of o = softmax(q K^T / sqrt(hd)) V per head: (dq, dK, dV)."""
    hd = q.shape[1] // H
    dO = _split(do, H)
    dV = P.transpose(0, 2, 1) @ dO
    dP = dO @ _split(V, H).transpose(0, 2, 1)
    dS = P * (dP - np.sum(P * dP, axis=-1, keepdims=True))
    dq = dS @ _split(K, H) / np.sqrt(hd)
    dK = dS.transpose(0, 2, 1) @ _split(q, H) / np.sqrt(hd)
    return _merge_heads(dq), _merge_heads(dK), _merge_heads(dV)


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def swiglu_f(y, w1, w3, w2):
    u1, u3 = y @ w1.T, y @ w3.T
    hs = u1 * sigmoid(u1) * u3
    return hs @ w2.T, (u1, u3, hs)


def swiglu_b(df, y, c, w1, w3, w2):
    """Adjoint of W2(silu(W1 y) * W3 y): (dy, dW1, dW3, dW2)."""
    u1, u3, hs = c
    sg = sigmoid(u1)
    dhs = df @ w2
    du3 = dhs * u1 * sg
    du1 = dhs * u3 * sg * (1.0 + u1 * (1.0 - sg))
    return du1 @ w1 + du3 @ w3, du1.T @ y, du3.T @ y, df.T @ hs


# ---------------------------------------------------------------------------
# the schedule
# ---------------------------------------------------------------------------

class ManualBPTT:
    def __init__(self, P: dict[str, np.ndarray], cfg: dict):
        self.P, self.cfg = P, cfg
        self.d, self.H, self.L, self.W = cfg["d"], cfg["n_heads"], cfg["n_layers"], cfg["window"]
        self.eps, self.base, self.alpha = cfg["rms_eps"], cfg["rope_base"], cfg["alpha"]
        self.tied = cfg.get("tied", 1)

    def _dn(self, name, l):
        return f"{name}.{l}" if self.tied else f"d{name}.{l}"

    def _g(self, name, l=None):
        return self.P[name if l is None else f"{name}.{l}"][0]

    # -- encoder (token-parallel) ------------------------------------------
    def encoder_f(self, tok):
        P, H, eps, base = self.P, self.H, self.eps, self.base
        S = tok.size
        pos = np.arange(S)
        causal = np.tril(np.ones((S, S), dtype=bool))
        h = P["emb"][tok].copy()
        caches = []
        for l in range(self.L):
            x, r1 = rms_f(h, self._g("g_ea", l), eps)
            q = rot(x @ P[f"wq.{l}"].T, pos, H, base)
            k = rot(x @ P[f"wk.{l}"].T, pos, H, base)
            v = x @ P[f"wv.{l}"].T
            o, A, _ = attn_f(q, k, v, H, causal)
            h2 = h + o @ P[f"wo.{l}"].T
            y, r2 = rms_f(h2, self._g("g_ef", l), eps)
            f, cf = swiglu_f(y, P[f"w1.{l}"], P[f"w3.{l}"], P[f"w2.{l}"])
            caches.append((h, x, r1, q, k, v, o, A, h2, y, r2, cf))
            h = h2 + f
        e = h
        n, rn = rms_f(e, self._g("g_mem"), eps)
        mem = [(rot(n @ P[f"wk_mem.{g}"].T, pos, H, base), n @ P[f"wv_mem.{g}"].T) for g in range(self.cfg["groups"])]
        return e, (caches, n, rn), mem

    def encoder_b(self, tok, e, enc_cache, de, dmem, G):
        P, H, base = self.P, self.H, self.base
        caches, n, rn = enc_cache
        pos = np.arange(tok.size)
        dn = np.zeros_like(n)
        for g, (dK, dV) in enumerate(dmem):
            dk = rot(dK, pos, H, base, -1.0)
            G[f"wk_mem.{g}"] += dk.T @ n
            G[f"wv_mem.{g}"] += dV.T @ n
            dn += dk @ P[f"wk_mem.{g}"] + dV @ P[f"wv_mem.{g}"]
        dx, dg = rms_b(dn, e, rn, self._g("g_mem"))
        G["g_mem"][0] += dg
        dh = de + dx
        for l in reversed(range(self.L)):
            h, x, r1, q, k, v, o, A, h2, y, r2, cf = caches[l]
            dy, dw1, dw3, dw2 = swiglu_b(dh, y, cf, P[f"w1.{l}"], P[f"w3.{l}"], P[f"w2.{l}"])
            G[f"w1.{l}"] += dw1
            G[f"w3.{l}"] += dw3
            G[f"w2.{l}"] += dw2
            dx2, dg = rms_b(dy, h2, r2, self._g("g_ef", l))
            G[f"g_ef.{l}"][0] += dg
            dh2 = dh + dx2
            G[f"wo.{l}"] += dh2.T @ o
            dq, dk, dv = attn_b(dh2 @ P[f"wo.{l}"], q, k, v, A, H)
            dq = rot(dq, pos, H, base, -1.0)
            dk = rot(dk, pos, H, base, -1.0)
            G[f"wq.{l}"] += dq.T @ x
            G[f"wk.{l}"] += dk.T @ x
            G[f"wv.{l}"] += dv.T @ x
            dxa = dq @ P[f"wq.{l}"] + dk @ P[f"wk.{l}"] + dv @ P[f"wv.{l}"]
            dx1, dg = rms_b(dxa, h, r1, self._g("g_ea", l))
            G[f"g_ea.{l}"][0] += dg
            dh = dh2 + dx1
        np.add.at(G["emb"], tok, dh)

    # -- one decoder transition ---------------------------------------------
    def step_f(self, t, et, s, win, mem):
        """Transition at 0-based position t.  win[l] maps position -> (k, v)
        rows and receives this position's entry.  Returns (s_t, cache)."""
        P, H, eps, base, L = self.P, self.H, self.eps, self.base, self.L
        s = s[None]
        et = et[None]
        if self.cfg.get("merge_kind", 0) == 0:
            rm, rr = rms_f(s, self._g("g_merge"), eps)
            c = np.concatenate([et, rm], axis=1)
            gate = sigmoid(c @ P["w_gate"].T + self._g("b_gate"))
            ws = rm @ P["w_state"].T
            z = et + self.alpha * gate * ws
            mc = (s, rm, rr, c, gate, ws)
        else:
            c = np.concatenate([et, s], axis=1)
            gate = sigmoid(c @ P["w_gate"].T)
            z = gate * et + (1.0 - gate) * s
            mc = (s, c, gate, et)
        lay = []
        for l in range(L):
            x, r1 = rms_f(z, self._g("g_dsa", l), eps)
            q = rot(x @ P[self._dn("wq", l)].T, [t], H, base)
            k = rot(x @ P[self._dn("wk", l)].T, [t], H, base)
            v = x @ P[self._dn("wv", l)].T
            win[l][t] = (k, v)
            js = [j for j in range(max(0, t - self.W + 1), t + 1)]
            Kw = np.concatenate([win[l][j][0] for j in js])
            Vw = np.concatenate([win[l][j][1] for j in js])
            o, A, _ = attn_f(q, Kw, Vw, H)
            b = z + o @ P[self._dn("wo", l)].T
            xm, r2 = rms_f(b, self._g("g_dmem", l), eps)
            qm = rot(xm @ P[f"wq_mem.{l}"].T, [t], H, base)
            g = 0 if self.cfg["groups"] == 1 else l
            om, Am, lse = attn_f(qm, mem[g][0][:t + 1], mem[g][1][:t + 1], H)
            a = b + om @ P[f"wo_mem.{l}"].T
            y, r3 = rms_f(a, self._g("g_dffn", l), eps)
            f, cf = swiglu_f(y, P[self._dn("w1", l)], P[self._dn("w3", l)], P[self._dn("w2", l)])
            lay.append((z, x, r1, q, js, Kw, Vw, o, A, b, xm, r2, qm, om, Am, lse, a, y, r3, cf))
            z = a + f
        n, rn = rms_f(z, self._g("g_out"), eps)
        logits = n @ P["w_out"].T
        return z[0], (mc, lay, z, n, rn, logits[0])

    # -- full replay --------------------------------------------------------
    def loss_and_grads(self, tok, wts, seg: int):
        """L_w and its gradient (name -> array), with decoder segments of
        ``seg`` steps recomputed from checkpoints during the backward pass."""
        P, H, L, base = self.P, self.H, self.L, self.base
        tok = np.asarray(tok, dtype=np.int64)
        S = tok.size
        G = {k: np.zeros_like(v) for k, v in P.items()}
        e, enc_cache, mem = self.encoder_f(tok)

        # forward: log-probs, keeping only the segment checkpoints
        starts = list(range(0, S - 1, seg))
        ckpt = {}
        s = P["s_star"][0].copy()
        win = [dict() for _ in range(L)]
        logp = np.zeros(S - 1)
        for t in range(S - 1):
            if t in starts:
                keep = range(max(0, t - self.W + 1), t)
                ckpt[t] = (s.copy(), [{j: win[l][j] for j in keep} for l in range(L)])
            s, c = self.step_f(t, e[t], s, win, mem)
            lg = c[5]
            mx = lg.max()
            logp[t] = lg[tok[t + 1]] - (mx + np.log(np.exp(lg - mx).sum()))
            for l in range(L):  # the ring holds W-1 entries after the step
                win[l].pop(t - self.W + 1, None)
        loss = -float(np.dot(wts, logp))

        # backward: segments in reverse
        de = np.zeros_like(e)
        dmem = [(np.zeros_like(K), np.zeros_like(V)) for K, V in mem]
        pend = [dict() for _ in range(L)]  # position -> (dk, dv) still owed to that position's step
        ds = np.zeros(self.d)
        for t0 in reversed(starts):
            t1 = min(t0 + seg, S - 1)
            s_in, win0 = ckpt[t0]
            win = [dict(w) for w in win0]
            s_prev, caches = s_in, []
            for t in range(t0, t1):  # recompute the segment
                s_new, c = self.step_f(t, e[t], s_prev, win, mem)
                caches.append((s_prev, c))
                s_prev = s_new
            # per-weight (dY, X) rows of this segment, reduced once at its end
            rows = {}

            def acc(name, dy, x):
                rows.setdefault(name, ([], []))
                rows[name][0].append(dy)
                rows[name][1].append(x)

            deferred = [[] for _ in range(L)]  # (t, qm, dom, lse) of the memory attention
            for t in reversed(range(t0, t1)):
                s_prev_t, (mc, lay, z_out, n, rn, logits) = caches[t - t0]
                p = np.exp(logits - logits.max())
                p /= p.sum()
                dlog = -wts[t] * (np.eye(logits.size)[tok[t + 1]] - p)
                acc("w_out", dlog[None], n)
                dn = dlog[None] @ P["w_out"]
                dx, dg = rms_b(dn, z_out, rn, self._g("g_out"))
                G["g_out"][0] += dg
                dz = ds[None] + dx
                for l in reversed(range(L)):
                    (z, x, r1, q, js, Kw, Vw, o, A, b, xm, r2, qm, om, Am, lse, a, y, r3, cf) = lay[l]
                    dy, dw1, dw3, dw2 = swiglu_b(dz, y, cf, P[self._dn("w1", l)], P[self._dn("w3", l)],
                                                 P[self._dn("w2", l)])
                    G[self._dn("w1", l)] += dw1
                    G[self._dn("w3", l)] += dw3
                    G[self._dn("w2", l)] += dw2
                    dxa, dg = rms_b(dy, a, r3, self._g("g_dffn", l))
                    G[f"g_dffn.{l}"][0] += dg
                    da = dz + dxa
                    acc(f"wo_mem.{l}", da, om)
                    dom = da @ P[f"wo_mem.{l}"]
                    g = 0 if self.cfg["groups"] == 1 else l
                    Km, Vm = mem[g][0][:t + 1], mem[g][1][:t + 1]
                    dqm, _, _ = attn_b(dom, qm, Km, Vm, Am, H)  # dK/dV deferred below
                    deferred[l].append((t, qm[0], dom[0], lse[:, 0]))
                    dqm = rot(dqm, [t], H, base, -1.0)
                    acc(f"wq_mem.{l}", dqm, xm)
                    dxm, dg = rms_b(dqm @ P[f"wq_mem.{l}"], b, r2, self._g("g_dmem", l))
                    G[f"g_dmem.{l}"][0] += dg
                    db = da + dxm
                    acc(self._dn("wo", l), db, o)
                    dq, dKw, dVw = attn_b(db @ P[self._dn("wo", l)], q, Kw, Vw, A, H)
                    for i, j in enumerate(js[:-1]):  # owed to earlier positions
                        pk, pv = pend[l].get(j, (0.0, 0.0))
                        pend[l][j] = (pk + dKw[i:i + 1], pv + dVw[i:i + 1])
                    pk, pv = pend[l].pop(t, (0.0, 0.0))  # complete: later steps are done
                    dk = rot(dKw[-1:] + pk, [t], H, base, -1.0)
                    dv = dVw[-1:] + pv
                    dq = rot(dq, [t], H, base, -1.0)
                    acc(self._dn("wq", l), dq, x)
                    acc(self._dn("wk", l), dk, x)
                    acc(self._dn("wv", l), dv, x)
                    dxs = dq @ P[self._dn("wq", l)] + dk @ P[self._dn("wk", l)] + dv @ P[self._dn("wv", l)]
                    dx1, dg = rms_b(dxs, z, r1, self._g("g_dsa", l))
                    G[f"g_dsa.{l}"][0] += dg
                    dz = db + dx1
                # merge
                if self.cfg.get("merge_kind", 0) == 0:
                    sv, rm, rr, c, gate, ws = mc
                    de[t] += dz[0]
                    dws = dz * self.alpha * gate
                    dgp = dz * self.alpha * ws * gate * (1.0 - gate)
                    acc("w_state", dws, rm)
                    acc("w_gate", dgp, c)
                    G["b_gate"][0] += dgp[0]
                    dc = dgp @ P["w_gate"]
                    de[t] += dc[0, :self.d]
                    drm = dws @ P["w_state"] + dc[:, self.d:]
                    dsv, dg = rms_b(drm, sv, rr, self._g("g_merge"))
                    G["g_merge"][0] += dg
                    ds = dsv[0]
                else:
                    sv, c, gate, et = mc
                    de[t] += (dz * gate)[0]
                    dgp = dz * (et - sv) * gate * (1.0 - gate)
                    acc("w_gate", dgp, c)
                    dc = dgp @ P["w_gate"]
                    de[t] += dc[0, :self.d]
                    ds = (dz * (1.0 - gate) + dc[:, self.d:])[0]
            # end of segment: one product per weight, one masked memory pass per layer
            for name, (dys, xs) in rows.items():
                G[name] += np.concatenate(dys).T @ np.concatenate(xs)
            for l in range(L):
                g = 0 if self.cfg["groups"] == 1 else l
                ts = np.array([r[0] for r in deferred[l]])
                Qm = np.stack([r[1] for r in deferred[l]])
                dOm = np.stack([r[2] for r in deferred[l]])
                lse = np.stack([r[3] for r in deferred[l]], axis=1)  # [H, n]
                K, V = mem[g]
                hd = self.d // H
                sc = _split(Qm, H) @ _split(K, H).transpose(0, 2, 1) / np.sqrt(hd)
                allowed = np.arange(K.shape[0])[None, :] <= ts[:, None]
                Pm = np.where(allowed[None], np.exp(sc - lse[..., None]), 0.0)
                dP = _split(dOm, H) @ _split(V, H).transpose(0, 2, 1)
                Dm = np.sum(_split(dOm, H) * _split(self._om(Pm, V, H), H), axis=-1, keepdims=True)
                dS = Pm * (dP - Dm)
                dmem[g][0][:] += _merge_heads(dS.transpose(0, 2, 1) @ _split(Qm, H)) / np.sqrt(hd)
                dmem[g][1][:] += _merge_heads(Pm.transpose(0, 2, 1) @ _split(dOm, H))
        assert all(not p for p in pend), "every SWA adjoint reaches its step"
        G["s_star"][0] += ds
        self.encoder_b(tok, e, enc_cache, de, dmem, G)
        return loss, logp, G

    @staticmethod
    def _om(Pm, V, H):
        return _merge_heads(Pm @ _split(V, H))
