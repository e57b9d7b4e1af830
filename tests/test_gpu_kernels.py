"""Kernel-level numerics of the decode attention (eq. 2.15 / eq. 2.8) against
a plain PyTorch fp32 reference of the same operation, through the C ABI's
op-level entry point.  Cases span one key, exact chunk boundaries (256),
ragged tails, several chunks (up to nine), head sizes 16/32/64/128/256 and
both storage types, with and without the rotary map on the query."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    import stateful_decoder_b200 as rlt
    return rlt, torch


def rope_table(torch, npos, hd, base=10000.0):
    i = torch.arange(hd // 2, dtype=torch.float64)
    p = torch.arange(npos, dtype=torch.float64)[:, None]
    ang = p * base ** (-2.0 * i / hd)
    return torch.stack([torch.cos(ang), torch.sin(ang)], dim=-1).float().contiguous()


def reference(torch, q, k, v, n, rope=None, qpos=0):
    B, H, _, hd = k.shape
    qh = q.double().view(B, H, hd)
    if rope is not None:
        c = rope[qpos, :, 0].double()
        s = rope[qpos, :, 1].double()
        a, b = qh[..., : hd // 2], qh[..., hd // 2:]
        qh = torch.cat([a * c - b * s, a * s + b * c], dim=-1)
    kk = k[:, :, :n].double()
    vv = v[:, :, :n].double()
    w = torch.softmax(torch.einsum("bhd,bhnd->bhn", qh, kk) / math.sqrt(hd), dim=-1)
    return torch.einsum("bhn,bhnd->bhd", w, vv).reshape(B, H * hd)


CASES = [  # B, H, hd, n, ld_t, dtype, rope
    (3, 2, 128, 1, 8, "bf16", False),
    (2, 4, 128, 256, 256, "bf16", True),
    (2, 4, 128, 257, 300, "bf16", False),
    (5, 2, 64, 700, 1024, "bf16", True),
    (1, 16, 128, 1023, 1024, "bf16", True),
    (2, 4, 16, 513, 600, "f32", True),
    (2, 2, 256, 300, 320, "bf16", True),
    (3, 1, 256, 100, 128, "f32", False),
    (2, 2, 64, 512, 520, "bf16", False),
    (2, 2, 64, 513, 520, "bf16", True),
    (1, 4, 32, 1100, 1200, "bf16", True),
    (1, 2, 16, 2100, 2200, "f32", True),
]


@pytest.mark.parametrize("B,H,hd,n,ld_t,dt,use_rope", CASES)
def test_prefix_attention_matches_torch(env, B, H, hd, n, ld_t, dt, use_rope):
    rlt, torch = env
    g = torch.Generator().manual_seed(B * 1000 + n)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    q = torch.randn(B, H * hd, generator=g).cuda()
    k = torch.randn(B, H, ld_t, hd, generator=g).to(tdt).cuda()
    v = torch.randn(B, H, ld_t, hd, generator=g).to(tdt).cuda()
    rope = rope_table(torch, 64, hd).cuda() if use_rope else None
    out = torch.zeros(B, H * hd, dtype=tdt, device="cuda")
    rlt.rlt_op_prefix_attention(q, k, v, n, out, rope_cs=rope, qpos=37)
    torch.cuda.synchronize()
    want = reference(torch, q.cpu(), k.float().cpu(), v.float().cpu(), n,
                     rope.cpu() if rope is not None else None, 37)
    tol = 1.5e-2 if dt == "bf16" else 2e-5  # bf16 output rounding vs fp32 arithmetic
    err = (out.double().cpu() - want).abs().max().item()
    assert err <= tol, err
