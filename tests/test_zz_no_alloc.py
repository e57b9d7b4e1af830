"""The allocation-free prefix attention (rlt_op_prefix_attention_noalloc) gives
the same output as the allocating entry point, bit for bit (the same kernels
run with the same chunking; only where the chunk partials live differs), on
several calls in a row (the shared static scratch keeps each call's
contents), and rejects a call
whose scratch would not fit.  Some callers cannot allocate device memory:
serving engines that hand all of the GPU's memory to their own pool, and
latency-critical paths that cannot take the device-wide synchronisation of
cudaMalloc/cudaFree; this entry point is for them.  The file sorts last so a
run that stops at the first failure has run every other test first."""
import pytest

pytestmark = pytest.mark.gpu


def _inputs(torch, B, H, hd, n, ld_t, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H * hd, generator=g).cuda()
    k = torch.randn(B, H, ld_t, hd, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(B, H, ld_t, hd, generator=g).to(torch.bfloat16).cuda()
    return q, k, v


def _rope(torch, npos, hd):
    i = torch.arange(hd // 2, dtype=torch.float64)
    p = torch.arange(npos, dtype=torch.float64)[:, None]
    ang = p * 10000.0 ** (-2.0 * i / hd)
    return torch.stack([torch.cos(ang), torch.sin(ang)], dim=-1).float().contiguous().cuda()


def test_noalloc_matches_allocating_entry_point_twice():
    import torch
    import stateful_decoder_b200 as rlt
    # first call: several 256-key chunks (uses the scratch); second call:
    # a different, smaller shape that reuses the same scratch slots; third:
    # the largest head size the entry points take
    for (B, H, hd, n, ld_t, seed) in ((4, 16, 128, 1000, 1024, 1), (3, 8, 128, 300, 512, 2),
                                      (2, 2, 256, 600, 640, 3)):
        rope = _rope(torch, 128, hd)
        q, k, v = _inputs(torch, B, H, hd, n, ld_t, seed)
        want = torch.zeros(B, H * hd, dtype=torch.bfloat16, device="cuda")
        got = torch.full((B, H * hd), 7.0, dtype=torch.bfloat16, device="cuda")
        rlt.rlt_op_prefix_attention(q, k, v, n, want, rope_cs=rope, qpos=99)
        rlt.rlt_op_prefix_attention_noalloc(q, k, v, n, got, rope_cs=rope, qpos=99)
        torch.cuda.synchronize()
        assert torch.equal(got, want), (got.float() - want.float()).abs().max().item()


def test_noalloc_rejects_oversized_scratch():
    import torch
    import stateful_decoder_b200 as rlt
    # 256 x 16 heads x 8 chunks x 130 floats = 4.26 M floats > 4 M
    B, H, n, ld_t = 256, 16, 2048, 2048
    q = torch.zeros(B, H * 128, device="cuda")
    k = torch.zeros(B, H, ld_t, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(B, H * 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rlt.RltError) as e:
        rlt.rlt_op_prefix_attention_noalloc(q, k, k, n, out)
    assert e.value.code == rlt.RLT_E_CAPACITY
