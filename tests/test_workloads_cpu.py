"""The seeded input recipe (workloads.py): same seed, same bytes; the Qwen3-8B-shaped
value distributions with the sink bias on each sequence's first keys and V rows of norm
sqrt(d)·exp(N(0, 0.5)); FP8 codes within e4m3 rounding of the BF16 tensors with scale
amax/448 rounded to float32; a paged cache that reproduces the contiguous K/V."""
import math

import numpy as np
import torch

from block_sparse_attention_oam_b200 import workloads as W

WL = W.QWEN_32K.with_(name="recipe", seqlens=(5000, 700), num_q_heads=4, num_kv_heads=2, seed=5)


def _same(a, b):
    return torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def test_seeded_and_deterministic():
    a, b = W.make_inputs(WL), W.make_inputs(WL)
    assert _same(a.q, b.q) and _same(a.k, b.k) and _same(a.v, b.v)
    c = W.make_inputs(WL.with_(seed=6))
    assert not _same(a.q, c.q) and not _same(a.k, c.k) and not _same(a.v, c.v)


def test_qwen_recipe_statistics():
    inp = W.make_inputs(WL)
    d = WL.head_dim
    q, k, v = inp.q.float(), inp.k.float(), inp.v.float()
    assert abs(float(q.mean())) < 3e-3 and abs(float(q.std()) * math.sqrt(d) - 1.0) < 0.01
    for t0, S in ((0, 5000), (5000, 700)):
        body = k[t0 + 128: t0 + S]
        assert abs(float(body.std()) * math.sqrt(d) - 1.0) < 0.02
        for h in range(WL.num_kv_heads):
            sink = float(k[t0: t0 + 128, h].mean(0).norm())      # 4/sqrt(d) = 0.354 plus noise ~0.09
            rest = float(k[t0 + 128: t0 + 256, h].mean(0).norm())
            assert 0.25 < sink < 0.46 and rest < 0.2, (t0, h, sink, rest)
    ln = torch.log(v.norm(dim=-1) / math.sqrt(d))
    assert abs(float(ln.mean())) < 0.02 and abs(float(ln.std()) - 0.5) < 0.02


def test_tiny_recipe():
    inp = W.make_inputs(W.TINY)
    q, k = inp.q.float(), inp.k.float()
    assert abs(float(q.std()) - 1.0) < 0.02
    for h in range(W.TINY.num_kv_heads):
        assert 3.5 < float(k[:64, h].mean(0).norm()) < 4.6      # the x4 unit direction
        assert float(k[64:128, h].mean(0).norm()) < 1.5


def test_fp8_codes_and_scales():
    ref = W.make_inputs(WL)
    inp = W.make_inputs(WL.with_(dtype="fp8_e4m3"))
    for name in ("q", "k", "v"):
        codes, scale, x = getattr(inp, name), getattr(inp, name + "_scale"), getattr(ref, name).float()
        assert codes.dtype == torch.float8_e4m3fn
        assert scale == float(np.float32(float(x.abs().max()) / W.FP8_E4M3_MAX))
        c = codes.float()
        assert float(c.abs().max()) == W.FP8_E4M3_MAX
        err = (c * scale - x).abs()
        bound = torch.maximum(x.abs() * 2.0 ** -4, torch.full_like(x, 2.0 ** -10 * scale)) * (1 + 1e-6)
        assert bool((err <= bound).all()), name


def test_paged_cache_reproduces_contiguous():
    wl = W.PAGED_VARLEN.with_(name="paged_recipe", seqlens=(300, 64, 129), num_q_heads=4, num_kv_heads=2, seed=9)
    inp = W.make_inputs(wl)
    P = wl.page_size
    used = inp.block_table[inp.block_table >= 0]
    assert sorted(used.tolist()) == list(range(inp.k_cache.shape[0]))       # every slot used once
    for b, S in enumerate(wl.seqlens):
        t0 = int(inp.cu_seqlens[b])
        t = np.arange(S)
        slots = inp.block_table[b, t // P]
        assert _same(inp.k_cache[slots, t % P], inp.k[t0: t0 + S])
        assert _same(inp.v_cache[slots, t % P], inp.v[t0: t0 + S])
        assert (inp.block_table[b, (S + P - 1) // P:] == -1).all()
