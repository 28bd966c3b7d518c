"""Seeded synthetic inputs for the Stem prefill path.

This module only draws random tensors and lays them out (token-major Q/K/V,
optional FP8-e4m3 quantisation with per-tensor scales, optional paged KV cache).
It holds none of the method's arithmetic: no pooling, scoring, budgeting,
selection or attention.  Both the CUDA path (through the C-ABI) and the CPU
oracle consume what it returns, so the two always see the same bytes.

Shapes follow the public descriptions of Stem (Tencent Hunyuan): block size 128,
keep fraction 25%, decay ratio 0.7, OAM weight 0.2, Qwen3-8B-shaped attention
(32 query heads, 8 KV heads, head dim 128) and contexts up to 128K tokens.
The pages measure on models and LongBench, which are not available; these
seeded tensors stand in for them.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

FP8_E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seqlens: tuple
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block: int
    keep: float
    dtype: str = "bf16"          # "bf16" or "fp8_e4m3"
    mu: float = 0.7
    beta: float = 0.2
    paged: bool = False
    page_size: int = 64
    style: str = "qwen"          # "tiny" or "qwen": value distribution recipe
    seed: int = 0
    shared_lists: bool = False   # one selection per KV group (an extension, not in the pages)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads the path is measured and checked on.
TINY = Workload("tiny_mha_s1024_b64", (1024,), 2, 2, 64, 64, 0.25, "bf16", style="tiny", seed=1)
QWEN_32K = Workload("qwen3_8b_layer_s32k_bf16", (32768,), 32, 8, 128, 128, 0.25, "bf16", seed=2)
LONG_128K_FP8 = Workload("qwen3_8b_layer_s128k_fp8", (131072,), 32, 8, 128, 128, 0.25, "fp8_e4m3", seed=3)
SWEEP_64K = Workload("qwen3_8b_layer_s64k_bf16", (65536,), 32, 8, 128, 128, 0.25, "bf16", seed=4)
SWEEP_KEEPS = (1.0, 0.5, 0.25, 0.2, 0.1)
PAGED_VARLEN = Workload("paged_varlen_4seq_16k_to_128k", (16384, 32768, 65536, 131072), 32, 8, 128, 128,
                        0.25, "bf16", paged=True, seed=5)

ALL = {w.name: w for w in (TINY, QWEN_32K, LONG_128K_FP8, SWEEP_64K, PAGED_VARLEN)}


@dataclasses.dataclass
class Inputs:
    """Device-ready inputs (CPU torch tensors in their storage dtype) plus the
    float64 values they represent (what the oracle consumes)."""
    wl: Workload
    cu_seqlens: np.ndarray            # int32 [num_seqs+1]
    q: torch.Tensor                   # [T, Hq, d] bf16 or float8_e4m3fn
    k: torch.Tensor                   # [T, Hkv, d] (logical token order)
    v: torch.Tensor                   # [T, Hkv, d]
    q_scale: float = 1.0
    k_scale: float = 1.0
    v_scale: float = 1.0
    # paged layout (only when wl.paged)
    k_cache: Optional[torch.Tensor] = None   # [num_slots, page, Hkv, d]
    v_cache: Optional[torch.Tensor] = None
    block_table: Optional[np.ndarray] = None  # int32 [num_seqs, max_pages]

    def dequant(self, which: str) -> np.ndarray:
        """float64 values of q/k/v exactly as the kernels see them."""
        t = getattr(self, which)
        s = getattr(self, which + "_scale")
        return t.float().numpy().astype(np.float64) * s


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream])))


def _trng(seed: int, stream: int) -> torch.Generator:
    """Seeded torch CPU generator for (workload seed, stream)."""
    return torch.Generator().manual_seed((int(seed) * 1_000_003 + int(stream)) & 0x7FFFFFFFFFFFFFFF)


def _unit_rows(rng, n, d):
    u = rng.standard_normal((n, d))
    return u / np.linalg.norm(u, axis=-1, keepdims=True)


_CHUNK = 4096   # tokens generated per step (small float32 buffers, reused)


def _gen_sequence_into(wl: Workload, seq_index: int, S: int, q_out, k_out, v_out) -> None:
    """Fill bf16 tensors q_out [S,Hq,d], k_out [S,Hkv,d], v_out [S,Hkv,d] for one sequence,
    _CHUNK tokens at a time (only the bf16 results are ever held at full size).
    Q, K ~ N(0,1)/sqrt(d) with a sink bias on the first 128 keys; V rows of norm
    sqrt(d) * exp(N(0, 0.5)) ("tiny": unit Q/K, a x4 sink direction on the first 64 keys,
    V rows scaled by exp(N(0, 0.5)))."""
    d, Hq, Hkv = wl.head_dim, wl.num_q_heads, wl.num_kv_heads
    base = 16 * seq_index
    rn, ru = (_rng(wl.seed, base + i) for i in (3, 4))
    gq, gk, gv = (_trng(wl.seed, base + i) for i in (0, 1, 2))
    log_norm = torch.from_numpy(rn.normal(0.0, 0.5, size=(S, Hkv)).astype(np.float32))
    u = torch.from_numpy(_unit_rows(ru, Hkv, d).astype(np.float32))   # sink direction per KV head
    tiny = wl.style == "tiny"
    inv = 1.0 if tiny else 1.0 / math.sqrt(d)
    nsink = min(64 if tiny else 128, S)
    sink = (4.0 if tiny else 4.0 * inv) * u
    n0 = min(_CHUNK, S)
    bq = torch.empty((n0, Hq, d), dtype=torch.float32)
    bk = torch.empty((n0, Hkv, d), dtype=torch.float32)
    bv = torch.empty((n0, Hkv, d), dtype=torch.float32)
    for t0 in range(0, S, _CHUNK):
        n = min(_CHUNK, S - t0)
        q, k, v = bq[:n], bk[:n], bv[:n]
        torch.randn((n, Hq, d), generator=gq, out=q)
        torch.randn((n, Hkv, d), generator=gk, out=k)
        torch.randn((n, Hkv, d), generator=gv, out=v)
        if not tiny:
            q.mul_(inv)
            k.mul_(inv)
        if t0 < nsink:
            k[: nsink - t0] += sink[None, :, :]
        ln = log_norm[t0: t0 + n]
        if tiny:
            v.mul_(torch.exp(ln)[:, :, None])
        else:
            v.div_(torch.linalg.vector_norm(v, dim=-1, keepdim=True))
            v.mul_((math.sqrt(d) * torch.exp(ln))[:, :, None])
        q_out[t0: t0 + n].copy_(q)
        k_out[t0: t0 + n].copy_(k)
        v_out[t0: t0 + n].copy_(v)


def _quant_fp8(x_bf16: torch.Tensor):
    """Per-tensor e4m3 codes and scale (amax / 448, a float32-representable value, so host
    float64 and device float32 agree exactly), a chunk of rows at a time."""
    amax = 0.0
    for t0 in range(0, x_bf16.shape[0], _CHUNK):
        amax = max(amax, float(x_bf16[t0: t0 + _CHUNK].abs().max()))
    scale = float(np.float32(amax / FP8_E4M3_MAX)) if amax > 0 else 1.0
    codes = torch.empty(x_bf16.shape, dtype=torch.float8_e4m3fn)
    for t0 in range(0, x_bf16.shape[0], _CHUNK):
        codes[t0: t0 + _CHUNK] = (x_bf16[t0: t0 + _CHUNK].float() / scale).to(torch.float8_e4m3fn)
    return codes, scale


def make_inputs(wl: Workload) -> Inputs:
    seqlens = [int(s) for s in wl.seqlens]
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    T = int(cu[-1])
    q = torch.empty((T, wl.num_q_heads, wl.head_dim), dtype=torch.bfloat16)
    k = torch.empty((T, wl.num_kv_heads, wl.head_dim), dtype=torch.bfloat16)
    v = torch.empty((T, wl.num_kv_heads, wl.head_dim), dtype=torch.bfloat16)
    for b, S in enumerate(seqlens):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        _gen_sequence_into(wl, b, S, q[t0:t1], k[t0:t1], v[t0:t1])
    inp = Inputs(wl, cu, q, k, v)
    if wl.dtype == "fp8_e4m3":
        inp.q, inp.q_scale = _quant_fp8(q)
        inp.k, inp.k_scale = _quant_fp8(k)
        inp.v, inp.v_scale = _quant_fp8(v)
    elif wl.dtype != "bf16":
        raise ValueError(wl.dtype)
    if wl.paged:
        _page(inp)
    return inp


def _page(inp: Inputs) -> None:
    """Scatter K/V into fixed-size pages at a seeded random permutation of slots."""
    wl = inp.wl
    P = wl.page_size
    pages_per_seq = [(s + P - 1) // P for s in wl.seqlens]
    num_slots = int(sum(pages_per_seq))
    max_pages = max(pages_per_seq)
    perm = _rng(wl.seed, 1000).permutation(num_slots).astype(np.int32)
    table = np.full((len(wl.seqlens), max_pages), -1, dtype=np.int32)
    Hkv, d = wl.num_kv_heads, wl.head_dim
    kc = torch.zeros((num_slots, P, Hkv, d), dtype=inp.k.dtype)
    vc = torch.zeros((num_slots, P, Hkv, d), dtype=inp.v.dtype)
    nxt = 0
    for b, S in enumerate(wl.seqlens):
        t0 = int(inp.cu_seqlens[b])
        for p in range(pages_per_seq[b]):
            slot = int(perm[nxt]); nxt += 1
            table[b, p] = slot
            n = min(P, S - p * P)
            kc[slot, :n] = inp.k[t0 + p * P: t0 + p * P + n]
            vc[slot, :n] = inp.v[t0 + p * P: t0 + p * P + n]
    inp.k_cache, inp.v_cache, inp.block_table = kc, vc, table

