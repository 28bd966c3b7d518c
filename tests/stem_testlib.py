"""Shared helpers for the GPU parity tests: run the oracle on a workload's inputs
(optionally on a subset of heads / rows) and move inputs to the device."""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from oracle import stem_oracle as O

BF16_TOL = 2e-2      # max-abs, bf16 output vs float64 oracle
FP8_TOL = 6e-2       # max-abs, fp8 path vs float64 oracle on the dequantised inputs
SCORE_RTOL = 1e-3    # relative, with a small absolute floor
SCORE_ATOL = 1e-5
SCORE_GAP = 1e-3     # end-to-end lists may differ only where the score gap is below this


def bf16_half_ulp(x):
    """Half a bf16 unit in the last place at |x| (8 significand bits): the rounding error the
    bf16 output format adds on its own to an exact result."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 8)


def out_bound(ref, base):
    """Element-wise bound for a bf16 output against the float64 oracle: `base` for the
    arithmetic (bf16 or FP8 operands, float32 accumulation) plus the output's own rounding."""
    return base + bf16_half_ulp(ref)


def out_excess(got, ref, base):
    """Largest (|got - ref| - bound); <= 0 means every element is within its bound."""
    return float((np.abs(got - ref) - out_bound(ref, base)).max())


def to_device(inp: W.Inputs):
    d = dict(q=inp.q.cuda(), k=inp.k.cuda(), v=inp.v.cuda(), paged=None)
    if inp.wl.paged:
        d["paged"] = S.PagedKV(inp.k_cache.cuda(), inp.v_cache.cuda(), torch.from_numpy(inp.block_table).cuda())
    return d


def seq_slices(inp: W.Inputs):
    cu = inp.cu_seqlens
    return [(int(cu[b]), int(cu[b + 1])) for b in range(len(cu) - 1)]


def oracle_pooled(inp: W.Inputs, b: int, heads=None):
    """Pooled Q/K/V terms of sequence b for q-heads `heads` (default all)."""
    wl = inp.wl
    t0, t1 = seq_slices(inp)[b]
    g = wl.num_q_heads // wl.num_kv_heads
    heads = list(range(wl.num_q_heads)) if heads is None else list(heads)
    kvh = sorted({h // g for h in heads})
    q = inp.q[t0:t1, heads].float().numpy().astype(np.float64) * inp.q_scale
    k = inp.k[t0:t1, kvh].float().numpy().astype(np.float64) * inp.k_scale
    v = inp.v[t0:t1, kvh].float().numpy().astype(np.float64) * inp.v_scale
    qbar = O.pool_mean(q, wl.block)
    kb = O.pool_mean(k, wl.block)
    lb = O.pool_log_norm(v, wl.block)
    # expand to per-q-head K/V terms
    pos = {kh: n for n, kh in enumerate(kvh)}
    kbar = np.stack([kb[pos[h // g]] for h in heads])
    lbar = np.stack([lb[pos[h // g]] for h in heads])
    return qbar, kbar, lbar


def oracle_scores(inp: W.Inputs, b: int, heads=None):
    qbar, kbar, lbar = oracle_pooled(inp, b, heads)
    # one kv-head per q-head after expansion: g = 1
    return O.oam_scores(qbar, kbar, lbar, inp.wl.softmax_scale, inp.wl.beta)


def gpu_scores_dense(scores_packed: np.ndarray, N: int, off: int) -> np.ndarray:
    """[H, packed] -> [H, N, N] lower triangle of one sequence (NaN above)."""
    H = scores_packed.shape[0]
    out = np.full((H, N, N), np.nan)
    r, c = np.tril_indices(N)
    out[:, r, c] = scores_packed[:, off: off + N * (N + 1) // 2]
    return out


def check_scores(gpu: np.ndarray, ref: np.ndarray):
    m = ~np.isnan(ref)
    err = np.abs(gpu[m] - ref[m])
    bound = SCORE_RTOL * np.abs(ref[m]) + SCORE_ATOL
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} scores off; worst err {err.max():.3e}"
    return float((err / (np.abs(ref[m]) + 1e-12)).max())


def oracle_dequant(inp: W.Inputs, which: str, t0: int, t1: int, heads=None):
    t = getattr(inp, which)[t0:t1]
    if heads is not None:
        t = t[:, heads]
    return t.float().numpy().astype(np.float64) * getattr(inp, which + "_scale")


def lists_from_csr(row_ptr: np.ndarray, col: np.ndarray, row0: int, N: int, h: int):
    return [list(col[h, row_ptr[row0 + i]: row_ptr[row0 + i + 1]]) for i in range(N)]


def attend_tiles(inp: W.Inputs, b: int, lists_by_head: dict, tiles):
    """Oracle attention of sequence b on tiles [(h, i)] with lists_by_head[h][i]."""
    wl = inp.wl
    t0, t1 = seq_slices(inp)[b]
    g = wl.num_q_heads // wl.num_kv_heads
    res = {}
    for h, i in tiles:
        q = oracle_dequant(inp, "q", t0, t1, [h])
        k = oracle_dequant(inp, "k", t0, t1, [h // g])
        v = oracle_dequant(inp, "v", t0, t1, [h // g])
        out, lse = O.attend(q, k, v, [lists_by_head[h]], wl.block, wl.softmax_scale, rows=[(0, i)])
        rows = slice(i * wl.block, min(t1 - t0, (i + 1) * wl.block))
        res[(h, i)] = (out[rows, 0, :], lse[0, rows])
    return res
