"""CPU oracle for the Stem sparse-attention prefill path.

TEST INFRASTRUCTURE ONLY.  This module is a plain, slow, float64 restatement of
what the path computes.  Only the test-suite, the smoke check and the timed CPU
baseline of the benchmark may import it; the product (the C-ABI library and its
Python binding) never does, and shares no code with it.

Sources (public web pages about Tencent Hunyuan's Stem, cited by page title and
section):
  [ARCH]  Tencent Cloud developer article "从Stem稀疏注意力看 大模型推理的架构取舍"
          sections "用架构师的眼睛看稀疏注意力", "TPD：优先级排序", "OAM：价值评估",
          "HPC-Stem：评估选块，快几十倍", "HPC-BSA：跳块零开销的秘密",
          "答案不在算法里".
  [WEDO]  wedoany.com news "腾讯混元 Stem 稀疏注意力" (TPD/OAM paragraph).
  [SETUP] setupai.cc digest "技術深入" list (TPD per-layer top-k keeps the
          initial tokens; OAM ranks by approximate output magnitude).

Where the pages leave a step open, the plainest reading consistent with the
rest is taken; each such reading is marked READING below.

Every function here is pinned by CPU tests against closed forms, a hand-worked
example, brute force on tiny inputs, or a library routine it reduces to
(``torch.nn.functional.scaled_dot_product_attention`` for keep = 1).
"""
from __future__ import annotations

import bisect
import math

import numpy as np

FLT_MIN = 2.0 ** -126


def num_blocks(seqlen: int, block: int) -> int:
    """Blocks of a sequence; a partial last block counts (READING: partial blocks
    are pooled over their valid tokens and causally masked)."""
    return (seqlen + block - 1) // block


# ---------------------------------------------------------------------------
# Pooling: compact per-block representations ([ARCH] "HPC-Stem：评估选块，快几十倍":
# per-block summaries of Q and K are precomputed so that one GEMM scores every
# block pair).  READING: the summary is the mean over the block's tokens.
# ---------------------------------------------------------------------------
def pool_mean(x: np.ndarray, block: int) -> np.ndarray:
    """x [S, H, d] -> [H, N, d]: mean of the rows of each block (valid rows only)."""
    S, H, d = x.shape
    N = num_blocks(S, block)
    out = np.zeros((H, N, d), dtype=np.float64)
    for i in range(N):
        rows = x[i * block: min(S, (i + 1) * block)].astype(np.float64)
        out[:, i, :] = rows.sum(axis=0) / rows.shape[0]
    return out


def pool_log_norm(v: np.ndarray, block: int) -> np.ndarray:
    """v [S, H, d] -> [H, N]: mean over the block of log ||v_t||_2 ([ARCH] "OAM：价值评估":
    the magnitude term is log||V_j||_2).  READING: per-token natural log of the L2
    norm, averaged over the block; a zero norm is clamped to FLT_MIN."""
    S, H, d = v.shape
    N = num_blocks(S, block)
    out = np.zeros((H, N), dtype=np.float64)
    for i in range(N):
        rows = v[i * block: min(S, (i + 1) * block)].astype(np.float64)
        norms = np.sqrt((rows * rows).sum(axis=-1))            # [n, H]
        logs = np.log(np.maximum(norms, FLT_MIN))
        out[:, i] = logs.sum(axis=0) / rows.shape[0]
    return out


# ---------------------------------------------------------------------------
# OAM score ([ARCH] "OAM：价值评估" and "HPC-Stem"): routing relevance (QK^T)
# plus beta * log||V_j||, beta = 0.2, purely additive: no softmax, no gather.
# READING: the routing term carries the softmax scale sigma (1/sqrt(d) by default).
# ---------------------------------------------------------------------------
def oam_scores(qbar, kbar, lbar, sigma: float, beta: float) -> np.ndarray:
    """qbar [Hq,N,d], kbar [Hkv,N,d], lbar [Hkv,N] -> s [Hq,N,N]; NaN above the diagonal.

    s[h,i,j] = sigma * <qbar[h,i], kbar[h//g,j]> + beta * lbar[h//g,j]   for j <= i
    """
    Hq, N, d = qbar.shape
    Hkv = kbar.shape[0]
    g = Hq // Hkv
    s = np.full((Hq, N, N), np.nan, dtype=np.float64)
    tri = np.tril(np.ones((N, N), dtype=bool))
    for h in range(Hq):
        kh = h // g
        full = sigma * (qbar[h] @ kbar[kh].T) + beta * lbar[kh][None, :]
        s[h][tri] = full[tri]
    return s


def pack_causal(s: np.ndarray) -> np.ndarray:
    """[H,N,N] lower triangle -> [H, N(N+1)/2], row i at offset i(i+1)/2."""
    H, N, _ = s.shape
    rows, cols = np.tril_indices(N)
    return s[:, rows, cols]


# ---------------------------------------------------------------------------
# TPD budget ([ARCH] "TPD：优先级排序"; [WEDO]): the per-position top-k budget
# decays linearly from the initial position to the end, the end keeping mu = 0.7
# of the initial budget, with the total unchanged (redistributed, not increased).
# READINGS:
#   * position = query block i; the budget is a keep *fraction* of the row's i+1
#     causal blocks: r_i = r_start * (1 - (1-mu) * i/(N-1)),  k_i = floor(r_i * (i+1));
#   * block 0 and the diagonal are forced and count toward k_i:
#     k_i = min(i+1, max(m_i, floor(r_start * w_i))),  m_i = min(2, i+1),
#     w_i = (1 - (1-mu)*i/(N-1)) * (i+1)   (w_0 = 1 when N = 1);
#   * the target total is T = round-half-up(keep * C), C = N(N+1)/2, clamped to
#     [2N-1, C] (the forced blocks alone are 2N-1);
#   * r_start is the midpoint of the first interval of r on which K(r) = sum k_i(r)
#     reaches T.  K only jumps at r = n / w_i for m_i < n <= i+1; past the last
#     jump the interval is unbounded and r_start = 2 * (last jump).
# ---------------------------------------------------------------------------
def tpd_weights(N: int, mu: float) -> np.ndarray:
    if N == 1:
        return np.ones(1)
    return np.array([(1.0 - (1.0 - mu) * i / (N - 1)) * (i + 1) for i in range(N)], dtype=np.float64)


def tpd_min_keep(N: int) -> np.ndarray:
    return np.minimum(2, np.arange(N) + 1)


def tpd_counts(r: float, N: int, mu: float) -> np.ndarray:
    w = tpd_weights(N, mu)
    i = np.arange(N)
    return np.minimum(i + 1, np.maximum(tpd_min_keep(N), np.floor(r * w).astype(np.int64)))


def tpd_target(N: int, keep: float) -> int:
    C = N * (N + 1) // 2
    T = int(math.floor(keep * C + 0.5))
    return max(2 * N - 1, min(C, T))


def tpd_jumps(N: int, mu: float) -> np.ndarray:
    """Sorted distinct values of r at which some k_i(r) increases."""
    w = tpd_weights(N, mu)
    m = tpd_min_keep(N)
    vals = [np.arange(m[i] + 1, i + 2, dtype=np.float64) / w[i] for i in range(N) if m[i] + 1 <= i + 1]
    if not vals:
        return np.zeros(0)
    return np.unique(np.concatenate(vals))


def tpd_plan(N: int, keep: float, mu: float):
    """Return (r_start, K_tot, k[N]) for one sequence of N blocks."""
    T = tpd_target(N, keep)
    b = tpd_jumps(N, mu)
    if b.size == 0:
        r = 1.0
        k = tpd_counts(r, N, mu)
        return r, int(k.sum()), k

    def midpoint(p):          # interval p lies between jump p-1 and jump p
        if p == 0:
            return b[0] / 2.0
        if p == b.size:
            return 2.0 * b[-1]
        return (b[p - 1] + b[p]) / 2.0

    totals = _KeyView(lambda p: int(tpd_counts(midpoint(p), N, mu).sum()), b.size + 1)
    p = bisect.bisect_left(totals, T)
    r = midpoint(p)
    k = tpd_counts(r, N, mu)
    return r, int(k.sum()), k


class _KeyView:
    """Lazy monotone sequence for bisect."""
    def __init__(self, f, n):
        self.f, self.n = f, n

    def __len__(self):
        return self.n

    def __getitem__(self, p):
        return self.f(p)


# ---------------------------------------------------------------------------
# Selection ([ARCH] "HPC-Stem" fuses budget generation with the top-k; the trunk
# argument of "用架构师的眼睛看稀疏注意力" keeps the initial block).  Block 0 and the
# diagonal are always kept; the other k_i - m_i come from blocks 1..i-1 ranked by
# (score descending, index ascending).  READING: NaN ranks as -inf.  The list is
# emitted in ascending block order (diagonal last).
# ---------------------------------------------------------------------------
def select_row(scores_row: np.ndarray, i: int, k_i: int) -> list:
    if i == 0:
        return [0]
    cand = np.arange(1, i)
    s = np.asarray(scores_row[1:i], dtype=np.float64)
    s = np.where(np.isnan(s), -np.inf, s)
    order = np.lexsort((cand, -s))          # primary: -s ascending; then index ascending
    chosen = cand[order[: k_i - 2]]
    return sorted([0, i] + [int(c) for c in chosen])


def select_all(s: np.ndarray, k: np.ndarray) -> list:
    """s [H,N,N] (dense lower triangle), k [N] -> lists[h][i]."""
    H, N, _ = s.shape
    return [[select_row(s[h, i, : i + 1], i, int(k[i])) for i in range(N)] for h in range(H)]


# ---------------------------------------------------------------------------
# One selection per KV group — an extension of this library, not in the pages.
# READING (own): the g q-heads that read one kv-head share one list per row.  The
# group's score of block j in row i is the sum over its q-heads, in head order, of
# their OAM scores, taken in float32 (the precision the device ranks in, so both
# sides rank the same numbers; the positive factor 1/g of a mean would not change the
# order).  Budget, forced blocks and tie rule are those of the per-head selection.
# ---------------------------------------------------------------------------
def group_scores(s: np.ndarray, g: int) -> np.ndarray:
    """s [Hq,N,N] -> [Hq/g, N, N] float32: the g heads of each group summed left to right."""
    Hq = s.shape[0]
    s32 = np.asarray(s, dtype=np.float32)
    out = np.empty((Hq // g,) + s.shape[1:], dtype=np.float32)
    for kh in range(Hq // g):
        acc = s32[kh * g].copy()
        for t in range(1, g):
            acc = np.add(acc, s32[kh * g + t], dtype=np.float32)
        out[kh] = acc
    return out


def select_all_shared(s: np.ndarray, k: np.ndarray, g: int) -> list:
    """s [Hq,N,N], k [N] -> lists[kh][i], one list per group of g q-heads."""
    return select_all(group_scores(s, g).astype(np.float64), k)


def expand_shared(lists_g: list, g: int) -> list:
    """Per-group lists -> per-q-head lists (q-head h uses group h // g)."""
    return [lists_g[h // g] for h in range(len(lists_g) * g)]


def to_csr(lists_per_seq: list, Hq: int):
    """lists_per_seq[b][h][i] -> (row_ptr [R+1] int32, col_idx [Hq, nnz] int32).
    row_ptr is shared by all heads (the budget does not depend on the head)."""
    lengths = [len(row) for seq in lists_per_seq for row in seq[0]]
    row_ptr = np.zeros(len(lengths) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(lengths)
    nnz = int(row_ptr[-1])
    col = np.zeros((Hq, nnz), dtype=np.int32)
    for h in range(Hq):
        flat = [c for seq in lists_per_seq for row in seq[h] for c in row]
        col[h] = flat
    return row_ptr.astype(np.int32), col


# ---------------------------------------------------------------------------
# Block-sparse causal attention ([ARCH] "HPC-BSA：跳块零开销的秘密": only the listed
# KV blocks are visited; a skipped block is mathematically the same as all its
# scores being -inf).  Written by deletion: the unlisted keys are simply absent.
# ---------------------------------------------------------------------------
def attend(q, k, v, lists, block: int, sigma: float, rows=None):
    """One sequence.  q [S,Hq,d], k/v [S,Hkv,d] float64; lists[h][i].
    rows: optional iterable of (h, i) q-tiles to compute (others left NaN).
    Returns out [S,Hq,d] and lse [Hq,S] (natural log)."""
    S, Hq, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    N = num_blocks(S, block)
    out = np.full((S, Hq, d), np.nan)
    lse = np.full((Hq, S), np.nan)
    todo = rows if rows is not None else [(h, i) for h in range(Hq) for i in range(N)]
    for h, i in todo:
        kh = h // g
        t = np.arange(i * block, min(S, (i + 1) * block))
        u = np.concatenate([np.arange(j * block, min(S, (j + 1) * block)) for j in lists[h][i]])
        logits = sigma * (q[t, h, :] @ k[u, kh, :].T)
        logits[u[None, :] > t[:, None]] = -np.inf
        m = logits.max(axis=1, keepdims=True)
        p = np.exp(logits - m)
        l = p.sum(axis=1, keepdims=True)
        out[t, h, :] = (p @ v[u, kh, :]) / l
        lse[h, t] = (m + np.log(l))[:, 0]
    return out, lse


def stem_sequence(q, k, v, block: int, keep: float, mu: float, beta: float, sigma: float,
                  rows=None, shared_lists: bool = False):
    """The whole path for one sequence: pool -> score -> plan -> select -> attend.
    shared_lists: one list per KV group (see select_all_shared)."""
    qbar, kbar, lbar = pool_mean(q, block), pool_mean(k, block), pool_log_norm(v, block)
    s = oam_scores(qbar, kbar, lbar, sigma, beta)
    N = qbar.shape[1]
    r, K, kk = tpd_plan(N, keep, mu)
    if shared_lists:
        g = q.shape[1] // k.shape[1]
        lists = expand_shared(select_all_shared(s, kk, g), g)
    else:
        lists = select_all(s, kk)
    out, lse = attend(q, k, v, lists, block, sigma, rows)
    return dict(qbar=qbar, kbar=kbar, lbar=lbar, scores=s, r_start=r, total=K, k=kk,
                lists=lists, out=out, lse=lse)
