"""The roofline's numerator: bench.selected_flops counts 4·d FLOPs (QKᵀ and PV, a
multiply-add each) per causally visible (query token, key token) pair of the listed
blocks.  Pinned by brute force over token pairs, by the dense count at keep = 1, and by
the selected-block figures of the 128K and 64K layers."""
import math

import numpy as np
import pytest

import bench
from block_sparse_attention_oam_b200 import stem as S
from oracle import stem_oracle as O


def _row_ptr(seqlens, block, keep, mu=0.7):
    rp = [0]
    for s in seqlens:
        k = O.tpd_plan(math.ceil(s / block), keep, mu)[2]
        for x in k:
            rp.append(rp[-1] + int(x))
    return np.asarray(rp, dtype=np.int64)


def _brute(seqlens, block, head_dim, heads, rp):
    """Visible (t, u) pairs of the listed blocks, counted token by token: every list keeps
    k_i blocks, block 0 and the diagonal among them, so any k_i of them give the same count
    as long as the diagonal is one of them (the budget does not depend on the choice)."""
    pairs = 0
    row0 = 0
    for s in seqlens:
        N = math.ceil(s / block)
        for i in range(N):
            k = int(rp[row0 + i + 1] - rp[row0 + i])
            listed = list(range(k - 1)) + [i]      # any k-1 earlier blocks plus the diagonal
            for t in range(i * block, min(s, (i + 1) * block)):
                for j in listed:
                    for u in range(j * block, min(s, (j + 1) * block)):
                        pairs += u <= t
        row0 += N
    return pairs * 4 * head_dim * heads


@pytest.mark.parametrize("seqlens,block,keep", [((300, 130), 64, 0.25), ((257,), 64, 0.5), ((64, 65, 1), 64, 0.3)])
def test_selected_flops_by_brute_force(seqlens, block, keep):
    rp = _row_ptr(seqlens, block, keep)
    prob = S.Problem([0] + list(np.cumsum(seqlens)), 3, 1, 32, block, keep=keep)
    assert bench.selected_flops(prob, rp, block, 32, seqlens) == _brute(seqlens, block, 32, 3, rp)


@pytest.mark.parametrize("seqlens", [(131072,), (300, 2112, 77), (16384, 32768, 65536, 131072)])
def test_keep_one_counts_the_dense_flops(seqlens):
    rp = _row_ptr(seqlens, 128, 1.0)
    prob = S.Problem([0] + list(np.cumsum(seqlens)), 32, 8, 128, 128, keep=1.0)
    assert bench.selected_flops(prob, rp, 128, 128, seqlens) == bench.dense_flops(seqlens, 32, 128)


def test_layer_figures():
    """Selected TFLOP of one Qwen3-8B-shaped layer at keep 0.25: 35.08 at 128K (140.74
    dense), 8.745 at 64K (35.18 dense)."""
    for s, sel, dense in ((131072, 35.08, 140.74), (65536, 8.745, 35.18)):
        rp = _row_ptr((s,), 128, 0.25)
        prob = S.Problem([0, s], 32, 8, 128, 128)
        assert abs(bench.selected_flops(prob, rp, 128, 128, (s,)) / 1e12 - sel) < 5e-3
        assert abs(bench.dense_flops((s,), 32, 128) / 1e12 - dense) < 5e-3
