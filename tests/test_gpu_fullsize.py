"""Parity at the full workload sizes, in the launch configuration bench.py times
(stem_score_select -> bsa_prefill), on outputs the oracle can compute one by one: every
score row of sampled q-heads (from stem_score), the selection of sampled heads
(bit-exact when fed the oracle's scores; the fused front's lists equal the score-matrix
path's on every head), and sampled attention tiles.  Also the largest supported
sequence (2048 blocks) and degenerate lengths."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from oracle import stem_oracle as O
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu

FULL = {
    "qwen3_8b_32k_bf16": W.QWEN_32K,
    "qwen3_8b_128k_fp8": W.LONG_128K_FP8,
    "qwen3_8b_64k_keep0.1": W.SWEEP_64K.with_(keep=0.1),
    "qwen3_8b_64k_keep1.0": W.SWEEP_64K.with_(keep=1.0),
    "paged_varlen_16k_to_128k": W.PAGED_VARLEN,
    "max_blocks_2048": W.QWEN_32K.with_(name="max_blocks", seqlens=(2048 * 128,), num_q_heads=2, num_kv_heads=1,
                                        head_dim=64, seed=31),
    "degenerate_lengths": W.QWEN_32K.with_(name="degenerate", seqlens=(1, 5, 127, 129, 256, 64), num_q_heads=4,
                                           num_kv_heads=2, block=64, seed=32),
}


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


def _run_path(wl, inp):
    """The bench's step (stem_score_select -> bsa_prefill) on one workspace, plus the
    score matrix and its selection (stem_score -> stem_select) for the checks."""
    prob = S.problem_for(wl, inp)
    sz = prob.sizes()
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    scores = torch.empty((wl.num_q_heads, sz["scores_per_head"]), dtype=torch.float32, device="cuda")
    rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty((wl.num_q_heads, sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
    out = torch.empty((sz["total_tokens"], wl.num_q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    S.stem_score(prob, dev["q"], dev["k"], dev["v"], dev["paged"], scores=scores, ws=ws)
    rp0, ci0 = S.stem_select(prob, scores, ws=ws)
    S.stem_score_select(prob, dev["q"], dev["k"], dev["v"], dev["paged"], rp, ci, ws=ws)
    S.bsa_prefill(prob, dev["q"], dev["k"], dev["v"], rp, ci, dev["paged"], out=out, ws=ws)
    S.query_status(ws)
    assert torch.equal(rp, rp0) and torch.equal(ci, ci0), "fused front differs from the score-matrix path"
    del rp0, ci0
    return prob, dev, ws, scores, rp, ci, out


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_sampled_parity(name):
    wl = FULL[name]
    inp = W.make_inputs(wl)
    prob, dev, ws, scores, rp, ci, out = _run_path(wl, inp)
    Hq = wl.num_q_heads
    heads = sorted({0, Hq - 1})
    tol = T.FP8_TOL if wl.dtype == "fp8_e4m3" else T.BF16_TOL
    scores_h = scores.cpu().numpy()
    rp_h, ci_h, out_h = rp.cpu().numpy(), ci.cpu().numpy(), out.float().cpu().numpy()

    # selection fed the oracle's (float32) scores on the sampled heads
    fed = scores_h.copy()
    off, row0, oracle_lists = 0, 0, []
    for b, (t0, t1) in enumerate(T.seq_slices(inp)):
        N = math.ceil((t1 - t0) / wl.block)
        ref = T.oracle_scores(inp, b, heads)                      # [len(heads), N, N]
        T.check_scores(T.gpu_scores_dense(scores_h[heads], N, off), ref)
        ref32 = ref.astype(np.float32)
        fed[heads, off: off + N * (N + 1) // 2] = O.pack_causal(ref32)
        k = O.tpd_plan(N, wl.keep, wl.mu)[2]
        oracle_lists.append(O.select_all(ref32.astype(np.float64), k))
        # end-to-end lists: equal to the oracle's except inside the score-gap band
        ora64 = O.select_all(ref, k)
        for n_h, h in enumerate(heads):
            gl = T.lists_from_csr(rp_h, ci_h, row0, N, h)
            _lists_within_gap(gl, ora64[n_h], ref[n_h])
        off += N * (N + 1) // 2
        row0 += N
    rp2, ci2 = S.stem_select(prob, torch.from_numpy(fed).cuda(), ws=ws)
    S.query_status(ws)
    rp2, ci2 = rp2.cpu().numpy(), ci2.cpu().numpy()
    assert np.array_equal(rp2, rp_h)
    row0 = 0
    for b, (t0, t1) in enumerate(T.seq_slices(inp)):
        N = math.ceil((t1 - t0) / wl.block)
        for n_h, h in enumerate(heads):
            got = T.lists_from_csr(rp2, ci2, row0, N, h)
            assert [list(map(int, x)) for x in got] == oracle_lists[b][n_h], (b, h)
        row0 += N

    # sampled attention tiles, against the oracle on the lists the GPU used
    row0 = 0
    g = Hq // wl.num_kv_heads
    for b, (t0, t1) in enumerate(T.seq_slices(inp)):
        N = math.ceil((t1 - t0) / wl.block)
        rows = sorted({0, min(1, N - 1), N // 2, N - 1})
        for h in heads:
            gl = [list(map(int, x)) for x in T.lists_from_csr(rp_h, ci_h, row0, N, h)]
            q = T.oracle_dequant(inp, "q", t0, t1, [h])
            k = T.oracle_dequant(inp, "k", t0, t1, [h // g])
            v = T.oracle_dequant(inp, "v", t0, t1, [h // g])
            ref, _ = O.attend(q, k, v, [gl], wl.block, wl.softmax_scale, rows=[(0, i) for i in rows])
            for i in rows:
                sl = slice(i * wl.block, min(t1 - t0, (i + 1) * wl.block))
                err = T.out_excess(out_h[t0:t1][sl, h], ref[sl, 0], tol)
                assert err <= 0, (name, b, h, i, err)
        row0 += N
    assert np.isfinite(out_h).all()


def _lists_within_gap(gpu_lists, ora_lists, s):
    for i, (gl, ol) in enumerate(zip(gpu_lists, ora_lists)):
        gl = [int(x) for x in gl]
        assert len(gl) == len(ol) and gl[0] == 0 and gl[-1] == i and gl == sorted(gl)
        if gl == ol:
            continue
        kth = min(s[i, j] for j in ol if 0 < j < i)
        for j in set(gl) - set(ol):
            assert s[i, j] >= kth - T.SCORE_GAP * max(1.0, abs(kth)), (i, j)
