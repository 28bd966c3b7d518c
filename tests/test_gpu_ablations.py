"""The two ablations the pages discuss, as run-time knobs of the same path, each held to
the parity bar of the default setting.

Tencent Cloud article "从Stem稀疏注意力看 大模型推理的架构取舍": section "TPD：优先级排序"
compares the decaying budget against a uniform one (mu = 1: every row keeps the same
fraction of its causal blocks); section "OAM：价值评估" compares the output-aware score
against the plain routing score (beta = 0: no log-norm term of V)."""
import dataclasses
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from oracle import stem_oracle as O
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu

BASE = {
    "bf16_gqa_s4096": W.QWEN_32K.with_(name="abl_bf16", seqlens=(4096,), num_q_heads=8, num_kv_heads=2, seed=41),
    "fp8_s4096": W.LONG_128K_FP8.with_(name="abl_fp8", seqlens=(4096,), num_q_heads=8, num_kv_heads=2, seed=42),
    "ragged_varlen": W.QWEN_32K.with_(name="abl_ragged", seqlens=(300, 2112, 1024), num_q_heads=4, num_kv_heads=2,
                                      seed=43),
}
ABLATIONS = {"beta0": dict(beta=0.0), "uniform_mu1": dict(mu=1.0), "both": dict(beta=0.0, mu=1.0)}

_cache = {}


def _inputs(name, ablation):
    """The base workload's inputs (the knobs do not change them) under the ablated settings."""
    if name not in _cache:
        _cache[name] = W.make_inputs(BASE[name])
    inp = _cache[name]
    return dataclasses.replace(inp, wl=inp.wl.with_(**ABLATIONS[ablation]))


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


def _nblocks(wl):
    return [math.ceil(s / wl.block) for s in wl.seqlens]


@pytest.mark.parametrize("ablation", list(ABLATIONS))
@pytest.mark.parametrize("name", list(BASE))
def test_ablation_scores_and_budgets(name, ablation):
    inp = _inputs(name, ablation)
    wl = inp.wl
    prob = S.problem_for(wl, inp)
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    scores = S.stem_score(prob, dev["q"], dev["k"], dev["v"], dev["paged"], ws=ws)
    rp, ci = S.stem_select(prob, scores, ws=ws)
    S.query_status(ws)
    scores, rp = scores.cpu().numpy(), rp.cpu().numpy()
    off, row0 = 0, 0
    for b, N in enumerate(_nblocks(wl)):
        T.check_scores(T.gpu_scores_dense(scores, N, off), T.oracle_scores(inp, b))
        # per-row budgets are the oracle's plan for these knobs, bit for bit
        k = np.asarray(O.tpd_plan(N, wl.keep, wl.mu)[2])
        np.testing.assert_array_equal(np.diff(rp[row0: row0 + N + 1]), k)
        if wl.mu == 1.0 and N > 1:
            # uniform budget: the kept fraction does not decay along the sequence
            r = O.tpd_plan(N, wl.keep, wl.mu)[0]
            i = np.arange(N)
            np.testing.assert_array_equal(k, np.minimum(i + 1, np.maximum(np.minimum(2, i + 1),
                                                                          np.floor(r * (i + 1)))))
        off += N * (N + 1) // 2
        row0 += N


@pytest.mark.parametrize("name", ["bf16_gqa_s4096", "fp8_s4096"])
def test_beta0_scores_do_not_depend_on_v(name):
    """With beta = 0 the score is the routing term alone: rescaling V rows changes nothing."""
    inp = _inputs(name, "beta0")
    prob = S.problem_for(inp.wl, inp)
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    a = S.stem_score(prob, dev["q"], dev["k"], dev["v"], ws=ws).cpu()
    v = dev["v"]
    v2 = v.view(torch.uint8).roll(5, 0).view(v.dtype).contiguous()   # other rows, other norms per block
    b = S.stem_score(prob, dev["q"], dev["k"], v2, ws=ws).cpu()
    S.query_status(ws)
    assert torch.equal(a, b)


@pytest.mark.parametrize("ablation", list(ABLATIONS))
@pytest.mark.parametrize("name", list(BASE))
def test_ablation_end_to_end(name, ablation):
    inp = _inputs(name, ablation)
    wl = inp.wl
    prob = S.problem_for(wl, inp)
    sz = prob.sizes()
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty((wl.num_q_heads, sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
    out = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], dev["paged"], row_ptr=rp, col_idx=ci, ws=ws)
    S.query_status(ws)
    rp, ci, out = rp.cpu().numpy(), ci.cpu().numpy(), out.float().cpu().numpy()
    tol = T.FP8_TOL if wl.dtype == "fp8_e4m3" else T.BF16_TOL
    g = wl.num_q_heads // wl.num_kv_heads
    row0 = 0
    for b, (t0, t1) in enumerate(T.seq_slices(inp)):
        N = _nblocks(wl)[b]
        s = T.oracle_scores(inp, b)
        ora = O.select_all(s, O.tpd_plan(N, wl.keep, wl.mu)[2])
        for h in range(wl.num_q_heads):
            gl = [list(map(int, x)) for x in T.lists_from_csr(rp, ci, row0, N, h)]
            for i, (gi, oi) in enumerate(zip(gl, ora[h])):
                assert len(gi) == len(oi) and gi[0] == 0 and gi[-1] == i and gi == sorted(gi)
                if gi != oi:
                    kth = min(s[h, i, j] for j in oi if 0 < j < i)
                    for j in set(gi) - set(oi):
                        assert s[h, i, j] >= kth - T.SCORE_GAP * max(1.0, abs(kth)), (h, i, j)
            q = T.oracle_dequant(inp, "q", t0, t1, [h])
            k = T.oracle_dequant(inp, "k", t0, t1, [h // g])
            v = T.oracle_dequant(inp, "v", t0, t1, [h // g])
            ref, _ = O.attend(q, k, v, [gl], wl.block, wl.softmax_scale)
            assert T.out_excess(out[t0:t1, h], ref[:, 0], tol) <= 0, (name, ablation, b, h)
        row0 += N
