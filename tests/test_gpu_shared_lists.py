"""One selection per KV group — an extension of this library, not in the pages (the
oracle's reading: the group's score of a block is the float32 sum, in head order, of its
q-heads' OAM scores; the per-head budget, forced blocks and tie rule apply unchanged).
Same bars as the per-head path: selection bit-exact on the oracle's scores, end-to-end
list differences only inside the score gap, outputs within the BF16/FP8 tolerances; and
the BSA kernel reading a shared list equals it reading the same list copied per head."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from oracle import stem_oracle as O
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu

CASES = {
    "bf16_g4": W.QWEN_32K.with_(name="sh_bf16_g4", seqlens=(4096,), num_q_heads=8, num_kv_heads=2, seed=61,
                                shared_lists=True),
    "fp8_g4": W.LONG_128K_FP8.with_(name="sh_fp8_g4", seqlens=(3072,), num_q_heads=8, num_kv_heads=2, seed=62,
                                    shared_lists=True),
    "ragged_g2": W.QWEN_32K.with_(name="sh_ragged_g2", seqlens=(300, 2112, 1024), num_q_heads=4, num_kv_heads=2,
                                  seed=63, shared_lists=True),
    "paged_g4": W.PAGED_VARLEN.with_(name="sh_paged_g4", seqlens=(1024, 2000), num_q_heads=8, num_kv_heads=2,
                                     seed=64, shared_lists=True),
}
_cache = {}


def _inputs(name):
    if name not in _cache:
        _cache[name] = W.make_inputs(CASES[name])
    return _cache[name]


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


def _nblocks(wl):
    return [math.ceil(s / wl.block) for s in wl.seqlens]


@pytest.mark.parametrize("keep", [0.25, 0.1, 0.6])
@pytest.mark.parametrize("name", list(CASES))
def test_shared_select_bit_exact_on_oracle_scores(name, keep):
    inp = _inputs(name)
    wl = inp.wl.with_(keep=keep)
    g = wl.num_q_heads // wl.num_kv_heads
    prob = S.problem_for(wl, inp)
    packed, lists = [], []
    for b, N in enumerate(_nblocks(wl)):
        s = T.oracle_scores(inp, b).astype(np.float32)          # the exact bytes both sides sum and rank
        packed.append(np.ascontiguousarray(O.pack_causal(s)))
        lists.append(O.select_all_shared(s.astype(np.float64), O.tpd_plan(N, keep, wl.mu)[2], g))
    scores = torch.from_numpy(np.concatenate(packed, axis=1)).cuda()
    ws = S.workspace(prob)
    rp, ci = S.stem_select(prob, scores, ws=ws)
    S.query_status(ws)
    assert ci.shape[0] == wl.num_kv_heads
    rp_o, ci_o = O.to_csr(lists, wl.num_kv_heads)
    np.testing.assert_array_equal(rp.cpu().numpy(), rp_o)
    np.testing.assert_array_equal(ci.cpu().numpy(), ci_o)


@pytest.mark.parametrize("name", list(CASES))
def test_shared_bsa_equals_the_list_copied_per_head(name):
    """Reading list h/g (shared) or list h of a per-head copy gives the same bytes."""
    inp = _inputs(name)
    wl = inp.wl
    g = wl.num_q_heads // wl.num_kv_heads
    prob = S.problem_for(wl, inp)
    prob_h = S.problem_for(wl.with_(shared_lists=False), inp)
    dev = T.to_device(inp)
    ws = S.workspace(prob_h)
    scores = S.stem_score(prob, dev["q"], dev["k"], dev["v"], dev["paged"], ws=ws)
    rp, ci = S.stem_select(prob, scores, ws=ws)
    out_shared = S.bsa_prefill(prob, dev["q"], dev["k"], dev["v"], rp, ci, dev["paged"], ws=ws)
    ci_per_head = ci.repeat_interleave(g, dim=0).contiguous()
    out_copy = S.bsa_prefill(prob_h, dev["q"], dev["k"], dev["v"], rp, ci_per_head, dev["paged"], ws=ws)
    S.query_status(ws)
    assert torch.equal(out_shared, out_copy)


@pytest.mark.parametrize("name", list(CASES))
def test_shared_stem_attention_end_to_end(name):
    inp = _inputs(name)
    wl = inp.wl
    g = wl.num_q_heads // wl.num_kv_heads
    prob = S.problem_for(wl, inp)
    sz = prob.sizes()
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
    out = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], dev["paged"], row_ptr=rp, col_idx=ci, ws=ws)
    S.query_status(ws)
    rp, ci, out = rp.cpu().numpy(), ci.cpu().numpy(), out.float().cpu().numpy()
    tol = T.FP8_TOL if wl.dtype == "fp8_e4m3" else T.BF16_TOL
    row0 = 0
    for b, (t0, t1) in enumerate(T.seq_slices(inp)):
        N = _nblocks(wl)[b]
        s = T.oracle_scores(inp, b)
        sg = O.group_scores(s, g).astype(np.float64)
        ora = O.select_all(sg, O.tpd_plan(N, wl.keep, wl.mu)[2])
        for kh in range(wl.num_kv_heads):
            gl = [list(map(int, x)) for x in T.lists_from_csr(rp, ci, row0, N, kh)]
            for i, (gi, oi) in enumerate(zip(gl, ora[kh])):
                assert len(gi) == len(oi) and gi[0] == 0 and gi[-1] == i and gi == sorted(gi)
                if gi != oi:
                    kth = min(sg[kh, i, j] for j in oi if 0 < j < i)
                    for j in set(gi) - set(oi):
                        assert sg[kh, i, j] >= kth - T.SCORE_GAP * max(1.0, abs(kth)), (kh, i, j)
            for h in range(kh * g, (kh + 1) * g):
                q = T.oracle_dequant(inp, "q", t0, t1, [h])
                k = T.oracle_dequant(inp, "k", t0, t1, [kh])
                v = T.oracle_dequant(inp, "v", t0, t1, [kh])
                ref, _ = O.attend(q, k, v, [gl], wl.block, wl.softmax_scale)
                assert T.out_excess(out[t0:t1, h], ref[:, 0], tol) <= 0, (name, b, h)
        row0 += N
