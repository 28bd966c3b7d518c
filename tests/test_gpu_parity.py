"""GPU parity: every stage of the CUDA path (through the C-ABI) against the
float64 oracle on the same seeded inputs.

Bars: scores within 1e-3 relative; selection bit-exact when fed the oracle's
scores; BF16 outputs within 2e-2 (FP8 6e-2) plus half a bf16 ulp of the oracle's
value (the output format's own rounding) element by element; end-to-end
lists differ from the oracle's only where the score gap is below 1e-3."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from oracle import stem_oracle as O
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu

# Small workloads that still span several tiles, GQA, a ragged tail, FP8 and paging.
SMALL = {
    "tiny": W.TINY,
    "gqa_s4096": W.QWEN_32K.with_(name="gqa_s4096", seqlens=(4096,), num_q_heads=8, num_kv_heads=2, seed=11),
    "fp8_s4096": W.LONG_128K_FP8.with_(name="fp8_s4096", seqlens=(4096,), num_q_heads=8, num_kv_heads=2, seed=12),
    "ragged_varlen": W.QWEN_32K.with_(name="ragged_varlen", seqlens=(300, 1024, 2112, 77), num_q_heads=4,
                                      num_kv_heads=2, seed=13),
    "paged_varlen": W.PAGED_VARLEN.with_(name="paged_varlen", seqlens=(1024, 300, 2112), num_q_heads=8,
                                         num_kv_heads=2, seed=14),
    "d64_b128": W.QWEN_32K.with_(name="d64_b128", seqlens=(2048,), num_q_heads=4, num_kv_heads=4, head_dim=64,
                                 seed=15),
    "d128_b64": W.QWEN_32K.with_(name="d128_b64", seqlens=(1536,), num_q_heads=4, num_kv_heads=1, block=64,
                                 seed=16),
    "fp8_paged_varlen": W.PAGED_VARLEN.with_(name="fp8_paged_varlen", seqlens=(1024, 300, 2112), num_q_heads=8,
                                             num_kv_heads=2, dtype="fp8_e4m3", seed=17),
    "fp8_ragged_varlen": W.LONG_128K_FP8.with_(name="fp8_ragged_varlen", seqlens=(300, 1024, 2112, 77), num_q_heads=4,
                                               num_kv_heads=2, seed=18),
    # an odd number of q-heads: the last head pair of every row has one head
    "odd_heads": W.QWEN_32K.with_(name="odd_heads", seqlens=(1500, 400), num_q_heads=3, num_kv_heads=1, seed=19),
    # the most sequences a batch may hold (STEM_MAX_SEQS), of seeded lengths 1..299
    "max_seqs_64": W.QWEN_32K.with_(name="max_seqs_64", seqlens=(
        177, 126, 107, 277, 114, 82, 263, 18, 133, 93, 9, 215, 298, 234, 97, 162, 254, 94, 128, 274,
        59, 278, 203, 131, 236, 123, 108, 184, 276, 214, 200, 186, 251, 130, 222, 133, 181, 194,
        110, 275, 73, 15, 223, 27, 163, 228, 51, 138, 173, 233, 150, 162, 166, 139, 10, 286, 250,
        111, 110, 194, 267, 163, 82, 34),
                                    num_q_heads=4, num_kv_heads=2, seed=20),
    # an odd number of (sequence, head pair) groups, with more units than SMs: the launches
    # that deal the units forwards and back
    "snake_bf16": W.QWEN_32K.with_(name="snake_bf16", seqlens=(9000, 6000, 4000), num_q_heads=2, num_kv_heads=1,
                                   block=64, seed=21),
    "snake_fp8": W.LONG_128K_FP8.with_(name="snake_fp8", seqlens=(20000,), num_q_heads=2, num_kv_heads=1, seed=22),
}

_cache = {}


def inputs(name):
    if name not in _cache:
        _cache[name] = W.make_inputs(SMALL[name])
    return _cache[name]


def _seq_blocks(wl):
    return [math.ceil(s / wl.block) for s in wl.seqlens]


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", list(SMALL))
def test_scores_match_oracle(name):
    inp = inputs(name)
    wl = inp.wl
    prob = S.problem_for(wl, inp)
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    scores = S.stem_score(prob, dev["q"], dev["k"], dev["v"], dev["paged"], ws=ws).cpu().numpy()
    S.query_status(ws)
    off = 0
    for b, N in enumerate(_seq_blocks(wl)):
        ref = T.oracle_scores(inp, b)
        T.check_scores(T.gpu_scores_dense(scores, N, off), ref)
        off += N * (N + 1) // 2


@pytest.mark.parametrize("name", ["tiny", "gqa_s4096", "ragged_varlen", "paged_varlen"])
@pytest.mark.parametrize("keep,mu", [(0.25, 0.7), (0.1, 0.7), (0.5, 1.0), (1.0, 0.7)])
def test_select_bit_exact_on_oracle_scores(name, keep, mu):
    inp = inputs(name)
    wl = inp.wl.with_(keep=keep, mu=mu)
    prob = S.problem_for(wl, inp)
    packed, lists = [], []
    for b, N in enumerate(_seq_blocks(wl)):
        s = T.oracle_scores(inp, b).astype(np.float32)            # the exact bytes both sides rank
        packed.append(np.ascontiguousarray(O.pack_causal(s)))
        k = O.tpd_plan(N, keep, mu)[2]
        lists.append(O.select_all(s.astype(np.float64), k))
    scores = torch.from_numpy(np.concatenate(packed, axis=1)).cuda()
    ws = S.workspace(prob)
    rp, ci = S.stem_select(prob, scores, ws=ws)
    S.query_status(ws)
    rp_o, ci_o = O.to_csr(lists, wl.num_q_heads)
    np.testing.assert_array_equal(rp.cpu().numpy(), rp_o)
    np.testing.assert_array_equal(ci.cpu().numpy(), ci_o)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_ties_and_nans_bit_exact(seed):
    """Integer-valued scores (many exact ties), -0.0, +-inf and NaN: the
    (score desc, index asc) rule with NaN ranked as -inf."""
    rng = np.random.default_rng(seed)
    seqlens = (128 * 70, 128 * 33)
    prob = S.Problem(np.concatenate([[0], np.cumsum(seqlens)]), 8, 2, 128, 128, keep=0.3)
    packed, lists = [], []
    for S_ in seqlens:
        N = S_ // 128
        s = rng.integers(-3, 4, size=(8, N, N)).astype(np.float32)
        s[rng.random(s.shape) < 0.05] = np.nan
        s[rng.random(s.shape) < 0.03] = -np.inf
        s[rng.random(s.shape) < 0.03] = np.inf
        s[rng.random(s.shape) < 0.05] = -0.0
        s[:, np.triu_indices(N, 1)[0], np.triu_indices(N, 1)[1]] = np.nan
        packed.append(np.ascontiguousarray(O.pack_causal(s)))
        lists.append(O.select_all(s.astype(np.float64), O.tpd_plan(N, 0.3, 0.7)[2]))
    scores = torch.from_numpy(np.concatenate(packed, axis=1)).cuda()
    ws = S.workspace(prob)
    rp, ci = S.stem_select(prob, scores, ws=ws)
    S.query_status(ws)
    rp_o, ci_o = O.to_csr(lists, 8)
    np.testing.assert_array_equal(rp.cpu().numpy(), rp_o)
    np.testing.assert_array_equal(ci.cpu().numpy(), ci_o)


def _oracle_csr(inp, keep=None):
    wl = inp.wl if keep is None else inp.wl.with_(keep=keep)
    lists = []
    for b, N in enumerate(_seq_blocks(wl)):
        s = T.oracle_scores(inp, b)
        lists.append(O.select_all(s, O.tpd_plan(N, wl.keep, wl.mu)[2]))
    return lists, O.to_csr(lists, wl.num_q_heads)


@pytest.mark.parametrize("name", list(SMALL))
def test_bsa_matches_oracle_attention(name):
    inp = inputs(name)
    wl = inp.wl
    prob = S.problem_for(wl, inp)
    dev = T.to_device(inp)
    lists, (rp, ci) = _oracle_csr(inp)
    ws = S.workspace(prob)
    T_ = sum(wl.seqlens)
    lse = torch.full((wl.num_q_heads, T_), float("nan"), dtype=torch.float32, device="cuda")
    out = S.bsa_prefill(prob, dev["q"], dev["k"], dev["v"], torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(),
                        dev["paged"], lse=lse, ws=ws)
    S.query_status(ws)
    out = out.float().cpu().numpy()
    lse = lse.cpu().numpy()
    tol = T.FP8_TOL if wl.dtype == "fp8_e4m3" else T.BF16_TOL
    worst = -np.inf
    for b, (t0, t1) in enumerate(T.seq_slices(inp)):
        N = _seq_blocks(wl)[b]
        for h in range(wl.num_q_heads):
            g = wl.num_q_heads // wl.num_kv_heads
            q = T.oracle_dequant(inp, "q", t0, t1, [h])
            k = T.oracle_dequant(inp, "k", t0, t1, [h // g])
            v = T.oracle_dequant(inp, "v", t0, t1, [h // g])
            ref, ref_lse = O.attend(q, k, v, [lists[b][h]], wl.block, wl.softmax_scale)
            err = T.out_excess(out[t0:t1, h, :], ref[:, 0, :], tol)
            worst = max(worst, err)
            assert err <= 0, (b, h, err)
            assert np.abs(lse[h, t0:t1] - ref_lse[0]).max() <= 2e-3 * max(1.0, np.abs(ref_lse).max())
    assert np.isfinite(out).all()


@pytest.mark.parametrize("name", ["tiny", "gqa_s4096", "paged_varlen", "fp8_s4096", "d128_b64"])
def test_dense_kernel_equals_keep_one_selection_and_oracle(name):
    inp = inputs(name)
    wl = inp.wl.with_(keep=1.0)
    prob = S.problem_for(wl, inp)
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    dense = S.bsa_dense_prefill(prob, dev["q"], dev["k"], dev["v"], dev["paged"], ws=ws)
    lists, (rp, ci) = _oracle_csr(inp, keep=1.0)
    assert all(lists[b][h][i] == list(range(i + 1)) for b in range(len(lists)) for h in range(wl.num_q_heads)
               for i in range(len(lists[b][h])))
    sparse = S.bsa_prefill(prob, dev["q"], dev["k"], dev["v"], torch.from_numpy(rp).cuda(),
                           torch.from_numpy(ci).cuda(), dev["paged"], ws=ws)
    S.query_status(ws)
    assert torch.equal(dense, sparse)                      # same kernel path, same visiting order
    # against the library routine the dense case reduces to (float64 SDPA on the CPU)
    out = dense.float().cpu().numpy()
    tol = T.FP8_TOL if wl.dtype == "fp8_e4m3" else T.BF16_TOL
    g = wl.num_q_heads // wl.num_kv_heads
    for (t0, t1) in T.seq_slices(inp):
        q = torch.from_numpy(T.oracle_dequant(inp, "q", t0, t1)).permute(1, 0, 2)[None]
        k = torch.from_numpy(np.repeat(T.oracle_dequant(inp, "k", t0, t1), g, axis=1)).permute(1, 0, 2)[None]
        v = torch.from_numpy(np.repeat(T.oracle_dequant(inp, "v", t0, t1), g, axis=1)).permute(1, 0, 2)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=wl.softmax_scale)
        ref = ref[0].permute(1, 0, 2).numpy()
        assert T.out_excess(out[t0:t1], ref, tol) <= 0


def _check_lists_within_gap(gpu_lists, ora_lists, scores):
    """Every block the GPU kept and the oracle did not must score within the gap
    of the oracle's k-th best candidate (the tie band); sizes must agree."""
    for i, (g, o) in enumerate(zip(gpu_lists, ora_lists)):
        assert len(g) == len(o) and g[0] == 0 and g[-1] == i and sorted(g) == list(g)
        if g == o:
            continue
        chosen_o = [j for j in o if 0 < j < i]
        kth = min(scores[i, j] for j in chosen_o)
        for j in set(g) - set(o):
            assert scores[i, j] >= kth - T.SCORE_GAP * max(1.0, abs(kth)), (i, j, scores[i, j], kth)


@pytest.mark.parametrize("name", list(SMALL))
def test_stem_attention_end_to_end(name):
    inp = inputs(name)
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
    row0 = 0
    for b, (t0, t1) in enumerate(T.seq_slices(inp)):
        N = _seq_blocks(wl)[b]
        s = T.oracle_scores(inp, b)
        ora = O.select_all(s, O.tpd_plan(N, wl.keep, wl.mu)[2])
        g = wl.num_q_heads // wl.num_kv_heads
        for h in range(wl.num_q_heads):
            gl = T.lists_from_csr(rp, ci, row0, N, h)
            _check_lists_within_gap(gl, ora[h], s[h])
            q = T.oracle_dequant(inp, "q", t0, t1, [h])
            k = T.oracle_dequant(inp, "k", t0, t1, [h // g])
            v = T.oracle_dequant(inp, "v", t0, t1, [h // g])
            ref, _ = O.attend(q, k, v, [[list(map(int, x)) for x in gl]], wl.block, wl.softmax_scale)
            assert T.out_excess(out[t0:t1, h], ref[:, 0], tol) <= 0
        row0 += N


def test_two_calls_same_result_and_status_clean():
    inp = inputs("gqa_s4096")
    prob = S.problem_for(inp.wl, inp)
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    a = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], ws=ws)
    b = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], ws=ws)
    assert S.query_status(ws) == S.STEM_OK
    assert torch.equal(a, b)


def test_corrupt_selection_reports_bounds_error():
    """A block index beyond the diagonal is caught by the kernel's own bounds
    check (clamped, flagged) and reported as STEM_ERR_BOUNDS; the GPU stays usable."""
    inp = inputs("gqa_s4096")
    prob = S.problem_for(inp.wl, inp)
    dev = T.to_device(inp)
    lists, (rp, ci) = _oracle_csr(inp)
    ci = ci.copy()
    ci[0, rp[5]] = 31                     # row 5 may only list blocks 0..5
    ws = S.workspace(prob)
    S.bsa_prefill(prob, dev["q"], dev["k"], dev["v"], torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(), ws=ws)
    with pytest.raises(S.StemError) as e:
        S.query_status(ws)
    assert e.value.status == S.STEM_ERR_BOUNDS
    S.stem_attention(prob, dev["q"], dev["k"], dev["v"], ws=ws)   # context still healthy
    assert S.query_status(ws) == S.STEM_OK


def test_list_not_ending_on_the_diagonal_reports_bounds_error():
    """The token-level causal mask applies to the last list entry, which must be the
    diagonal block; a list that ends elsewhere (every entry still within 0..i) is
    flagged by the kernel and reported as STEM_ERR_BOUNDS."""
    inp = inputs("gqa_s4096")
    prob = S.problem_for(inp.wl, inp)
    dev = T.to_device(inp)
    lists, (rp, ci) = _oracle_csr(inp)
    ci = ci.copy()
    assert ci[1, rp[6] - 1] == 5
    ci[1, rp[6] - 1] = 4                  # row 5 of head 1 now ends on block 4
    ws = S.workspace(prob)
    S.bsa_prefill(prob, dev["q"], dev["k"], dev["v"], torch.from_numpy(rp).cuda(), torch.from_numpy(ci).cuda(), ws=ws)
    with pytest.raises(S.StemError) as e:
        S.query_status(ws)
    assert e.value.status == S.STEM_ERR_BOUNDS
    S.stem_attention(prob, dev["q"], dev["k"], dev["v"], ws=ws)
    assert S.query_status(ws) == S.STEM_OK


@pytest.mark.parametrize("bad", ["past_end", "negative"])
def test_corrupt_page_slot_reports_bounds_error_in_scoring(bad):
    """A block-table entry outside the cache (within a sequence's pages) is caught by
    the pooling kernel, which reads slot 0 instead and reports STEM_ERR_BOUNDS before
    the attention kernel runs; the GPU stays usable."""
    inp = inputs("paged_varlen")
    prob = S.problem_for(inp.wl, inp)
    dev = T.to_device(inp)
    paged = dev["paged"]
    table = paged.block_table.clone()
    num_slots = paged.k_cache.shape[0]
    table[1, 2] = num_slots + 7 if bad == "past_end" else -3   # sequence 1 has 5 pages
    bad_paged = S.PagedKV(paged.k_cache, paged.v_cache, table)
    ws = S.workspace(prob)
    S.stem_score(prob, dev["q"], None, None, bad_paged, ws=ws)
    with pytest.raises(S.StemError) as e:
        S.query_status(ws)
    assert e.value.status == S.STEM_ERR_BOUNDS
    S.stem_score(prob, dev["q"], None, None, paged, ws=ws)
    assert S.query_status(ws) == S.STEM_OK
