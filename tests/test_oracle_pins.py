"""Pins for the CPU oracle: each check compares it with something other than
itself (closed forms, a hand-worked example, brute force on tiny inputs, or a
library routine the case reduces to)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import stem_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "hand_4block.json")


def _gold():
    with open(GOLD) as f:
        return json.load(f)


# ----------------------------------------------------------------- pooling
def test_pool_mean_constant_and_ramp_blocks():
    B, H, d = 4, 3, 5
    rng = np.random.default_rng(0)
    c = rng.standard_normal((3, H, d))
    x = np.repeat(c, B, axis=0)                       # block i is constant c_i
    np.testing.assert_array_equal(O.pool_mean(x, B), c.transpose(1, 0, 2))
    # arithmetic progression a + t*delta over the block: mean = a + delta*(n-1)/2
    a, delta = 1.5, 0.25
    t = np.arange(B, dtype=np.float64)
    x = (a + delta * t)[:, None, None] * np.ones((B, H, d))
    assert np.allclose(O.pool_mean(x, B), a + delta * (B - 1) / 2, rtol=0, atol=1e-15)


def test_pool_mean_partial_block_uses_valid_rows_only():
    x = np.zeros((6, 1, 1))
    x[4:, 0, 0] = [2.0, 4.0]                          # last block of size 4 has 2 valid rows
    assert O.pool_mean(x, 4)[0, 1, 0] == 3.0


def test_pool_log_norm_closed_forms():
    B, H, d = 4, 2, 3
    rng = np.random.default_rng(1)
    dirs = rng.standard_normal((2 * B, H, d))
    dirs /= np.linalg.norm(dirs, axis=-1, keepdims=True)
    c = np.array([[0.3, -1.2], [2.0, 0.0]])           # [block, head]
    v = dirs * np.exp(np.repeat(c, B, axis=0))[:, :, None]
    assert np.allclose(O.pool_log_norm(v, B), c.T, atol=1e-14)
    # alternating norms e^a, e^b -> (a+b)/2
    v2 = dirs[:B].copy()
    v2[0::2] *= math.e ** 1.0
    v2[1::2] *= math.e ** -3.0
    assert np.allclose(O.pool_log_norm(v2, B), -1.0, atol=1e-14)
    # zero rows are clamped to FLT_MIN
    assert O.pool_log_norm(np.zeros((B, 1, d)), B)[0, 0] == math.log(2.0 ** -126)


# ----------------------------------------------------------------- scoring
def test_scores_beta0_onehot_keys_read_q_component():
    Hq, Hkv, N, d = 4, 2, 5, 6
    rng = np.random.default_rng(2)
    qbar = rng.standard_normal((Hq, N, d))
    kbar = np.zeros((Hkv, N, d))
    for kh in range(Hkv):
        for j in range(N):
            kbar[kh, j, (j + 2 * kh) % d] = 1.0
    s = O.oam_scores(qbar, kbar, rng.standard_normal((Hkv, N)), sigma=0.5, beta=0.0)
    for h in range(Hq):
        kh = h // (Hq // Hkv)                          # GQA: q-head h reads kv-head h // g
        for i in range(N):
            for j in range(N):
                if j <= i:
                    assert s[h, i, j] == 0.5 * qbar[h, i, (j + 2 * kh) % d]
                else:
                    assert np.isnan(s[h, i, j])


def test_scores_magnitude_term_is_additive_and_shift_invariant_for_selection():
    Hq, Hkv, N, d = 2, 1, 9, 4
    rng = np.random.default_rng(3)
    qbar, kbar, lbar = rng.standard_normal((Hq, N, d)), rng.standard_normal((Hkv, N, d)), rng.standard_normal((Hkv, N))
    s0 = O.oam_scores(qbar, kbar, lbar, 0.3, 0.0)
    s1 = O.oam_scores(qbar, kbar, lbar, 0.3, 0.2)
    tri = ~np.isnan(s0)
    assert np.allclose((s1 - s0)[tri], (0.2 * np.broadcast_to(lbar[0][None, None, :], s0.shape))[tri])
    s2 = O.oam_scores(qbar, kbar, lbar + 7.0, 0.3, 0.2)        # constant shift of log||v||
    k = O.tpd_plan(N, 0.5, 0.7)[2]
    assert O.select_all(s1, k) == O.select_all(s2, k)


# ----------------------------------------------------------------- TPD budget
def test_hand_example_budget():
    g = _gold()
    N = 4
    assert np.allclose(O.tpd_weights(N, 0.7), g["expect"]["weights"], atol=1e-15)
    assert O.tpd_target(N, 0.8) == g["expect"]["target"]
    r, K, k = O.tpd_plan(N, 0.8, 0.7)
    assert list(k) == g["expect"]["k"] and K == 8
    assert abs(r - g["expect"]["r_start"]) < 1e-12
    assert 3 / 2.8 < r < 3 / 2.4


def test_decay_ratio_end_keeps_mu_of_start():
    for N in (2, 16, 256, 1024):
        w = O.tpd_weights(N, 0.7)
        frac = w / (np.arange(N) + 1)                      # keep fraction per row / r_start
        assert frac[0] == 1.0 and abs(frac[-1] - 0.7) < 1e-15
        assert np.all(np.diff(frac) < 0)                   # linear decay


@pytest.mark.parametrize("N,keep", [(16, 0.25), (256, 0.25), (1024, 0.25), (512, 1.0), (512, 0.5),
                                    (512, 0.25), (512, 0.2), (512, 0.1), (128, 0.25), (3, 0.5), (7, 0.9)])
def test_budget_sum_matches_target(N, keep):
    r, K, k = O.tpd_plan(N, keep, 0.7)
    C = N * (N + 1) // 2
    T = O.tpd_target(N, keep)
    assert T == max(2 * N - 1, min(C, math.floor(keep * C + 0.5)))
    assert K == int(k.sum()) == T                           # no coincident jumps at these sizes
    assert k[0] == 1 and np.all(k[1:] >= 2) and np.all(k <= np.arange(N) + 1)


def test_budget_edge_cases():
    for N in (1, 2, 5, 64):
        r, K, k = O.tpd_plan(N, 1.0, 0.7)
        assert list(k) == list(range(1, N + 1))             # keep = 1: dense causal
        r, K, k = O.tpd_plan(N, 1e-6, 0.7)
        assert K == 2 * N - 1                               # forced blocks only
    # mu = 1: uniform keep fraction, k_i = clamp(floor(r (i+1)))
    r, K, k = O.tpd_plan(64, 0.3, 1.0)
    i = np.arange(64)
    assert np.array_equal(k, np.minimum(i + 1, np.maximum(np.minimum(2, i + 1), np.floor(r * (i + 1)))))


@pytest.mark.parametrize("N", [3, 4, 8, 17, 40, 64])
@pytest.mark.parametrize("keep", [0.15, 0.25, 0.5, 0.8])
def test_budget_against_exhaustive_r_scan(N, keep):
    """Brute force: evaluate the total at just above every value n / w_i (n = 1..N,
    every row), i.e. on every interval where any floor can change.  The smallest
    total >= T must be K_tot, reached with the same k vector as at r_start."""
    T = O.tpd_target(N, keep)
    r0, K, k = O.tpd_plan(N, keep, 0.7)
    w = O.tpd_weights(N, 0.7)
    i = np.arange(N)
    cands = np.sort(np.concatenate([np.arange(1, N + 1) / wi for wi in w]))
    probes = np.concatenate([[cands[0] / 2], cands * (1 + 1e-11)])
    kk = np.minimum(i + 1, np.maximum(np.minimum(2, i + 1), np.floor(probes[:, None] * w[None, :])))
    tot = kk.sum(1)
    first = np.argmax(tot >= T)
    assert tot[first] == K
    assert np.array_equal(kk[first], k)


@pytest.mark.parametrize("S,B,T_expect", [(1024, 64, 34), (32768, 128, 8224), (131072, 128, 131200),
                                          (65536, 128, 32832), (16384, 128, 2064)])
def test_budget_at_workload_sizes(S, B, T_expect):
    N = S // B
    r, K, k = O.tpd_plan(N, 0.25, 0.7)
    C = N * (N + 1) // 2
    assert T_expect == math.floor(0.25 * C + 0.5)
    assert K == int(k.sum()) == T_expect


# ----------------------------------------------------------------- selection
def _dominance_ok(s, i, chosen):
    """Every chosen candidate beats every unchosen one under (score desc, index asc)."""
    cand = set(range(1, i))
    sel = set(chosen) - {0, i}
    key = lambda j: (-(s[j] if not np.isnan(s[j]) else -np.inf), j)
    return all(key(a) < key(b) for a in sel for b in cand - sel)


@pytest.mark.parametrize("seed", range(6))
def test_select_brute_force_small(seed):
    rng = np.random.default_rng(seed)
    for N in range(1, 9):
        s = rng.integers(-2, 3, size=(N, N)).astype(np.float64)  # many exact ties
        if seed % 2:
            s[rng.random((N, N)) < 0.1] = np.nan
        for i in range(N):
            for k_i in range(min(2, i + 1), i + 2):
                got = O.select_row(s[i, : i + 1], i, k_i)
                valid = [sorted({0, i} | set(c)) for c in itertools.combinations(range(1, i), k_i - min(2, i + 1))]
                winners = [c for c in valid if _dominance_ok(s[i], i, c)]
                assert len(winners) == 1 and got == winners[0]
                assert got[0] == 0 and got[-1] == i and len(got) == k_i


def test_hand_example_selection_and_csr():
    g = _gold()
    q, k, v = (np.array(g[n], dtype=np.float64)[:, None, :] for n in ("q", "k", "v"))
    p = g["params"]
    res = O.stem_sequence(q, k, v, 2, p["keep"], p["mu"], p["beta"], p["sigma"])
    e = g["expect"]
    assert np.array_equal(res["qbar"][0], e["qbar"]) and np.array_equal(res["kbar"][0], e["kbar"])
    assert np.allclose(res["lbar"][0], e["lbar"], atol=1e-15)
    assert np.allclose(res["scores"][0, 3], e["score_row3"], atol=1e-15)
    row_ptr, col = O.to_csr([res["lists"]], 1)
    assert list(row_ptr) == e["row_ptr"] and list(col[0]) == e["col_idx"]
    assert np.allclose(res["out"][0, 0], e["out_token0"]) and np.allclose(res["out"][1, 0], e["out_token1"])
    a = 1 / math.sqrt(2)
    ea = math.exp(a)
    assert np.allclose(res["out"][6, 0], [(2 + ea) / (3 + 2 * ea), (1 + ea) / (3 + 2 * ea)], atol=1e-14)
    # OAM changes the choice
    var = g["variant_oam_changes_choice"]
    res2 = O.stem_sequence(q, k, np.array(var["v"])[:, None, :], 2, p["keep"], p["mu"], p["beta"], p["sigma"])
    assert np.allclose(res2["lbar"][0], var["lbar"], atol=1e-15)
    assert res2["lists"][0][3] == var["row3"]
    # forced blocks only
    fo = g["variant_forced_only"]
    res3 = O.stem_sequence(q, k, v, 2, fo["keep"], p["mu"], p["beta"], p["sigma"])
    assert res3["total"] == fo["target"] and res3["lists"][0] == fo["lists"]


# ----------------------------------------------------------------- attention
def _sdpa(q, k, v, sigma, mask=None, causal=False):
    # torch layout [B, H, S, d]; GQA by repeating kv heads
    g = q.shape[1] // k.shape[1]
    Q = torch.from_numpy(q).permute(1, 0, 2)[None]
    K = torch.from_numpy(np.repeat(k, g, axis=1)).permute(1, 0, 2)[None]
    V = torch.from_numpy(np.repeat(v, g, axis=1)).permute(1, 0, 2)[None]
    o = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, is_causal=causal, scale=sigma)
    return o[0].permute(1, 0, 2).numpy()


def test_keep_one_is_dense_causal_attention():
    rng = np.random.default_rng(5)
    S, Hq, Hkv, d, B = 80, 4, 2, 8, 16                      # 5 blocks
    q, k, v = rng.standard_normal((S, Hq, d)), rng.standard_normal((S, Hkv, d)), rng.standard_normal((S, Hkv, d))
    res = O.stem_sequence(q, k, v, B, 1.0, 0.7, 0.2, 0.3)
    assert all(res["lists"][h][i] == list(range(i + 1)) for h in range(Hq) for i in range(5))
    ref = _sdpa(q, k, v, 0.3, causal=True)
    assert np.allclose(res["out"], ref, atol=1e-12)
    # LSE: log sum_u exp(sigma q.k_u) over the causal keys, checked on a few rows by brute force
    for (t, h) in [(0, 0), (37, 3), (79, 1)]:
        lg = [0.3 * q[t, h] @ k[u, h // 2] for u in range(t + 1)]
        assert abs(res["lse"][h, t] - math.log(sum(math.exp(x) for x in lg))) < 1e-12


def test_skipped_blocks_equal_minus_infinity_scores():
    """Deleting unlisted blocks (the oracle) == masking their logits with -inf (library)."""
    rng = np.random.default_rng(6)
    S, Hq, Hkv, d, B = 96, 2, 1, 8, 16                      # 6 blocks, partial budget
    q, k, v = rng.standard_normal((S, Hq, d)), rng.standard_normal((S, Hkv, d)), rng.standard_normal((S, Hkv, d))
    res = O.stem_sequence(q, k, v, B, 0.4, 0.7, 0.2, 0.25)
    for h in range(Hq):
        mask = np.full((S, S), -np.inf)
        for i in range(6):
            for j in res["lists"][h][i]:
                mask[i * B:(i + 1) * B, j * B:(j + 1) * B] = 0.0
        mask[np.triu_indices(S, 1)] = -np.inf
        ref = _sdpa(q[:, h:h + 1], k, v, 0.25, mask=torch.from_numpy(mask)[None, None])
        assert np.allclose(res["out"][:, h:h + 1], ref, atol=1e-12)
    assert any(len(res["lists"][0][i]) < i + 1 for i in range(6))   # something was skipped


def test_forced_only_row_by_hand():
    """A row keeping only block 0 and the diagonal: softmax over exactly those keys."""
    rng = np.random.default_rng(7)
    B, d = 4, 3
    S = 4 * B
    q, k, v = rng.standard_normal((S, 1, d)), rng.standard_normal((S, 1, d)), rng.standard_normal((S, 1, d))
    lists = [[[0], [0, 1], [0, 2], [0, 3]]]
    out, _ = O.attend(q, k, v, lists, B, 1.0)
    t = 13                                                  # block 3, row 1: keys 0..3 and 12, 13
    keys = [0, 1, 2, 3, 12, 13]
    w = np.array([math.exp(float(q[t, 0] @ k[u, 0])) for u in keys])
    expect = sum(wi * v[u, 0] for wi, u in zip(w, keys)) / w.sum()
    assert np.allclose(out[t, 0], expect, atol=1e-13)


# ------------------------------------------------------ one selection per KV group
# (an extension of this library, not in the pages: group score = float32 sum of the
# group's q-head scores, then the per-head selection rules)
def test_shared_lists_group_of_one_is_the_per_head_selection():
    rng = np.random.default_rng(21)
    s = rng.standard_normal((3, 9, 9)).astype(np.float32).astype(np.float64)
    k = O.tpd_plan(9, 0.4, 0.7)[2]
    assert np.array_equal(O.group_scores(s, 1), s.astype(np.float32))
    assert O.select_all_shared(s, k, 1) == O.select_all(s, k)


def test_shared_lists_identical_heads_give_the_head_lists():
    """Groups of identical heads (integer scores, so every float32 sum is exact): the group's
    list is each member head's own list."""
    rng = np.random.default_rng(22)
    for g in (2, 3, 4):
        base = rng.integers(-3, 4, size=(2, 10, 10)).astype(np.float64)
        s = np.repeat(base, g, axis=0)
        k = O.tpd_plan(10, 0.35, 0.7)[2]
        shared = O.select_all_shared(s, k, g)
        own = O.select_all(s, k)
        for h in range(2 * g):
            assert shared[h // g] == own[h]


@pytest.mark.parametrize("seed", range(4))
def test_shared_lists_brute_force_small(seed):
    """Integer scores (exact sums in any order): every group list is the unique subset that
    the (summed score descending, index ascending) order puts first."""
    rng = np.random.default_rng(30 + seed)
    g, N = 2, 8
    s = rng.integers(-2, 3, size=(2 * g, N, N)).astype(np.float64)
    k = O.tpd_plan(N, 0.45, 0.7)[2]
    shared = O.select_all_shared(s, k, g)
    for kh in range(2):
        tot = sum(s[kh * g + t] for t in range(g))       # float64 sum of small integers: exact
        for i in range(N):
            got = shared[kh][i]
            m = min(2, i + 1)
            valid = [sorted({0, i} | set(c)) for c in itertools.combinations(range(1, i), int(k[i]) - m)]
            winners = [c for c in valid if _dominance_ok(tot[i], i, c)]
            assert len(winners) == 1 and got == winners[0]
            assert got[0] == 0 and got[-1] == i and len(got) == k[i]


def test_shared_lists_keep_one_is_dense_causal_attention():
    rng = np.random.default_rng(23)
    S, Hq, Hkv, d, B = 64, 4, 2, 8, 16
    q, k, v = rng.standard_normal((S, Hq, d)), rng.standard_normal((S, Hkv, d)), rng.standard_normal((S, Hkv, d))
    res = O.stem_sequence(q, k, v, B, 1.0, 0.7, 0.2, 0.3, shared_lists=True)
    assert np.allclose(res["out"], _sdpa(q, k, v, 0.3, causal=True), atol=1e-12)


def test_shared_lists_members_of_a_group_read_the_same_blocks():
    rng = np.random.default_rng(24)
    S, Hq, Hkv, d, B = 160, 8, 2, 8, 16                      # g = 4, 10 blocks
    q, k, v = rng.standard_normal((S, Hq, d)), rng.standard_normal((S, Hkv, d)), rng.standard_normal((S, Hkv, d))
    res = O.stem_sequence(q, k, v, B, 0.3, 0.7, 0.2, 0.3, shared_lists=True)
    for h in range(Hq):
        assert res["lists"][h] == res["lists"][(h // 4) * 4]
        assert [len(r) for r in res["lists"][h]] == list(res["k"])
