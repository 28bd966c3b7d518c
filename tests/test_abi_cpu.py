"""CPU-only checks of the C-ABI library: it loads, exports every function the
header declares, its host-side planner agrees with the oracle's, and bad
arguments are rejected before anything touches a GPU."""
import ctypes
import math

import numpy as np
import pytest

from block_sparse_attention_oam_b200 import build as B
from block_sparse_attention_oam_b200 import stem as S
from oracle import stem_oracle as O


@pytest.fixture(scope="module")
def L():
    B.build()
    return S.lib()


def test_library_exports_every_declared_function(L):
    names = S.header_functions()
    expect = {"stem_query_sizes", "stem_workspace_size", "stem_tpd_plan", "stem_score", "stem_select",
              "stem_score_select",
              "bsa_prefill", "bsa_dense_prefill", "stem_attention", "stem_query_status", "stem_reset_status",
              "stem_status_string", "stem_last_error", "stem_attention_noalloc", "stem_debug_inject",
              "stem_attention_host"}
    assert expect <= set(names), set(names)
    for n in names:
        assert hasattr(L, n), n


@pytest.mark.parametrize("N", [1, 2, 3, 4, 5, 16, 17, 64, 100, 256, 512, 1024, 2048])
@pytest.mark.parametrize("keep", [0.01, 0.1, 0.2, 0.25, 0.5, 0.8, 1.0])
@pytest.mark.parametrize("mu", [0.7, 1.0, 0.3])
def test_host_planner_matches_oracle(L, N, keep, mu):
    r, tot = S.tpd_plan(N, keep, mu)
    r_o, tot_o, k_o = O.tpd_plan(N, keep, mu)
    assert tot == tot_o
    assert r == r_o                         # same jump values, same midpoint: identical doubles
    assert int(O.tpd_counts(r, N, mu).sum()) == tot


def test_planner_rejects_bad_arguments(L):
    for args in [(0, 0.25, 0.7), (4, 0.0, 0.7), (4, 1.5, 0.7), (4, 0.25, 0.0), (4, 0.25, 1.2)]:
        with pytest.raises(S.StemError) as e:
            S.tpd_plan(*args)
        assert e.value.status == S.STEM_ERR_INVALID


def test_query_sizes_match_oracle_counts(L):
    seqlens = [300, 1024, 2048 + 64]
    p = S.Problem(np.concatenate([[0], np.cumsum(seqlens)]), 8, 2, 128, 128)
    sz = p.sizes()
    Ns = [math.ceil(s / 128) for s in seqlens]
    assert sz["num_rows"] == sum(Ns)
    assert sz["scores_per_head"] == sum(n * (n + 1) // 2 for n in Ns)
    assert sz["nnz_per_head"] == sum(O.tpd_plan(n, 0.25, 0.7)[1] for n in Ns)
    assert sz["total_tokens"] == sum(seqlens)
    assert sz["workspace_bytes"] >= 4 * (8 * sz["scores_per_head"] + 8 * sz["nnz_per_head"])


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, S.STEM_ERR_UNSUPPORTED),
    ("block_size", 32, S.STEM_ERR_UNSUPPORTED),
    ("num_kv_heads", 3, S.STEM_ERR_INVALID),
    ("keep", 0.0, S.STEM_ERR_INVALID),
    ("mu", 0.0, S.STEM_ERR_INVALID),
])
def test_problem_validation(L, field, value, status):
    kw = dict(cu_seqlens=[0, 1024], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=128)
    kw[field] = value
    with pytest.raises(S.StemError) as e:
        S.Problem(**kw).sizes()
    assert e.value.status == status


def test_fp8_shape_limits_and_bad_seqlens(L):
    with pytest.raises(S.StemError) as e:
        S.Problem([0, 1024], 2, 2, 64, 64, dtype="fp8_e4m3").sizes()
    assert e.value.status == S.STEM_ERR_UNSUPPORTED
    with pytest.raises(S.StemError) as e:
        S.Problem([0, 512, 512], 2, 2, 64, 64).sizes()       # empty sequence
    assert e.value.status == S.STEM_ERR_INVALID
    with pytest.raises(S.StemError) as e:
        S.Problem([0, 128 * 4096], 2, 2, 64, 128).sizes()   # more blocks than supported
    assert e.value.status == S.STEM_ERR_UNSUPPORTED


def test_batch_size_limit(L):
    """STEM_MAX_SEQS sequences are accepted, one more is refused on the host."""
    cu = [64 * b for b in range(65)]
    assert S.Problem(cu, 4, 2, 128, 64).sizes()["num_rows"] == 64
    with pytest.raises(S.StemError) as e:
        S.Problem(cu + [cu[-1] + 64], 4, 2, 128, 64).sizes()
    assert e.value.status == S.STEM_ERR_INVALID


def test_entry_points_reject_before_launch(L):
    """Null pointers and a short workspace are refused on the host (no CUDA call)."""
    p = S.Problem([0, 1024], 2, 2, 64, 64)
    fake = ctypes.c_void_p(0x1000)          # never dereferenced: validation fails first
    st = L.stem_score(p.c, None, fake, fake, None, fake, fake, 1 << 30, None)
    assert st == S.STEM_ERR_INVALID
    st = L.stem_score(p.c, fake, fake, fake, None, fake, fake, 16, None)
    assert st == S.STEM_ERR_WORKSPACE
    st = L.bsa_prefill(p.c, fake, fake, fake, None, None, fake, fake, None, fake, 1 << 30, None)
    assert st == S.STEM_ERR_INVALID
    st = L.stem_score_select(p.c, fake, fake, fake, None, None, fake, fake, 1 << 30, None)
    assert st == S.STEM_ERR_INVALID                           # no row_ptr
    st = L.stem_score_select(p.c, fake, fake, fake, None, fake, fake, fake, 16, None)
    assert st == S.STEM_ERR_WORKSPACE
    st = L.stem_attention(None, fake, fake, fake, None, fake, None, None, None, fake, 1 << 30, None)
    assert st == S.STEM_ERR_INVALID
    assert b"NULL" in L.stem_last_error()
    assert L.stem_status_string(S.STEM_ERR_TIMEOUT) == b"device pipeline wait timed out"


def test_host_entry_rejects_before_launch(L):
    """stem_attention_host refuses NULL host buffers, a negative group count and a
    short workspace on the host, before any copy or launch."""
    p = S.Problem([0, 1024], 2, 2, 64, 64)
    fake = ctypes.c_void_p(0x1000)

    def call(q_host=fake, out_host=fake, groups=0, ws_bytes=1 << 30):
        return L.stem_attention_host(p.c, q_host, fake, fake, fake, fake, fake, None, out_host, fake, None, None,
                                     None, groups, fake, ws_bytes, None)

    assert call(q_host=None) == S.STEM_ERR_INVALID
    assert b"host" in L.stem_last_error()
    assert call(out_host=None) == S.STEM_ERR_INVALID
    assert call(groups=-1) == S.STEM_ERR_INVALID
    assert call(ws_bytes=16) == S.STEM_ERR_WORKSPACE


def test_host_entry_binding_checks_host_tensors(L):
    """The binding refuses device or non-contiguous host tensors before calling the library."""
    import torch
    p = S.Problem([0, 256], 2, 2, 64, 64)
    q = torch.zeros((256, 2, 64), dtype=torch.bfloat16)
    strided = torch.zeros((256, 2, 128), dtype=torch.bfloat16)[:, :, ::2]
    with pytest.raises(ValueError, match="k_host"):
        S.stem_attention_host(p, q, strided, q, q, q, q, out_host=q, out=q, ws=torch.zeros(1 << 20, dtype=torch.uint8))


def test_shared_lists_sizes_and_validation(L):
    """One selection per KV group: col_idx has Hkv rows; any other flag value is refused."""
    cu = np.array([0, 1024, 3000])
    per_head = S.Problem(cu, 8, 2, 128, 128).sizes()
    shared = S.Problem(cu, 8, 2, 128, 128, shared_lists=True).sizes()
    assert per_head["list_heads"] == 8 and shared["list_heads"] == 2
    assert shared["nnz_per_head"] == per_head["nnz_per_head"]
    assert shared["workspace_bytes"] < per_head["workspace_bytes"]
    p = S.Problem(cu, 8, 2, 128, 128)
    p._c.shared_lists = 2
    st = L.stem_query_sizes(p.c, ctypes.byref(S._Sizes()))
    assert st == S.STEM_ERR_INVALID
