"""stem_attention_host: the whole path from host buffers, one group of kv-heads at a time,
each group's copies overlapping the other groups' work.  Every head's arithmetic is
independent of the other heads, so the output, the log-sum-exp and the selection equal
stem_attention's bit for bit, for contiguous and paged caches, BF16 and FP8, per-head and
shared lists, and any number of groups (G = 1, 2, 4 below; an odd number of q-heads per
group in the ragged case; the first and last groups in two halves where they hold one
kv-head and a multiple of 4 q-heads)."""
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu

CASES = {
    "fp8_gqa_s4096": W.LONG_128K_FP8.with_(name="host_fp8", seqlens=(4096,), num_q_heads=8, num_kv_heads=4, seed=61),
    "bf16_shared_lists": W.QWEN_32K.with_(name="host_shared", seqlens=(2048, 1000), num_q_heads=8, num_kv_heads=2,
                                         shared_lists=True, seed=64),
    "bf16_ragged_varlen": W.QWEN_32K.with_(name="host_bf16", seqlens=(300, 2112, 1024), num_q_heads=6,
                                          num_kv_heads=2, seed=62),
    "bf16_paged_varlen": W.PAGED_VARLEN.with_(name="host_paged", seqlens=(2048, 640, 4096), num_q_heads=4,
                                             num_kv_heads=2, seed=63),
    # one kv-head and 4 q-heads per group: the first and last groups run in two halves
    "bf16_halves": W.QWEN_32K.with_(name="host_halves", seqlens=(2048, 700), num_q_heads=16, num_kv_heads=4,
                                    seed=65),
    "fp8_halves": W.LONG_128K_FP8.with_(name="host_fp8_halves", seqlens=(3000,), num_q_heads=8, num_kv_heads=2,
                                        seed=66),
    "paged_halves": W.PAGED_VARLEN.with_(name="host_paged_halves", seqlens=(1500, 4096), num_q_heads=8,
                                         num_kv_heads=2, seed=67),
}

_cache = {}


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


def _setup(name):
    if name not in _cache:
        inp = W.make_inputs(CASES[name])
        prob = S.problem_for(inp.wl, inp)
        dev = T.to_device(inp)
        sz = prob.sizes()
        ref_rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
        ref_ci = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
        ref_lse = torch.empty((inp.wl.num_q_heads, sz["total_tokens"]), dtype=torch.float32, device="cuda")
        ws = S.workspace(prob)
        ref = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], dev["paged"], lse=ref_lse, row_ptr=ref_rp,
                               col_idx=ref_ci, ws=ws)
        S.query_status(ws)
        _cache[name] = (inp, prob, dev, ref.cpu(), ref_lse.cpu(), ref_rp.cpu(), ref_ci.cpu())
    return _cache[name]


@pytest.mark.parametrize("groups", [0, 1, 2, 3, 100])
@pytest.mark.parametrize("name", list(CASES))
def test_host_entry_equals_device_entry(name, groups):
    inp, prob, dev, ref, ref_lse, ref_rp, ref_ci = _setup(name)
    paged = dev["paged"]
    if paged is None:
        k_host, v_host = inp.k.pin_memory(), inp.v.pin_memory()
        k, v = torch.empty_like(dev["k"]), torch.empty_like(dev["v"])
        pg = None
    else:
        # the call fills the device caches from the host ones
        k_host, v_host = inp.k_cache.pin_memory(), inp.v_cache.pin_memory()
        k = v = None
        pg = S.PagedKV(torch.zeros_like(paged.k_cache), torch.zeros_like(paged.v_cache), paged.block_table)
    q_host = inp.q.pin_memory()
    q = torch.empty_like(dev["q"])
    out = torch.full_like(ref.cuda(), float("nan"))
    out_host = torch.full(tuple(ref.shape), float("nan"), dtype=torch.bfloat16).pin_memory()
    sz = prob.sizes()
    rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
    lse = torch.empty((inp.wl.num_q_heads, sz["total_tokens"]), dtype=torch.float32, device="cuda")
    ws = S.workspace(prob)
    got = S.stem_attention_host(prob, q_host, k_host, v_host, q, k, v, pg, out_host=out_host, out=out, lse=lse,
                                row_ptr=rp, col_idx=ci, out_groups=groups, ws=ws)
    S.query_status(ws)   # synchronises the stream the copies joined
    assert got.data_ptr() == out_host.data_ptr()
    assert torch.equal(out_host.view(torch.int16), ref.view(torch.int16))
    # the device buffer holds O staged group by group: group g's q-heads contiguous, and a
    # group run in two halves (the first and last, with one kv-head and a multiple of 4
    # q-heads per group, two or more groups, per-head lists) its halves one after the other
    wl = inp.wl
    G = max(c for c in range(1, wl.num_kv_heads + 1) if wl.num_kv_heads % c == 0 and c <= (groups or 8))
    hg = wl.num_q_heads // G
    halves = G >= 2 and wl.num_kv_heads // G == 1 and not wl.shared_lists and hg % 4 == 0
    pieces = []
    for g in range(G):
        parts = 2 if halves and g in (0, G - 1) else 1
        for p_ in range(parts):
            h0 = g * hg + p_ * hg // parts
            pieces.append(ref[:, h0:h0 + hg // parts].contiguous().flatten())
    staged = torch.cat(pieces)
    assert torch.equal(out.cpu().flatten().view(torch.int16), staged.view(torch.int16))
    assert torch.equal(lse.cpu(), ref_lse)
    assert torch.equal(rp.cpu(), ref_rp) and torch.equal(ci.cpu(), ref_ci)
