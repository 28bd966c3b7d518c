"""Canary guards around every buffer the path writes (a check that stands in for a memory
sanitizer): each output, selection, score and workspace buffer is carved out of a larger
allocation whose 4 KiB before and after hold a sentinel pattern; after each entry point
runs, the sentinels must be intact and the read-only inputs unchanged.  The workloads
cover ragged tails, varlen batches, paging, FP8, d = 64, block 64 and a single head pair."""
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes of sentinel on each side (keeps the payload 256-byte aligned)
SENTINEL = 0xA5

CASES = {
    "ragged_varlen": W.QWEN_32K.with_(name="ragged_varlen", seqlens=(300, 1024, 2112, 77), num_q_heads=4,
                                      num_kv_heads=2, seed=71),
    "paged_varlen": W.PAGED_VARLEN.with_(name="paged_varlen", seqlens=(1024, 300, 2112), num_q_heads=8,
                                         num_kv_heads=2, seed=72),
    "fp8_ragged": W.LONG_128K_FP8.with_(name="fp8_ragged", seqlens=(2000, 130), num_q_heads=8, num_kv_heads=2,
                                        seed=73),
    "d64_b64_shared": W.QWEN_32K.with_(name="d64_b64_shared", seqlens=(1000, 64, 1), num_q_heads=4,
                                       num_kv_heads=2, head_dim=64, block=64, shared_lists=True, seed=74),
    # one head pair, more q-block rows than SMs: the attention launch deals its units
    # forwards and back (an odd number of groups)
    "single_pair": W.QWEN_32K.with_(name="single_pair", seqlens=(12000,), num_q_heads=2, num_kv_heads=1,
                                    block=64, seed=75),
}


class Guarded:
    """A device (or pinned host) buffer of `shape` and `dtype` between two sentinel guards."""

    def __init__(self, shape, dtype, device="cuda", pinned=False):
        n = 1
        for x in shape:
            n *= x
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        body = (nbytes + 255) // 256 * 256
        self.raw = torch.full((GUARD + body + GUARD,), SENTINEL, dtype=torch.uint8, device=device)
        if pinned:
            self.raw = self.raw.pin_memory()
        self.nbytes = nbytes
        self.t = self.raw[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def intact(self):
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.nbytes:]
        return bool((head == SENTINEL).all()) and bool((tail == SENTINEL).all())


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


def _setup(name):
    wl = CASES[name]
    inp = W.make_inputs(wl)
    prob = S.problem_for(wl, inp)
    sz = prob.sizes()
    dev = T.to_device(inp)
    snap = {k: v.clone() for k, v in dev.items() if isinstance(v, torch.Tensor)}
    if dev["paged"] is not None:
        snap["k_cache"] = dev["paged"].k_cache.clone()
        snap["v_cache"] = dev["paged"].v_cache.clone()
        snap["block_table"] = dev["paged"].block_table.clone()
    return wl, inp, prob, sz, dev, snap


def _inputs_unchanged(dev, snap):
    for k in ("q", "k", "v"):
        assert torch.equal(dev[k], snap[k]), f"input {k} was written"
    if dev["paged"] is not None:
        assert torch.equal(dev["paged"].k_cache, snap["k_cache"])
        assert torch.equal(dev["paged"].v_cache, snap["v_cache"])
        assert torch.equal(dev["paged"].block_table, snap["block_table"])


@pytest.mark.parametrize("name", list(CASES))
def test_device_entry_points_write_only_their_buffers(name):
    wl, inp, prob, sz, dev, snap = _setup(name)
    T_, Hq, d = sz["total_tokens"], wl.num_q_heads, wl.head_dim
    ws = Guarded((sz["workspace_bytes"],), torch.uint8)
    ws.t.zero_()
    scores = Guarded((Hq, sz["scores_per_head"]), torch.float32)
    rp = Guarded((sz["num_rows"] + 1,), torch.int32)
    ci = Guarded((sz["list_heads"], sz["nnz_per_head"]), torch.int32)
    out = Guarded((T_, Hq, d), torch.bfloat16)
    lse = Guarded((Hq, T_), torch.float32)
    S.stem_score(prob, dev["q"], dev["k"], dev["v"], dev["paged"], scores=scores.t, ws=ws.t)
    S.stem_select(prob, scores.t, rp.t, ci.t, ws=ws.t)
    S.stem_score_select(prob, dev["q"], dev["k"], dev["v"], dev["paged"], rp.t, ci.t, ws=ws.t)
    S.bsa_prefill(prob, dev["q"], dev["k"], dev["v"], rp.t, ci.t, dev["paged"], out=out.t, lse=lse.t, ws=ws.t)
    S.bsa_dense_prefill(prob, dev["q"], dev["k"], dev["v"], dev["paged"], out=out.t, lse=lse.t, ws=ws.t)
    S.stem_attention(prob, dev["q"], dev["k"], dev["v"], dev["paged"], out=out.t, lse=lse.t, row_ptr=rp.t,
                     col_idx=ci.t, ws=ws.t)
    assert S.query_status(ws.t) == S.STEM_OK
    for nm, g in (("workspace", ws), ("scores", scores), ("row_ptr", rp), ("col_idx", ci), ("out", out),
                  ("lse", lse)):
        assert g.intact(), f"{nm}: a guard byte changed"
    _inputs_unchanged(dev, snap)
    assert torch.isfinite(out.t.float()).all()


@pytest.mark.parametrize("name", ["ragged_varlen", "paged_varlen", "fp8_ragged"])
def test_host_entry_writes_only_its_buffers(name):
    """stem_attention_host overwrites its device staging buffers (documented) and its host
    output, nothing around them; its host inputs stay as they were."""
    wl, inp, prob, sz, dev, snap = _setup(name)
    T_, Hq, d = sz["total_tokens"], wl.num_q_heads, wl.head_dim
    hq = inp.q.pin_memory()
    hk = (inp.k_cache if wl.paged else inp.k).pin_memory()
    hv = (inp.v_cache if wl.paged else inp.v).pin_memory()
    hq0, hk0, hv0 = hq.clone(), hk.clone(), hv.clone()
    ws = Guarded((sz["workspace_bytes"],), torch.uint8)
    ws.t.zero_()
    qd = Guarded(tuple(hq.shape), hq.dtype)
    kd = Guarded(tuple(hk.shape), hk.dtype)
    vd = Guarded(tuple(hv.shape), hv.dtype)
    out = Guarded((T_, Hq, d), torch.bfloat16)
    hout = Guarded((T_, Hq, d), torch.bfloat16, device="cpu", pinned=True)
    paged = None
    if wl.paged:
        paged = S.PagedKV(kd.t, vd.t, dev["paged"].block_table)
    S.stem_attention_host(prob, hq, hk, hv, qd.t, kd.t, vd.t, paged, out_host=hout.t, out=out.t, ws=ws.t)
    torch.cuda.synchronize()
    assert S.query_status(ws.t) == S.STEM_OK
    for nm, g in (("workspace", ws), ("q staging", qd), ("k staging", kd), ("v staging", vd), ("out", out),
                  ("host out", hout)):
        assert g.intact(), f"{nm}: a guard byte changed"
    assert torch.equal(hq, hq0) and torch.equal(hk, hk0) and torch.equal(hv, hv0)
    ref = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], dev["paged"])
    assert torch.equal(hout.t, ref.cpu())
