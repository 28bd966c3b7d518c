"""stem_attention_noalloc: the whole prefill path for callers that cannot
allocate device memory (a plugin host whose framework owns the GPU's memory, a
serving loop that must not allocate while running).  Its scratch is a fixed
array inside the library, so the only buffers the caller passes are its inputs
and outputs.  It must give the same result as stem_attention with a caller
workspace, call after call, and refuse problems too large for the array.

This file is named to be collected last, so a failure here never hides the
result of another test."""
import numpy as np
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu

CASES = {
    "gqa_s4096": W.QWEN_32K.with_(name="gqa_s4096", seqlens=(4096,), num_q_heads=8, num_kv_heads=2, seed=21),
    "paged_varlen": W.PAGED_VARLEN.with_(name="paged_varlen", seqlens=(1024, 300, 2112), num_q_heads=8,
                                         num_kv_heads=2, seed=22),
    "fp8_s2048": W.LONG_128K_FP8.with_(name="fp8_s2048", seqlens=(2048,), num_q_heads=4, num_kv_heads=1, seed=23),
}


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_workspace_entry_point_twice(name):
    """Same kernels on the same inputs as stem_attention: the outputs and the selection
    are bit-identical, call after call, and a call after the first allocates nothing
    (neither torch's allocator nor the device's free memory moves)."""
    wl = CASES[name]
    inp = W.make_inputs(wl)
    prob = S.problem_for(wl, inp)
    sz = prob.sizes()
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    rp_ref = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
    ci_ref = torch.empty((wl.num_q_heads, sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
    ref = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], dev["paged"], row_ptr=rp_ref, col_idx=ci_ref, ws=ws)
    S.query_status(ws)
    rp = torch.full_like(rp_ref, -1)
    ci = torch.full_like(ci_ref, -1)
    out = torch.empty_like(ref)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        rp.fill_(-1)
        ci.fill_(-1)
        out.zero_()
        status.fill_(-1)
        torch.cuda.synchronize()
        free0, alloc0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        S.stem_attention_noalloc(prob, dev["q"], dev["k"], dev["v"], dev["paged"], out=out, row_ptr=rp, col_idx=ci,
                                 status=status)
        torch.cuda.synchronize()
        free1, alloc1 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        if call > 0:   # the first call on a device may load the library's kernels
            assert alloc1 == alloc0, f"call {call}: torch allocated {alloc1 - alloc0} bytes"
            assert free1 == free0, f"call {call}: device free memory moved by {free0 - free1} bytes"
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item())}"
        assert torch.equal(rp, rp_ref) and torch.equal(ci, ci_ref), f"call {call}: selection differs"
        assert torch.equal(out, ref), f"call {call}: output differs from stem_attention's"


def test_noalloc_refuses_problems_larger_than_its_scratch():
    wl = W.LONG_128K_FP8                       # needs about 105 MB of scratch
    prob = S.problem_for(wl)
    assert prob.sizes()["workspace_bytes"] > 32 << 20
    q = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(S.StemError) as e:
        S.stem_attention_noalloc(prob, q, q, q, out=q)
    assert e.value.status == S.STEM_ERR_WORKSPACE
    assert "static scratch" in str(e.value)
