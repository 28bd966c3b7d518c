"""The kv-head split of one layer (bench.py under torchrun) on one GPU: every rank's share
of the heads, run through stem_attention as a problem of its own, gives exactly the
whole problem's output heads, log-sum-exp and lists (every step of the path stays inside
a kv-head group), for BF16, FP8 (whose per-tensor scales stay the whole tensors') and a
paged cache, and the head-major gather lays them out as the one-GPU output."""
import pytest
import torch

from block_sparse_attention_oam_b200 import sharding as SH
from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu

CASES = {
    "bf16": W.QWEN_32K.with_(name="shard_bf16", seqlens=(2048, 700), num_q_heads=16, num_kv_heads=4, seed=81),
    "fp8": W.LONG_128K_FP8.with_(name="shard_fp8", seqlens=(3000,), num_q_heads=16, num_kv_heads=4, seed=82),
    "paged": W.PAGED_VARLEN.with_(name="shard_paged", seqlens=(1500, 640), num_q_heads=8, num_kv_heads=4, seed=83),
}


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


def _run(inp):
    prob = S.problem_for(inp.wl, inp)
    sz = prob.sizes()
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
    lse = torch.empty((inp.wl.num_q_heads, sz["total_tokens"]), dtype=torch.float32, device="cuda")
    out = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], dev["paged"], lse=lse, row_ptr=rp, col_idx=ci, ws=ws)
    assert S.query_status(ws) == S.STEM_OK
    return out, lse, rp, ci


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("name", list(CASES))
def test_shards_reproduce_the_whole_layer(name, world):
    wl = CASES[name]
    inp = W.make_inputs(wl)
    out, lse, rp, ci = _run(inp)
    parts = []
    for r in range(world):
        sh = SH.head_shard(wl.num_q_heads, wl.num_kv_heads, world, r)
        o, l, rp_r, ci_r = _run(SH.shard_inputs(inp, sh))
        assert torch.equal(o, out[:, sh.q0:sh.q1])
        assert torch.equal(l, lse[sh.q0:sh.q1])
        assert torch.equal(rp_r, rp) and torch.equal(ci_r, ci[sh.q0:sh.q1])
        parts.append(o)
    gathered = torch.stack(parts)                    # what all_gather_into_tensor assembles, rank-major
    assert torch.equal(SH.token_major(gathered), out)
