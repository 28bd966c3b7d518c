"""The fused front (stem_score_select: scores computed inside the budgeted top-k straight
from the pooled block summaries, no score matrix) against the two-launch path through the
score matrix (stem_score -> stem_select), which the oracle parity tests pin: the selections
must be identical bit for bit, since both compute every score with the same float32
operations in the same order.  Also: the fused front leaves the workspace's score region
untouched, and attention over its lists equals stem_attention (which runs the two-launch
front) bit for bit."""
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from tests import stem_testlib as T
from tests.test_gpu_parity import SMALL

pytestmark = pytest.mark.gpu

CASES = dict(SMALL)
CASES.update({
    "gqa_shared": SMALL["gqa_s4096"].with_(name="gqa_shared", shared_lists=True),
    "paged_shared": SMALL["paged_varlen"].with_(name="paged_shared", shared_lists=True),
    "fp8_shared": SMALL["fp8_s4096"].with_(name="fp8_shared", shared_lists=True),
    "keep_one": SMALL["gqa_s4096"].with_(name="keep_one", keep=1.0),
    "keep_tiny": SMALL["gqa_s4096"].with_(name="keep_tiny", keep=0.02),
    "uniform_mu": SMALL["ragged_varlen"].with_(name="uniform_mu", mu=1.0),
    "beta_zero": SMALL["ragged_varlen"].with_(name="beta_zero", beta=0.0),
    "g8_per_head": W.QWEN_32K.with_(name="g8_per_head", seqlens=(3000,), num_q_heads=16, num_kv_heads=2, seed=61),
    "g8_shared": W.QWEN_32K.with_(name="g8_shared", seqlens=(3000,), num_q_heads=16, num_kv_heads=2, seed=61,
                                  shared_lists=True),
    "g6_per_head": W.QWEN_32K.with_(name="g6_per_head", seqlens=(2200,), num_q_heads=6, num_kv_heads=1, seed=62),
})

_cache = {}


def inputs(name):
    if name not in _cache:
        _cache[name] = W.make_inputs(CASES[name])
    return _cache[name]


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    torch.cuda.synchronize()


def _two_launch(prob, dev, ws):
    scores = S.stem_score(prob, dev["q"], dev["k"], dev["v"], dev["paged"], ws=ws)
    return S.stem_select(prob, scores, ws=ws)


@pytest.mark.parametrize("name", list(CASES))
def test_fused_front_selection_equals_the_score_matrix_path(name):
    inp = inputs(name)
    prob = S.problem_for(inp.wl, inp)
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    rp0, ci0 = _two_launch(prob, dev, ws)
    rp1, ci1 = S.stem_score_select(prob, dev["q"], dev["k"], dev["v"], dev["paged"], ws=ws)
    assert S.query_status(ws) == S.STEM_OK
    assert torch.equal(rp1, rp0)
    assert torch.equal(ci1, ci0), f"{int((ci1 != ci0).sum())} list entries differ"


@pytest.mark.parametrize("name", ["gqa_s4096", "fp8_s4096", "paged_varlen", "gqa_shared", "d128_b64"])
def test_fused_front_leaves_the_score_matrix_untouched_and_feeds_the_same_attention(name):
    inp = inputs(name)
    prob = S.problem_for(inp.wl, inp)
    sz = prob.sizes()
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    rp0, ci0 = _two_launch(prob, dev, ws)
    ref = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], dev["paged"], ws=ws)
    S.query_status(ws)
    ws.fill_(0xFF)                                  # every byte the call does not write stays 0xFF
    ws[:256].zero_()                                # the status word
    rp, ci = S.stem_score_select(prob, dev["q"], dev["k"], dev["v"], dev["paged"], ws=ws)
    out = S.bsa_prefill(prob, dev["q"], dev["k"], dev["v"], rp, ci, dev["paged"], ws=ws)
    assert S.query_status(ws) == S.STEM_OK
    assert torch.equal(rp, rp0) and torch.equal(ci, ci0)
    assert torch.equal(out, ref)
    # the score matrix region (Hq x scores_per_head floats) is one untouched run of 0xFF bytes
    score_bytes = prob.num_q_heads * sz["scores_per_head"] * 4
    untouched = (ws == 0xFF).to(torch.int32)
    run = torch.cumsum(untouched, 0)
    starts = torch.nonzero(torch.diff(untouched, prepend=torch.zeros(1, dtype=torch.int32, device=ws.device)) == 1)
    ends = torch.nonzero(torch.diff(untouched, append=torch.zeros(1, dtype=torch.int32, device=ws.device)) == -1)
    longest = int((run[ends[:, 0]] - run[starts[:, 0]] + 1).max()) if len(starts) else 0
    assert longest >= score_bytes, f"longest untouched run {longest} < score matrix {score_bytes} bytes"
