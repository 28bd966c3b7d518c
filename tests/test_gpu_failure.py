"""Failure detection on the GPU without a fault: a withheld K tile makes one CTA's
bounded pipeline wait run out; the kernel reports STEM_ERR_TIMEOUT through the
workspace status word, releases its resources, and the next call succeeds."""
import pytest
import torch

from block_sparse_attention_oam_b200 import stem as S
from block_sparse_attention_oam_b200 import workloads as W
from tests import stem_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    yield
    S.debug_inject(0)
    torch.cuda.synchronize()


def test_stalled_pipeline_reports_timeout_and_gpu_stays_usable():
    wl = W.QWEN_32K.with_(name="stall", seqlens=(2048,), num_q_heads=4, num_kv_heads=2, seed=41)
    inp = W.make_inputs(wl)
    prob = S.problem_for(wl, inp)
    dev = T.to_device(inp)
    ws = S.workspace(prob)
    S.debug_inject(1)
    S.stem_attention(prob, dev["q"], dev["k"], dev["v"], ws=ws)
    with pytest.raises(S.StemError) as e:
        S.query_status(ws)
    assert e.value.status == S.STEM_ERR_TIMEOUT
    # the request was consumed: the next call runs normally and matches a clean run
    out = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], ws=ws)
    assert S.query_status(ws) == S.STEM_OK
    ws2 = S.workspace(prob)
    ref = S.stem_attention(prob, dev["q"], dev["k"], dev["v"], ws=ws2)
    assert S.query_status(ws2) == S.STEM_OK
    assert torch.equal(out, ref)
    assert torch.isfinite(out.float()).all()


def test_injection_mode_validation():
    with pytest.raises(S.StemError):
        S.debug_inject(7)
