"""One layer split across ranks by KV-head group (every step of the path stays inside a
(kv-head, its q-heads) group), then one all-gather of the output heads.  On two and four
gloo ranks on the CPU: each rank runs the float64 oracle on its shard of a GQA workload
(the path's arithmetic, on the CPU), the gathered heads in the one-GPU layout equal the
whole problem's output and selection, and the head partition is validated."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from block_sparse_attention_oam_b200 import sharding as SH  # noqa: E402
from block_sparse_attention_oam_b200 import workloads as W  # noqa: E402

WL = W.QWEN_32K.with_(name="gqa_s640", seqlens=(640, 384), num_q_heads=8, num_kv_heads=4, seed=31)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_layer(inp):
    """Oracle output [T, Hq, d] and per-sequence lists of a workload's inputs."""
    from oracle import stem_oracle as O
    wl = inp.wl
    outs, lists = [], []
    for b in range(len(wl.seqlens)):
        t0, t1 = int(inp.cu_seqlens[b]), int(inp.cu_seqlens[b + 1])
        res = O.stem_sequence(inp.dequant("q")[t0:t1], inp.dequant("k")[t0:t1], inp.dequant("v")[t0:t1], wl.block,
                              wl.keep, wl.mu, wl.beta, wl.softmax_scale)
        outs.append(res["out"])
        lists.append(res["lists"])
    return np.concatenate(outs, axis=0), lists


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = W.make_inputs(WL)                      # every rank draws the same layer
        sh = SH.head_shard(WL.num_q_heads, WL.num_kv_heads, world, rank)
        part = SH.shard_inputs(inp, sh)
        out, lists = _oracle_layer(part)
        gathered = SH.gather_heads(torch.from_numpy(out), dist)
        got_lists = [None] * world
        dist.all_gather_object(got_lists, lists)
        if rank == 0:
            q.put(("ok", SH.token_major(gathered).numpy(), got_lists))
    except Exception as e:  # noqa: BLE001 - reported to the test
        q.put(("error", repr(e), None))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def _run(world, timeout=300):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = q.get(timeout=timeout)
    for p in procs:
        p.join(timeout)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    return res


@pytest.mark.parametrize("world", [2, 4])
def test_sharded_layer_gathers_to_the_one_gpu_result(world):
    status, out, got_lists = _run(world)
    assert status == "ok", out
    full_out, full_lists = _oracle_layer(W.make_inputs(WL))
    assert out.shape == full_out.shape
    assert np.array_equal(out, full_out)            # heads are independent: bit-identical
    kpr = WL.num_kv_heads // world
    g = WL.num_q_heads // WL.num_kv_heads
    for r in range(world):
        for b in range(len(WL.seqlens)):
            for hl in range(kpr * g):
                assert got_lists[r][b][hl] == full_lists[b][r * kpr * g + hl]


def test_head_shard_partition():
    parts = [SH.head_shard(32, 8, 4, r) for r in range(4)]
    assert [(p.q0, p.q1, p.k0, p.k1) for p in parts] == [(0, 8, 0, 2), (8, 16, 2, 4), (16, 24, 4, 6), (24, 32, 6, 8)]
    for p in parts:                                  # local q-head j reads local kv-head j // g = global h // g - k0
        for h in range(p.q0, p.q1):
            assert (h - p.q0) // 4 == h // 4 - p.k0
    assert SH.head_shard(32, 8, 1, 0) == SH.HeadShard(0, 1, 0, 32, 0, 8)
    with pytest.raises(ValueError):
        SH.head_shard(32, 8, 3, 0)                   # 8 kv-heads do not split over 3 ranks
    with pytest.raises(ValueError):
        SH.head_shard(32, 8, 2, 2)


def test_shard_inputs_slices_heads_and_pages():
    wl = W.PAGED_VARLEN.with_(name="paged_small", seqlens=(300, 200), num_q_heads=8, num_kv_heads=4, seed=32)
    inp = W.make_inputs(wl)
    sh = SH.head_shard(8, 4, 2, 1)
    part = SH.shard_inputs(inp, sh)
    assert part.wl.num_q_heads == 4 and part.wl.num_kv_heads == 2
    assert torch.equal(part.q, inp.q[:, 4:8]) and part.q.is_contiguous()
    assert torch.equal(part.k, inp.k[:, 2:4]) and torch.equal(part.v, inp.v[:, 2:4])
    assert torch.equal(part.k_cache, inp.k_cache[:, :, 2:4]) and torch.equal(part.v_cache, inp.v_cache[:, :, 2:4])
    assert part.block_table is inp.block_table
