"""Benchmark of the Stem sparse-attention prefill path on B200.

One step = one pass of the whole hot path over one layer's synthetic inputs, exactly
what stem_attention runs: stem_score (Q/K/V pooled in one launch, then the block-score
GEMM) -> stem_select (budget + top-k) -> bsa_prefill, inputs resident in HBM.  The fused
operator stem_score_select is timed beside it.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: one Qwen3-8B-shaped layer at 128K tokens in FP8-e4m3, keep 25% (the
headline).  The same line also carries a record per other workload of the suite (the
1024-token tiny case, the 32K BF16 layer, the 64K BF16 layer with its density sweep and
the paged varlen batch), unless --no-extra.

With N > 1 (torchrun) the layer is split by KV-head group: rank r runs the path on
kv-heads [r*Hkv/N, (r+1)*Hkv/N) and their q-heads, then one NCCL all-gather collects the
output heads; the step time (gather included) is the max over ranks, and the value is
the time of that one layer (strong scaling).
"""
from __future__ import annotations

import argparse
import copy
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_oam_b200 import sharding as SH     # noqa: E402
from block_sparse_attention_oam_b200 import stem as S          # noqa: E402
from block_sparse_attention_oam_b200 import workloads as W     # noqa: E402

METRIC = "Stem prefill ms/layer at 128K, 25% budget; effective TFLOP/s vs B200 peak"
BF16_DATASHEET_TFLOPS = 2250.0
FP8_DATASHEET_TFLOPS = 4500.0
FP8_OVER_BF16 = 2.0          # nominal dense FP8 / BF16 tensor throughput ratio
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DENSE_LAUNCHES = 5           # timed launches of the dense comparator (after one untimed)
CPU_SAMPLE_BLOCKS = 64       # q-blocks of head 0 the oracle attends in a CPU sample
L2_BYTES = 126 << 20
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one bsa_kernel launch,
# from an ncu capture of that launch on the named workload.  A figure holds only for the
# kernel source and the input generator it was taken on: KERNEL_SOURCES are hashed and
# compared, and a stale figure reports null.
KERNEL_SOURCES = ("block_sparse_attention_oam_b200/csrc/stem_bsa.cu", "block_sparse_attention_oam_b200/csrc/stem_internal.cuh",
                  "block_sparse_attention_oam_b200/workloads.py")
MEASURED_TRAFFIC = {
    # (workload, keep, mu, beta): (bytes per launch, sha256 of KERNEL_SOURCES)
    ("qwen3_8b_layer_s128k_fp8", 0.25, 0.7, 0.2): (2.135398400e+09, "7ff6c04c831ac2d39aa79a018dff8a0044ecd1af6603009b8a3c7cd10daccc03"),
    ("qwen3_8b_layer_s64k_bf16", 0.25, 0.7, 0.2): (1.408879872e+09, "7ff6c04c831ac2d39aa79a018dff8a0044ecd1af6603009b8a3c7cd10daccc03"),
}


def kernel_sha256() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(wl) -> float | None:
    """Bytes per bsa_kernel launch measured on this workload with the current kernel source,
    else None (another workload, or the kernel changed since the counters were taken)."""
    rec = None if wl.shared_lists else MEASURED_TRAFFIC.get((wl.name, wl.keep, wl.mu, wl.beta))
    if rec is None or rec[1] != kernel_sha256():
        return None
    return rec[0]


def max_over_ranks(ms: float, dist, device="cuda") -> float:
    """The slowest rank's time (every rank gets it); `dist` None on one GPU."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK, "fallback"


def selected_flops(prob: S.Problem, row_ptr: np.ndarray, block: int, head_dim: int, seqlens) -> float:
    """Algorithmic FLOPs of the listed blocks: QK^T and PV over B x B tiles (2 x 2B^2 d),
    the diagonal block counted as its causal half; ragged tails counted by valid tokens."""
    flops = 0.0
    row0 = 0
    for S_ in seqlens:
        N = math.ceil(S_ / block)
        k = np.diff(row_ptr[row0: row0 + N + 1]).astype(np.float64)
        rows = np.minimum(block, S_ - np.arange(N) * block).astype(np.float64)
        # off-diagonal blocks: rows x block keys (the last block may be ragged only on the diagonal)
        flops += float(np.sum((k - 1) * rows * block) * 4 * head_dim)
        flops += float(np.sum(rows * (rows + 1) / 2) * 4 * head_dim)
        row0 += N
    return flops * prob.num_q_heads


def dense_flops(seqlens, num_q_heads, head_dim):
    return float(sum(s * (s + 1) / 2 for s in seqlens)) * 4 * head_dim * num_q_heads


class Clocks:
    """nvidia-smi sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit()) if rows else None,
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ the oracle on the CPU
def cpu_sample(inp: W.Inputs, n_blocks: int = CPU_SAMPLE_BLOCKS):
    """Time the float64 oracle (as it stands) on a fixed, bounded sample of the workload on
    the host cores and extrapolate to ms per layer: pool + score + plan + select for q-head 0
    over all rows (scaled by the head count), attention for the first `n_blocks` q-blocks of
    a seeded permutation of head 0's rows (scaled by selected blocks to every head and row).
    The sample is the same every time, so the GPU arm's cpu_baseline and the reference arm
    time the same work."""
    from oracle import stem_oracle as O
    from threadpoolctl import threadpool_info
    wl = inp.wl
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    h = 0
    g = wl.num_q_heads // wl.num_kv_heads
    t_sel = t_att = 0.0
    blocks_done = blocks_total = rows_done = 0
    cu = inp.cu_seqlens
    per_seq = max(1, n_blocks // len(wl.seqlens))
    wall0 = time.perf_counter()
    for b, S_ in enumerate(wl.seqlens):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        N = math.ceil(S_ / wl.block)
        q = inp.q[t0:t1, [h]].float().numpy().astype(np.float64) * inp.q_scale
        k = inp.k[t0:t1, [h // g]].float().numpy().astype(np.float64) * inp.k_scale
        v = inp.v[t0:t1, [h // g]].float().numpy().astype(np.float64) * inp.v_scale
        c0 = time.perf_counter()
        qbar, kbar, lbar = O.pool_mean(q, wl.block), O.pool_mean(k, wl.block), O.pool_log_norm(v, wl.block)
        s = O.oam_scores(qbar, kbar, lbar, wl.softmax_scale, wl.beta)
        kk = O.tpd_plan(N, wl.keep, wl.mu)[2]
        lists = O.select_all(s, kk)
        t_sel += (time.perf_counter() - c0) * wl.num_q_heads
        blocks_total += int(np.sum(kk)) * wl.num_q_heads
        order = np.random.default_rng(1000 + b).permutation(N)[:per_seq]
        c0 = time.perf_counter()
        for i in order:
            O.attend(q, k, v, lists, wl.block, wl.softmax_scale, rows=[(0, int(i))])
            blocks_done += len(lists[0][i])
            rows_done += 1
        t_att += time.perf_counter() - c0
    wall = time.perf_counter() - wall0
    ms = (t_sel + t_att * blocks_total / max(1, blocks_done)) * 1e3
    return {"value": ms, "unit": "ms/layer", "cores": threads, "kind": "oracle", "extrapolated": True,
            "sample_wall_ms": wall * 1e3,
            "sample": f"float64 oracle on q-head 0: pool+score+select over all rows (x{wl.num_q_heads} heads), "
                      f"attention on {rows_done} seeded q-blocks ({blocks_done} of {blocks_total} selected "
                      f"blocks), extrapolated by selected blocks"}


def run_reference(args, wl):
    """Reference arm: the oracle itself, timed as it stands on the host cores; each step is
    the fixed sample of cpu_sample (the GPU arm's cpu_baseline times the same sample)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = W.make_inputs(wl)
    vals = [cpu_sample(inp) for _ in range(args.warmup + args.steps)]
    timed = vals[args.warmup:]
    v = statistics.mean(x["value"] for x in timed)
    wall = statistics.mean(x["sample_wall_ms"] for x in timed)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "ms/layer", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall, "higher_is_better": False,
            "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "extrapolated": True,
            "extrapolation": "value: one layer's time extrapolated from each step's bounded sample; "
                             "ms_per_step: the sample's own wall time",
            "config": {"workload": wl.name, "seq_len": list(wl.seqlens), "keep": wl.keep, "block": wl.block,
                       "heads": [wl.num_q_heads, wl.num_kv_heads], "head_dim": wl.head_dim},
            "cpu_baseline": {"value": v, "unit": "ms/layer", "cores": timed[-1]["cores"], "kind": "oracle",
                             "extrapolated": True, "sample": timed[-1]["sample"]},
            "e2e": {"value": v, "unit": "ms/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the GPU arm
class Layer:
    """One workload's inputs on this rank's device (its heads' share under N > 1)."""

    def __init__(self, wl, rank=0, world=1):
        inp = W.make_inputs(wl)                      # every rank draws the same layer
        self.shard = SH.head_shard(wl.num_q_heads, wl.num_kv_heads, world, rank)
        if world > 1:
            inp = SH.shard_inputs(inp, self.shard)
        self.inp = inp
        self.wl = inp.wl
        self.prob = S.problem_for(self.wl, inp)
        sz = self.prob.sizes()
        self.sz = sz
        self.q, self.k, self.v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
        self.paged = None
        if self.wl.paged:
            self.paged = S.PagedKV(inp.k_cache.cuda(), inp.v_cache.cuda(), torch.from_numpy(inp.block_table).cuda())
        self.ws = S.workspace(self.prob)
        self.scores = torch.empty((self.wl.num_q_heads, sz["scores_per_head"]), dtype=torch.float32, device="cuda")
        self.rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
        self.ci = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
        self.out = torch.empty((sz["total_tokens"], self.wl.num_q_heads, self.wl.head_dim), dtype=torch.bfloat16,
                               device="cuda")

    def with_keep(self, keep):
        """The same inputs and buffers under another keep fraction (a new problem, workspace
        and selection)."""
        other = copy.copy(self)
        other.wl = self.wl.with_(keep=keep)
        other.prob = S.problem_for(other.wl, self.inp)
        other.sz = other.prob.sizes()
        other.ws = S.workspace(other.prob)
        other.ci = torch.empty((other.sz["list_heads"], other.sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
        return other

    def front(self):
        S.stem_score(self.prob, self.q, self.k, self.v, self.paged, scores=self.scores, ws=self.ws)
        S.stem_select(self.prob, self.scores, self.rp, self.ci, ws=self.ws)

    def bsa(self):
        S.bsa_prefill(self.prob, self.q, self.k, self.v, self.rp, self.ci, self.paged, out=self.out, ws=self.ws)


def _events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def time_dense(layer, dist):
    """The dense causal kernel on the same inputs: one untimed launch, then DENSE_LAUNCHES
    launches each between CUDA events; the mean, max over ranks."""
    stream = torch.cuda.current_stream()
    S.bsa_dense_prefill(layer.prob, layer.q, layer.k, layer.v, layer.paged, out=layer.out, ws=layer.ws)
    ev = [_events(2) for _ in range(DENSE_LAUNCHES)]
    for a, b in ev:
        a.record(stream)
        S.bsa_dense_prefill(layer.prob, layer.q, layer.k, layer.v, layer.paged, out=layer.out, ws=layer.ws)
        b.record(stream)
    torch.cuda.synchronize()
    S.query_status(layer.ws)
    return max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in ev), dist)


def measure(layer, steps, warmup, dist=None, with_clocks=False):
    """Warm-up, then `steps` timed steps bracketed by a barrier and synchronisations, with
    CUDA events per stage on the launching stream.  Returns the record of this workload."""
    wl, prob = layer.wl, layer.prob
    world = 1 if dist is None else dist.get_world_size()
    stream = torch.cuda.current_stream()
    gathered = None
    if world > 1:
        gathered = torch.empty((world,) + tuple(layer.out.shape), dtype=layer.out.dtype, device="cuda")

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        S.stem_score(prob, layer.q, layer.k, layer.v, layer.paged, scores=layer.scores, ws=layer.ws)
        if ev is not None:
            ev[1].record(stream)
        S.stem_select(prob, layer.scores, layer.rp, layer.ci, ws=layer.ws)
        if ev is not None:
            ev[2].record(stream)
        layer.bsa()
        if ev is not None:
            ev[3].record(stream)
        if gathered is not None:
            SH.gather_heads(layer.out, dist, gathered)
            if ev is not None:
                ev[4].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    S.query_status(layer.ws)
    # inputs smaller than twice the L2 (126 MB): flush it before every timed step (writing a
    # 512 MB buffer, outside the step's events) and time the steps one by one
    in_bytes = sum(t.numel() * t.element_size() for t in (layer.q, layer.k, layer.v))
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda") if in_bytes < 2 * L2_BYTES else None
    evs = [_events(5) for _ in range(steps)]
    clocks = Clocks(torch.cuda.current_device()) if with_clocks else None
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.start()
    t_start, t_end = _events(2)
    t_start.record(stream)
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    if dist is not None:
        dist.barrier()
    S.query_status(layer.ws)
    last = 4 if gathered is not None else 3
    if flush is None:
        step_ms = max_over_ranks(t_start.elapsed_time(t_end) / steps, dist)
    else:
        step_ms = max_over_ranks(statistics.mean(e[0].elapsed_time(e[last]) for e in evs), dist)
    del flush
    st_score = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    st_select = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    st_bsa = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    stages = {"score": st_score, "select": st_select, "bsa": st_bsa}
    if gathered is not None:
        stages["gather"] = statistics.mean(e[3].elapsed_time(e[4]) for e in evs)

    # the fused operator (stem_score_select: scores inside the selection, no score
    # matrix) on the same inputs, for comparison; its lists must equal the step's
    rp2, ci2 = torch.empty_like(layer.rp), torch.empty_like(layer.ci)
    S.stem_score_select(prob, layer.q, layer.k, layer.v, layer.paged, rp2, ci2, ws=layer.ws)
    fev = [_events(2) for _ in range(3)]
    for a, b in fev:
        a.record(stream)
        S.stem_score_select(prob, layer.q, layer.k, layer.v, layer.paged, rp2, ci2, ws=layer.ws)
        b.record(stream)
    torch.cuda.synchronize()
    S.query_status(layer.ws)
    fused_ms = statistics.mean(a.elapsed_time(b) for a, b in fev)
    same = bool(torch.equal(rp2, layer.rp) and torch.equal(ci2, layer.ci))
    del rp2, ci2

    rp_h = layer.rp.cpu().numpy()
    fp8 = wl.dtype == "fp8_e4m3"
    flops_sel = selected_flops(prob, rp_h, wl.block, wl.head_dim, wl.seqlens)
    flops_dense = dense_flops(wl.seqlens, wl.num_q_heads, wl.head_dim)
    bsa_ms = max_over_ranks(st_bsa, dist)
    peaks, peak_src = measured_peaks()
    peak = peaks["bf16_tflops_sustained"] * (FP8_OVER_BF16 if fp8 else 1.0)
    # the layer's FLOPs: this rank's heads times the ranks (every rank has the same share)
    flops_sel_all, flops_dense_all = flops_sel * world, flops_dense * world
    achieved = flops_sel / (bsa_ms * 1e-3) / 1e12
    datasheet = FP8_DATASHEET_TFLOPS if fp8 else BF16_DATASHEET_TFLOPS
    rec = {
        "value": step_ms, "unit": "ms/layer", "steps": steps, "warmup": warmup, "ms_per_step": step_ms,
        "dtype": "e4m3" if fp8 else "bf16",
        "config": {"workload": wl.name if world == 1 else f"{wl.name} (heads {layer.shard.q0}..{layer.shard.q1 - 1} of "
                                                           f"{wl.num_q_heads * world} on rank {layer.shard.rank})",
                   "seq_len": list(wl.seqlens), "keep": wl.keep, "mu": wl.mu, "beta": wl.beta,
                   "shared_lists": wl.shared_lists, "block": wl.block,
                   "heads": [wl.num_q_heads * world, wl.num_kv_heads * world], "head_dim": wl.head_dim,
                   "paged": wl.paged, "l2": "inputs larger than L2 (no flush)" if in_bytes >= 2 * L2_BYTES
                   else "L2 flushed before every timed step (512 MB written outside the step's events)"},
        "stages_ms": stages,
        "score_select_frac": (st_score + st_select) / step_ms,
        "fused_front": {"ms": fused_ms, "lists_equal": same,
                        "note": "stem_score_select (scores computed inside the selection, no score matrix) "
                                "on the same inputs; not in the step, which runs stem_score + stem_select"},
        "selected_tflop": flops_sel_all / 1e12, "dense_tflop": flops_dense_all / 1e12,
        "effective_tflops": {"bsa": achieved * world, "prefill": flops_sel_all / (step_ms * 1e-3) / 1e12,
                             "bsa_frac_of_datasheet": achieved / datasheet,
                             "datasheet_tflops": datasheet},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": measured_traffic(wl) if world == 1 else None,
                     "peak_source": f"{peak_src} bf16_tflops_sustained" + (" x2 (fp8 nominal ratio)" if fp8 else ""),
                     "kernel": "bsa_kernel", "per": "one GPU" if world == 1 else "one rank's launch"},
        "gpu_launches": (4 + (1 if fp8 else 0)) * steps,
    }
    if clk is not None:
        rec["clocks"] = clk
    return rec


def add_dense(rec, layer, dist):
    dense_ms = time_dense(layer, dist)
    rec["dense"] = {"bsa_dense_ms": dense_ms, "launches": DENSE_LAUNCHES,
                    "speedup_prefill_vs_dense": dense_ms / rec["ms_per_step"],
                    "dense_tflops": rec["dense_tflop"] / (dense_ms * 1e-3)}


def add_graph(rec, layer, steps, dist):
    """The whole path (every kernel of stem_attention) replayed as one CUDA graph, inputs
    resident: what the per-call launch overhead costs."""
    stream = torch.cuda.current_stream()
    graph, _ = S.capture_attention(layer.prob, layer.q, layer.k, layer.v, layer.paged, out=layer.out, ws=layer.ws)
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    a, b = _events(2)
    a.record(stream)
    for _ in range(steps):
        graph.replay()
    b.record(stream)
    torch.cuda.synchronize()
    rec["graph"] = {"ms_per_step": max_over_ranks(a.elapsed_time(b) / steps, dist),
                    "kernels_per_replay": 4 + (1 if layer.wl.dtype == "fp8_e4m3" else 0),
                    "note": "stem_attention captured in one CUDA graph, inputs resident"}
    del graph
    S.query_status(layer.ws)


def add_e2e(rec, layer, steps, dist):
    """End to end through the C-ABI with host buffers: stem_attention_host copies Q/K/V
    (pinned) to the device, runs the path and copies O back, every step, kv-head group by
    group, the copies overlapping the work.  Under N > 1 each rank does this for its own
    heads (its output heads land in its host buffer; no gather)."""
    stream = torch.cuda.current_stream()
    inp, wl = layer.inp, layer.wl
    hq = inp.q.pin_memory()
    hk = (inp.k_cache if wl.paged else inp.k).pin_memory()
    hv = (inp.v_cache if wl.paged else inp.v).pin_memory()
    hout = torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory()
    k = layer.paged.k_cache if wl.paged else layer.k
    v = layer.paged.v_cache if wl.paged else layer.v

    def e2e_step():
        S.stem_attention_host(layer.prob, hq, hk, hv, layer.q, k, v, layer.paged, out_host=hout, out=layer.out,
                              ws=layer.ws)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    a, b = _events(2)
    a.record(stream)
    for _ in range(steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    S.query_status(layer.ws)
    e2e_ms = max_over_ranks(a.elapsed_time(b) / steps, dist)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    rec["e2e"] = {"value": e2e_ms, "unit": "ms/layer", "steps": steps, "h2d_bytes_per_step": h2d,
                  "d2h_bytes_per_step": hout.numel() * hout.element_size()}


def sweep(wl, steps, warmup):
    """Density sweep on one workload: BSA latency against the selected FLOPs for every keep
    fraction of the suite, next to the dense kernel (the pages report the latency as close
    to linear in density), with a least-squares line of ms on selected TFLOP."""
    rows = []
    dense_ms = None
    point = None
    base = Layer(wl)
    for keep in W.SWEEP_KEEPS:
        layer = base.with_keep(keep)
        stream = torch.cuda.current_stream()
        layer.front()
        for _ in range(warmup):
            layer.bsa()
        evs = [_events(2) for _ in range(steps)]
        for a, b in evs:
            a.record(stream)
            layer.bsa()
            b.record(stream)
        torch.cuda.synchronize()
        S.query_status(layer.ws)
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        fl = selected_flops(layer.prob, layer.rp.cpu().numpy(), wl.block, wl.head_dim, wl.seqlens)
        if dense_ms is None:
            dense_ms = time_dense(layer, None)
        rows.append({"keep": keep, "selected_tflop": fl / 1e12, "bsa_ms": ms, "tflops": fl / (ms * 1e-3) / 1e12,
                     "fraction_of_dense_time": ms / dense_ms})
        if keep == wl.keep:
            point = measure(layer, steps, warmup)
            point["dense"] = {"bsa_dense_ms": dense_ms, "launches": DENSE_LAUNCHES,
                              "speedup_prefill_vs_dense": dense_ms / point["ms_per_step"],
                              "dense_tflops": point["dense_tflop"] / (dense_ms * 1e-3)}
    x = np.array([r["selected_tflop"] for r in rows])
    y = np.array([r["bsa_ms"] for r in rows])
    slope, icpt = np.polyfit(x, y, 1)
    r2 = 1.0 - float(np.sum((y - (slope * x + icpt)) ** 2) / np.sum((y - y.mean()) ** 2))
    return point, {"workload": wl.name, "dense_ms": dense_ms, "steps": steps, "rows": rows,
                   "fit": {"ms_per_tflop": float(slope), "intercept_ms": float(icpt), "r2": r2}}


def run_sweep_only(args):
    if args.sweep_workload is not None:
        wl = W.ALL[args.sweep_workload]
    else:
        wl = W.ALL[args.workload] if args.workload != W.LONG_128K_FP8.name else W.SWEEP_64K
    _, sw = sweep(wl, args.steps, args.warmup)
    sw["metric"] = "BSA latency vs density (linear fit of ms on selected TFLOP)"
    print(json.dumps(sw), flush=True)


def extra_records(args):
    """The rest of the suite on one GPU: the tiny case, the 32K BF16 layer, the 64K BF16
    layer (keep 25% and the density sweep) and the paged varlen batch."""
    steps = min(args.steps, 10)
    warmup = max(3, args.warmup)
    out = {}
    for wl in (W.TINY, W.QWEN_32K, W.PAGED_VARLEN):
        layer = Layer(wl)
        rec = measure(layer, steps, warmup)
        add_dense(rec, layer, None)
        if not args.no_cpu_baseline:
            rec["cpu_baseline"] = cpu_sample(layer.inp)
        out[wl.name] = rec
        del layer
        torch.cuda.empty_cache()
    point, sw = sweep(W.SWEEP_64K, steps, warmup)
    if not args.no_cpu_baseline:
        point["cpu_baseline"] = cpu_sample(W.make_inputs(W.SWEEP_64K))
    out[W.SWEEP_64K.name] = point
    torch.cuda.empty_cache()
    return out, sw


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=W.LONG_128K_FP8.name, choices=sorted(W.ALL))
    ap.add_argument("--keep", type=float, default=None)
    ap.add_argument("--mu", type=float, default=None, help="end-to-start budget ratio (1 = uniform budget)")
    ap.add_argument("--beta", type=float, default=None, help="weight of the log-norm term (0 = routing score only)")
    ap.add_argument("--shared-lists", action="store_true",
                    help="one selection per KV group (an extension of this library, not in the pages)")
    ap.add_argument("--seqlen", type=int, default=None, help="replace the workload's sequences by one of this length")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads of the suite")
    ap.add_argument("--sweep-workload", default=None, choices=sorted(W.ALL),
                    help="the workload --sweep runs on (default: the 64K BF16 layer)")
    ap.add_argument("--sweep", action="store_true", help="only the density sweep (keep 1.0 .. 0.1) against the dense kernel")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    wl = W.ALL[args.workload]
    if args.keep is not None:
        wl = wl.with_(keep=args.keep)
    if args.mu is not None:
        wl = wl.with_(mu=args.mu)
    if args.beta is not None:
        wl = wl.with_(beta=args.beta)
    if args.shared_lists:
        wl = wl.with_(shared_lists=True)
    if args.seqlen is not None:
        wl = wl.with_(seqlens=(args.seqlen,), name=f"{wl.name}@{args.seqlen}")
    if args.impl == "reference":
        run_reference(args, wl)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the path has no CPU fallback)")
    if args.sweep:
        S.lib()
        run_sweep_only(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    S.lib()

    layer = Layer(wl, rank, world)
    rec = measure(layer, args.steps, args.warmup, dist, with_clocks=True)
    if not args.no_dense:
        add_dense(rec, layer, dist)
    if not args.no_graph:
        add_graph(rec, layer, args.steps, dist)
    if not args.no_e2e:
        add_e2e(rec, layer, args.steps, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_sample(layer.inp)
    del layer
    torch.cuda.empty_cache()
    extra = sweep_rec = None
    if world == 1 and not args.no_extra:
        extra, sweep_rec = extra_records(args)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        clocks = rec.pop("clocks", None)
        line = {"metric": METRIC, "value": rec["value"], "unit": "ms/layer", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": False,
                "scaling": "strong", "vs_baseline": None, "dtype": rec["dtype"], "data": "synthetic",
                "config": dict(rec["config"], parallelism=f"kv-head groups over {world} GPUs" if world > 1 else "none")}
        for k in ("stages_ms", "score_select_frac", "fused_front", "selected_tflop", "dense_tflop",
                  "effective_tflops", "roofline", "gpu_launches", "dense", "graph", "e2e", "cpu_baseline"):
            if k in rec:
                line[k] = rec[k]
        line["clocks"] = clocks
        if extra is not None:
            line["workloads"] = extra
            line["density_sweep"] = sweep_rec
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
