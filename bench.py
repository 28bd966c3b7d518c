"""Benchmark of the Stem sparse-attention prefill path on B200.

One step = one pass of the whole hot path over one layer's synthetic inputs
(stem_score -> stem_select -> bsa_prefill, i.e. what stem_attention runs), inputs
resident in HBM.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: one Qwen3-8B-shaped layer at 128K tokens in FP8-e4m3, keep 25%.
With N > 1 (torchrun) every rank runs its own replica (the path has no exchange
step); the device time is the max over ranks.
"""
from __future__ import annotations

import argparse
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

from block_sparse_attention_oam_b200 import stem as S          # noqa: E402
from block_sparse_attention_oam_b200 import workloads as W     # noqa: E402

METRIC = "Stem prefill ms/layer at 128K, 25% budget; effective TFLOP/s vs B200 peak"
BF16_DATASHEET_TFLOPS = 2250.0
FP8_OVER_BF16 = 2.0          # nominal dense FP8 / BF16 tensor throughput ratio
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_STEP = 6         # pool(Q), pool(K), pool(V), score, select, bsa (+1 for FP8: its first-row bsa launch)
# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one bsa_kernel launch, from
# an ncu capture of that launch on the named workload (summaries under profiles/).  A figure
# holds only for the kernel source and the input generator it was taken on: KERNEL_SOURCES
# are hashed and compared.
KERNEL_SOURCES = ("block_sparse_attention_oam_b200/csrc/stem_bsa.cu", "block_sparse_attention_oam_b200/csrc/stem_internal.cuh",
                  "block_sparse_attention_oam_b200/workloads.py")
MEASURED_TRAFFIC = {
    # (workload, keep, mu, beta): (bytes per launch, sha256 of KERNEL_SOURCES, profile summary)
    ("qwen3_8b_layer_s128k_fp8", 0.25, 0.7, 0.2): (2.14e9, "0faad37df4b9e65bfff87e4099340736e40601ecb236c8f7db3406492db9a144",
                                         "profiles/launches_s128k_fp8_keep25.md"),
    ("qwen3_8b_layer_s64k_bf16", 0.25, 0.7, 0.2): (1.409e9, "0faad37df4b9e65bfff87e4099340736e40601ecb236c8f7db3406492db9a144",
                                         "profiles/bsa_kernel_bf16_s64k_keep25.md"),
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
    """The slowest replica's time (every rank gets it); `dist` None on one GPU."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def ms_per_layer(step_ms_max: float, world: int) -> float:
    """Replicas each process one layer per step: the job's time per layer is the slowest
    replica's step time over the layers processed by all of them."""
    return step_ms_max / world


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


def cpu_baseline(inp: W.Inputs, rp: np.ndarray, ci: np.ndarray, budget_s: float = 15.0):
    """Time the float64 oracle (as it stands) on a bounded sample of the workload on
    the host cores and scale to ms per layer: pool + score + select for one q-head
    (all rows), attention for a seeded subset of that head's q-blocks, extrapolated
    by selected blocks to all heads."""
    from oracle import stem_oracle as O
    from threadpoolctl import threadpool_info
    wl = inp.wl
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    h = 0
    g = wl.num_q_heads // wl.num_kv_heads
    t_sel = 0.0
    t_att = 0.0
    blocks_done = 0
    blocks_total = int(ci.shape[1]) * wl.num_q_heads
    rng = np.random.default_rng(0)
    row0 = 0
    cu = inp.cu_seqlens
    sample_rows = 0
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
        order = rng.permutation(N)
        c0 = time.perf_counter()
        for i in order:
            O.attend(q, k, v, lists, wl.block, wl.softmax_scale, rows=[(0, int(i))])
            blocks_done += len(lists[0][i])
            sample_rows += 1
            if time.perf_counter() - c0 > budget_s / len(wl.seqlens):
                break
        t_att += time.perf_counter() - c0
        row0 += N
    ms = (t_sel + t_att * blocks_total / max(1, blocks_done)) * 1e3
    return {"value": ms, "unit": "ms/layer", "cores": threads, "kind": "oracle",
            "sample": f"float64 oracle on q-head 0: pool+score+select over all rows (x{wl.num_q_heads} heads), "
                      f"attention on {sample_rows} seeded q-blocks ({blocks_done} of {blocks_total} selected "
                      f"blocks), extrapolated by selected blocks"}


def run_reference(args, wl):
    """Reference arm: the oracle itself, timed as it stands on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    inp = W.make_inputs(wl)
    from oracle import stem_oracle as O
    # the oracle's own selection gives the CSR the sample needs
    rows, cols = [], []
    for S_ in wl.seqlens:
        N = math.ceil(S_ / wl.block)
        rows.append(O.tpd_plan(N, wl.keep, wl.mu)[2])
    k = np.concatenate(rows)
    rp = np.concatenate([[0], np.cumsum(k)]).astype(np.int32)
    ci = np.zeros((wl.num_q_heads, int(rp[-1])), dtype=np.int32)
    vals = []
    for _ in range(args.warmup + args.steps):
        vals.append(cpu_baseline(inp, rp, ci, budget_s=max(2.0, 20.0 / (args.warmup + args.steps))))
    timed = vals[args.warmup:]
    v = statistics.mean(x["value"] for x in timed)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "ms/layer", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "seq_len": list(wl.seqlens), "keep": wl.keep, "block": wl.block,
                       "heads": [wl.num_q_heads, wl.num_kv_heads], "head_dim": wl.head_dim},
            "cpu_baseline": {"value": v, "unit": "ms/layer", "cores": timed[-1]["cores"], "kind": "oracle",
                             "sample": timed[-1]["sample"]},
            "e2e": {"value": v, "unit": "ms/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """Density sweep: BSA latency against the selected FLOPs for several keep
    fractions on one workload, next to the dense kernel (the pages report the
    latency as close to linear in density)."""
    wl = W.ALL[args.workload] if args.workload != W.LONG_128K_FP8.name else W.SWEEP_64K
    inp = W.make_inputs(wl)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    stream = torch.cuda.current_stream()
    rows = []
    dense_ms = None
    for keep in W.SWEEP_KEEPS:
        prob = S.problem_for(wl.with_(keep=keep), inp)
        sz = prob.sizes()
        ws = S.workspace(prob)
        scores = torch.empty((wl.num_q_heads, sz["scores_per_head"]), dtype=torch.float32, device="cuda")
        rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
        ci = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
        out = torch.empty((sz["total_tokens"], wl.num_q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
        S.stem_score(prob, q, k, v, scores=scores, ws=ws)
        S.stem_select(prob, scores, rp, ci, ws=ws)
        for _ in range(args.warmup):
            S.bsa_prefill(prob, q, k, v, rp, ci, out=out, ws=ws)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in evs:
            a.record(stream)
            S.bsa_prefill(prob, q, k, v, rp, ci, out=out, ws=ws)
            b.record(stream)
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        fl = selected_flops(prob, rp.cpu().numpy(), wl.block, wl.head_dim, wl.seqlens)
        if dense_ms is None:
            for _ in range(args.warmup):
                S.bsa_dense_prefill(prob, q, k, v, out=out, ws=ws)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(args.steps):
                S.bsa_dense_prefill(prob, q, k, v, out=out, ws=ws)
            b.record(stream)
            torch.cuda.synchronize()
            dense_ms = a.elapsed_time(b) / args.steps
        S.query_status(ws)
        rows.append({"keep": keep, "selected_tflop": fl / 1e12, "bsa_ms": ms, "tflops": fl / (ms * 1e-3) / 1e12,
                     "fraction_of_dense_time": ms / dense_ms})
    x = np.array([r["selected_tflop"] for r in rows])
    y = np.array([r["bsa_ms"] for r in rows])
    slope, icpt = np.polyfit(x, y, 1)
    r2 = 1.0 - float(np.sum((y - (slope * x + icpt)) ** 2) / np.sum((y - y.mean()) ** 2))
    line = {"metric": "BSA latency vs density (linear fit of ms on selected TFLOP)", "workload": wl.name,
            "dtype": "e4m3" if wl.dtype == "fp8_e4m3" else "bf16", "steps": args.steps, "warmup": args.warmup,
            "dense_ms": dense_ms, "sweep": rows,
            "fit": {"ms_per_tflop": float(slope), "intercept_ms": float(icpt), "r2": r2}}
    print(json.dumps(line), flush=True)


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
    ap.add_argument("--sweep", action="store_true", help="density sweep (keep 1.0 .. 0.1) against the dense kernel")
    args = ap.parse_args()
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
    if args.sweep:
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device (the path has no CPU fallback)")
        S.lib()
        run_sweep(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the path has no CPU fallback)")
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    S.lib()

    inp = W.make_inputs(wl.with_(seed=wl.seed + 1000 * rank))
    prob = S.problem_for(wl, inp)
    sz = prob.sizes()
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    paged = None
    if wl.paged:
        paged = S.PagedKV(inp.k_cache.cuda(), inp.v_cache.cuda(), torch.from_numpy(inp.block_table).cuda())
    ws = S.workspace(prob)
    scores = torch.empty((wl.num_q_heads, sz["scores_per_head"]), dtype=torch.float32, device="cuda")
    rp = torch.empty(sz["num_rows"] + 1, dtype=torch.int32, device="cuda")
    ci = torch.empty((sz["list_heads"], sz["nnz_per_head"]), dtype=torch.int32, device="cuda")
    out = torch.empty((sz["total_tokens"], wl.num_q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        S.stem_score(prob, q, k, v, paged, scores=scores, ws=ws)
        if ev is not None:
            ev[1].record(stream)
        S.stem_select(prob, scores, rp, ci, ws=ws)
        if ev is not None:
            ev[2].record(stream)
        S.bsa_prefill(prob, q, k, v, rp, ci, paged, out=out, ws=ws)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    S.query_status(ws)
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = Clocks(torch.cuda.current_device())
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if dist is not None:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    st_score = [e[0].elapsed_time(e[1]) for e in evs]
    st_select = [e[1].elapsed_time(e[2]) for e in evs]
    st_bsa = [e[2].elapsed_time(e[3]) for e in evs]
    S.query_status(ws)
    total_ms = max_over_ranks(total_ms, dist)

    rp_h = rp.cpu().numpy()
    flops_sel = selected_flops(prob, rp_h, wl.block, wl.head_dim, wl.seqlens)
    flops_dense = dense_flops(wl.seqlens, wl.num_q_heads, wl.head_dim)
    bsa_ms = statistics.mean(st_bsa)
    step_ms = total_ms / args.steps
    peaks, peak_src = measured_peaks()
    fp8 = wl.dtype == "fp8_e4m3"
    peak = peaks["bf16_tflops_sustained"] * (FP8_OVER_BF16 if fp8 else 1.0)
    achieved = flops_sel / (bsa_ms * 1e-3) / 1e12

    result = {
        "metric": METRIC, "value": ms_per_layer(step_ms, world), "unit": "ms/layer", "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "seq_len": list(wl.seqlens), "keep": wl.keep, "mu": wl.mu,
                   "beta": wl.beta, "shared_lists": wl.shared_lists, "block": wl.block, "heads": [wl.num_q_heads, wl.num_kv_heads],
                   "head_dim": wl.head_dim, "paged": wl.paged, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2 (no flush)"},
        "stages_ms": {"score": statistics.mean(st_score), "select": statistics.mean(st_select), "bsa": bsa_ms},
        "score_select_frac": (statistics.mean(st_score) + statistics.mean(st_select)) / step_ms,
        "selected_tflop": flops_sel / 1e12, "dense_tflop": flops_dense / 1e12,
        "effective_tflops": {"bsa": achieved, "prefill": flops_sel / (step_ms * 1e-3) / 1e12,
                             "bsa_frac_of_bf16_datasheet": achieved / BF16_DATASHEET_TFLOPS},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": measured_traffic(wl),
                     "peak_source": f"{peak_src} bf16_tflops_sustained" + (" x2 (fp8 nominal ratio)" if fp8 else ""),
                     "kernel": "bsa_kernel"},
        "gpu_launches": (KERNELS_PER_STEP + (1 if fp8 else 0)) * args.steps,
        "clocks": clk,
    }

    if not args.no_dense:
        dt = []
        for i in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            S.bsa_dense_prefill(prob, q, k, v, paged, out=out, ws=ws)
            b.record(stream)
            torch.cuda.synchronize()
            if i > 0:
                dt.append(a.elapsed_time(b))
        dense_ms = statistics.mean(dt)
        result["dense"] = {"bsa_dense_ms": dense_ms, "speedup_prefill_vs_dense": dense_ms / step_ms,
                           "dense_tflops": flops_dense / (dense_ms * 1e-3) / 1e12}
        S.query_status(ws)

    if not args.no_graph:
        # the whole path (every kernel of stem_attention) replayed as one CUDA graph,
        # inputs resident: what the per-call launch overhead costs
        graph, _ = S.capture_attention(prob, q, k, v, paged, out=out, ws=ws)
        for _ in range(2):
            graph.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        g_ms = a.elapsed_time(b) / args.steps
        g_ms = max_over_ranks(g_ms, dist)
        result["graph"] = {"ms_per_step": g_ms, "kernels_per_replay": KERNELS_PER_STEP + (1 if fp8 else 0),
                           "note": "stem_attention captured in one CUDA graph, inputs resident"}
        del graph
        S.query_status(ws)

    if not args.no_e2e:
        # end to end through the C-ABI with host buffers: stem_attention_host copies Q/K/V
        # (pinned) to the device, runs the path and copies O back, every step, group of
        # kv-heads by group, the copies overlapping the work.
        hq, hk, hv = inp.q.pin_memory(), (inp.k_cache if wl.paged else inp.k).pin_memory(), \
            (inp.v_cache if wl.paged else inp.v).pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            S.stem_attention_host(prob, hq, hk, hv, q, k, v, paged, out_host=hout, out=out, ws=ws)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        a.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms = a.elapsed_time(b) / n_e2e
        e2e_ms = max_over_ranks(e2e_ms, dist)
        h2d = hq.numel() * hq.element_size() + hk.numel() * hk.element_size() + hv.numel() * hv.element_size()
        result["e2e"] = {"value": ms_per_layer(e2e_ms, world), "unit": "ms/layer", "h2d_bytes_per_step": h2d,
                         "d2h_bytes_per_step": hout.numel() * hout.element_size()}
        S.query_status(ws)

    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(inp, rp_h, ci.cpu().numpy())

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


if __name__ == "__main__":
    main()
