#!/usr/bin/env python
"""Benchmark of the DSA forward hot path (lightning indexer -> top-k -> sparse MLA) on B200.

One step = one ``dsa_forward`` call over the whole workload (all query rows: chunked
indexer + top-k, then the sparse MLA), inputs resident in HBM.  Default workload: one
32K-token prefill (topk 2048).  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

N > 1 (launched by torchrun) runs N independent replicas, one per GPU: the path has no
exchange step on one problem, so there is no collective on the data path; the timing is
the max over ranks and ``value`` counts the tokens all ranks processed.

``--impl reference`` times the fp64 CPU oracle on the host cores (bounded row samples of
the same workload); it is the slow reference arm, not a GPU implementation.
"""
from __future__ import annotations

import argparse
import hashlib
import json
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

import dsa_synth  # noqa: E402

METRIC = "DSA fwd tokens/s at 32K prefill (indexer+topk+sparse MLA); decode µs/step"
L2_BYTES = 126 * 1024 * 1024
FLOP_PER_PAIR_INDEXER = 64 * 128 * 2            # per causal (query, key) pair
FLOP_PER_PAIR_MLA = 128 * (576 + 512) * 2       # per (query, selected key) pair, 128 heads

# ncu DRAM traffic (read + write bytes per launch) of each kernel, recorded against the
# sha256 of the source file it was captured from; reported only while the source is
# unchanged.
TRAFFIC = {
    # ncu capture of the 4096-query prefill launch (persistent pairs): 1.141 GB of DRAM
    # traffic (642 MB read, 499 MB written: q reads and out writes, both proportional to the
    # query count; kv rows come from L2), scaled x8 to the 32768-query launch of the 32K step
    # (that prefill only: at 128K the kv rows no longer fit in L2)
    "sparse_mla": {"bytes_per_launch": 1.140993e9 * 8, "total_q": 32768, "src_sha": "ad33592d1748a857"},
}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d.get("bf16_tflops_sustained"),
                    src="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def _src_sha(name: str) -> str:
    p = os.path.join(ROOT, "attention_lightning_indexer_b200", "csrc", name)
    try:
        return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]
    except OSError:
        return ""


# ----------------------------------------------------------------- distributed

def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _init_pg(ws, local, backend="nccl"):
    if ws <= 1:
        return None
    import datetime

    import torch.distributed as dist

    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def _barrier(dist):
    if dist is not None:
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def _max_over_ranks(dist, x: float) -> float:
    if dist is None:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not self.uuid.startswith("GPU-"):
                self.uuid = "GPU-" + self.uuid
        except Exception:
            self.uuid = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.uuid:
                cmd.insert(1, f"--id={self.uuid}")
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ----------------------------------------------------------------- workload facts

def _pairs(inp):
    """(causal indexer pairs, selected MLA pairs, top-k algorithmic bytes) of a workload."""
    cu_q = inp["cu_q"].cpu().numpy().astype(np.int64)
    cu_k = inp["cu_k"].cpu().numpy().astype(np.int64)
    k = inp["topk"]
    idx_pairs = mla_pairs = topk_bytes = 0
    for b in range(len(cu_q) - 1):
        lq, lk = cu_q[b + 1] - cu_q[b], cu_k[b + 1] - cu_k[b]
        n = np.arange(lk - lq, lk, dtype=np.int64) + 1          # visible keys per query row
        idx_pairs += int(n.sum())
        mla_pairs += int(np.minimum(n, k).sum())
        topk_bytes += int((4 * n * (n > k)).sum()) + 4 * k * int(lq)
    return idx_pairs, mla_pairs, topk_bytes


def _tokens(inp):
    return int(inp["total_q"])


def _config(args, inp, chunk, ws):
    """The workload's `config`, the same for both arms (how each arm runs it is stated in its
    own keys: `cpu_baseline.sample` for the reference arm)."""
    return {"workload": args.workload, "global_batch": ws * inp["batch"], "seq_len": int(inp["max_len_k"]),
            "topk": inp["topk"], "chunk_q": chunk, "parallelism": f"replicas x{ws}",
            "l2": "flushed between timed steps (2 x 126 MB write) and inputs > L2"}


# Longest key sequence the library's forward attends in the dense (masked) form alone
# (include/dsa.h, dsa_forward).
DENSE_KV_THRESHOLD = 3584


def _attention_launches(p) -> int:
    """Attention launches of one dsa_forward call on a prefill without split partials: the
    dense form alone for short key sequences; in one packed, unpaged sequence the rows whose
    visible keys all fit in topk take the dense form and the rest the gathered form."""
    if not p.block_table and p.max_len_k <= DENSE_KV_THRESHOLD:
        return 1
    T = p.total_q
    R = min(max(p.topk - (p.total_k - T), 0), T) if not p.cu_q and not p.block_table else 0
    return 2 if 0 < R < T else 1


# ----------------------------------------------------------------- our arm

def _forward_args(inp):
    fp8 = "q_idx8" in inp
    blocks = "q_scale_ue8m0" in inp
    return dict(q_idx=inp["q_idx8"] if fp8 else inp["q_idx"], k_idx=inp["k_idx8"] if fp8 else inp["k_idx"],
                q_scale=inp["q_scale_ue8m0"] if blocks else inp.get("q_scale"),
                k_scale=inp["k_scale_ue8m0"] if blocks else inp.get("k_scale"))


def run_ours(args, ws, rank, local, dist):
    import attention_lightning_indexer_b200 as dsa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = dsa_synth.WORKLOADS[args.workload]
    inp = dsa_synth.make_workload(args.workload, seed=args.seed, device=dev)
    chunk = args.chunk if args.chunk is not None else wl.chunk
    p = dsa.problem_from_inputs(inp)
    fa = _forward_args(inp)
    T = inp["total_q"]
    out = torch.empty((T, 128, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, 128), dtype=torch.float32, device=dev)
    wsb = torch.empty(dsa.dsa_forward_workspace_size(p, chunk), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(o=out, l=lse, q=inp["q"], kv=inp["kv"], qi=fa["q_idx"], ki=fa["k_idx"], w=inp["w"]):
        dsa.dsa_forward(p, qi, ki, w, q, kv, o, l, wsb, chunk_q=chunk, q_scale=fa["q_scale"],
                        k_scale=fa["k_scale"], stream=stream)

    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    dsa.dsa_check_device_errors()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    _barrier(dist)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()                      # evict L2 between timed steps (outside the events)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    _barrier(dist)
    clk = clocks.stop()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = _max_over_ranks(dist, sum(step_ms))
    dsa.dsa_check_device_errors()

    tokens = _tokens(inp)
    n_chunks = (T + (chunk or T) - 1) // (chunk or T)
    launches_per_step = 2 * n_chunks + _attention_launches(p)
    res = {
        "metric": METRIC,
        "value": ws * tokens * args.steps / (total_ms / 1e3),
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if "q_idx8" not in inp else "e4m3 indexer + bf16 attention",
        "data": "synthetic (seeded; shapes and distributions of the workload recipe)",
        "config": _config(args, inp, chunk, ws),
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }

    if rank == 0 and not args.no_breakdown:
        res["roofline"], res["kernels"] = _breakdown(dsa, p, inp, fa, chunk, dev, stream, flush)
    if args.workload != "decode_b64" and not args.no_decode:
        res["decode"] = _decode_secondary(dsa, args, rank, dev, stream, flush, dist)
    if not args.no_e2e:
        res["e2e"] = _e2e(dsa, p, inp, fa, chunk, dev, stream, args, ws, dist)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = _cpu_baseline(inp, args.cpu_rows, args.seed)
    if rank == 0:
        print(json.dumps(res), flush=True)


def _capture(step, dev):
    """One call of step() captured as a CUDA graph (on a side stream, as capture needs)."""
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream(dev))
    torch.cuda.synchronize(dev)
    return graph


def _decode_secondary(dsa, args, rank, dev, stream, flush, dist):
    """The metric's second half: decode microseconds per step (64 sequences, one query
    each, contexts ~U[8192, 65536]), timed like the main step (events, L2 flushed between
    steps, max over ranks)."""
    inp = dsa_synth.make_workload("decode_b64", seed=args.seed, device=dev)
    p = dsa.problem_from_inputs(inp)
    fa = _forward_args(inp)
    T = inp["total_q"]
    out = torch.empty((T, 128, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, 128), dtype=torch.float32, device=dev)
    wsb = torch.empty(dsa.dsa_forward_workspace_size(p, 0), dtype=torch.uint8, device=dev)

    def step(st=stream):
        dsa.dsa_forward(p, fa["q_idx"], fa["k_idx"], inp["w"], inp["q"], inp["kv"], out, lse, wsb, chunk_q=0,
                        stream=st)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    n = max(args.steps, 10)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    def timed(run):
        _barrier(dist)
        for i in range(n):
            flush.zero_()
            starts[i].record(stream)
            run()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        _barrier(dist)
        return _max_over_ranks(dist, sum(s.elapsed_time(e) for s, e in zip(starts, ends))) / n * 1e3

    # A serving loop captures its decode step once and replays it: the step as a CUDA graph
    # of its kernel launches, replayed on the bench stream (the eager time is reported too).
    graph = _capture(step, dev)
    us_graph = timed(graph.replay)
    us_eager = timed(step)
    dsa.dsa_check_device_errors()
    res = {"workload": "decode_b64", "us_per_step": us_graph, "cuda_graph": True, "us_per_step_eager": us_eager,
           "steps": n, "batch": inp["batch"], "mean_context": float(inp["total_k"]) / inp["batch"],
           "gpu_launches_per_step": 3, "higher_is_better": False}
    del graph
    # the same step with the key caches in shuffled 64-token pages (block table)
    pg = dsa_synth.to_paged(inp, page_size=64, seed=args.seed + 7)
    pp = dsa.problem_from_inputs(pg)
    def step_paged(st=stream):
        dsa.dsa_forward(pp, pg["q_idx"], pg["k_idx"], pg["w"], pg["q"], pg["kv"], out, lse, wsb, chunk_q=0, stream=st)

    for _ in range(3):
        step_paged()
    graph = _capture(step_paged, dev)
    res["us_per_step_paged_cache"] = timed(graph.replay)
    dsa.dsa_check_device_errors()
    del graph, pg
    # a small batch (8 sequences, the same context range): too few tokens to fill the SMs,
    # so the attention splits each index row over several CTA pairs and merges by lse
    sb = dsa_synth.make_decode(8, 8192, 65536, topk=inp["topk"], seed=args.seed + 11, device=dev)
    ps = dsa.problem_from_inputs(sb)
    out_s = torch.empty((sb["total_q"], 128, 512), dtype=torch.bfloat16, device=dev)
    lse_s = torch.empty((sb["total_q"], 128), dtype=torch.float32, device=dev)
    ws_s = torch.empty(dsa.dsa_forward_workspace_size(ps, 0), dtype=torch.uint8, device=dev)
    def step_small(st=stream):
        dsa.dsa_forward(ps, sb["q_idx"], sb["k_idx"], sb["w"], sb["q"], sb["kv"], out_s, lse_s, ws_s, stream=st)

    for _ in range(3):
        step_small()
    graph = _capture(step_small, dev)
    res["small_batch"] = {"batch": 8, "mean_context": float(sb["total_k"]) / 8, "gpu_launches_per_step": 4,
                          "cuda_graph": True, "us_per_step": timed(graph.replay)}
    dsa.dsa_check_device_errors()
    del graph, sb, ws_s
    if rank == 0 and not args.no_breakdown:
        res["roofline"], res["kernels"] = _breakdown(dsa, p, inp, fa, 0, dev, stream, flush, decode=True)
    return res


def _breakdown(dsa, p, inp, fa, chunk, dev, stream, flush, reps=2, decode=False):
    """Average device time of each kernel of the step: each call is captured once as a CUDA
    graph (its host-side argument set-up happens at capture) and replayed between CUDA events
    on the bench stream, L2 flushed before.  Prefill kernels run for milliseconds and replay
    once per flush.  Decode kernels run for tens of microseconds, where one launch's latency
    would count in full although the step overlaps it: they replay 10 times back to back per
    flush (the indexer's keys and the attention's rows still come from HBM, the top-k's
    score rows from L2 as in the step, right after the indexer wrote them)."""
    T = inp["total_q"]
    chunk = chunk or T
    ld = dsa.scores_ld(inp["max_len_k"])
    scores = torch.empty((chunk, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((T, inp["topk"]), dtype=torch.int32, device=dev)
    out = torch.empty((T, 128, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, 128), dtype=torch.float32, device=dev)
    t_idx = t_topk = t_mla = 0.0
    n_idx = n_topk = n_mla = 0

    back_to_back = 10 if decode else 1

    def timed(call):
        graph = _capture(call, dev)
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            for _ in range(back_to_back):
                graph.replay()
            b.record(stream)
        b.synchronize()
        del graph
        return a.elapsed_time(b) / back_to_back

    for _ in range(reps):
        for r0 in range(0, T, chunk):
            rc = min(chunk, T - r0)
            t_idx += timed(lambda st: dsa.dsa_indexer_scores(p, fa["q_idx"], fa["k_idx"], inp["w"], scores,
                                                             row_begin=r0, row_count=rc, q_scale=fa["q_scale"],
                                                             k_scale=fa["k_scale"], stream=st))
            t_topk += timed(lambda st: dsa.dsa_topk(p, scores, idx[r0:r0 + rc], row_begin=r0, row_count=rc,
                                                    stream=st))
            n_idx += 1
            n_topk += 1
        t_mla += timed(lambda st: dsa.dsa_sparse_mla_fwd(p, inp["q"], inp["kv"], idx, out, lse, stream=st))
        n_mla += 1
    idx_pairs, mla_pairs, topk_bytes = _pairs(inp)
    pk = _peaks()
    fp8 = "q_idx8" in inp
    idx_peak = pk["bf16"] * (2.0 if fp8 else 1.0)
    kernels = {
        "indexer": {"ms_per_launch": t_idx / n_idx, "launches_per_step": n_idx // reps,
                    "ms_per_step": t_idx / reps, "tflops": idx_pairs * FLOP_PER_PAIR_INDEXER / (t_idx / reps) / 1e9,
                    "peak_tflops": idx_peak},
        "topk": {"ms_per_launch": t_topk / n_topk, "launches_per_step": n_topk // reps, "ms_per_step": t_topk / reps,
                 "gbs": topk_bytes / (t_topk / reps) / 1e6, "peak_gbs": pk["hbm_gbs"]},
        "sparse_mla": {"ms_per_launch": t_mla / n_mla, "launches_per_step": 1, "ms_per_step": t_mla / reps,
                       "tflops": mla_pairs * FLOP_PER_PAIR_MLA / (t_mla / reps) / 1e9, "peak_tflops": pk["bf16"]},
    }
    # algorithmic HBM bytes of each kernel (decode is bandwidth-bound throughout)
    T, k = inp["total_q"], inp["topk"]
    eb = 1 if fp8 else 2
    idx_bytes = (inp["total_k"] * 128 * eb + T * 64 * 128 * eb + T * 64 * 4 + 4 * idx_pairs
                 + (4 * (T + inp["total_k"]) if fp8 else 0))
    mla_bytes = mla_pairs * 1152 + T * 128 * (576 + 512) * 2 + T * 128 * 4 + T * k * 4
    for name, nbytes in (("indexer", idx_bytes), ("sparse_mla", mla_bytes)):
        kernels[name]["gbs"] = nbytes / (kernels[name]["ms_per_step"]) / 1e6
        kernels[name]["peak_gbs"] = pk["hbm_gbs"]
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    kd = kernels[dom]
    src = {"indexer": "indexer_tc.cuh", "topk": "topk.cuh", "sparse_mla": "sparse_mla_pair.cuh"}[dom]
    tr = TRAFFIC.get(dom)
    traffic = (tr["bytes_per_launch"] if tr and tr.get("src_sha") == _src_sha(src) and not decode
               and inp["total_q"] == tr.get("total_q") and "q_idx8" not in inp else None)
    if dom == "topk" or decode:
        roof = {"bound": "hbm", "achieved": kd["gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": kd["gbs"] / pk["hbm_gbs"], "traffic": traffic}
    else:
        roof = {"bound": "tensor", "achieved": kd["tflops"], "peak": kd["peak_tflops"], "unit": "TFLOP/s",
                "frac": kd["tflops"] / kd["peak_tflops"], "traffic": traffic}
    roof.update({"kernel": dom, "peak_source": pk["src"] + " (MEASURED_PEAKS burst figure)"
                 if pk["src"] == "measured" else "fallback"})
    return roof, kernels


def _e2e(dsa, p, inp, fa, chunk, dev, stream, args, ws, dist):
    """Same metric end to end through the public calls with host buffers: every step copies
    its inputs from pinned host memory, runs the path and copies out + lse back, all inside
    the timed region.  The step is pipelined over the query chunks on three streams: the
    chunk's indexer inputs and q go up (copy stream), indexer -> top-k -> sparse MLA run on
    the chunk (compute stream, the MLA on the chunk's rows as a sub-problem whose queries are
    the last rows of a prefix of the sequence), and the chunk's out / lse come down (second
    copy stream), so the two copy directions and the kernels overlap.  Ragged batches run as
    one chunk."""
    fp8 = "q_idx8" in inp
    qi_name, ki_name = ("q_idx8", "k_idx8") if fp8 else ("q_idx", "k_idx")
    key_names = [n for n in (ki_name, "k_scale", "kv") if n in inp]
    row_names = [n for n in (qi_name, "q_scale", "w", "q") if n in inp]
    names = key_names + row_names
    host = {n: inp[n].cpu().pin_memory() for n in names}
    devb = {n: torch.empty_like(inp[n]) for n in names}
    T = inp["total_q"]
    ragged = p.cu_q is not None
    ch = T if (ragged or not chunk) else min(chunk, args.e2e_chunk)
    chunks = [(r0, min(ch, T - r0)) for r0 in range(0, T, ch)]
    out = torch.empty((T, 128, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((T, 128), dtype=torch.float32, device=dev)
    idx = torch.empty((T, inp["topk"]), dtype=torch.int32, device=dev)
    scores = torch.empty((ch, dsa.scores_ld(inp["max_len_k"])), dtype=torch.float32, device=dev)
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_cmp = stream
    ev = lambda: torch.cuda.Event()                                   # noqa: E731
    last = {"keys_free": None, "rows_free": [None] * len(chunks), "out_free": [None] * len(chunks)}

    def mla_sub(r0, rc):
        if ragged:
            return p
        return dsa.make_problem(1, rc, r0 + rc, rc, r0 + rc, inp["topk"], sm_scale=p.sm_scale)

    subs = [mla_sub(r0, rc) for r0, rc in chunks]

    def step():
        # keys (and kv) once per step, after the previous step's last kernel that reads them
        if last["keys_free"] is not None:
            s_in.wait_event(last["keys_free"])
        with torch.cuda.stream(s_in):
            for n in key_names:
                devb[n].copy_(host[n], non_blocking=True)
        keys_in = ev()
        keys_in.record(s_in)
        rows_in = []
        for c, (r0, rc) in enumerate(chunks):
            if last["rows_free"][c] is not None:
                s_in.wait_event(last["rows_free"][c])
            with torch.cuda.stream(s_in):
                for n in row_names:
                    devb[n][r0:r0 + rc].copy_(host[n][r0:r0 + rc], non_blocking=True)
            e = ev()
            e.record(s_in)
            rows_in.append(e)
        s_cmp.wait_event(keys_in)
        for c, (r0, rc) in enumerate(chunks):
            s_cmp.wait_event(rows_in[c])
            dsa.dsa_indexer_scores(p, devb[qi_name], devb[ki_name], devb["w"], scores, row_begin=r0, row_count=rc,
                                   q_scale=devb.get("q_scale"), k_scale=devb.get("k_scale"), stream=s_cmp)
            dsa.dsa_topk(p, scores, idx[r0:r0 + rc], row_begin=r0, row_count=rc, stream=s_cmp)
            if last["out_free"][c] is not None:
                s_cmp.wait_event(last["out_free"][c])
            dsa.dsa_sparse_mla_fwd(subs[c], devb["q"][r0:r0 + rc], devb["kv"], idx[r0:r0 + rc], out[r0:r0 + rc],
                                   lse[r0:r0 + rc], stream=s_cmp)
            done = ev()
            done.record(s_cmp)
            last["rows_free"][c] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                out_h[r0:r0 + rc].copy_(out[r0:r0 + rc], non_blocking=True)
                lse_h[r0:r0 + rc].copy_(lse[r0:r0 + rc], non_blocking=True)
            e = ev()
            e.record(s_out)
            last["out_free"][c] = e
        kf = ev()
        kf.record(s_cmp)
        last["keys_free"] = kf

    step()
    torch.cuda.synchronize(dev)
    steps = max(1, min(args.steps, 3))
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    _barrier(dist)
    torch.cuda.synchronize(dev)
    a.record(s_in)
    for _ in range(steps):
        step()
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize(dev)
    _barrier(dist)
    ms = _max_over_ranks(dist, a.elapsed_time(b)) / steps
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
    # the pipelined calls must give exactly what dsa_forward gives on the same inputs
    out_ref, lse_ref = torch.empty_like(out), torch.empty_like(lse)
    wsb = torch.empty(dsa.dsa_forward_workspace_size(p, ch), dtype=torch.uint8, device=dev)
    dsa.dsa_forward(p, devb[qi_name], devb[ki_name], devb["w"], devb["q"], devb["kv"], out_ref, lse_ref, wsb,
                    chunk_q=ch, q_scale=devb.get("q_scale"), k_scale=devb.get("k_scale"), stream=s_cmp)
    torch.cuda.synchronize(dev)
    same = bool(torch.equal(out_h, out_ref.cpu()) and torch.equal(lse_h, lse_ref.cpu()))
    return {"value": ws * _tokens(inp) / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "pipelined": f"{len(chunks)} query chunks over 3 streams (H2D / kernels / D2H)",
            "gpu_launches_per_step": 3 * len(chunks), "identical_to_dsa_forward": same}


# ----------------------------------------------------------------- oracle (CPU) arms

def _oracle_inputs_host(inp):
    """Host copies the oracle reads: full key-side tensors, query-side tensors stay on device."""
    keys = {n: inp[n].cpu() for n in ("k_idx", "k_idx8", "k_scale", "kv") if n in inp}
    return keys


def _oracle_forward_rows(inp, keys, rows):
    import oracle

    rt = torch.from_numpy(rows)
    cu_q = inp["cu_q"].cpu().numpy()
    cu_k = inp["cu_k"].cpu().numpy()
    dev_rows = rt.to(inp["w"].device)
    w = inp["w"][dev_rows].cpu()
    q = inp["q"][dev_rows].cpu()
    if "q_idx8" in inp:
        sc = oracle.indexer_fp8(inp["q_idx8"][dev_rows].cpu(), inp["q_scale"][dev_rows].cpu(), w, keys["k_idx8"],
                                keys["k_scale"], rows=rows, cu_q=cu_q, cu_k=cu_k, ld=inp["max_len_k"])
    else:
        sc = oracle.indexer(inp["q_idx"][dev_rows].cpu(), w, keys["k_idx"], rows=rows, cu_q=cu_q, cu_k=cu_k,
                            ld=inp["max_len_k"])
    ix = oracle.topk(sc, inp["topk"], rows=rows, cu_q=cu_q, cu_k=cu_k)
    oracle.sparse_mla(q, keys["kv"], ix, dsa_synth.SM_SCALE, rows=rows, cu_q=cu_q, cu_k=cu_k)


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def _cpu_baseline(inp, n_rows, seed, target_s=12.0):
    """The oracle as it stands on the host cores, on uniformly drawn query rows of the
    same workload.  A first draw of `n_rows` rows calibrates the per-row time; the timed
    sample is then sized to about `target_s` seconds of CPU work."""
    import oracle

    keys = _oracle_inputs_host(inp)
    rng = np.random.default_rng(seed + 1234)
    T = inp["total_q"]
    cal = np.sort(rng.choice(T, size=min(n_rows, T), replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    _oracle_forward_rows(inp, keys, cal)
    per_row = (time.perf_counter() - t0) / len(cal)
    n = int(min(T, max(len(cal), target_s / max(per_row, 1e-6))))
    rows = np.sort(rng.choice(T, size=n, replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    _oracle_forward_rows(inp, keys, rows)
    dt = time.perf_counter() - t0
    return {"value": len(rows) / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "cpu_model": _cpu_model(),
            "sample": f"{len(rows)} uniformly drawn query rows of the same workload (full indexer row, top-k, "
                      f"sparse MLA per row), fp64, {dt:.1f} s of CPU work"}


def run_reference(args, ws, rank, local):
    if rank != 0:
        return
    import oracle

    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    inp = dsa_synth.make_workload(args.workload, seed=args.seed, device=dev)
    keys = _oracle_inputs_host(inp)
    rng = np.random.default_rng(args.seed + 99)
    per_step = min(args.cpu_rows, inp["total_q"])

    def step():
        rows = np.sort(rng.choice(inp["total_q"], size=per_step, replace=False)).astype(np.int64)
        _oracle_forward_rows(inp, keys, rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = per_step * args.steps / dt
    wl = dsa_synth.WORKLOADS[args.workload]
    res = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; same recipe)",
        "config": _config(args, inp, args.chunk if args.chunk is not None else wl.chunk, ws),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "cpu_model": _cpu_model(),
                         "sample": f"{per_step} uniformly drawn query rows per step of the same workload, fp64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(res), flush=True)


def run_kernel(args, local):
    """One kernel entry point on a bounded slice of the workload, for profilers: the
    indexer or top-k on the last (heaviest) chunk of query rows, or the sparse MLA on
    `--rows` query rows (the last ones).  Prints one JSON line with the mean device time."""
    import attention_lightning_indexer_b200 as dsa

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl = dsa_synth.WORKLOADS[args.workload]
    if args.kernel == "cache_write":
        return _run_cache_write(args, dsa, dev)
    need_latent = args.kernel in ("sparse_mla", "dense_mla")
    inp = dsa_synth.make_workload(args.workload, seed=args.seed, device=dev, with_latent=need_latent)
    p = dsa.problem_from_inputs(inp)
    fa = _forward_args(inp)
    T = inp["total_q"]
    rows = min(T, args.rows or (args.chunk or wl.chunk or T))
    r0 = T - rows
    ld = dsa.scores_ld(inp["max_len_k"])
    stream = torch.cuda.current_stream(dev)
    if args.kernel in ("indexer_topk", "indexer_topk_streaming"):
        # the selection of the whole workload in its chunks: two passes through score rows,
        # or the streaming path (no score rows); the same indices either way
        ch = args.chunk or wl.chunk or T
        idx = torch.empty((T, inp["topk"]), dtype=torch.int32, device=dev)
        if args.kernel == "indexer_topk":
            scores = torch.empty((min(ch, T), ld), dtype=torch.float32, device=dev)

            def fn():
                for c0 in range(0, T, ch):
                    rc = min(ch, T - c0)
                    dsa.dsa_indexer_scores(p, fa["q_idx"], fa["k_idx"], inp["w"], scores, row_begin=c0, row_count=rc,
                                           q_scale=fa["q_scale"], k_scale=fa["k_scale"], stream=stream)
                    dsa.dsa_topk(p, scores, idx[c0:c0 + rc], row_begin=c0, row_count=rc, stream=stream)
        else:
            ws_s = torch.empty(dsa.dsa_indexer_topk_streaming_workspace_size(p, ch), dtype=torch.uint8, device=dev)
            fn = lambda: dsa.dsa_indexer_topk_streaming(p, fa["q_idx"], fa["k_idx"], inp["w"], idx, ws_s,
                                                        chunk_q=ch, q_scale=fa["q_scale"], k_scale=fa["k_scale"],
                                                        stream=stream)
        rows, r0 = T, 0
    elif args.kernel in ("indexer", "topk"):
        scores = torch.empty((rows, ld), dtype=torch.float32, device=dev)
        idx = torch.empty((rows, inp["topk"]), dtype=torch.int32, device=dev)
        dsa.dsa_indexer_scores(p, fa["q_idx"], fa["k_idx"], inp["w"], scores, row_begin=r0, row_count=rows,
                               q_scale=fa["q_scale"], k_scale=fa["k_scale"], stream=stream)
        if args.kernel == "indexer":
            fn = lambda: dsa.dsa_indexer_scores(p, fa["q_idx"], fa["k_idx"], inp["w"], scores, row_begin=r0,
                                                row_count=rows, q_scale=fa["q_scale"], k_scale=fa["k_scale"],
                                                stream=stream)
        else:
            fn = lambda: dsa.dsa_topk(p, scores, idx, row_begin=r0, row_count=rows, stream=stream)
    else:
        # index set: the GPU top-k of the GPU scores, chunk by chunk, for the last `rows` rows
        idx = torch.empty((T, inp["topk"]), dtype=torch.int32, device=dev)
        ch = args.chunk or wl.chunk or T
        scores = torch.empty((min(ch, rows), ld), dtype=torch.float32, device=dev)
        for c0 in range(r0, T, ch):
            rc = min(ch, T - c0)
            dsa.dsa_indexer_scores(p, fa["q_idx"], fa["k_idx"], inp["w"], scores, row_begin=c0, row_count=rc,
                                   q_scale=fa["q_scale"], k_scale=fa["k_scale"], stream=stream)
            dsa.dsa_topk(p, scores, idx[c0:c0 + rc], row_begin=c0, row_count=rc, stream=stream)
        del scores
        sub = dsa.make_problem(1, rows, inp["total_k"], rows, inp["max_len_k"], inp["topk"]) if p.cu_q is None else p
        q = inp["q"][r0:]
        out = torch.empty((rows, 128, 512), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((rows, 128), dtype=torch.float32, device=dev)
        ix = idx[r0:]
        if args.kernel == "dense_mla":      # the same attention in the dense (masked MHA) form
            fn = lambda: dsa.dsa_dense_mla_fwd(sub, q, inp["kv"], ix, out, lse, stream=stream)
        else:
            fn = lambda: dsa.dsa_sparse_mla_fwd(sub, q, inp["kv"], ix, out, lse, stream=stream)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize(dev)
    dsa.dsa_check_device_errors()
    ms = a.elapsed_time(b) / args.steps
    print(json.dumps({"kernel": args.kernel, "workload": args.workload, "rows": rows, "row_begin": r0,
                      "ms_per_launch": ms}), flush=True)


def _run_cache_write(args, dsa, dev):
    """The key-cache write of the workload's tokens (all of them), HBM-bound: per token 256 B +
    1152 B read and written."""
    inp = dsa_synth.make_workload(args.workload, seed=args.seed, device=dev, with_latent=True)
    n = inp["total_k"]
    g = torch.Generator(device=dev).manual_seed(args.seed)
    k_raw = torch.randn(n, 128, generator=g, device=dev).to(torch.bfloat16)
    kv_raw = inp["kv"]
    pos = torch.arange(n, dtype=torch.int32, device=dev)
    rows = torch.arange(n, dtype=torch.int32, device=dev)
    ln_w, ln_b = torch.ones(128, device=dev), torch.zeros(128, device=dev)
    rms_w = torch.ones(512, device=dev)
    inv_freq = torch.rand(32, generator=g, device=dev)
    kc = torch.empty(n, 128, dtype=torch.bfloat16, device=dev)
    kvc = torch.empty(n, 576, dtype=torch.bfloat16, device=dev)
    fn = lambda: dsa.dsa_cache_write(k_raw, kv_raw, pos, rows, ln_w, ln_b, rms_w, inv_freq, kc, kvc)  # noqa: E731
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        fn()
    ts = []
    for _ in range(args.steps):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    dsa.dsa_check_device_errors()
    ms = statistics.median(ts)
    nbytes = n * (2 * (128 + 576) * 2 + 8)
    print(json.dumps({"kernel": "cache_write", "workload": args.workload, "tokens": n, "ms_per_launch": ms,
                      "gbs": nbytes / ms / 1e6, "peak_gbs": _peaks()["hbm_gbs"]}), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="prefill_32k", choices=sorted(dsa_synth.WORKLOADS))
    ap.add_argument("--chunk", type=int, default=None, help="query rows per indexer/top-k chunk (0 = all)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-rows", type=int, default=48, help="oracle rows per CPU sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode_b64 secondary measurement")
    ap.add_argument("--e2e-chunk", type=int, default=2048, help="query rows per pipelined chunk of the e2e step")
    ap.add_argument("--kernel", choices=("indexer", "topk", "indexer_topk", "indexer_topk_streaming", "sparse_mla",
                                         "dense_mla", "cache_write"), default=None,
                    help="time one kernel on a bounded slice (for profilers) instead of the full step")
    ap.add_argument("--rows", type=int, default=0, help="query rows for --kernel (default: one chunk)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    ws, rank, local = _dist()
    if args.kernel is not None:
        run_kernel(args, local)
        return
    if args.impl == "reference":
        run_reference(args, ws, rank, local)
        return
    dist = _init_pg(ws, local)
    try:
        run_ours(args, ws, rank, local, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
