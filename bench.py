#!/usr/bin/env python
"""Decode-step benchmark of the RTPurbo attention hot path on B200.

One step = one decode step of the workload: every layer's rtp_decode_step (indexer scoring,
sort-free top-p, compaction, sparse + window attention) for every sequence of the batch.
Prints ONE JSON line (rank 0).

  python bench.py [--gpus N --steps K --warmup W] [--workload ctx_1m] [--top-p 0.9]
  python bench.py --impl reference ...   # the fp64 CPU oracle on the host cores

Timing: the step is captured once as a CUDA graph (all layers), replayed W times untimed,
then K times between CUDA events on the launch stream, bracketed by a barrier and a
device synchronisation; the max over ranks is reported. The step reads several GB from HBM,
far more than the 126 MB L2, so no flush is needed between steps.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode steps/s and effective HBM GB/s (% of roofline) at 128K–1M ctx"
ROW_BYTES = 2 * 128 * 2      # one token's K and V rows (bf16, head_dim 128)
# DRAM traffic of attend_kernel from one ncu capture (the attend_kernel summary under
# profiles/): ctx_1m layer 2, 448.90 MB read + 3.53 MB written for 869 997 tokens x 512 B of
# algorithmic bytes. It is scaled to a bench launch by that launch's algorithmic bytes, and
# reported only while the kernel's sources are the ones that were captured.
ATTEND_NCU = {"source_sha256_16": "d0fb486cbd2e21fb", "traffic_bytes": 448.899328e6 + 3.533312e6,
              "algorithmic_bytes": 869997 * 512}
IDX_BYTES = 16 * 2           # one token's indexer key (fp16, 16 dims)
L2_FLUSH_BELOW = 1 << 30    # steps reading less than this are timed with L2 flushed
BROAD_TOKENS = 16384         # a layer whose retrieval head selects more is a broad-query layer


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
                "samples": len(rows)}


def step_bytes(plan, sel_counts) -> tuple[int, int, int]:
    """Algorithmic HBM bytes of one step: indexer keys of every retrieval head (N x 32 B),
    selected K/V rows (|S| x 512 B) and window K/V rows (|T| x 512 B).
    Returns (total, attend_bytes, indexer_bytes)."""
    idx = att = 0
    for l in range(plan.num_layers):
        for b in range(plan.batch):
            N = int(plan.seq_lens[b])
            for h in range(plan.num_kv_heads):
                att += int(sel_counts[l][b, h]) * ROW_BYTES
                if plan.retrieval[l, h]:
                    idx += N * IDX_BYTES
    return idx + att, att, idx


def exact_top_p_counts(plan, layers, top_p: float) -> list[int]:
    """Size of the exact (sort-based) top-p set of every retrieval head of the workload, for the
    overshoot statistic of the histogram selection: scores 0.25 q_idx . k_idx in fp32, masses
    exp(s - s_max), the shortest prefix of the descending order whose mass reaches p of the total
    (cumulative sums in fp64). A measurement aid run with torch ops, not part of the path."""
    import torch
    out = []
    for l, li in enumerate(layers):
        for b in range(plan.batch):
            N = int(plan.seq_lens[b])
            for h in range(plan.num_kv_heads):
                if not plan.retrieval[l, h]:
                    continue
                k = li.k_idx[b, h, :N].float()
                s = (k @ li.q_idx[b, h].float()) * 0.25
                w = torch.exp(s - s.max()).double()
                c = torch.cumsum(torch.sort(w, descending=True).values, 0)
                out.append(int(torch.searchsorted(c, top_p * c[-1]).item()) + 1)
    return out


def cpu_sample_layers(plan, per_kind: int = 2):
    """A bounded sample of the workload for the CPU oracle (about 10 s of fp64 work at 1M
    context): per_kind layers with a broad (diffuse or flat) retrieval query, with a
    concentrated one and with local heads only."""
    from head_wise_sparse_retrieval_b200 import workloads as W
    pick = []
    for cond in (lambda l: ((plan.kind[l] == W.KIND_DIFFUSE) | (plan.kind[l] == W.KIND_FLAT)).any(),
                 lambda l: (plan.kind[l] == W.KIND_CONC).any(),
                 lambda l: not plan.retrieval[l].any()):
        got = 0
        for l in range(plan.num_layers):
            if got < per_kind and cond(l) and l not in pick:
                pick.append(l)
                got += 1
    return pick or [0]


def oracle_step_bytes(plan, layer_fn):
    """Algorithmic bytes of a full step from the oracle's own token sets: it scores every
    retrieval head and runs the histogram top-p on it; local heads use the window set."""
    import oracle
    from head_wise_sparse_retrieval_b200 import workloads as W
    p = float(np.float32(plan.top_p))
    total = 0
    for l in range(plan.num_layers):
        li = layer_fn(l) if plan.retrieval[l].any() else None
        for b in range(plan.batch):
            N = int(plan.seq_lens[b])
            for h in range(plan.num_kv_heads):
                if plan.retrieval[l, h]:
                    s = oracle.indexer_scores(W.to_host_u16(li.q_idx[b, h]),
                                              W.to_host_u16(li.k_idx[b, h, :N]), 0.25)
                    total += N * IDX_BYTES + oracle.hist_topp(s, p).sel.size * ROW_BYTES
                else:
                    total += oracle.window_sink_set(N, plan.window, plan.sinks).size * ROW_BYTES
        del li
    return total


def oracle_units(plan, layer_fn, layers):
    """Host copies of the sampled layers, cut into one-head units (layer, b, kvh): each is a
    one-KV-head layer for the oracle as it stands (its G query heads, its caches)."""
    from head_wise_sparse_retrieval_b200 import workloads as W
    G = plan.num_q_heads // plan.num_kv_heads
    units = []
    for l in layers:
        li = layer_fn(l)
        q, qi = W.to_host_u16(li.q), W.to_host_u16(li.q_idx)
        kc, vc, ki = W.to_host_u16(li.k_cache), W.to_host_u16(li.v_cache), W.to_host_u16(li.k_idx)
        for b in range(plan.batch):
            N = int(plan.seq_lens[b])
            for h in range(plan.num_kv_heads):
                ret = bool(plan.retrieval[l, h])
                units.append(dict(
                    layer=l, ret=ret, N=N,
                    args=dict(q=q[b:b + 1, h * G:(h + 1) * G], q_idx=qi[b:b + 1, h:h + 1],
                              k_cache=kc[b:b + 1, h:h + 1, :N], v_cache=vc[b:b + 1, h:h + 1, :N],
                              k_idx=ki[b:b + 1, h:h + 1, :N],
                              seq_lens=np.array([N], np.int64),
                              retrieval_mask=np.array([1 if ret else 0], np.uint8))))
        del li
    return units


def oracle_units_run(plan, units, threads):
    """Runs the oracle (fp64 C, one thread per call) over the units on `threads` host threads
    (ctypes releases the GIL in the calls). Returns (wall seconds, algorithmic bytes)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    p = float(np.float32(plan.top_p))

    def one(u):
        _, nsel = oracle.decode_layer(**u["args"], top_p=p, window=plan.window, sinks=plan.sinks,
                                      num_threads=1)
        return int(nsel[0, 0]) * ROW_BYTES + (u["N"] * IDX_BYTES if u["ret"] else 0)

    # the longest units first, so that the pool does not end on one of them
    order = sorted(units, key=lambda u: -(u["N"] if u["ret"] else min(u["N"], plan.window)))
    t = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        nbytes = sum(ex.map(one, order))
    return time.perf_counter() - t, nbytes


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def attend_source_hash() -> str:
    """Hash of the attention kernel's sources (the kernel and its tile step), to tell whether
    the recorded ncu traffic still describes the kernel that runs."""
    import hashlib
    h = hashlib.sha256()
    for f in ("attend_kernel.cu", "attend_tile.cuh"):
        with open(os.path.join(ROOT, "head_wise_sparse_retrieval_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def step_read_bytes(plan) -> int:
    """An upper bound of the bytes a step reads, from the shapes alone: every retrieval head's
    indexer keys and all of its N tokens, every local head's window set."""
    total = 0
    for l in range(plan.num_layers):
        for b in range(plan.batch):
            N = int(plan.seq_lens[b])
            for h in range(plan.num_kv_heads):
                if plan.retrieval[l, h]:
                    total += N * (IDX_BYTES + ROW_BYTES)
                else:
                    total += min(N, plan.window + plan.sinks) * ROW_BYTES
    return total


def prefill_key_counts(plan, masks: dict, T: int, dense: bool) -> tuple[int, int]:
    """(rows, fills) of a T-token prompt through every layer: rows = the sum over prompt rows of
    their key-set sizes (i + 1, or at most window + sinks for a local head): the attention's
    work; fills = the key rows gathered into shared memory, one union set per pair of rows."""
    W, S = plan.window, plan.sinks
    n = np.arange(1, T + 1, dtype=np.int64)
    rows_full, rows_win = int(n.sum()), int(np.minimum(n, W + S).sum())
    lo = np.arange(0, T, 2, dtype=np.int64)
    hi = np.minimum(lo + 1, T - 1)
    fill_full = int((hi + 1).sum())
    fill_win = int(np.where(lo + 1 > W + S, S + W + (hi - lo), hi + 1).sum())
    B, Hkv = plan.batch, plan.num_kv_heads
    if dense:
        k = plan.num_layers * B * Hkv
        return k * rows_full, k * fill_full
    rows = fills = 0
    for m, ls in masks.items():
        nret = int(np.frombuffer(m, np.uint8).astype(bool).sum())
        rows += len(ls) * B * (nret * rows_full + (Hkv - nret) * rows_win)
        fills += len(ls) * B * (nret * fill_full + (Hkv - nret) * fill_win)
    return rows, fills


def prefill_leg(h, plan, kcache, vcache, dev, stream, T: int) -> dict:
    """A T-token prompt through every layer (rtp_prefill with the layer's retrieval mask), and the
    same with every head dense (the kernel's full causal attention): one call per distinct mask,
    timed with CUDA events on the launch stream after a warm-up call, summed over the layers."""
    import torch
    B, Hq, Hkv, L = plan.batch, plan.num_q_heads, plan.num_kv_heads, plan.num_layers
    gen = torch.Generator(device=dev).manual_seed(7)
    q = torch.randn(B, Hq, T, 128, generator=gen, device=dev).to(torch.bfloat16)
    out = torch.empty(B, Hq, T, 128, dtype=torch.float32, device=dev)
    seq = torch.full((B,), T, dtype=torch.int32, device=dev)
    masks = {}
    for l in range(L):
        masks.setdefault(bytes(plan.retrieval[l].astype(np.uint8)), []).append(l)

    def timed(mask, dense):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            h.prefill(q, kcache, vcache, seq, mask, out, dense=dense, stream=stream)
            e0.record(stream)
            h.prefill(q, kcache, vcache, seq, mask, out, dense=dense, stream=stream)
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    per_mask = {m: timed(np.frombuffer(m, np.uint8).copy(), False) for m in masks}
    sparse_ms = sum(per_mask[m] * len(ls) for m, ls in masks.items())
    dense_ms = timed(np.zeros(Hkv, np.uint8), True) * L
    rows_s, fills_s = prefill_key_counts(plan, masks, T, False)
    rows_d, fills_d = prefill_key_counts(plan, masks, T, True)
    flop_per_row = 2 * 2 * (Hq // Hkv) * 128  # S = K Q^T and O += V^T P^T, per query head
    return {"prompt_tokens": T, "layers": L, "ms_sparse": sparse_ms, "ms_dense": dense_ms,
            "speedup_vs_dense": dense_ms / sparse_ms,
            "per_layer_ms": {"".join(str(x) for x in m): per_mask[m] for m in masks},
            "smem_fill_tbs": {"sparse": fills_s * ROW_BYTES / (sparse_ms * 1e-3) / 1e12,
                              "dense": fills_d * ROW_BYTES / (dense_ms * 1e-3) / 1e12},
            "tflops": {"sparse": rows_s * flop_per_row / (sparse_ms * 1e-3) / 1e12,
                       "dense": rows_d * flop_per_row / (dense_ms * 1e-3) / 1e12},
            "kernel": "prefill_kernel",
            "note": ("each pair of prompt rows gathers the union of its key sets from L2 into "
                     "shared memory once per KV head; the pages quote their prefill speed-up "
                     "against FlashAttention-2 on H20 (2.83x at 32K), context only")}


def config_of(plan, world: int) -> dict:
    """The workload both arms measure (the same keys and values for the GPU arm and the
    reference arm); how each arm times it is reported under "protocol"."""
    return {"workload": plan.name, "layers": plan.num_layers, "batch": plan.batch,
            "ctx": plan.ctx, "q_heads": plan.num_q_heads, "kv_heads": plan.num_kv_heads,
            "head_dim": 128, "idx_dim": 16, "retrieval_kv_heads": int(plan.retrieval.sum()),
            "top_p": plan.top_p, "window": plan.window, "sinks": plan.sinks,
            "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": (f"L2 (126 MB) flushed before every timed step: a step reads less than "
                   f"{L2_FLUSH_BELOW >> 20} MB" if step_read_bytes(plan) < L2_FLUSH_BELOW else
                   "no flush: a step reads far more than the 126 MB L2")}


def dist_env() -> tuple[int, int, int]:
    """(world, rank, local rank) as torchrun sets them; (1, 0, 0) without torchrun."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(local: int):
    """One process per GPU over NCCL (gloo when no GPU is visible, for the host-side tests),
    with a short timeout so that ranks waiting on a dead peer end with an error."""
    import datetime
    import torch
    import torch.distributed as dist
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    else:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of x over all ranks (x itself on one rank): a multi-GPU step takes as long as
    its slowest replica."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world: int, ms_per_step: float) -> float:
    """Whole-job decode steps per second: every rank decodes its own step (replicas), so the
    job finishes world steps per max-over-ranks step time."""
    return world * 1e3 / ms_per_step


def run_reference(args, plan, rank, world):
    """--impl reference: the fp64 CPU oracle on the host cores, each step a bounded sample of
    the same workload (one sampled layer), its time scaled to a full step by bytes."""
    if rank != 0:
        return
    import torch
    import oracle
    from head_wise_sparse_retrieval_b200 import workloads as W
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    layers = cpu_sample_layers(plan)  # two of each kind: more one-head units than host threads
    threads = oracle.max_threads()
    layer_fn = lambda l: W.make_layer(plan, l, dev)
    full = oracle_step_bytes(plan, layer_fn)
    units = oracle_units(plan, layer_fn, layers)
    cores = min(threads, len(units))
    times = []
    for i in range(args.warmup + args.steps):
        secs, nbytes = oracle_units_run(plan, units, threads)
        if i >= args.warmup:
            times.append(secs * full / max(nbytes, 1))
    sec_per_step = float(np.mean(times))
    value = 1.0 / sec_per_step
    sample = (f"each step: layers {layers} of {plan.name} (broad-query, concentrated-query, "
              f"local-only), {len(units)} one-head units over {cores} host threads "
              f"({cpu_model()}); fp64 oracle wall time scaled to a full step by algorithmic "
              f"bytes ({full} B per step from the oracle's own selections)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec_per_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(plan, world),
            "protocol": {"timing": "host wall clock around the oracle calls of each step",
                         "sample": "bounded sample of the workload, scaled by bytes"},
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores,
                             "kind": "oracle", "sample": sample, "cpu_model": cpu_model(),
                             "host_threads": threads},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["rtp", "reference"], default="rtp")
    ap.add_argument("--workload", default="ctx_1m",
                    choices=["tiny", "one_layer", "batch_decode", "long_context", "ctx_1m"])
    ap.add_argument("--top-p", type=float, default=None)
    ap.add_argument("--layers", type=int, default=None, help="fewer layers (debug only)")
    ap.add_argument("--ctx", type=int, default=None, help="other context length (debug only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--p-sweep", default="0.8,0.95",
                    help="other top-p values timed the same way (comma list; empty: none)")
    ap.add_argument("--k-sweep", default="2048,4096,16384",
                    help="fixed top-k values (through the same histogram) timed the same way")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--prefill-t", type=int, default=32768,
                    help="prompt length of the prefill leg (the pages' prefill table starts at 32K)")
    ap.add_argument("--single-layer", type=int, default=None,
                    help="profiling case: only this layer of the workload, decoded --reps times")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--single-launch", action="store_true",
                    help="--single-layer: run the layer as one fused launch")
    ap.add_argument("--prefill-case", type=int, default=None,
                    help="profiling case: rtp_prefill of a prompt of this many tokens with the "
                         "mask of the workload's first layer that has a retrieval head, --reps "
                         "calls")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    import torch
    import torch.distributed as dist
    from head_wise_sparse_retrieval_b200 import rtp
    from head_wise_sparse_retrieval_b200 import workloads as W

    world, rank, local = dist_env()
    if world > 1:
        init_dist(local)

    plan = W.plan(args.workload, top_p=args.top_p, num_layers=args.layers, ctx=args.ctx)

    if args.impl == "reference":
        run_reference(args, plan, rank, world)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return

    rtp.load()
    dev = torch.device("cuda", local if world > 1 else 0)
    if args.prefill_case is not None:  # small case for ncu captures of the prefill kernel
        T = args.prefill_case
        B, Hq, Hkv = plan.batch, plan.num_q_heads, plan.num_kv_heads
        l = next(i for i in range(plan.num_layers) if plan.retrieval[i].any())
        gen = torch.Generator(device=dev).manual_seed(T)
        q = torch.randn(B, Hq, T, 128, generator=gen, device=dev).to(torch.bfloat16)
        k = torch.randn(B, Hkv, T, 128, generator=gen, device=dev).to(torch.bfloat16)
        v = torch.randn(B, Hkv, T, 128, generator=gen, device=dev).to(torch.bfloat16)
        seq = torch.full((B,), T, dtype=torch.int32, device=dev)
        out = torch.empty(B, Hq, T, 128, dtype=torch.float32, device=dev)
        h = rtp.Handle(rtp.config_for(plan, max_ctx=T), dev.index)
        for _ in range(args.reps):
            h.prefill(q, k, v, seq, plan.retrieval[l], out)
        torch.cuda.synchronize()
        status = h.device_status()
        h.close()
        print(json.dumps({"prefill_case": T, "workload": plan.name, "mask_of_layer": l,
                          "retrieval": plan.retrieval[l].tolist(), "reps": args.reps,
                          "device_status": status}))
        if status:
            raise SystemExit(1)
        return
    if args.single_layer is not None:  # small case for ncu captures (one layer, a few calls)
        l = args.single_layer
        li = W.make_layer(plan, l, dev)
        h = rtp.Handle(rtp.config_for(plan), dev.index)
        out = torch.empty((plan.batch, plan.num_q_heads, 128), dtype=torch.float32, device=dev)
        cnt = torch.empty((plan.batch, plan.num_kv_heads), dtype=torch.int32, device=dev)
        for _ in range(args.reps):
            h.decode_step(l, rtp.layer_from(li), plan.retrieval[l], plan.top_p, out, cnt,
                          single_launch=args.single_launch)
        torch.cuda.synchronize()
        status = h.device_status()
        h.close()
        print(json.dumps({"single_layer": l, "workload": plan.name, "reps": args.reps,
                          "retrieval": plan.retrieval[l].tolist(),
                          "token_sets": cnt.cpu().tolist(), "device_status": status}))
        if status:
            raise SystemExit(1)
        return
    torch.cuda.set_device(dev)
    L, B, Hq, Hkv = plan.num_layers, plan.batch, plan.num_q_heads, plan.num_kv_heads

    t_gen = time.perf_counter()
    layers = [W.make_layer(plan, l, dev) for l in range(L)]
    torch.cuda.synchronize()
    t_gen = time.perf_counter() - t_gen
    outs = [torch.empty((B, Hq, 128), dtype=torch.float32, device=dev) for _ in range(L)]
    cnts = [torch.empty((B, Hkv), dtype=torch.int32, device=dev) for _ in range(L)]
    h = rtp.Handle(rtp.config_for(plan), dev.index)
    views = [rtp.layer_from(li) for li in layers]
    stream = torch.cuda.Stream(device=dev)

    def step(dense=False):
        for l in range(L):
            if dense:
                h.dense_decode(views[l], outs[l], stream=stream)
            else:
                h.decode_step(l, views[l], plan.retrieval[l], plan.top_p, outs[l], cnts[l],
                              stream=stream)

    # eager step: checks the path end to end and gives the token-set sizes
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    status = h.device_status()
    if status:
        raise SystemExit(f"device status 0x{status:x} after the eager step")
    sel = [c.cpu().numpy() for c in cnts]
    total_bytes, attend_bytes, idx_bytes = step_bytes(plan, sel)

    # capture the whole step as one CUDA graph
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    with torch.cuda.stream(stream):  # a graph replays on the current stream
        for _ in range(args.warmup):
            g.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(dev.index if world == 1 else local)
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    # A step that reads less than several times the 126 MB L2 could find part of its inputs
    # still in L2 from the previous replay: then L2 is flushed (a 512 MB write) before every
    # timed replay, outside its event pair. Larger steps are timed back to back. The rule uses
    # the shapes only (step_read_bytes), so both arms state the same in their config.
    flush = step_read_bytes(plan) < L2_FLUSH_BELOW
    scratch = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if flush else None
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        if flush:
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for a0, a1 in ev:
                scratch.fill_(1)
                a0.record(stream)
                g.replay()
                a1.record(stream)
        else:
            e0.record(stream)
            for _ in range(args.steps):
                g.replay()
            e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if rank == 0 else {}
    step_ms = (sum(a0.elapsed_time(a1) for a0, a1 in ev) if flush
               else e0.elapsed_time(e1)) / args.steps
    ms = max_over_ranks(step_ms, world, dev)
    del g, scratch

    # per-kernel durations (CUDA events around each launch on the launch stream), read layer
    # by layer so that they can be split by layer class as well
    def layer_class(l):
        ret = plan.retrieval[l].astype(bool)
        if not ret.any():
            return "local_only"
        big = max(int(sel[l][b, k]) for b in range(B) for k in range(Hkv) if ret[k])
        return "broad_retrieval" if big > BROAD_TOKENS else "concentrated_retrieval"

    h.profile(True)
    prof_steps = max(3, min(args.steps, 10))
    acc = {k: [0.0, 0] for k in rtp.KERNEL_CLASSES}
    by_class = {}
    for _ in range(prof_steps):
        with torch.cuda.stream(stream):
            step()
        # in launch order, per layer: [select,] attend[, merge] (a layer of local heads only is
        # one attention launch that merges inside, when the handle has its cluster size)
        launches = h.profile_launches()
        at = 0
        for l in range(L):
            got = []  # this layer's launches: [select,] attend[, merge]
            while at < len(launches):
                kind, t_ms = launches[at]
                if got and got[-1][0] in ("attend", "fused") and kind != "merge":
                    break  # the next layer's first launch
                at += 1
                got.append((kind, t_ms))
                if kind == "merge":
                    break  # the layer's last launch
            # a local-only layer without a merge launch ran as one cluster launch
            name = layer_class(l)
            if name == "local_only" and all(k != "merge" for k, _ in got):
                name = "local_only_cluster"
            c = by_class.setdefault(name, {"attend_ms": 0.0, "attend_n": 0, "attend_bytes": 0,
                                           "select_ms": 0.0, "select_n": 0, "select_bytes": 0})
            for kind, t_ms in got:
                acc[kind][0] += t_ms
                acc[kind][1] += 1
                if kind == "select":
                    c["select_ms"] += t_ms
                    c["select_n"] += 1
                    c["select_bytes"] += sum(int(plan.seq_lens[b]) * IDX_BYTES for b in range(B)
                                             for k in range(Hkv) if plan.retrieval[l, k])
                elif kind == "attend":
                    c["attend_ms"] += t_ms
                    c["attend_n"] += 1
                    c["attend_bytes"] += int(sel[l].sum()) * ROW_BYTES
    h.profile(False)
    kern = {k: {"ms_total_per_step": v[0] / prof_steps, "launches_per_step": v[1] / prof_steps}
            for k, v in acc.items() if v[1]}
    # launches of the step as counted by the library's per-launch events ([select,] attend
    # [, merge] per layer: the merge folds into the attention launch when its grid fits at once)
    launches_per_step = round(sum(v[1] for v in acc.values()) / prof_steps)
    # the dominant kernel, attend_kernel: the attention launches of every layer that did not run
    # as one cluster launch
    split = [c for n, c in by_class.items() if n != "local_only_cluster"]
    att_n = sum(c["attend_n"] for c in split)
    att_ms = sum(c["attend_ms"] for c in split) / max(att_n, 1)
    att_bytes_per_launch = sum(c["attend_bytes"] for c in split) / max(att_n, 1)
    hbm, peak_kind = _peaks()
    att_gbs = att_bytes_per_launch / (att_ms * 1e-3) / 1e9
    # the attention launches split by layer class, and the selection launches (indexer keys)
    classes = {}
    sel_ms = sel_n = sel_b = 0
    for name, c in sorted(by_class.items()):
        if c["attend_n"]:
            per_ms = c["attend_ms"] / c["attend_n"]
            per_b = c["attend_bytes"] / c["attend_n"]
            gbs = per_b / (per_ms * 1e-3) / 1e9
            classes[("head_cluster_kernel_local_only" if name == "local_only_cluster"
                     else "attend_" + name)] = {
                "launches_per_step": c["attend_n"] / prof_steps, "per_launch_ms": per_ms,
                "algorithmic_bytes_per_launch": per_b, "achieved": gbs, "frac": gbs / hbm}
        sel_ms += c["select_ms"]
        sel_n += c["select_n"]
        sel_b += c["select_bytes"]
    if sel_n:
        per_ms, per_b = sel_ms / sel_n, sel_b / sel_n
        gbs = per_b / (per_ms * 1e-3) / 1e9
        classes["select_kernel"] = {"launches_per_step": sel_n / prof_steps,
                                    "per_launch_ms": per_ms, "algorithmic_bytes_per_launch": per_b,
                                    "achieved": gbs, "frac": gbs / hbm}
    traffic = None
    if attend_source_hash() == ATTEND_NCU["source_sha256_16"]:
        traffic = att_bytes_per_launch * ATTEND_NCU["traffic_bytes"] / ATTEND_NCU["algorithmic_bytes"]

    # the same step at other p (the 1M-context configuration sweeps p over 0.8 / 0.9 / 0.95)
    # and with the fixed top-k of the pages' top-k / top-p comparison (2k / 4k / 16k)
    def time_variant(pv, kv, ready=False, single=False):
        def run():
            for l in range(L):
                h.decode_step(l, views[l], plan.retrieval[l], pv, outs[l], cnts[l],
                              stream=stream, top_k=kv, inputs_ready=ready, single_launch=single)
        with torch.cuda.stream(stream):
            run()
        torch.cuda.synchronize()
        sel_v = [c.cpu().numpy() for c in cnts]
        bytes_v = step_bytes(plan, sel_v)[0]
        gv = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gv, stream=stream):
            run()
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                gv.replay()
        torch.cuda.synchronize()
        v0 = torch.cuda.Event(enable_timing=True)
        v1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        with torch.cuda.stream(stream):
            v0.record(stream)
            for _ in range(args.steps):
                gv.replay()
            v1.record(stream)
        torch.cuda.synchronize()
        vms = max_over_ranks(v0.elapsed_time(v1) / args.steps, world, dev)
        n_v = [int(x[b, k]) for l, x in enumerate(sel_v) for b in range(B) for k in range(Hkv)
               if plan.retrieval[l, k]]
        del gv
        return {"ms_per_step": vms, "steps_per_s": throughput(world, vms),
                "effective_gbs": bytes_v / (vms * 1e-3) / 1e9,
                "roofline_frac_step": bytes_v / (vms * 1e-3) / 1e9 / hbm,
                "algorithmic_bytes_per_step": bytes_v,
                "mean_selected": float(np.mean(n_v)) if n_v else 0.0}

    p_sweep = {ps.strip(): time_variant(float(ps), 0)
               for ps in args.p_sweep.split(",") if ps.strip()}
    k_sweep = {ks.strip(): time_variant(plan.top_p, int(ks))
               for ks in args.k_sweep.split(",") if ks.strip()}
    # the same step with rtp_layer_io.inputs_ready: every input is resident before the step,
    # so each layer's scoring / local attention streams while the previous launch drains
    chained = time_variant(plan.top_p, 0, ready=True)
    # the same step with every layer as one fused launch (rtp_layer_io.single_launch)
    try:
        single = time_variant(plan.top_p, 0, single=True)
    except rtp.RtpError as e:  # shapes beyond the single-launch limits
        single = {"unsupported": str(e)}

    # indexer production of one layer (q_idx and the new k_idx row of every KV head), timed as a
    # CUDA graph of 100 calls; W is random (no trained weights), the row goes to a scratch cache
    G = Hq // Hkv
    gen = torch.Generator(device=dev).manual_seed(99)
    q_pre = torch.randn(B, Hq, 128, generator=gen, device=dev).to(torch.bfloat16)
    k_pre = torch.randn(B, Hkv, 128, generator=gen, device=dev).to(torch.bfloat16)
    w_q = (0.03 * torch.randn(Hkv, 16, G * 128, generator=gen, device=dev)).to(torch.bfloat16)
    w_k = (0.1 * torch.randn(Hkv, 16, 128, generator=gen, device=dev)).to(torch.bfloat16)
    qi_s = torch.empty(B, Hkv, 16, dtype=torch.float16, device=dev)
    ki_s = torch.empty(B, Hkv, plan.max_ctx, 16, dtype=torch.float16, device=dev)
    seq_d = layers[0].seq_lens
    with torch.cuda.stream(stream):
        h.indexer_append(q_pre, k_pre, w_q, w_k, seq_d, qi_s, ki_s, stream=stream)
    torch.cuda.synchronize()
    gi = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gi, stream=stream):
        for _ in range(100):
            h.indexer_append(q_pre, k_pre, w_q, w_k, seq_d, qi_s, ki_s, stream=stream)
    with torch.cuda.stream(stream):
        gi.replay()
        i0 = torch.cuda.Event(enable_timing=True)
        i1 = torch.cuda.Event(enable_timing=True)
        i0.record(stream)
        gi.replay()
        i1.record(stream)
    torch.cuda.synchronize()
    ius = i0.elapsed_time(i1) * 1e3 / 100
    ibytes = 2 * (w_q.numel() + w_k.numel() + q_pre.numel() + k_pre.numel() + 2 * B * Hkv * 16)
    indexer = {"us_per_call": ius, "bytes_per_call": ibytes,
               "effective_gbs": ibytes / (ius * 1e-6) / 1e9,
               "shape": {"batch": B, "q_heads": Hq, "kv_heads": Hkv, "r": 16}}
    del gi, ki_s

    # prefill of a prompt through every layer's mask, against dense prefill on the same kernel
    prefill = None
    if not args.no_prefill and args.prefill_t <= plan.max_ctx:
        prefill = prefill_leg(h, plan, layers[0].k_cache, layers[0].v_cache, dev, stream,
                              args.prefill_t)

    # dense decode on the same caches (the speedup denominator)
    dense = None
    if not args.no_dense:
        gd = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gd, stream=stream):
            step(dense=True)
        with torch.cuda.stream(stream):
            for _ in range(3):
                gd.replay()
        torch.cuda.synchronize()
        nd = max(3, min(args.steps, 5))
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            d0.record(stream)
            for _ in range(nd):
                gd.replay()
            d1.record(stream)
        torch.cuda.synchronize()
        dms = d0.elapsed_time(d1) / nd
        dense_bytes = sum(int(plan.seq_lens[b]) * ROW_BYTES for b in range(B)) * Hkv * L
        dense = {"ms_per_step": dms, "speedup": dms / ms,
                 "effective_gbs": dense_bytes / (dms * 1e-3) / 1e9}
        del gd

    # end to end through the host-buffer entry point: pinned host queries in, outputs out
    e2e = None
    if not args.no_e2e:
        q_h = torch.stack([li.q for li in layers]).cpu().pin_memory()
        qi_h = torch.stack([li.q_idx for li in layers]).cpu().pin_memory()
        seq_h = layers[0].seq_lens.cpu().pin_memory()
        out_h = torch.empty((L, B, Hq, 128), dtype=torch.float32).pin_memory()
        masks = plan.retrieval.astype(np.uint8)
        for _ in range(2):
            h.decode_step_host(q_h, qi_h, seq_h, views, masks, plan.top_p, out_h, stream=stream)
        ne = max(3, min(args.steps, 10))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        x0 = torch.cuda.Event(enable_timing=True)
        x1 = torch.cuda.Event(enable_timing=True)
        x0.record(stream)
        for _ in range(ne):
            h.decode_step_host(q_h, qi_h, seq_h, views, masks, plan.top_p, out_h, stream=stream)
        x1.record(stream)
        torch.cuda.synchronize()
        xms = max_over_ranks(x0.elapsed_time(x1) / ne, world, dev)
        e2e = {"value": throughput(world, xms), "unit": "steps/s",
               "h2d_bytes_per_step": int(q_h.numel() * 2 + qi_h.numel() * 2 + seq_h.numel() * 4),
               "d2h_bytes_per_step": int(out_h.numel() * 4), "ms_per_step": xms}

    # CPU baseline: the oracle on a bounded sample of the workload (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        picks = cpu_sample_layers(plan)
        threads = oracle.max_threads()
        full = oracle_step_bytes(plan, lambda l: layers[l])
        units = oracle_units(plan, lambda l: layers[l], picks)
        secs, sbytes = oracle_units_run(plan, units, threads)
        del units
        est = secs * full / max(sbytes, 1)
        cpu = {"value": 1.0 / est, "unit": "steps/s",
               "cores": int(min(threads, len(picks) * B * Hkv)), "kind": "oracle",
               "sample": (f"layers {picks} of {plan.name} (broad-query, concentrated-query and "
                          f"local-only layers) as {len(picks) * B * Hkv} one-head units on "
                          f"{threads} host threads, {secs:.1f} s of fp64 oracle wall time, "
                          f"scaled to a full step by algorithmic bytes"),
               "cpu_model": cpu_model(), "host_threads": threads}

    value = throughput(world, ms)
    eff_gbs = total_bytes / (ms * 1e-3) / 1e9
    n_sel = [int(s[b, k]) for l, s in enumerate(sel) for b in range(B) for k in range(Hkv)
             if plan.retrieval[l, k]]
    n_exact = exact_top_p_counts(plan, layers, plan.top_p) if n_sel else []
    over = [a - e for a, e in zip(n_sel, n_exact)]
    over_rel = [a / e - 1.0 for a, e in zip(n_sel, n_exact)]
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_of(plan, world),
        "protocol": {"timing": "CUDA graph of all layers, CUDA events on the launch stream"},
        "effective_gbs": eff_gbs,
        "roofline_frac_step": eff_gbs / hbm,
        # the same against the data-sheet HBM3e figure of a B200 (8 TB/s), for context
        "roofline_frac_step_nominal_8tbs": eff_gbs / 8000.0,
        "algorithmic_bytes_per_step": total_bytes,
        "bytes_breakdown": {"indexer": idx_bytes, "attend_kv": attend_bytes},
        "roofline": {"bound": "hbm", "kernel": "attend_kernel", "achieved": att_gbs,
                     "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": att_gbs / hbm, "traffic": traffic,
                     "per_launch_ms": att_ms, "algorithmic_bytes_per_launch": att_bytes_per_launch,
                     "classes": classes,
                     "class_rule": (f"broad_retrieval: a retrieval head selected more than "
                                    f"{BROAD_TOKENS} tokens; concentrated_retrieval: retrieval "
                                    f"heads all at or below; local_only: no retrieval head "
                                    f"(head_cluster_kernel when such a layer runs as one "
                                    f"cluster launch)")},
        "kernels": kern,
        "selection": {"retrieval_heads": len(n_sel),
                      "mean_selected": float(np.mean(n_sel)) if n_sel else 0.0,
                      "max_selected": int(max(n_sel)) if n_sel else 0,
                      "mean_exact_top_p": float(np.mean(n_exact)) if n_exact else 0.0,
                      "overshoot_tokens_mean": float(np.mean(over)) if over else 0.0,
                      "overshoot_rel_mean": float(np.mean(over_rel)) if over_rel else 0.0},
        "p_sweep": p_sweep,
        "k_sweep": k_sweep,
        "chained": chained,
        "single_launch": single,
        "indexer_append": indexer,
        "prefill": prefill,
        "dense": dense,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "setup_s": t_gen,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    h.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
