"""Helpers for comparing the CUDA library (through its C-ABI binding) with the fp64 oracle.

Inputs come from head_wise_sparse_retrieval_b200.workloads only; the oracle reads host copies
of those same tensors and never anything the CUDA path produced.

Tolerances (fixed by the method's stated bar):
  * selections: the same token sets, except tokens whose fp64 scaled score lies within 1e-5 of
    a bin edge (they may fall on either side in fp32); a different threshold bin is accepted
    only when the oracle's suffix mass at the disputed boundary is within 1e-6 * C_0 of
    p * C_0 ("threshold-ambiguous");
  * outputs, absolute (the method's stated bar): max |gpu - oracle| <= 1e-2 and
    mean |gpu - oracle| <= 1e-3 per head and per layer, against O1 over the oracle's set;
  * outputs, relative (per head, G x 128 values): max |err| <= 1e-2 * max |ref| + 1e-6 and
    mean |err| <= 1e-2 * mean |ref| + 1e-6, against O1 recomputed over the GPU's own set, so
    that a broad head whose output is ~1e-3 in size cannot pass with a wrong or half-sized
    result. The bound comes from the kernel's arithmetic: the softmax weights are rounded to
    bf16 (relative error at most 2^-9, about uniform, so of standard deviation 2^-9/sqrt(3))
    and the normaliser is summed from the same rounded weights, so the output is a convex
    combination with perturbed weights: err = sum_n p_n d_n (v_n - o) / sum_n p_n. For the
    random values of these workloads both err and o scale as sqrt(sum p_n^2) / sum p_n, and
    their ratio is about 2^-9/sqrt(3) = 1.1e-3; 1e-2 leaves a margin of about 9x. A head
    concentrated on a few tokens has |err| <= 2^-9 |v_a - v_b| with |o| of order one.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

import oracle
from head_wise_sparse_retrieval_b200 import rtp
from head_wise_sparse_retrieval_b200 import workloads as W

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
REL = 1e-2
REL_FLOOR = 1e-6
EDGE_TOL = 1e-5
AMBIG_TOL = 1e-6


def u16(t: torch.Tensor) -> np.ndarray:
    return W.to_host_u16(t)


@dataclass
class HeadOracle:
    is_ret: bool
    N: int
    sel: np.ndarray                 # ascending positions (selection or window set)
    out: np.ndarray                 # [G, D] fp64
    scores: np.ndarray | None = None
    hist: oracle.HistSelection | None = None


def oracle_head(li: W.LayerInputs, b: int, kvh: int, is_ret: bool, top_p: float, G: int,
                window: int = 8192, sinks: int = 4, dense: bool = False,
                top_k: int = 0) -> HeadOracle:
    """The oracle's result for one (b, KV head), from host copies of only what it reads."""
    N = int(li.seq_lens[b].item())
    q = u16(li.q[b, kvh * G:(kvh + 1) * G])
    if dense:
        sel = np.arange(N, dtype=np.int64)
        hs, s = None, None
    elif is_ret:
        s = oracle.indexer_scores(u16(li.q_idx[b, kvh]), u16(li.k_idx[b, kvh, :N]), 0.25)
        if top_k > 0:
            hs = oracle.hist_topk(s, top_k)
        else:
            hs = oracle.hist_topp(s, float(np.float32(top_p)))
        sel = hs.sel
    else:
        sel = oracle.window_sink_set(N, window, sinks)
        hs, s = None, None
    rows = torch.as_tensor(sel, device=li.k_cache.device)
    k = u16(li.k_cache[b, kvh].index_select(0, rows))
    v = u16(li.v_cache[b, kvh].index_select(0, rows))
    out = oracle.sparse_attention(q, k, v, np.arange(sel.size), 1.0 / math.sqrt(128))
    return HeadOracle(is_ret, N, sel, out, s, hs)


@dataclass
class SelectionReport:
    n_oracle: int
    n_gpu: int
    n_exact: int
    edge_tokens: int
    ambiguous: bool
    bstar_oracle: int
    bstar_gpu: int


def check_selection(gpu_sel: np.ndarray, gpu_bstar: int, ho: HeadOracle, top_p: float,
                    exact: bool = True) -> SelectionReport:
    s = ho.scores
    hs = ho.hist
    p = float(np.float32(top_p))
    ambiguous = False
    ref_bstar = hs.bstar
    if gpu_bstar != hs.bstar:
        # the suffix mass at the disputed boundary must sit within AMBIG_TOL of p * C_0
        C0 = hs.suffix[0]
        lo_b, hi_b = sorted((gpu_bstar, hs.bstar))
        near = [abs(hs.suffix[b] - p * C0) <= AMBIG_TOL * C0 for b in range(lo_b, hi_b + 1)]
        assert any(near), (f"threshold bin differs: gpu {gpu_bstar}, oracle {hs.bstar}; "
                           f"C_b/C_0 = {[hs.suffix[b] / C0 for b in range(lo_b, hi_b + 1)]}, p={p}")
        ambiguous = True
        ref_bstar = gpu_bstar
    ref = set(np.nonzero(hs.bins >= ref_bstar)[0].tolist())
    got = set(gpu_sel.tolist())
    diff = np.array(sorted(ref ^ got), dtype=np.int64)
    if diff.size:
        s_max = s.max()
        x = (s[diff] - (s_max - 16.0)) * 16.0
        dist = np.abs(x - np.round(x)) / 16.0
        bad = diff[dist >= EDGE_TOL]
        assert bad.size == 0, (f"{bad.size} selection differences away from bin edges, e.g. "
                               f"{bad[:8].tolist()} (oracle bins {hs.bins[bad[:8]].tolist()}, "
                               f"b* {hs.bstar})")
    assert np.all(np.diff(gpu_sel) > 0), "selection must be strictly ascending"
    n_exact = oracle.exact_topp(s, p).size if exact else -1
    return SelectionReport(len(ref), len(got), n_exact, int(diff.size), ambiguous, hs.bstar,
                           gpu_bstar)


def check_selection_topk(gpu_sel: np.ndarray, gpu_bstar: int, ho: HeadOracle,
                         k: int) -> SelectionReport:
    """Fixed top-k: b* is the bin of the k-th highest score, so a different b* is accepted only
    when some token lies within EDGE_TOL of a bin edge between the two (its fp32 bin can
    differ, which moves the counts)."""
    s, hs = ho.scores, ho.hist
    s_max = s.max()
    ambiguous = False
    ref_bstar = hs.bstar
    if gpu_bstar != hs.bstar:
        lo_b, hi_b = sorted((gpu_bstar, hs.bstar))
        edges = (s_max - 16.0) + np.arange(lo_b, hi_b + 2) / 16.0
        near = np.abs(s[:, None] - edges[None, :]).min() < EDGE_TOL
        assert near, f"threshold bin differs: gpu {gpu_bstar}, oracle {hs.bstar}, k={k}"
        ambiguous = True
        ref_bstar = gpu_bstar
    ref = set(np.nonzero(hs.bins >= ref_bstar)[0].tolist())
    got = set(gpu_sel.tolist())
    diff = np.array(sorted(ref ^ got), dtype=np.int64)
    if diff.size:
        x = (s[diff] - (s_max - 16.0)) * 16.0
        dist = np.abs(x - np.round(x)) / 16.0
        bad = diff[dist >= EDGE_TOL]
        assert bad.size == 0, f"{bad.size} selection differences away from bin edges"
    assert np.all(np.diff(gpu_sel) > 0), "selection must be strictly ascending"
    assert len(got) >= min(k, s.size)
    n_exact = oracle.exact_topk(s, k).size
    return SelectionReport(len(ref), len(got), n_exact, int(diff.size), ambiguous, hs.bstar,
                           gpu_bstar)


def check_output(gpu: np.ndarray, ref: np.ndarray, what: str = "",
                 own: np.ndarray | None = None):
    """One head's output ([G, 128]) against the oracle: the absolute bar against ref (O1 over
    the oracle's set) and the relative bar against own (O1 over the GPU's set; ref when the
    sets agree)."""
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    g = gpu.astype(np.float64)
    err = np.abs(g - ref)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e}, mean-abs {mean:.3e}"
    base = ref if own is None else own
    rerr = np.abs(g - base)
    rmx, rmean = float(rerr.max()), float(rerr.mean())
    lim_mx = REL * float(np.abs(base).max()) + REL_FLOOR
    lim_mean = REL * float(np.abs(base).mean()) + REL_FLOOR
    assert rmx <= lim_mx and rmean <= lim_mean, (
        f"{what}: relative bar: max |err| {rmx:.3e} > {lim_mx:.3e} or mean |err| {rmean:.3e} > "
        f"{lim_mean:.3e} (max |ref| {float(np.abs(base).max()):.3e})")
    return mx, mean


def own_set_output(li: W.LayerInputs, b: int, kvh: int, G: int, sel: np.ndarray) -> np.ndarray:
    """O1 recomputed by the oracle over the positions the GPU selected (to tell kernel error
    from a selection that differs at bin edges)."""
    q = u16(li.q[b, kvh * G:(kvh + 1) * G])
    rows = torch.as_tensor(np.asarray(sel, np.int64), device=li.k_cache.device)
    k = u16(li.k_cache[b, kvh].index_select(0, rows))
    v = u16(li.v_cache[b, kvh].index_select(0, rows))
    return oracle.sparse_attention(q, k, v, np.arange(len(sel)), 1.0 / math.sqrt(128))


def make_handle(plan: W.Plan, **cfg_overrides) -> rtp.Handle:
    return rtp.Handle(rtp.config_for(plan, **cfg_overrides), 0)


def run_layer(h: rtp.Handle, plan: W.Plan, li: W.LayerInputs, layer: int, top_p=None,
              dense=False, top_k: int = 0, single_launch: bool = False):
    B, Hq, Hkv = plan.batch, plan.num_q_heads, plan.num_kv_heads
    out = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=li.q.device)
    cnt = torch.full((B, Hkv), -1, dtype=torch.int32, device=li.q.device)
    L = rtp.layer_from(li)
    if dense:
        h.dense_decode(L, out)
    else:
        h.decode_step(layer, L, plan.retrieval[layer], plan.top_p if top_p is None else top_p,
                      out, cnt, top_k=top_k, single_launch=single_launch)
    torch.cuda.synchronize()
    return out, cnt


@dataclass
class LayerReport:
    heads: list = field(default_factory=list)
    max_abs: float = 0.0
    mean_abs: float = 0.0


def check_layer(h: rtp.Handle, plan: W.Plan, li: W.LayerInputs, layer: int, top_p=None,
                heads=None, exact=True, top_k: int = 0,
                single_launch: bool = False) -> LayerReport:
    """Run one layer on the GPU and compare every (or the given) head with the oracle."""
    p = plan.top_p if top_p is None else top_p
    out, cnt = run_layer(h, plan, li, layer, p, top_k=top_k, single_launch=single_launch)
    assert h.device_status() == 0
    G = plan.group
    rep = LayerReport()
    errs = []
    todo = heads if heads is not None else [(b, k) for b in range(plan.batch)
                                            for k in range(plan.num_kv_heads)]
    out_h = out.cpu().numpy()
    cnt_h = cnt.cpu().numpy()
    for b, kvh in todo:
        is_ret = bool(plan.retrieval[layer, kvh])
        ho = oracle_head(li, b, kvh, is_ret, p, G, plan.window, plan.sinks, top_k=top_k)
        info = {"b": b, "kvh": kvh, "ret": is_ret, "n_sel": int(ho.sel.size)}
        if is_ret:
            gsel = h.selection(b, kvh)
            gb, _ = h.threshold(b, kvh)
            if top_k > 0:
                sr = check_selection_topk(gsel, gb, ho, top_k)
            else:
                sr = check_selection(gsel, gb, ho, p, exact=exact)
            info["sel"] = sr
            assert cnt_h[b, kvh] == gsel.size
            own = None
            if sr.edge_tokens == 0 and not sr.ambiguous:
                assert gsel.size == ho.sel.size
            else:  # the sets differ at bin edges: isolate the kernel's error on its own set
                own = own_set_output(li, b, kvh, G, gsel)
                info["own_set"] = True
        else:
            assert cnt_h[b, kvh] == ho.sel.size
            own = None
        g = out_h[b, kvh * G:(kvh + 1) * G]
        mx, mean = check_output(g, ho.out, f"layer {layer} b {b} kvh {kvh}", own)
        errs.append(np.abs(g - ho.out))
        rep.heads.append(info)
    e = np.concatenate([x.ravel() for x in errs])
    rep.max_abs, rep.mean_abs = float(e.max()), float(e.mean())
    assert rep.mean_abs <= MEAN_ABS
    return rep
