"""Seeded synthetic inputs for the decode-step attention (shared by the tests and bench.py).

This module only draws inputs. It holds none of the method's arithmetic: no indexer score,
histogram, selection or attention is computed here. The shapes follow the five workloads
the method is measured on (names below); the value distributions follow the pages' own
descriptions of the two query regimes (xllm-io paper review, section 三 "洞察 3: 动态 Top-P
选择", Figures 3(a) and 3(b)): a broad query whose mass spreads over thousands of tokens,
and a needle-in-a-haystack query where a few tokens carry nearly all of it.

Recipe (per layer, seeded by (workload seed, layer)):
  * K, V caches: bf16 ~ N(0, 1), layout [B, Hkv, max_ctx, 128];
  * queries q: bf16 ~ N(0, 1), layout [B, Hq, 128];
  * indexer keys: fp16 ~ N(0, 1), layout [B, Hkv, max_ctx, 16];
  * indexer query of a retrieval head: q_idx = 4 * sigma * u (u a random unit vector), so that
    with the 1/4 indexer scale the background scores are N(0, sigma^2):
      - "conc":    sigma = 1 and n needles whose keys are alpha * (0.9 u + sqrt(0.19) w), w a
                   random unit vector orthogonal to u; alpha is set in closed form from the
                   expected background mass N * exp(1/2) so that the needles carry about 97%
                   of the mass (the pages' NIAH example has 2 tokens carrying 96.6%);
      - "diffuse": sigma = 2.39 (about 8k tokens for 90% of the mass at 64K context, the
                   pages' broad query needs ~8.5k);
      - "flat":    sigma = 0.5 (near-uniform mass; the bandwidth worst case);
  * positions >= seq_len may be poisoned with NaN so that any read past the context shows.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

KIND_LOCAL, KIND_CONC, KIND_DIFFUSE, KIND_FLAT = 0, 1, 2, 3
KIND_NAMES = {KIND_LOCAL: "local", KIND_CONC: "conc", KIND_DIFFUSE: "diffuse", KIND_FLAT: "flat"}
SIGMA = {KIND_CONC: 1.0, KIND_DIFFUSE: 2.39, KIND_FLAT: 0.5}
NEEDLE_MASS = 0.97
NEEDLE_COS = 0.9


@dataclass
class Plan:
    """Structure of one workload: shapes, head roles and query regimes (all host-side)."""
    name: str
    num_layers: int
    batch: int
    num_q_heads: int
    num_kv_heads: int
    ctx: int
    max_ctx: int
    top_p: float
    seed: int
    head_dim: int = 128
    idx_dim: int = 16
    window: int = 8192
    sinks: int = 4
    retrieval: np.ndarray = field(default=None)   # [L, Hkv] uint8
    kind: np.ndarray = field(default=None)        # [L, B, Hkv] int8 (KIND_*)
    n_needles: np.ndarray = field(default=None)   # [L, B, Hkv] int32 (conc heads)
    seq_lens: np.ndarray = field(default=None)    # [B] int64

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def describe(self) -> dict:
        kinds = {KIND_NAMES[k]: int((self.kind == k).sum()) for k in (1, 2, 3)}
        return {
            "workload": self.name, "layers": self.num_layers, "batch": self.batch,
            "q_heads": self.num_q_heads, "kv_heads": self.num_kv_heads,
            "head_dim": self.head_dim, "idx_dim": self.idx_dim, "ctx": self.ctx,
            "window": self.window, "sinks": self.sinks, "top_p": self.top_p,
            "retrieval_kv_heads": int(self.retrieval.sum()), "query_kinds": kinds,
            "seed": self.seed,
        }


def _rng(seed: int, *salt: int) -> np.random.Generator:
    return np.random.default_rng([seed, *salt])


def plan(name: str, *, top_p: float | None = None, ctx: int | None = None,
         num_layers: int | None = None, query: str | None = None,
         seq_lens: list[int] | None = None) -> Plan:
    """The five workloads:

    tiny          1 layer, B=1, 8 q / 1 KV head, N=4096, one retrieval head, 3 needles, seed 0
    one_layer     1 layer, B=1, 32 q / 4 KV, N=65536; KV head 0 retrieval, 1-3 local; the query
                  is "conc" (2-8 needles), "diffuse" or "flat" (``query=``), seed 1
    batch_decode  1 layer, B=8, 32 q / 4 KV, N=131072, KV head 0 retrieval with 1-64 needles
                  per sequence, seed 2
    long_context  48 layers, B=2, 32 q / 4 KV, N=524288, 29 of 192 KV heads retrieval (by
                  seed); half the retrieval queries conc, half diffuse, seed 3
    ctx_1m        48 layers, B=1, 32 q / 4 KV, N=1048576, 29 retrieval heads; 14 flat and 15
                  conc; p in {0.8, 0.9, 0.95}, seed 4
    """
    if name == "tiny":
        p = Plan(name, 1, 1, 8, 1, 4096, 4096, 0.9, 0)
        p.retrieval = np.ones((1, 1), np.uint8)
        p.kind = np.full((1, 1, 1), KIND_CONC, np.int8)
        p.n_needles = np.full((1, 1, 1), 3, np.int32)
    elif name == "one_layer":
        p = Plan(name, 1, 1, 32, 4, 65536, 65536, 0.9, 1)
        p.retrieval = np.array([[1, 0, 0, 0]], np.uint8)
        q = query or "conc"
        kind = {"conc": KIND_CONC, "diffuse": KIND_DIFFUSE, "flat": KIND_FLAT}[q]
        p.kind = np.zeros((1, 1, 4), np.int8)
        p.kind[0, 0, 0] = kind
        p.n_needles = np.zeros((1, 1, 4), np.int32)
        p.n_needles[0, 0, 0] = int(_rng(1, 11).integers(2, 9)) if kind == KIND_CONC else 0
        p.name = f"one_layer/{q}"
    elif name == "batch_decode":
        p = Plan(name, 1, 8, 32, 4, 131072, 131072, 0.9, 2)
        p.retrieval = np.array([[1, 0, 0, 0]], np.uint8)
        p.kind = np.zeros((1, 8, 4), np.int8)
        p.kind[0, :, 0] = KIND_CONC
        p.n_needles = np.zeros((1, 8, 4), np.int32)
        p.n_needles[0, :, 0] = _rng(2, 11).integers(1, 65, size=8)
    elif name in ("long_context", "ctx_1m"):
        big = name == "ctx_1m"
        seed = 4 if big else 3
        B = 1 if big else 2
        N = 1048576 if big else 524288
        p = Plan(name, 48, B, 32, 4, N, N, 0.9, seed)
        L, H = 48, 4
        r = _rng(seed, 11)
        flat = np.zeros(L * H, np.uint8)
        flat[r.permutation(L * H)[:29]] = 1
        p.retrieval = flat.reshape(L, H)
        p.kind = np.zeros((L, B, H), np.int8)
        p.n_needles = np.zeros((L, B, H), np.int32)
        inst = [(l, b, h) for l in range(L) for h in range(H) if p.retrieval[l, h]
                for b in range(B)]
        order = r.permutation(len(inst))
        n_other = 14 if big else len(inst) // 2
        other = KIND_FLAT if big else KIND_DIFFUSE
        for rank, i in enumerate(order):
            l, b, h = inst[i]
            if rank < n_other:
                p.kind[l, b, h] = other
            else:
                p.kind[l, b, h] = KIND_CONC
                p.n_needles[l, b, h] = int(r.integers(2, 9))
    else:
        raise ValueError(f"unknown workload {name!r}")

    if top_p is not None:
        p.top_p = float(top_p)
    if ctx is not None:
        p.ctx = p.max_ctx = int(ctx)
    if num_layers is not None and num_layers < p.num_layers:
        p.num_layers = int(num_layers)
        p.retrieval = p.retrieval[:num_layers].copy()
        p.kind = p.kind[:num_layers].copy()
        p.n_needles = p.n_needles[:num_layers].copy()
    if seq_lens is not None:
        assert len(seq_lens) == p.batch
        p.seq_lens = np.asarray(seq_lens, np.int64)
        p.max_ctx = max(p.max_ctx, int(p.seq_lens.max()))
    else:
        p.seq_lens = np.full(p.batch, p.ctx, np.int64)
    return p


def custom(*, batch: int, num_q_heads: int, num_kv_heads: int, seq_lens, max_ctx: int,
           retrieval, kinds, n_needles=None, top_p: float = 0.9, seed: int = 0,
           window: int = 8192, sinks: int = 4, name: str = "custom") -> Plan:
    """A one-layer plan of arbitrary shape (edge cases: ragged lengths, tiny contexts, ...)."""
    H = num_kv_heads
    p = Plan(name, 1, batch, num_q_heads, H, int(max(seq_lens)), max_ctx, top_p, seed,
             window=window, sinks=sinks)
    p.retrieval = np.asarray(retrieval, np.uint8).reshape(1, H)
    p.kind = np.asarray(kinds, np.int8).reshape(1, batch, H)
    p.n_needles = (np.zeros((1, batch, H), np.int32) if n_needles is None
                   else np.asarray(n_needles, np.int32).reshape(1, batch, H))
    p.seq_lens = np.asarray(seq_lens, np.int64)
    assert p.seq_lens.max() <= max_ctx
    return p


def _unit(r: np.random.Generator, dim: int) -> np.ndarray:
    u = r.standard_normal(dim)
    return u / np.linalg.norm(u)


@dataclass
class LayerInputs:
    q: torch.Tensor          # [B, Hq, D] bf16
    q_idx: torch.Tensor      # [B, Hkv, r] fp16
    k_cache: torch.Tensor    # [B, Hkv, max_ctx, D] bf16
    v_cache: torch.Tensor    # [B, Hkv, max_ctx, D] bf16
    k_idx: torch.Tensor      # [B, Hkv, max_ctx, r] fp16
    seq_lens: torch.Tensor   # [B] int32
    needles: dict            # (b, kvh) -> np.ndarray of planted positions


def make_layer(p: Plan, layer: int, device="cpu", poison_tail: bool = False) -> LayerInputs:
    """Draw one layer's inputs on ``device`` (torch generator seeded by (seed, layer))."""
    dev = torch.device(device)
    B, Hq, H, D, R, Nmax = p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.idx_dim, p.max_ctx
    g = torch.Generator(device=dev)
    g.manual_seed(int(p.seed) * 1_000_003 + 7919 * int(layer) + 1)
    q = torch.randn((B, Hq, D), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    k_cache = torch.randn((B, H, Nmax, D), generator=g, device=dev, dtype=torch.bfloat16)
    v_cache = torch.randn((B, H, Nmax, D), generator=g, device=dev, dtype=torch.bfloat16)
    k_idx = torch.randn((B, H, Nmax, R), generator=g, device=dev, dtype=torch.float16)

    r = _rng(p.seed, 101, layer)
    q_idx = np.zeros((B, H, R), np.float64)
    needles: dict = {}
    for b in range(B):
        N = int(p.seq_lens[b])
        for h in range(H):
            u = _unit(r, R)
            kind = int(p.kind[layer, b, h]) if p.retrieval[layer, h] else KIND_LOCAL
            sigma = SIGMA.get(kind, 1.0)
            q_idx[b, h] = 4.0 * sigma * u
            if kind == KIND_CONC:
                n = int(max(1, min(p.n_needles[layer, b, h], N)))
                pos = np.sort(r.choice(N, size=n, replace=False))
                # needle score so that n needles carry NEEDLE_MASS of the expected total mass
                s_needle = math.log(NEEDLE_MASS / (1 - NEEDLE_MASS) * N * math.exp(0.5) / n)
                alpha = s_needle / NEEDLE_COS
                w = r.standard_normal(R)
                w -= w.dot(u) * u
                w /= np.linalg.norm(w)
                key = alpha * (NEEDLE_COS * u + math.sqrt(1 - NEEDLE_COS ** 2) * w)
                kt = torch.tensor(key, dtype=torch.float16, device=dev)
                k_idx[b, h, torch.as_tensor(pos, device=dev)] = kt
                needles[(b, h)] = pos
    q_idx_t = torch.tensor(q_idx, dtype=torch.float16, device=dev)

    if poison_tail:
        for b in range(B):
            N = int(p.seq_lens[b])
            if N < Nmax:
                k_cache[b, :, N:] = float("nan")
                v_cache[b, :, N:] = float("nan")
                k_idx[b, :, N:] = float("nan")
    seq = torch.tensor(p.seq_lens, dtype=torch.int32, device=dev)
    return LayerInputs(q, q_idx_t, k_cache, v_cache, k_idx, seq, needles)


def to_host_u16(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of a bf16 / fp16 tensor as a numpy uint16 array (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def with_top_p(p: Plan, top_p: float) -> Plan:
    return replace(p, top_p=float(top_p))
