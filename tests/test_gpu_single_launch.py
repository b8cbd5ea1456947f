"""The single-launch layer (rtp_layer_io.single_launch: selection, gather and merge in one
cooperative launch, the selection kept in per-tile bit masks) against the fp64 oracle, and its
selection against the three-launch path's, token for token."""
import numpy as np
import pytest
import torch

from head_wise_sparse_retrieval_b200 import rtp
from head_wise_sparse_retrieval_b200 import workloads as W

from parity_utils import MAX_ABS, MEAN_ABS, check_layer, make_handle, run_layer

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rtp.load()


def _run(plan, layer=0, top_p=None, poison=False, exact=True, top_k=0, **cfg):
    li = W.make_layer(plan, layer, DEV, poison_tail=poison)
    with make_handle(plan, **cfg) as h:
        rep = check_layer(h, plan, li, layer, top_p, exact=exact, top_k=top_k,
                          single_launch=True)
    return rep


def _same_selection_as_three_launches(plan, layer=0, top_k=0):
    """Both paths bin the same fp32 scores: their selections and counts must be identical."""
    li = W.make_layer(plan, layer, DEV)
    ret = [(b, k) for b in range(plan.batch) for k in range(plan.num_kv_heads)
           if plan.retrieval[layer, k]]
    with make_handle(plan) as h:
        o3, c3 = run_layer(h, plan, li, layer, top_k=top_k)
        s3 = {bk: h.selection(*bk) for bk in ret}
        t3 = {bk: h.threshold(*bk) for bk in ret}
        o1, c1 = run_layer(h, plan, li, layer, top_k=top_k, single_launch=True)
        assert h.device_status() == 0
        s1 = {bk: h.selection(*bk) for bk in ret}
        t1 = {bk: h.threshold(*bk) for bk in ret}
    assert torch.equal(c1, c3)
    for bk in ret:
        assert np.array_equal(s1[bk], s3[bk]), bk
        assert t1[bk] == t3[bk], bk
    # different split-K cuts (and so different running maxima for the bf16 probabilities):
    # both outputs are within the oracle tolerance, so within twice it of each other
    d = (o1 - o3).abs()
    assert float(d.max()) <= 2 * MAX_ABS and float(d.mean()) <= 2 * MEAN_ABS


def test_tiny_selects_the_needles():
    p = W.plan("tiny")
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        check_layer(h, p, li, 0, single_launch=True)
        sel = h.selection(0, 0)
    assert sel.tolist() == li.needles[(0, 0)].tolist()


@pytest.mark.parametrize("query", ["conc", "diffuse", "flat"])
def test_one_layer(query):
    p = W.plan("one_layer", query=query)
    _run(p)
    _same_selection_as_three_launches(p)


def test_batch_decode_full_size():
    p = W.plan("batch_decode")
    rep = _run(p, exact=False)
    assert len(rep.heads) == 32
    _same_selection_as_three_launches(p)


@pytest.mark.parametrize("seq_lens", [
    [1, 2, 3, 4, 5, 17, 64, 65],
    [4095, 4096, 4097, 8191, 8192, 8193, 8196, 8197],
    [20000, 1, 12345, 8197, 16384, 16385, 3, 9000],
])
def test_ragged_lengths_and_poisoned_tail(seq_lens):
    """Ragged contexts around the 64-token ownership tiles, the 16-token MMA tiles and the
    window; the cache beyond N is NaN so any read past the context shows up."""
    B = len(seq_lens)
    kinds = [[W.KIND_DIFFUSE, W.KIND_LOCAL, W.KIND_CONC, W.KIND_FLAT] for _ in range(B)]
    needles = [[0, 0, 3, 0] for _ in range(B)]
    p = W.custom(batch=B, num_q_heads=32, num_kv_heads=4, seq_lens=seq_lens,
                 max_ctx=max(seq_lens) + 37, retrieval=[1, 0, 1, 1], kinds=kinds,
                 n_needles=needles, seed=sum(seq_lens) % 1000)
    _run(p, poison=True)
    _same_selection_as_three_launches(p)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_group_sizes(G):
    H = 3
    p = W.custom(batch=2, num_q_heads=H * G, num_kv_heads=H, seq_lens=[9000, 3000],
                 max_ctx=9001, retrieval=[1, 0, 1],
                 kinds=[[W.KIND_DIFFUSE, 0, W.KIND_CONC]] * 2, n_needles=[[0, 0, 5]] * 2,
                 seed=G)
    _run(p)


@pytest.mark.parametrize("top_p", [0.01, 0.5, 0.95, 1.0])
def test_top_p_values(top_p):
    p = W.custom(batch=1, num_q_heads=16, num_kv_heads=2, seq_lens=[30000], max_ctx=30000,
                 retrieval=[1, 1], kinds=[[W.KIND_DIFFUSE, W.KIND_FLAT]], seed=7)
    rep = _run(p, top_p=top_p)
    if top_p == 1.0:
        assert all(h["sel"].n_gpu == 30000 for h in rep.heads)


@pytest.mark.parametrize("query", ["diffuse", "conc"])
@pytest.mark.parametrize("k", [1, 2048, 16384])
def test_fixed_top_k(query, k):
    p = W.plan("one_layer", query=query)
    rep = _run(p, top_k=k)
    r = rep.heads[0]["sel"]
    assert r.n_gpu >= k and r.n_exact == k
    _same_selection_as_three_launches(p, top_k=k)


def test_fixed_top_k_beyond_n_selects_everything():
    seq = [100, 5000, 40000, 3]
    p = W.custom(batch=4, num_q_heads=16, num_kv_heads=2, seq_lens=seq, max_ctx=40000,
                 retrieval=[1, 1], kinds=[[W.KIND_DIFFUSE, W.KIND_FLAT]] * 4, seed=31)
    rep = _run(p, top_k=4096, poison=True)
    for h in rep.heads:
        n = seq[h["b"]]
        assert h["sel"].n_gpu == n if n <= 4096 else h["sel"].n_gpu >= 4096


def test_local_heads_only():
    p = W.custom(batch=3, num_q_heads=32, num_kv_heads=4, seq_lens=[100, 9000, 8196],
                 max_ctx=9000, retrieval=[0, 0, 0, 0], kinds=[[0, 0, 0, 0]] * 3, seed=5)
    _run(p)


def test_all_retrieval_heads_mixed_densities():
    """A needle head and a flat head in one layer: the round-robin ownership keeps every CTA's
    share of both."""
    p = W.custom(batch=2, num_q_heads=32, num_kv_heads=4, seq_lens=[40000, 25000],
                 max_ctx=40000, retrieval=[1, 1, 1, 1],
                 kinds=[[W.KIND_CONC, W.KIND_DIFFUSE, W.KIND_FLAT, W.KIND_CONC]] * 2,
                 n_needles=[[1, 0, 0, 64]] * 2, seed=11)
    _run(p)
    _same_selection_as_three_launches(p)


def test_deterministic_reruns():
    p = W.plan("one_layer", query="flat")
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        o1, c1 = run_layer(h, p, li, 0, single_launch=True)
        o2, c2 = run_layer(h, p, li, 0, single_launch=True)
    assert torch.equal(o1, o2) and torch.equal(c1, c2)


def test_cuda_graph_replay_matches_eager():
    p = W.custom(batch=2, num_q_heads=32, num_kv_heads=4, seq_lens=[30000, 12000],
                 max_ctx=30000, retrieval=[1, 0, 0, 1],
                 kinds=[[W.KIND_FLAT, 0, 0, W.KIND_CONC]] * 2, n_needles=[[0, 0, 0, 4]] * 2,
                 seed=3)
    li = W.make_layer(p, 0, DEV)
    L = rtp.layer_from(li)
    with make_handle(p) as h:
        eager, _ = run_layer(h, p, li, 0, single_launch=True)
        out = torch.zeros_like(eager)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            h.decode_step(0, L, p.retrieval[0], p.top_p, out, stream=s, single_launch=True)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(3):  # back-to-back launches reuse the workspace
                h.decode_step(0, L, p.retrieval[0], p.top_p, out, single_launch=True)
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
        assert h.device_status() == 0
        del g


def test_unsupported_shapes_are_refused_before_any_launch():
    # B * Hkv above the single-launch tables
    p = W.custom(batch=20, num_q_heads=32, num_kv_heads=4, seq_lens=[100] * 20, max_ctx=100,
                 retrieval=[1, 0, 0, 0], kinds=[[W.KIND_FLAT, 0, 0, 0]] * 20, seed=1)
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        with pytest.raises(rtp.RtpError, match="single launch"):
            run_layer(h, p, li, 0, single_launch=True)
        run_layer(h, p, li, 0)  # the three-launch path still serves it


@pytest.mark.slow
def test_ctx_1m_sampled_layers():
    """Full-size 1M-token layers of the 48-layer workload in single-launch mode: a layer with a
    flat retrieval head, one with a needle head, one with local heads only."""
    p = W.plan("ctx_1m")
    flat = [l for l in range(48) if (p.kind[l] == W.KIND_FLAT).any()]
    conc = [l for l in range(48) if (p.kind[l] == W.KIND_CONC).any()]
    none = [l for l in range(48) if not p.retrieval[l].any()]
    with make_handle(p) as h:
        for l in (flat[0], conc[0], none[0]):
            li = W.make_layer(p, l, DEV)
            check_layer(h, p, li, l, exact=False, single_launch=True)
            del li
            torch.cuda.empty_cache()


def test_largest_single_launch_layer():
    """B * Hkv = 64, the largest layer the single-launch tables take, with ragged contexts."""
    B, Hkv = 16, 4
    seqs = [1 + 997 * b for b in range(B)]
    kinds = [[W.KIND_DIFFUSE, W.KIND_LOCAL, W.KIND_CONC, W.KIND_FLAT] for _ in range(B)]
    p = W.custom(batch=B, num_q_heads=32, num_kv_heads=Hkv, seq_lens=seqs, max_ctx=max(seqs),
                 retrieval=[1, 0, 1, 1], kinds=kinds, n_needles=[[0, 0, 3, 0]] * B, seed=23)
    li = W.make_layer(p, 0, DEV)
    heads = [(b, k) for b in (0, 1, 7, 15) for k in range(Hkv)]
    with make_handle(p) as h:
        check_layer(h, p, li, 0, heads=heads, exact=False, single_launch=True)
    _same_selection_as_three_launches(p)
