"""Parity of the CUDA library (called through its C-ABI) with the fp64 oracle, on a B200."""
import numpy as np
import pytest
import torch

from head_wise_sparse_retrieval_b200 import rtp
from head_wise_sparse_retrieval_b200 import workloads as W

from parity_utils import (check_layer, check_output, make_handle, oracle_head, run_layer,
                          MEAN_ABS)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rtp.load()


def _run(plan, layer=0, top_p=None, heads=None, poison=False, exact=True, top_k=0, **cfg):
    li = W.make_layer(plan, layer, DEV, poison_tail=poison)
    with make_handle(plan, **cfg) as h:
        rep = check_layer(h, plan, li, layer, top_p, heads, exact=exact, top_k=top_k)
    return rep


def test_tiny_selects_the_needles():
    p = W.plan("tiny")
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        rep = check_layer(h, p, li, 0)
        sel = h.selection(0, 0)
    assert sel.tolist() == li.needles[(0, 0)].tolist()
    assert rep.heads[0]["sel"].n_gpu == 3


@pytest.mark.parametrize("query", ["conc", "diffuse", "flat"])
def test_one_layer(query):
    p = W.plan("one_layer", query=query)
    rep = _run(p)
    r = rep.heads[0]["sel"]
    if query == "conc":
        assert r.n_gpu <= 16
    if query == "diffuse":
        assert 3000 < r.n_gpu < 30000
    assert r.n_exact <= r.n_gpu


def test_batch_decode_full_size():
    p = W.plan("batch_decode")
    rep = _run(p, exact=False)
    assert len(rep.heads) == 32


@pytest.mark.parametrize("seq_lens", [
    [1, 2, 3, 4, 5, 17, 64, 65],
    [4095, 4096, 4097, 8191, 8192, 8193, 8196, 8197],
    [20000, 1, 12345, 8197, 16384, 16385, 3, 9000],
])
def test_ragged_lengths_and_poisoned_tail(seq_lens):
    """Ragged contexts around tile, chunk and window boundaries; the cache beyond N is NaN so
    any read past the context shows up in the output."""
    B = len(seq_lens)
    kinds = [[W.KIND_DIFFUSE, W.KIND_LOCAL, W.KIND_CONC, W.KIND_FLAT] for _ in range(B)]
    needles = [[0, 0, 3, 0] for _ in range(B)]
    p = W.custom(batch=B, num_q_heads=32, num_kv_heads=4, seq_lens=seq_lens,
                 max_ctx=max(seq_lens) + 37, retrieval=[1, 0, 1, 1], kinds=kinds,
                 n_needles=needles, seed=sum(seq_lens) % 1000)
    _run(p, poison=True)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_group_sizes(G):
    H = 3
    p = W.custom(batch=2, num_q_heads=H * G, num_kv_heads=H, seq_lens=[9000, 3000],
                 max_ctx=9001, retrieval=[1, 0, 1],
                 kinds=[[W.KIND_DIFFUSE, 0, W.KIND_CONC]] * 2, n_needles=[[0, 0, 5]] * 2,
                 seed=G)
    _run(p)


@pytest.mark.parametrize("top_p", [0.01, 0.5, 0.8, 0.95, 1.0])
def test_top_p_values(top_p):
    p = W.custom(batch=1, num_q_heads=16, num_kv_heads=2, seq_lens=[30000], max_ctx=30000,
                 retrieval=[1, 1], kinds=[[W.KIND_DIFFUSE, W.KIND_FLAT]], seed=7)
    rep = _run(p, top_p=top_p)
    if top_p == 1.0:
        assert all(h["sel"].n_gpu == 30000 for h in rep.heads)


@pytest.mark.parametrize("query", ["diffuse", "flat", "conc"])
@pytest.mark.parametrize("k", [1, 2048, 4096, 16384])
def test_fixed_top_k(query, k):
    """Fixed top-k through the histogram (the pages' top-2k / 4k / 16k): every bin from the top
    until the bins hold k tokens."""
    p = W.plan("one_layer", query=query)
    rep = _run(p, top_k=k)
    r = rep.heads[0]["sel"]
    assert r.n_gpu >= k and r.n_exact == k


def test_fixed_top_k_ragged_and_beyond_n():
    seq = [100, 5000, 40000, 3]
    kinds = [[W.KIND_DIFFUSE, W.KIND_FLAT]] * 4
    p = W.custom(batch=4, num_q_heads=16, num_kv_heads=2, seq_lens=seq, max_ctx=40000,
                 retrieval=[1, 1], kinds=kinds, seed=31)
    rep = _run(p, top_k=4096, poison=True)
    for h in rep.heads:
        n = seq[h["b"]]
        assert h["sel"].n_gpu == n if n <= 4096 else h["sel"].n_gpu >= 4096


def test_small_window_and_no_sinks():
    p = W.custom(batch=2, num_q_heads=16, num_kv_heads=2, seq_lens=[5000, 100], max_ctx=5000,
                 retrieval=[0, 0], kinds=[[0, 0]] * 2, seed=9, window=777, sinks=0)
    _run(p, window=777, sinks=0)


@pytest.mark.parametrize("B,Hkv,G,seq_lens", [
    (1, 1, 8, [9000]),                       # one head: the most clusters per head
    (1, 2, 8, [8197]),                       # two heads, window + sinks + 1 tokens
    (1, 4, 8, [20000]),                      # the ctx_1m head layout
    (2, 4, 4, [8196, 70]),                   # the whole context at and under window + sinks
    (3, 4, 8, [1, 17, 12001]),               # 12 heads; contexts shorter than the cluster
    (37, 1, 2, [3 + 331 * b for b in range(37)]),  # 37 heads: the smallest cluster
    (40, 1, 1, [5000] * 40),                 # more heads than that serves: the split launches
])
def test_local_only_layers(B, Hkv, G, seq_lens):
    """Layers without retrieval heads run as one launch of one or more thread-block clusters
    per KV head when the SMs allow (the cluster merges its CTAs' pieces itself, through L2 after
    a cluster barrier), else as the split attention and merge launches; every
    head against the oracle, with the cache past each context poisoned, bit-identical reruns,
    and the launch count of the path that ran."""
    p = W.custom(batch=B, num_q_heads=Hkv * G, num_kv_heads=Hkv, seq_lens=seq_lens,
                 max_ctx=max(seq_lens) + 5, retrieval=[0] * Hkv, kinds=[[0] * Hkv] * B,
                 seed=B * 10 + Hkv)
    li = W.make_layer(p, 0, DEV, poison_tail=True)
    with make_handle(p) as h:
        h.profile(True)
        check_layer(h, p, li, 0)
        kinds = [k for k, _ in h.profile_launches()]
        h.profile(False)
        a, _ = run_layer(h, p, li, 0)
        # reruns back to back: a value read before another thread or CTA wrote it would change
        # from run to run
        again = [run_layer(h, p, li, 0)[0] for _ in range(8)]
    for b in again:
        assert torch.equal(a, b)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    if sms // (B * Hkv) >= 4:
        assert kinds == ["attend"], kinds  # the merge is inside the launch
    else:
        assert kinds == ["attend", "merge"], kinds


def test_all_retrieval_heads():
    p = W.custom(batch=2, num_q_heads=32, num_kv_heads=4, seq_lens=[40000, 25000],
                 max_ctx=40000, retrieval=[1, 1, 1, 1],
                 kinds=[[W.KIND_CONC, W.KIND_DIFFUSE, W.KIND_FLAT, W.KIND_CONC]] * 2,
                 n_needles=[[1, 0, 0, 64]] * 2, seed=11)
    _run(p)


@pytest.mark.slow
def test_selection_ranges_beyond_on_chip_capacity():
    """Eight retrieval slots of 655 360 tokens: each selection CTA scores more tokens than it
    keeps in shared memory, so part of its scores and bins go through the global spill
    buffers, and its histogram is flushed in more than one chunk."""
    N = 655360
    kinds = [[W.KIND_CONC, W.KIND_DIFFUSE, W.KIND_FLAT, W.KIND_CONC],
             [W.KIND_DIFFUSE, W.KIND_CONC, W.KIND_CONC, W.KIND_FLAT]]
    p = W.custom(batch=2, num_q_heads=32, num_kv_heads=4, seq_lens=[N, N - 4321], max_ctx=N,
                 retrieval=[1, 1, 1, 1], kinds=kinds, n_needles=[[2, 0, 0, 7], [0, 5, 3, 0]],
                 seed=21)
    assert sum(p.seq_lens) * 4 > 148 * 2 * 16384  # more than the CTAs keep on chip
    _run(p, exact=False)


@pytest.mark.parametrize("B,Hq,Hkv", [(1, 32, 4), (8, 32, 4), (3, 16, 8), (2, 8, 8)])
def test_indexer_append_matches_oracle(B, Hq, Hkv):
    """rtp_indexer_append: q_idx and the new k_idx row agree with the fp64 oracle rounded to
    fp16 (fp32 accumulation may differ by one fp16 unit next to a rounding boundary); only row
    N_b - 1 of the selected heads changes and q_idx of unselected heads is left alone."""
    import oracle
    G, D, r, max_ctx = Hq // Hkv, 128, 16, 300
    g = torch.Generator(device=DEV).manual_seed(B * 100 + Hq + Hkv)
    bf = lambda *sh, sd=1.0: (torch.randn(*sh, generator=g, device=DEV) * sd).to(torch.bfloat16)
    q_pre, k_pre = bf(B, Hq, D), bf(B, Hkv, D)
    w_q, w_k = bf(Hkv, r, G * D, sd=0.03), bf(Hkv, r, D, sd=0.1)
    seq = torch.tensor([max_ctx - 7 * b for b in range(B)], dtype=torch.int32, device=DEV)
    k_idx = torch.randn(B, Hkv, max_ctx, r, generator=g, device=DEV).to(torch.float16)
    q_idx = torch.full((B, Hkv, r), 7.0, dtype=torch.float16, device=DEV)
    k_before, q_before = k_idx.clone(), q_idx.clone()
    mask = np.array([(h + 1) % 3 != 0 for h in range(Hkv)], np.uint8)
    p = W.custom(batch=B, num_q_heads=Hq, num_kv_heads=Hkv, seq_lens=seq.tolist(),
                 max_ctx=max_ctx, retrieval=[0] * Hkv, kinds=[[0] * Hkv] * B)
    with make_handle(p) as h:
        h.indexer_append(q_pre, k_pre, w_q, w_k, seq, q_idx, k_idx, head_mask=mask)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    qi, ki = oracle.indexer_project(W.to_host_u16(q_pre), W.to_host_u16(k_pre),
                                    W.to_host_u16(w_q), W.to_host_u16(w_k))
    ulp = lambda a, b: np.abs(a.astype(np.int32) - b.astype(np.int32))
    gq = q_idx.cpu().numpy().view(np.uint16).astype(np.int16)
    gk = k_idx.cpu().numpy().view(np.uint16)
    exact = total = 0
    for b in range(B):
        n = int(seq[b])
        for hh in range(Hkv):
            if not mask[hh]:
                assert torch.equal(q_idx[b, hh], q_before[b, hh])
                assert torch.equal(k_idx[b, hh], k_before[b, hh])
                continue
            want_q = qi[b, hh].astype(np.float16).view(np.int16)
            want_k = ki[b, hh].astype(np.float16).view(np.int16)
            got_k = gk[b, hh, n - 1].astype(np.int16)
            assert ulp(gq[b, hh], want_q).max() <= 1 and ulp(got_k, want_k).max() <= 1
            exact += int((gq[b, hh] == want_q).sum() + (got_k == want_k).sum())
            total += 2 * r
            others = torch.ones(max_ctx, dtype=torch.bool)
            others[n - 1] = False
            assert torch.equal(k_idx[b, hh][others.to(DEV)], k_before[b, hh][others.to(DEV)])
    assert exact >= 0.97 * total


def test_dense_decode_matches_oracle():
    p = W.custom(batch=2, num_q_heads=32, num_kv_heads=4, seq_lens=[33000, 7],
                 max_ctx=33000, retrieval=[1, 0, 0, 0],
                 kinds=[[W.KIND_CONC, 0, 0, 0]] * 2, n_needles=[[3, 0, 0, 0]] * 2, seed=12)
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        out, _ = run_layer(h, p, li, 0, dense=True)
    out = out.cpu().numpy()
    for b in range(2):
        for kvh in range(4):
            ho = oracle_head(li, b, kvh, False, 0.9, 8, dense=True)
            check_output(out[b, kvh * 8:(kvh + 1) * 8], ho.out, f"dense b{b} kvh{kvh}")


def test_p_one_equals_dense():
    p = W.custom(batch=1, num_q_heads=16, num_kv_heads=2, seq_lens=[20000], max_ctx=20000,
                 retrieval=[1, 1], kinds=[[W.KIND_CONC, W.KIND_DIFFUSE]],
                 n_needles=[[4, 0]], seed=13)
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        sparse, cnt = run_layer(h, p, li, 0, top_p=1.0)
        dense, _ = run_layer(h, p, li, 0, dense=True)
    assert cnt.cpu().tolist() == [[20000, 20000]]
    assert torch.equal(sparse, dense)


def test_deterministic_reruns():
    p = W.plan("one_layer", query="diffuse")
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        o1, c1 = run_layer(h, p, li, 0)
        s1 = h.selection(0, 0)
        o2, c2 = run_layer(h, p, li, 0)
        s2 = h.selection(0, 0)
    assert torch.equal(o1, o2) and torch.equal(c1, c2) and np.array_equal(s1, s2)


def test_cuda_graph_replay_matches_eager():
    p = W.plan("one_layer", query="conc")
    li = W.make_layer(p, 0, DEV)
    L = rtp.layer_from(li)
    with make_handle(p) as h:
        eager, _ = run_layer(h, p, li, 0)
        out = torch.zeros_like(eager)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            h.decode_step(0, L, p.retrieval[0], p.top_p, out, stream=s)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        out.zero_()
        with torch.cuda.graph(g):
            h.decode_step(0, L, p.retrieval[0], p.top_p, out)
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
        del g


def test_host_buffer_entry_matches_device_entry():
    p = W.plan("long_context", num_layers=2, ctx=20000)
    lis = [W.make_layer(p, l, DEV) for l in range(2)]
    with make_handle(p) as h:
        dev_out = [run_layer(h, p, li, l)[0] for l, li in enumerate(lis)]
        q = torch.stack([li.q for li in lis]).cpu().pin_memory()
        qi = torch.stack([li.q_idx for li in lis]).cpu().pin_memory()
        seq = lis[0].seq_lens.cpu().pin_memory()
        out = torch.empty((2,) + tuple(dev_out[0].shape), dtype=torch.float32).pin_memory()
        views = [rtp.layer_from(li) for li in lis]
        h.decode_step_host(q, qi, seq, views, p.retrieval, p.top_p, out)
        for l in range(2):
            assert torch.equal(out[l], dev_out[l].cpu())
        # a second call replays the captured launches on new queries from the same staging
        for li in lis:
            li.q.neg_()
        dev_out2 = [run_layer(h, p, li, l)[0] for l, li in enumerate(lis)]
        q2 = torch.stack([li.q for li in lis]).cpu().pin_memory()
        h.decode_step_host(q2, qi, seq, views, p.retrieval, p.top_p, out)
        for l in range(2):
            assert torch.equal(out[l], dev_out2[l].cpu())
            assert not torch.equal(dev_out2[l], dev_out[l])
        # other masks: the launches are captured again
        masks = p.retrieval.copy()
        masks[0] = 1 - masks[0]
        dev_out3 = []
        for l, li in enumerate(lis):
            o = torch.empty_like(dev_out2[l])
            h.decode_step(l, rtp.layer_from(li), masks[l], p.top_p, o)
            dev_out3.append(o)
        h.decode_step_host(q2, qi, seq, views, masks, p.top_p, out)
        for l in range(2):
            assert torch.equal(out[l], dev_out3[l].cpu())


def test_inputs_ready_chaining_matches_strict_ordering():
    """Layers launched back to back with inputs_ready (selection scoring and local-only
    attention start before the previous launch finishes) give bit-identical outputs and
    selections to the strictly ordered launches."""
    p = W.plan("long_context", num_layers=6, ctx=30000)
    lis = [W.make_layer(p, l, DEV) for l in range(6)]
    B, Hq, Hkv = p.batch, p.num_q_heads, p.num_kv_heads
    with make_handle(p) as h:
        res = {}
        for ready in (False, True):
            outs = [torch.full((B, Hq, 128), float("nan"), device=DEV) for _ in lis]
            cnts = [torch.full((B, Hkv), -1, dtype=torch.int32, device=DEV) for _ in lis]
            for rep in range(3):
                for l, li in enumerate(lis):
                    h.decode_step(l, rtp.layer_from(li), p.retrieval[l], p.top_p, outs[l],
                                  cnts[l], inputs_ready=ready)
            torch.cuda.synchronize()
            assert h.device_status() == 0
            res[ready] = ([o.cpu() for o in outs], [c.cpu() for c in cnts])
    assert any(p.retrieval[l].any() for l in range(6)) and not all(p.retrieval[l].any()
                                                                    for l in range(6))
    for l in range(6):
        assert torch.equal(res[True][0][l], res[False][0][l])
        assert torch.equal(res[True][1][l], res[False][1][l])


def test_bounded_wait_runs_out_and_is_reported():
    """Failure detection without a GPU fault: one selection CTA withholds its barrier arrival,
    the other CTAs' bounded waits (2 ms here) run out, the launch ends by itself and the status
    word reports the timeout; the handle then decodes normally."""
    p = W.plan("one_layer", query="conc")
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        out = torch.empty((1, 32, 128), dtype=torch.float32, device=DEV)
        assert h.device_status() == 0
        h.selftest_wait_timeout(0, rtp.layer_from(li), p.retrieval[0], p.top_p, out,
                                wait_ns=2_000_000)
        code = h.device_status()
        assert code & rtp.DEV_WAIT_TIMEOUT, hex(code)
        assert h.device_status() == 0  # read and cleared
        with pytest.raises(rtp.RtpError):
            h.selection(0, 0)  # the self-test's lists are not meaningful
        check_layer(h, p, li, 0)


def test_bad_seq_len_is_reported_not_faulted():
    p = W.custom(batch=2, num_q_heads=8, num_kv_heads=1, seq_lens=[100, 50], max_ctx=128,
                 retrieval=[1], kinds=[[W.KIND_CONC]] * 2, n_needles=[[2]] * 2, seed=14)
    li = W.make_layer(p, 0, DEV)
    li.seq_lens[1] = 1000  # beyond max_ctx: clamped on the device, reported in the status word
    with make_handle(p) as h:
        out, _ = run_layer(h, p, li, 0)
        code = h.device_status()
        assert code & rtp.DEV_BAD_SEQLEN
        assert h.device_status() == 0  # reading clears it
    assert torch.isfinite(out[0]).all()


def test_negative_top_k_is_rejected():
    p = W.plan("tiny")
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        out = torch.empty((1, 8, 128), dtype=torch.float32, device=DEV)
        with pytest.raises(rtp.RtpError) as e:
            h.decode_step(0, rtp.layer_from(li), [1], 0.9, out, top_k=-1)
        assert e.value.status == rtp.RTP_ERR_INVALID_ARG
        h.decode_step(0, rtp.layer_from(li), [1], 0.0, out, top_k=5)  # top_p ignored
        torch.cuda.synchronize()
        assert h.selection(0, 0).size >= 5


def test_host_side_argument_errors():
    p = W.plan("tiny")
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        out = torch.empty((1, 8, 128), dtype=torch.float32, device=DEV)
        L = rtp.layer_from(li)
        with pytest.raises(rtp.RtpError) as e:
            h.decode_step(0, L, [1], 0.0, out)
        assert e.value.status == rtp.RTP_ERR_INVALID_ARG
        with pytest.raises(rtp.RtpError):
            h.decode_step(0, L, [1], 1.5, out)
        with pytest.raises(rtp.RtpError):
            h.decode_step(1, L, [1], 0.9, out)  # layer out of range
        bad = rtp.Layer(li.q, li.q_idx, li.k_cache.view(-1)[1:], li.v_cache, li.k_idx, li.seq_lens)
        with pytest.raises(rtp.RtpError):
            h.decode_step(0, bad, [1], 0.9, out)  # misaligned cache pointer
        with pytest.raises(rtp.RtpError):
            h.selection(0, 0)  # no successful decode_step yet


@pytest.mark.slow
@pytest.mark.parametrize("name", ["long_context", "ctx_1m"])
def test_long_configs_sampled_layers(name):
    """Full-size layers of the 48-layer workloads, in the launch configuration the benchmark
    times (one call per layer, same handle configuration); every head of the sampled layers is
    compared with the oracle."""
    p = W.plan(name)
    # a layer with a conc retrieval head, one with a diffuse/flat one, one with none
    conc = [l for l in range(48) if (p.kind[l] == W.KIND_CONC).any()]
    other = [l for l in range(48) if ((p.kind[l] == W.KIND_DIFFUSE) |
                                      (p.kind[l] == W.KIND_FLAT)).any()]
    none = [l for l in range(48) if not p.retrieval[l].any()]
    layers = [conc[0], other[0], none[0]]
    with make_handle(p) as h:
        for l in layers:
            li = W.make_layer(p, l, DEV)
            check_layer(h, p, li, l, exact=False)
            del li
            torch.cuda.empty_cache()


def test_maximum_head_count():
    """B * Hkv = 1024 heads (the largest layer the library takes), 256 retrieval slots and
    32 768 merge units, ragged contexts from 1 to 300 tokens; sampled heads against the
    oracle."""
    B, Hkv, G = 64, 16, 8
    rng = np.random.default_rng(5)
    seqs = [int(x) for x in rng.integers(1, 301, B)]
    ret = [1 if k % 4 == 0 else 0 for k in range(Hkv)]
    kinds = [[(W.KIND_DIFFUSE if (b + k) % 2 else W.KIND_CONC) if ret[k] else W.KIND_LOCAL
              for k in range(Hkv)] for b in range(B)]
    needles = [[2 if kinds[b][k] == W.KIND_CONC else 0 for k in range(Hkv)] for b in range(B)]
    p = W.custom(batch=B, num_q_heads=Hkv * G, num_kv_heads=Hkv, seq_lens=seqs, max_ctx=300,
                 retrieval=ret, kinds=kinds, n_needles=needles, seed=17)
    heads = [(b, k) for b in (0, 1, 31, 62, 63) for k in (0, 3, 4, 12, 15)]
    _run(p, heads=heads, exact=False)


def test_profiling_and_nvtx_do_not_change_results():
    """Per-launch events (rtp_profile_launches) report each layer's launches in order, and
    neither they nor NVTX ranges change the outputs (bit-equal to a plain run)."""
    p = W.custom(batch=2, num_q_heads=32, num_kv_heads=4, seq_lens=[20000, 9000],
                 max_ctx=20000, retrieval=[1, 0, 1, 0],
                 kinds=[[W.KIND_DIFFUSE, 0, W.KIND_CONC, 0]] * 2, n_needles=[[0, 0, 4, 0]] * 2,
                 seed=23)
    li = W.make_layer(p, 0, DEV)
    with make_handle(p) as h:
        plain, _ = run_layer(h, p, li, 0)
        h.profile(True)
        h.nvtx(True)
        profiled, _ = run_layer(h, p, li, 0)
        dense, _ = run_layer(h, p, li, 0, dense=True)
        launches = h.profile_launches()
        h.profile(False)
        h.nvtx(False)
    assert torch.equal(plain, profiled)
    assert [k for k, _ in launches] == ["select", "attend", "merge", "attend", "merge"]
    assert all(ms > 0 for _, ms in launches)
    check_output(dense.cpu().numpy()[0, 0:8], oracle_head(li, 0, 0, False, 0.9, 8,
                                                          dense=True).out, "dense after profiling")


@pytest.mark.slow
def test_largest_context_with_tied_scores_selects_every_token():
    """The largest cache a handle takes (max_ctx = 2^24 - 1) with a zero indexer query: every
    score ties at s_max = 0, every token falls in bin 255 with mass 1, and the 64-bit sums of
    2^-40 fixed-point masses reach (2^24 - 1) * 2^40, just below 2^64. A wrapped sum would move
    b* off bin 255 and drop tokens. With a zero query as well the attention weights are
    uniform, so the output is the mean of V over all tokens (computed here by torch in fp64)."""
    N = (1 << 24) - 1
    g = torch.Generator(device=DEV).manual_seed(77)
    k = torch.randn((1, 1, N, 128), generator=g, device=DEV, dtype=torch.bfloat16)
    v = torch.randn((1, 1, N, 128), generator=g, device=DEV, dtype=torch.bfloat16)
    k_idx = torch.randn((1, 1, N, 16), generator=g, device=DEV, dtype=torch.float16)
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device=DEV)
    q_idx = torch.zeros((1, 1, 16), dtype=torch.float16, device=DEV)
    seq = torch.tensor([N], dtype=torch.int32, device=DEV)
    p = W.custom(batch=1, num_q_heads=8, num_kv_heads=1, seq_lens=[N], max_ctx=N,
                 retrieval=[1], kinds=[[W.KIND_FLAT]], seed=77)
    out = torch.full((1, 8, 128), float("nan"), dtype=torch.float32, device=DEV)
    cnt = torch.full((1, 1), -1, dtype=torch.int32, device=DEV)
    with make_handle(p) as h:
        h.decode_step(0, rtp.Layer(q, q_idx, k, v, k_idx, seq), np.array([1], np.uint8), 0.9,
                      out, cnt)
        torch.cuda.synchronize()
        assert h.device_status() == 0
        bstar, s_max = h.threshold(0, 0)
    assert int(cnt.item()) == N
    assert (bstar, s_max) == (255, 0.0)
    ref = v[0, 0].double().mean(dim=0).cpu().numpy()
    got = out[0].cpu().numpy()
    for g_ in range(8):
        check_output(got[g_:g_ + 1], ref[None, :], f"mean of V, query head {g_}")
