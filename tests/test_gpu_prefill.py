"""Prefill attention (rtp_prefill) against the fp64 oracle, through the C-ABI, on a B200.

Row i of a prompt attends over {j <= i} for a retrieval head (or with dense set) and over the
sinks and the last `window` positions up to i for a local head (the gist.science technical
summary, Methodology 1): the decode output of a context of i + 1 tokens. Each test compares the
rows it names with oracle.prefill_rows under the same absolute and relative bars as the decode
parity tests.
"""
import numpy as np
import pytest
import torch

from head_wise_sparse_retrieval_b200 import rtp
from head_wise_sparse_retrieval_b200 import workloads as W

from parity_utils import check_output, make_handle

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rtp.load()


def _inputs(B, Hq, Hkv, t_max, max_ctx, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    bf = lambda *sh: torch.randn(*sh, generator=g, device=DEV).to(torch.bfloat16)
    return bf(B, Hq, t_max, 128), bf(B, Hkv, max_ctx, 128), bf(B, Hkv, max_ctx, 128)


def _plan(B, Hq, Hkv, seqs, max_ctx, **kw):
    return W.custom(batch=B, num_q_heads=Hq, num_kv_heads=Hkv, seq_lens=seqs, max_ctx=max_ctx,
                    retrieval=[0] * Hkv, kinds=[[0] * Hkv] * B, **kw)


def _check_rows(out, q, k, v, seqs, G, mask, heads, rows_of, window, sinks, dense_all=False):
    import oracle
    for b, hq in heads:
        T = seqs[b]
        kvh = hq // G
        rows = np.asarray(rows_of(T), np.int64)
        dense = dense_all or bool(mask[kvh])
        ref = oracle.prefill_rows(W.to_host_u16(q[b, hq, rows]), W.to_host_u16(k[b, kvh, :T]),
                                  W.to_host_u16(v[b, kvh, :T]), rows, dense, window, sinks)
        got = out[b, hq, rows].cpu().numpy()
        check_output(got, ref, f"prefill b {b} head {hq}")


@pytest.mark.parametrize("window,sinks", [(128, 4), (100, 0), (64, 64), (1, 4)])
def test_prefill_small_window_every_row(window, sinks):
    """A window far below the prompt length, every row of a local and a retrieval head of both
    sequences: rows before and after the window's reach, ragged prompts below t_max; rows past a
    prompt's length are left untouched."""
    B, Hq, Hkv, seqs, t_max = 2, 16, 2, [300, 1000], 1000
    q, k, v = _inputs(B, Hq, Hkv, t_max, 1024, seed=window + sinks)
    seq = torch.tensor(seqs, dtype=torch.int32, device=DEV)
    mask = np.array([1, 0], np.uint8)
    p = _plan(B, Hq, Hkv, seqs, 1024, window=window, sinks=sinks)
    out = torch.full((B, Hq, t_max, 128), float("nan"), device=DEV)
    with make_handle(p, window=window, sinks=sinks) as h:
        h.prefill(q, k, v, seq, mask, out)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    _check_rows(out, q, k, v, seqs, Hq // Hkv, mask, [(0, 0), (0, 9), (1, 3), (1, 15)],
                lambda T: range(T), window, sinks)
    assert torch.isnan(out[0, :, 300:]).all()  # rows past T_b are not written
    assert torch.isfinite(out[1]).all()


def test_prefill_pages_window_around_its_reach():
    """Window 8192 + 4 sinks on a 9000-token prompt: rows on both sides of the window's reach,
    for a local and a retrieval head."""
    B, Hq, Hkv, seqs = 1, 16, 2, [9000]
    q, k, v = _inputs(B, Hq, Hkv, 9000, 9000, seed=5)
    seq = torch.tensor(seqs, dtype=torch.int32, device=DEV)
    mask = np.array([0, 1], np.uint8)
    p = _plan(B, Hq, Hkv, seqs, 9000)
    out = torch.empty((B, Hq, 9000, 128), device=DEV)
    rows = lambda T: [0, 1, 3, 4, 15, 16, 17, 63, 64, 65, 4000, 8190, 8191, 8192, 8195, 8196,
                      8197, 8260, 8961, 8999]
    with make_handle(p) as h:
        h.prefill(q, k, v, seq, mask, out)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    _check_rows(out, q, k, v, seqs, 8, mask, [(0, 0), (0, 7), (0, 8), (0, 15)], rows, 8192, 4)


@pytest.mark.parametrize("G", [1, 4])
def test_prefill_dense_flag_and_group_sizes(G):
    """dense != 0 gives full causal attention on every head, whatever the mask; groups smaller
    than the MMA's 8 columns."""
    Hkv = 3
    B, Hq, seqs, t_max = 2, Hkv * G, [777, 130], 800
    q, k, v = _inputs(B, Hq, Hkv, t_max, 800, seed=G)
    seq = torch.tensor(seqs, dtype=torch.int32, device=DEV)
    mask = np.array([0, 1, 0], np.uint8)
    p = _plan(B, Hq, Hkv, seqs, 800, window=50, sinks=2)
    out = torch.empty((B, Hq, t_max, 128), device=DEV)
    with make_handle(p, window=50, sinks=2) as h:
        h.prefill(q, k, v, seq, mask, out, dense=True)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    heads = [(0, 0), (0, Hq - 1), (1, Hq // 2)]
    _check_rows(out, q, k, v, seqs, G, mask, heads, lambda T: range(T), 50, 2, dense_all=True)


def test_prefill_local_heads_of_a_layer_mask():
    """Mixed mask with several query heads per group written by one warp: every query head of
    a local and of a retrieval KV head, sampled rows."""
    B, Hq, Hkv, seqs, t_max = 1, 32, 4, [3000], 3000
    q, k, v = _inputs(B, Hq, Hkv, t_max, 3000, seed=11)
    seq = torch.tensor(seqs, dtype=torch.int32, device=DEV)
    mask = np.array([0, 0, 1, 0], np.uint8)
    p = _plan(B, Hq, Hkv, seqs, 3000, window=1024, sinks=4)
    out = torch.empty((B, Hq, t_max, 128), device=DEV)
    with make_handle(p, window=1024, sinks=4) as h:
        h.prefill(q, k, v, seq, mask, out)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    rows = lambda T: [0, 7, 1027, 1028, 1029, 2047, 2999]
    heads = [(0, hq) for hq in list(range(8, 16)) + list(range(16, 24))]
    _check_rows(out, q, k, v, seqs, 8, mask, heads, rows, 1024, 4)


def test_prefill_covering_window_equals_dense_and_reruns_bit_equal():
    """A window covering the whole prompt makes a local head's prefill full causal attention:
    the same kernel arithmetic, so bit-equal to dense; and a rerun is bit-identical."""
    B, Hq, Hkv, seqs, t_max = 1, 8, 1, [2000], 2000
    q, k, v = _inputs(B, Hq, Hkv, t_max, 2000, seed=9)
    seq = torch.tensor(seqs, dtype=torch.int32, device=DEV)
    p = _plan(B, Hq, Hkv, seqs, 2000, window=4096, sinks=4)
    outs = [torch.empty((B, Hq, t_max, 128), device=DEV) for _ in range(3)]
    with make_handle(p, window=4096, sinks=4) as h:
        h.prefill(q, k, v, seq, np.array([0], np.uint8), outs[0])
        h.prefill(q, k, v, seq, np.array([0], np.uint8), outs[1])
        h.prefill(q, k, v, seq, np.array([0], np.uint8), outs[2], dense=True)
        torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(outs[0], outs[2])
    _check_rows(outs[0], q, k, v, seqs, 8, np.array([1], np.uint8), [(0, 0), (0, 5)],
                lambda T: [0, 1, 999, 1999], 4096, 4)


def test_prefill_clamps_a_bad_length_and_reports_it():
    """A prompt length above t_max is clamped to t_max and flagged in the device status word;
    the rows computed are those of the clamped length."""
    B, Hq, Hkv, t_max = 1, 8, 1, 500
    q, k, v = _inputs(B, Hq, Hkv, t_max, 512, seed=3)
    p = _plan(B, Hq, Hkv, [500], 512, window=64, sinks=4)
    out_bad = torch.empty((B, Hq, t_max, 128), device=DEV)
    out_ok = torch.empty((B, Hq, t_max, 128), device=DEV)
    with make_handle(p, window=64, sinks=4) as h:
        h.prefill(q, k, v, torch.tensor([t_max], dtype=torch.int32, device=DEV),
                  np.array([0], np.uint8), out_ok)
        torch.cuda.synchronize()
        assert h.device_status() == 0
        h.prefill(q, k, v, torch.tensor([t_max + 7], dtype=torch.int32, device=DEV),
                  np.array([0], np.uint8), out_bad)
        torch.cuda.synchronize()
        assert h.device_status() & rtp.DEV_BAD_SEQLEN
    assert torch.equal(out_bad, out_ok)


def test_prefill_rejects_bad_arguments_before_launch():
    """t_max beyond the cache and a NULL pointer are refused on the host, nothing launched."""
    B, Hq, Hkv = 1, 8, 1
    q, k, v = _inputs(B, Hq, Hkv, 65, 64, seed=1)  # t_max 65 > max_ctx 64
    seq = torch.tensor([64], dtype=torch.int32, device=DEV)
    out = torch.full((B, Hq, 65, 128), 3.0, device=DEV)
    p = _plan(B, Hq, Hkv, [64], 64)
    with make_handle(p) as h:
        with pytest.raises(rtp.RtpError) as e:
            h.prefill(q, k, v, seq, np.array([1], np.uint8), out)
        assert e.value.status == rtp.RTP_ERR_INVALID_ARG
        io = rtp.PrefillIO(q[:, :, :64].contiguous().data_ptr(), k.data_ptr(), None,
                           seq.data_ptr(), np.array([0], np.uint8).ctypes.data_as(
                               rtp.ctypes.POINTER(rtp.ctypes.c_uint8)), out.data_ptr(), 64, 0)
        assert rtp.load().rtp_prefill(h._h, rtp.ctypes.byref(io), None) == rtp.RTP_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert bool((out == 3.0).all())
