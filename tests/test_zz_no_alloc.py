"""The no-allocation attention entry point, rtp_window_attention_noalloc.

It serves callers that cannot allocate device memory -- an engine that hands out memory only
from its own pre-planned pool, or a latency-critical path where cudaMalloc (which can
synchronise the device) must not run. Its scratch is a fixed device array inside the library.

These tests call it through the C-ABI twice in a row, after a first call that does the one-time
look-up of the array's address, and check:
  * each result against the handle-based entry point's: bit-identical to rtp_dense_decode (the
    same attention and merge kernels on the same grid), and for local heads within the parity
    bars of rtp_decode_step, which runs a layer of local heads as one cluster launch that merges
    inside the launch instead (another summation order), as well as against the
    oracle;
  * the caching allocator's allocated and reserved bytes do not move across the two calls;
  * a handle created earlier for a larger layer still decodes correctly afterwards (the
    kernel's shared-memory limit is shared with every handle and must never be lowered).
The file is collected last on purpose, so that a failure here comes after every other test.
"""
import numpy as np
import pytest
import torch

from head_wise_sparse_retrieval_b200 import rtp
from head_wise_sparse_retrieval_b200 import workloads as W

from parity_utils import check_layer, check_output, make_handle, oracle_head, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rtp.load()


def _big_plan():
    """48 KV heads over 12 sequences (more than the no-alloc layer's 12), two of them retrieval
    heads, so the handle's attention and selection need more shared memory than the call's."""
    B = 12
    return W.custom(batch=B, num_q_heads=32, num_kv_heads=4, seq_lens=[3000 + 37 * b for b in range(B)],
                    max_ctx=3500, retrieval=[1, 0, 1, 0],
                    kinds=[[W.KIND_DIFFUSE, 0, W.KIND_CONC, 0]] * B,
                    n_needles=[[0, 0, 3, 0]] * B, seed=41)


@pytest.mark.parametrize("dense", [False, True])
def test_noalloc_matches_handle_entry_points_on_two_calls(dense):
    big = _big_plan()
    big_li = W.make_layer(big, 0, "cuda")
    p = W.custom(batch=3, num_q_heads=32, num_kv_heads=4, seq_lens=[20000, 9000, 5],
                 max_ctx=20011, retrieval=[0, 0, 0, 0], kinds=[[0, 0, 0, 0]] * 3, seed=31)
    li = W.make_layer(p, 0, "cuda")
    with make_handle(big) as hb:  # exists before the no-alloc calls
        with make_handle(p) as h:
            ref, _ = run_layer(h, p, li, 0, dense=dense)
        outs = [torch.full_like(ref, float("nan")) for _ in range(3)]
        kw = dict(window=p.window, sinks=p.sinks, dense=dense)
        # first call on the device: looks up the scratch array's address
        rtp.window_attention_noalloc(li.q, li.k_cache, li.v_cache, li.seq_lens, outs[0], **kw)
        torch.cuda.synchronize()
        alloc0, reserved0 = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
        for call in (1, 2):
            rtp.window_attention_noalloc(li.q, li.k_cache, li.v_cache, li.seq_lens, outs[call],
                                         **kw)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == alloc0
        assert torch.cuda.memory_reserved() == reserved0
        for call in (1, 2):
            if dense:
                assert torch.equal(outs[call], ref), f"call {call}: differs from the handle path"
            else:
                got, want = outs[call].cpu().numpy(), ref.cpu().numpy().astype(np.float64)
                for b in range(p.batch):
                    for kvh in range(p.num_kv_heads):
                        if int(p.seq_lens[b]) > 0:
                            check_output(got[b, kvh * 8:(kvh + 1) * 8], want[b, kvh * 8:(kvh + 1) * 8],
                                         f"call {call} b{b} kvh{kvh} vs the handle path")
        # and against the oracle on a few heads (the handle path's own parity is tested elsewhere)
        out_h = outs[2].cpu().numpy()
        for b, kvh in [(0, 0), (1, 3), (2, 1)]:
            ho = oracle_head(li, b, kvh, False, 0.9, 8, p.window, p.sinks, dense=dense)
            check_output(out_h[b, kvh * 8:(kvh + 1) * 8], ho.out, f"noalloc b{b} kvh{kvh}")
        # the larger handle decodes after the no-alloc calls
        rep = check_layer(hb, big, big_li, 0, heads=[(0, 0), (5, 1), (11, 2), (7, 3)],
                          exact=False)
        assert len(rep.heads) == 4


def test_noalloc_rejects_sizes_beyond_its_scratch():
    B, H = 17, 4  # 68 KV heads > RTP_NOALLOC_MAX_HEADS
    q = torch.zeros((B, 8 * H, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((B, H, 16, 128), dtype=torch.bfloat16, device="cuda")
    seq = torch.full((B,), 16, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, 8 * H, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(rtp.RtpError) as e:
        rtp.window_attention_noalloc(q, kc, kc, seq, out)
    assert e.value.status == rtp.RTP_ERR_UNSUPPORTED
    assert "RTP_NOALLOC_MAX_HEADS" in str(e.value)
