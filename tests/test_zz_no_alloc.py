"""The no-allocation attention entry point, rtp_window_attention_noalloc.

It serves callers that cannot allocate device memory -- an engine that hands out memory only
from its own pre-planned pool, or a latency-critical path where cudaMalloc (which can
synchronise the device) must not run. Its scratch is a fixed device array inside the library.
These tests call it through the C-ABI twice in a row and compare each result with the handle-
based entry points (rtp_decode_step for local heads, rtp_dense_decode), within the tolerances
of the other parity tests. The file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from head_wise_sparse_retrieval_b200 import rtp
from head_wise_sparse_retrieval_b200 import workloads as W

from parity_utils import MAX_ABS, MEAN_ABS, make_handle, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    rtp.load()


@pytest.mark.parametrize("dense", [False, True])
def test_noalloc_matches_handle_entry_points_on_two_calls(dense):
    p = W.custom(batch=3, num_q_heads=32, num_kv_heads=4, seq_lens=[20000, 9000, 5],
                 max_ctx=20011, retrieval=[0, 0, 0, 0], kinds=[[0, 0, 0, 0]] * 3, seed=31)
    li = W.make_layer(p, 0, "cuda")
    with make_handle(p) as h:
        ref, _ = run_layer(h, p, li, 0, dense=dense)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        rtp.window_attention_noalloc(li.q, li.k_cache, li.v_cache, li.seq_lens, out,
                                     window=p.window, sinks=p.sinks, dense=dense)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), f"call {call}: non-finite output"
        err = (out - ref).abs()
        assert float(err.max()) <= MAX_ABS, f"call {call}: max-abs {float(err.max()):.3e}"
        assert float(err.mean()) <= MEAN_ABS, f"call {call}: mean-abs {float(err.mean()):.3e}"


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
