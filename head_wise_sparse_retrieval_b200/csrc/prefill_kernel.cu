// prefill_kernel.cu -- causal attention over every position of a prompt (sm_100a).
//
// Follows the gist.science technical summary, Methodology 1 (during prefill the retrieval heads
// keep, and attend over, the full KV cache; the local heads keep a sliding window with attention
// sinks) and "Full Attention Strikes Back ..." (xllm-io paper review), section 五 测试配置
// (window 8192, 4 sinks) and its prefill speed-up table. Row i (0-based position) of a prompt
// attends over the set a decode step over the first i + 1 tokens uses:
//   retrieval head (or dense):  { j : j <= i }
//   local head:                 { 0 .. sinks-1 } U { i+1-window .. i }   (all i + 1 when they meet)
// o_i = sum_j softmax_j(q_i . k_j / sqrt(d_h)) v_j, for the G query heads of the KV head.
//
// Work item = (b, KV head, row i): one decode problem whose token set is the row's set above,
// attended by one warp with the decode attention's tile step (attend_tile.cuh): 16-token tiles
// gathered by the warp's own 3-stage cp.async pipeline, S^T = K Q^T on the tensor cores with the
// G query heads of the group as N = 8, online softmax, O^T += V^T P^T. A warp owns an item's
// whole token set, so nothing is merged across warps or CTAs. The grid is persistent (every CTA
// resident); warps take items round-robin, head by head, each head's last rows first.
#include "attend_tile.cuh"
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kPW = kPrefillWarps;
constexpr int kPT = kPW * 32;
constexpr int kPDepth = 3;  // cp.async stages per warp

// B operand of the S MMA for row i: b0 = q[g][16 ks + 2t, +1], b1 = q[g][16 ks + 8 + 2t, +1] for
// query head g = lane / 4 < G of the group (zeros above). Rows of one head are t_max apart.
__device__ __forceinline__ void load_q_rows(uint32_t (&qf)[8][2], const __nv_bfloat16* q0,
                                            size_t head_stride, int G, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const bool valid = g < G;
  const uint32_t* qrow =
      reinterpret_cast<const uint32_t*>(q0 + (valid ? (size_t)g * head_stride : 0));
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    qf[ks][0] = valid ? qrow[ks * 8 + t] : 0u;
    qf[ks][1] = valid ? qrow[ks * 8 + 4 + t] : 0u;
  }
}

}  // namespace

size_t prefill_smem_bytes() { return (size_t)kPW * kPDepth * kWarpStage; }

__global__ void __launch_bounds__(kPT, 2) prefill_kernel(const PrefillArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t my_stages = smem_u32(smem) + (uint32_t)warp * kPDepth * kWarpStage;
  const uint64_t policy = l2_policy_evict_first();
  const float scale_log2 = a.attn_scale_log2;
  const int BH = a.B * a.Hkv;
  const long long items = (long long)BH * a.t_max;
  const size_t head_stride = (size_t)a.t_max * kHeadDim;  // one query head's rows

  for (long long it = (long long)blockIdx.x * kPW + warp; it < items;
       it += (long long)gridDim.x * kPW) {
    // item -> ((b, KV head), row i): heads one after the other, each from its last row (the
    // longest set) down, so that warp w takes every nw-th row of every head (balanced) and
    // the warps of a CTA take adjacent rows of one head (nearly the same key tiles)
    const int bh = (int)(it / a.t_max);
    const int i = a.t_max - 1 - (int)(it - (long long)bh * a.t_max);
    const int b = bh / a.Hkv, kvh = bh - b * a.Hkv;
    int T = __ldg(a.seq_lens + b);
    if (T < 1 || T > a.t_max) {  // clamped and reported
      if (lane == 0) atomicOr(a.status, kDevBadSeqlen);
      T = T < 1 ? 1 : a.t_max;
    }
    if (i >= T) continue;  // the same for the whole warp
    const unsigned long long mword = kvh < 64 ? a.ret_bits0 : kvh < 128 ? a.ret_bits1
                                   : kvh < 192 ? a.ret_bits2 : a.ret_bits3;
    const bool local = !a.dense && !((mword >> (kvh & 63)) & 1ull);
    // the row's set in ascending order: ranks k < n1 are positions k, the rest lo2 + (k - n1)
    const int N = i + 1;
    int n1 = N, lo2 = N;
    if (local && N > a.window + a.sinks) {
      n1 = a.sinks;
      lo2 = N - a.window;
    }
    const int len = n1 + (N - lo2);
    const int ntiles = (len + kTile - 1) / kTile;

    const size_t head = (size_t)b * a.Hkv + kvh;
    const __nv_bfloat16* kbase = a.k_cache + head * (size_t)a.max_ctx * kHeadDim;
    const __nv_bfloat16* vbase = a.v_cache + head * (size_t)a.max_ctx * kHeadDim;
    uint32_t qf[8][2];
    load_q_rows(qf, a.q + ((size_t)(b * a.Hq + kvh * a.G) * a.t_max + i) * kHeadDim, head_stride,
                a.G, lane);

    // lane l < 16: position of token l of tile s (unused past the set)
    auto tile_pos = [&](int s) {
      const int k = s * kTile + lane;
      if (lane >= kTile || k >= len) return -1;
      return k < n1 ? k : lo2 + (k - n1);
    };
    auto issue = [&](int s) {  // one commit group per tile slot, empty past the set
      if (s < ntiles)
        gather_tile(my_stages + (uint32_t)(s % kPDepth) * kWarpStage, kbase, vbase, T,
                    tile_pos(s), min(kTile, len - s * kTile), lane, policy, a.status);
      cp_async_commit();
    };
    for (int s = 0; s < kPDepth - 1; ++s) issue(s);

    TileAcc st;
    st.init();
    for (int s = 0; s < ntiles; ++s) {
      issue(s + kPDepth - 1);
      cp_async_wait<kPDepth - 1>();  // tile s landed
      __syncwarp();
      attend_tile(my_stages + (uint32_t)(s % kPDepth) * kWarpStage, qf,
                  min(kTile, len - s * kTile), scale_log2, lane, st);
      __syncwarp();  // the stage is refilled kPDepth - 1 tiles later
    }
    cp_async_wait<0>();  // the trailing empty groups; the stages are free for the next item
    __syncwarp();

    // l over the 8 lanes of a column (query head), then out = O / l
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, o);
      st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, o);
    }
    const int g = lane >> 2, t = lane & 3;
    const float inv0 = 1.f / st.l0, inv1 = 1.f / st.l1;
    float* o0 = a.out + ((size_t)(b * a.Hq + kvh * a.G + 2 * t) * a.t_max + i) * kHeadDim;
    float* o1 = o0 + head_stride;
    const bool h0 = 2 * t < a.G, h1 = 2 * t + 1 < a.G;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {  // acc[mt]: dims 16 mt + g (c0, c1) and + 8 (c2, c3)
      const int d = 16 * mt + g;
      if (h0) {
        o0[d] = st.acc[mt][0] * inv0;
        o0[d + 8] = st.acc[mt][2] * inv0;
      }
      if (h1) {
        o1[d] = st.acc[mt][1] * inv1;
        o1[d + 8] = st.acc[mt][3] * inv1;
      }
    }
  }
}

}  // namespace rtp
