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
// Work item = (b, KV head, rows 2p and 2p + 1): two decode problems whose token sets differ in
// at most two positions, attended by one warp over the union of the two sets with the decode
// attention's gather (attend_tile.cuh): 16-token tiles from the warp's own 2-stage cp.async
// pipeline. Each tile's K and V fragments are loaded from shared memory once and used by both
// rows: S^T = K Q^T on the tensor cores with the G query heads of the group as N = 8, per row;
// each row masks the tokens outside its own set, keeps its own online softmax (log2 domain) and
// adds O^T += V^T P^T. A warp owns an item's whole token set, so nothing is merged across warps
// or CTAs. The grid is persistent (every CTA resident); warps take items round-robin, head by
// head, each head's last rows first.
#include "attend_tile.cuh"
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kPW = kPrefillWarps;
constexpr int kPT = kPW * 32;
constexpr int kPDepth = 2;  // cp.async stages per warp (12 warps per SM hide the latency)

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

// Row r of a prompt has key j in its set: j <= r, and for a local head j < sinks or j > r - window.
__device__ __forceinline__ bool in_row_set(int j, int r, bool local, int window, int sinks) {
  return j <= r && (!local || j < sinks || j > r - window);
}

// The online-softmax update of one row for one tile: x[0..3] are its scaled scores (tokens g, g,
// g + 8, g + 8; query heads 2t, 2t + 1), masked to -inf outside the row's set. Returns P (bf16,
// transposed for the B operand of O^T += V^T P^T). A row whose maximum is still -inf (no key of
// its set seen yet) keeps zero weights.
__device__ __forceinline__ void row_softmax(float (&x)[4], TileAcc& st, uint32_t& pb0,
                                            uint32_t& pb1) {
  float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  const float mn0 = fmaxf(st.m0, mx0), mn1 = fmaxf(st.m1, mx1);
  if (__any_sync(0xffffffffu, mn0 > st.m0 || mn1 > st.m1)) {  // rescale when a max grows
    const float al0 = (mn0 > st.m0) ? exp2f(st.m0 - mn0) : 1.f;
    const float al1 = (mn1 > st.m1) ? exp2f(st.m1 - mn1) : 1.f;
    st.l0 *= al0;
    st.l1 *= al1;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      st.acc[mt][0] *= al0;
      st.acc[mt][1] *= al1;
      st.acc[mt][2] *= al0;
      st.acc[mt][3] *= al1;
    }
    st.m0 = mn0;
    st.m1 = mn1;
  }
  const float b0 = (st.m0 == -INFINITY) ? 0.f : st.m0;  // exp2(-inf - 0) = 0
  const float b1 = (st.m1 == -INFINITY) ? 0.f : st.m1;
  const uint32_t p01 = pack_bf16x2(exp2f(x[0] - b0), exp2f(x[1] - b1));
  const uint32_t p23 = pack_bf16x2(exp2f(x[2] - b0), exp2f(x[3] - b1));
  st.l0 += bf16_lo(p01) + bf16_lo(p23);
  st.l1 += bf16_hi(p01) + bf16_hi(p23);
  pb0 = movmatrix_trans(p01);
  pb1 = movmatrix_trans(p23);
}

// One tile for the two rows rr[0] >= rr[1] of an item: the stage at kb holds n valid tokens
// whose positions sit in lanes 0..15 of pos.
__device__ __forceinline__ void prefill_tile2(uint32_t kb, const uint32_t (&qf)[2][8][2], int n,
                                              int pos, const int (&rr)[2], bool local,
                                              int window, int sinks, float scale_log2,
                                              int lane, TileAcc (&st)[2]) {
  const int g = lane >> 2;
  const int k_row = (lane & 7) + ((lane >> 3) & 1) * 8, k_col = lane >> 4;
  const int v_row = kTile + (lane & 7) + (lane >> 4) * 8, v_col = (lane >> 3) & 1;
  // positions of this lane's tokens g and g + 8
  const int p_lo = __shfl_sync(0xffffffffu, pos, g);
  const int p_hi = __shfl_sync(0xffffffffu, pos, g + 8);
  uint32_t pb[2][2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    // S^T (16 tokens x 8 heads) = K (16 x 128) . Q_r^T (128 x 8), two accumulator chains; the
    // K fragments are read from shared memory again for the second row (fewer live registers)
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ks += 2) {
      uint32_t fa[4], fb[4];
      ldmatrix_x4(fa, kb + tile_swz(k_row, 2 * ks + k_col));
      ldmatrix_x4(fb, kb + tile_swz(k_row, 2 * ks + 2 + k_col));
      mma_bf16_16816(sa, fa, qf[r][ks][0], qf[r][ks][1]);
      mma_bf16_16816(sb, fb, qf[r][ks + 1][0], qf[r][ks + 1][1]);
    }
    const bool v_lo = g < n && in_row_set(p_lo, rr[r], local, window, sinks);
    const bool v_hi = g + 8 < n && in_row_set(p_hi, rr[r], local, window, sinks);
    float x[4];
    x[0] = v_lo ? (sa[0] + sb[0]) * scale_log2 : -INFINITY;
    x[1] = v_lo ? (sa[1] + sb[1]) * scale_log2 : -INFINITY;
    x[2] = v_hi ? (sa[2] + sb[2]) * scale_log2 : -INFINITY;
    x[3] = v_hi ? (sa[3] + sb[3]) * scale_log2 : -INFINITY;
    row_softmax(x, st[r], pb[r][0], pb[r][1]);
  }
  // O^T (128 dims x 8 heads) += V^T (128 x 16 tokens) . P^T (16 x 8), per row
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    uint32_t fv[4];
    ldmatrix_x4_trans(fv, kb + tile_swz(v_row, 2 * mt + v_col));
    mma_bf16_16816(st[0].acc[mt], fv, pb[0][0], pb[0][1]);
    mma_bf16_16816(st[1].acc[mt], fv, pb[1][0], pb[1][1]);
  }
}

}  // namespace

size_t prefill_smem_bytes() { return (size_t)kPW * kPDepth * kWarpStage; }

// The bound of 3 CTAs per SM caps the registers at 170 (the two rows' accumulators and queries
// stay in registers; a few item-level values spill); 64 KB of stages per CTA admit three CTAs
// per SM in shared memory as well.
__global__ void __launch_bounds__(kPT, 3) prefill_kernel(const PrefillArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t my_stages = smem_u32(smem) + (uint32_t)warp * kPDepth * kWarpStage;
  const uint64_t policy = l2_policy_evict_first();
  const float scale_log2 = a.attn_scale_log2;
  const int BH = a.B * a.Hkv;
  const int pairs = (a.t_max + 1) / 2;  // rows 2p, 2p + 1 of each head
  const long long items = (long long)BH * pairs;
  const size_t head_stride = (size_t)a.t_max * kHeadDim;  // one query head's rows

  for (long long it = (long long)blockIdx.x * kPW + warp; it < items;
       it += (long long)gridDim.x * kPW) {
    // item -> ((b, KV head), row pair p): heads one after the other, each from its last rows
    // (the longest sets) down, so that warp w takes every nw-th pair of every head (balanced)
    // and the warps of a CTA take adjacent rows of one head (nearly the same key tiles)
    const int bh = (int)(it / pairs);
    const int p = pairs - 1 - (int)(it - (long long)bh * pairs);
    const int b = bh / a.Hkv, kvh = bh - b * a.Hkv;
    int T = __ldg(a.seq_lens + b);
    if (T < 1 || T > a.t_max) {  // clamped and reported
      if (lane == 0) atomicOr(a.status, kDevBadSeqlen);
      T = T < 1 ? 1 : a.t_max;
    }
    const int lo = 2 * p;
    if (lo >= T) continue;  // the same for the whole warp
    const int hi = min(lo + 1, T - 1);  // == lo: a single row (the last of an odd prompt)
    const int rr[2] = {hi, lo};
    const unsigned long long mword = kvh < 64 ? a.ret_bits0 : kvh < 128 ? a.ret_bits1
                                   : kvh < 192 ? a.ret_bits2 : a.ret_bits3;
    const bool local = !a.dense && !((mword >> (kvh & 63)) & 1ull);
    // the union of the two rows' sets, ascending: ranks k < n1 are positions k, the rest
    // lo2 + (k - n1), up to hi. Row lo's set is [0, S) U [lo + 1 - W, lo] once lo + 1 > W + S,
    // and then row hi's is inside [0, S) U [lo + 1 - W, hi]; before that the union is [0, hi].
    int n1 = hi + 1, lo2 = hi + 1;
    if (local && lo + 1 > a.window + a.sinks) {
      n1 = a.sinks;
      lo2 = lo + 1 - a.window;
    }
    const int len = n1 + (hi + 1 - lo2);
    const int ntiles = (len + kTile - 1) / kTile;

    const size_t head = (size_t)b * a.Hkv + kvh;
    const __nv_bfloat16* kbase = a.k_cache + head * (size_t)a.max_ctx * kHeadDim;
    const __nv_bfloat16* vbase = a.v_cache + head * (size_t)a.max_ctx * kHeadDim;
    const __nv_bfloat16* qg = a.q + (size_t)(b * a.Hq + kvh * a.G) * head_stride;
    uint32_t qf[2][8][2];
    load_q_rows(qf[0], qg + (size_t)hi * kHeadDim, head_stride, a.G, lane);
    load_q_rows(qf[1], qg + (size_t)lo * kHeadDim, head_stride, a.G, lane);

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

    TileAcc st[2];
    st[0].init();
    st[1].init();
    for (int s = 0; s < ntiles; ++s) {
      issue(s + kPDepth - 1);
      const int pos = tile_pos(s);
      cp_async_wait<kPDepth - 1>();  // tile s landed
      __syncwarp();
      prefill_tile2(my_stages + (uint32_t)(s % kPDepth) * kWarpStage, qf,
                    min(kTile, len - s * kTile), pos, rr, local, a.window, a.sinks, scale_log2,
                    lane, st);
      __syncwarp();  // the stage is refilled kPDepth - 1 tiles later
    }
    cp_async_wait<0>();  // the trailing empty groups; the stages are free for the next item
    __syncwarp();

    // per row: l over the 8 lanes of a column (query head), then out = O / l
    const int g = lane >> 2, t = lane & 3;
    const bool h0 = 2 * t < a.G, h1 = 2 * t + 1 < a.G;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if (r == 1 && lo == hi) break;  // a single row: written once
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        st[r].l0 += __shfl_xor_sync(0xffffffffu, st[r].l0, o);
        st[r].l1 += __shfl_xor_sync(0xffffffffu, st[r].l1, o);
      }
      const float inv0 = 1.f / st[r].l0, inv1 = 1.f / st[r].l1;
      float* o0 = a.out + ((size_t)(b * a.Hq + kvh * a.G + 2 * t) * a.t_max + rr[r]) * kHeadDim;
      float* o1 = o0 + head_stride;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {  // acc[mt]: dims 16 mt + g (c0, c1) and + 8 (c2, c3)
        const int d = 16 * mt + g;
        if (h0) {
          o0[d] = st[r].acc[mt][0] * inv0;
          o0[d + 8] = st[r].acc[mt][2] * inv0;
        }
        if (h1) {
          o1[d] = st[r].acc[mt][1] * inv1;
          o1[d + 8] = st[r].acc[mt][3] * inv1;
        }
      }
    }
  }
}

}  // namespace rtp
