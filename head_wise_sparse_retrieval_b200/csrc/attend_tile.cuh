// attend_tile.cuh -- the attention tile step shared by attend_kernel (attend_kernel.cu) and the
// single-launch layer (fused_kernel.cu), sm_100a.
//
// Follows "Full Attention Strikes Back ..." (xllm-io paper review), section 三, 核心公式 /
// 自适应稀疏注意力: O_h(m) = sum_{n in S} softmax_S(q^T k_n / sqrt(d_h)) v_n, computed by one
// warp 16 tokens at a time for the G <= 8 query heads of a KV head (the GQA group shares the
// token set S):
//   * gather_tile: the tile's 16 K rows and 16 V rows (256 B each) into the warp's stage with
//     16-byte cp.async (L2 evict-first); rows past the tile's n tokens are zero-filled, not
//     read. Shared-memory rows are XOR-swizzled so that the 8 rows an ldmatrix reads hit 8
//     different bank groups;
//   * attend_tile: S^T (16 tokens x 8 heads) = K Q^T on the tensor cores (warp MMA m16n8k16,
//     bf16 in, fp32 accumulate), online softmax in the log2 domain (rescaled only when a
//     maximum grows), P rounded to bf16 and transposed in registers (movmatrix), and
//     O^T (128 dims x 8 heads) += V^T P^T. The normaliser l is summed from the same rounded P.
#pragma once

#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

constexpr int kTile = 16;                          // tokens per warp tile
constexpr int kWarpStage = 2 * kTile * kRowBytes;  // one stage: 16 K rows, then 16 V rows

// Byte offset of 16-byte column c of row r in a stage: 256-byte rows, the column XOR-swizzled
// with the row.
__device__ __forceinline__ uint32_t tile_swz(int r, int c) {
  return (uint32_t)(r * kRowBytes + ((c ^ (r & 7)) << 4));
}

// Size and position of the window + sinks set of a local head with N tokens: the first S
// positions and the last W, as a set union (all N when they overlap).
__device__ __forceinline__ int window_len(int N, int W, int S) {
  return (N <= W + S) ? N : W + S;
}
__device__ __forceinline__ int window_pos(int r, int N, int W, int S) {
  return (N <= W + S) ? r : (r < S ? r : N - W + (r - S));
}

// Gathers a tile's K and V rows into `stage`: lane l copies 16-byte column c = l % 16 of rows
// 2i + l / 16; the cache positions come from lanes 0..15 of pos. A position outside [0, N) (a
// corrupted list) is replaced by 0 and reported once per tile; rows past n are zero-filled.
// One commit group is left to the caller.
__device__ __forceinline__ void gather_tile(uint32_t stage, const __nv_bfloat16* kbase,
                                            const __nv_bfloat16* vbase, int N, int pos, int n,
                                            int lane, uint64_t policy, unsigned* status) {
  const int c = lane & 15, par = lane >> 4;
  // tile_swz(2i + par, c) = (2i + par) * 256 + ((c ^ ((2i + par) & 7)) << 4)
  //                       = par * 256 + 512 i + (((c ^ par) ^ 2 (i & 3)) << 4)
  const uint32_t lane_base = stage + (uint32_t)par * kRowBytes;
  const int cx = c ^ par;
  const __nv_bfloat16* kcol = kbase + c * 8;
  const __nv_bfloat16* vcol = vbase + c * 8;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kTile / 2; ++i) {
    const int row = 2 * i + par;
    const int p = __shfl_sync(0xffffffffu, pos, row);
    const bool valid = row < n;
    const bool in = (unsigned)p < (unsigned)N;
    bad |= valid && !in;
    const size_t off = (valid && in) ? (size_t)p * kHeadDim : 0;
    const unsigned bytes = valid ? 16u : 0u;
    const uint32_t dst = lane_base + 512u * i + ((uint32_t)(cx ^ (2 * (i & 3))) << 4);
    cp_async_16(dst, kcol + off, bytes, policy);
    cp_async_16(dst + kTile * kRowBytes, vcol + off, bytes, policy);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, kDevBadIndex);
}

// A warp's running attention state for its 8 query-head columns: the maxima m (log2 domain)
// and sums l of query heads 2t and 2t + 1 (t = lane % 4), and O^T in MMA accumulator layout.
struct TileAcc {
  float m0, m1, l0, l1;
  float acc[8][4];
  __device__ __forceinline__ void init() {
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  }
};

// Loads Q^T as the MMA's B operand for query heads g = lane / 4 < G (zeros above):
// b0 = q[g][16 ks + 2t, +1], b1 = q[g][16 ks + 8 + 2t, +1].
__device__ __forceinline__ void load_q_frag(uint32_t (&qf)[8][2], const __nv_bfloat16* qgroup,
                                            int G, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const bool valid = g < G;
  const uint32_t* qrow = reinterpret_cast<const uint32_t*>(qgroup + (valid ? g : 0) * kHeadDim);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    qf[ks][0] = valid ? qrow[ks * 8 + t] : 0u;
    qf[ks][1] = valid ? qrow[ks * 8 + 4 + t] : 0u;
  }
}

// One tile of the online-softmax attention over the stage at kb holding n valid tokens
// (n >= 1; token 0 of a piece's first tile is always valid, so the maxima stay finite).
__device__ __forceinline__ void attend_tile(uint32_t kb, const uint32_t (&qf)[8][2], int n,
                                            float scale_log2, int lane, TileAcc& st) {
  const int g = lane >> 2;
  // ldmatrix rows / 16-byte columns this lane addresses (before the swizzle)
  const int k_row = (lane & 7) + ((lane >> 3) & 1) * 8, k_col = lane >> 4;
  const int v_row = kTile + (lane & 7) + (lane >> 4) * 8, v_col = (lane >> 3) & 1;
  // S^T (16 tokens x 8 heads) = K (16 x 128) . Q^T (128 x 8), two accumulator chains
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int ks = 0; ks < 8; ks += 2) {
    uint32_t fa[4], fb[4];
    ldmatrix_x4(fa, kb + tile_swz(k_row, 2 * ks + k_col));
    ldmatrix_x4(fb, kb + tile_swz(k_row, 2 * ks + 2 + k_col));
    mma_bf16_16816(sa, fa, qf[ks][0], qf[ks][1]);
    mma_bf16_16816(sb, fb, qf[ks + 1][0], qf[ks + 1][1]);
  }
  // rows: token g (c0: head 2t, c1: head 2t+1) and token g+8 (c2, c3)
  float x0 = (sa[0] + sb[0]) * scale_log2, x1 = (sa[1] + sb[1]) * scale_log2;
  float x2 = (sa[2] + sb[2]) * scale_log2, x3 = (sa[3] + sb[3]) * scale_log2;
  if (g >= n) x0 = x1 = -INFINITY;
  if (g + 8 >= n) x2 = x3 = -INFINITY;
  float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  const float mn0 = fmaxf(st.m0, mx0), mn1 = fmaxf(st.m1, mx1);  // finite: token 0 is valid
  if (__any_sync(0xffffffffu, mn0 > st.m0 || mn1 > st.m1)) {   // rescale when a max grows
    const float al0 = exp2f(st.m0 - mn0), al1 = exp2f(st.m1 - mn1);
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
  const uint32_t p01 = pack_bf16x2(exp2f(x0 - st.m0), exp2f(x1 - st.m1));
  const uint32_t p23 = pack_bf16x2(exp2f(x2 - st.m0), exp2f(x3 - st.m1));
  st.l0 += bf16_lo(p01) + bf16_lo(p23);
  st.l1 += bf16_hi(p01) + bf16_hi(p23);
  // P^T as the B operand: transpose the 8x8 (token x head) blocks in registers
  const uint32_t pb0 = movmatrix_trans(p01);
  const uint32_t pb1 = movmatrix_trans(p23);
  // O^T (128 dims x 8 heads) += V^T (128 x 16 tokens) . P^T (16 x 8)
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    uint32_t fv[4];
    ldmatrix_x4_trans(fv, kb + tile_swz(v_row, 2 * mt + v_col));
    mma_bf16_16816(st.acc[mt], fv, pb0, pb1);
  }
}

}  // namespace rtp
