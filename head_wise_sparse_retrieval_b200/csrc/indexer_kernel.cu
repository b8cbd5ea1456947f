// indexer_kernel.cu -- indexer production at decode (sm_100a).
//
// Follows "Full Attention Strikes Back ..." (xllm-io paper review), section 三, 核心公式 /
// 自适应稀疏注意力: the retrieval score s_h(m,n) = (W^Q_h q^pre_{m,h})^T (W^K_h k^pre_{n,h})
// uses low-rank projections of the queries and keys taken before RoPE. At a decode step the
// current token contributes one indexer query per KV head and one new indexer-key row:
//   q_idx[b][h][i]        = fp16( sum_{j < G*D} Wq[h][i][j] * q_pre[b][h*G + j/D][j%D] )
//   k_idx[b][h][N_b-1][i] = fp16( sum_{d < D}   Wk[h][i][d] * k_pre[b][h][d] )
// with the G query heads of the KV head's group concatenated head-major.
//
// One warp per output i of one (b, selected KV head): kIdxSplit CTAs of kIdxWarps warps cover
// the r = 16 outputs. Lane l owns the 16-byte chunks l, l + 32, ... of the G*D-long weight row
// (at most 4) and chunk l of the D-long key row (lanes 0..15). The weights are model constants:
// they are loaded before the wait for the preceding launch, so only the activations q_pre /
// k_pre sit on the dependent path. Each lane sums its chunks in order in fp32, a fixed xor
// shuffle tree adds the 32 lanes, and the result is rounded to fp16 once. Zero chunks past
// G * D add exact zeros.
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kChunk = 8;                                  // bf16 per 16-byte load
constexpr int kQIter = kMaxGroup * kHeadDim / kChunk / 32;  // weight chunks per lane (4)

__device__ __forceinline__ float dot8(const uint4& w, const uint4& x, float acc) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc = fmaf(bf16_lo(wv[k]), bf16_lo(xv[k]), acc);
    acc = fmaf(bf16_hi(wv[k]), bf16_hi(xv[k]), acc);
  }
  return acc;
}

}  // namespace

__global__ void __launch_bounds__(kIdxWarps * 32) indexer_kernel(const IndexerArgs x) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int unit = blockIdx.x / kIdxSplit;                 // (b, selected head)
  const int i = (blockIdx.x - unit * kIdxSplit) * kIdxWarps + warp;  // output 0..15
  const int b = unit / x.nsel, hs = unit - b * x.nsel;
  const int h = x.heads[hs];
  const int nq = x.G * kHeadDim / kChunk;                  // chunks of the query row

  // the weights first: they do not depend on the preceding launch
  const uint4* wq = reinterpret_cast<const uint4*>(x.w_q + ((size_t)h * kIdxDim + i) * nq * kChunk);
  const uint4* wk = reinterpret_cast<const uint4*>(x.w_k + ((size_t)h * kIdxDim + i) * kHeadDim);
  uint4 wv[kQIter];
#pragma unroll
  for (int k = 0; k < kQIter; ++k) {
    const int c = lane + 32 * k;
    wv[k] = c < nq ? __ldg(wq + c) : make_uint4(0, 0, 0, 0);
  }
  const uint4 wkv = lane < kHeadDim / kChunk ? __ldg(wk + lane) : make_uint4(0, 0, 0, 0);

  pdl_wait();
  pdl_launch_dependents();
  const uint4* qg = reinterpret_cast<const uint4*>(
      x.q_pre + ((size_t)b * x.Hq + (size_t)h * x.G) * kHeadDim);
  const uint4* kh = reinterpret_cast<const uint4*>(x.k_pre + ((size_t)b * x.Hkv + h) * kHeadDim);
  uint4 xv[kQIter];
#pragma unroll
  for (int k = 0; k < kQIter; ++k) {
    const int c = lane + 32 * k;
    xv[k] = c < nq ? __ldcg(qg + c) : make_uint4(0, 0, 0, 0);
  }
  const uint4 kv = lane < kHeadDim / kChunk ? __ldcg(kh + lane) : make_uint4(0, 0, 0, 0);
  const int n_raw = x.seq_lens[b];
  float aq = 0.f;
#pragma unroll
  for (int k = 0; k < kQIter; ++k) aq = dot8(wv[k], xv[k], aq);
  float ak = dot8(wkv, kv, 0.f);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    aq += __shfl_xor_sync(0xffffffffu, aq, o);
    ak += __shfl_xor_sync(0xffffffffu, ak, o);
  }
  if (lane == 0) {
    int n = n_raw;
    if (n < 1 || n > x.max_ctx) {
      atomicOr(x.status, kDevBadSeqlen);
      n = n < 1 ? 1 : x.max_ctx;
    }
    x.q_idx[((size_t)b * x.Hkv + h) * kIdxDim + i] = __float2half_rn(aq);
    x.k_idx[(((size_t)b * x.Hkv + h) * x.max_ctx + (n - 1)) * kIdxDim + i] = __float2half_rn(ak);
  }
}

}  // namespace rtp
