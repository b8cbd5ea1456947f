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
// One CTA per (b, selected KV head), 128 threads: thread t owns output i = t / 8 and the
// 16-byte chunks t % 8, t % 8 + 8, ... of the weight row (all loaded before any sum); the 8
// partial sums of an output are added by a fixed shuffle tree (fp32 throughout, rounded to
// fp16 once). Zero chunks past G * D add exact zeros, so the sums do not depend on G.
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kIdxThreads = 128;
constexpr int kChunk = 8;  // bf16 per 16-byte load

__device__ __forceinline__ float dot8(const uint4& w, const uint4& x) {
  const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
  const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    acc = fmaf(bf16_lo(wv[k]), bf16_lo(xv[k]), acc);
    acc = fmaf(bf16_hi(wv[k]), bf16_hi(xv[k]), acc);
  }
  return acc;
}

}  // namespace

__global__ void __launch_bounds__(kIdxThreads) indexer_kernel(const IndexerArgs x) {
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x / x.nsel, hs = blockIdx.x - b * x.nsel;
  const int h = x.heads[hs];
  const int i = tid >> 3, part = tid & 7;  // output i of 16, partial 0..7
  const int GD = x.G * kHeadDim;

  // q_idx: the weight row and the group's queries, 16-byte chunks part, part + 8, ...
  const uint4* wq = reinterpret_cast<const uint4*>(x.w_q + ((size_t)h * kIdxDim + i) * GD);
  const uint4* qg = reinterpret_cast<const uint4*>(
      x.q_pre + ((size_t)b * x.Hq + (size_t)h * x.G) * kHeadDim);
  // G <= 8, so a thread has at most 16 chunks: all loads are issued before the sums
  constexpr int kMaxIter = kMaxGroup * kHeadDim / kChunk / 8;
  uint4 wv[kMaxIter], xv[kMaxIter];
#pragma unroll
  for (int k = 0; k < kMaxIter; ++k) {
    const int c = part + 8 * k;
    const bool in = c < GD / kChunk;
    wv[k] = in ? __ldg(wq + c) : make_uint4(0, 0, 0, 0);
    xv[k] = in ? __ldg(qg + c) : make_uint4(0, 0, 0, 0);
  }
  float aq = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxIter; ++k) aq += dot8(wv[k], xv[k]);
  // k_idx row: D = 128 -> 16 chunks, two per partial
  const uint4* wk = reinterpret_cast<const uint4*>(x.w_k + ((size_t)h * kIdxDim + i) * kHeadDim);
  const uint4* kh = reinterpret_cast<const uint4*>(x.k_pre + ((size_t)b * x.Hkv + h) * kHeadDim);
  float ak = dot8(__ldg(wk + part), __ldg(kh + part));
  ak += dot8(__ldg(wk + part + 8), __ldg(kh + part + 8));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {  // lanes 8j .. 8j+7 hold the partials of one output
    aq += __shfl_xor_sync(0xffffffffu, aq, o);
    ak += __shfl_xor_sync(0xffffffffu, ak, o);
  }
  if (part == 0) {
    int n = x.seq_lens[b];
    if (n < 1 || n > x.max_ctx) {
      atomicOr(x.status, kDevBadSeqlen);
      n = n < 1 ? 1 : x.max_ctx;
    }
    x.q_idx[((size_t)b * x.Hkv + h) * kIdxDim + i] = __float2half_rn(aq);
    x.k_idx[(((size_t)b * x.Hkv + h) * x.max_ctx + (n - 1)) * kIdxDim + i] = __float2half_rn(ak);
  }
}

}  // namespace rtp
