// select_kernels.cu -- the sort-free top-p selection of the retrieval heads (sm_100a).
//
// Follows "Full Attention Strikes Back ..." (xllm-io paper review), section 三:
//   核心公式 / 自适应稀疏注意力  s_h(m,n) = (W^Q q^pre)^T (W^K k^pre),  S_h(m) = Top-P(s_h, p)
//   硬件感知解码内核            top-p without sorting, over a 256-bin histogram (O(1) per head)
// and the gist.science technical summary, Methodology 3 (mass accumulated until p is reached).
//
// Three launches per layer, each over (chunk, retrieval slot) with PDL between them:
//   score_kernel   streams the N x 16 fp16 indexer keys once (two 16-byte loads per token,
//                  a lane pair per token), writes the fp32 scaled scores (they stay in L2)
//                  and one maximum per 1024-token chunk;
//   hist_kernel    s_max = max of the chunk maxima; bins every score relative to s_max and
//                  adds exp(s - s_max) to 256 shared bins in 2^-40 fixed point
//                  (integer adds: the result does not depend on the order of arrival); the
//                  last CTA of a slot (atomic ticket, no waiting) scans the bins from the top
//                  with one warp and writes b*;
//                  The same CTAs count tokens per bin and chunk, so once b* is known the last
//                  CTA also writes how many tokens each chunk selects and their prefix;
//   compact_kernel re-bins with the same function and writes the selected positions, in
//                  ascending order, into one dense list (each chunk at its prefix offset).
// Bins need the global s_max, so the scores make one round trip through L2 (4 B per token
// against 32 B of indexer keys read from HBM).
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

__device__ __forceinline__ int clamp_seq_len(const LayerArgs& a, int b, unsigned* status,
                                             bool report) {
  int n = a.seq_lens[b];
  if (n < 1 || n > a.max_ctx) {
    if (report) atomicOr(status, kDevBadSeqlen);
    n = n < 1 ? 1 : a.max_ctx;
  }
  return n;
}

__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kSelThreads / 32; ++i) r = fmaxf(r, red[i]);
  __syncthreads();
  return r;
}

// ---- 1. indexer scores -------------------------------------------------------------------

__global__ void __launch_bounds__(kSelThreads) score_kernel(const LayerArgs a, const Workspace w) {
  __shared__ float red[kSelThreads / 32];
  pdl_wait();
  const int slot = blockIdx.y;
  const int b = slot / a.nret, kvh = a.ret_kvh[slot % a.nret];
  const int N = clamp_seq_len(a, b, w.status, blockIdx.x == 0 && threadIdx.x == 0);

  if (blockIdx.x == 0) {  // reset what the next two kernels accumulate into
    w.hist[(size_t)slot * kBins + threadIdx.x] = 0ull;
    if (threadIdx.x == 0) w.ticket_hist[slot] = 0u;
  }
  pdl_launch_dependents();

  const int n0 = blockIdx.x * kScoreChunk;
  if (n0 >= N) return;
  const int n1 = min(n0 + kScoreChunk, N);

  // a lane pair per token: the even lane holds dims 0..7, the odd lane dims 8..15
  const int half = threadIdx.x & 1, pair = threadIdx.x >> 1;
  const size_t head = (size_t)b * a.Hkv + kvh;
  float q[8];
  {
    const uint4 qv = *reinterpret_cast<const uint4*>(a.q_idx + head * kIdxDim + half * 8);
    const __half2* h2 = reinterpret_cast<const __half2*>(&qv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h2[i]);
      q[2 * i] = f.x;
      q[2 * i + 1] = f.y;
    }
  }
  const uint4* keys = reinterpret_cast<const uint4*>(a.k_idx + head * (size_t)a.max_ctx * kIdxDim);
  float* sc = w.scores + (size_t)slot * w.ld;

  constexpr int kIter = kScoreChunk / (kSelThreads / 2);  // 8 tokens per lane pair
  uint4 kv[kIter];
#pragma unroll
  for (int it = 0; it < kIter; ++it) {
    const int n = n0 + it * (kSelThreads / 2) + pair;
    kv[it] = (n < n1) ? __ldcs(keys + 2 * (size_t)n + half) : make_uint4(0, 0, 0, 0);
  }
  float mx = -INFINITY;
#pragma unroll
  for (int it = 0; it < kIter; ++it) {
    const int n = n0 + it * (kSelThreads / 2) + pair;
    const __half2* h2 = reinterpret_cast<const __half2*>(&kv[it]);
    float p[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h2[i]);
      p[2 * i] = __fmul_rn(q[2 * i], f.x);       // fp16 x fp16 products are exact in fp32
      p[2 * i + 1] = __fmul_rn(q[2 * i + 1], f.y);
    }
    // pairwise sum: 8 products, then the partner lane's 8
    const float s01 = __fadd_rn(p[0], p[1]), s23 = __fadd_rn(p[2], p[3]);
    const float s45 = __fadd_rn(p[4], p[5]), s67 = __fadd_rn(p[6], p[7]);
    const float part = __fadd_rn(__fadd_rn(s01, s23), __fadd_rn(s45, s67));
    const float other = __shfl_xor_sync(0xffffffffu, part, 1);
    const float s = __fmul_rn(__fadd_rn(part, other), a.idx_scale);
    if (n < n1) {
      if (half == 0) sc[n] = s;
      mx = fmaxf(mx, s);
    }
  }
  mx = block_max_256(mx, red);
  if (threadIdx.x == 0) w.chunk_max[(size_t)slot * w.n_score_chunks + blockIdx.x] = mx;
}

// ---- 2. mass histogram + threshold bin + chunk offsets ------------------------------------

// Block-wide exclusive scan of one int per thread (256 threads); returns the block total.
__device__ __forceinline__ int block_excl_scan_256(int v, int& excl, int* warp_tot) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int k = 0; k < kSelThreads / 32; ++k) {
    const int t = warp_tot[k];
    before += (k < warp) ? t : 0;
    all += t;
  }
  __syncthreads();
  excl = before + x - v;
  return all;
}

// Loads the kPerThread consecutive scores of this thread (positions n..n+kPerThread-1), with
// -inf past n1.
__device__ __forceinline__ void load_scores(const float* sc, int n, int n1, float (&v)[kPerThread]) {
  if (n + kPerThread <= n1) {
#pragma unroll
    for (int k = 0; k < kPerThread; k += 4) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>(sc + n + k));
      v[k] = f.x;
      v[k + 1] = f.y;
      v[k + 2] = f.z;
      v[k + 3] = f.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) v[k] = (n + k < n1) ? __ldcg(sc + n + k) : -INFINITY;
  }
}

__global__ void __launch_bounds__(kSelThreads) hist_kernel(const LayerArgs a, const Workspace w) {
  // Per-warp histograms of the 2^-40 fixed-point masses, split into 32-bit low and high words
  // (native shared-memory atomics; the carry of the low word is detected from the returned old
  // value), and one token-count histogram. Integer sums: exact, independent of arrival order.
  constexpr int kWarps = kSelThreads / 32;
  __shared__ uint32_t wlo[kWarps][kBins];
  __shared__ uint32_t whi[kWarps][kBins];
  __shared__ uint32_t cnt[kBins];
  __shared__ float red[kWarps];
  __shared__ int warp_tot[kWarps];
  __shared__ int is_last, bstar_s, carry_s;
  for (int i = threadIdx.x; i < kWarps * kBins; i += kSelThreads) {
    (&wlo[0][0])[i] = 0u;  // before the dependency wait: overlaps the previous kernel
    (&whi[0][0])[i] = 0u;
  }
  cnt[threadIdx.x] = 0u;
  pdl_wait();
  pdl_launch_dependents();

  const int slot = blockIdx.y;
  const int b = slot / a.nret;
  const int N = clamp_seq_len(a, b, w.status, false);
  const int n0 = blockIdx.x * kSelChunk;
  if (n0 >= N) return;
  const int n1 = min(n0 + kSelChunk, N);
  const int warp = threadIdx.x >> 5;

  // s_max over the chunk maxima of the whole context (max is order-independent)
  const int nsc = (N + kScoreChunk - 1) / kScoreChunk;
  float m = -INFINITY;
  for (int i = threadIdx.x; i < nsc; i += kSelThreads)
    m = fmaxf(m, __ldcg(w.chunk_max + (size_t)slot * w.n_score_chunks + i));
  const float s_max = block_max_256(m, red);  // also orders the zero fill before the adds

  const float* sc = w.scores + (size_t)slot * w.ld;
  float sv[kPerThread];
  load_scores(sc, n0 + threadIdx.x * kPerThread, n1, sv);
  uint32_t* lo_h = wlo[warp];
  uint32_t* hi_h = whi[warp];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const float s = sv[k];
    if (s == -INFINITY) continue;
    const int bin = score_bin(s, s_max, a.bin_scale);
    const float wgt = expf(s - s_max);                       // in (0, 1]
    const unsigned long long fx = __float2ull_rn(wgt * 1099511627776.0f);  // * 2^40, exact
    const uint32_t lo = (uint32_t)fx;
    uint32_t hi = (uint32_t)(fx >> 32);
    if (lo) {
      const uint32_t old = atomicAdd(lo_h + bin, lo);
      hi += (old + lo < old) ? 1u : 0u;                      // carry out of the low word
    }
    if (hi) atomicAdd(hi_h + bin, hi);
    atomicAdd(cnt + bin, 1u);
  }
  __syncthreads();
  {
    unsigned long long v = 0ull;
#pragma unroll
    for (int k = 0; k < kWarps; ++k)
      v += ((unsigned long long)whi[k][threadIdx.x] << 32) + wlo[k][threadIdx.x];
    if (v) atomicAdd(w.hist + (size_t)slot * kBins + threadIdx.x, v);
    w.chunk_bins[((size_t)slot * w.n_sel_chunks + blockIdx.x) * kBins + threadIdx.x] =
        cnt[threadIdx.x];
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned nhc = (unsigned)((N + kSelChunk - 1) / kSelChunk);
    is_last = (atomicAdd(w.ticket_hist + slot, 1u) == nhc - 1u);
    carry_s = 0;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();

  // ---- last CTA of this slot: b* by one warp (8 bins per lane, suffix sums from the top) ----
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    unsigned long long v[8], lane_sum = 0ull;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[i] = __ldcg(w.hist + (size_t)slot * kBins + lane * 8 + i);
      lane_sum += v[i];
    }
    unsigned long long incl = lane_sum;  // sum over lanes >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    const unsigned long long total = __shfl_sync(0xffffffffu, incl, 0);
    const double target = (double)a.top_p * (double)total;
    unsigned long long c = incl - lane_sum;  // mass of the bins above this lane's
    int best = -1;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      c += v[i];
      if (best < 0 && (double)c >= target) best = lane * 8 + i;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    if (lane == 0) {
      bstar_s = best < 0 ? 0 : best;
      w.mass_total[slot] = total;
    }
  }
  __syncthreads();
  const int bs = bstar_s;

  // ---- selected tokens per chunk (bins >= b*) and their exclusive prefix ----
  const int nch = (N + kSelChunk - 1) / kSelChunk;
  int* off = w.chunk_off + (size_t)slot * (w.n_sel_chunks + 1);
  for (int base = 0; base < nch; base += kSelThreads) {
    const int cc = base + threadIdx.x;
    int v = 0;
    if (cc < nch) {
      const uint32_t* row = w.chunk_bins + ((size_t)slot * w.n_sel_chunks + cc) * kBins;
      int bb = bs;
      for (; bb < kBins && (bb & 3); ++bb) v += (int)__ldcg(row + bb);
      for (; bb < kBins; bb += 4) {
        const uint4 q = __ldcg(reinterpret_cast<const uint4*>(row + bb));
        v += (int)(q.x + q.y + q.z + q.w);
      }
    }
    int excl;
    const int all = block_excl_scan_256(v, excl, warp_tot);
    const int carry = carry_s;
    if (cc < nch) off[cc] = carry + excl;
    __syncthreads();
    if (threadIdx.x == 0) carry_s = carry + all;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int total = carry_s;
    off[nch] = total;
    w.bstar[slot] = bs;
    w.s_max[slot] = s_max;
    w.sel_total[slot] = total;
    w.sel_n[slot] = N;
    w.ticket_hist[slot] = 0u;
  }
}

// ---- 3. compaction: the selected positions, ascending, into one dense list -----------------

__global__ void __launch_bounds__(kSelThreads) compact_kernel(const LayerArgs a,
                                                              const Workspace w) {
  __shared__ int warp_tot[kSelThreads / 32];
  pdl_wait();
  pdl_launch_dependents();

  const int slot = blockIdx.y;
  const int b = slot / a.nret;
  const int N = clamp_seq_len(a, b, w.status, false);
  const int n0 = blockIdx.x * kSelChunk;
  if (n0 >= N) return;
  const int n1 = min(n0 + kSelChunk, N);
  const int bstar = __ldcg(w.bstar + slot);
  const float s_max = __ldcg(w.s_max + slot);
  const int base = __ldcg(w.chunk_off + (size_t)slot * (w.n_sel_chunks + 1) + blockIdx.x);
  const float* sc = w.scores + (size_t)slot * w.ld;
  int* out = w.sel_idx + (size_t)slot * w.ld;

  const int n = n0 + threadIdx.x * kPerThread;  // this thread's kPerThread consecutive tokens
  float sv[kPerThread];
  load_scores(sc, n, n1, sv);
  unsigned flags = 0u;
#pragma unroll
  for (int k = 0; k < kPerThread; ++k)
    if (sv[k] != -INFINITY && score_bin(sv[k], s_max, a.bin_scale) >= bstar) flags |= 1u << k;
  int excl;
  block_excl_scan_256(__popc(flags), excl, warp_tot);
  int at = base + excl;
#pragma unroll
  for (int k = 0; k < kPerThread; ++k)
    if (flags & (1u << k)) out[at++] = n + k;
}

}  // namespace rtp
