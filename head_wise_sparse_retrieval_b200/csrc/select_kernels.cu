// select_kernels.cu -- the sort-free top-p selection of the retrieval heads (sm_100a).
//
// Follows "Full Attention Strikes Back ..." (xllm-io paper review), section 三:
//   核心公式 / 自适应稀疏注意力  s_h(m,n) = (W^Q q^pre)^T (W^K k^pre),  S_h(m) = Top-P(s_h, p)
//   硬件感知解码内核            top-p without sorting, over a 256-bin histogram (O(1) per head),
//                              scoring and selection in one launch
// and the gist.science technical summary, Methodology 3 (mass accumulated until p is reached).
//
// One persistent cooperative launch per layer selects the tokens of every retrieval slot
// (slot = b * nret + j for the j-th retrieval KV head). The indexer keys of all slots are laid
// end to end and cut into one equal range per CTA; a CTA keeps the scores of its range in its
// own shared memory (ranges longer than kScoreCap spill the rest to global buffers; the host
// launches the variant without spill code when no range can be that long). Three phases, two
// grid barriers (bounded waits):
//   1. scores: a lane pair reads a token's 32 bytes with two 16-byte loads (double-buffered),
//      the scaled fp32 score is kept, and each CTA records the max of each slot it scores;
//   2. histogram: s_max of a slot = the atomic max of its CTAs' maxima (order-preserving
//      integer keys, cleared after the second barrier); every score is binned relative
//      to s_max and exp(s - s_max) is added in 2^-40 fixed point to per-warp shared bins
//      (32-bit words, exact integer sums whatever the order). The CTA adds its masses to one
//      of kHistCopies copies of the slot's global histogram (integer atomics, spread over the
//      copies) and stores, per bin b, how many of its tokens fall in bins >= b;
//   3. compaction: each CTA sums the copies, finds b* with a CTA-wide suffix scan over the
//      bins, reads the counts at b* of the CTAs before it (one coalesced load) for its offset,
//      and writes its selected positions, ascending, into one dense list per slot.
// Phases 2 and 3 bin the same fp32 scores with score_bin, so counts and flags agree exactly.
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kWarpsSel = kSelThreads / 32;
static_assert(kSelThreads == kBins, "phase 3 gives one bin to each thread");

__device__ __forceinline__ int clamp_seq_len(const LayerArgs& a, int b, unsigned* status,
                                             bool report) {
  int n = __ldcg(a.seq_lens + b);
  if (n < 1 || n > a.max_ctx) {
    if (report) atomicOr(status, kDevBadSeqlen);
    n = n < 1 ? 1 : a.max_ctx;
  }
  return n;
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kWarpsSel; ++i) r = fmaxf(r, red[i]);
  return r;
}

__device__ __forceinline__ int block_sum(int v, int* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int r = 0;
#pragma unroll
  for (int i = 0; i < kWarpsSel; ++i) r += red[i];
  return r;
}

// Block-wide exclusive scan of one int per thread; returns the block total.
__device__ __forceinline__ int block_excl_scan(int v, int& excl, int* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) red[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int k = 0; k < kWarpsSel; ++k) {
    const int t = red[k];
    before += (k < warp) ? t : 0;
    all += t;
  }
  excl = before + x - v;
  return all;
}

// Inclusive suffix sum over the CTA's threads (thread i gets the sum of threads >= i).
template <typename T>
__device__ __forceinline__ T block_suffix_sum(T v, T* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  T x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  __syncthreads();
  if (lane == 0) red[warp] = x;
  __syncthreads();
  T after = 0;
#pragma unroll
  for (int k = 0; k < kWarpsSel; ++k) after += (k > warp) ? red[k] : (T)0;
  return x + after;
}

// Slot sizes (clamped sequence lengths) and their prefix sums into soff[0 .. S]. report: flag
// out-of-range lengths in the status word.
__device__ void slot_offsets(const LayerArgs& a, int S, long long* soff, unsigned* status,
                             bool report) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int s = tid; s < S; s += kSelThreads)
    soff[s + 1] = clamp_seq_len(a, s / a.nret, status, report && (s % a.nret) == 0);
  __syncthreads();
  if (warp == 0) {  // inclusive scan, 32 slots at a time
    long long carry = 0;
    for (int base = 0; base < S; base += 32) {
      const int i = base + lane;
      long long x = (i < S) ? soff[i + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (i < S) soff[i + 1] = carry + x;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) soff[0] = 0;
  }
  __syncthreads();
}

// Largest s < S with off[s] <= x (off ascending, off[0] = 0 <= x < off[S]).
__device__ __forceinline__ int upper_slot(const long long* off, int S, long long x) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The scores (fp32) and bins (one byte) of this CTA's range: the first kScoreCap of each in
// shared memory, the rest (if any) in the global spill buffers at their slot positions. When
// the whole range fits (the usual case) the loops index shared memory directly.
template <bool kFits>
struct Scores {
  float* sm;              // shared, indexed by position in the CTA range
  unsigned char* smb;
  float* glob;            // global spill buffers
  unsigned char* globb;
  size_t ld;
  long long t0;           // range start (concatenated coordinates)
  const long long* soff;
  __device__ float* at(int s, int n) const {
    const long long i = soff[s] + n - t0;
    if (kFits) return sm + i;
    return (i < kScoreCap) ? sm + i : glob + (size_t)s * ld + n;
  }
  __device__ unsigned char* bin_at(int s, int n) const {
    const long long i = soff[s] + n - t0;
    if (kFits) return smb + i;
    return (i < kScoreCap) ? smb + i : globb + (size_t)s * ld + n;
  }
};

}  // namespace

size_t select_smem_bytes(int slots) {
  return (size_t)kScoreCap * 5 + (size_t)(slots + 1) * 8;
}

template <bool kFits>
__device__ __forceinline__ void select_body(const LayerArgs& a, const Workspace& w,
                                            const SelectArgs& x) {
  extern __shared__ __align__(16) unsigned char dsm[];
  __shared__ uint32_t wlo[kWarpsSel][kBins];   // per-warp fixed-point masses, bits 0..19
  __shared__ uint32_t whi[kWarpsSel][kBins];   // bits 20..40
  __shared__ uint32_t cnt[kBins];              // tokens per bin in the segment
  __shared__ float redf[kWarpsSel];
  __shared__ int redi[kWarpsSel];
  __shared__ int aborted;
  __shared__ int bstar_s;

  __shared__ unsigned long long red64[kWarpsSel];
  __shared__ unsigned long long bin0_mass;     // bin 0's fixed-point mass in the chunk

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.B * a.nret;
  float* s_scores = reinterpret_cast<float*>(dsm);
  unsigned char* s_bins = dsm + (size_t)kScoreCap * 4;
  long long* soff = reinterpret_cast<long long*>(dsm + (size_t)kScoreCap * 5);
  if (tid == 0) aborted = 0;

  // Nothing this kernel writes is read by the launch before it (the previous layer's merge),
  // and the selection lists it overwrites were consumed before that merge began. So when the
  // caller vouches that the inputs are ready (a.early), the wait moves to the kernel's end:
  // it still finishes only after its predecessor, which the next launch relies on.
  if (!a.early) pdl_wait();
  pdl_launch_dependents();

  slot_offsets(a, S, soff, w.status, blockIdx.x == 0);
  if (blockIdx.x == 0) {  // phase 2 accumulates into these
    for (int i = tid; i < kHistCopies * S * kBins; i += kSelThreads) w.hist[i] = 0ull;
    if (x.top_k > 0)
      for (int i = tid; i < kHistCopies * S * kBins; i += kSelThreads) x.hist_cnt[i] = 0u;
  }

  const long long T = soff[S];
  const long long P = min((long long)gridDim.x, T);
  const bool active = (long long)blockIdx.x < P;
  const long long t0 = active ? floor_div((long long)blockIdx.x * T, P) : 0;
  const long long t1 = active ? floor_div(((long long)blockIdx.x + 1) * T, P) : 0;
  const Scores<kFits> sc{s_scores, s_bins, w.scores, w.bins, (size_t)w.ld, t0, soff};

  // ---- phase 1: indexer scores of this CTA's range -----------------------------------------
  // One thread per token: the 16 fp16 dims of the key arrive as two 16-byte loads, the score
  // is (dot8(dims 0-7) + dot8(dims 8-15)) * scale with the products summed pairwise in fp32.
  if (active) {
    int s = upper_slot(soff, S, t0);
    for (long long t = t0; t < t1; ++s) {
      const int n0 = (int)(t - soff[s]);
      const int n1 = (int)(min(t1, soff[s + 1]) - soff[s]);
      t = soff[s] + n1;
      const int b = s / a.nret, kvh = a.ret_kvh[s % a.nret];
      const size_t head = (size_t)b * a.Hkv + kvh;
      const uint4 qlo = *reinterpret_cast<const uint4*>(a.q_idx + head * kIdxDim);
      const uint4 qhi = *reinterpret_cast<const uint4*>(a.q_idx + head * kIdxDim + 8);
      const uint4* keys =
          reinterpret_cast<const uint4*>(a.k_idx + head * (size_t)a.max_ctx * kIdxDim);
      float* srow = sc.at(s, 0);  // kFits: the slot's scores in this CTA's shared memory
      constexpr int kUnroll = kScoreUnroll / 2;  // tokens per thread per batch (two loads each)
      float mx = -INFINITY;
      uint4 kv[2 * kUnroll], nx[2 * kUnroll];
      auto load_batch = [&](uint4 (&dst)[2 * kUnroll], int base) {
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int n = base + u * kSelThreads + tid;
          const bool in = n < n1;
          dst[2 * u] = in ? __ldcs(keys + 2 * (size_t)n) : make_uint4(0, 0, 0, 0);
          dst[2 * u + 1] = in ? __ldcs(keys + 2 * (size_t)n + 1) : make_uint4(0, 0, 0, 0);
        }
      };
      load_batch(kv, n0);
      for (int base = n0; base < n1; base += kSelThreads * kUnroll) {
        if (base + kSelThreads * kUnroll < n1) load_batch(nx, base + kSelThreads * kUnroll);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int n = base + u * kSelThreads + tid;
          const float sv = __fmul_rn(__fadd_rn(dot8_f16(qlo, kv[2 * u]), dot8_f16(qhi, kv[2 * u + 1])),
                                     a.idx_scale);
          if (n < n1) {
            if (kFits) srow[n] = sv;
            else *sc.at(s, n) = sv;
            mx = fmaxf(mx, sv);
          }
        }
#pragma unroll
        for (int u = 0; u < 2 * kUnroll; ++u) kv[u] = nx[u];
      }
      mx = block_max(mx, redf);
      if (tid == 0) atomicMax(w.smax_key + s, float_key(mx));
    }
  }
  grid_barrier(w.grid_bar, w.status, &aborted, x.wait_ns, x.withhold_cta);

  // ---- phase 2: mass histogram and token counts of this CTA's segments ---------------------
  if (active) {
    int s = upper_slot(soff, S, t0);
    for (long long t = t0; t < t1; ++s) {
      const int n0 = (int)(t - soff[s]);
      const int n1 = (int)(min(t1, soff[s + 1]) - soff[s]);
      t = soff[s] + n1;
      const long long c0 = cta_of(soff[s], T, P);
      // s_max of the slot: the atomic max over the CTAs that scored it
      const float s_max = key_float(__ldcg(w.smax_key + s));
      for (int i = tid; i < kWarpsSel * kBins; i += kSelThreads) {
        (&wlo[0][0])[i] = 0u;
        (&whi[0][0])[i] = 0u;
      }
      cnt[tid] = 0u;
      __syncthreads();  // the zero fill comes before the adds
      const int copy = (int)(blockIdx.x % kHistCopies);
      // bits 0..19 and 20..40 of the 2^-40 weights go to separate 32-bit words, so that no add
      // needs the old value: a warp adds at most kScoreCap / 8 tokens to a bin before the flush
      for (int k0 = n0; k0 < n1; k0 += kScoreCap) {
        const int k1 = min(n1, k0 + kScoreCap);
        if (k0 != n0) {
          for (int i = tid; i < kWarpsSel * kBins; i += kSelThreads) {
            (&wlo[0][0])[i] = 0u;
            (&whi[0][0])[i] = 0u;
          }
        }
        if (tid == 0) bin0_mass = 0ull;
        __syncthreads();
        // Bin 0 takes every score below the range: for a query with a few dominant tokens that
        // is most of the slot, and shared atomics on that one bin would serialise the warp.
        // Its tokens are summed in registers instead, then once per warp.
        unsigned long long m0 = 0ull;
        unsigned n0cnt = 0u;
        // on chip, the slot's rows are plain offsets into shared memory (computed once here:
        // the bin stores below would otherwise make the compiler reload the slot offsets)
        const float* srow = sc.at(s, 0);
        unsigned char* brow = sc.bin_at(s, 0);
#pragma unroll 4
        for (int n = k0 + tid; n < k1; n += kSelThreads) {
          const float v = kFits ? srow[n] : *sc.at(s, n);
          const int bin = score_bin(v, s_max, a.bin_scale);
          if (kFits) brow[n] = (unsigned char)bin;
          else *sc.bin_at(s, n) = (unsigned char)bin;
          const float wgt = expf(v - s_max);                          // in (0, 1]
          const unsigned long long fx = __float2ull_rn(wgt * 1099511627776.0f);  // * 2^40, exact
          if (bin == 0) {
            m0 += fx;
            ++n0cnt;
          } else {
            atomicAdd(&wlo[warp][bin], (uint32_t)fx & 0xFFFFFu);
            atomicAdd(&whi[warp][bin], (uint32_t)(fx >> 20));
            atomicAdd(&cnt[bin], 1u);
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          m0 += __shfl_xor_sync(0xffffffffu, m0, o);
          n0cnt += __shfl_xor_sync(0xffffffffu, n0cnt, o);
        }
        if (lane == 0 && n0cnt) {
          atomicAdd(&bin0_mass, m0);
          atomicAdd(&cnt[0], n0cnt);
        }
        __syncthreads();
        unsigned long long v = (tid == 0) ? bin0_mass : 0ull;
#pragma unroll
        for (int k = 0; k < kWarpsSel; ++k)
          v += ((unsigned long long)whi[k][tid] << 20) + wlo[k][tid];
        if (v) atomicAdd(w.hist + ((size_t)copy * S + s) * kBins + tid, v);
        __syncthreads();  // the per-warp words are read before the next chunk clears them
      }
      if (x.top_k > 0 && cnt[tid])  // fixed top-k: the slot's token count per bin
        atomicAdd(x.hist_cnt + ((size_t)copy * S + s) * kBins + tid, cnt[tid]);
      // tokens of this CTA in bins >= tid, stored bin-major so that phase 3 reads one column
      const unsigned ge = block_suffix_sum<unsigned>(cnt[tid], reinterpret_cast<unsigned*>(redi));
      w.cta_ge[((size_t)s * kBins + tid) * gridDim.x + blockIdx.x] = ge;
      if (blockIdx.x == c0 && tid == 0) w.s_max[s] = s_max;
      __syncthreads();
    }
  }
  grid_barrier(w.grid_bar, w.status, &aborted, x.wait_ns, -1);
  if (blockIdx.x == 0 && !aborted)  // every CTA read the maxima before this barrier
    for (int s = tid; s < S; s += kSelThreads) w.smax_key[s] = 0u;

  // ---- phase 3: b*, offsets and the dense selected list -----------------------------------
  if (active) {
    int s = upper_slot(soff, S, t0);
    for (long long t = t0; t < t1; ++s) {
      const int n0 = (int)(t - soff[s]);
      const int n1 = (int)(min(t1, soff[s + 1]) - soff[s]);
      t = soff[s] + n1;
      const int c0 = (int)cta_of(soff[s], T, P), c1 = (int)cta_of(soff[s + 1] - 1, T, P);
      const bool first = (int)blockIdx.x == c0;
      // b*: thread tid owns bin tid; the copies are summed, then a suffix scan from the top
      // bin gives each bin's mass at or above it
      unsigned long long hv = 0ull;
#pragma unroll
      for (int k = 0; k < kHistCopies; ++k)
        hv += __ldcg(w.hist + ((size_t)k * S + s) * kBins + tid);
      const unsigned long long sfx = block_suffix_sum<unsigned long long>(hv, red64);
      __syncthreads();
      if (tid == 0) red64[0] = sfx;  // the total C_0
      if (tid == 0) bstar_s = 0;
      __syncthreads();
      const unsigned long long total = red64[0];
      const double target = (double)a.top_p * (double)total;
      const unsigned long long above = sfx - hv;  // mass of the bins above tid
      if (x.top_k > 0) {
        // fixed top-k: the highest bin whose suffix count reaches k (none: every token)
        unsigned hc = 0u;
#pragma unroll
        for (int k = 0; k < kHistCopies; ++k) hc += __ldcg(x.hist_cnt + ((size_t)k * S + s) * kBins + tid);
        const unsigned cs = block_suffix_sum<unsigned>(hc, reinterpret_cast<unsigned*>(redi));
        const unsigned kk = (unsigned)x.top_k;
        if (cs >= kk && (tid == kBins - 1 || cs - hc < kk)) bstar_s = tid;
      } else if ((double)sfx >= target && (tid == kBins - 1 || !((double)above >= target))) {
        bstar_s = tid;  // the highest bin whose suffix mass reaches p * C_0 (one thread)
      }
      __syncthreads();
      const int bs = bstar_s;
      if (first && tid == 0) w.mass_total[s] = total;
      // selected tokens of the slot's CTAs before this one (first CTA: of all, for |S|)
      const int r0 = c0, r1 = first ? c1 + 1 : (int)blockIdx.x;
      const unsigned* col = w.cta_ge + ((size_t)s * kBins + bs) * gridDim.x;
      int mine = 0;
      for (int c = r0 + tid; c < r1; c += kSelThreads) mine += (int)__ldcg(col + c);
      const int sum_rows = block_sum(mine, redi);
      int base = first ? 0 : sum_rows;
      if (first && tid == 0) {
        w.bstar[s] = bs;
        w.sel_total[s] = sum_rows;
        w.sel_n[s] = (int)(soff[s + 1] - soff[s]);
      }
      int* out = w.sel_idx + (size_t)s * w.ld;
      const unsigned char* brow = sc.bin_at(s, 0);  // on chip: the slot's bins in shared memory
      // ordered compaction: warp w takes 32 x kPerThread consecutive tokens of each round, one
      // ballot per 32; the warps' counts are scanned, then each warp writes its tokens in order
      constexpr int kWarpSpan = 32 * kPerThread;
      for (int rb = n0; rb < n1; rb += kWarpsSel * kWarpSpan) {
        const int wb = rb + warp * kWarpSpan;
        unsigned bal[kPerThread];
        int wcnt = 0;
#pragma unroll
        for (int k = 0; k < kPerThread; ++k) {
          const int n = wb + 32 * k + lane;
          const int nc = min(n, n1 - 1);  // in range: no branch around the load
          const int bin = kFits ? brow[nc] : *sc.bin_at(s, nc);
          const bool f = n < n1 && bin >= bs;
          bal[k] = __ballot_sync(0xffffffffu, f);
          wcnt += __popc(bal[k]);
        }
        int wexcl;
        const int all = block_excl_scan(lane == 0 ? wcnt : 0, wexcl, redi);
        int at = base + __shfl_sync(0xffffffffu, wexcl, 0);
        const unsigned lt = (1u << lane) - 1u;
#pragma unroll
        for (int k = 0; k < kPerThread; ++k) {
          // in range by construction; after an abandoned barrier the offsets may be stale, so
          // the row's capacity is still checked
          const int dst = at + __popc(bal[k] & lt);
          if (bal[k] & (1u << lane)) {
            if ((unsigned)dst < (unsigned)w.ld) out[dst] = wb + 32 * k + lane;
            else atomicOr(w.status, kDevBadIndex);
          }
          at += __popc(bal[k]);
        }
        base += all;
      }
      __syncthreads();
    }
  }
  if (a.early) pdl_wait();
}

__global__ void __launch_bounds__(kSelThreads, 2) select_kernel_onchip(const LayerArgs a,
                                                                       const Workspace w,
                                                                       const SelectArgs x) {
  select_body<true>(a, w, x);
}

__global__ void __launch_bounds__(kSelThreads, 2) select_kernel_spill(const LayerArgs a,
                                                                      const Workspace w,
                                                                      const SelectArgs x) {
  select_body<false>(a, w, x);
}

}  // namespace rtp
