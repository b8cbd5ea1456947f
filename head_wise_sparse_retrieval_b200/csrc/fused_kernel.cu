// fused_kernel.cu -- one decode layer (retrieval and local heads) in one launch (sm_100a).
//
// Follows "Full Attention Strikes Back ..." (xllm-io paper review), section 三:
//   核心公式 / 自适应稀疏注意力   s_h(m,n) = (W^Q q^pre)^T (W^K k^pre), S_h(m) = Top-P(s_h, p),
//                                O_h(m) = exact softmax attention over S_h(m);
//   硬件感知解码内核             top-p without sorting over a 256-bin histogram, scoring and
//                                selection fused into one launch;
// and the gist.science technical summary, Methodology 1 (local heads: 4 sinks and the last
// 8192 positions) and 3 (mass accumulated until p is reached).
//
// It computes what select_kernel + attend_kernel + merge_kernel compute, bin for bin and token
// for token, in one cooperative launch of one CTA per SM, without a list of selected positions:
//   ownership  the tokens of every retrieval slot (slot = b * nret + j) are cut into 64-token
//              tiles; the tiles of all slots, laid end to end, are dealt round-robin (tile g to
//              CTA g mod P). Every CTA thus holds about 1/P of every slot, so the scoring work
//              and the gather work left by the selection are balanced whatever the slots'
//              selection densities are;
//   phase 1    each warp streams its tiles' indexer keys through a 4-stage cp.async ring and
//              keeps the fp32 scores in shared memory; the CTA's maximum of each slot goes into
//              a global atomic max over order-preserving integer keys;
//   phase 2    (grid barrier) bins and 2^-40 fixed-point masses, as in select_kernel, into the
//              slot's global histogram copies, with the token count of every bin;
//   phase 3    (grid barrier) one thread per bin sums the copies, CTA-wide suffix scans of
//              mass and count give b* and |S|; each CTA turns its bins into one 64-bit selection
//              mask per tile and an exclusive prefix of the masks' popcounts;
//   phase 4    the CTA's selected tokens of a slot are split evenly over its warps; a warp reads
//              its positions straight from the masks (a cursor over its tiles) and gathers the K/V
//              rows with 16-byte cp.async into a 3-stage ring; the local heads' window sets are cut
//              into P contiguous ranges as in attend_kernel. The math is attend_kernel's (warp MMA
//              with the GQA group as N = 8, online softmax in the log2 domain, fixed-order merge
//              of the warps). A (head, CTA) piece goes to a partial, or to the output when one
//              CTA holds the whole head;
//   phase 5    (grid barrier) the CTAs merge the split heads by log-sum-exp, one (head, query
//              head, 32 dimensions) unit at a time, every sum in a fixed order.
// All waits are bounded (kDevWaitTimeout); after a timed-out barrier the CTA stops.
#include "attend_tile.cuh"
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kW = kFusedWarps;
constexpr int kT = kFusedThreads;
constexpr int kDepth = 3;                                  // gather stages per warp
constexpr int kOwn = kFusedOwnTok;
constexpr int kRing = 4;                                   // indexer-key stages per warp
constexpr int kRegion = kW * kDepth * kWarpStage;          // 192 KB, reused by every phase
constexpr int kKeyStage = kOwn * kIdxDim * 2;              // one tile of indexer keys (2 KB)
constexpr int kRingBytes = kW * kRing * kKeyStage;         // phase 1: [0, 64 KB)
constexpr int kCapTokens = kFusedCapTiles * kOwn;
constexpr int kScoresOff = kRingBytes;                     // phase 1-2: fp32 scores
constexpr int kWHistOff = kCapTokens;                      // phase 2: per-warp mass words,
constexpr int kWHistBytes = 2 * kW * kBins * 4;            // after the bins, inside the ring
constexpr int kOPitch = kHeadDim + 4;
constexpr int kCombFloats = kMaxGroup * kOPitch + kW * kMaxGroup * 2 + kMaxGroup * 2;
constexpr int kBitsOff = kRegion;                          // u64 mask per own tile
constexpr int kPreOff = kBitsOff + kFusedCapTiles * 8;     // int prefix [kFusedCapTiles + 1]
constexpr int kCombOff = kPreOff + ((kFusedCapTiles + 1) * 4 + 15) / 16 * 16;
constexpr int kSmemBytes = kCombOff + kCombFloats * 4;
constexpr int kMergeRows = kT / 8;                         // pieces one merge pass loads
constexpr int kMergeRegs = 5;                              // passes kept in registers (160)
constexpr int kMaxH = kFusedMaxHeads;

static_assert(kScoresOff + 4 * kCapTokens <= kRegion, "the scores fit the region");
static_assert(kWHistOff + kWHistBytes <= kRingBytes, "bins and words overlay the key ring");
static_assert(kCapTokens / kW <= 4096, "a warp adds at most 4096 20-bit halves to a word");
static_assert(kFusedCapTiles <= 2 * kT, "the popcount prefix takes two tiles per thread");
static_assert(kT == kBins, "phase 2 flushes one bin per thread");
static_assert(2 * 1024 * 4 + 256 + kW * 8 * 16 <= kRegion, "merge arrays fit the region");


// Position of the k-th (0-based) set bit of x, k < popc(x): halving the window by popcounts.
__device__ __forceinline__ int nth_set32(unsigned x, int k) {
  int pos = 0;
#pragma unroll
  for (int sh = 16; sh > 0; sh >>= 1) {
    const int c = __popc(x & ((1u << sh) - 1u));
    if (k >= c) {
      k -= c;
      x >>= sh;
      pos += sh;
    }
  }
  return pos;
}
__device__ __forceinline__ int nth_set64(unsigned long long m, int k) {
  const unsigned lo = (unsigned)m;
  const int cl = __popc(lo);
  return k < cl ? nth_set32(lo, k) : 32 + nth_set32((unsigned)(m >> 32), k - cl);
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
  for (int k = 0; k < kW; ++k) after += (k > warp) ? red[k] : (T)0;
  return x + after;
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
  for (int k = 0; k < kW; ++k) {
    const int t = red[k];
    before += (k < warp) ? t : 0;
    all += t;
  }
  excl = before + x - v;
  return all;
}

// A head's rows and token set.
struct HeadRef {
  const __nv_bfloat16* kbase;
  const __nv_bfloat16* vbase;
  int N;
};

// Gathers the tile's K and V rows into the stage (attend_tile.cuh).
__device__ __forceinline__ void issue_tile(uint32_t stage, const HeadRef& h, int pos, int n,
                                           int lane, uint64_t policy, unsigned* status) {
  gather_tile(stage, h.kbase, h.vbase, h.N, pos, n, lane, policy, status);
}

// Per-CTA tables, built in the prologue.
struct Tables {
  int N[kMaxH];          // retrieval slot: clamped sequence length
  int G[kMaxH + 1];      // first global ownership tile of the slot (prefix of ceil(N / 64))
  int O[kMaxH + 1];      // first own tile of the slot in this CTA's order (clamped to the cap)
  int first[kMaxH];      // the slot's first tile owned by this CTA (>= G[s] + tiles: none)
  int pidx[kMaxH];       // this CTA's piece of the slot, counted from pb[s]
  int pb[kMaxH + 1];     // first piece of the slot (prefix of min(P, tiles)); pb[S]: local pieces
  unsigned key[kMaxH];   // this CTA's max score of the slot, as a key
  float smax[kMaxH];
  int bstar[kMaxH];
  int sel[kMaxH];        // |S| of the slot
  long long loff[kMaxH + 1];  // local heads: prefix of the window-set sizes
  int lhd[kMaxH];        // head of local ordinal
  int lord[kMaxH];       // local ordinal of head (or -1)
  int seq[kMaxH];        // clamped N of sequence b
  int nloc;
};

// The units of this CTA's work, in order: the retrieval slots it owns tiles of, then the
// segments of its range of the local heads' concatenated window sets. ra, rb: this warp's part
// (CTA selection ranks of the slot, or window ranks of the head).
struct Unit {
  int kind;  // 0 retrieval, 1 local
  int idx;   // slot, or local ordinal
  int hd;    // b * Hkv + kvh
  int ra, rb;
  int r0, r1;  // local: the CTA's segment of the head
};

struct UnitWalk {
  int s;            // next retrieval slot to consider
  long long t, t1;  // local range still to walk
  int lh;           // local ordinal holding t
  __device__ void begin(const Tables& tb, long long t0, long long tend) {
    s = 0;
    t = t0;
    t1 = tend;
    int lo = 0, hi = tb.nloc - 1;  // local head with loff[lh] <= t0 < loff[lh + 1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tb.loff[mid] <= t0) lo = mid; else hi = mid - 1;
    }
    lh = lo;
  }
  __device__ bool next(const Tables& tb, const LayerArgs& a, const int* pre, int S, int warp,
                       Unit& u) {
    while (s < S) {
      const int sl = s++;
      if (tb.O[sl + 1] > tb.O[sl]) {
        const int base = pre[tb.O[sl]], cnt = pre[tb.O[sl + 1]] - base;
        u.kind = 0;
        u.idx = sl;
        u.hd = (sl / a.nret) * a.Hkv + a.ret_kvh[sl % a.nret];
        u.ra = base + (int)(((long long)cnt * warp) / kW);
        u.rb = base + (int)(((long long)cnt * (warp + 1)) / kW);
        u.r0 = u.r1 = 0;
        return true;
      }
    }
    while (t < t1 && lh < tb.nloc) {
      const long long hend = min(t1, tb.loff[lh + 1]);
      if (hend > t) {
        const int len = (int)(hend - t);
        u.kind = 1;
        u.idx = lh;
        u.hd = tb.lhd[lh];
        u.r0 = (int)(t - tb.loff[lh]);
        u.r1 = (int)(hend - tb.loff[lh]);
        u.ra = u.r0 + (int)(((long long)len * warp) / kW);
        u.rb = u.r0 + (int)(((long long)len * (warp + 1)) / kW);
        t = hend;
        ++lh;
        return true;
      }
      ++lh;
    }
    return false;
  }
};

}  // namespace

size_t fused_smem_bytes() { return (size_t)kSmemBytes; }

__global__ void __launch_bounds__(kT, 1) fused_layer_kernel(const LayerArgs a, const Workspace w,
                                                            const FusedArgs f) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ Tables tb;
  __shared__ uint32_t sCnt[kBins];
  __shared__ int sRed[kW];
  __shared__ unsigned long long sRed64[kW];
  __shared__ unsigned sRedU[kW];
  __shared__ int sB;
  __shared__ unsigned long long sTot;
  __shared__ int aborted;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = (int)gridDim.x, cta = (int)blockIdx.x;
  const int S = a.B * a.nret, nheads = a.B * a.Hkv;
  float* scores = reinterpret_cast<float*>(smem + kScoresOff);
  unsigned char* bins = smem;
  unsigned long long* bits = reinterpret_cast<unsigned long long*>(smem + kBitsOff);
  int* pre = reinterpret_cast<int*>(smem + kPreOff);
  float* sComb = reinterpret_cast<float*>(smem + kCombOff);
  const uint64_t policy = l2_policy_evict_first();

  if (tid == 0) aborted = 0;
  // the workspace is the previous launch's until it has finished
  pdl_wait();
  pdl_launch_dependents();

  // ---- prologue: sequence lengths, slot and local-head tables ------------------------------
  for (int b = tid; b < a.B; b += kT) {
    int n = a.seq_lens[b];
    if (n < 1 || n > a.max_ctx) {
      if (cta == 0) atomicOr(w.status, kDevBadSeqlen);
      n = n < 1 ? 1 : a.max_ctx;
    }
    tb.seq[b] = n;
  }
  for (int s = tid; s < S; s += kT) tb.key[s] = 0u;
  for (int hd = tid; hd < nheads; hd += kT) tb.lord[hd] = -1;
  if (cta == 0)  // phase 2 accumulates into these
    for (int i = tid; i < kHistCopies * S * kBins; i += kT) {
      w.hist[i] = 0ull;
      f.hist_cnt[i] = 0u;
    }
  __syncthreads();
  if (warp == 0) {
    int cg = 0, co = 0, cp = 0;
    for (int base = 0; base < S; base += 32) {
      const int s = base + lane;
      const bool v = s < S;
      const int n = v ? tb.seq[s / a.nret] : 0;
      const int tiles = (n + kOwn - 1) / kOwn;
      int xi = tiles;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, xi, o);
        if (lane >= o) xi += y;
      }
      const int g0 = cg + xi - tiles;
      int r = (cta - g0) % P;  // this CTA's first tile of the slot is g0 + r
      if (r < 0) r += P;
      const int first = g0 + r;
      const int own = (v && first < g0 + tiles) ? (g0 + tiles - 1 - first) / P + 1 : 0;
      const int pidx = r;  // the owners of the slot's tiles, from its first tile on
      const int pc = v ? min(P, tiles) : 0;
      int yi = own, zi = pc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y1 = __shfl_up_sync(0xffffffffu, yi, o);
        const int z1 = __shfl_up_sync(0xffffffffu, zi, o);
        if (lane >= o) {
          yi += y1;
          zi += z1;
        }
      }
      if (v) {
        tb.N[s] = n;
        tb.G[s] = g0;
        tb.first[s] = first;
        tb.pidx[s] = pidx;
        tb.O[s] = min(co + yi - own, kFusedCapTiles);
        tb.pb[s] = cp + zi - pc;
      }
      cg += __shfl_sync(0xffffffffu, xi, 31);
      co += __shfl_sync(0xffffffffu, yi, 31);
      cp += __shfl_sync(0xffffffffu, zi, 31);
    }
    if (lane == 0) {
      tb.G[S] = cg;
      tb.O[S] = min(co, kFusedCapTiles);
      tb.pb[S] = cp;
      if (co > kFusedCapTiles) atomicOr(w.status, kDevBadIndex);  // the host rules this out
    }
  } else if (warp == 1) {
    int cnt = 0;
    long long acc = 0;
    for (int base = 0; base < nheads; base += 32) {
      const int hd = base + lane;
      const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
      const bool loc = hd < nheads && a.slot_of_kvh[kvh] < 0;
      const unsigned bal = __ballot_sync(0xffffffffu, loc);
      const int ord = cnt + __popc(bal & ((1u << lane) - 1u));
      long long li = loc ? window_len(tb.seq[b], a.window, a.sinks) : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, li, o);
        if (lane >= o) li += y;
      }
      if (loc) {
        tb.lhd[ord] = hd;
        tb.lord[hd] = ord;
        tb.loff[ord + 1] = acc + li;
      }
      acc += __shfl_sync(0xffffffffu, li, 31);
      cnt += __popc(bal);
    }
    if (lane == 0) {
      tb.loff[0] = 0;
      tb.nloc = cnt;
    }
  }
  __syncthreads();
  const int ownT = tb.O[S];
  // first token of own tile o of slot s, in the slot
  auto tile_n0 = [&](int o, int s) {  // a CTA's consecutive tiles of a slot are P apart
    return (tb.first[s] + P * (o - tb.O[s]) - tb.G[s]) * kOwn;
  };

  // ---- phase 1: indexer scores of the own tiles ---------------------------------------------
  if (S > 0) {
    const uint32_t ring = smem_u32(smem) + warp * kRing * kKeyStage;
    const int nmine = ownT > warp ? (ownT - warp + kW - 1) / kW : 0;
    int s_iss = 0;
    auto issue_keys = [&](int i) {  // the keys of this warp's tile i; one commit group
      const int o = warp + kW * i;
      if (i < nmine) {
        while (tb.O[s_iss + 1] <= o) ++s_iss;
        const int b = s_iss / a.nret, kvh = a.ret_kvh[s_iss % a.nret];
        const __half* keys = a.k_idx + ((size_t)b * a.Hkv + kvh) * a.max_ctx * kIdxDim;
        const int n0 = tile_n0(o, s_iss);
        const int valid = min(kOwn, tb.N[s_iss] - n0);
        const uint32_t dst = ring + (i % kRing) * kKeyStage;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int ch = lane + 32 * j;  // 16-byte chunk: token ch / 2, half ch % 2
          const int tok = ch >> 1;
          const bool in = tok < valid;
          const __half* src = keys + (size_t)(n0 + (in ? tok : 0)) * kIdxDim + (ch & 1) * 8;
          cp_async_16(dst + ch * 16, src, in ? 16u : 0u, policy);
        }
      }
      cp_async_commit();
    };
    for (int i = 0; i < kRing - 1; ++i) issue_keys(i);
    int s_cur = 0, run = -1;
    uint4 qv = make_uint4(0, 0, 0, 0);  // this lane's 8 fp16 dims of the slot's indexer query
    float mx = -INFINITY;
    auto flush_max = [&]() {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) atomicMax(&tb.key[run], float_key(mx));
    };
    for (int i = 0; i < nmine; ++i) {
      issue_keys(i + kRing - 1);
      cp_async_wait<kRing - 1>();
      __syncwarp();
      const int o = warp + kW * i;
      while (tb.O[s_cur + 1] <= o) ++s_cur;
      if (s_cur != run) {
        if (run >= 0) flush_max();
        run = s_cur;
        mx = -INFINITY;
        const int b = run / a.nret, kvh = a.ret_kvh[run % a.nret];
        qv = *reinterpret_cast<const uint4*>(
            a.q_idx + ((size_t)b * a.Hkv + kvh) * kIdxDim + (lane & 1) * 8);
      }
      const int valid = min(kOwn, tb.N[run] - tile_n0(o, run));
      const unsigned char* st = smem + (warp * kRing + i % kRing) * kKeyStage;
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        const int tok = pp * 16 + (lane >> 1);
        const uint4 kv = *reinterpret_cast<const uint4*>(st + (tok * 2 + (lane & 1)) * 16);
        // the selection kernel's arithmetic: this half's 8 exact products summed pairwise in
        // fp32 (mixed-precision FMAs), then the other half's sum added
        const float part = dot8_f16(qv, kv);
        const float other = __shfl_xor_sync(0xffffffffu, part, 1);
        const float sv = __fmul_rn(__fadd_rn(part, other), a.idx_scale);
        if (tok < valid) {
          if ((lane & 1) == 0) scores[o * kOwn + tok] = sv;
          mx = fmaxf(mx, sv);
        }
      }
      __syncwarp();  // the stage is refilled kRing - 1 tiles later
    }
    if (run >= 0) flush_max();
    cp_async_wait<0>();
    __syncthreads();
    for (int s = tid; s < S; s += kT)
      if (tb.O[s + 1] > tb.O[s]) atomicMax(f.smax_key + s, tb.key[s]);
    grid_barrier(f.bar, w.status, &aborted, f.wait_ns, -1);  // S is the same for every CTA
    if (aborted) return;
  }

  // ---- phase 2: bins, masses and counts of the own tokens -----------------------------------
  if (S > 0) {
    for (int s = tid; s < S; s += kT) tb.smax[s] = key_float(__ldcg(f.smax_key + s));
    uint32_t* wlo = reinterpret_cast<uint32_t*>(smem + kWHistOff);
    uint32_t* whi = wlo + kW * kBins;
    const int copy = cta % kHistCopies;
    for (int s = 0; s < S; ++s) {
      const int o0 = tb.O[s], o1 = tb.O[s + 1];
      if (o1 <= o0) continue;  // the same for every thread of the CTA
      for (int i = tid; i < kW * kBins; i += kT) {
        wlo[i] = 0u;
        whi[i] = 0u;
      }
      sCnt[tid] = 0u;
      __syncthreads();  // (and, for the first slot, the s_max table)
      const float smax = tb.smax[s];
      const int ntok = (o1 - o0) * kOwn;
      for (int i = tid; i < ntok; i += kT) {
        const int o = o0 + i / kOwn, tok = i % kOwn;
        if (tile_n0(o, s) + tok < tb.N[s]) {
          const int idx = o * kOwn + tok;
          const float v = scores[idx];
          const int bin = score_bin(v, smax, a.bin_scale);
          bins[idx] = (unsigned char)bin;
          const float wgt = expf(v - smax);  // in (0, 1]
          const unsigned long long fx = __float2ull_rn(wgt * 1099511627776.0f);  // * 2^40, exact
          atomicAdd(&wlo[warp * kBins + bin], (uint32_t)fx & 0xFFFFFu);
          atomicAdd(&whi[warp * kBins + bin], (uint32_t)(fx >> 20));
          atomicAdd(&sCnt[bin], 1u);
        }
      }
      __syncthreads();
      unsigned long long v = 0ull;
#pragma unroll
      for (int k = 0; k < kW; ++k)
        v += ((unsigned long long)whi[k * kBins + tid] << 20) + wlo[k * kBins + tid];
      const size_t hi = ((size_t)copy * S + s) * kBins + tid;
      if (v) atomicAdd(w.hist + hi, v);
      if (sCnt[tid]) atomicAdd(f.hist_cnt + hi, sCnt[tid]);
      __syncthreads();  // the words are read before the next slot clears them
    }
    grid_barrier(f.bar, w.status, &aborted, f.wait_ns, -1);
    if (aborted) return;
  }

  // ---- phase 3: b* of every slot, the CTA's selection masks and their prefix ----------------
  if (S > 0) {
    for (int s = 0; s < S; ++s) {
      // thread tid owns bin tid: the copies summed, then suffix sums from the top bin
      unsigned long long hv = 0ull;
      unsigned hc = 0u;
#pragma unroll
      for (int k = 0; k < kHistCopies; ++k) {
        const size_t hb = ((size_t)k * S + s) * kBins + tid;
        hv += __ldcg(w.hist + hb);
        hc += __ldcg(f.hist_cnt + hb);
      }
      const unsigned long long sfx = block_suffix_sum<unsigned long long>(hv, sRed64);
      const unsigned cfx = block_suffix_sum<unsigned>(hc, sRedU);
      if (tid == 0) {
        sTot = sfx;  // C_0
        sB = 0;      // fixed top-k above the slot's size: every token
      }
      __syncthreads();
      const unsigned long long total = sTot;
      const double target = (double)a.top_p * (double)total;
      // the highest bin whose suffix reaches the target (suffix sums fall with the bin)
      const bool q = (f.top_k > 0) ? (cfx >= (unsigned)f.top_k) : ((double)sfx >= target);
      const bool q_above = tid + 1 < kBins &&
                           ((f.top_k > 0) ? (cfx - hc >= (unsigned)f.top_k)
                                          : ((double)(sfx - hv) >= target));
      if (q && !q_above) {
        sB = tid;
        tb.sel[s] = (int)cfx;
      }
      __syncthreads();
      if (tid == 0) {
        const int bs = sB;
        tb.bstar[s] = bs;
        if (bs == 0) tb.sel[s] = (int)cfx;  // (also when no bin qualified)
        if (cta == 0) {  // what the debug calls read
          w.bstar[s] = bs;
          w.sel_total[s] = tb.sel[s];
          w.sel_n[s] = tb.N[s];
          w.mass_total[s] = total;
          w.s_max[s] = tb.smax[s];
        }
      }
      __syncthreads();
    }
    if (cta == 0)  // every CTA read the maxima before the second barrier
      for (int s = tid; s < S; s += kT) f.smax_key[s] = 0u;
    // selection masks: bit i of tile o is token i of the tile (in range, bin >= b*)
    {
      int s = 0;
      for (int o = warp; o < ownT; o += kW) {
        while (tb.O[s + 1] <= o) ++s;
        const int n0 = tile_n0(o, s);
        const int valid = min(kOwn, tb.N[s] - n0);
        const int bs = tb.bstar[s];
        const unsigned char* bt = bins + o * kOwn;
        const bool f0 = lane < valid && bt[lane] >= bs;
        const bool f1 = lane + 32 < valid && bt[lane + 32] >= bs;
        const unsigned lo = __ballot_sync(0xffffffffu, f0), hi = __ballot_sync(0xffffffffu, f1);
        const unsigned long long m = ((unsigned long long)hi << 32) | lo;
        if (lane == 0) {
          bits[o] = m;
          f.sel_bits[(size_t)s * f.ldw + n0 / kOwn] = m;
        }
      }
    }
    __syncthreads();
    {
      const int o0 = 2 * tid;
      const int c0 = o0 < ownT ? __popcll(bits[o0]) : 0;
      const int c1 = o0 + 1 < ownT ? __popcll(bits[o0 + 1]) : 0;
      int excl;
      const int all = block_excl_scan(c0 + c1, excl, sRed);
      if (o0 < ownT) pre[o0] = excl;
      if (o0 + 1 < ownT) pre[o0 + 1] = excl + c0;
      if (tid == 0) pre[ownT] = all;
    }
  } else if (tid == 0) {
    pre[0] = 0;
  }
  if (cta == 0 && a.sel_count)
    for (int hd = tid; hd < nheads; hd += kT) {
      const int b = hd / a.Hkv, kvh = hd - b * a.Hkv, j = a.slot_of_kvh[kvh];
      a.sel_count[hd] =
          j >= 0 ? tb.sel[b * a.nret + j] : window_len(tb.seq[b], a.window, a.sinks);
    }
  __syncthreads();

  // ---- phase 4: gather and attention, unit by unit ------------------------------------------
  const long long Wt = tb.nloc > 0 ? tb.loff[tb.nloc] : 0;
  const long long Ploc = min((long long)P, Wt);
  const bool has_loc = cta < Ploc;
  const long long lt0 = has_loc ? floor_div((long long)cta * Wt, Ploc) : 0;
  const long long lt1 = has_loc ? floor_div(((long long)cta + 1) * Wt, Ploc) : 0;
  const uint32_t my_stages = smem_u32(smem) + warp * kDepth * kWarpStage;

  auto head_of = [&](const Unit& u) {
    HeadRef h;
    const size_t off = (size_t)u.hd * a.max_ctx * kHeadDim;
    h.kbase = a.k_cache + off;
    h.vbase = a.v_cache + off;
    h.N = u.kind == 0 ? tb.N[u.idx] : tb.seq[u.hd / a.Hkv];
    return h;
  };

  // load side: this warp's tiles across the units, positions from the masks or the window
  UnitWalk lw;
  lw.begin(tb, lt0, lt1);
  Unit lu;
  HeadRef lh{};
  int lrem = 0, co = 0, co_end = 0, cr = 0;
  unsigned long long cm = 0ull;
  auto issue = [&](int i) {  // loads of this warp's next tile into stage i % kDepth; one group
    while (lrem == 0) {
      if (!lw.next(tb, a, pre, S, warp, lu)) break;
      lrem = lu.rb - lu.ra;
      if (lrem == 0) continue;
      lh = head_of(lu);
      if (lu.kind == 0) {  // the own tile holding CTA rank ra, then skip the ranks before it
        int lo = tb.O[lu.idx], hi = tb.O[lu.idx + 1] - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (pre[mid] <= lu.ra) lo = mid; else hi = mid - 1;
        }
        co = lo;
        co_end = tb.O[lu.idx + 1];
        cm = bits[co];
        const int k = lu.ra - pre[co];
        if (k > 0) {
          const int p = nth_set64(cm, k - 1);
          cm &= ~((2ull << p) - 1ull);
        }
      } else {
        cr = lu.ra;
      }
    }
    if (lrem > 0) {
      const int need = min(kTile, lrem);
      int pos = -1;
      if (lu.kind == 0) {
        int filled = 0;
        while (filled < need) {
          while (cm == 0ull && co + 1 < co_end) cm = bits[++co];
          if (cm == 0ull) {  // fewer selected tokens than ranks: cannot happen
            if (lane == 0) atomicOr(w.status, kDevBadIndex);
            break;
          }
          const int cnt = __popcll(cm);
          const int take = min(cnt, need - filled);
          const int j = lane - filled;
          if (j >= 0 && j < take) pos = tile_n0(co, lu.idx) + nth_set64(cm, j);
          if (take == cnt) {
            cm = 0ull;
          } else {
            const int p = nth_set64(cm, take - 1);
            cm &= ~((2ull << p) - 1ull);
          }
          filled += take;
        }
      } else {
        if (lane < need) pos = window_pos(cr + lane, lh.N, a.window, a.sinks);
        cr += need;
      }
      lrem -= need;
      issue_tile(my_stages + (i % kDepth) * kWarpStage, lh, pos, need, lane, policy, w.status);
    }
    cp_async_commit();
  };
  for (int i = 0; i < kDepth - 1; ++i) issue(i);

  // math side: the same units in the same order
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const float scale_log2 = a.attn_scale_log2;
  int done = 0;
  UnitWalk mw;
  mw.begin(tb, lt0, lt1);
  Unit u;
  while (mw.next(tb, a, pre, S, warp, u)) {
    const int b = u.hd / a.Hkv, kvh = u.hd - b * a.Hkv;
    uint32_t qf[8][2];
    load_q_frag(qf, a.q + ((size_t)b * a.Hq + (size_t)kvh * a.G) * kHeadDim, a.G, lane);
    TileAcc st;
    st.init();
    const int len_w = u.rb - u.ra;
    for (int r = 0; r < len_w; r += kTile, ++done) {
      issue(done + kDepth - 1);
      cp_async_wait<kDepth - 1>();
      __syncwarp();
      const int n = min(kTile, len_w - r);
      attend_tile(my_stages + (done % kDepth) * kWarpStage, qf, n, scale_log2, lane, st);
      __syncwarp();  // the stage is refilled kDepth - 1 tiles later
    }

    // ---- end of the unit: merge the warps, write the piece or the output ----
    if (u.kind == 0 && pre[tb.O[u.idx + 1]] == pre[tb.O[u.idx]]) {
      // none of the slot's selected tokens is in this CTA's tiles (the same for every warp):
      // an empty piece, m = -inf and l = 0 (phase 5 gives it the factor 0 and skips its O)
      float* pc = f.partials + (size_t)(tb.pb[u.idx] + tb.pidx[u.idx]) * kPartFloats;
      if (tid < a.G) {
        pc[kPartO + tid] = -INFINITY;
        pc[kPartO + kMaxGroup + tid] = 0.f;
      }
      continue;
    }
    float* sO = sComb;                                   // [8][kOPitch]
    float* sML = sComb + kMaxGroup * kOPitch;            // [kW][8][2]
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      st.l0 += __shfl_xor_sync(0xffffffffu, st.l0, o);
      st.l1 += __shfl_xor_sync(0xffffffffu, st.l1, o);
    }
    if (g == 0) {
      sML[(warp * kMaxGroup + 2 * t) * 2] = st.m0;
      sML[(warp * kMaxGroup + 2 * t) * 2 + 1] = st.l0;
      sML[(warp * kMaxGroup + 2 * t + 1) * 2] = st.m1;
      sML[(warp * kMaxGroup + 2 * t + 1) * 2 + 1] = st.l1;
    }
    __syncthreads();
    {
      float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
      for (int wq = 0; wq < kW; ++wq) {
        M0 = fmaxf(M0, sML[(wq * kMaxGroup + 2 * t) * 2]);
        M1 = fmaxf(M1, sML[(wq * kMaxGroup + 2 * t + 1) * 2]);
      }
      const float f0 = (st.m0 == -INFINITY) ? 0.f : exp2f(st.m0 - M0);  // 0: a warp without tokens
      const float f1 = (st.m1 == -INFINITY) ? 0.f : exp2f(st.m1 - M1);
#pragma unroll
      for (int wq = 0; wq < kW; ++wq) {
        if (warp == wq) {
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            float* r0p = sO + (2 * t) * kOPitch + 16 * mt + g;
            float* r1p = sO + (2 * t + 1) * kOPitch + 16 * mt + g;
            if (wq == 0) {
              r0p[0] = st.acc[mt][0] * f0;
              r1p[0] = st.acc[mt][1] * f1;
              r0p[8] = st.acc[mt][2] * f0;
              r1p[8] = st.acc[mt][3] * f1;
            } else {
              r0p[0] += st.acc[mt][0] * f0;
              r1p[0] += st.acc[mt][1] * f1;
              r0p[8] += st.acc[mt][2] * f0;
              r1p[8] += st.acc[mt][3] * f1;
            }
          }
        }
        __syncthreads();
      }
    }
    // a retrieval slot has one piece per CTA owning its tiles; a local head one per CTA whose
    // range meets it (index CTA + ordinal, as in attend_kernel)
    bool single;
    int piece;
    if (u.kind == 0) {
      single = min(P, tb.G[u.idx + 1] - tb.G[u.idx]) == 1;
      piece = tb.pb[u.idx] + tb.pidx[u.idx];
    } else {
      const int len = (int)(tb.loff[u.idx + 1] - tb.loff[u.idx]);
      single = u.r0 == 0 && u.r1 == len;
      piece = tb.pb[S] + cta + u.idx;
    }
    float* sFin = sML + kW * kMaxGroup * 2;  // [8][2]: M, then L (1 / L for a whole head)
    if (tid < a.G) {
      float M = -INFINITY;
#pragma unroll
      for (int wq = 0; wq < kW; ++wq) M = fmaxf(M, sML[(wq * kMaxGroup + tid) * 2]);
      float L = 0.f;
#pragma unroll
      for (int wq = 0; wq < kW; ++wq) {
        const float mw = sML[(wq * kMaxGroup + tid) * 2];
        if (mw != -INFINITY) L += sML[(wq * kMaxGroup + tid) * 2 + 1] * exp2f(mw - M);
      }
      sFin[2 * tid] = M;
      sFin[2 * tid + 1] = single ? 1.f / L : L;
    }
    __syncthreads();
    for (int e = tid; e < kMaxGroup * 16; e += kT) {
      const int jq = e >> 4, d0 = (e & 15) * 8;
      if (jq < a.G) {
        const float4* src = reinterpret_cast<const float4*>(sO + jq * kOPitch + d0);
        float4 o0 = src[0], o1 = src[1];
        float4* dst;
        if (single) {
          const float inv = sFin[2 * jq + 1];
          o0.x *= inv; o0.y *= inv; o0.z *= inv; o0.w *= inv;
          o1.x *= inv; o1.y *= inv; o1.z *= inv; o1.w *= inv;
          dst = reinterpret_cast<float4*>(
              a.out + ((size_t)b * a.Hq + (size_t)kvh * a.G + jq) * kHeadDim + d0);
        } else {
          float* pc = f.partials + (size_t)piece * kPartFloats;
          dst = reinterpret_cast<float4*>(pc + jq * kHeadDim + d0);
          if ((e & 15) == 0) {
            pc[kPartO + jq] = sFin[2 * jq];
            pc[kPartO + kMaxGroup + jq] = sFin[2 * jq + 1];
          }
        }
        dst[0] = o0;
        dst[1] = o1;
      }
    }
    __syncthreads();  // sComb is reused by the next unit
  }
  cp_async_wait<0>();  // the stages become the merge arrays
  grid_barrier(f.bar, w.status, &aborted, f.wait_ns, -1);
  if (aborted) return;

  // ---- phase 5: merge the split heads ------------------------------------------------------
  // unit (head hd, query head jq, quarter qtr); pieces i = 0 .. n-1 at base + i:
  //   out = sum_i f_i O_i / sum_i f_i l_i,  f_i = 2^(m_i - max m)  (0 for an empty piece)
  float* sF = reinterpret_cast<float*>(smem);
  float* sL = sF + 1024;
  float* red = sL + 1024;
  float4* racc = reinterpret_cast<float4*>(smem + 2 * 1024 * 4 + 256);  // [kW][8]
  const int units = nheads * a.G * 4;
  const int rr = tid >> 3, c8 = tid & 7;
  for (int un = cta; un < units; un += P) {
    const int hd = un / (a.G * 4), jq = (un >> 2) % a.G, qtr = un & 3;
    const int b = hd / a.Hkv, kvh = hd - b * a.Hkv, j = a.slot_of_kvh[kvh];
    int base, n;
    if (j >= 0) {
      const int s = b * a.nret + j;
      n = min(P, tb.G[s + 1] - tb.G[s]);
      base = tb.pb[s];
    } else {
      const int lh = tb.lord[hd];
      const int cf = (int)cta_of(tb.loff[lh], Wt, Ploc);
      const int cl = (int)cta_of(tb.loff[lh + 1] - 1, Wt, Ploc);
      n = cl - cf + 1;
      base = tb.pb[S] + cf + lh;
    }
    if (n <= 1) continue;  // written by phase 4
    const float* pb = f.partials + (size_t)base * kPartFloats;
    const int col = jq * kHeadDim + qtr * 32 + c8 * 4;
    float4 ov[kMergeRegs];
#pragma unroll
    for (int k = 0; k < kMergeRegs; ++k) {
      const int i = rr + k * kMergeRows;
      ov[k] = (i < n) ? __ldcg(reinterpret_cast<const float4*>(pb + (size_t)i * kPartFloats + col))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mx = -INFINITY;
    for (int i = tid; i < n; i += kT) {
      const float m = __ldcg(pb + (size_t)i * kPartFloats + kPartO + jq);
      sL[i] = __ldcg(pb + (size_t)i * kPartFloats + kPartO + kMaxGroup + jq);
      sF[i] = m;
      mx = fmaxf(mx, m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int k = 1; k < kW; ++k) M = fmaxf(M, red[k]);
    float ls = 0.f;
    for (int i = tid; i < n; i += kT) {
      const float m = sF[i];
      const float fi = (m == -INFINITY) ? 0.f : exp2f(m - M);
      sF[i] = fi;
      ls += sL[i] * fi;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    __syncthreads();  // every thread has read red[] (the maxima)
    if (lane == 0) red[warp] = ls;
    __syncthreads();  // red[] holds the l sums, sF[] the factors
    float L = 0.f;
#pragma unroll
    for (int k = 0; k < kW; ++k) L += red[k];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kMergeRegs; ++k) {
      const int i = rr + k * kMergeRows;
      if (i < n) {
        const float fi = sF[i];
        if (fi != 0.f) {
          acc.x += ov[k].x * fi; acc.y += ov[k].y * fi; acc.z += ov[k].z * fi; acc.w += ov[k].w * fi;
        }
      }
    }
    for (int i = rr + kMergeRegs * kMergeRows; i < n; i += kMergeRows) {
      const float fi = sF[i];
      if (fi != 0.f) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(pb + (size_t)i * kPartFloats + col));
        acc.x += v.x * fi; acc.y += v.y * fi; acc.z += v.z * fi; acc.w += v.w * fi;
      }
    }
    // rows of a warp: lanes c8, c8 + 8, c8 + 16, c8 + 24; then the warps in order
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) {
      acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
      acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
      acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
      acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
    if (lane < 8) racc[warp * 8 + lane] = acc;
    __syncthreads();
    if (tid < 8) {
      float4 o = racc[tid];
#pragma unroll
      for (int k = 1; k < kW; ++k) {
        const float4 v = racc[k * 8 + tid];
        o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
      }
      const float inv = 1.f / L;
      float4* dst = reinterpret_cast<float4*>(
          a.out + ((size_t)b * a.Hq + (size_t)kvh * a.G + jq) * kHeadDim + qtr * 32 + tid * 4);
      *dst = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    }
    __syncthreads();  // the arrays are reused by the next unit
  }
}

}  // namespace rtp
