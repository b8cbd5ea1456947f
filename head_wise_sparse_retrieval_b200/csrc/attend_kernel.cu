// attend_kernel.cu -- exact softmax attention over a token set per KV head (sm_100a).
//
// Follows "Full Attention Strikes Back ..." (xllm-io paper review), section 三, 核心公式 /
// 自适应稀疏注意力:  O_h(m) = sum_{n in S_h(m)} softmax_{S_h(m)}(q^T k_n / sqrt(d_h)) v_n,
// with S_h the selected set of a retrieval head, and section 五 测试配置 / gist.science
// Methodology 1 for local heads (S = 4 sinks U the last 8192 positions).
//
// One persistent launch per layer covers every (b, KV head) of the layer. The token sets of
// all heads are laid end to end (retrieval: the |S| selected positions; local: the window
// set; dense mode: all N) and the concatenation is cut into P equal ranges, one per CTA
// (split-K, balanced to the token). A CTA cuts its range, head by head, into 16-token tiles
// dealt round-robin to its warps. Each warp runs its own kAttendDepth-deep pipeline:
//   * positions: the selected list (prefetched one tile ahead, so the load overlaps the
//     math) or window arithmetic;
//   * data: each tile's 16 K rows and 16 V rows (256 B each) are gathered with 16-byte
//     cp.async (L2 evict-first; rows past the end of a head are zero-filled, not read);
//   * math on the tensor cores (mma m16n8k16, bf16 in, fp32 accumulate) with the 8 query
//     heads of the GQA group as N = 8, so every fetched row serves the whole group:
//     S^T = K Q^T, online softmax in the log2 domain, P rounded to bf16 and transposed in
//     registers (movmatrix), O^T += V^T P^T.
// At the end of a head's piece the warps merge (m, l, O) through shared memory. A head split
// over several CTAs writes one partial per CTA; a two-level tree of atomic tickets (fan-in 16,
// nothing waits) lets the last CTA of each group and then of the head merge the partials in a
// fixed order (log-sum-exp) and write the output.
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kWarps = kAttendWarps;
constexpr int kTile = 16;
constexpr int kDepth = kAttendDepth;
constexpr int kWarpStage = 2 * kTile * kRowBytes;          // 16 K rows then 16 V rows
constexpr int kOPitch = kHeadDim + 4;                      // padded row of the merge buffer
constexpr int kCombFloats = kMaxGroup * kOPitch + kWarps * kMaxGroup * 2;
constexpr int kMaxMerge = 2 * kMergeFanIn;                 // sources of one merge
constexpr int kMergeBatch = 4;                             // sources loaded per round trip

// Shared memory: per-warp stages, the warp-merge buffer, then the head tables sized by the
// layer (B * Hkv + 1 offsets, B lengths).
struct SmemLayout {
  static constexpr size_t stage_off = 0;
  static constexpr size_t comb_off = stage_off + (size_t)kWarps * kDepth * kWarpStage;
  static constexpr size_t hoff_off = comb_off + (size_t)kCombFloats * 4;
  __host__ __device__ static size_t seq_off(int nheads) { return hoff_off + (size_t)(nheads + 1) * 8; }
  __host__ __device__ static size_t total(int nheads, int batch) {
    return seq_off(nheads) + (size_t)batch * 4;
  }
};

// Byte offset of 16-byte column c of row r inside a stage: rows are 256 B, the column is
// XOR-swizzled with the row so that the 8 rows an ldmatrix reads hit 8 different bank groups.
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * kRowBytes + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ int window_len(int N, int W, int S) {
  return (N <= W + S) ? N : W + S;
}
__device__ __forceinline__ int window_pos(int r, int N, int W, int S) {
  return (N <= W + S) ? r : (r < S ? r : N - W + (r - S));
}

// CTA whose range [floor(c T / P), floor((c+1) T / P)) holds position x (0 <= x < T, P <= T).
__device__ __forceinline__ long long cta_of(long long x, long long T, long long P) {
  return ((x + 1) * P + T - 1) / T - 1;
}

// The segments of this CTA's range, head by head, in order.
struct Walk {
  const long long* off;
  int nheads;
  long long t, t1;
  int h;
  __device__ void begin(const long long* o, int nh, long long t0, long long tend) {
    off = o;
    nheads = nh;
    t = t0;
    t1 = tend;
    int lo = 0, hi = nh - 1;  // head with off[h] <= t0 < off[h+1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= t0) lo = mid; else hi = mid - 1;
    }
    h = lo;
  }
  __device__ bool next(int& head, int& r0, int& r1) {  // next non-empty segment
    while (t < t1 && h < nheads) {
      const long long hend = min(t1, off[h + 1]);
      if (hend > t) {
        head = h;
        r0 = (int)(t - off[h]);
        r1 = (int)(hend - off[h]);
        t = hend;
        ++h;
        return true;
      }
      ++h;
    }
    return false;
  }
};

// A head's token set and where its rows live.
struct HeadRef {
  const __nv_bfloat16* kbase;
  const __nv_bfloat16* vbase;
  const int* sel;  // selected list (retrieval), else nullptr
  int N;
  int window;      // 1: local head (window + sinks), 0: dense or retrieval
};

__device__ __forceinline__ HeadRef head_ref(const LayerArgs& a, const Workspace& w,
                                            const int* sSeq, int hd) {
  const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
  const size_t head = (size_t)b * a.Hkv + kvh;
  HeadRef r;
  r.kbase = a.k_cache + head * (size_t)a.max_ctx * kHeadDim;
  r.vbase = a.v_cache + head * (size_t)a.max_ctx * kHeadDim;
  r.N = sSeq[b];
  const int j = a.dense ? -1 : a.slot_of_kvh[kvh];
  r.sel = (j >= 0) ? w.sel_idx + (size_t)(b * a.nret + j) * w.ld : nullptr;
  r.window = (!a.dense && j < 0) ? 1 : 0;
  return r;
}

// Walks this warp's tiles k = w, w + kWarps, ... across the CTA's segments (for the loads,
// which run ahead of the math). Tile k of a segment starting at global tile index kb covers
// ranks r0 + 16 (k - kb) ... of its head.
struct TileIter {
  Walk walk;
  int hd, r0, r1, kb, nt;
  bool have;
  __device__ void begin(const long long* off, int nheads, long long t0, long long t1) {
    walk.begin(off, nheads, t0, t1);
    kb = 0;
    nt = 0;
    have = false;
  }
  // Moves to the segment holding tile k (k never decreases). False past the last tile.
  __device__ bool locate(int k) {
    while (!have || k >= kb + nt) {
      if (have) kb += nt;
      if (!walk.next(hd, r0, r1)) return false;
      nt = (r1 - r0 + kTile - 1) / kTile;
      have = true;
    }
    return true;
  }
};

// Lane l < 16 returns the cache position of token l of the tile (rank r), -1 past n. For a
// retrieval head the load is issued here and consumed one tile later.
__device__ __forceinline__ int tile_positions(const HeadRef& h, const LayerArgs& a, int r, int n,
                                              int lane) {
  if (lane >= n || lane >= kTile) return -1;
  const int rank = r + lane;
  if (h.sel) return __ldcg(h.sel + rank);
  return h.window ? window_pos(rank, h.N, a.window, a.sinks) : rank;
}

// Gathers the tile's K and V rows into the stage: lane l copies 16-byte column c = l % 16 of
// rows 2i + l / 16; the positions come from lanes 0..15 of pos.
__device__ __forceinline__ void issue_tile(uint32_t stage, const HeadRef& h, int pos, int n,
                                           int lane, uint64_t policy, unsigned* status) {
  const int c = lane & 15, par = lane >> 4;
#pragma unroll
  for (int i = 0; i < kTile / 2; ++i) {
    const int row = 2 * i + par;
    int p = __shfl_sync(0xffffffffu, pos, row);
    const bool valid = row < n;
    if (valid && (p < 0 || p >= h.N)) {
      if (c == 0) atomicOr(status, kDevBadIndex);
      p = 0;
    }
    const size_t off = valid ? (size_t)p * kHeadDim + c * 8 : 0;
    const unsigned bytes = valid ? 16u : 0u;
    cp_async_16(stage + swz(row, c), h.kbase + off, bytes, policy);
    cp_async_16(stage + swz(kTile + row, c), h.vbase + off, bytes, policy);
  }
}

// Log-sum-exp merge of n partials (o[8][128], m[8], l[8]), n <= kMaxMerge, by the 128 threads
// of the CTA. (m, l) of every source go through shared memory in one round trip; then thread
// tid owns query head jq = tid / 16 and dimensions 8 (tid % 16) .. +7 and issues the 16-byte
// loads of kMergeBatch sources at a time. final: out[jq][d] = O / L; otherwise dst receives a partial.
__device__ void merge_partials(int n, int G, bool final, float* dst, const float* const* src,
                               float (*mM)[kMaxGroup], float (*mF)[kMaxGroup], float* mL,
                               int tid) {
  __syncthreads();  // src[] written
  for (int e = tid; e < n * 2 * kMaxGroup; e += kAttendThreads) {
    const int i = e / (2 * kMaxGroup), r = e % (2 * kMaxGroup);
    const float v = __ldcg(src[i] + kPartO + r);  // m[0..7] then l[0..7]
    if (r < kMaxGroup) mM[i][r] = v; else mF[i][r - kMaxGroup] = v;
  }
  __syncthreads();
  if (tid < G) {
    float M = -INFINITY;
    for (int i = 0; i < n; ++i) M = fmaxf(M, mM[i][tid]);
    float L = 0.f;
    for (int i = 0; i < n; ++i) {
      const float f = exp2f(mM[i][tid] - M);
      L += mF[i][tid] * f;
      mF[i][tid] = f;  // the l slot now holds the scale factor of source i
    }
    mL[tid] = L;
    mM[0][tid] = M;    // source 0's m is no longer needed
  }
  __syncthreads();
  const int jq = tid >> 4, d0 = (tid & 15) * 8;
  if (jq < G) {
    float4 o0 = make_float4(0.f, 0.f, 0.f, 0.f), o1 = o0;
    for (int i0 = 0; i0 < n; i0 += kMergeBatch) {
      float4 v0[kMergeBatch], v1[kMergeBatch];
#pragma unroll
      for (int i = 0; i < kMergeBatch; ++i) {
        if (i0 + i < n) {
          const float4* p = reinterpret_cast<const float4*>(src[i0 + i] + jq * kHeadDim + d0);
          v0[i] = __ldcg(p);
          v1[i] = __ldcg(p + 1);
        }
      }
#pragma unroll
      for (int i = 0; i < kMergeBatch; ++i) {
        if (i0 + i < n) {
          const float f = mF[i0 + i][jq];
          o0.x += v0[i].x * f; o0.y += v0[i].y * f; o0.z += v0[i].z * f; o0.w += v0[i].w * f;
          o1.x += v1[i].x * f; o1.y += v1[i].y * f; o1.z += v1[i].z * f; o1.w += v1[i].w * f;
        }
      }
    }
    if (final) {
      const float inv = 1.f / mL[jq];
      float4* q = reinterpret_cast<float4*>(dst + (size_t)jq * kHeadDim + d0);
      q[0] = make_float4(o0.x * inv, o0.y * inv, o0.z * inv, o0.w * inv);
      q[1] = make_float4(o1.x * inv, o1.y * inv, o1.z * inv, o1.w * inv);
    } else {
      float4* q = reinterpret_cast<float4*>(dst + jq * kHeadDim + d0);
      q[0] = o0;
      q[1] = o1;
      if ((tid & 15) == 0) {
        dst[kPartO + jq] = mM[0][jq];
        dst[kPartO + kMaxGroup + jq] = mL[jq];
      }
    }
  }
  __syncthreads();  // scratch reusable
}

}  // namespace

size_t attend_smem_bytes(int nheads, int batch) { return SmemLayout::total(nheads, batch); }

__global__ void __launch_bounds__(kAttendThreads, kAttendCtasPerSm) attend_kernel(
    const LayerArgs a, const Workspace w) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int nheads = a.B * a.Hkv;
  float* sComb = reinterpret_cast<float*>(smem + SmemLayout::comb_off);
  long long* sOff = reinterpret_cast<long long*>(smem + SmemLayout::hoff_off);
  int* sSeq = reinterpret_cast<int*>(smem + SmemLayout::seq_off(nheads));
  __shared__ int is_last;
  __shared__ const float* msrc[kMaxMerge];
  __shared__ float mM[kMaxMerge][kMaxGroup];
  __shared__ float mF[kMaxMerge][kMaxGroup];
  __shared__ float mL[kMaxGroup];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  pdl_wait();

  // ---- the layer's heads and their token-set lengths --------------------------------------
  for (int b = tid; b < a.B; b += kAttendThreads) {
    const int n = a.seq_lens[b];
    sSeq[b] = n < 1 ? 1 : (n > a.max_ctx ? a.max_ctx : n);
  }
  __syncthreads();
  for (int hd = tid; hd < nheads; hd += kAttendThreads) {
    const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
    const int N = sSeq[b];
    int len;
    const bool ret = !a.dense && a.slot_of_kvh[kvh] >= 0;
    if ((a.heads == kHeadsLocal && ret) || (a.heads == kHeadsRetrieval && !ret)) {
      len = 0;  // another launch of this layer covers the head
    } else if (a.dense) {
      len = N;
    } else if (ret) {
      len = __ldcg(w.sel_total + b * a.nret + a.slot_of_kvh[kvh]);
      len = len < 1 ? 1 : (len > N ? N : len);
    } else {
      len = window_len(N, a.window, a.sinks);
    }
    sOff[hd + 1] = len;
  }
  __syncthreads();
  if (warp == 0) {  // inclusive scan of the lengths, 32 heads at a time
    long long carry = 0;
    for (int base = 0; base < nheads; base += 32) {
      const int i = base + lane;
      long long x = (i < nheads) ? sOff[i + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (i < nheads) sOff[i + 1] = carry + x;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) sOff[0] = 0;
  }
  __syncthreads();
  pdl_launch_dependents();

  // P = min(grid, T) CTAs take part, so every range is non-empty and the pieces of a head are
  // exactly the CTAs c_first..c_last (the ticket count of its merge)
  const long long T = sOff[nheads];
  const long long P = min((long long)gridDim.x, T);  // T >= 1: the launch covers >= 1 head
  if ((long long)blockIdx.x >= P) return;
  const long long t0 = (long long)blockIdx.x * T / P;
  const long long t1 = ((long long)blockIdx.x + 1) * T / P;

  // total tiles of this CTA (segments are few)
  int ktot = 0;
  {
    Walk cnt;
    cnt.begin(sOff, nheads, t0, t1);
    int hd, r0, r1;
    while (cnt.next(hd, r0, r1)) ktot += (r1 - r0 + kTile - 1) / kTile;
  }

  const uint64_t policy = l2_policy_evict_first();
  const uint32_t my_stages = smem_u32(smem + SmemLayout::stage_off) + warp * kDepth * kWarpStage;

  // ---- load side: this warp's tiles k = warp + kWarps i, positions one tile ahead ----------
  TileIter iss;
  iss.begin(sOff, nheads, t0, t1);
  HeadRef pf_h{};
  int pf_r = 0, pf_n = 0, pf_pos = -1, pf_hd = -1;
  auto prefetch = [&](int i) {  // positions of warp tile i (pf_n = 0 past the end)
    const int k = warp + kWarps * i;
    pf_n = 0;
    pf_pos = -1;
    if (k < ktot && iss.locate(k)) {
      if (iss.hd != pf_hd) {
        pf_hd = iss.hd;
        pf_h = head_ref(a, w, sSeq, pf_hd);
      }
      pf_r = iss.r0 + (k - iss.kb) * kTile;
      pf_n = min(kTile, iss.r1 - pf_r);
      pf_pos = tile_positions(pf_h, a, pf_r, pf_n, lane);
    }
  };
  auto issue = [&](int i) {  // loads of warp tile i (positions prefetched); one commit group
    if (pf_n > 0)
      issue_tile(my_stages + (i % kDepth) * kWarpStage, pf_h, pf_pos, pf_n, lane, policy,
                 w.status);
    cp_async_commit();
  };
  for (int s = 0; s < kDepth - 1; ++s) {
    prefetch(s);
    issue(s);
  }
  prefetch(kDepth - 1);

  // ---- math side: segment by segment ----
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const float scale_log2 = a.attn_scale_log2;
  // ldmatrix rows / 16-byte columns this lane addresses (before the swizzle)
  const int k_row = (lane & 7) + ((lane >> 3) & 1) * 8, k_col = lane >> 4;
  const int v_row = kTile + (lane & 7) + (lane >> 4) * 8, v_col = (lane >> 3) & 1;
  int done = 0;     // warp tiles computed
  int kseg = 0;     // global tile index of the current segment's first tile
  Walk walk;
  walk.begin(sOff, nheads, t0, t1);
  int hd, r0, r1;
  while (walk.next(hd, r0, r1)) {
    const int nt = (r1 - r0 + kTile - 1) / kTile;
    const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
    // Q^T as the B operand: b0 = q[g][16ks + 2t, +1], b1 = q[g][16ks + 8 + 2t, +1]
    uint32_t qf[8][2];
    {
      const bool valid = g < a.G;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          a.q + ((size_t)b * a.Hq + (size_t)kvh * a.G + (valid ? g : 0)) * kHeadDim);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        qf[ks][0] = valid ? qrow[ks * 8 + t] : 0u;
        qf[ks][1] = valid ? qrow[ks * 8 + 4 + t] : 0u;
      }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    for (int k = warp + kWarps * done; k < kseg + nt; k += kWarps, ++done) {
      // keep kDepth - 1 tiles in flight: issue warp tile done + kDepth - 1, then prefetch the
      // positions of the one after (their load overlaps this tile's math)
      issue(done + kDepth - 1);
      prefetch(done + kDepth);
      cp_async_wait<kDepth - 1>();
      __syncwarp();

      const int n = min(kTile, r1 - (r0 + (k - kseg) * kTile));  // valid tokens of this tile
      const uint32_t kb = my_stages + (done % kDepth) * kWarpStage;
      // S^T (16 tokens x 8 heads) = K (16 x 128) . Q^T (128 x 8), two accumulator chains
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ks += 2) {
        uint32_t fa[4], fb[4];
        ldmatrix_x4(fa, kb + swz(k_row, 2 * ks + k_col));
        ldmatrix_x4(fb, kb + swz(k_row, 2 * ks + 2 + k_col));
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
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: token 0 is valid
      if (__any_sync(0xffffffffu, mn0 > m0 || mn1 > m1)) {  // rescale only when a max grows
        const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[mt][0] *= al0;
          acc[mt][1] *= al1;
          acc[mt][2] *= al0;
          acc[mt][3] *= al1;
        }
        m0 = mn0;
        m1 = mn1;
      }
      const uint32_t p01 = pack_bf16x2(exp2f(x0 - m0), exp2f(x1 - m1));
      const uint32_t p23 = pack_bf16x2(exp2f(x2 - m0), exp2f(x3 - m1));
      l0 += bf16_lo(p01) + bf16_lo(p23);
      l1 += bf16_hi(p01) + bf16_hi(p23);
      // P^T as the B operand: transpose the 8x8 (token x head) blocks in registers
      const uint32_t pb0 = movmatrix_trans(p01);
      const uint32_t pb1 = movmatrix_trans(p23);
      // O^T (128 dims x 8 heads) += V^T (128 x 16 tokens) . P^T (16 x 8)
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t fv[4];
        ldmatrix_x4_trans(fv, kb + swz(v_row, 2 * mt + v_col));
        mma_bf16_16816(acc[mt], fv, pb0, pb1);
      }
      __syncwarp();  // the stage is refilled kDepth - 1 tiles later
    }
    kseg += nt;

    // ---- end of this head's piece: merge the warps ----------------------------------------
    // (m, l) per warp and head through shared memory; each warp rescales its O in registers
    // to the common max, then the warps add O into one buffer in a fixed order.
    float* sO = sComb;                                   // [8][kOPitch]
    float* sML = sComb + kMaxGroup * kOPitch;            // [kWarps][8][2]
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    if (g == 0) {
      sML[(warp * kMaxGroup + 2 * t) * 2] = m0;
      sML[(warp * kMaxGroup + 2 * t) * 2 + 1] = l0;
      sML[(warp * kMaxGroup + 2 * t + 1) * 2] = m1;
      sML[(warp * kMaxGroup + 2 * t + 1) * 2 + 1] = l1;
    }
    __syncthreads();
    {
      float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
      for (int wq = 0; wq < kWarps; ++wq) {
        M0 = fmaxf(M0, sML[(wq * kMaxGroup + 2 * t) * 2]);
        M1 = fmaxf(M1, sML[(wq * kMaxGroup + 2 * t + 1) * 2]);
      }
      const float f0 = (m0 == -INFINITY) ? 0.f : exp2f(m0 - M0);  // 0: a warp without tokens
      const float f1 = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M1);
#pragma unroll
      for (int wq = 0; wq < kWarps; ++wq) {
        if (warp == wq) {
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            float* r0p = sO + (2 * t) * kOPitch + 16 * mt + g;
            float* r1p = sO + (2 * t + 1) * kOPitch + 16 * mt + g;
            if (wq == 0) {
              r0p[0] = acc[mt][0] * f0;
              r1p[0] = acc[mt][1] * f1;
              r0p[8] = acc[mt][2] * f0;
              r1p[8] = acc[mt][3] * f1;
            } else {
              r0p[0] += acc[mt][0] * f0;
              r1p[0] += acc[mt][1] * f1;
              r0p[8] += acc[mt][2] * f0;
              r1p[8] += acc[mt][3] * f1;
            }
          }
        }
        __syncthreads();
      }
    }

    const long long hb = sOff[hd], he = sOff[hd + 1];
    const int c_first = (int)cta_of(hb, T, P), c_last = (int)cta_of(he - 1, T, P);
    const int d = tid;  // 0..127: one output dimension per thread
    float* out_h = a.out + ((size_t)b * a.Hq + (size_t)kvh * a.G) * kHeadDim;
    const bool single = (c_first == c_last);
    float* piece = w.partials + ((size_t)blockIdx.x + hd) * kPartFloats;
    for (int jq = 0; jq < a.G; ++jq) {
      float M = -INFINITY;
#pragma unroll
      for (int wq = 0; wq < kWarps; ++wq) M = fmaxf(M, sML[(wq * kMaxGroup + jq) * 2]);
      float L = 0.f;
#pragma unroll
      for (int wq = 0; wq < kWarps; ++wq) {
        const float mw = sML[(wq * kMaxGroup + jq) * 2];
        if (mw != -INFINITY) L += sML[(wq * kMaxGroup + jq) * 2 + 1] * exp2f(mw - M);
      }
      const float O = sO[jq * kOPitch + d];
      if (single) {
        out_h[(size_t)jq * kHeadDim + d] = O / L;
      } else {
        piece[jq * kHeadDim + d] = O;
        if (d == 0) {
          piece[kPartO + jq] = M;
          piece[kPartO + kMaxGroup + jq] = L;
        }
      }
    }
    if (a.sel_count && (int)blockIdx.x == c_first && tid == 0) a.sel_count[hd] = (int)(he - hb);
    if (!single) {
      // Two-level merge tree over the pieces of this head, fan-in kMergeFanIn: the last CTA of
      // each aligned group of kMergeFanIn CTAs merges the group's pieces, the last group merges
      // the groups. Tickets only: nothing waits.
      const int gi = (int)blockIdx.x / kMergeFanIn;
      const int g_first = c_first / kMergeFanIn, g_last = c_last / kMergeFanIn;
      const int gs = max(c_first, gi * kMergeFanIn);
      const int ge = min(c_last, gi * kMergeFanIn + kMergeFanIn - 1);
      bool holds_group = true;
      if (ge > gs) {
        __syncthreads();  // the piece is written (CTA scope); thread 0 publishes it (gpu scope)
        unsigned* tk = w.ticket_group + (size_t)hd * w.n_merge_groups + gi;
        if (tid == 0) {
          __threadfence();
          is_last = (atomicAdd(tk, 1u) == (unsigned)(ge - gs));
          if (is_last) __threadfence();
        }
        __syncthreads();
        holds_group = is_last;
        if (holds_group) {
          if (tid < ge - gs + 1)
            msrc[tid] = w.partials + ((size_t)(gs + tid) + hd) * kPartFloats;
          const bool final_merge = (g_first == g_last);
          float* dst = final_merge ? out_h
                                   : w.group_partials +
                                         ((size_t)hd * w.n_merge_groups + gi) * kPartFloats;
          merge_partials(ge - gs + 1, a.G, final_merge, dst, msrc, mM, mF, mL, tid);
          if (tid == 0) *tk = 0u;
          if (final_merge) holds_group = false;
        }
      }
      if (holds_group) {  // this CTA holds group gi's merged result: join the head's merge
        __syncthreads();
        if (tid == 0) {
          __threadfence();
          is_last = (atomicAdd(w.ticket_attend + hd, 1u) == (unsigned)(g_last - g_first));
          if (is_last) __threadfence();
        }
        __syncthreads();
        if (is_last) {
          const int ng = g_last - g_first + 1;
          if (tid < ng) {
            const int gg = g_first + tid;
            const int s0 = max(c_first, gg * kMergeFanIn);
            const int s1 = min(c_last, gg * kMergeFanIn + kMergeFanIn - 1);
            msrc[tid] = (s1 > s0) ? w.group_partials + ((size_t)hd * w.n_merge_groups + gg) *
                                                           kPartFloats
                                  : w.partials + ((size_t)s0 + hd) * kPartFloats;
          }
          merge_partials(ng, a.G, true, out_h, msrc, mM, mF, mL, tid);
          if (tid == 0) w.ticket_attend[hd] = 0u;
        }
      }
    }
    __syncthreads();  // sComb is reused by the next piece
  }
  cp_async_wait<0>();  // nothing may land in shared memory after the CTA exits
}

}  // namespace rtp
