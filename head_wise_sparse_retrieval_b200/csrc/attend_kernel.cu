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
//   * positions: the selected list, loaded two tiles before the tile's data is requested (the
//     index round trip overlaps two tiles of streaming), or window arithmetic;
//   * data: each tile's 16 K rows and 16 V rows (256 B each) are gathered with 16-byte
//     cp.async (L2 evict-first; rows past the end of a head are zero-filled, not read);
//   * math on the tensor cores (mma m16n8k16, bf16 in, fp32 accumulate) with the 8 query
//     heads of the GQA group as N = 8, so every fetched row serves the whole group:
//     S^T = K Q^T, online softmax in the log2 domain, P rounded to bf16 and transposed in
//     registers (movmatrix), O^T += V^T P^T.
// At the end of a head's piece the warps merge (m, l, O) through shared memory. A head held by
// one CTA is written out there; a head split over several CTAs leaves one partial per CTA, and
// merge_kernel (the next launch on the stream) combines them by log-sum-exp in a fixed order.
#include "attend_tile.cuh"
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kWarps = kAttendWarps;
constexpr int kDepth = kAttendDepth;
constexpr int kOPitch = kHeadDim + 4;                      // padded row of the merge buffer
constexpr int kCombFloats = kMaxGroup * kOPitch + kWarps * kMaxGroup * 2 + kMaxGroup * 2;
constexpr int kMergeRows = kMergeThreads / 8;              // pieces a merge pass loads at once
constexpr int kMergeRegs = 20;                             // passes kept in registers (320 pieces)

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

// Size of head hd's token set (retrieval: |S| from the selection, clamped to [1, N]; local:
// the window set; dense: N), N = seq_lens[b] clamped to [1, max_ctx]. The attention split and
// the merge both derive the pieces of a head from these sizes.
__device__ __forceinline__ int head_len(const LayerArgs& a, const Workspace& w, int hd, int* N_out) {
  const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
  const bool ret = !a.dense && a.slot_of_kvh[kvh] >= 0;
  const int n = a.seq_lens[b];  // both loads in flight together
  const int ns = ret ? __ldcg(w.sel_total + b * a.nret + a.slot_of_kvh[kvh]) : 0;
  const int N = n < 1 ? 1 : (n > a.max_ctx ? a.max_ctx : n);
  if (N_out) *N_out = N;
  if (a.dense) return N;
  if (ret) return ns < 1 ? 1 : (ns > N ? N : ns);
  return window_len(N, a.window, a.sinks);
}

// How a layer's heads are cut over the attention grid, from their token-set sizes. A head of
// at most kTinyLen tokens (a concentrated query's few selected positions) takes a CTA of its
// own when such heads are few (at most grid / 8, and the others keep a token per CTA):
// otherwise the CTA holding it would also hold pieces of its neighbours and run an end-of-piece
// merge for each. The other heads' sets are laid end to end (the tiny heads with no tokens) and
// cut into P equal ranges, CTAs 0 .. P-1; the tiny heads follow in head order, CTAs P .. P +
// ntiny - 1, each a single piece. Without such heads, or with too many, every set is laid end
// to end (ntiny = 0). One warp calls it: off[1 .. nheads] hold the sizes on entry and the
// inclusive scan of the laid-out sizes on return (off[0] = 0); every lane returns the same
// values, including the head and size of CTA cta when it is a tiny head's (else -1, 0).
constexpr int kTinyLen = 4 * kTile;
struct HeadSplit {
  long long T, P;   // laid-out tokens, CTAs that cut them
  int ntiny;        // heads with a CTA of their own
  int tiny_head, tiny_len;
};
__device__ HeadSplit split_heads(long long* off, int nheads, int grid, int cta, int lane) {
  int ntiny = 0;
  long long tbig = 0, tall = 0;
  for (int base = 0; base < nheads; base += 32) {
    const int i = base + lane;
    const long long len = (i < nheads) ? off[i + 1] : 0;
    const bool tiny = i < nheads && len <= kTinyLen;
    ntiny += __popc(__ballot_sync(0xffffffffu, tiny));
    long long big = tiny ? 0 : len, all = len;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      big += __shfl_xor_sync(0xffffffffu, big, o);
      all += __shfl_xor_sync(0xffffffffu, all, o);
    }
    tbig += big;
    tall += all;
  }
  const bool use = ntiny >= 1 && ntiny < nheads && 8 * ntiny <= grid && tbig >= grid - ntiny;
  HeadSplit r;
  r.ntiny = use ? ntiny : 0;
  r.T = use ? tbig : tall;
  r.P = min((long long)(grid - r.ntiny), r.T);
  r.tiny_head = -1;
  r.tiny_len = 0;
  const long long k = (long long)cta - r.P;  // this CTA's rank among the tiny heads' CTAs
  if (use && k >= 0 && k < ntiny) {
    int seen = 0;
    for (int base = 0; base < nheads; base += 32) {
      const int i = base + lane;
      const long long len = (i < nheads) ? off[i + 1] : 0;
      const unsigned m = __ballot_sync(0xffffffffu, i < nheads && len <= kTinyLen);
      const int here = __popc(m);
      if (r.tiny_head < 0 && k < seen + here) {
        const int l = __fns(m, 0, (int)(k - seen) + 1);  // lane of the (k - seen)-th set bit
        r.tiny_head = base + l;
        r.tiny_len = (int)__shfl_sync(0xffffffffu, len, l);
      }
      seen += here;
    }
  }
  long long carry = 0;
  for (int base = 0; base < nheads; base += 32) {  // inclusive scan, 32 heads at a time
    const int i = base + lane;
    const long long len = (i < nheads) ? off[i + 1] : 0;
    long long x = (use && len <= kTinyLen) ? 0 : len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    __syncwarp();  // every lane has read its size before any is overwritten
    if (i < nheads) off[i + 1] = carry + x;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) off[0] = 0;
  __syncwarp();
  return r;
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

// Gathers the tile's K and V rows into the stage (attend_tile.cuh): rows past n are
// zero-filled, a position outside [0, N) is replaced by 0 and reported.
__device__ __forceinline__ void issue_tile(uint32_t stage, const HeadRef& h, int pos, int n,
                                           int lane, uint64_t policy, unsigned* status) {
  gather_tile(stage, h.kbase, h.vbase, h.N, pos, n, lane, policy, status);
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

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Without retrieval heads nothing here depends on the launch before (the previous layer's
  // merge, which reads the partials this kernel writes). When the caller vouches that the
  // inputs are ready, the wait moves to just before the first write.
  const bool early = a.early && (a.nret == 0 || a.dense);
  if (!early) pdl_wait();

  // ---- the layer's heads and their token-set lengths --------------------------------------
  for (int hd = tid; hd < nheads; hd += kAttendThreads) {
    int N;
    const int len = head_len(a, w, hd, &N);
    if (hd % a.Hkv == 0) sSeq[hd / a.Hkv] = N;
    sOff[hd + 1] = len;
  }
  __syncthreads();
  __shared__ long long sSplit[2];  // P, and the end of this CTA's laid-out coordinates
  __shared__ int sRole;            // 0: a range of the laid-out sets, 1: a tiny head, 2: none
  if (warp == 0) {
    // P CTAs cut the laid-out sets, so every range is non-empty and the pieces of a head are
    // exactly the CTAs c_first..c_last. A tiny head's CTA sees the sets as if its head were the
    // only one: sizes 0 before it, its size from it on.
    const HeadSplit sp = split_heads(sOff, nheads, (int)gridDim.x, (int)blockIdx.x, lane);
    if (sp.tiny_head >= 0)
      for (int h = lane; h <= nheads; h += 32) sOff[h] = (h > sp.tiny_head) ? sp.tiny_len : 0;
    if (lane == 0) {
      sSplit[0] = sp.P;
      sSplit[1] = sp.tiny_head >= 0 ? sp.tiny_len : sp.T;
      sRole = ((long long)blockIdx.x < sp.P) ? 0 : (sp.tiny_head >= 0 ? 1 : 2);
    }
  }
  __syncthreads();
  pdl_launch_dependents();
  if (sRole == 2) return;
  long long t0, t1;
  if (sRole == 0) {
    const long long P = sSplit[0], T = sSplit[1];
    t0 = floor_div((long long)blockIdx.x * T, P);
    t1 = floor_div(((long long)blockIdx.x + 1) * T, P);
  } else {
    t0 = 0;
    t1 = sSplit[1];
  }

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
  // Two position slots: A holds the next tile to issue, B the one after. fill() loads a tile's
  // positions into B; issue() requests the data of A's tile, then A takes B.
  HeadRef fill_h{}, iss_h{};
  int fill_hd = -1, iss_hd = -1;
  int a_hd = -1, a_n = 0, a_pos = -1, b_hd = -1, b_n = 0, b_pos = -1;
  auto fill = [&](int i) {  // positions of warp tile i into B (b_n = 0 past the end)
    const int k = warp + kWarps * i;
    b_n = 0;
    b_pos = -1;
    if (k < ktot && iss.locate(k)) {
      if (iss.hd != fill_hd) {
        fill_hd = iss.hd;
        fill_h = head_ref(a, w, sSeq, fill_hd);
      }
      const int r = iss.r0 + (k - iss.kb) * kTile;
      b_hd = fill_hd;
      b_n = min(kTile, iss.r1 - r);
      b_pos = tile_positions(fill_h, a, r, b_n, lane);
    }
  };
  auto shift = [&]() {
    a_hd = b_hd;
    a_n = b_n;
    a_pos = b_pos;
  };
  auto issue = [&](int i) {  // loads of warp tile i (A's positions); one commit group
    if (a_n > 0) {
      if (a_hd != iss_hd) {
        iss_hd = a_hd;
        iss_h = head_ref(a, w, sSeq, iss_hd);
      }
      issue_tile(my_stages + (i % kDepth) * kWarpStage, iss_h, a_pos, a_n, lane, policy,
                 w.status);
    }
    cp_async_commit();
  };
  for (int s = 0; s < kDepth - 1; ++s) {
    fill(s);
    shift();
    issue(s);
  }
  fill(kDepth - 1);
  shift();
  fill(kDepth);

  // ---- math side: segment by segment ----
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const float scale_log2 = a.attn_scale_log2;
  int done = 0;     // warp tiles computed
  int kseg = 0;     // global tile index of the current segment's first tile
  Walk walk;
  walk.begin(sOff, nheads, t0, t1);
  int hd, r0, r1;
  while (walk.next(hd, r0, r1)) {
    const int nt = (r1 - r0 + kTile - 1) / kTile;
    const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
    uint32_t qf[8][2];
    load_q_frag(qf, a.q + ((size_t)b * a.Hq + (size_t)kvh * a.G) * kHeadDim, a.G, lane);
    TileAcc st;
    st.init();

    for (int k = warp + kWarps * done; k < kseg + nt; k += kWarps, ++done) {
      // keep kDepth - 1 tiles in flight: issue warp tile done + kDepth - 1, then prefetch the
      // positions of the one after (their load overlaps this tile's math)
      issue(done + kDepth - 1);
      shift();
      fill(done + kDepth + 1);
      cp_async_wait<kDepth - 1>();
      __syncwarp();

      const int n = min(kTile, r1 - (r0 + (k - kseg) * kTile));  // valid tokens of this tile
      attend_tile(my_stages + (done % kDepth) * kWarpStage, qf, n, scale_log2, lane, st);
      __syncwarp();  // the stage is refilled kDepth - 1 tiles later
    }
    kseg += nt;

    if (early) pdl_wait();  // the partials below may still be read by the previous merge
    // ---- end of this head's piece: merge the warps ----------------------------------------
    // (m, l) per warp and head through shared memory; each warp rescales its O in registers
    // to the common max, then the warps add O into one buffer in a fixed order.
    float* sO = sComb;                                   // [8][kOPitch]
    float* sML = sComb + kMaxGroup * kOPitch;            // [kWarps][8][2]
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
      for (int wq = 0; wq < kWarps; ++wq) {
        M0 = fmaxf(M0, sML[(wq * kMaxGroup + 2 * t) * 2]);
        M1 = fmaxf(M1, sML[(wq * kMaxGroup + 2 * t + 1) * 2]);
      }
      const float f0 = (st.m0 == -INFINITY) ? 0.f : exp2f(st.m0 - M0);  // 0: a warp without tokens
      const float f1 = (st.m1 == -INFINITY) ? 0.f : exp2f(st.m1 - M1);
#pragma unroll
      for (int wq = 0; wq < kWarps; ++wq) {
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

    // this CTA holds the head's first piece when its segment starts at rank 0, the last when
    // it ends at the head's size; one piece covering both is the whole head
    const int len = (int)(sOff[hd + 1] - sOff[hd]);
    const bool first_piece = (r0 == 0), last_piece = (r1 == len);
    const bool single = first_piece && last_piece;
    float* sFin = sML + kWarps * kMaxGroup * 2;  // [8][2]: M, then L (1 / L for a whole head)
    if (tid < a.G) {  // the piece's (M, L) per query head, over the warps
      float M = -INFINITY;
#pragma unroll
      for (int wq = 0; wq < kWarps; ++wq) M = fmaxf(M, sML[(wq * kMaxGroup + tid) * 2]);
      float L = 0.f;
#pragma unroll
      for (int wq = 0; wq < kWarps; ++wq) {
        const float mw = sML[(wq * kMaxGroup + tid) * 2];
        if (mw != -INFINITY) L += sML[(wq * kMaxGroup + tid) * 2 + 1] * exp2f(mw - M);
      }
      sFin[2 * tid] = M;
      sFin[2 * tid + 1] = single ? 1.f / L : L;
    }
    __syncthreads();
    // output or partial: thread tid writes query head tid / 16, dimensions 8 (tid % 16) .. +7
    // (two 16-byte stores); with fewer than 128 threads the loop covers the rest
    for (int e = tid; e < kMaxGroup * 16; e += kAttendThreads) {
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
          float* piece = w.partials + ((size_t)blockIdx.x + hd) * kPartFloats;
          dst = reinterpret_cast<float4*>(piece + jq * kHeadDim + d0);
          if ((e & 15) == 0) {
            piece[kPartO + jq] = sFin[2 * jq];
            piece[kPartO + kMaxGroup + jq] = sFin[2 * jq + 1];
          }
        }
        dst[0] = o0;
        dst[1] = o1;
      }
    }
    if (tid == 0) {  // merge_kernel reads the head's piece range (CTAs first .. last)
      if (first_piece) w.head_pieces[hd].x = (int)blockIdx.x;
      if (last_piece) w.head_pieces[hd].y = (int)blockIdx.x;
      if (a.sel_count && first_piece) a.sel_count[hd] = len;
    }
    __syncthreads();  // sComb is reused by the next piece
  }
  cp_async_wait<0>();  // nothing may land in shared memory after the CTA exits
}

// Combines the pieces of every head that the attention launch split over several CTAs.
// Unit u = (head hd, query head jq of the group, quarter qtr of the 128 dimensions); one CTA of
// kMergeThreads threads per unit. With M = max_i m_i and f_i = 2^(m_i - M) over the pieces
// i = 0 .. n-1 of the head (in CTA order):  out[jq][d] = sum_i f_i O_i[jq][d] / sum_i f_i l_i.
// Every sum runs in a fixed order (per-thread strides, then fixed shuffle and shared-memory
// trees), so the result does not depend on timing. The first kMergeRows * kMergeRegs pieces'
// O rows are loaded before the maxima are known, so m, l and O arrive in one round trip.
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const LayerArgs a,
                                                              const Workspace w) {
  __shared__ float sF[kMaxPieces];  // m_i, then the factor f_i
  __shared__ float sL[kMaxPieces];
  __shared__ float red[kMergeThreads / 32];
  __shared__ float4 racc[kMergeThreads / 32][8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = tid >> 3, c = tid & 7;  // piece row, 16-byte column of the 32-dim quarter
  const int nheads = a.B * a.Hkv;
  const int units = merge_units(nheads, a.G);
  // The pieces of a head follow from the split of the concatenated token sets, which depends
  // only on the head sizes: for layers of at most kMergeDirectHeads heads they are computed
  // here, before the wait for the attention launch, from the lengths and the selection sizes.
  // Both were complete before the attention launch passed its own wait, and this launch is
  // only released by the attention launch after that point. Larger layers read the ranges the
  // attention launch recorded, after the wait.
  __shared__ long long mOff[kMergeDirectHeads + 1];
  __shared__ long long mSplit[2];  // T and P of the attention launch's split
  const bool direct = nheads <= kMergeDirectHeads;
  if (direct && warp == 0) {  // the attention launch's split of the same sizes
    for (int i = lane; i < nheads; i += 32) mOff[i + 1] = head_len(a, w, i, nullptr);
    __syncwarp();
    const HeadSplit sp = split_heads(mOff, nheads, a.attend_grid, -1, lane);
    if (lane == 0) {
      mSplit[0] = sp.T;
      mSplit[1] = sp.P;
    }
  }
  __syncthreads();
  pdl_wait();
  pdl_launch_dependents();
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int hd = u / (a.G * 4), jq = (u >> 2) % a.G, qtr = u & 3;
    int c_first, n;
    if (direct) {
      if (mOff[hd + 1] == mOff[hd]) continue;  // a tiny head: its own CTA wrote it out
      const long long T = mSplit[0], P = mSplit[1];
      c_first = (int)cta_of(mOff[hd], T, P);
      n = (int)cta_of(mOff[hd + 1] - 1, T, P) - c_first + 1;
    } else {
      const int2 pr = __ldcg(w.head_pieces + hd);
      c_first = pr.x;
      n = pr.y - pr.x + 1;
    }
    if (n <= 1) continue;  // written by the attention launch
    const float* base = w.partials + (size_t)(c_first + hd) * kPartFloats;
    const int col = jq * kHeadDim + qtr * 32 + c * 4;
    float4 ov[kMergeRegs];
#pragma unroll
    for (int k = 0; k < kMergeRegs; ++k) {
      const int i = r + k * kMergeRows;
      ov[k] = (i < n) ? __ldcg(reinterpret_cast<const float4*>(base + (size_t)i * kPartFloats + col))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mx = -INFINITY;
    for (int i = tid; i < n; i += kMergeThreads) {
      const float m = __ldcg(base + (size_t)i * kPartFloats + kPartO + jq);
      sL[i] = __ldcg(base + (size_t)i * kPartFloats + kPartO + kMaxGroup + jq);
      sF[i] = m;
      mx = fmaxf(mx, m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float M = red[0];
#pragma unroll
    for (int k = 1; k < kMergeThreads / 32; ++k) M = fmaxf(M, red[k]);
    float ls = 0.f;
    for (int i = tid; i < n; i += kMergeThreads) {
      const float f = exp2f(sF[i] - M);
      sF[i] = f;
      ls += sL[i] * f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    __syncthreads();  // every thread has read red[] (the maxima)
    if (lane == 0) red[warp] = ls;
    __syncthreads();  // red[] holds the l sums, sF[] the factors
    float L = 0.f;
#pragma unroll
    for (int k = 0; k < kMergeThreads / 32; ++k) L += red[k];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kMergeRegs; ++k) {
      const int i = r + k * kMergeRows;
      if (i < n) {
        const float f = sF[i];
        acc.x += ov[k].x * f; acc.y += ov[k].y * f; acc.z += ov[k].z * f; acc.w += ov[k].w * f;
      }
    }
    for (int i = r + kMergeRegs * kMergeRows; i < n; i += kMergeRows) {  // long heads only
      const float4 v = __ldcg(reinterpret_cast<const float4*>(base + (size_t)i * kPartFloats + col));
      const float f = sF[i];
      acc.x += v.x * f; acc.y += v.y * f; acc.z += v.z * f; acc.w += v.w * f;
    }
    // rows r of a warp: (tid >> 3) & 3; add them (lanes c, c + 8, c + 16, c + 24), then warps
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) {
      acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
      acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
      acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
      acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
    if (lane < 8) racc[warp][lane] = acc;
    __syncthreads();
    if (tid < 8) {
      float4 o = racc[0][tid];
#pragma unroll
      for (int k = 1; k < kMergeThreads / 32; ++k) {
        const float4 v = racc[k][tid];
        o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w;
      }
      const float inv = 1.f / L;
      const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
      float4* dst = reinterpret_cast<float4*>(
          a.out + ((size_t)b * a.Hq + (size_t)kvh * a.G + jq) * kHeadDim + qtr * 32 + tid * 4);
      *dst = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
    }
    __syncthreads();  // shared arrays are reused by the next unit
  }
}

}  // namespace rtp
