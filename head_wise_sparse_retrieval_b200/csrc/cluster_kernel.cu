// cluster_kernel.cu -- one decode layer whose KV heads are all local heads (sm_100a).
//
// Follows "Full Attention Strikes Back ..." (xllm-io paper review), section 五 测试配置, and the
// gist.science technical summary, Methodology 1: a local head attends over its 4 sink tokens and
// the last 8192 positions,  O_h = sum_{n in T} softmax_T(q^T k_n / sqrt(d_h)) v_n  with
// T = {0 .. sinks-1} U {N-window .. N-1} (all N positions when they meet).
//
// A layer without retrieval heads needs no selection, and every head's set size follows from
// its sequence length. One thread-block cluster of C CTAs (one CTA per SM) takes one (b, KV
// head): CTA rank r attends over ranks [r T / C, (r + 1) T / C) of the head's set with the decode
// attention's tile step (attend_tile.cuh: 16-token tiles gathered by per-warp cp.async
// pipelines, warp MMA with the G query heads as N = 8, online softmax). The CTA's warps merge
// their (m, l, O) through shared memory; the C pieces of the head are merged by the cluster
// itself, in a fixed order: every CTA stores its piece to its slot in global memory, one cluster
// barrier orders the stores before the reads, and rank r reads its share of every piece from L2
// (one round trip) and writes the r-th C-th of the head's G * 128 output values. No merge launch
// follows.
#include <cooperative_groups.h>

#include "attend_tile.cuh"
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace cg = cooperative_groups;

namespace rtp {

namespace {

constexpr int kW = kClusterWarps;
constexpr int kD = kClusterDepth;
constexpr int kT = kW * 32;
constexpr int kElems = kMaxGroup * kHeadDim;  // one head's output values (8 query heads x 128)

// Shared memory: the warps' stages, then each warp's maximum m (log2 domain) and sum l per query
// head. At the end the stages hold the warps' rescaled O for the CTA-level merge.
struct CSmem {
  static constexpr size_t stage_off = 0;
  static constexpr size_t ml_off = (size_t)kW * kD * kWarpStage;  // per warp: m[8], l[8]
  static constexpr size_t total = ml_off + (size_t)kW * kMaxGroup * 2 * 4;
};

// A warp's O in its slot of the stages, rows of kSlotPitch floats: the pitch makes the MMA
// fragment's stores (query heads 2t, 2t + 1 of lanes t = 0..3) fall in different banks.
constexpr int kSlotPitch = kHeadDim + 4;
constexpr int kSlotFloats = kMaxGroup * kSlotPitch;
static_assert((size_t)kW * kSlotFloats * 4 <= CSmem::ml_off, "the warps' O fit in the stages");

}  // namespace

size_t cluster_smem_bytes() { return CSmem::total; }

__global__ void __launch_bounds__(kT, 1) head_cluster_kernel(const LayerArgs a, const Workspace w) {
  extern __shared__ __align__(128) unsigned char smem[];
  float* sML = reinterpret_cast<float*>(smem + CSmem::ml_off);
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int hd = (int)blockIdx.x / C;  // the grid is one cluster per (b, KV head)
  const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // When the caller vouches that the inputs are ready, the wait moves to just before the first
  // store to the pieces' slots, which the launch before may still read; this launch then still
  // completes after its predecessor.
  if (!a.early) pdl_wait();
  int N = __ldg(a.seq_lens + b);
  if (N < 1 || N > a.max_ctx) {  // clamped and reported
    if (tid == 0 && rank == 0) atomicOr(w.status, kDevBadSeqlen);
    N = N < 1 ? 1 : a.max_ctx;
  }
  pdl_launch_dependents();
  const int len = window_len(N, a.window, a.sinks);
  const int r0 = (int)((long long)rank * len / C), r1 = (int)((long long)(rank + 1) * len / C);
  const int nt = (r1 - r0 + kTile - 1) / kTile;  // tiles of this CTA's range
  const int my_n = (nt > warp) ? (nt - warp + kW - 1) / kW : 0;  // tiles warp, warp + kW, ...

  const size_t head = (size_t)b * a.Hkv + kvh;
  const __nv_bfloat16* kbase = a.k_cache + head * (size_t)a.max_ctx * kHeadDim;
  const __nv_bfloat16* vbase = a.v_cache + head * (size_t)a.max_ctx * kHeadDim;
  const uint64_t policy = l2_policy_evict_first();
  const uint32_t my_stages = smem_u32(smem + CSmem::stage_off) + (uint32_t)warp * kD * kWarpStage;
  // tile i of this warp: ranks r0 + 16 (warp + kW i) ...; lane l < 16 gets its token's position
  auto tile_n = [&](int i) { return min(kTile, r1 - (r0 + (warp + kW * i) * kTile)); };
  auto issue = [&](int i) {  // one commit group per tile slot, empty past the warp's tiles
    if (i < my_n) {
      const int n = tile_n(i);
      const int rk = r0 + (warp + kW * i) * kTile + lane;
      const int pos = (lane < n) ? window_pos(rk, N, a.window, a.sinks) : -1;
      gather_tile(my_stages + (uint32_t)(i % kD) * kWarpStage, kbase, vbase, N, pos, n, lane,
                  policy, w.status);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int s = 0; s < kD - 1; ++s) issue(s);
  uint32_t qf[8][2];
  load_q_frag(qf, a.q + ((size_t)b * a.Hq + (size_t)kvh * a.G) * kHeadDim, a.G, lane);
  TileAcc st;
  st.init();
  const float scale_log2 = a.attn_scale_log2;
  for (int i = 0; i < my_n; ++i) {
    issue(i + kD - 1);
    cp_async_wait<kD - 1>();  // tile i landed
    __syncwarp();
    attend_tile(my_stages + (uint32_t)(i % kD) * kWarpStage, qf, tile_n(i), scale_log2, lane, st);
    __syncwarp();  // the stage is refilled kD - 1 tiles later
  }
  cp_async_wait<0>();  // the trailing empty groups; the stages are free from here

  // ---- the CTA's piece: merge the warps ------------------------------------------------------
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
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
  {  // each warp writes its O, rescaled to the CTA maximum, into its own slot of the stages
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int wq = 0; wq < kW; ++wq) {
      M0 = fmaxf(M0, sML[(wq * kMaxGroup + 2 * t) * 2]);
      M1 = fmaxf(M1, sML[(wq * kMaxGroup + 2 * t + 1) * 2]);
    }
    const float f0 = (st.m0 == -INFINITY) ? 0.f : exp2f(st.m0 - M0);  // 0: a warp without tokens
    const float f1 = (st.m1 == -INFINITY) ? 0.f : exp2f(st.m1 - M1);
    float* wo = reinterpret_cast<float*>(smem + CSmem::stage_off) + (size_t)warp * kSlotFloats;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      wo[(2 * t) * kSlotPitch + 16 * mt + g] = st.acc[mt][0] * f0;
      wo[(2 * t + 1) * kSlotPitch + 16 * mt + g] = st.acc[mt][1] * f1;
      wo[(2 * t) * kSlotPitch + 16 * mt + g + 8] = st.acc[mt][2] * f0;
      wo[(2 * t + 1) * kSlotPitch + 16 * mt + g + 8] = st.acc[mt][3] * f1;
    }
  }
  __syncthreads();  // every warp's slot is written

  // ---- the head: merge the cluster's pieces through global memory -------------------------
  // Each CTA stores its piece (m, l, O) in its slot of cluster_parts; after one cluster barrier
  // (release / acquire at cluster scope) rank r reads its share of every piece from L2 in one
  // round trip. In early mode the launch before may still read the slots: wait for it first.
  if (a.early) pdl_wait();
  float* part = w.cluster_parts + ((size_t)hd * C + rank) * kClusterPartFloats;
  if (tid < kMaxGroup) {  // the piece's (m, l) per query head, over the warps
    float M = -INFINITY;
#pragma unroll
    for (int wq = 0; wq < kW; ++wq) M = fmaxf(M, sML[(wq * kMaxGroup + tid) * 2]);
    float L = 0.f;
#pragma unroll
    for (int wq = 0; wq < kW; ++wq) {
      const float mw = sML[(wq * kMaxGroup + tid) * 2];
      if (mw != -INFINITY) L += sML[(wq * kMaxGroup + tid) * 2 + 1] * exp2f(mw - M);
    }
    part[tid] = M;
    part[kMaxGroup + tid] = L;
  }
  {  // O of the piece: the warps' slots added in warp order, stored to the slot directly
    const float* wo = reinterpret_cast<const float*>(smem + CSmem::stage_off);
    for (int e = tid; e < kElems; e += kT) {
      const int at = (e / kHeadDim) * kSlotPitch + e % kHeadDim;
      float v = 0.f;
#pragma unroll
      for (int wq = 0; wq < kW; ++wq) v += wo[(size_t)wq * kSlotFloats + at];
      part[2 * kMaxGroup + e] = v;
    }
  }
  cluster.sync();  // every piece of the head is in global memory
  {
    // rank r writes output values [r E / C, (r + 1) E / C) of the G * 128 (E) of the head, at
    // most 8 * 128 / kMinCluster = kT of them: one per thread, with M = max_c m_c and
    // f_c = 2^(m_c - M): out = sum_c f_c O_c / sum_c f_c l_c, the pieces in rank order
    static_assert(kMaxGroup * kHeadDim / kMinCluster <= kT, "one output per thread");
    const int E = a.G * kHeadDim;
    const int e0 = (int)((long long)rank * E / C), e1 = (int)((long long)(rank + 1) * E / C);
    const int e = e0 + tid;
    if (e < e1) {
      const int jq = e / kHeadDim;
      const float* head_parts = w.cluster_parts + (size_t)hd * C * kClusterPartFloats;
      float oc[kMaxCluster], mc[kMaxCluster], lc[kMaxCluster];
#pragma unroll
      for (int c = 0; c < kMaxCluster; ++c) {  // every load in flight together
        const float* pc = head_parts + (size_t)c * kClusterPartFloats;
        const bool in = c < C;
        oc[c] = in ? __ldcg(pc + 2 * kMaxGroup + e) : 0.f;
        mc[c] = in ? __ldcg(pc + jq) : -INFINITY;
        lc[c] = in ? __ldcg(pc + kMaxGroup + jq) : 0.f;
      }
      float M = -INFINITY;
#pragma unroll
      for (int c = 0; c < kMaxCluster; ++c) M = fmaxf(M, mc[c]);
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int c = 0; c < kMaxCluster; ++c) {
        if (mc[c] == -INFINITY) continue;  // a CTA without tokens, or past the cluster
        const float f = exp2f(mc[c] - M);
        L += lc[c] * f;
        O += oc[c] * f;
      }
      a.out[((size_t)b * a.Hq + (size_t)kvh * a.G) * kHeadDim + e] = O / L;
    }
    if (tid == 0 && rank == 0 && a.sel_count) a.sel_count[hd] = len;
  }
}

}  // namespace rtp
