// attend_kernel.cu -- exact softmax attention over a token set per KV head (sm_100a).
//
// Follows "Full Attention Strikes Back ..." (xllm-io paper review), section 三, 核心公式 /
// 自适应稀疏注意力:  O_h(m) = sum_{n in S_h(m)} softmax_{S_h(m)}(q^T k_n / sqrt(d_h)) v_n,
// with S_h the selected set of a retrieval head, and section 五 测试配置 / gist.science
// Methodology 1 for local heads (S = 4 sinks U the last 8192 positions).
//
// One persistent launch per layer covers every (b, KV head) of the layer. The token sets of
// all heads are laid end to end (retrieval: |S| selected positions; local: the window set;
// dense mode: all N) and the concatenation is cut into gridDim.x equal ranges, one per CTA
// (split-K, balanced to the token). A CTA walks its range head by head:
//   producer warp   maps each rank to a cache row (selected list / window arithmetic), and
//                   gathers K and V rows (256 B each) into a 4-stage shared-memory ring with
//                   1-D bulk async copies completing on mbarriers (evict-first in L2);
//   4 consumer warps each take 16 tokens of a 64-token stage: S^T = K Q^T and O^T += V^T P^T
//                   on the tensor cores (m16n8k16, bf16 in, fp32 accumulate) with the 8 query
//                   heads of the GQA group as the N=8 dimension, so each fetched row serves the
//                   whole group; online softmax in the log2 domain; P is rounded to bf16 and
//                   transposed in registers (movmatrix) to feed the second MMA.
// At the end of a head's piece the 4 warps merge (m, l, O) through shared memory; a head
// split over several CTAs writes partials, and the last CTA to finish it (atomic ticket, no
// waiting) merges the partials in a fixed order (log-sum-exp combine) and writes the output.
#include "rtp_device.cuh"
#include "rtp_kernels.h"

namespace rtp {

namespace {

constexpr int kStageBytes = kAttendTile * kRowPitch;   // one K (or V) stage
constexpr int kCombFloats = kAttendConsumerWarps * kMaxGroup * kPartStride;

struct SmemLayout {
  static constexpr size_t k_off = 0;
  static constexpr size_t v_off = k_off + (size_t)kAttendStages * kStageBytes;
  static constexpr size_t comb_off = v_off + (size_t)kAttendStages * kStageBytes;
  static constexpr size_t hoff_off = comb_off + (size_t)kCombFloats * 4;
  static constexpr size_t coff_off = hoff_off + (size_t)(kMaxAttendHeads + 1) * 8;
};

__device__ __forceinline__ int window_len(int N, int W, int S) {
  return (N <= W + S) ? N : W + S;
}
__device__ __forceinline__ int window_pos(int r, int N, int W, int S) {
  return (N <= W + S) ? r : (r < S ? r : N - W + (r - S));
}

__device__ __forceinline__ int seq_len_of(const LayerArgs& a, int b) {
  const int n = a.seq_lens[b];
  return n < 1 ? 1 : (n > a.max_ctx ? a.max_ctx : n);
}

// CTA whose range [floor(c T / P), floor((c+1) T / P)) holds position x (0 <= x < T).
__device__ __forceinline__ long long cta_of(long long x, long long T, long long P) {
  return ((x + 1) * P + T - 1) / T - 1;
}

// The segments of this CTA's range, head by head. Producer and consumers run the same walk.
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
  // next non-empty segment: head h, ranks [r0, r1)
  __device__ bool next(int& head, int& r0, int& r1) {
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

}  // namespace

size_t attend_smem_bytes(int n_sel_chunks) {
  return SmemLayout::coff_off + (size_t)(n_sel_chunks + 1) * 4;
}

__global__ void __launch_bounds__(kAttendThreads, 1) attend_kernel(const LayerArgs a,
                                                                   const Workspace w) {
  extern __shared__ __align__(128) unsigned char smem[];
  unsigned char* sK = smem + SmemLayout::k_off;
  unsigned char* sV = smem + SmemLayout::v_off;
  float* sComb = reinterpret_cast<float*>(smem + SmemLayout::comb_off);
  long long* sOff = reinterpret_cast<long long*>(smem + SmemLayout::hoff_off);
  int* sChunkOff = reinterpret_cast<int*>(smem + SmemLayout::coff_off);
  __shared__ __align__(8) uint64_t full_bar[kAttendStages];
  __shared__ __align__(8) uint64_t empty_bar[kAttendStages];
  __shared__ volatile int abort_flag;
  __shared__ int is_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- prologue that touches only shared memory: overlaps the previous kernel (PDL) ----
  {
    uint4* z = reinterpret_cast<uint4*>(smem);
    const int n16 = (int)(SmemLayout::comb_off / 16);
    for (int i = tid; i < n16; i += kAttendThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  if (tid == 0) {
    for (int s = 0; s < kAttendStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kAttendConsumerWarps);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();  // zero fill (generic proxy) before the bulk copies (async proxy)

  pdl_wait();

  // ---- the layer's heads and their token-set lengths --------------------------------------
  const int nheads = a.B * a.Hkv;
  for (int hd = tid; hd < nheads; hd += kAttendThreads) {
    const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
    const int N = seq_len_of(a, b);
    int len;
    if (a.dense) {
      len = N;
    } else if (a.slot_of_kvh[kvh] >= 0) {
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

  const long long T = sOff[nheads];
  const long long P = gridDim.x;
  const long long t0 = (long long)blockIdx.x * T / P;
  const long long t1 = ((long long)blockIdx.x + 1) * T / P;
  if (t0 >= t1) return;

  Walk walk;
  walk.begin(sOff, nheads, t0, t1);
  int hd, r0, r1;

  if (warp == kAttendConsumerWarps) {
    // ================================ producer ================================
    const uint64_t policy = l2_policy_evict_first();
    unsigned it = 0;
    while (walk.next(hd, r0, r1)) {
      const int b = hd / a.Hkv, kvh = hd - b * a.Hkv;
      const int N = seq_len_of(a, b);
      const int j = a.dense ? -1 : a.slot_of_kvh[kvh];
      const int slot = b * a.nret + j;
      int nch = 0;
      const int* sel = nullptr;
      if (j >= 0) {
        nch = (N + kSelChunk - 1) / kSelChunk;
        const int* coff = w.chunk_off + (size_t)slot * (w.n_sel_chunks + 1);
        for (int i = lane; i <= nch; i += 32) sChunkOff[i] = __ldcg(coff + i);
        sel = w.sel_idx + (size_t)slot * a.max_ctx;
        __syncwarp();
      }
      const size_t head = (size_t)b * a.Hkv + kvh;
      const __nv_bfloat16* kbase = a.k_cache + head * (size_t)a.max_ctx * kHeadDim;
      const __nv_bfloat16* vbase = a.v_cache + head * (size_t)a.max_ctx * kHeadDim;

      for (int r = r0; r < r1; r += kAttendTile, ++it) {
        const int n = min(kAttendTile, r1 - r);
        const int stage = it % kAttendStages;
        const unsigned round = it / kAttendStages;
        mbar_wait_bounded(&empty_bar[stage], (round & 1u) ^ 1u, w.status, &abort_flag);

        int pos[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = lane + 32 * u;
          pos[u] = -1;
          if (i < n) {
            const int rank = r + i;
            int p;
            if (j < 0) {
              p = a.dense ? rank : window_pos(rank, N, a.window, a.sinks);
            } else if (rank >= sChunkOff[nch]) {
              p = -1;  // beyond the selected list (cannot happen: |S| >= 1 and len <= |S|)
            } else {
              int lo = 0, hi = nch - 1;  // chunk c with off[c] <= rank < off[c+1]
              while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (sChunkOff[mid] <= rank) lo = mid; else hi = mid - 1;
              }
              p = __ldcg(sel + (size_t)lo * kSelChunk + (rank - sChunkOff[lo]));
            }
            if (p < 0 || p >= N) {
              atomicOr(w.status, kDevBadIndex);
              p = 0;
            }
            pos[u] = p;
          }
        }
        if (lane == 0) mbar_arrive_expect_tx(&full_bar[stage], (unsigned)n * 2u * kRowBytes);
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (pos[u] >= 0) {
            const int i = lane + 32 * u;
            const size_t row = (size_t)pos[u] * kHeadDim;
            bulk_g2s(sK + stage * kStageBytes + i * kRowPitch, kbase + row, kRowBytes,
                     &full_bar[stage], policy);
            bulk_g2s(sV + stage * kStageBytes + i * kRowPitch, vbase + row, kRowBytes,
                     &full_bar[stage], policy);
          }
        }
      }
    }
    return;
  }

  // ================================ consumers ================================
  const int g = lane >> 2, t = lane & 3;  // MMA fragment coordinates
  const float scale_log2 = a.attn_scale_log2;
  // ldmatrix row addresses (byte offsets inside a stage)
  const int k_row = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int k_col = (lane >> 4) * 16;
  const int v_row = (lane & 7) + (lane >> 4) * 8;
  const int v_col = ((lane >> 3) & 1) * 16;
  const int i0 = warp * 16;
  unsigned it = 0;

  while (walk.next(hd, r0, r1)) {
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

    for (int r = r0; r < r1; r += kAttendTile, ++it) {
      const int n = min(kAttendTile, r1 - r);
      const int stage = it % kAttendStages;
      const unsigned round = it / kAttendStages;
      mbar_wait_bounded(&full_bar[stage], round & 1u, w.status, &abort_flag);
      const int nv = n - i0;
      if (nv > 0) {
        const uint32_t kb = smem_u32(sK + stage * kStageBytes + i0 * kRowPitch);
        const uint32_t vb = smem_u32(sV + stage * kStageBytes + i0 * kRowPitch);
        // S^T (16 tokens x 8 heads) = K (16 x 128) . Q^T (128 x 8), two accumulator chains
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t ka = kb + k_row * kRowPitch + k_col;
#pragma unroll
        for (int ks = 0; ks < 8; ks += 2) {
          uint32_t fa[4], fb[4];
          ldmatrix_x4(fa, ka + ks * 32);
          ldmatrix_x4(fb, ka + (ks + 1) * 32);
          mma_bf16_16816(sa, fa, qf[ks][0], qf[ks][1]);
          mma_bf16_16816(sb, fb, qf[ks + 1][0], qf[ks + 1][1]);
        }
        // rows: token g (c0: head 2t, c1: head 2t+1) and token g+8 (c2, c3)
        float x0 = (sa[0] + sb[0]) * scale_log2, x1 = (sa[1] + sb[1]) * scale_log2;
        float x2 = (sa[2] + sb[2]) * scale_log2, x3 = (sa[3] + sb[3]) * scale_log2;
        if (g >= nv) x0 = x1 = -INFINITY;
        if (g + 8 >= nv) x2 = x3 = -INFINITY;
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: token 0 is valid
        const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        const uint32_t p01 = pack_bf16x2(exp2f(x0 - mn0), exp2f(x1 - mn1));
        const uint32_t p23 = pack_bf16x2(exp2f(x2 - mn0), exp2f(x3 - mn1));
        l0 = l0 * al0 + bf16_lo(p01) + bf16_lo(p23);
        l1 = l1 * al1 + bf16_hi(p01) + bf16_hi(p23);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[mt][0] *= al0;
          acc[mt][1] *= al1;
          acc[mt][2] *= al0;
          acc[mt][3] *= al1;
        }
        // P^T as the B operand: transpose the 8x8 (token x head) blocks in registers
        const uint32_t pb0 = movmatrix_trans(p01);
        const uint32_t pb1 = movmatrix_trans(p23);
        // O^T (128 dims x 8 heads) += V^T (128 x 16 tokens) . P^T (16 x 8)
        const uint32_t va = vb + v_row * kRowPitch + v_col;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          uint32_t fv[4];
          ldmatrix_x4_trans(fv, va + mt * 32);
          mma_bf16_16816(acc[mt], fv, pb0, pb1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[stage]);
    }

    // ---- end of this head's piece: merge the 4 warps --------------------------------------
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    {
      float* c0 = sComb + (warp * kMaxGroup + 2 * t) * kPartStride;
      float* c1 = c0 + kPartStride;
      if (g == 0) {
        c0[0] = m0;
        c0[1] = l0;
        c1[0] = m1;
        c1[1] = l1;
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        c0[2 + 16 * mt + g] = acc[mt][0];
        c1[2 + 16 * mt + g] = acc[mt][1];
        c0[2 + 16 * mt + g + 8] = acc[mt][2];
        c1[2 + 16 * mt + g + 8] = acc[mt][3];
      }
    }
    named_barrier_sync(1, kAttendConsumerWarps * 32);

    const long long hb = sOff[hd], he = sOff[hd + 1];
    const long long c_first = cta_of(hb, T, P), c_last = cta_of(he - 1, T, P);
    const bool single = (c_first == c_last);
    const int d = tid;  // 0..127: one output dimension per consumer thread
    float* part = w.partials + ((size_t)blockIdx.x + hd) * kMaxGroup * kPartStride;
    for (int jq = 0; jq < a.G; ++jq) {
      float M = -INFINITY;
#pragma unroll
      for (int wq = 0; wq < kAttendConsumerWarps; ++wq)
        M = fmaxf(M, sComb[(wq * kMaxGroup + jq) * kPartStride]);
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int wq = 0; wq < kAttendConsumerWarps; ++wq) {
        const float* c = sComb + (wq * kMaxGroup + jq) * kPartStride;
        const float f = exp2f(c[0] - M);
        L += c[1] * f;
        O += c[2 + d] * f;
      }
      if (single) {
        a.out[((size_t)b * a.Hq + (size_t)kvh * a.G + jq) * kHeadDim + d] = O / L;
      } else {
        float* pj = part + jq * kPartStride;
        if (d == 0) {
          pj[0] = M;
          pj[1] = L;
        }
        pj[2 + d] = O;
      }
    }
    if (a.sel_count && blockIdx.x == c_first && tid == 0) a.sel_count[hd] = (int)(he - hb);
    if (!single) {
      __threadfence();
      named_barrier_sync(1, kAttendConsumerWarps * 32);
      if (tid == 0)
        is_last = (atomicAdd(w.ticket_attend + hd, 1u) == (unsigned)(c_last - c_first));
      named_barrier_sync(1, kAttendConsumerWarps * 32);
      if (is_last) {
        __threadfence();
        const int npieces = (int)(c_last - c_first + 1);
        for (int jq = 0; jq < a.G; ++jq) {
          float M = -INFINITY;
          for (int pc = 0; pc < npieces; ++pc) {
            const float* pp = w.partials +
                              ((size_t)(c_first + pc) + hd) * kMaxGroup * kPartStride +
                              jq * kPartStride;
            M = fmaxf(M, __ldcg(pp));
          }
          float L = 0.f, O = 0.f;
          for (int pc = 0; pc < npieces; ++pc) {
            const float* pp = w.partials +
                              ((size_t)(c_first + pc) + hd) * kMaxGroup * kPartStride +
                              jq * kPartStride;
            const float f = exp2f(__ldcg(pp) - M);
            L += __ldcg(pp + 1) * f;
            O += __ldcg(pp + 2 + d) * f;
          }
          a.out[((size_t)b * a.Hq + (size_t)kvh * a.G + jq) * kHeadDim + d] = O / L;
        }
        if (tid == 0) w.ticket_attend[hd] = 0u;
      }
    }
    named_barrier_sync(1, kAttendConsumerWarps * 32);  // sComb is reused by the next piece
  }
}

}  // namespace rtp
