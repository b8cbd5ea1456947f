// rtp_kernels.h -- launch arguments shared by the host code and the kernels of librtp.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace rtp {

constexpr int kMaxKvHeads = 256;

// Device workspace owned by a handle. Slot = b * nret + j for the j-th retrieval KV head of
// the current layer (the workspace is sized for nret = Hkv).
struct Workspace {
  float* scores;                  // [slots][max_ctx]        scaled indexer scores
  float* chunk_max;               // [slots][n_score_chunks] per-CTA maxima of the scores
  unsigned long long* hist;       // [slots][256]            fixed-point (2^-40) bin masses
  float* s_max;                   // [slots]
  int* bstar;                     // [slots]
  unsigned long long* mass_total; // [slots]                 C_0 in fixed point
  int* sel_idx;                   // [slots][max_ctx]        selected positions, per 8192-chunk
  int* chunk_cnt;                 // [slots][n_sel_chunks]   selected per chunk
  int* chunk_off;                 // [slots][n_sel_chunks+1] exclusive prefix of chunk_cnt
  int* sel_total;                 // [slots]                 |S|
  int* sel_n;                     // [slots]                 N the selection was made over
  unsigned* ticket_hist;          // [slots]
  unsigned* ticket_compact;       // [slots]
  unsigned* ticket_attend;        // [B*Hkv]
  float* partials;                // [(attend_ctas + B*Hkv)][8][2 + 128]
  unsigned* status;               // [1] RTP_DEV_* bits
  int n_score_chunks;             // ceil(max_ctx / kScoreChunk)
  int n_sel_chunks;               // ceil(max_ctx / kSelChunk)
};

struct LayerArgs {
  const __nv_bfloat16* q;         // [B][Hq][128]
  const __half* q_idx;            // [B][Hkv][16]
  const __nv_bfloat16* k_cache;   // [B][Hkv][max_ctx][128]
  const __nv_bfloat16* v_cache;   // [B][Hkv][max_ctx][128]
  const __half* k_idx;            // [B][Hkv][max_ctx][16]
  const int* seq_lens;            // [B]
  float* out;                     // [B][Hq][128]
  int* sel_count;                 // [B][Hkv] or nullptr
  int B, Hq, Hkv, G, max_ctx, window, sinks, nret;
  int dense;                      // every head attends over all N tokens
  float top_p, idx_scale, attn_scale_log2, bin_scale;
  short ret_kvh[kMaxKvHeads];     // KV head of retrieval index j (j < nret)
  short slot_of_kvh[kMaxKvHeads]; // retrieval index j of KV head kvh, or -1 for a local head
};

// Kernel entry points (defined in select_kernels.cu / attend_kernel.cu).
__global__ void score_kernel(const LayerArgs a, const Workspace w);
__global__ void hist_kernel(const LayerArgs a, const Workspace w);
__global__ void compact_kernel(const LayerArgs a, const Workspace w);
__global__ void attend_kernel(const LayerArgs a, const Workspace w);

constexpr int kAttendConsumerWarps = 4;
constexpr int kAttendThreads = (kAttendConsumerWarps + 1) * 32;
constexpr int kAttendTile = 16 * kAttendConsumerWarps;   // tokens per pipeline stage
constexpr int kAttendStages = 4;
constexpr int kRowBytes = 128 * 2;                       // one K or V row in HBM
constexpr int kRowPitch = kRowBytes + 16;                // padded row in shared memory
constexpr int kMaxAttendHeads = 1024;                    // B * Hkv per layer

size_t attend_smem_bytes(int n_sel_chunks);

}  // namespace rtp
