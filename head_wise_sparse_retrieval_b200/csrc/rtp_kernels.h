// rtp_kernels.h -- launch arguments shared by the host code and the kernels of librtp.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace rtp {

constexpr int kMaxKvHeads = 256;

// Largest cache a handle takes. The selection sums each token's mass exp(s - s_max) in (0, 1]
// as an integer of 2^-40 units (at most 2^40 per token) into 64-bit bins and a 64-bit total,
// so N tokens must satisfy N * 2^40 < 2^64: N <= 2^24 - 1.
constexpr int kMaxCtx = (1 << 24) - 1;

// Device workspace owned by a handle. Slot = b * nret + j for the j-th retrieval KV head of
// the current layer (the workspace is sized for nret = Hkv).
struct Workspace {
  float* scores;                  // [slots][ld]             scaled indexer scores (spill)
  unsigned char* bins;            // [slots][ld]             their histogram bins (spill)
  unsigned* smax_key;             // [slots]                 atomic max of the CTAs' maxima
                                  //                         (float_key); 0 between launches
  unsigned long long* hist;       // [kHistCopies][slots][256] fixed-point (2^-40) bin masses
  float* s_max;                   // [slots]
  int* bstar;                     // [slots]
  unsigned long long* mass_total; // [slots]                 C_0 in fixed point
  int* sel_idx;                   // [slots][ld]             selected positions, ascending
  uint32_t* cta_ge;               // [slots][256][select_ctas] tokens of a CTA in bins >= b
  int* sel_total;                 // [slots]                 |S|
  int* sel_n;                     // [slots]                 N the selection was made over
  unsigned* grid_bar;             // [0]: grid barrier counter of the selection kernel
  float* partials;                // [(attend_ctas + B*Hkv)][kPartFloats]  piece of CTA c, head h at c + h
  int2* head_pieces;              // [B*Hkv]                 first and last attention CTA of a head
  float* cluster_parts;           // [B*Hkv*C][kClusterPartFloats] pieces of the cluster launch
  unsigned* status;               // [1] RTP_DEV_* bits
  int ld;                         // per-slot stride of scores / sel_idx: max_ctx rounded up to 64
};

// Selection-only arguments (kept apart from LayerArgs, which the attention launches share).
struct SelectArgs {
  int top_k;                      // > 0: b* by token count (fixed top-k) instead of mass
  unsigned* hist_cnt;             // [kHistCopies][slots][256] tokens per bin (top-k only)
  unsigned long long wait_ns;     // limit of every grid-barrier wait
  int withhold_cta;               // self-test: CTA that skips its first arrival, else -1
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
  int attend_grid;                // CTAs of the attention launch (the merge derives the split)
  int early;                      // the caller vouches the inputs are complete before the
                                  // preceding launch ends: kernels may read them before waiting
};

// Single-launch layer (fused_kernel.cu): selection, gather and merge in one cooperative launch
// of one CTA per SM. The retrieval slots' tokens are owned in 64-token tiles dealt round-robin
// to the CTAs; a CTA holds at most kFusedCapTiles of them on chip.
constexpr int kFusedWarps = 8;
constexpr int kFusedThreads = kFusedWarps * 32;
constexpr int kFusedOwnTok = 64;                         // tokens per ownership tile
constexpr int kFusedMaxHeads = 64;                       // B * Hkv of a single-launch layer
constexpr int kFusedCapTiles = 448;                      // ownership tiles a CTA keeps on chip
constexpr int kFusedBarWord = 64;                        // its grid_bar word (own cache line)
struct FusedArgs {
  int top_k;                      // > 0: b* by token count (fixed top-k)
  unsigned* hist_cnt;             // [kHistCopies][slots][256] tokens per bin
  unsigned* smax_key;             // [slots] order-preserving key of s_max; 0 between launches
  unsigned long long* sel_bits;   // [slots][ldw] selection mask of each 64-token tile
  float* partials;                // [slots * P + P + B*Hkv][kPartFloats] pieces
  unsigned* bar;                  // grid-barrier counter of this kernel
  unsigned long long wait_ns;     // limit of every grid-barrier wait
  int ldw;                        // per-slot stride of sel_bits (words)
};
__global__ void fused_layer_kernel(const LayerArgs a, const Workspace w, const FusedArgs f);
size_t fused_smem_bytes();

// Layers whose KV heads are all local heads (cluster_kernel.cu): one thread-block cluster of
// up to kMaxCluster CTAs (one per SM) per (b, KV head), its pieces merged through distributed
// shared memory.
constexpr int kClusterWarps = 8;
constexpr int kClusterDepth = 3;                         // cp.async stages per warp
constexpr int kMaxCluster = 16;                          // CTAs of one cluster (non-portable > 8)
constexpr int kMinCluster = 4;                           // below this the split launches serve better
constexpr int kClusterMaxSet = 65536;                    // window + sinks of a cluster layer
constexpr int kClusterPartFloats = 2 * 8 + 8 * 128;      // a cluster CTA's piece: m[8], l[8], O
__global__ void head_cluster_kernel(const LayerArgs a, const Workspace w);
size_t cluster_smem_bytes();

// Prefill (prefill_kernel.cu): attention of every position of a prompt, over all earlier
// positions for retrieval heads (or every head, dense), over sinks + window for local heads.
// Persistent grid; one warp per work item (b, KV head, row).
constexpr int kPrefillWarps = 4;
struct PrefillArgs {
  const __nv_bfloat16* q;         // [B][Hq][t_max][128]
  const __nv_bfloat16* k_cache;   // [B][Hkv][max_ctx][128], rows < T_b hold the prompt
  const __nv_bfloat16* v_cache;
  const int* seq_lens;            // [B] prompt lengths T_b
  float* out;                     // [B][Hq][t_max][128]
  unsigned* status;
  // retrieval KV heads: bit kvh of the 256-bit mask
  unsigned long long ret_bits0, ret_bits1, ret_bits2, ret_bits3;
  int B, Hq, Hkv, G, max_ctx, t_max, window, sinks, dense;
  float attn_scale_log2;
};
__global__ void prefill_kernel(const PrefillArgs a);
size_t prefill_smem_bytes();

// Indexer production at decode (indexer_kernel.cu).
struct IndexerArgs {
  const __nv_bfloat16* q_pre;     // [B][Hq][128]
  const __nv_bfloat16* k_pre;     // [B][Hkv][128]
  const __nv_bfloat16* w_q;       // [Hkv][16][G*128]
  const __nv_bfloat16* w_k;       // [Hkv][16][128]
  const int* seq_lens;            // [B]
  __half* q_idx;                  // [B][Hkv][16]
  __half* k_idx;                  // [B][Hkv][max_ctx][16], row N_b - 1 written
  unsigned* status;
  int Hq, Hkv, G, max_ctx;
  int nsel;                       // KV heads produced, listed in heads[]
  short heads[kMaxKvHeads];
};
__global__ void indexer_kernel(const IndexerArgs x);
constexpr int kIdxWarps = 4;                             // outputs (one per warp) of a CTA
constexpr int kIdxSplit = 16 / kIdxWarps;                // CTAs per (b, KV head): r = 16

// Kernel entry points (defined in select_kernels.cu / attend_kernel.cu).
// Cooperative launches. _onchip: every CTA's range fits in shared memory (no spill code);
// _spill: longer ranges keep the rest of their scores and bins in the global workspace.
__global__ void select_kernel_onchip(const LayerArgs a, const Workspace w, const SelectArgs x);
__global__ void select_kernel_spill(const LayerArgs a, const Workspace w, const SelectArgs x);
__global__ void attend_kernel(const LayerArgs a, const Workspace w);
__global__ void merge_kernel(const LayerArgs a, const Workspace w);

#ifndef RTP_ATTEND_WARPS
#define RTP_ATTEND_WARPS 4
#endif
#ifndef RTP_ATTEND_DEPTH
#define RTP_ATTEND_DEPTH 3
#endif
constexpr int kAttendWarps = RTP_ATTEND_WARPS;           // warps per attention CTA
constexpr int kAttendDepth = RTP_ATTEND_DEPTH;           // cp.async stages per warp
constexpr int kAttendCtasPerSm = 2;                      // resident attention CTAs per SM
constexpr int kAttendThreads = kAttendWarps * 32;
constexpr int kRowBytes = 128 * 2;                       // one K or V row
constexpr int kMaxAttendHeads = 1024;                    // B * Hkv per layer
constexpr int kMaxSelSlots = kMaxAttendHeads;            // retrieval slots per layer
constexpr int kMaxSelectCtasPerSm = 2;                   // resident selection CTAs per SM
// 16-byte key loads a selection thread keeps in flight per batch (two batches are in flight;
// 10 and 12 measured slower on the 1M-context step)
constexpr int kScoreUnroll = 8;
constexpr int kScoreCap = 16384;                         // scores a selection CTA keeps on chip
constexpr int kHistCopies = 8;                           // copies of each slot's histogram
size_t select_smem_bytes(int slots);
constexpr int kMaxPieces = 1024;                         // attention CTAs (pieces of one head)
constexpr int kMergeThreads = 128;
constexpr int kMergeDirectHeads = 64;                    // heads whose pieces the merge derives
// merge units: (head, query head of the group, quarter of the 128 dimensions)
__host__ __device__ inline int merge_units(int nheads, int G) { return nheads * G * 4; }

size_t attend_smem_bytes(int nheads, int batch);
void set_last_error(const char* msg);  // the reason rtp_last_error reports on this thread

// Raises a kernel's cudaFuncAttributeMaxDynamicSharedMemorySize on the current device to at
// least `bytes`, never lowering it. The attribute is one setting per kernel and device for the
// whole process, shared by every handle and by the no-allocation entry point: lowering it for a
// smaller layer would make a larger handle's later launches fail. Thread-safe.
cudaError_t raise_smem_limit(const void* kernel, size_t bytes);

}  // namespace rtp
