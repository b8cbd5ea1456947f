// rtp_api.cu -- host side of librtp: argument checks, workspace, launches (C-ABI of rtp.h).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "rtp.h"
#include "rtp_device.cuh"
#include "rtp_kernels.h"

using namespace rtp;

struct rtp_handle {
  rtp_config cfg;
  int device = 0;
  int num_sms = 0;
  int G = 0;
  int attend_grid = 0;
  int select_grid = 0;
  size_t select_smem = 0;
  size_t attend_smem = 0;
  void* ws_mem = nullptr;
  size_t ws_bytes = 0;
  Workspace ws{};
  unsigned* hist_cnt = nullptr;  // selection token counts per bin (fixed top-k)
  // single-launch layers (fused_layer_kernel): one CTA per SM, when B * Hkv <= kFusedMaxHeads
  bool fused_ok = false;
  int fused_grid = 0;
  size_t fused_smem = 0;
  FusedArgs fx{};
  int prefill_grid = 0;  // persistent prefill launch: every CTA resident at once
  // layers without retrieval heads: one cluster of cluster_size CTAs per (b, KV head), or 0
  int cluster_size = 0;
  size_t cluster_smem = 0;
  // staging for rtp_decode_step_host
  void* stage_q = nullptr;
  void* stage_qidx = nullptr;
  int* stage_seq = nullptr;
  float* stage_out = nullptr;
  // bookkeeping of the last rtp_decode_step, for the debug getters
  bool last_valid = false;
  cudaStream_t last_stream = nullptr;
  int last_nret = 0;
  bool last_fused = false;  // the selection is in the masks, not the position lists
  short last_slot_of_kvh[kMaxKvHeads];
  // rtp_decode_step_host replays the layer sequence as a CUDA graph, captured once per
  // (layer count, p, cache pointers, masks) on a stream of the handle
  cudaStream_t cap_stream = nullptr;
  cudaGraphExec_t step_exec = nullptr;
  int step_layers = 0;
  float step_p = 0.f;
  std::vector<const void*> step_ptrs;
  std::vector<uint8_t> step_masks;
  // NVTX ranges around each call's launches (rtp_nvtx_enable)
  bool nvtx = false;
  // kernel profiling (rtp_profile_enable)
  bool prof = false;
  std::vector<cudaEvent_t> prof_ev;   // 2 per launch
  std::vector<int> prof_kind;
  int prof_used = 0;
  bool prof_overflow = false;
};

namespace {

thread_local char g_err[256] = "";

rtp_status fail(rtp_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return s;
}

rtp_status ok() {
  g_err[0] = '\0';
  return RTP_OK;
}

rtp_status cuda_fail(cudaError_t e, const char* what) {
  return fail(RTP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

rtp_status check_config(const rtp_config* c) {
  if (!c) return fail(RTP_ERR_INVALID_ARG, "config is NULL");
  if (c->num_layers < 1) return fail(RTP_ERR_INVALID_ARG, "num_layers must be >= 1");
  if (c->batch < 1) return fail(RTP_ERR_INVALID_ARG, "batch must be >= 1");
  if (c->num_kv_heads < 1 || c->num_kv_heads > kMaxKvHeads)
    return fail(RTP_ERR_INVALID_ARG, "num_kv_heads must be in [1, %d]", kMaxKvHeads);
  if (c->num_q_heads < 1 || c->num_q_heads % c->num_kv_heads != 0)
    return fail(RTP_ERR_INVALID_ARG, "num_q_heads must be a positive multiple of num_kv_heads");
  if ((long long)c->batch * c->num_kv_heads > kMaxAttendHeads)
    return fail(RTP_ERR_UNSUPPORTED, "batch * num_kv_heads must be <= %d", kMaxAttendHeads);
  const int G = c->num_q_heads / c->num_kv_heads;
  if (G > kMaxGroup) return fail(RTP_ERR_UNSUPPORTED, "GQA group size %d > %d", G, kMaxGroup);
  if (c->head_dim != kHeadDim) return fail(RTP_ERR_UNSUPPORTED, "head_dim must be 128");
  if (c->idx_dim != kIdxDim) return fail(RTP_ERR_UNSUPPORTED, "idx_dim must be 16");
  if (c->num_bins != kBins) return fail(RTP_ERR_UNSUPPORTED, "num_bins must be 256");
  if (c->max_ctx < 1 || c->max_ctx > kMaxCtx)
    return fail(RTP_ERR_INVALID_ARG,
                "max_ctx must be in [1, 2^24 - 1] (the 64-bit fixed-point mass sums)");
  if (c->window < 1) return fail(RTP_ERR_INVALID_ARG, "window must be >= 1");
  if (c->sinks < 0) return fail(RTP_ERR_INVALID_ARG, "sinks must be >= 0");
  if (c->window > (1 << 28) || c->sinks > (1 << 28))
    return fail(RTP_ERR_INVALID_ARG, "window and sinks must be <= 2^28");
  if (!(c->idx_range > 0.f) || !std::isfinite(c->idx_range))
    return fail(RTP_ERR_INVALID_ARG, "idx_range must be finite and > 0");
  if (!(c->idx_scale > 0.f) || !std::isfinite(c->idx_scale))
    return fail(RTP_ERR_INVALID_ARG, "idx_scale must be finite and > 0");
  if (!(c->attn_scale > 0.f) || !std::isfinite(c->attn_scale))
    return fail(RTP_ERR_INVALID_ARG, "attn_scale must be finite and > 0");
  return RTP_OK;
}

struct WsPlan {
  size_t off[21];
  size_t total;
};

// Byte offsets of the workspace arrays (each 256-byte aligned).
WsPlan plan_workspace(const rtp_config* c, int attend_grid, int select_grid, int fused_grid,
                      int cluster_ctas) {
  const size_t slots = (size_t)c->batch * c->num_kv_heads;
  const size_t nmax = round_up((size_t)c->max_ctx, 64);  // per-slot stride (16-byte loads)
  const bool fused = slots <= (size_t)kFusedMaxHeads;
  const size_t sizes[] = {
      slots * nmax * 4,                      // 0 scores
      slots * 4,                             // 1 smax_key
      (size_t)kHistCopies * slots * kBins * 8,  // 2 hist
      slots * 4,                             // 3 s_max
      slots * 4,                             // 4 bstar
      slots * 8,                             // 5 mass_total
      slots * nmax * 4,                      // 6 sel_idx
      slots * (size_t)select_grid * kBins * 4,  // 7 cta_ge
      slots * nmax,                          // 8 bins
      slots * 4,                             // 9 sel_total
      slots * 4,                             // 10 sel_n
      (size_t)(2 + (4 * kMaxAttendHeads + 15) / 16) * 4,  // 11 grid_bar
      4,                                     // 12 (unused)
      slots * 8,                             // 13 head_pieces
      ((size_t)attend_grid + slots) * kPartFloats * 4,  // 14 partials
      256,                                   // 15 status
      (size_t)kHistCopies * slots * kBins * 4,  // 16 hist_cnt
      fused ? slots * 4 : 0,                 // 17 smax_key
      fused ? slots * (nmax / 64) * 8 : 0,   // 18 sel_bits
      fused ? (slots * fused_grid + fused_grid + slots) * kPartFloats * 4 : 0,  // 19 pieces
      (size_t)cluster_ctas * kClusterPartFloats * 4,  // 20 cluster_parts (B*Hkv*C <= #SMs)
  };
  WsPlan p{};
  size_t at = 0;
  for (size_t i = 0; i < sizeof sizes / sizeof sizes[0]; ++i) {
    p.off[i] = at;
    at = round_up(at + sizes[i], 256);
  }
  p.total = at;
  return p;
}

template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel k, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       bool cooperative, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

rtp_status check_io(const rtp_handle* h, const rtp_layer_io* io, bool need_idx) {
  if (!io) return fail(RTP_ERR_INVALID_ARG, "io is NULL");
  if (!io->q || !io->k_cache || !io->v_cache || !io->seq_lens || !io->out)
    return fail(RTP_ERR_INVALID_ARG, "q, k_cache, v_cache, seq_lens and out must be non-NULL");
  if (!aligned16(io->q) || !aligned16(io->k_cache) || !aligned16(io->v_cache) ||
      !aligned16(io->out))
    return fail(RTP_ERR_INVALID_ARG, "q, k_cache, v_cache and out must be 16-byte aligned");
  if (((uintptr_t)io->seq_lens & 3u) || ((uintptr_t)io->sel_count & 3u))
    return fail(RTP_ERR_INVALID_ARG, "seq_lens and sel_count must be 4-byte aligned");
  if (need_idx) {
    if (!io->q_idx || !io->k_idx)
      return fail(RTP_ERR_INVALID_ARG, "q_idx and k_idx are required for retrieval heads");
    if (!aligned16(io->q_idx) || !aligned16(io->k_idx))
      return fail(RTP_ERR_INVALID_ARG, "q_idx and k_idx must be 16-byte aligned");
    if (io->top_k < 0) return fail(RTP_ERR_INVALID_ARG, "top_k must be >= 0");
    if (io->top_k == 0 && !(io->top_p > 0.f && io->top_p <= 1.f))
      return fail(RTP_ERR_INVALID_ARG, "top_p must be in (0, 1]");
  }
  (void)h;
  return RTP_OK;
}

LayerArgs make_args(const rtp_handle* h, const rtp_layer_io* io) {
  LayerArgs a;
  memset(&a, 0, sizeof a);
  a.q = static_cast<const __nv_bfloat16*>(io->q);
  a.q_idx = static_cast<const __half*>(io->q_idx);
  a.k_cache = static_cast<const __nv_bfloat16*>(io->k_cache);
  a.v_cache = static_cast<const __nv_bfloat16*>(io->v_cache);
  a.k_idx = static_cast<const __half*>(io->k_idx);
  a.seq_lens = io->seq_lens;
  a.out = io->out;
  a.sel_count = io->sel_count;
  a.B = h->cfg.batch;
  a.Hq = h->cfg.num_q_heads;
  a.Hkv = h->cfg.num_kv_heads;
  a.G = h->G;
  a.max_ctx = h->cfg.max_ctx;
  a.window = h->cfg.window;
  a.sinks = h->cfg.sinks;
  a.top_p = io->top_p;
  a.early = io->inputs_ready ? 1 : 0;
  a.idx_scale = h->cfg.idx_scale;
  a.attn_scale_log2 = (float)((double)h->cfg.attn_scale * 1.4426950408889634);
  a.bin_scale = (float)((double)kBins / (double)h->cfg.idx_range);
  for (int k = 0; k < kMaxKvHeads; ++k) a.slot_of_kvh[k] = -1;
  return a;
}

constexpr int kProfCapacity = 1024;

// Launches one kernel, bracketed by profiling events when the handle has profiling enabled.
template <typename Kernel, typename... Args>
cudaError_t launch_one(rtp_handle* h, int kind, Kernel k, dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, bool cooperative, Args... args) {
  const bool prof = h->prof && h->prof_used < kProfCapacity;
  if (h->prof && !prof) h->prof_overflow = true;
  if (prof) cudaEventRecord(h->prof_ev[2 * h->prof_used], s);
  cudaError_t e = launch_pdl(k, grid, block, smem, s, cooperative, args...);
  if (prof && e == cudaSuccess) {
    cudaEventRecord(h->prof_ev[2 * h->prof_used + 1], s);
    h->prof_kind[h->prof_used++] = kind;
  }
  return e;
}

// Whether the layer fits the single-launch kernel: B * Hkv within its tables, and the ownership
// tiles of the worst case (every N_b = max_ctx) within each CTA's on-chip share.
bool fused_fits(const rtp_handle* h, const LayerArgs& a) {
  if (!h->fused_ok || a.dense) return false;
  const long long tiles =
      (long long)a.B * a.nret * ((a.max_ctx + kFusedOwnTok - 1) / kFusedOwnTok);
  return (tiles + h->fused_grid - 1) / h->fused_grid <= kFusedCapTiles;
}

rtp_status enqueue_fused(rtp_handle* h, const LayerArgs& a, cudaStream_t s, int top_k) {
  if (!fused_fits(h, a))
    return fail(RTP_ERR_UNSUPPORTED,
                "single launch: needs B*Hkv <= %d and B*nret*ceil(max_ctx/64) <= %d*%d",
                kFusedMaxHeads, h->fused_grid, kFusedCapTiles);
  FusedArgs f = h->fx;
  f.top_k = top_k;
  const cudaError_t e = launch_one(h, 3, fused_layer_kernel, dim3(h->fused_grid),
                                   dim3(kFusedThreads), h->fused_smem, s, true, a, h->ws, f);
  return e == cudaSuccess ? RTP_OK : cuda_fail(e, "fused_layer_kernel launch");
}

// A launch of head_cluster_kernel: one cluster of h->cluster_size CTAs per (b, KV head), with
// the programmatic-dependent-launch attribute of the other launches.
cudaError_t launch_cluster(rtp_handle* h, const LayerArgs& a, cudaStream_t s) {
  const bool prof = h->prof && h->prof_used < kProfCapacity;
  if (h->prof && !prof) h->prof_overflow = true;
  if (prof) cudaEventRecord(h->prof_ev[2 * h->prof_used], s);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(a.B * a.Hkv * h->cluster_size));
  cfg.blockDim = dim3(kClusterWarps * 32);
  cfg.dynamicSmemBytes = h->cluster_smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)h->cluster_size;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, head_cluster_kernel, a, h->ws);
  if (prof && e == cudaSuccess) {
    cudaEventRecord(h->prof_ev[2 * h->prof_used + 1], s);
    h->prof_kind[h->prof_used++] = 1;  // an attention launch (its merge is inside)
  }
  return e;
}

rtp_status enqueue_layer(rtp_handle* h, const LayerArgs& a0, cudaStream_t s, int top_k = 0,
                         unsigned long long wait_ns = kWaitLimitNs, int withhold_cta = -1) {
  cudaError_t e;
  if (!a0.dense && a0.nret == 0 && h->cluster_size > 0) {  // local heads only: one launch
    e = launch_cluster(h, a0, s);
    return e == cudaSuccess ? RTP_OK : cuda_fail(e, "head_cluster_kernel launch");
  }
  if (!a0.dense && a0.nret > 0) {
    SelectArgs x;
    x.top_k = top_k;
    x.hist_cnt = h->hist_cnt;
    x.wait_ns = wait_ns;
    x.withhold_cta = withhold_cta;
    // the ranges are at most ceil(B * nret * max_ctx / grid) tokens: on chip when that fits
    const long long worst = (long long)a0.B * a0.nret * a0.max_ctx;
    const bool fits = (worst + h->select_grid - 1) / h->select_grid <= kScoreCap;
    e = launch_one(h, 0, fits ? select_kernel_onchip : select_kernel_spill, dim3(h->select_grid),
                   dim3(kSelThreads), h->select_smem, s, true, a0, h->ws, x);
    if (e != cudaSuccess) return cuda_fail(e, "select_kernel launch");
  }
  if (withhold_cta >= 0) return RTP_OK;  // self-test: the selection alone
  LayerArgs a = a0;
  a.attend_grid = h->attend_grid;
  e = launch_one(h, 1, attend_kernel, dim3(h->attend_grid), dim3(kAttendThreads), h->attend_smem,
                 s, false, a, h->ws);
  if (e != cudaSuccess) return cuda_fail(e, "attend_kernel launch");
  e = launch_one(h, 2, merge_kernel, dim3(merge_units(a.B * a.Hkv, a.G)), dim3(kMergeThreads),
                 0, s, false, a, h->ws);
  return e == cudaSuccess ? RTP_OK : cuda_fail(e, "merge_kernel launch");
}

// An NVTX range around the launches of one call, when the handle has NVTX enabled (the ranges
// cost nothing without a profiler attached, but stay off by default).
struct NvtxRange {
  bool on;
  NvtxRange(const rtp_handle* h, const char* fmt, int x, int y) : on(h->nvtx) {
    if (!on) return;
    char name[96];
    snprintf(name, sizeof name, fmt, x, y);
    nvtxRangePushA(name);
  }
  ~NvtxRange() {
    if (on) nvtxRangePop();
  }
};

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
    if (prev != dev) cudaSetDevice(dev);
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

}  // namespace

namespace rtp {
// Records the reason returned by rtp_last_error on this thread (used by noalloc.cu).
void set_last_error(const char* msg) { snprintf(g_err, sizeof g_err, "%s", msg); }

cudaError_t raise_smem_limit(const void* kernel, size_t bytes) {
  static std::mutex mu;  // the read and the raise are one step for concurrent callers
  std::lock_guard<std::mutex> lock(mu);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);  // the current device's setting
  if (e != cudaSuccess) return e;
  if (bytes <= (size_t)fa.maxDynamicSharedSizeBytes) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}
}  // namespace rtp

extern "C" {

void rtp_config_default(rtp_config* c, int num_layers, int batch, int num_q_heads,
                        int num_kv_heads, int max_ctx) {
  if (!c) return;
  c->num_layers = num_layers;
  c->batch = batch;
  c->num_q_heads = num_q_heads;
  c->num_kv_heads = num_kv_heads;
  c->head_dim = 128;
  c->idx_dim = 16;
  c->max_ctx = max_ctx;
  c->window = 8192;
  c->sinks = 4;
  c->num_bins = 256;
  c->idx_range = 16.0f;
  c->idx_scale = 0.25f;
  c->attn_scale = (float)(1.0 / std::sqrt(128.0));
}

size_t rtp_workspace_bytes(const rtp_config* cfg) {
  if (check_config(cfg) != RTP_OK) return 0;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return plan_workspace(cfg, sms * kAttendCtasPerSm, sms * kMaxSelectCtasPerSm, sms, sms).total;
}

rtp_status rtp_create(const rtp_config* cfg, int device, rtp_handle** out) {
  if (!out) return fail(RTP_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  rtp_status st = check_config(cfg);
  if (st != RTP_OK) return st;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceCount");
  if (device < 0 || device >= ndev)
    return fail(RTP_ERR_INVALID_ARG, "device %d out of range (%d devices)", device, ndev);
  DeviceGuard guard(device);

  rtp_handle* h = new rtp_handle();
  h->cfg = *cfg;
  h->device = device;
  h->G = cfg->num_q_heads / cfg->num_kv_heads;
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, device);
  h->attend_grid = h->num_sms * kAttendCtasPerSm;  // persistent: every CTA resident
  if (h->attend_grid > kMaxPieces) h->attend_grid = kMaxPieces;

  h->select_smem = select_smem_bytes(cfg->batch * cfg->num_kv_heads);
  e = raise_smem_limit((const void*)select_kernel_onchip, h->select_smem);
  if (e == cudaSuccess) e = raise_smem_limit((const void*)select_kernel_spill, h->select_smem);
  int sel_per_sm = 0, sel_per_sm_spill = 0;
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&sel_per_sm, select_kernel_onchip,
                                                      kSelThreads, h->select_smem);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&sel_per_sm_spill, select_kernel_spill,
                                                      kSelThreads, h->select_smem);
  if (sel_per_sm_spill < sel_per_sm) sel_per_sm = sel_per_sm_spill;  // one grid for both
  if (e != cudaSuccess || sel_per_sm < 1) {
    delete h;
    return e != cudaSuccess ? cuda_fail(e, "occupancy of select_kernel")
                            : fail(RTP_ERR_UNSUPPORTED, "select_kernel does not fit an SM");
  }
  if (sel_per_sm > kMaxSelectCtasPerSm) sel_per_sm = kMaxSelectCtasPerSm;
  h->select_grid = h->num_sms * sel_per_sm;  // cooperative: every CTA resident at once
  h->fused_grid = h->num_sms;  // one CTA per SM
  const WsPlan p = plan_workspace(cfg, h->attend_grid, h->select_grid, h->fused_grid, h->num_sms);
  const size_t L = (size_t)cfg->num_layers, B = (size_t)cfg->batch;
  const size_t q_bytes = L * B * cfg->num_q_heads * kHeadDim * 2;
  const size_t qi_bytes = L * B * cfg->num_kv_heads * kIdxDim * 2;
  const size_t out_bytes = L * B * cfg->num_q_heads * kHeadDim * 4;
  const size_t stage_q_off = p.total;
  const size_t stage_qi_off = round_up(stage_q_off + q_bytes, 256);
  const size_t stage_seq_off = round_up(stage_qi_off + qi_bytes, 256);
  const size_t stage_out_off = round_up(stage_seq_off + B * 4, 256);
  h->ws_bytes = round_up(stage_out_off + out_bytes, 256);

  e = cudaMalloc(&h->ws_mem, h->ws_bytes);
  if (e != cudaSuccess) {
    const size_t bytes = h->ws_bytes;
    delete h;
    cudaGetLastError();
    return fail(RTP_ERR_OOM, "cudaMalloc of %zu workspace bytes failed", bytes);
  }
  e = cudaMemset(h->ws_mem, 0, h->ws_bytes);
  if (e != cudaSuccess) {
    cudaFree(h->ws_mem);
    delete h;
    return cuda_fail(e, "cudaMemset");
  }
  char* base = static_cast<char*>(h->ws_mem);
  Workspace& w = h->ws;
  w.scores = reinterpret_cast<float*>(base + p.off[0]);
  w.smax_key = reinterpret_cast<unsigned*>(base + p.off[1]);
  w.hist = reinterpret_cast<unsigned long long*>(base + p.off[2]);
  w.s_max = reinterpret_cast<float*>(base + p.off[3]);
  w.bstar = reinterpret_cast<int*>(base + p.off[4]);
  w.mass_total = reinterpret_cast<unsigned long long*>(base + p.off[5]);
  w.sel_idx = reinterpret_cast<int*>(base + p.off[6]);
  w.cta_ge = reinterpret_cast<uint32_t*>(base + p.off[7]);
  w.bins = reinterpret_cast<unsigned char*>(base + p.off[8]);
  w.sel_total = reinterpret_cast<int*>(base + p.off[9]);
  w.sel_n = reinterpret_cast<int*>(base + p.off[10]);
  w.grid_bar = reinterpret_cast<unsigned*>(base + p.off[11]);
  w.head_pieces = reinterpret_cast<int2*>(base + p.off[13]);
  w.cluster_parts = reinterpret_cast<float*>(base + p.off[20]);
  w.partials = reinterpret_cast<float*>(base + p.off[14]);
  w.status = reinterpret_cast<unsigned*>(base + p.off[15]);
  h->hist_cnt = reinterpret_cast<unsigned*>(base + p.off[16]);
  h->fx.hist_cnt = h->hist_cnt;
  h->fx.smax_key = reinterpret_cast<unsigned*>(base + p.off[17]);
  h->fx.sel_bits = reinterpret_cast<unsigned long long*>(base + p.off[18]);
  h->fx.partials = reinterpret_cast<float*>(base + p.off[19]);
  h->fx.bar = w.grid_bar + kFusedBarWord;
  h->fx.wait_ns = kWaitLimitNs;
  h->fx.ldw = (int)(round_up((size_t)cfg->max_ctx, 64) / 64);
  w.ld = (int)round_up((size_t)cfg->max_ctx, 64);
  h->stage_q = base + stage_q_off;
  h->stage_qidx = base + stage_qi_off;
  h->stage_seq = reinterpret_cast<int*>(base + stage_seq_off);
  h->stage_out = reinterpret_cast<float*>(base + stage_out_off);

  h->attend_smem = attend_smem_bytes(cfg->batch * cfg->num_kv_heads, cfg->batch);
  int max_optin = 0;
  cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (h->attend_smem + 4096 > (size_t)max_optin / kAttendCtasPerSm) {
    cudaFree(h->ws_mem);
    delete h;
    return fail(RTP_ERR_UNSUPPORTED, "max_ctx too large for the attention kernel's shared memory");
  }
  e = raise_smem_limit((const void*)attend_kernel, h->attend_smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(attend_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) {
    cudaFree(h->ws_mem);
    delete h;
    return cuda_fail(e, "cudaFuncSetAttribute(attend_kernel)");
  }
  if ((long long)cfg->batch * cfg->num_kv_heads <= kFusedMaxHeads &&
      fused_smem_bytes() <= (size_t)max_optin) {
    h->fused_smem = fused_smem_bytes();
    int per_sm = 0;
    e = raise_smem_limit((const void*)fused_layer_kernel, h->fused_smem);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused_layer_kernel,
                                                        kFusedThreads, h->fused_smem);
    if (e != cudaSuccess) {
      cudaFree(h->ws_mem);
      delete h;
      return cuda_fail(e, "cudaFuncSetAttribute(fused_layer_kernel)");
    }
    h->fused_ok = per_sm >= 1;  // the grid is one CTA per SM, all resident at once
  }
  {  // layers of local heads only: the largest cluster (kMinCluster .. kMaxCluster CTAs, one
     // per SM) of which B * Hkv fit at once (else the largest of which one fits), when the SMs
     // are enough for B * Hkv such clusters
    const int nheads = cfg->batch * cfg->num_kv_heads;
    int c = h->num_sms / nheads;
    if (c > kMaxCluster) c = kMaxCluster;
    h->cluster_smem = cluster_smem_bytes();
    if (c >= kMinCluster && cfg->window + cfg->sinks <= kClusterMaxSet &&
        h->cluster_smem <= (size_t)max_optin) {
      e = raise_smem_limit((const void*)head_cluster_kernel, h->cluster_smem);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(head_cluster_kernel,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      for (; e == cudaSuccess && c >= kMinCluster; --c) {
        cudaLaunchConfig_t lc = {};
        lc.gridDim = dim3((unsigned)(nheads * c));
        lc.blockDim = dim3(kClusterWarps * 32);
        lc.dynamicSmemBytes = h->cluster_smem;
        cudaLaunchAttribute at;
        at.id = cudaLaunchAttributeClusterDimension;
        at.val.clusterDim.x = (unsigned)c;
        at.val.clusterDim.y = 1;
        at.val.clusterDim.z = 1;
        lc.attrs = &at;
        lc.numAttrs = 1;
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, head_cluster_kernel, &lc) != cudaSuccess) {
          cudaGetLastError();  // an unsupported size: try a smaller one
          continue;
        }
        if (nclusters >= 1 && h->cluster_size == 0) h->cluster_size = c;  // the largest that fits
        if (nclusters >= nheads) {  // one wave
          h->cluster_size = c;
          break;
        }
      }
      if (e != cudaSuccess) {
        cudaFree(h->ws_mem);
        delete h;
        return cuda_fail(e, "cudaFuncSetAttribute(head_cluster_kernel)");
      }
    }
  }
  {  // prefill: a persistent grid of as many CTAs as fit at once (at most three per SM)
    int per_sm = 0;
    e = raise_smem_limit((const void*)prefill_kernel, prefill_smem_bytes());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prefill_kernel,
                                                        kPrefillWarps * 32, prefill_smem_bytes());
    if (e != cudaSuccess) {
      cudaFree(h->ws_mem);
      delete h;
      return cuda_fail(e, "cudaFuncSetAttribute(prefill_kernel)");
    }
    h->prefill_grid = h->num_sms * (per_sm < 3 ? per_sm : 3);
  }
  *out = h;
  return ok();
}

rtp_status rtp_destroy(rtp_handle* h) {
  if (!h) return ok();
  DeviceGuard guard(h->device);
  cudaDeviceSynchronize();
  for (cudaEvent_t ev : h->prof_ev) cudaEventDestroy(ev);
  if (h->step_exec) cudaGraphExecDestroy(h->step_exec);
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);

  cudaError_t e = cudaFree(h->ws_mem);
  delete h;
  if (e != cudaSuccess) return cuda_fail(e, "cudaFree");
  return ok();
}

rtp_status rtp_decode_step(rtp_handle* h, int layer, const rtp_layer_io* io, void* stream) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  if (layer < 0 || layer >= h->cfg.num_layers)
    return fail(RTP_ERR_INVALID_ARG, "layer %d outside [0, %d)", layer, h->cfg.num_layers);
  if (!io) return fail(RTP_ERR_INVALID_ARG, "io is NULL");
  if (!io->retrieval_mask) return fail(RTP_ERR_INVALID_ARG, "retrieval_mask is NULL");
  LayerArgs a = make_args(h, io);
  a.nret = 0;
  for (int kvh = 0; kvh < a.Hkv; ++kvh) {
    if (io->retrieval_mask[kvh]) {
      a.slot_of_kvh[kvh] = (short)a.nret;
      a.ret_kvh[a.nret++] = (short)kvh;
    }
  }
  rtp_status st = check_io(h, io, a.nret > 0);
  if (st != RTP_OK) return st;
  DeviceGuard guard(h->device);
  NvtxRange range(h, "rtp_decode_step layer %d (%d retrieval KV heads)", layer, a.nret);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool single = io->single_launch != 0;
  st = single ? enqueue_fused(h, a, s, io->top_k) : enqueue_layer(h, a, s, io->top_k);
  if (st != RTP_OK) return st;
  h->last_fused = single;
  h->last_valid = true;
  h->last_stream = s;
  h->last_nret = a.nret;
  memcpy(h->last_slot_of_kvh, a.slot_of_kvh, sizeof h->last_slot_of_kvh);
  return ok();
}

rtp_status rtp_indexer_append(rtp_handle* h, const rtp_indexer_io* io, void* stream) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  if (!io || !io->q_pre || !io->k_pre || !io->w_q || !io->w_k || !io->seq_lens || !io->q_idx ||
      !io->k_idx)
    return fail(RTP_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(io->q_pre) || !aligned16(io->k_pre) || !aligned16(io->w_q) ||
      !aligned16(io->w_k) || !aligned16(io->q_idx) || !aligned16(io->k_idx) ||
      ((uintptr_t)io->seq_lens & 3u))
    return fail(RTP_ERR_INVALID_ARG, "pointers must be 16-byte aligned (seq_lens 4)");
  IndexerArgs x;
  memset(&x, 0, sizeof x);
  x.q_pre = static_cast<const __nv_bfloat16*>(io->q_pre);
  x.k_pre = static_cast<const __nv_bfloat16*>(io->k_pre);
  x.w_q = static_cast<const __nv_bfloat16*>(io->w_q);
  x.w_k = static_cast<const __nv_bfloat16*>(io->w_k);
  x.seq_lens = io->seq_lens;
  x.q_idx = static_cast<__half*>(io->q_idx);
  x.k_idx = static_cast<__half*>(io->k_idx);
  x.status = h->ws.status;
  x.Hq = h->cfg.num_q_heads;
  x.Hkv = h->cfg.num_kv_heads;
  x.G = h->G;
  x.max_ctx = h->cfg.max_ctx;
  for (int k = 0; k < x.Hkv; ++k)
    if (!io->head_mask || io->head_mask[k]) x.heads[x.nsel++] = (short)k;
  if (x.nsel == 0) return ok();
  DeviceGuard guard(h->device);
  NvtxRange range(h, "rtp_indexer_append (%d x %d KV heads)", h->cfg.batch, x.nsel);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(h->cfg.batch * x.nsel * kIdxSplit);
  cfg.blockDim = dim3(kIdxWarps * 32);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, indexer_kernel, x);
  return e == cudaSuccess ? ok() : cuda_fail(e, "indexer_kernel launch");
}

rtp_status rtp_selftest_wait_timeout(rtp_handle* h, int layer, const rtp_layer_io* io,
                                     uint64_t wait_ns, void* stream) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  if (layer < 0 || layer >= h->cfg.num_layers)
    return fail(RTP_ERR_INVALID_ARG, "layer %d outside [0, %d)", layer, h->cfg.num_layers);
  if (!io || !io->retrieval_mask) return fail(RTP_ERR_INVALID_ARG, "io or its mask is NULL");
  if (wait_ns < 1000 || wait_ns > 1000000000ull)
    return fail(RTP_ERR_INVALID_ARG, "wait_ns must be in [1 us, 1 s]");
  LayerArgs a = make_args(h, io);
  a.nret = 0;
  for (int kvh = 0; kvh < a.Hkv; ++kvh) {
    if (io->retrieval_mask[kvh]) {
      a.slot_of_kvh[kvh] = (short)a.nret;
      a.ret_kvh[a.nret++] = (short)kvh;
    }
  }
  if (a.nret == 0) return fail(RTP_ERR_INVALID_ARG, "the mask has no retrieval head");
  rtp_status st = check_io(h, io, true);
  if (st != RTP_OK) return st;
  DeviceGuard guard(h->device);
  st = enqueue_layer(h, a, static_cast<cudaStream_t>(stream), io->top_k, wait_ns, 0);
  if (st != RTP_OK) return st;
  h->last_valid = false;  // its selection lists are not meaningful
  return ok();
}

rtp_status rtp_prefill(rtp_handle* h, const rtp_prefill_io* io, void* stream) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  if (!io || !io->q || !io->k_cache || !io->v_cache || !io->seq_lens || !io->out ||
      !io->retrieval_mask)
    return fail(RTP_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned16(io->q) || !aligned16(io->k_cache) || !aligned16(io->v_cache) ||
      !aligned16(io->out) || ((uintptr_t)io->seq_lens & 3u))
    return fail(RTP_ERR_INVALID_ARG, "pointers must be 16-byte aligned (seq_lens 4)");
  if (io->t_max < 1 || io->t_max > h->cfg.max_ctx)
    return fail(RTP_ERR_INVALID_ARG, "t_max %d outside [1, max_ctx = %d]", io->t_max,
                h->cfg.max_ctx);
  if ((long long)h->cfg.batch * h->cfg.num_kv_heads * io->t_max > 0x7fffffffLL)
    return fail(RTP_ERR_UNSUPPORTED, "batch * num_kv_heads * t_max must be < 2^31");
  if (h->prefill_grid < 1) return fail(RTP_ERR_UNSUPPORTED, "prefill_kernel does not fit an SM");
  PrefillArgs a;
  memset(&a, 0, sizeof a);
  a.q = static_cast<const __nv_bfloat16*>(io->q);
  a.k_cache = static_cast<const __nv_bfloat16*>(io->k_cache);
  a.v_cache = static_cast<const __nv_bfloat16*>(io->v_cache);
  a.seq_lens = io->seq_lens;
  a.out = io->out;
  a.status = h->ws.status;
  a.B = h->cfg.batch;
  a.Hq = h->cfg.num_q_heads;
  a.Hkv = h->cfg.num_kv_heads;
  a.G = h->G;
  a.max_ctx = h->cfg.max_ctx;
  a.t_max = io->t_max;
  a.window = h->cfg.window;
  a.sinks = h->cfg.sinks;
  a.dense = io->dense ? 1 : 0;
  a.attn_scale_log2 = (float)((double)h->cfg.attn_scale * 1.4426950408889634);
  unsigned long long bits[4] = {0ull, 0ull, 0ull, 0ull};
  for (int k = 0; k < a.Hkv; ++k)
    if (io->retrieval_mask[k]) bits[k >> 6] |= 1ull << (k & 63);
  a.ret_bits0 = bits[0];
  a.ret_bits1 = bits[1];
  a.ret_bits2 = bits[2];
  a.ret_bits3 = bits[3];
  // one warp per (b, KV head, pair of rows)
  const long long warps = (long long)a.B * a.Hkv * ((a.t_max + 1) / 2);
  const long long need = (warps + kPrefillWarps - 1) / kPrefillWarps;
  const int grid = need < h->prefill_grid ? (int)need : h->prefill_grid;
  DeviceGuard guard(h->device);
  NvtxRange range(h, "rtp_prefill (t_max %d, dense %d)", io->t_max, a.dense);
  // a plain launch (no programmatic dependency): the kernel starts after the preceding work on
  // the stream has completed
  prefill_kernel<<<grid, kPrefillWarps * 32, prefill_smem_bytes(),
                   static_cast<cudaStream_t>(stream)>>>(a);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ok() : cuda_fail(e, "prefill_kernel launch");
}

rtp_status rtp_dense_decode(rtp_handle* h, const rtp_layer_io* io, void* stream) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  rtp_status st = check_io(h, io, false);
  if (st != RTP_OK) return st;
  LayerArgs a = make_args(h, io);
  a.dense = 1;
  a.nret = 0;
  DeviceGuard guard(h->device);
  NvtxRange range(h, "rtp_dense_decode (%d x %d KV heads)", a.B, a.Hkv);
  st = enqueue_layer(h, a, static_cast<cudaStream_t>(stream));
  return st == RTP_OK ? ok() : st;
}

rtp_status rtp_decode_step_host(rtp_handle* h, int num_layers, const void* q_host,
                                const void* q_idx_host, const int32_t* seq_lens_host,
                                const void* const* k_cache, const void* const* v_cache,
                                const void* const* k_idx, const uint8_t* masks, float top_p,
                                float* out_host, void* stream) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  if (num_layers < 1 || num_layers > h->cfg.num_layers)
    return fail(RTP_ERR_INVALID_ARG, "num_layers outside [1, %d]", h->cfg.num_layers);
  if (!q_host || !seq_lens_host || !k_cache || !v_cache || !masks || !out_host)
    return fail(RTP_ERR_INVALID_ARG, "a required host pointer is NULL");
  const rtp_config& c = h->cfg;
  const size_t L = (size_t)num_layers, B = (size_t)c.batch;
  const size_t q_layer = B * c.num_q_heads * kHeadDim;       // elements per layer
  const size_t qi_layer = B * c.num_kv_heads * kIdxDim;
  bool any_ret = false;
  for (size_t i = 0; i < L * c.num_kv_heads; ++i) any_ret |= masks[i] != 0;
  if (any_ret && (!q_idx_host || !k_idx))
    return fail(RTP_ERR_INVALID_ARG, "q_idx_host and k_idx are required for retrieval heads");
  for (int b = 0; b < c.batch; ++b)
    if (seq_lens_host[b] < 1 || seq_lens_host[b] > c.max_ctx)
      return fail(RTP_ERR_INVALID_ARG, "seq_lens_host[%d] = %d outside [1, %d]", b,
                  seq_lens_host[b], c.max_ctx);
  DeviceGuard guard(h->device);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(h->stage_q, q_host, L * q_layer * 2, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && any_ret)
    e = cudaMemcpyAsync(h->stage_qidx, q_idx_host, L * qi_layer * 2, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(h->stage_seq, seq_lens_host, B * 4, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
  // the layers read and write only the staging buffers and the caller's caches, so the launch
  // sequence is the same from call to call while the pointers, masks and p are
  auto enqueue_all = [&](cudaStream_t st_stream) -> rtp_status {
    for (int l = 0; l < num_layers; ++l) {
      rtp_layer_io io;
      memset(&io, 0, sizeof io);
      io.q = static_cast<const char*>(h->stage_q) + (size_t)l * q_layer * 2;
      io.q_idx = static_cast<const char*>(h->stage_qidx) + (size_t)l * qi_layer * 2;
      io.k_cache = k_cache[l];
      io.v_cache = v_cache[l];
      io.k_idx = k_idx ? k_idx[l] : nullptr;
      io.seq_lens = h->stage_seq;
      io.retrieval_mask = masks + (size_t)l * c.num_kv_heads;
      io.top_p = top_p;
      io.out = h->stage_out + (size_t)l * q_layer;
      io.inputs_ready = 1;  // staged before the first launch; the caches do not change
      rtp_status st = rtp_decode_step(h, l, &io, st_stream);
      if (st != RTP_OK) return st;
    }
    return RTP_OK;
  };
  if (h->prof) {  // profiling events cannot sit in a graph: launch eagerly
    rtp_status st = enqueue_all(s);
    if (st != RTP_OK) return st;
  } else {
    std::vector<const void*> ptrs(3 * L);
    for (size_t l = 0; l < L; ++l) {
      ptrs[3 * l] = k_cache[l];
      ptrs[3 * l + 1] = v_cache[l];
      ptrs[3 * l + 2] = k_idx ? k_idx[l] : nullptr;
    }
    std::vector<uint8_t> mk(masks, masks + L * c.num_kv_heads);
    const bool reuse = h->step_exec && h->step_layers == num_layers && h->step_p == top_p &&
                       h->step_ptrs == ptrs && h->step_masks == mk;
    if (!reuse) {
      if (h->step_exec) {
        cudaGraphExecDestroy(h->step_exec);
        h->step_exec = nullptr;
      }
      if (!h->cap_stream) {
        e = cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreate");
      }
      e = cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal);
      if (e != cudaSuccess) return cuda_fail(e, "cudaStreamBeginCapture");
      rtp_status st = enqueue_all(h->cap_stream);
      cudaGraph_t graph = nullptr;
      e = cudaStreamEndCapture(h->cap_stream, &graph);
      if (st != RTP_OK) {
        if (graph) cudaGraphDestroy(graph);
        return st;
      }
      if (e != cudaSuccess) return cuda_fail(e, "cudaStreamEndCapture");
      e = cudaGraphInstantiate(&h->step_exec, graph, 0);
      cudaGraphDestroy(graph);
      if (e != cudaSuccess) {
        h->step_exec = nullptr;
        return cuda_fail(e, "cudaGraphInstantiate");
      }
      h->step_layers = num_layers;
      h->step_p = top_p;
      h->step_ptrs = std::move(ptrs);
      h->step_masks = std::move(mk);
    }
    e = cudaGraphLaunch(h->step_exec, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGraphLaunch");
    h->last_stream = s;
  }
  e = cudaMemcpyAsync(out_host, h->stage_out, L * q_layer * 4, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  return ok();
}

static rtp_status last_slot(rtp_handle* h, int b, int kvh, int* slot) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  if (!h->last_valid) return fail(RTP_ERR_INVALID_ARG, "no rtp_decode_step on this handle yet");
  if (b < 0 || b >= h->cfg.batch || kvh < 0 || kvh >= h->cfg.num_kv_heads)
    return fail(RTP_ERR_INVALID_ARG, "(b, kvh) = (%d, %d) out of range", b, kvh);
  const int j = h->last_slot_of_kvh[kvh];
  if (j < 0) return fail(RTP_ERR_INVALID_ARG, "kv head %d was local in the last call", kvh);
  *slot = b * h->last_nret + j;
  return RTP_OK;
}

rtp_status rtp_get_selection(rtp_handle* h, int b, int kvh, int32_t* idx_out, int64_t cap,
                             int64_t* count) {
  int slot = 0;
  rtp_status st = last_slot(h, b, kvh, &slot);
  if (st != RTP_OK) return st;
  if (!count) return fail(RTP_ERR_INVALID_ARG, "count is NULL");
  if (cap > 0 && !idx_out) return fail(RTP_ERR_INVALID_ARG, "idx_out is NULL");
  DeviceGuard guard(h->device);
  cudaError_t e = cudaStreamSynchronize(h->last_stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int total = 0, n = 0;
  e = cudaMemcpy(&total, h->ws.sel_total + slot, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&n, h->ws.sel_n + slot, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  *count = total;
  if (cap <= 0) return ok();
  const int64_t k = total < cap ? total : cap;
  if (h->last_fused) {  // expand the slot's tile masks (bit i of word t: token 64 t + i)
    const int words = (n + kFusedOwnTok - 1) / kFusedOwnTok;
    std::vector<unsigned long long> m((size_t)words);
    e = cudaMemcpy(m.data(), h->fx.sel_bits + (size_t)slot * h->fx.ldw, (size_t)words * 8,
                   cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
    int64_t at = 0;
    for (int t = 0; t < words && at < k; ++t)
      for (int i = 0; i < 64 && at < k; ++i)
        if ((m[(size_t)t] >> i) & 1ull) idx_out[at++] = t * kFusedOwnTok + i;
    return ok();
  }
  e = cudaMemcpy(idx_out, h->ws.sel_idx + (size_t)slot * h->ws.ld, (size_t)k * 4,
                 cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  return ok();
}

rtp_status rtp_get_threshold(rtp_handle* h, int b, int kvh, int* bstar, float* s_max) {
  int slot = 0;
  rtp_status st = last_slot(h, b, kvh, &slot);
  if (st != RTP_OK) return st;
  if (!bstar || !s_max) return fail(RTP_ERR_INVALID_ARG, "bstar and s_max must be non-NULL");
  DeviceGuard guard(h->device);
  cudaError_t e = cudaStreamSynchronize(h->last_stream);
  if (e == cudaSuccess) e = cudaMemcpy(bstar, h->ws.bstar + slot, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(s_max, h->ws.s_max + slot, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  return ok();
}

rtp_status rtp_get_device_status(rtp_handle* h, uint32_t* code) {
  if (!h || !code) return fail(RTP_ERR_INVALID_ARG, "handle and code must be non-NULL");
  DeviceGuard guard(h->device);
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(code, h->ws.status, 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(h->ws.status, 0, 4);
  // a barrier that timed out leaves its counter mid-count: start the next launch from zero
  if (e == cudaSuccess && (*code & kDevWaitTimeout)) {
    e = cudaMemset(h->ws.grid_bar, 0, (kFusedBarWord + 1) * 4);
    if (e == cudaSuccess)  // a stopped selection may leave maxima behind
      e = cudaMemset(h->ws.smax_key, 0, (size_t)h->cfg.batch * h->cfg.num_kv_heads * 4);
    if (e == cudaSuccess && h->fused_ok)  // a stopped single launch may leave maxima behind
      e = cudaMemset(h->fx.smax_key, 0, (size_t)h->cfg.batch * h->cfg.num_kv_heads * 4);
  }
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
  if (*code) return fail(RTP_ERR_DEVICE_STATUS, "device status 0x%x", *code);
  return ok();
}

rtp_status rtp_nvtx_enable(rtp_handle* h, int enable) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  h->nvtx = enable != 0;
  return ok();
}

rtp_status rtp_profile_enable(rtp_handle* h, int enable) {
  if (!h) return fail(RTP_ERR_INVALID_ARG, "handle is NULL");
  DeviceGuard guard(h->device);
  if (enable && h->prof_ev.empty()) {
    h->prof_ev.resize(2 * kProfCapacity);
    h->prof_kind.resize(kProfCapacity);
    for (auto& ev : h->prof_ev) {
      cudaError_t e = cudaEventCreate(&ev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
    }
  }
  h->prof = enable != 0;
  h->prof_used = 0;
  h->prof_overflow = false;
  return ok();
}

rtp_status rtp_profile_read(rtp_handle* h, double* ms, int64_t* launches) {
  if (!h || !ms || !launches) return fail(RTP_ERR_INVALID_ARG, "NULL argument");
  DeviceGuard guard(h->device);
  for (int k = 0; k < 4; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  for (int i = 0; i < h->prof_used; ++i) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(h->prof_ev[2 * i + 1]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, h->prof_ev[2 * i], h->prof_ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    ms[h->prof_kind[i]] += t;
    launches[h->prof_kind[i]] += 1;
  }
  const bool overflow = h->prof_overflow;
  h->prof_used = 0;
  h->prof_overflow = false;
  if (overflow) return fail(RTP_ERR_INVALID_ARG, "profiling pool overflowed; read more often");
  return ok();
}

rtp_status rtp_profile_launches(rtp_handle* h, double* ms, int32_t* kind, int64_t cap,
                                int64_t* count) {
  if (!h || !count || (cap > 0 && (!ms || !kind)))
    return fail(RTP_ERR_INVALID_ARG, "NULL argument");
  DeviceGuard guard(h->device);
  const int n = h->prof_used;
  *count = n;
  for (int i = 0; i < n && i < cap; ++i) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(h->prof_ev[2 * i + 1]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, h->prof_ev[2 * i], h->prof_ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventElapsedTime");
    ms[i] = t;
    kind[i] = h->prof_kind[i];
  }
  const bool overflow = h->prof_overflow || n > cap;
  h->prof_used = 0;
  h->prof_overflow = false;
  if (overflow) return fail(RTP_ERR_INVALID_ARG, "more launches recorded than cap (or the pool)");
  return ok();
}

const char* rtp_status_string(rtp_status s) {
  switch (s) {
    case RTP_OK: return "RTP_OK";
    case RTP_ERR_INVALID_ARG: return "RTP_ERR_INVALID_ARG";
    case RTP_ERR_UNSUPPORTED: return "RTP_ERR_UNSUPPORTED";
    case RTP_ERR_OOM: return "RTP_ERR_OOM";
    case RTP_ERR_CUDA: return "RTP_ERR_CUDA";
    case RTP_ERR_DEVICE_STATUS: return "RTP_ERR_DEVICE_STATUS";
  }
  return "RTP_ERR_UNKNOWN";
}

const char* rtp_last_error(void) { return g_err; }

}  // extern "C"
