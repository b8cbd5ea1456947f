// noalloc.cu -- rtp_window_attention_noalloc: window / dense attention with no allocation.
//
// For callers that cannot allocate device memory (a serving engine that owns every byte
// through its own pool, or a latency-critical path where cudaMalloc, which may synchronise the
// device, must not run). The attention kernels' only scratch -- split-K partials, the piece
// ranges the merge reads and a status word -- lives in the file-scope device array below, of
// a fixed size that bounds the call (at most RTP_NOALLOC_MAX_HEADS KV heads per call and at most
// RTP_NOALLOC_MAX_CTAS attention CTAs). Host code never touches the array by name: its device
// address is looked up once per device with cudaGetSymbolAddress and passed to the kernel.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "rtp.h"
#include "rtp_device.cuh"
#include "rtp_kernels.h"

using namespace rtp;

namespace {

constexpr int kNaHeads = RTP_NOALLOC_MAX_HEADS;
constexpr int kNaCtas = RTP_NOALLOC_MAX_CTAS;
constexpr size_t kNaPartOff = 0;
constexpr size_t kNaPartBytes = (size_t)(kNaCtas + kNaHeads) * kPartFloats * 4;
constexpr size_t kNaHeadOff = kNaPartOff + kNaPartBytes;           // piece ranges, then status
constexpr size_t kNaStatusOff = kNaHeadOff + (size_t)kNaHeads * 8;
constexpr size_t kNaUsed = kNaStatusOff + 256;
static_assert(kNaUsed <= RTP_NOALLOC_SCRATCH_BYTES, "no-alloc scratch too small");
static_assert(kNaCtas <= kMaxPieces, "the merge holds one factor per attention CTA");
static_assert(kNaHeadOff % 256 == 0, "aligned piece ranges");

// The scratch of every rtp_window_attention_noalloc call on this device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[RTP_NOALLOC_SCRATCH_BYTES];

struct DeviceSetup {
  bool ready = false;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
  int num_sms = 0;
};
constexpr int kMaxDevices = 64;
DeviceSetup g_setup[kMaxDevices];
std::mutex g_setup_mutex;

rtp_status na_fail(rtp_status s, const char* msg) {
  set_last_error(msg);
  return s;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" rtp_status rtp_window_attention_noalloc(const rtp_noalloc_params* p, const void* q,
                                                   const void* k_cache, const void* v_cache,
                                                   const int32_t* seq_lens, float* out,
                                                   void* stream) {
  if (!p || !q || !k_cache || !v_cache || !seq_lens || !out)
    return na_fail(RTP_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(seq_lens, 4))
    return na_fail(RTP_ERR_INVALID_ARG, "device pointers must be 16-byte aligned (seq_lens 4)");
  if (p->batch < 1 || p->num_kv_heads < 1 || p->num_q_heads < 1 ||
      p->num_q_heads % p->num_kv_heads != 0)
    return na_fail(RTP_ERR_INVALID_ARG, "batch, heads: positive, Hq a multiple of Hkv");
  if ((long long)p->batch * p->num_kv_heads > kNaHeads)
    return na_fail(RTP_ERR_UNSUPPORTED,
                   "batch * num_kv_heads exceeds RTP_NOALLOC_MAX_HEADS (the scratch limit)");
  if (p->num_q_heads / p->num_kv_heads > kMaxGroup)
    return na_fail(RTP_ERR_UNSUPPORTED, "GQA group size above 8");
  if (p->max_ctx < 1 || p->max_ctx > (1 << 28) || p->window < 1 || p->window > (1 << 28) ||
      p->sinks < 0 || p->sinks > (1 << 28))
    return na_fail(RTP_ERR_INVALID_ARG, "max_ctx, window or sinks out of range");
  if (!(p->attn_scale > 0.f) || !(p->attn_scale < 1e30f))
    return na_fail(RTP_ERR_INVALID_ARG, "attn_scale must be finite and > 0");

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return na_fail(RTP_ERR_CUDA, "cannot query the current device");
  DeviceSetup setup;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    DeviceSetup& s = g_setup[dev];
    if (!s.ready) {  // once per device, with that device current
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return na_fail(RTP_ERR_CUDA, "cudaGetSymbolAddress of the scratch array failed");
      }
      e = cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return na_fail(RTP_ERR_CUDA, "cannot query the SM count");
      s.scratch = static_cast<unsigned char*>(ptr);
      s.ready = true;
    }
    setup = s;
  }

  const int nheads = p->batch * p->num_kv_heads;
  const size_t smem = attend_smem_bytes(nheads, p->batch);
  // the dynamic shared memory limit is a per-kernel setting shared with every handle; it is
  // only ever raised (a handle created earlier for a larger layer keeps its size), and raising
  // it is not an allocation
  e = raise_smem_limit((const void*)attend_kernel, smem);
  if (e != cudaSuccess) return na_fail(RTP_ERR_CUDA, "cannot set the kernel's shared memory");

  LayerArgs a;
  memset(&a, 0, sizeof a);
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  a.v_cache = static_cast<const __nv_bfloat16*>(v_cache);
  a.seq_lens = seq_lens;
  a.out = out;
  a.B = p->batch;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = p->num_q_heads / p->num_kv_heads;
  a.max_ctx = p->max_ctx;
  a.window = p->window;
  a.sinks = p->sinks;
  a.nret = 0;
  a.dense = p->dense ? 1 : 0;
  a.attn_scale_log2 = (float)((double)p->attn_scale * 1.4426950408889634);
  for (int k = 0; k < kMaxKvHeads; ++k) a.slot_of_kvh[k] = -1;

  Workspace w;
  memset(&w, 0, sizeof w);
  unsigned char* base = setup.scratch;
  w.partials = reinterpret_cast<float*>(base + kNaPartOff);
  w.head_pieces = reinterpret_cast<int2*>(base + kNaHeadOff);
  w.status = reinterpret_cast<unsigned*>(base + kNaStatusOff);

  // Nothing in the array needs to start at zero: the attention launch writes the piece range of
  // every head and every partial the merge reads; status bits only accumulate.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int grid = setup.num_sms * kAttendCtasPerSm;
  if (grid > kNaCtas) grid = kNaCtas;
  a.attend_grid = grid;
  attend_kernel<<<grid, kAttendThreads, smem, s>>>(a, w);
  e = cudaGetLastError();
  if (e != cudaSuccess) return na_fail(RTP_ERR_CUDA, "attention kernel launch failed");
  merge_kernel<<<merge_units(nheads, a.G), kMergeThreads, 0, s>>>(a, w);
  e = cudaGetLastError();
  if (e != cudaSuccess) return na_fail(RTP_ERR_CUDA, "merge kernel launch failed");
  set_last_error("");
  return RTP_OK;
}
