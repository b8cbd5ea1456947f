/*
 * rtp.h -- C-ABI of the B200 decode-step attention of RTPurbo (head-wise sparse retrieval).
 *
 * One call computes one layer of one decode step for a batch of sequences:
 *
 *   retrieval KV head (mask != 0), per sequence b with context N = seq_lens[b]:
 *     s_n  = idx_scale * q_idx . k_idx[n]                       n < N      (indexer score)
 *     bin  = clamp(floor((s_n - (s_max - idx_range)) * 256 / idx_range), 0, 255)
 *     w_n  = exp(s_n - s_max);  M_b = sum_{bin(n)=b} w_n;  C_b = M_255 + ... + M_b
 *     b*   = max{ b : C_b >= top_p * C_0 };  S = { n : bin(n) >= b* }  (sort-free top-p)
 *     o_g  = sum_{n in S} softmax_S(attn_scale * q_g . k_n) v_n   for the G query heads g
 *            of the KV head's GQA group (they share S)
 *   local KV head (mask == 0):
 *     the same o_g over T = {0 .. sinks-1} U {N-window .. N-1} (clipped to [0, N))
 *
 * Passages this follows (page title, then section / equation):
 *   "Full Attention Strikes Back: Transferring Full Attention into Sparse within Hundred
 *   Training Steps" (xllm-io paper review):
 *     - section 三, 核心公式 / 自适应稀疏注意力: the low-rank indexer score s_h(m,n), taken
 *       before RoPE, the sparse attention O_h(m) over S_h(m), and S_h(m) = Top-P(s_h, p);
 *     - section 三, 硬件感知解码内核: sort-free top-p over a 256-bin histogram whose size does
 *       not depend on the sequence length, scoring and selection fused;
 *     - section 五, 测试配置: window 8192, 4 sink tokens, low-rank size 16, top-p 0.9.
 *   "Technical Summary: Full Attention Strikes Back ..." (gist.science), Methodology 1 and 3:
 *     local heads use a sliding window with attention sinks; retrieval heads select tokens
 *     in decode by accumulating low-dimensional attention mass until p is reached.
 *   The pages leave the bin edges, the indexer scale and the handling of GQA groups open;
 *   the rules above are the readings this library implements.
 *
 * Conventions for every entry point:
 *   - All tensors are row-major and contiguous. bf16 / fp16 tensors are passed as void*
 *     (16-bit IEEE bfloat16 / binary16 values). Device pointers must be 16-byte aligned.
 *   - The caller owns every buffer passed in. The handle owns only its workspace.
 *   - Every call returns an rtp_status. Arguments are checked on the host before any
 *     launch; on error nothing is enqueued. rtp_last_error() gives a one-line reason
 *     (thread-local, valid until the next call on the same thread).
 *   - Streams are cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - One handle serves one stream at a time: calls that overlap on the GPU through the
 *     same handle race on its workspace.
 */
#ifndef RTP_H
#define RTP_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RTP_API __attribute__((visibility("default")))
#else
#define RTP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RTP_OK = 0,
    RTP_ERR_INVALID_ARG = 1,   /* a NULL / misaligned pointer, a size out of range, ... */
    RTP_ERR_UNSUPPORTED = 2,   /* a valid configuration this build does not implement    */
    RTP_ERR_OOM = 3,           /* device workspace allocation failed (rtp_create only)   */
    RTP_ERR_CUDA = 4,          /* a CUDA runtime call failed                             */
    RTP_ERR_DEVICE_STATUS = 5  /* the kernels reported a problem (rtp_get_device_status) */
} rtp_status;

/* Device status bits, reported by rtp_get_device_status. */
#define RTP_DEV_BAD_SEQLEN   0x1u  /* a seq_lens[b] outside [1, max_ctx]; it was clamped   */
#define RTP_DEV_WAIT_TIMEOUT 0x2u  /* a bounded in-kernel wait gave up (output invalid)     */
#define RTP_DEV_BAD_INDEX    0x4u  /* a token index outside [0, N) was about to be read     */

typedef struct rtp_handle rtp_handle;

typedef struct {
    int num_layers;    /* layers of the model; rtp_decode_step's layer is checked against it   */
    int batch;         /* B, >= 1                                                              */
    int num_q_heads;   /* Hq; Hq % Hkv == 0                                                    */
    int num_kv_heads;  /* Hkv, 1 .. 256; G = Hq / Hkv must be 1 .. 8                           */
    int head_dim;      /* D, 128 only                                                          */
    int idx_dim;       /* r, 16 only                                                           */
    int max_ctx;       /* cache capacity per (b, KV head), 1 .. 2^24 - 1 (16 777 215): the
                          selection sums token masses as 64-bit integers of 2^-40 units    */
    int window;        /* local-head sliding window, >= 1 (8192)                               */
    int sinks;         /* local-head sink tokens, >= 0 (4)                                     */
    int num_bins;      /* histogram bins, 256 only                                             */
    float idx_range;   /* the bins cover [s_max - idx_range, s_max], > 0 (16)                  */
    float idx_scale;   /* indexer score scale, > 0 (1/sqrt(16) = 0.25)                         */
    float attn_scale;  /* attention logit scale, > 0 (1/sqrt(128))                            */
} rtp_config;

/* Fills *cfg with the pages' configuration for the given shape: head_dim 128, idx_dim 16,
 * window 8192, sinks 4, 256 bins over a range of 16, idx_scale 0.25, attn_scale 1/sqrt(128). */
RTP_API void rtp_config_default(rtp_config *cfg, int num_layers, int batch, int num_q_heads,
                        int num_kv_heads, int max_ctx);

/* Bytes of device workspace rtp_create allocates for cfg (0 if cfg is invalid). */
RTP_API size_t rtp_workspace_bytes(const rtp_config *cfg);

/* Creates a handle on CUDA device `device` and allocates its workspace, sized for the worst
 * case (every KV head a retrieval head selecting all max_ctx tokens), so that no later call
 * allocates. Errors: RTP_ERR_INVALID_ARG (bad cfg or out == NULL), RTP_ERR_UNSUPPORTED
 * (head_dim, idx_dim, num_bins or G outside what is implemented), RTP_ERR_OOM, RTP_ERR_CUDA. */
RTP_API rtp_status rtp_create(const rtp_config *cfg, int device, rtp_handle **out);

/* Frees the workspace and the handle. NULL is accepted. Synchronises the device first. */
RTP_API rtp_status rtp_destroy(rtp_handle *h);

typedef struct {
    const void *q;           /* bf16 [B][Hq][D], device: the current token's queries (RoPE'd)    */
    const void *q_idx;       /* fp16 [B][Hkv][r], device: indexer queries W^Q q^pre; read for
                                retrieval heads only (may be NULL when the mask has none)        */
    const void *k_cache;     /* bf16 [B][Hkv][max_ctx][D], device: keys (RoPE'd)                 */
    const void *v_cache;     /* bf16 [B][Hkv][max_ctx][D], device: values                        */
    const void *k_idx;       /* fp16 [B][Hkv][max_ctx][r], device: indexer keys W^K k^pre; read
                                for retrieval heads only (may be NULL when the mask has none)    */
    const int32_t *seq_lens; /* [B], device: N_b, 1 <= N_b <= max_ctx. The caches already hold
                                the current token at position N_b - 1.                          */
    const uint8_t *retrieval_mask; /* [Hkv], HOST: nonzero marks a retrieval KV head           */
    float top_p;             /* 0 < top_p <= 1                                                   */
    float *out;              /* fp32 [B][Hq][D], device: attention output                        */
    int32_t *sel_count;      /* optional [B][Hkv], device: receives |S| for retrieval heads and
                                |T| for local heads; NULL to skip                                */
    int32_t top_k;           /* 0: top-p selection. k > 0: fixed top-k through the same 256-bin
                                histogram (the pages' top-k / top-p comparison): every bin from
                                the top down until the bins hold >= k tokens, all N_b tokens
                                when k >= N_b; top_p is then ignored.                           */
    int32_t inputs_ready;    /* 0 (safe default): the layer's kernels wait for the preceding
                                launch on the stream before reading anything. Nonzero: the caller
                                vouches that q, q_idx, seq_lens and the caches are complete before
                                that launch ends (e.g. layer after layer of one step with every
                                input already resident), so the selection scores and the
                                attention of a layer without retrieval heads stream their inputs
                                while the previous launch drains; they still wait before
                                writing anything the previous layer may read.                   */
    int32_t single_launch;   /* 0 (default): the selection, attention and merge launches above.
                                Nonzero: the whole layer in ONE cooperative launch of one CTA per
                                SM (the pages' fused scoring + selection, extended through the
                                gather): the retrieval slots' tokens are owned in 64-token tiles
                                dealt round-robin to the CTAs, the selection stays in on-chip
                                bit masks (no position list) and the split heads are merged after
                                a grid barrier. Same selection and outputs as the default path.
                                Needs B * Hkv <= 64 and B * nret * ceil(max_ctx / 64) <= 448 per
                                SM, else RTP_ERR_UNSUPPORTED (nothing enqueued); inputs_ready is
                                ignored (the launch always waits for the preceding one).          */
} rtp_layer_io;

/* Enqueues one layer of the decode step on `stream`. A layer with retrieval heads is three
 * kernels: the selection, the attention of every head (split over the SMs), and the merge of
 * the split heads. A layer of local heads only is one kernel when the handle's B * Hkv leaves at
 * least 4 SMs per KV head (and window + sinks <= 65536): one thread-block cluster per KV head,
 * whose CTAs merge the head's pieces inside the launch; otherwise attention and
 * merge as above. Asynchronous: no host synchronisation,
 * no allocation, capturable in a CUDA graph (the mask is read on the host at call time and the
 * launch shapes depend only on cfg and the mask). Errors (nothing enqueued): RTP_ERR_INVALID_ARG
 * for a NULL handle / io / required pointer, a misaligned device pointer, top_k < 0, top_p
 * outside (0, 1] when top_k is 0, or layer outside [0, num_layers); RTP_ERR_CUDA if a launch fails. Problems only the device
 * can see (seq_lens) are reported through rtp_get_device_status. */
RTP_API rtp_status rtp_decode_step(rtp_handle *h, int layer, const rtp_layer_io *io, void *stream);

/* ---- Indexer production at decode ----------------------------------------------------
 * [R] section 三 核心公式 / 自适应稀疏注意力: the retrieval score uses low-rank projections of
 * the query and key taken before RoPE, s_h(m,n) = (W^Q_h q^pre_{m,h})^T (W^K_h k^pre_{n,h}).
 * rtp_indexer_append produces, for the current token of every sequence b and every selected
 * KV head h, the indexer query of rtp_decode_step and the new indexer-key cache row:
 *   q_idx[b][h][i]         = fp16( sum_{j < G*D} w_q[h][i][j] * q_pre[b][h*G + j/D][j%D] )
 *   k_idx[b][h][N_b-1][i]  = fp16( sum_{d < D}   w_k[h][i][d] * k_pre[b][h][d] )
 * (the G query heads of the KV head's group concatenated head-major; fp32 accumulation,
 * rounded to nearest fp16 once). All pointers are device memory, 16-byte aligned except
 * seq_lens (4). The weights w_q and w_k are read before the kernel waits for the preceding
 * launch on the stream, so that launch must not write them (model weights are constant
 * during decode); q_pre, k_pre and seq_lens are read after the wait. Errors:
 * RTP_ERR_INVALID_ARG for NULL / misaligned pointers; a seq_lens entry outside [1, max_ctx]
 * is clamped and reported in the device status word. */
typedef struct {
    const void *q_pre;       /* bf16 [B][Hq][D]: pre-RoPE queries of the current token         */
    const void *k_pre;       /* bf16 [B][Hkv][D]: pre-RoPE key of the current token            */
    const void *w_q;         /* bf16 [Hkv][r][G*D]                                             */
    const void *w_k;         /* bf16 [Hkv][r][D]                                               */
    const int32_t *seq_lens; /* [B]: the current token is at position N_b - 1                  */
    const uint8_t *head_mask;/* [Hkv], HOST: heads to produce (NULL: every head)               */
    void *q_idx;             /* fp16 [B][Hkv][r], written for the selected heads               */
    void *k_idx;             /* fp16 [B][Hkv][max_ctx][r]: row N_b - 1 of the selected heads   */
} rtp_indexer_io;

RTP_API rtp_status rtp_indexer_append(rtp_handle *h, const rtp_indexer_io *io, void *stream);

/* ---- Prefill ---------------------------------------------------------------------------
 * gist.science technical summary, Methodology 1: during prefill the retrieval heads keep, and
 * attend over, the full KV cache, and the local heads a sliding window with attention sinks;
 * "Full Attention Strikes Back ..." (xllm-io paper review) section 五 测试配置 (window 8192,
 * 4 sinks) and its prefill speed-up table. For every prompt position i < T_b of sequence b and
 * every query head hq of KV head kvh = hq / G:
 *   out[b][hq][i] = sum_{j in K_i} softmax_{K_i}(attn_scale * q[b][hq][i] . k_j) v_j
 *   K_i = { j : j <= i }                                          retrieval head, or dense != 0
 *   K_i = { 0 .. sinks-1 } U { i+1-window .. i } (all j <= i when they meet)   local head
 * i.e. the decode output of a context of i + 1 tokens (window and sinks from the config). The
 * caller has written the prompt's keys and values into rows 0 .. T_b - 1 of the caches. Rows
 * i >= T_b of out are not written. One launch, no host synchronisation, no allocation; the
 * kernel starts once the preceding work on the stream has completed. Errors (nothing
 * enqueued): RTP_ERR_INVALID_ARG for a NULL / misaligned pointer or t_max outside
 * [1, max_ctx]; RTP_ERR_UNSUPPORTED for batch * num_kv_heads * t_max >= 2^31. A seq_lens entry
 * outside [1, t_max] is clamped and reported in the device status word. */
typedef struct {
    const void *q;           /* bf16 [B][Hq][t_max][D], device: the prompt's queries           */
    const void *k_cache;     /* bf16 [B][Hkv][max_ctx][D], device                              */
    const void *v_cache;     /* bf16 [B][Hkv][max_ctx][D], device                              */
    const int32_t *seq_lens; /* [B], device: prompt lengths T_b                                */
    const uint8_t *retrieval_mask; /* [Hkv], HOST: nonzero marks a retrieval KV head           */
    float *out;              /* fp32 [B][Hq][t_max][D], device: rows < T_b written             */
    int32_t t_max;           /* rows per head of q and out, 1 .. max_ctx                      */
    int32_t dense;           /* nonzero: every head attends over all j <= i (full causal
                                attention, the speed-up denominator)                          */
} rtp_prefill_io;

RTP_API rtp_status rtp_prefill(rtp_handle *h, const rtp_prefill_io *io, void *stream);

/* Dense full attention over all N_b tokens for every KV head (top_p, q_idx, k_idx and the mask
 * are ignored). The speedup denominator: same caches, same kernels, no selection. */
RTP_API rtp_status rtp_dense_decode(rtp_handle *h, const rtp_layer_io *io, void *stream);

/* Host-buffer variant of a whole decode step over `num_layers` layers: copies the queries
 * q_host (bf16 [L][B][Hq][D]) and q_idx_host (fp16 [L][B][Hkv][r]) and seq_lens_host
 * (int32 [B]) from host memory to the handle's device staging, runs rtp_decode_step for each
 * layer l with the device caches k_cache[l], v_cache[l], k_idx[l] and the host mask
 * masks[l * Hkv ...], and copies the fp32 outputs back into out_host ([L][B][Hq][D]).
 * Host buffers should be pinned for the copies to be asynchronous. Synchronises `stream`
 * before returning (the outputs are in out_host on return). Staging is allocated by
 * rtp_create for cfg.num_layers layers. The layer launches are captured once into a CUDA
 * graph on a stream of the handle (created on first use) and replayed on `stream` while
 * num_layers, top_p, the cache pointers and the masks stay the same; a change re-captures.
 * While profiling is enabled the layers are launched one by one instead. Must not be called
 * while `stream` is being captured. Errors as rtp_decode_step. */
RTP_API rtp_status rtp_decode_step_host(rtp_handle *h, int num_layers, const void *q_host,
                                const void *q_idx_host, const int32_t *seq_lens_host,
                                const void *const *k_cache, const void *const *v_cache,
                                const void *const *k_idx, const uint8_t *masks, float top_p,
                                float *out_host, void *stream);

/* Debug / parity: the ascending token positions selected for (b, kvh) by the most recent
 * rtp_decode_step on this handle (which must have marked kvh as a retrieval head).
 * Synchronises that call's stream. Writes min(cap, |S|) positions to idx_out (HOST) and |S| to
 * *count. Errors: RTP_ERR_INVALID_ARG (no such head in the last call, NULL count). */
RTP_API rtp_status rtp_get_selection(rtp_handle *h, int b, int kvh, int32_t *idx_out, int64_t cap,
                             int64_t *count);

/* Debug / parity: the threshold bin b* and the maximum indexer score s_max (fp32) the most
 * recent rtp_decode_step used for (b, kvh). Synchronises that call's stream. */
RTP_API rtp_status rtp_get_threshold(rtp_handle *h, int b, int kvh, int *bstar, float *s_max);

/* Kernel profiling. While enabled, every kernel that rtp_decode_step / rtp_dense_decode
 * launches on this handle is bracketed by two CUDA events recorded on the launch stream (the
 * events are created here, so the decode calls still allocate nothing). Do not enable it while
 * capturing a CUDA graph. Kernel classes: 0 selection (indexer score, histogram top-p,
 * compaction), 1 attention (including the cluster launch of a layer of local heads only, which
 * merges inside), 2 merge of split heads' partials, 3 the single-launch layer
 * (rtp_layer_io.single_launch). The event pool holds 1024
 * launches; rtp_profile_read empties it. Errors: RTP_ERR_CUDA if the events cannot be created. */
RTP_API rtp_status rtp_profile_enable(rtp_handle *h, int enable);

/* The same recorded launches one by one, in launch order: ms[i] and kind[i] (the classes of
 * rtp_profile_read) for i < min(cap, *count), *count = the number recorded. Synchronises them
 * and empties the pool. Errors: RTP_ERR_INVALID_ARG for NULL arguments, or when more launches
 * were recorded than cap (the first cap are still written) or than the pool holds. */
RTP_API rtp_status rtp_profile_launches(rtp_handle *h, double *ms, int32_t *kind, int64_t cap,
                                        int64_t *count);

/* NVTX ranges. While enabled (off by default), every rtp_decode_step, rtp_dense_decode and
 * rtp_indexer_append call on this handle pushes one NVTX range around its launches, named for
 * the call, the layer and its retrieval-head count ("rtp_decode_step layer 7 (1 retrieval KV
 * heads)"), so that a timeline profiler shows each layer's kernels under one label. The
 * ranges are host-side markers: they cost nothing without a profiler attached and are legal
 * during stream capture. Errors: RTP_ERR_INVALID_ARG for a NULL handle. */
RTP_API rtp_status rtp_nvtx_enable(rtp_handle *h, int enable);

/* Synchronises the recorded launches, adds their durations (ms) and counts per kernel class
 * into ms[4] and launches[4] (overwritten), and empties the pool. */
RTP_API rtp_status rtp_profile_read(rtp_handle *h, double *ms, int64_t *launches);

/* Self-test of failure detection without a GPU fault: enqueues the selection of one layer (as
 * rtp_decode_step would, attention not launched) with CTA 0 withholding its arrival at the
 * first grid barrier and every barrier wait limited to wait_ns (1 us .. 1 s). The other CTAs'
 * waits run out, the launch ends on its own, and RTP_DEV_WAIT_TIMEOUT is set in the device
 * status word; rtp_get_device_status reports it and clears the barrier state, after which the
 * handle decodes normally. The selection lists it leaves are not meaningful (the debug
 * getters refuse them). The pages describe no such call. Errors: RTP_ERR_INVALID_ARG for a
 * mask without retrieval heads or wait_ns out of range, otherwise as rtp_decode_step. */
RTP_API rtp_status rtp_selftest_wait_timeout(rtp_handle *h, int layer, const rtp_layer_io *io,
                                             uint64_t wait_ns, void *stream);

/* Reads and clears the device status word (RTP_DEV_* bits) after synchronising the device.
 * After RTP_DEV_WAIT_TIMEOUT it also resets the selection kernel's grid-barrier counter, so
 * that later calls on the handle start from a clean barrier. Returns RTP_ERR_DEVICE_STATUS
 * when a bit was set, RTP_OK otherwise. */
RTP_API rtp_status rtp_get_device_status(rtp_handle *h, uint32_t *code);

/* ---- Attention without any allocation --------------------------------------------------
 * The pages describe no such call; it exists for callers that cannot allocate device memory:
 * engines that plan every byte up front and hand out memory only from their own pool, and
 * latency-critical paths where cudaMalloc (which may synchronise the device) must not run.
 * rtp_create allocates a workspace; this entry point needs no handle: its only scratch (the
 * split-K partials and head offsets of the attention kernels) is a file-scope device array of
 * RTP_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until the process exits.
 *
 * It computes, for every (b, KV head), the attention over the window + sink set of a local
 * head (dense == 0) or over all N_b tokens (dense != 0), exactly as rtp_decode_step does for a
 * local head and rtp_dense_decode for any head. Layouts as in rtp_layer_io: q bf16 [B][Hq][128],
 * k_cache / v_cache bf16 [B][Hkv][max_ctx][128], seq_lens int32 [B] (device), out fp32
 * [B][Hq][128]; device pointers, 16-byte aligned (seq_lens 4-byte aligned).
 *
 * Limits: batch * num_kv_heads <= RTP_NOALLOC_MAX_HEADS, G = Hq / Hkv in 1..8, max_ctx in
 * [1, 2^28], window >= 1, sinks >= 0; larger sizes return RTP_ERR_UNSUPPORTED with a message.
 * It calls no cudaMalloc / cudaFree and no allocating library routine. The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress) with that device current;
 * make that first call before any stream capture. Every call shares the one array, which keeps
 * the last call's contents, none of which a later call reads before writing it.
 * Calls that overlap on the GPU (different streams, or the same array used from two threads'
 * streams at once) race on the array. Device-side problems (a seq_lens entry outside
 * [1, max_ctx], which is clamped) are not reported by this call. */
#define RTP_NOALLOC_MAX_HEADS 64
#define RTP_NOALLOC_MAX_CTAS 296
#define RTP_NOALLOC_SCRATCH_BYTES 8388608

typedef struct {
    int batch, num_q_heads, num_kv_heads, max_ctx, window, sinks;  /* head_dim is 128 */
    float attn_scale;                                                /* e.g. 1/sqrt(128)  */
    int dense;                                                       /* 0: window + sinks */
} rtp_noalloc_params;

RTP_API rtp_status rtp_window_attention_noalloc(const rtp_noalloc_params *p, const void *q,
                                                const void *k_cache, const void *v_cache,
                                                const int32_t *seq_lens, float *out,
                                                void *stream);

/* Static string for a status code. */
RTP_API const char *rtp_status_string(rtp_status s);

/* One-line reason for the last error returned on this thread ("" if none). */
RTP_API const char *rtp_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RTP_H */
