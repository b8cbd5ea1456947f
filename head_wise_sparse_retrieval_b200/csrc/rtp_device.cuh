// rtp_device.cuh -- device-side building blocks shared by the kernels of librtp (sm_100a).
//
// Inline PTX wrappers for: programmatic dependent launch, GPU-scope atomics and acquire loads,
// asynchronous copies global -> shared (cp.async), ldmatrix, movmatrix and the warp-level
// bf16 MMA used to spare the FP32 pipes in the gather kernel.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace rtp {

constexpr int kHeadDim = 128;            // D
constexpr int kIdxDim = 16;              // r
constexpr int kBins = 256;               // histogram bins
constexpr int kSelThreads = 256;
constexpr int kPerThread = 16;           // consecutive tokens per thread in the compaction
constexpr int kMaxGroup = 8;             // query heads per KV head handled by one MMA column set
// a partial of one KV head's attention: o[8][128] (unnormalised), then m[8] (log2 domain), l[8]
constexpr int kPartO = kMaxGroup * kHeadDim;
constexpr int kPartFloats = kPartO + 2 * kMaxGroup;

// Device status bits (mirrors include/rtp.h).
constexpr unsigned kDevBadSeqlen = 0x1u;
constexpr unsigned kDevWaitTimeout = 0x2u;
constexpr unsigned kDevBadIndex = 0x4u;

// Bounded waits give up after this long (ns of %globaltimer) and report kDevWaitTimeout.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// ---- programmatic dependent launch ------------------------------------------------------

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Atomic add at GPU scope with release (publishes the writes the thread ordered before it) and
// acquire (later reads see what other releasing threads published) semantics.
__device__ __forceinline__ unsigned atomic_add_acq_rel_gpu(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v)
               : "memory");
  return old;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// floor(num / den) for 0 <= num < 2^53 and den >= 1, without a 64-bit integer division: the
// double quotient is within one of the result, and one integer check each way corrects it.
__device__ __forceinline__ long long floor_div(long long num, long long den) {
  long long q = (long long)((double)num / (double)den);
  if (q * den > num) --q;
  else if ((q + 1) * den <= num) ++q;
  return q;
}

// CTA c whose range [floor(c T / P), floor((c + 1) T / P)) holds position x, for 0 <= x < T,
// 1 <= P <= T and (x + 1) P + T < 2^53.
__device__ __forceinline__ long long cta_of(long long x, long long T, long long P) {
  return floor_div((x + 1) * P + T - 1, T) - 1;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Grid-wide barrier of a cooperative launch (every CTA is resident), one counter whose top bit
// flips once per barrier: CTA 0 adds 2^31 - (P - 1), every other CTA adds 1, so the low 31
// bits (0 between barriers) reach 2^31 and carry into the top bit exactly at the last arrival.
// The add has release semantics (it publishes the CTA's writes) and the polling load acquire
// semantics. The wait gives up after limit_ns, sets kDevWaitTimeout and makes later
// barriers of the CTA return at once, so the kernel ends (the host then clears the counter).
// withhold: a CTA index that does not arrive (self-test of the bounded wait), or -1.
__device__ inline void grid_barrier(unsigned* bar, unsigned* status, int* aborted,
                                    unsigned long long limit_ns, int withhold) {
  __syncthreads();
  if (threadIdx.x == 0 && !*aborted && (int)blockIdx.x == withhold) {
    *aborted = 1;  // never arrives: every other CTA's wait runs out
  } else if (threadIdx.x == 0 && !*aborted) {
    const unsigned inc = (blockIdx.x == 0) ? 0x80000000u - (gridDim.x - 1u) : 1u;
    const unsigned old = atomic_add_acq_rel_gpu(bar, inc);
    const unsigned long long t0 = global_ns();
    unsigned it = 0;
    while (((ld_acquire_gpu(bar) ^ old) & 0x80000000u) == 0u) {
      if ((++it & 255u) == 0 && global_ns() - t0 > limit_ns) {
        atomicOr(status, kDevWaitTimeout);
        *aborted = 1;
        break;
      }
    }
  }
  __syncthreads();
}

// Order-preserving map of a float to an unsigned key (larger float, larger key; 0 is below
// every key of a float, so 0 means "none").
__device__ __forceinline__ unsigned float_key(float x) {
  const unsigned u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// ---- shared memory and asynchronous copies -----------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 16-byte asynchronous copy global -> shared (L2 only, evict-first). src_bytes = 0 reads
// nothing and fills the 16 bytes with zeros (ragged tiles).
__device__ __forceinline__ void cp_async_16(uint32_t smem_dst, const void* gmem_src,
                                            unsigned src_bytes, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(smem_dst),
               "l"(gmem_src), "r"(src_bytes), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- warp-level matrix fragments ----------------------------------------------------------

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D = A(16x16, row) * B(16x8, col) + D, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// ---- indexer score arithmetic --------------------------------------------------------------
//
// fp16 x fp16 products are exact in fp32 (11-bit significands, no overflow or underflow), so
// the fp32 sum of two products, rounded once, is fma(a0, b0, a1 * b1): mixed-precision FMAs
// with fp16 operands give it without converting the operands. The -0 addend keeps a zero
// product's sign, so the result equals __fadd_rn(__fmul_rn(a0, b0), __fmul_rn(a1, b1)).
__device__ __forceinline__ float dot2_f16(uint32_t a2, uint32_t b2) {
  float d;
  asm("{\n\t.reg .f16 al, ah, bl, bh;\n\t.reg .f32 p;\n\t"
      "mov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.f16 p, ah, bh, 0f80000000;\n\t"
      "fma.rn.f32.f16 %0, al, bl, p;\n\t}"
      : "=f"(d)
      : "r"(a2), "r"(b2));
  return d;
}

// Sum of the 8 products of two fp16 8-vectors (16 bytes each) in the fixed order
// ((p0 + p1) + (p2 + p3)) + ((p4 + p5) + (p6 + p7)), fp32.
__device__ __forceinline__ float dot8_f16(const uint4& a, const uint4& b) {
  const float s01 = dot2_f16(a.x, b.x), s23 = dot2_f16(a.y, b.y);
  const float s45 = dot2_f16(a.z, b.z), s67 = dot2_f16(a.w, b.w);
  return __fadd_rn(__fadd_rn(s01, s23), __fadd_rn(s45, s67));
}

// ---- the histogram bin of a scaled indexer score -------------------------------------------
//
// bin = clamp(256 + floor((s - s_max) * bin_scale), 0, 255), bin_scale = 256 / idx_range.
// This equals floor((s - (s_max - idx_range)) * 256 / idx_range) clamped to [0, 255]. Every
// kernel that bins a score calls this one function on the same fp32 inputs, so a token counted
// in bin b by the histogram is selected by the compaction exactly when b >= b*.
__device__ __forceinline__ int score_bin(float s, float s_max, float bin_scale) {
  const float t = __fmul_rn(__fsub_rn(s, s_max), bin_scale);
  const float f = floorf(t);                      // <= 0 for s <= s_max
  const float c = fminf(fmaxf(f + 256.0f, 0.0f), 255.0f);
  return static_cast<int>(c);
}

}  // namespace rtp
