// Micro-benchmarks of the B200 issue pipes and of a streaming read, the ceilings
// that decode attention on CUDA cores is measured against.
//
// Every kernel does a fixed, bounded amount of work (no waits, no data-dependent
// loops) and writes one value per thread so that nothing is optimised away.  The
// caller times the launch on its stream; kvq_microbench returns the launch's
// work count (multiply-adds, or bytes for the read), so rate = work / time.
//
// Kinds (each thread runs `iters` rounds of 8 independent chains):
//   KVQ_UB_FFMA   fp32 fma             1 multiply-add per instruction
//   KVQ_UB_DP2A   dp2a.lo.s32.u32      2 multiply-adds per instruction
//   KVQ_UB_DP4A   dp4a.s32.u32         4 multiply-adds per instruction
//   KVQ_UB_FMA2   fma.rn.f32x2         2 multiply-adds per instruction
//   KVQ_UB_MIX    dp2a and fp32 fma interleaved one to one (3 per pair)
//   KVQ_UB_READ   16-byte loads of a device buffer, grid-stride (bytes)
#include "kvq_internal.h"

namespace kvq {

namespace {
constexpr int UB_THREADS = 256;

template <int KIND>
__global__ void __launch_bounds__(UB_THREADS) ubench_alu(int iters, uint32_t seed, unsigned long long* sink) {
  const uint32_t t = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t q = seed * 0x9E3779B1u + t;
  if (KIND == KVQ_UB_FFMA || KIND == KVQ_UB_MIX) {
    float a[8], b = __uint_as_float(0x3f800001u + (t & 7)), c = 1e-7f;
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = (float)(t + k);
    int d[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) d[k] = (int)(t * (k + 1));
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        a[k] = fmaf(a[k], b, c);
        if (KIND == KVQ_UB_MIX) asm volatile("dp2a.lo.s32.u32 %0, %1, %2, %0;" : "+r"(d[k]) : "r"(q), "r"(q ^ k));
      }
    }
    float s = 0.f;
    int e = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) { s += a[k]; e += d[k]; }
    sink[t] = (unsigned long long)__float_as_uint(s) + (unsigned long long)(uint32_t)e;
  } else if (KIND == KVQ_UB_DP2A || KIND == KVQ_UB_DP4A) {
    int d[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) d[k] = (int)(t * (k + 1));
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (KIND == KVQ_UB_DP2A) asm volatile("dp2a.lo.s32.u32 %0, %1, %2, %0;" : "+r"(d[k]) : "r"(q), "r"(q ^ k));
        else asm volatile("dp4a.s32.u32 %0, %1, %2, %0;" : "+r"(d[k]) : "r"(q), "r"(q ^ k));
      }
    }
    int e = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) e += d[k];
    sink[t] = (unsigned long long)(uint32_t)e;
  } else {                                        // KVQ_UB_FMA2
    uint64_t a[8];
    uint64_t b, c;
    asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(1.0000001f), "f"(0.9999999f));
    asm("mov.b64 %0, {%1, %2};" : "=l"(c) : "f"(1e-7f), "f"(2e-7f));
#pragma unroll
    for (int k = 0; k < 8; ++k) asm("mov.b64 %0, {%1, %2};" : "=l"(a[k]) : "f"((float)t), "f"((float)k));
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int k = 0; k < 8; ++k) asm volatile("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(a[k]) : "l"(b), "l"(c));
    }
    uint64_t s = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) s ^= a[k];
    sink[t] = s;
  }
}

__global__ void __launch_bounds__(UB_THREADS) ubench_read(const uint4* __restrict__ buf, size_t n16, int passes,
                                                          unsigned long long* sink) {
  const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  uint32_t x = 0;
  for (int pass = 0; pass < passes; ++pass)
    for (size_t i = t; i < n16; i += stride) {
      const uint4 v = __ldcs(buf + i);
      x ^= v.x ^ v.y ^ v.z ^ v.w;
    }
  sink[t] = x;
}
}  // namespace

cudaError_t launch_microbench(int kind, int iters, const void* buf, size_t buf_bytes, unsigned long long* sink,
                              int ctas, cudaStream_t s, double* work) {
  const size_t threads = (size_t)ctas * UB_THREADS;
  switch (kind) {
    case KVQ_UB_FFMA: ubench_alu<KVQ_UB_FFMA><<<ctas, UB_THREADS, 0, s>>>(iters, 1u, sink); *work = 8.0 * iters * threads; break;
    case KVQ_UB_DP2A: ubench_alu<KVQ_UB_DP2A><<<ctas, UB_THREADS, 0, s>>>(iters, 2u, sink); *work = 16.0 * iters * threads; break;
    case KVQ_UB_DP4A: ubench_alu<KVQ_UB_DP4A><<<ctas, UB_THREADS, 0, s>>>(iters, 3u, sink); *work = 32.0 * iters * threads; break;
    case KVQ_UB_FMA2: ubench_alu<KVQ_UB_FMA2><<<ctas, UB_THREADS, 0, s>>>(iters, 4u, sink); *work = 16.0 * iters * threads; break;
    case KVQ_UB_MIX: ubench_alu<KVQ_UB_MIX><<<ctas, UB_THREADS, 0, s>>>(iters, 5u, sink); *work = 24.0 * iters * threads; break;
    case KVQ_UB_READ: {
      const size_t n16 = buf_bytes / 16;
      ubench_read<<<ctas, UB_THREADS, 0, s>>>(reinterpret_cast<const uint4*>(buf), n16, iters, sink);
      *work = (double)n16 * 16.0 * iters;
    } break;
    default: return cudaErrorInvalidValue;
  }
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace kvq
