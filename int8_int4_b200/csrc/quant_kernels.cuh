// quant_kernels.cuh -- the HBM-bound quantisers: per-row symmetric int8
// (q8 weight pack and per-token activation quantisation, one rule) and the
// q4 group-32 nibble pack.
//
// "What aria is" (aria project page): weights are packed from fp16 down to 8
// or 4 bits. "Results": W8A8 quantises activations to 8 bits as well. Both
// quotients are IEEE fp32 divisions (__fdiv_rn) rounded half-to-even
// (__float2int_rn), so the codes are a pure function of the input bits.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"

namespace aria {

constexpr int kRowThreads = 256;
constexpr int kRowCached = 4;  // 16-byte chunks kept in registers per thread

__device__ __forceinline__ float absmax8(const uint4& v) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  __half2 m = __habs2(h[0]);
  m = __hmax2(m, __habs2(h[1]));
  m = __hmax2(m, __habs2(h[2]));
  m = __hmax2(m, __habs2(h[3]));
  return fmaxf(__low2float(m), __high2float(m));
}

__device__ __forceinline__ int quant_i8(float x, float s) {
  int q = __float2int_rn(__fdiv_rn(x, s));
  return max(-127, min(127, q));
}

// 8 fp16 -> 8 int8 codes packed in a uint2
__device__ __forceinline__ uint2 quant8_i8(const uint4& v, float s, bool zero) {
  const __half* h = reinterpret_cast<const __half*>(&v);
  uint32_t w[2] = {0u, 0u};
  if (!zero) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t b = static_cast<uint32_t>(quant_i8(__half2float(h[i]), s)) & 0xFFu;
      w[i >> 2] |= b << (8 * (i & 3));
    }
  }
  return make_uint2(w[0], w[1]);
}

// A GEMM loads its first packed weight tiles (with TMA, the async proxy)
// before it waits for the preceding kernel. A pack kernel therefore never
// lets its successor start early, and every thread ends with its stores
// ordered at GPU scope and toward the async proxy, so that the pack's
// completion implies that a following GEMM's tile loads see the bytes.
__device__ __forceinline__ void publish_packed_stores() {
  __threadfence();
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// One CTA per row: s[r] = absmax / 127, q = clamp(rhe(x / s), -127, 127).
// Row r of X starts 16-byte aligned (K % 8 == 0); the first kRowCached
// chunks of each thread stay in registers between the two passes.
// `early_dependents`: let the next kernel in the stream start its set-up
// now (activation quantisation). Weight packing passes false and publishes
// its stores (see publish_packed_stores).
__global__ void __launch_bounds__(kRowThreads) row_quant_i8_kernel(const __half* __restrict__ X,
                                                                   int K, int8_t* __restrict__ Q,
                                                                   float* __restrict__ S,
                                                                   bool early_dependents) {
  __shared__ float warp_max[kRowThreads / 32];
  pdl_wait();  // X may be written by the preceding kernel
  if (early_dependents) pdl_launch_dependents();
  const int64_t r = blockIdx.x;
  const int nchunk = K >> 3;
  const uint4* xr = reinterpret_cast<const uint4*>(X + r * static_cast<int64_t>(K));
  uint2* qr = reinterpret_cast<uint2*>(Q + r * static_cast<int64_t>(K));

  uint4 cache[kRowCached];
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < kRowCached; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nchunk) {
      cache[i] = ld_dep_v4(xr + c);
      a = fmaxf(a, absmax8(cache[i]));
    }
  }
  for (int c = threadIdx.x + kRowCached * kRowThreads; c < nchunk; c += kRowThreads)
    a = fmaxf(a, absmax8(ld_dep_v4(xr + c)));

#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = a;
  __syncthreads();
  a = warp_max[0];
#pragma unroll
  for (int w = 1; w < kRowThreads / 32; ++w) a = fmaxf(a, warp_max[w]);

  const float s = __fdiv_rn(a, 127.0f);
  const bool zero = (a == 0.0f);
  if (threadIdx.x == 0) S[r] = s;
#pragma unroll
  for (int i = 0; i < kRowCached; ++i) {
    const int c = threadIdx.x + i * kRowThreads;
    if (c < nchunk) qr[c] = quant8_i8(cache[i], s, zero);
  }
  for (int c = threadIdx.x + kRowCached * kRowThreads; c < nchunk; c += kRowThreads)
    qr[c] = quant8_i8(ld_dep_v4(xr + c), s, zero);
  if (!early_dependents) publish_packed_stores();
}

// q4 pack: one thread per 16-byte chunk (8 consecutive k of one row); four
// consecutive lanes form a group of 32 and share its absmax by shuffles.
// s16 = fp16_rn(absmax / 7); code = clamp(rhe(w / float(s16)), -7, 7) + 8,
// even k in the low nibble. Loop bounds are warp-uniform so every lane
// takes part in the shuffles. No early start of the next kernel, and the
// stores are published before the threads exit (see publish_packed_stores).
__global__ void __launch_bounds__(256) pack_q4_kernel(const __half* __restrict__ W,
                                                      int64_t nchunk,
                                                      uint32_t* __restrict__ P,
                                                      __half* __restrict__ S) {
  pdl_wait();
  const uint4* w4 = reinterpret_cast<const uint4*>(W);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x; base < nchunk;
       base += stride) {
    const int64_t c = base + threadIdx.x;
    const bool live = c < nchunk;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (live) v = ld_dep_v4(w4 + c);
    float a = absmax8(v);
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    const __half s16 = __float2half_rn(__fdiv_rn(a, 7.0f));
    const float sf = __half2float(s16);
    const __half* h = reinterpret_cast<const __half*>(&v);
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = 0;
      if (sf != 0.0f) q = max(-7, min(7, __float2int_rn(__fdiv_rn(__half2float(h[i]), sf))));
      word |= static_cast<uint32_t>(q + 8) << (4 * i);
    }
    if (live) {
      P[c] = word;
      if ((c & 3) == 0) S[c >> 2] = s16;
    }
  }
  publish_packed_stores();
}

}  // namespace aria
