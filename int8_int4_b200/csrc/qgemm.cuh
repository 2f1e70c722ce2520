// qgemm.cuh -- quantized GEMMs on the 5th-generation tensor cores (tcgen05).
//
// "Results" (aria project page): the transformer runs at q8 or q4 weight-only
// precision, or as W8A8 with 8-bit arithmetic on integer tensor cores; the
// steering direction ("Steering is real") is added to one block's output.
//
// One kernel template serves all formats. Orientation is swapped: the MMA's
// 128-row A operand is a tile of 128 output channels (weight rows) and the
// MMA's N operand is a tile of BN tokens, so one kernel covers M = 1 .. 4096
// without padding the token dimension to 128. Both operands are K-major in
// the 128-byte swizzled shared-memory layout.
//
// Warp roles (256 threads, one CTA per SM):
//   warp 0      TMA producer of weight tiles (raw packed bytes for q8/q4, the
//               int8 A operand itself for W8A8)
//   warp 1      TMEM allocator and single-thread tcgen05.mma issuer
//   warp 2      TMA producer of activation tiles (fp16 for q8/q4, int8 W8A8)
//   warps 4..7  q8/q4: dequantise raw weights into fp16 A tiles (one weight
//               row per thread, exact int8->fp16, fp16 code*scale for q4);
//               then the epilogue: TMEM -> registers -> scale, bias, steer ->
//               fp16 stores (fp64 arithmetic for W8A8).
// Split-K: when the output tiles are too few to cover the SMs, a cluster of S
// CTAs shares one output tile, each taking a contiguous K range; partial
// accumulators are summed through distributed shared memory in fixed rank
// order (deterministic, no global scratch).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"

namespace aria {

enum GemmKind : int { kQ8 = 1, kQ4 = 2, kW8A8 = 3, kS32 = 4 };

constexpr int kGemmThreads = 256;
constexpr int kTileN = 128;            // weight rows per tile (MMA M)
constexpr uint32_t kATile = 16384;     // 128 rows x 128 bytes
constexpr uint32_t kQ4ScaleTile = 2048;  // 128 rows x 8 fp16 scales

struct GemmParams {
  int M, N, K;
  int BN;                 // tokens per tile (MMA N): multiple of 16, <= 256
  int units;              // K units: 128 (q8, W8A8) or 256 (q4) elements
  int splits;             // CTAs per cluster along K
  int n_raw, n_a, n_x;    // ring depths
  uint32_t off_raw, off_a, off_x, off_bar;
  uint32_t raw_stage, x_stage;
  uint32_t tmem_cols;
  const float* sw;        // per-channel weight scale (q8, W8A8)
  const float* sx;        // per-token activation scale (W8A8)
  const __half* bias;     // [N] or null
  const float* steer;     // [N] or null (null also when alpha == 0)
  float alpha;
  void* Y;                // fp16 [M,N], or int32 [M,N] for kS32
};

template <int KIND>
struct KindTraits {
  static constexpr bool kDequant = (KIND == kQ8 || KIND == kQ4);
  static constexpr bool kF16 = kDequant;                    // MMA kind::f16 vs kind::i8
  static constexpr int kKbPerUnit = KIND == kQ8 ? 2 : (KIND == kQ4 ? 4 : 1);
  static constexpr int kXElemsPerKb = kF16 ? 64 : 128;      // 128 bytes of K per row
};

// ---------------------------------------------------------------- dequant ---
__device__ __forceinline__ uint32_t h2_sub_mul(uint32_t v, uint32_t bias2, uint32_t s2) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  h = __hmul2(__hsub2(h, *reinterpret_cast<__half2*>(&bias2)), *reinterpret_cast<__half2*>(&s2));
  return *reinterpret_cast<uint32_t*>(&h);
}

// 4 signed bytes -> 4 fp16 (exact): 0x64XX is 1024 + XX, XX = byte ^ 0x80.
__device__ __forceinline__ void i8x4_to_h(uint32_t x, uint32_t& lo, uint32_t& hi) {
  const uint32_t xb = x ^ 0x80808080u;
  const uint32_t k1152 = 0x64806480u;  // {1152, 1152}
  uint32_t a = __byte_perm(xb, 0x64646464u, 0x4140);
  uint32_t b = __byte_perm(xb, 0x64646464u, 0x4342);
  __half2 ha = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<const __half2*>(&k1152));
  __half2 hb = __hsub2(*reinterpret_cast<__half2*>(&b), *reinterpret_cast<const __half2*>(&k1152));
  lo = *reinterpret_cast<uint32_t*>(&ha);
  hi = *reinterpret_cast<uint32_t*>(&hb);
}

// 8 offset-binary nibbles (k0 in bits 0..3) -> 8 fp16 values (code * s), in k order.
__device__ __forceinline__ uint4 nib8_to_h(uint32_t x, uint32_t s2) {
  const uint32_t magic = 0x64006400u;   // 1024 in both halves
  const uint32_t k1032 = 0x64086408u;   // {1032, 1032} = 1024 + offset 8
  const uint32_t a = (x & 0x000F000Fu) | magic;           // {k0, k4}
  const uint32_t b = ((x >> 4) & 0x000F000Fu) | magic;    // {k1, k5}
  const uint32_t c = ((x >> 8) & 0x000F000Fu) | magic;    // {k2, k6}
  const uint32_t d = ((x >> 12) & 0x000F000Fu) | magic;   // {k3, k7}
  uint4 r;
  r.x = h2_sub_mul(__byte_perm(a, b, 0x5410), k1032, s2);  // {k0, k1}
  r.y = h2_sub_mul(__byte_perm(c, d, 0x5410), k1032, s2);  // {k2, k3}
  r.z = h2_sub_mul(__byte_perm(a, b, 0x7632), k1032, s2);  // {k4, k5}
  r.w = h2_sub_mul(__byte_perm(c, d, 0x7632), k1032, s2);  // {k6, k7}
  return r;
}

// byte offset of 16-byte chunk j of row r in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw128(uint32_t r, uint32_t j) {
  return r * 128u + ((j ^ (r & 7u)) << 4);
}

// ---------------------------------------------------------------- epilogue --
template <int KIND>
__device__ __forceinline__ __half epi_value(uint32_t acc_bits, int m, int n, const GemmParams& p) {
  if constexpr (KIND == kW8A8) {
    // fp64: ((acc * s_x) * s_w) + bias + alpha*v, each step rounded once, no
    // contraction, then one rounding to fp16
    double t = __dmul_rn(__dmul_rn(static_cast<double>(static_cast<int32_t>(acc_bits)),
                                   static_cast<double>(__ldg(p.sx + m))),
                         static_cast<double>(__ldg(p.sw + n)));
    if (p.bias) t = __dadd_rn(t, static_cast<double>(__half2float(p.bias[n])));
    if (p.steer)
      t = __dadd_rn(t, __dmul_rn(static_cast<double>(p.alpha), static_cast<double>(__ldg(p.steer + n))));
    return __double2half(t);
  } else {
    float y = __uint_as_float(acc_bits);
    if constexpr (KIND == kQ8) y = __fmul_rn(y, __ldg(p.sw + n));
    if (p.bias) y = __fadd_rn(y, __half2float(p.bias[n]));
    if (p.steer) y = __fmaf_rn(p.alpha, __ldg(p.steer + n), y);
    return __float2half_rn(y);
  }
}

template <int KIND>
__device__ __forceinline__ uint32_t reduce_add(uint32_t a, uint32_t b) {
  if constexpr (KIND == kW8A8 || KIND == kS32)
    return static_cast<uint32_t>(static_cast<int32_t>(a) + static_cast<int32_t>(b));
  else
    return __float_as_uint(__uint_as_float(a) + __uint_as_float(b));
}

// ------------------------------------------------------------------ kernel --
template <int KIND>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmS,
                 const __grid_constant__ CUtensorMap tmX, const GemmParams p) {
  using T = KindTraits<KIND>;
  extern __shared__ uint8_t dyn_smem[];
  // 1024-byte alignment of the shared-window address (128-byte swizzle atoms)
  const uint32_t base_u32 = smem_u32(dyn_smem);
  uint8_t* smem = dyn_smem + (((base_u32 + 1023u) & ~1023u) - base_u32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = p.splits > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int n0 = blockIdx.y * kTileN;
  const int m0 = blockIdx.z * p.BN;
  const int u_begin = static_cast<int>(static_cast<int64_t>(p.units) * rank / p.splits);
  const int u_end = static_cast<int>(static_cast<int64_t>(p.units) * (rank + 1) / p.splits);
  const int nu = u_end - u_begin;
  const int nkb = nu * T::kKbPerUnit;

  uint8_t* raw = smem + p.off_raw;
  uint8_t* abuf = smem + p.off_a;
  uint8_t* xbuf = smem + p.off_x;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + p.n_raw;
  uint64_t* a_full = raw_empty + p.n_raw;
  uint64_t* a_empty = a_full + p.n_a;
  uint64_t* x_full = a_empty + p.n_a;
  uint64_t* x_empty = x_full + p.n_x;
  uint64_t* acc_full = x_empty + p.n_x;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.n_raw; ++i) {
      mbar_init(raw_full + i, 1);
      mbar_init(raw_empty + i, 128);
    }
    for (int i = 0; i < p.n_a; ++i) {
      mbar_init(a_full + i, T::kDequant ? 128 : 1);
      mbar_init(a_empty + i, 1);
    }
    for (int i = 0; i < p.n_x; ++i) {
      mbar_init(x_full + i, 1);
      mbar_init(x_empty + i, 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
    if constexpr (KIND == kQ4) prefetch_tmap(&tmS);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // counters kept for the teardown drain of copies in flight
  int issued_w = 0, issued_x = 0;

  if (warp == 0) {
    // ------------------------------------------------ weight tile producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();  // weights are read once
      if constexpr (T::kDequant) {
        for (int i = 0; i < nu; ++i) {
          const int s = i % p.n_raw;
          const uint32_t ph = (i / p.n_raw) & 1;
          if (!mbar_wait(raw_empty + s, ph ^ 1, abort_flag, 1)) break;
          uint8_t* dst = raw + s * p.raw_stage;
          const int u = u_begin + i;
          if constexpr (KIND == kQ8) {
            mbar_arrive_expect_tx(raw_full + s, kATile);
            tma_load_2d(&tmW, raw_full + s, dst, u * 128, n0, pol);
          } else {
            mbar_arrive_expect_tx(raw_full + s, kATile + kQ4ScaleTile);
            tma_load_2d(&tmW, raw_full + s, dst, u * 128, n0, pol);       // 256 k as bytes
            tma_load_2d(&tmS, raw_full + s, dst + kATile, u * 8, n0, pol);  // 8 group scales
          }
          ++issued_w;
        }
      } else {
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = kb % p.n_a;
          const uint32_t ph = (kb / p.n_a) & 1;
          if (!mbar_wait(a_empty + s, ph ^ 1, abort_flag, 2)) break;
          mbar_arrive_expect_tx(a_full + s, kATile);
          tma_load_2d(&tmW, a_full + s, abuf + s * kATile, (u_begin + kb) * 128, n0, pol);
          ++issued_w;
        }
      }
    }
  } else if (warp == 2) {
    // -------------------------------------------- activation tile producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();   // re-read by every weight tile
      const int kx0 = u_begin * T::kKbPerUnit;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % p.n_x;
        const uint32_t ph = (kb / p.n_x) & 1;
        if (!mbar_wait(x_empty + s, ph ^ 1, abort_flag, 3)) break;
        mbar_arrive_expect_tx(x_full + s, p.x_stage);
        tma_load_2d(&tmX, x_full + s, xbuf + s * p.x_stage, (kx0 + kb) * T::kXElemsPerKb, m0, pol);
        ++issued_x;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = T::kF16 ? idesc_f16_f32(p.BN) : idesc_s8_s32(p.BN);
      bool ok = true;
      for (int kb = 0; kb < nkb && ok; ++kb) {
        const int sa = kb % p.n_a, sx = kb % p.n_x;
        ok = mbar_wait(a_full + sa, (kb / p.n_a) & 1, abort_flag, 4) &&
             mbar_wait(x_full + sx, (kb / p.n_x) & 1, abort_flag, 5);
        if (!ok) break;
        tc_fence_after();
        const uint64_t ad = sdesc_sw128(smem_u32(abuf + sa * kATile));
        const uint64_t bd = sdesc_sw128(smem_u32(xbuf + sx * p.x_stage));
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // 4 x 32 bytes of K per 128-byte block
          if constexpr (T::kF16)
            umma_f16(tmem_base, ad + 2 * j, bd + 2 * j, idesc, (kb | j) != 0);
          else
            umma_i8(tmem_base, ad + 2 * j, bd + 2 * j, idesc, (kb | j) != 0);
        }
        umma_commit(a_empty + sa);
        umma_commit(x_empty + sx);
      }
      umma_commit(acc_full);  // also fires when nothing was issued
    }
  } else if (warp >= 4) {
    const int t = threadIdx.x - 128;  // weight row within the tile == TMEM lane
    bool ok = true;
    if constexpr (T::kDequant) {
      // ------------------------------------------------------ dequantise
      int ia = 0;
      for (int i = 0; i < nu && ok; ++i) {
        const int s = i % p.n_raw;
        if (!(ok = mbar_wait(raw_full + s, (i / p.n_raw) & 1, abort_flag, 6))) break;
        const uint8_t* src = raw + s * p.raw_stage;
        uint4 v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c)
          v[c] = *reinterpret_cast<const uint4*>(src + sw128(t, c));
        uint4 sc = make_uint4(0, 0, 0, 0);
        if constexpr (KIND == kQ4) sc = *reinterpret_cast<const uint4*>(src + kATile + t * 16);
        mbar_arrive(raw_empty + s);
        constexpr int kHalves = T::kKbPerUnit;  // A tiles produced per raw stage
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
          const int sa = ia % p.n_a;
          if (!(ok = mbar_wait(a_empty + sa, ((ia / p.n_a) & 1) ^ 1, abort_flag, 7))) break;
          uint8_t* dst = abuf + sa * kATile;
          if constexpr (KIND == kQ8) {
            // raw chunks 4h..4h+3 (16 int8 each) -> fp16 chunks 0..7 of this tile
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint4 w = v[4 * h + cc];
              uint4 o0, o1;
              i8x4_to_h(w.x, o0.x, o0.y);
              i8x4_to_h(w.y, o0.z, o0.w);
              i8x4_to_h(w.z, o1.x, o1.y);
              i8x4_to_h(w.w, o1.z, o1.w);
              *reinterpret_cast<uint4*>(dst + sw128(t, 2 * cc)) = o0;
              *reinterpret_cast<uint4*>(dst + sw128(t, 2 * cc + 1)) = o1;
            }
          } else {
            // raw chunks 2h, 2h+1 (one 32-k group each) -> fp16 chunks 0..7
            const uint32_t* scw = reinterpret_cast<const uint32_t*>(&sc);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int c = 2 * h + g;
              const uint32_t spair = scw[c >> 1];
              const uint32_t s2 = (c & 1) ? __byte_perm(spair, 0, 0x3232) : __byte_perm(spair, 0, 0x1010);
              const uint4 w = v[c];
              *reinterpret_cast<uint4*>(dst + sw128(t, 4 * g + 0)) = nib8_to_h(w.x, s2);
              *reinterpret_cast<uint4*>(dst + sw128(t, 4 * g + 1)) = nib8_to_h(w.y, s2);
              *reinterpret_cast<uint4*>(dst + sw128(t, 4 * g + 2)) = nib8_to_h(w.z, s2);
              *reinterpret_cast<uint4*>(dst + sw128(t, 4 * g + 3)) = nib8_to_h(w.w, s2);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(a_full + sa);
          ++ia;
        }
      }
    }
    // ----------------------------------------------------------- epilogue
    ok = mbar_wait(acc_full, 0, abort_flag, 8);
    ok = __all_sync(0xffffffffu, ok);  // warp-uniform before .sync.aligned TMEM loads
    tc_fence_after();
    const uint32_t trow = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int n = n0 + t;
    if (p.splits == 1) {
      if (ok) {
        for (int cb = 0; cb < p.BN / 16; ++cb) {
          uint32_t r[16];
          tmem_ld16(trow + cb * 16, r);
          tmem_ld_wait();
          if (n < p.N) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int m = m0 + cb * 16 + i;
              if (m < p.M) {
                if constexpr (KIND == kS32)
                  reinterpret_cast<int32_t*>(p.Y)[static_cast<int64_t>(m) * p.N + n] = static_cast<int32_t>(r[i]);
                else
                  reinterpret_cast<__half*>(p.Y)[static_cast<int64_t>(m) * p.N + n] = epi_value<KIND>(r[i], m, n, p);
              }
            }
          }
        }
      }
    } else {
      // partial tile -> own shared memory, red[m_local][128] (32-bit words)
      fence_proxy_async_smem();
      uint32_t* red = reinterpret_cast<uint32_t*>(smem);
      for (int cb = 0; cb < p.BN / 16; ++cb) {
        uint32_t r[16];
        tmem_ld16(trow + cb * 16, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) red[(cb * 16 + i) * 128 + t] = ok ? r[i] : 0u;
      }
    }
  }

  // ------------------------------------------- split-K: cluster reduction
  if (p.splits > 1) {
    __syncwarp();
    cluster_sync();
    if (warp >= 4) {
      const int t = threadIdx.x - 128;
      const int mb = p.BN * rank / p.splits, me = p.BN * (rank + 1) / p.splits;
      const uint32_t red_u32 = smem_u32(smem);
      const int items = (me - mb) * 32;
      for (int it = t; it < items; it += 128) {
        const int ml = mb + (it >> 5);
        const int nl = (it & 31) * 4;
        const uint32_t off = red_u32 + static_cast<uint32_t>((ml * 128 + nl) * 4);
        uint4 acc = ld_dsmem_v4(mapa_shared(off, 0));
        for (int q = 1; q < p.splits; ++q) {
          const uint4 v = ld_dsmem_v4(mapa_shared(off, q));
          acc.x = reduce_add<KIND>(acc.x, v.x);
          acc.y = reduce_add<KIND>(acc.y, v.y);
          acc.z = reduce_add<KIND>(acc.z, v.z);
          acc.w = reduce_add<KIND>(acc.w, v.w);
        }
        const int m = m0 + ml, n = n0 + nl;
        if (m < p.M && n < p.N) {  // N % 16 == 0: all four columns are in range
          const int64_t o = static_cast<int64_t>(m) * p.N + n;
          if constexpr (KIND == kS32) {
            *reinterpret_cast<uint4*>(reinterpret_cast<int32_t*>(p.Y) + o) = acc;
          } else {
            __half h[4] = {epi_value<KIND>(acc.x, m, n, p), epi_value<KIND>(acc.y, m, n + 1, p),
                           epi_value<KIND>(acc.z, m, n + 2, p), epi_value<KIND>(acc.w, m, n + 3, p)};
            *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(p.Y) + o) = *reinterpret_cast<uint2*>(h);
          }
        }
      }
    }
    __syncwarp();
    cluster_sync();
  }

  // ---------------------------------------------------------------- teardown
  if (*abort_flag && lane == 0) {
    // drain copies still in flight into this CTA's shared memory
    if (warp == 0) {
      const int nring = T::kDequant ? p.n_raw : p.n_a;
      uint64_t* full = T::kDequant ? raw_full : a_full;
      for (int i = (issued_w > nring ? issued_w - nring : 0); i < issued_w; ++i)
        mbar_wait_drain(full + (i % nring), (i / nring) & 1);
    } else if (warp == 2) {
      for (int i = (issued_x > p.n_x ? issued_x - p.n_x : 0); i < issued_x; ++i)
        mbar_wait_drain(x_full + (i % p.n_x), (i / p.n_x) & 1);
    } else if (warp == 1) {
      mbar_wait_drain(acc_full, 0);  // MMAs issued before the abort have finished
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace aria
