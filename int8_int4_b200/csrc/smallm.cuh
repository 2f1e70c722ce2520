// smallm.cuh -- the few-token weight-only GEMM (M <= 16 tokens): q8, q4 and
// fp16 weights streamed from HBM once.
//
// "Results" (aria project page): the transformer's linears at q8 / q4 weight-
// only precision (and fp16); at a handful of tokens each call is a pass over
// the weights, so its speed is set by how fast they stream from HBM, and in a
// layer sequence by how much of that streaming overlaps the preceding layer.
//
// Work split: the N weight rows are divided into balanced ranges, one per
// cluster of S CTAs (S = 1: a lone CTA); the S CTAs of a cluster split K into
// equal slices. Every CTA copies all of its weight bytes (its rows x its K
// slice, plus the q4 group scales) into shared memory with bulk copies
// BEFORE the dependency wait of programmatic dependent launch, and lets its
// own successor start at once: the weight stream of a launch overlaps the
// tail of the preceding one. Only then does it wait, read the activations
// (L2-resident: just written by the preceding kernel) into registers, and
// run the products on the tensor cores with mma.sync m16n8k16: the 16-row
// operand is 16 weight rows, the 8-wide operand 8 tokens (two blocks of 8
// for 9..16 tokens), so no token padding beyond 8 / 16 is computed. The
// eight warps take interleaved 64-wide K chunks; their partial sums meet in
// shared memory and are added in warp order, and the S partials of a cluster
// in rank order through distributed shared memory (deterministic). The fused
// epilogue (q8 channel scale, bias, steering, one rounding to fp16) follows.
//
// Within a 64-wide K chunk, lane (g, q) = (lane / 4, lane % 4) holds the 16
// consecutive k values [16q, 16q + 16) of one weight row and of one token;
// m16n8k16 step j (0..3) takes values 4j .. 4j + 3 of them in the
// instruction's k positions {2q, 2q + 1, 2q + 8, 2q + 9}. The same
// permutation of k applies to both operands, so the dot products are
// unchanged and every operand load is a 16-byte vector.
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "qgemm.cuh"

namespace aria {

constexpr int kSmThreads = 256;
constexpr int kSmWarps = kSmThreads / 32;
// floats per (warp, token) row of the warp reduction for GP 16-row groups
// per pass: 16 GP + 4 makes the fragment stores bank-conflict-free
__host__ __device__ constexpr int sm_red_stride(int gp) { return gp * 16 + 4; }

struct SmallParams {
  int M, N, K;
  int S;                  // CTAs per cluster (K slices)
  int kslice;             // K elements per CTA (multiple of 64; of 256 for q4)
  int rows_base, rows_rem;  // cluster c owns rows_base + (c < rows_rem) rows
  int r_pad;              // 16-aligned maximum rows per cluster
  uint32_t wrow;          // shared-memory bytes per weight row (slice bytes + 16)
  uint32_t off_sc, off_red, off_part, off_bar, off_sw;  // shared-memory offsets (weights at 0)
  const uint8_t* W;       // q8 int8 [N,K]; q4 uint8 [N,K/2]; fp16 [N,K]
  const __half* Wsc;      // q4 group scales [N,K/32]
  const float* sw;        // q8 channel scales [N]
  const __half* X;        // [M,K]
  const __half* bias;     // [N] or null
  const float* steer;     // [N] or null
  int trace_launch;       // trace builds: the launch's index since the trace was cleared
  float alpha;
  const float* alpha_dev;
  __half* Y;              // [M,N]
};

template <int KIND>
struct SmallTraits {
  // bytes of one weight row per K element, as a ratio (q4: 1/2)
  static constexpr int kNum = KIND == kF16 ? 2 : 1;
  static constexpr int kDen = KIND == kQ4 ? 2 : 1;
};

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16 consecutive weights of one row (this lane's k values of a chunk) as 8
// fp16 pairs in k order. q8: int8 codes, exact (the channel scale is applied
// in the epilogue); q4: fp16((code - 8) * s16); fp16: as stored.
template <int KIND>
__device__ __forceinline__ void load_w16(const uint8_t* rowp, int kc, int q, uint32_t s2,
                                         uint32_t (&h)[8]) {
  if constexpr (KIND == kQ8) {
    const uint4 w = *reinterpret_cast<const uint4*>(rowp + kc * 64 + 16 * q);
    i8x4_to_h(w.x, h[0], h[1]);
    i8x4_to_h(w.y, h[2], h[3]);
    i8x4_to_h(w.z, h[4], h[5]);
    i8x4_to_h(w.w, h[6], h[7]);
  } else if constexpr (KIND == kQ4) {
    const uint2 w = *reinterpret_cast<const uint2*>(rowp + kc * 32 + 8 * q);
    const uint4 lo = nib8_to_h(w.x, s2);
    const uint4 hi = nib8_to_h(w.y, s2);
    h[0] = lo.x; h[1] = lo.y; h[2] = lo.z; h[3] = lo.w;
    h[4] = hi.x; h[5] = hi.y; h[6] = hi.z; h[7] = hi.w;
  } else {
    const uint4 a = *reinterpret_cast<const uint4*>(rowp + kc * 128 + 32 * q);
    const uint4 b = *reinterpret_cast<const uint4*>(rowp + kc * 128 + 32 * q + 16);
    h[0] = a.x; h[1] = a.y; h[2] = a.z; h[3] = a.w;
    h[4] = b.x; h[5] = b.y; h[6] = b.z; h[7] = b.w;
  }
}

// TB token blocks of 8 (M <= 8: 1; M <= 16: 2); CH: K chunks per warp held in
// registers (the planner keeps kslice / 64 / 8 <= CH); GP: 16-row groups
// accumulated in registers per pass over the chunks.
// At most 128 registers per thread (two CTAs per SM): a launch's CTAs can
// then sit beside those of the preceding launch while both stream weights.
template <int KIND, int TB, int CH, int GP>
__global__ void __launch_bounds__(kSmThreads, 2) smallm_kernel(const SmallParams p) {
  using Tr = SmallTraits<KIND>;
  extern __shared__ __align__(128) uint8_t sm[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, q = lane & 3;
  const int rank = p.S > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int cl = blockIdx.x / p.S;
  const int R = p.rows_base + (cl < p.rows_rem ? 1 : 0);
  const int r0 = cl * p.rows_base + min(cl, p.rows_rem);
  const int k0 = rank * p.kslice;
  const uint32_t slice_bytes = static_cast<uint32_t>(p.kslice) * Tr::kNum / Tr::kDen;
  const int64_t row_bytes = static_cast<int64_t>(p.K) * Tr::kNum / Tr::kDen;
  const uint32_t sc_bytes = KIND == kQ4 ? static_cast<uint32_t>(p.kslice / 32) * 2u : 0u;
  uint8_t* wsm = sm;
  __half* scs = reinterpret_cast<__half*>(sm + p.off_sc);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + p.off_bar);

  if (tid == 0) {
    ARIA_STAMP(0);
    mbar_init(bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(R) * (slice_bytes + sc_bytes));
  }
  __syncthreads();
  // ---- all weight bytes of this CTA, before the dependency wait: every
  // thread issues the bulk copies of its share of the rows (one warp issuing
  // them all serialises the requests)
  {
    const uint64_t pol = policy_evict_first();  // streamed once
    for (int r = tid; r < R; r += kSmThreads) {
      const int64_t n = r0 + r;
      bulk_g2s(wsm + r * p.wrow, p.W + n * row_bytes + static_cast<int64_t>(k0) * Tr::kNum / Tr::kDen,
               slice_bytes, bar, pol);
      if constexpr (KIND == kQ4)
        bulk_g2s(scs + r * (p.kslice / 32), p.Wsc + n * (p.K / 32) + k0 / 32, sc_bytes, bar, pol);
    }
  }
  // q8: the channel scales of the CTA's rows (part of the pack, like the
  // weights) into shared memory, also before the wait
  float* s_sw = reinterpret_cast<float*>(sm + p.off_sw);
  if constexpr (KIND == kQ8)
    for (int r = tid; r < R; r += kSmThreads) s_sw[r] = __ldg(p.sw + r0 + r);
  if (tid == 0) ARIA_STAMP(1);
  pdl_launch_dependents();  // the next launch may start streaming its own weights
  pdl_wait();               // X, the epilogue operands and Y belong to the stream order
  if (tid == 0) ARIA_STAMP(2);

  // ---- this warp's activation chunks into registers: token tb*8 + g4,
  // k values [k0 + 64c + 16q, +16) as two 16-byte vectors
  const int nch = p.kslice / 64;
  uint4 xa[CH][TB], xb[CH][TB];
#pragma unroll
  for (int i = 0; i < CH; ++i) {
    const int c = warp + i * kSmWarps;
#pragma unroll
    for (int tb = 0; tb < TB; ++tb) {
      const int t = tb * 8 + g4;
      xa[i][tb] = make_uint4(0u, 0u, 0u, 0u);
      xb[i][tb] = make_uint4(0u, 0u, 0u, 0u);
      if (c < nch && t < p.M) {
        const uint4* src = reinterpret_cast<const uint4*>(p.X + static_cast<int64_t>(t) * p.K + k0 + c * 64 + 16 * q);
        xa[i][tb] = ld_dep_v4(src);
        xb[i][tb] = ld_dep_v4(src + 1);
      }
    }
  }

  // ---- weights landed (bounded wait; on timeout the status word records it)
  if (!mbar_try_wait(bar, 0)) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, 0)) {
      if (globaltimer() - t0 > kWaitLimitNs) {
        atomicOr(&g_status, kStatusTimeout);
        atomicExch(&g_wait_site, 20u);
        mbar_wait_drain(bar, 0);  // the copies must land before shared memory is reused
        break;
      }
    }
  }
  if (tid == 0) ARIA_STAMP(3);

  constexpr int NT = TB * 8;  // tokens per warp tile
  const int groups = (R + 15) >> 4;
  constexpr int rs = sm_red_stride(GP);
  const int ps = p.r_pad + 4;                                     // cluster partial row stride
  float* red = reinterpret_cast<float*>(sm + p.off_red);         // [warp][token][rs]
  float* part = reinterpret_cast<float*>(sm + p.off_part);       // [token][ps]
  for (int gp = 0; gp < groups; gp += GP) {
    float acc[GP][TB][4];
#pragma unroll
    for (int gi = 0; gi < GP; ++gi)
#pragma unroll
      for (int tb = 0; tb < TB; ++tb)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[gi][tb][e] = 0.0f;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const int c = warp + i * kSmWarps;
      if (c >= nch) break;
#pragma unroll
      for (int gi = 0; gi < GP; ++gi) {
        const int g = gp + gi;
        if (g >= groups) break;
        const int ra = g * 16 + g4, rb = ra + 8;
        uint32_t ha[8], hb[8];
        uint32_t sa = 0u, sb = 0u;
        if constexpr (KIND == kQ4) {
          // this lane's 16 k values lie in group (64c + 16q) / 32 of the slice
          const int gi32 = c * 2 + (q >> 1);
          const uint16_t va = ra < R ? __half_as_ushort(scs[ra * (p.kslice / 32) + gi32]) : 0;
          const uint16_t vb = rb < R ? __half_as_ushort(scs[rb * (p.kslice / 32) + gi32]) : 0;
          sa = static_cast<uint32_t>(va) * 0x10001u;
          sb = static_cast<uint32_t>(vb) * 0x10001u;
        }
        if (ra < R) {
          load_w16<KIND>(wsm + ra * p.wrow, c, q, sa, ha);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) ha[e] = 0u;
        }
        if (rb < R) {
          load_w16<KIND>(wsm + rb * p.wrow, c, q, sb, hb);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) hb[e] = 0u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t a[4] = {ha[2 * j], hb[2 * j], ha[2 * j + 1], hb[2 * j + 1]};
#pragma unroll
          for (int tb = 0; tb < TB; ++tb) {
            const uint4& x = j < 2 ? xa[i][tb] : xb[i][tb];
            const uint32_t b0 = (j & 1) ? x.z : x.x;
            const uint32_t b1 = (j & 1) ? x.w : x.y;
            mma_16816(acc[gi][tb], a, b0, b1);
          }
        }
      }
    }
    // partial sums of this pass: red[warp][token][row]
    __syncthreads();  // the previous pass's reduction has read red
#pragma unroll
    for (int gi = 0; gi < GP; ++gi) {
      const int g = gp + gi;
      if (g >= groups) break;
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) {
        const int t = tb * 8 + 2 * q;
        const int row = (g - gp) * 16 + g4;
        float* base = red + (warp * NT + t) * rs;
        base[row] = acc[gi][tb][0];
        base[rs + row] = acc[gi][tb][1];
        base[row + 8] = acc[gi][tb][2];
        base[rs + row + 8] = acc[gi][tb][3];
      }
    }
    __syncthreads();
    // add the warps' partials in warp order: one output (token, row) per step
    const int prow = min(groups - gp, GP) * 16;
    for (int idx = tid; idx < NT * prow; idx += kSmThreads) {
      const int t = idx / prow, row = idx % prow;
      const int rl = gp * 16 + row;  // row within the cluster's range
      float s = 0.0f;
#pragma unroll
      for (int w = 0; w < kSmWarps; ++w) s += red[(w * NT + t) * rs + row];
      if (p.S > 1) {
        part[t * ps + rl] = s;
      } else if (t < p.M && rl < R) {
        const int n = r0 + rl;
        float y = s;
        if constexpr (KIND == kQ8) y = __fmul_rn(y, s_sw[rl]);
        if (p.bias) y = __fadd_rn(y, __half2float(p.bias[n]));
        if (p.steer) {
          const float a = p.alpha_dev ? *p.alpha_dev : p.alpha;
          if (a != 0.0f) y = __fmaf_rn(a, ld_dep_f32(p.steer + n), y);
        }
        p.Y[static_cast<int64_t>(t) * p.N + n] = __float2half_rn(y);
      }
    }
  }

  if (tid == 0) ARIA_STAMP(4);
  if (p.S > 1) {
    // rank r finishes rows [R*r/S, R*(r+1)/S) of the cluster's range: the S
    // partials through distributed shared memory, added in rank order
    cluster_sync();
    const int rb0 = R * rank / p.S, rb1 = R * (rank + 1) / p.S;
    const int nr = rb1 - rb0;
    if (tid == 0) ARIA_STAMP(5);
    const uint32_t part_u32 = smem_u32(sm + p.off_part);
    const float a = p.steer ? (p.alpha_dev ? *p.alpha_dev : p.alpha) : 0.0f;
    for (int idx = tid; idx < p.M * nr; idx += kSmThreads) {
      const int t = idx / nr, rl = rb0 + idx % nr;
      const uint32_t off = static_cast<uint32_t>((t * ps + rl) * 4);
      float s = 0.0f;
      for (int r = 0; r < p.S; ++r) s += __uint_as_float(ld_dsmem_u32(mapa_shared(part_u32 + off, r)));
      const int n = r0 + rl;
      float y = s;
      if constexpr (KIND == kQ8) y = __fmul_rn(y, s_sw[rl]);
      if (p.bias) y = __fadd_rn(y, __half2float(p.bias[n]));
      if (a != 0.0f) y = __fmaf_rn(a, ld_dep_f32(p.steer + n), y);
      p.Y[static_cast<int64_t>(t) * p.N + n] = __float2half_rn(y);
    }
    cluster_sync();  // no CTA leaves while a peer still reads its partials
  }
  if (tid == 0) ARIA_STAMP(6);
}

}  // namespace aria
