// qgemm.cuh -- quantized GEMMs on the 5th-generation tensor cores (tcgen05).
//
// "Results" (aria project page): the transformer runs at fp16, at q8 or q4
// weight-only precision, or as W8A8 with 8-bit arithmetic on integer tensor
// cores; the steering direction ("Steering is real") is added to one block's
// output, with a strength that may live in device memory so that a captured
// graph follows a schedule ("Live steering while streaming").
//
// One kernel template serves all formats. Orientation is swapped: the MMA's
// 128-row A operand is a tile of 128 output channels (weight rows) and the
// MMA's N operand is a tile of BN tokens, so one kernel covers M = 1 .. 4096
// without padding the token dimension to 128. Both operands are K-major in
// the 128-byte swizzled shared-memory layout.
//
// Persistent, warp-specialised CTA (one per SM). The producer and MMA roles
// run as converged warps: every lane waits on the barriers, one lane issues
// (TMA by lane 0, tcgen05.mma / commit by elect.sync), which keeps the issue
// loops on the uniform datapath.
//   warp 0       TMA producer of weight tiles (raw packed bytes for q8/q4; for
//                W8A8 and fp16 the weight and activation tiles of each stage). The
//                first ring of weight tiles is loaded before the wait on the
//                preceding kernel (programmatic dependent launch).
//   warp 1       TMEM allocator (two accumulator buffers) and MMA issuer
//   warp 2       q8/q4: TMA producer of activation tiles
//   warps 4..7   epilogue: TMEM -> registers -> scale, bias, steer -> fp16 ->
//                transposed through shared memory -> coalesced 16-byte stores;
//                overlaps the next tile's mainloop through the second
//                accumulator buffer (W8A8 and fp16 use warps 8..11 for it as well)
//   warps 8..11  q8/q4: dequantise raw weights into fp16 A tiles (one weight
//                row per thread; exact int8 -> fp16; fp16 code*scale for q4);
//                they take part in the epilogue of the CTA's last tile. When
//                each CTA has one tile, the A tiles are written to tensor
//                memory (tcgen05.st, a row per TMEM lane) and the MMA reads A
//                from there: shared memory then holds only the activation and
//                raw-weight rings, which can be nearly twice as deep; for
//                q4, warps 4..7, idle until the tile's accumulator is
//                complete, dequantise the odd K blocks while warps 8..11
//                take the even ones
// Rings of shared-memory stages with mbarriers connect the roles; every wait
// is bounded. Split-K (few output tiles): a cluster of S CTAs shares one tile,
// each taking a contiguous K range; all warps then sum the partial
// accumulators through distributed shared memory in fixed rank order
// (deterministic, no global scratch).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"
#include "quant_kernels.cuh"

namespace aria {

enum GemmKind : int { kQ8 = 1, kQ4 = 2, kW8A8 = 3, kS32 = 4, kF16 = 5 };

constexpr int kTileN = 128;              // weight rows per tile (MMA M)
constexpr uint32_t kATile = 16384;       // 128 rows x 128 bytes
constexpr uint32_t kQ4ScaleTile = 2048;  // 128 rows x 8 fp16 scales
constexpr uint32_t kAccCols = 256;       // TMEM columns per accumulator buffer
constexpr int kEpiRows = 16;             // tokens per epilogue store box
constexpr int kTileBnMax = 256;          // largest token tile (MMA N)
constexpr int kL2Ahead = 4;              // weight units prefetched into L2 ahead of the TMA loads

struct GemmParams {
  int M, N, K;
  int BN;                 // tokens per tile (MMA N): multiple of 16, <= 256
  int units;              // K units: 128 (q8, W8A8), 256 (q4) or 64 (fp16) elements
  int splits;             // CTAs per cluster along K (1 = persistent over tiles)
  int tiles_n, tiles;     // weight-row tiles, total output tiles
  int n_raw, n_a, n_x;    // ring depths (raw packed weights; stages of A + X; n_x == n_a)
  uint32_t off_raw, off_a, off_x, off_stage, off_sxd, off_bar;
  uint32_t raw_stage, x_stage;
  const float* sw;        // per-channel weight scale (q8, W8A8)
  const float* sx;        // per-token activation scale (W8A8)
  const __half* bias;     // [N] or null
  const float* steer;     // [N] or null (null also when a host alpha is 0)
  float alpha;
  const float* alpha_dev; // device alpha, read after the dependency wait; null: use `alpha`
  // W8A8 with the activation quantisation in the same launch (null: X is
  // already quantised): fp16 X, and the workspace that receives its codes
  // and token scales (read back through tmX and sx) and holds the grid
  // barrier {arrivals, generation}
  const __half* xf16;
  int8_t* xq_ws;
  float* sx_ws;
  unsigned* gbar;
  // failure-detection self-test: the limit of every bounded wait (0: the
  // default kWaitLimitNs) and, for W8A8 / fp16, a hook that withholds the
  // first stage of each CTA's first tile so that the waits on it run out
  uint64_t wait_ns;
  int drop_first_stage;
  // q8/q4 with one tile per CTA: the dequantised weights (the MMA's A
  // operand) go to tensor memory, columns [kAccCols + 32 s, +32) for stage s,
  // instead of shared memory; the accumulator keeps columns [0, BN)
  int tmem_a;
  // the CTA's last tile: warps 0..3, done with their roles, take a third of
  // its epilogue chunks (their store boxes fit in the activation ring)
  int helpers;
  int trace_launch;       // trace builds: the launch's index since the trace was cleared
  void* Y;                // fp16 [M,N], or int32 [M,N] for kS32 (split-K path)
};

template <int KIND>
struct KindTraits {
  static constexpr bool kDequant = (KIND == kQ8 || KIND == kQ4);
  static constexpr bool kMmaF16 = kDequant || KIND == kF16; // MMA kind::f16 vs kind::i8
  static constexpr int kKbPerUnit = KIND == kQ8 ? 2 : (KIND == kQ4 ? 4 : 1);
  static constexpr int kXElemsPerKb = kMmaF16 ? 64 : 128;   // 128 bytes of K per row
  // x coordinate step of one K unit in the weight tensor map: 128 bytes of
  // packed weights (q8, q4, W8A8) or 64 fp16 weights (fp16)
  static constexpr int kWUnitX = KIND == kF16 ? 64 : 128;
  static constexpr int kThreads = 384;
  static constexpr int kEpiWarps = kDequant ? 4 : 8;   // W8A8 / S32 / fp16 use warps 8..11 for the epilogue too
  static constexpr uint32_t kOutBytes = KIND == kS32 ? 4 : 2;
  static constexpr uint32_t kStageBuf = kEpiRows * 32 * kOutBytes;  // one warp's store box
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
// Per output channel n (one per epilogue thread), the constants of the fused
// epilogue, loaded once per tile.
template <int KIND>
struct RowConst {
  float sw = 0.0f, bias = 0.0f, alpha = 0.0f, v = 0.0f;  // all formats (W8A8: fp32 copies)
  float av_hi = 0.0f, av_lo = 0.0f;                      // W8A8: alpha*v = av_hi + av_lo exactly
  float sw_up = 0.0f, sw_dn = 0.0f;                      // W8A8: sw * (1 +- 2^-22), rounded
  bool has_bias = false, has_steer = false;
};

// The steering strength of this launch: the host value, or the device value
// (read after the dependency wait, so a preceding kernel may have written
// it). A zero strength skips the add entirely, which keeps the output
// bit-identical to an unsteered call.
__device__ __forceinline__ float steer_alpha(const GemmParams& p) {
  return p.alpha_dev ? *p.alpha_dev : p.alpha;
}

// The per-channel inputs of the epilogue as loaded (no arithmetic on them
// yet), so that a CTA can issue the loads for its next tile early and use
// them a tile later.
struct RowRaw {
  float sw = 0.0f, v = 0.0f;
  unsigned short bias = 0;  // fp16 bits
};

template <int KIND>
__device__ __forceinline__ RowRaw row_raw(int n, const GemmParams& p) {
  RowRaw r;
  if (n >= p.N) return r;
  if constexpr (KIND == kW8A8 || KIND == kQ8) r.sw = __ldg(p.sw + n);
  if (p.bias) r.bias = __half_as_ushort(p.bias[n]);
  if (p.steer) r.v = ld_dep_f32(p.steer + n);
  return r;
}

// `alpha`: the launch's steering strength (steer_alpha), 0 without steering
template <int KIND>
__device__ __forceinline__ RowConst<KIND> row_const_from(const RowRaw& r, int n, const GemmParams& p,
                                                        float alpha) {
  RowConst<KIND> c;
  if (n >= p.N) return c;
  c.has_bias = p.bias != nullptr;
  c.has_steer = p.steer != nullptr && alpha != 0.0f;
  if constexpr (KIND == kW8A8) {
    c.sw = r.sw;
    c.sw_up = __fmul_rn(c.sw, 1.0f + 0x1p-22f);
    c.sw_dn = __fmul_rn(c.sw, 1.0f - 0x1p-22f);
    if (c.has_bias) c.bias = __half2float(__ushort_as_half(r.bias));
    if (c.has_steer) {
      c.alpha = alpha;
      c.v = r.v;
      c.av_hi = __fmul_rn(c.alpha, c.v);
      c.av_lo = __fmaf_rn(c.alpha, c.v, -c.av_hi);  // exact remainder of the product
    }
  } else {
    if constexpr (KIND == kQ8) c.sw = r.sw;
    if (c.has_bias) c.bias = __half2float(__ushort_as_half(r.bias));
    if (c.has_steer) {
      c.alpha = alpha;
      c.v = r.v;
    }
  }
  return c;
}

template <int KIND>
__device__ __forceinline__ RowConst<KIND> row_const(int n, const GemmParams& p) {
  return row_const_from<KIND>(row_raw<KIND>(n, p), n, p, p.steer ? steer_alpha(p) : 0.0f);
}

// W8A8 reference sequence: ((acc * s_x) * s_w) + bias + alpha*v in fp64, each
// step rounded once (no contraction), then one rounding to fp16.
__device__ __noinline__ __half epi_w8a8_fp64(int32_t acc, float sx, float sw, float bias, float alpha,
                                             float v, bool has_bias, bool has_steer) {
  double t = __dmul_rn(__dmul_rn(static_cast<double>(acc), static_cast<double>(sx)),
                       static_cast<double>(sw));
  if (has_bias) t = __dadd_rn(t, static_cast<double>(bias));
  if (has_steer)  // a product of two fp32 values is exact in fp64
    t = __dadd_rn(t, __dmul_rn(static_cast<double>(alpha), static_cast<double>(v)));
  return __double2half(t);
}

// Knuth's two-sum: s + e == a + b exactly
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
  s = __fadd_rn(a, b);
  const float bb = __fsub_rn(s, a);
  e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}

// The same value, rounded to fp16, without fp64 arithmetic. The exact real
// value E = acc*s_x*s_w + bias + alpha*v is carried as an unevaluated sum
// yh + yl of two fp32 numbers (error-free products by fma, error-free sums by
// two-sum), accurate to about 2^-46 relative. Rounding E to fp16 then needs
// only yh, except when yh lies exactly on a midpoint between two fp16
// values, where the sign of yl decides. The result equals the fp64
// reference except if E lies within ~2^-46 of an fp16 midpoint (both are
// then within one fp16 ulp). |acc| >= 2^22 takes the fp64 sequence.
//
// w8a8_round() is the straight-line common path: it returns RN16(yh) and
// sets `rare` when the result may need the midpoint fix-up (or the fp64
// path), which w8a8_fixup() then applies. Keeping the common path free of
// branches lets a chunk of elements be evaluated interleaved.
struct W8A8Val {
  float yh, yl;
};

__device__ __forceinline__ __half w8a8_round(int32_t acc, float sx, const RowConst<kW8A8>& c,
                                             W8A8Val& v, bool& rare) {
  const float a = __fsub_rn(__int_as_float(acc + 0x4B400000), 12582912.0f);  // exact if |acc| < 2^22
  const float ph = __fmul_rn(sx, c.sw);
  const float pl = __fmaf_rn(sx, c.sw, -ph);        // sx*sw == ph + pl
  float yh = __fmul_rn(a, ph);
  float yl = __fmaf_rn(a, ph, -yh);                 // a*ph == yh + yl
  yl = __fmaf_rn(a, pl, yl);                        // + a*pl (error ~2^-48 |yh|)
  float e;
  if (c.has_bias) {
    two_sum(yh, c.bias, yh, e);
    yl = __fadd_rn(yl, e);
  }
  if (c.has_steer) {
    two_sum(yh, c.av_hi, yh, e);
    yl = __fadd_rn(yl, __fadd_rn(e, c.av_lo));
  }
  const float s = __fadd_rn(yh, yl);                // renormalise: |yl| <= ulp(yh)/2
  yl = __fsub_rn(yl, __fsub_rn(s, yh));
  yh = s;
  v.yh = yh;
  v.yl = yl;
  // An fp32 value can sit exactly on an fp16 rounding midpoint only if the 13
  // bits below fp16 precision read 1000000000000 (fp16-normal range), or if it
  // lies in the fp16-subnormal range.
  const uint32_t yb = __float_as_uint(yh) & 0x7FFFFFFFu;
  rare = (yl != 0.0f && ((yb & 0x1FFFu) == 0x1000u || yb < 0x38800000u)) ||
         acc <= -(1 << 22) || acc >= (1 << 22);
  return __float2half_rn(yh);
}

__device__ __noinline__ __half w8a8_fixup(__half h, int32_t acc, float sx, float sw, float bias,
                                          float alpha, float v, bool has_bias, bool has_steer,
                                          float yh, float yl) {
  if (acc <= -(1 << 22) || acc >= (1 << 22))
    return epi_w8a8_fp64(acc, sx, sw, bias, alpha, v, has_bias, has_steer);
  // midpoint case: |yh| exactly halfway between |h| and its neighbour
  const float ay = fabsf(yh);
  const float yl_away = yh < 0.0f ? -yl : yl;       // yl measured away from zero
  if (ay == 65520.0f) {
    // the midpoint between the largest finite value and overflow: the
    // conversion ties up to infinity, but a value just below it (yl pointing
    // toward zero) rounds to the largest finite magnitude 65504
    if (yl_away < 0.0f)
      return __ushort_as_half(static_cast<unsigned short>((__half_as_ushort(h) & 0x8000u) | 0x7BFFu));
    return h;
  }
  const float ar = fabsf(__half2float(h));
  const float d = __fsub_rn(ay, ar);                // exact (Sterbenz, or ar == 0)
  if (d != 0.0f && ar < 65504.0f) {
    const uint32_t hb = __half_as_ushort(h) & 0x7FFFu;
    float half_gap;
    if (hb < 0x0400u) {
      half_gap = 0x1p-25f;                          // zero / subnormal spacing 2^-24
    } else {
      const int e16 = static_cast<int>(hb >> 10) - 15;
      const bool down_binade = (d < 0.0f) && ((hb & 0x3FFu) == 0u) && hb > 0x0400u;
      half_gap = ldexpf(1.0f, e16 - (down_binade ? 12 : 11));
    }
    if (fabsf(d) == half_gap) {
      // yh on the midpoint: yl != 0 decides the side; with yl == 0 the value
      // is the midpoint itself and the conversion's tie-to-even stands
      if (yl_away != 0.0f && (yl_away > 0.0f) == (d > 0.0f)) {
        const uint32_t nb = d > 0.0f ? hb + 1u : hb - 1u;
        h = __ushort_as_half(static_cast<unsigned short>((__half_as_ushort(h) & 0x8000u) | nb));
      }
    }
  }
  return h;
}

// No bias and no steering. With t = fl(fl(acc) * s_x), the two products
// y_up = fl(t * fl(s_w (1 + 2^-22))) and y_dn = fl(t * fl(s_w (1 - 2^-22)))
// bracket the reference value E = fl64(fl64(acc * s_x) * s_w): for
// |acc| < 2^24 (fl(acc) exact) the three fp32 roundings on each side (t, the
// scaled s_w, the product) move a value by at most 3 * 2^-24 relative, and
// E differs from the exact product by about 2^-52: less than the 2^-22
// margin. Rounding to fp16 is monotonic, so if y_up and y_dn round to the
// same fp16 value, E does too. One packed conversion rounds both; the halves
// differ for about 0.07 % of elements (E near an fp16 rounding midpoint),
// which the caller recomputes with the fp64 sequence, as it does for
// |acc| >= 2^24 (w8a8_acc_big).
__device__ __forceinline__ uint32_t w8a8_plain_pair(int32_t acc, float sx, float sw_up, float sw_dn) {
  const float t = __fmul_rn(__int2float_rn(acc), sx);
  const float yu = __fmul_rn(t, sw_up);
  const float yd = __fmul_rn(t, sw_dn);
  uint32_t pk;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(pk) : "f"(yu), "f"(yd));
  return pk;  // low half RN16(y_dn), high half RN16(y_up)
}

__device__ __forceinline__ bool pair_split(uint32_t pk) { return (pk >> 16) != (pk & 0xFFFFu); }

__device__ __forceinline__ bool w8a8_acc_big(int32_t acc) {
  return static_cast<uint32_t>(acc) + (1u << 24) >= (1u << 25);  // |acc| >= 2^24
}

__device__ __forceinline__ __half epi_w8a8(int32_t acc, float sx, const RowConst<kW8A8>& c) {
  W8A8Val v;
  bool rare;
  const __half h = w8a8_round(acc, sx, c, v, rare);
  if (!rare) return h;
  return w8a8_fixup(h, acc, sx, c.sw, c.bias, c.alpha, c.v, c.has_bias, c.has_steer, v.yh, v.yl);
}

// q8 / q4 / fp16: fp32, (acc * s_w) (q8 only) + bias, then + alpha*v[n] (one
// fma), one rounding to fp16
template <int KIND>
__device__ __forceinline__ __half epi_wo(float acc, const RowConst<KIND>& c) {
  float y = acc;
  if constexpr (KIND == kQ8) y = __fmul_rn(y, c.sw);
  if (c.has_bias) y = __fadd_rn(y, c.bias);
  if (c.has_steer) y = __fmaf_rn(c.alpha, c.v, y);
  return __float2half_rn(y);
}

template <int KIND>
__device__ __forceinline__ uint32_t reduce_add(uint32_t a, uint32_t b) {
  if constexpr (KIND == kW8A8 || KIND == kS32)
    return static_cast<uint32_t>(static_cast<int32_t>(a) + static_cast<int32_t>(b));
  else
    return __float_as_uint(__uint_as_float(a) + __uint_as_float(b));
}

// Epilogue of one 16-column chunk for the calling warp, in two halves so the
// caller can release the accumulator buffer between them.
// compute: TMEM (row base `tacc` = this warp's 32 lanes of the buffer) ->
// registers -> scale / bias / steer -> fp16 -> 32x16 box in `sbuf`.
template <int KIND>
__device__ __forceinline__ void epilogue_chunk_compute(int c, uint32_t tacc, int lane, uint8_t* sbuf,
                                                       const RowConst<KIND>& rc, const float* sxs) {
    uint32_t r[16];
    tmem_ld16(tacc + c * 16, r);
    // transpose the warp's 32 channels x 16 tokens through shared memory
    // ([16][32] box), then coalesced 16-byte stores along the channels.
    // All shared-memory reads come before the first store into the box, and
    // the 16 results are computed into registers first, so the elements are
    // independent instruction streams.
    __half h[16];
    if constexpr (KIND == kW8A8) {
      float sxv[16];  // the chunk's 16 token scales, read while the TMEM load is in flight
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 f = reinterpret_cast<const float4*>(sxs + c * 16)[q];
        sxv[4 * q + 0] = f.x;
        sxv[4 * q + 1] = f.y;
        sxv[4 * q + 2] = f.z;
        sxv[4 * q + 3] = f.w;
      }
      tmem_ld_wait();
      // common path, straight-line over the chunk; each lane then redoes its
      // own flagged elements (registers selected by index, no TMEM re-read)
      uint32_t rare_mask = 0;
      if (!rc.has_bias && !rc.has_steer) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t pk = w8a8_plain_pair(static_cast<int32_t>(r[i]), sxv[i], rc.sw_up, rc.sw_dn);
          h[i] = __ushort_as_half(static_cast<unsigned short>(pk & 0xFFFFu));
          rare_mask |= static_cast<uint32_t>(pair_split(pk) | w8a8_acc_big(static_cast<int32_t>(r[i]))) << i;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          bool rare;
          W8A8Val vv;
          h[i] = w8a8_round(static_cast<int32_t>(r[i]), sxv[i], rc, vv, rare);
          rare_mask |= static_cast<uint32_t>(rare) << i;
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) reinterpret_cast<__half*>(sbuf)[i * 32 + lane] = h[i];
      while (rare_mask) {
        const int i = __ffs(rare_mask) - 1;
        rare_mask &= rare_mask - 1;
        uint32_t a1 = r[0];
        float sxi = sxv[0];
#pragma unroll
        for (int k = 1; k < 16; ++k) {
          if (k == i) {
            a1 = r[k];
            sxi = sxv[k];
          }
        }
        __half hv;
        if (!rc.has_bias && !rc.has_steer) {
          hv = epi_w8a8_fp64(static_cast<int32_t>(a1), sxi, rc.sw, 0.0f, 0.0f, 0.0f, false, false);
        } else {
          bool rare;
          W8A8Val vv;
          const __half h0 = w8a8_round(static_cast<int32_t>(a1), sxi, rc, vv, rare);
          hv = w8a8_fixup(h0, static_cast<int32_t>(a1), sxi, rc.sw, rc.bias, rc.alpha, rc.v,
                          rc.has_bias, rc.has_steer, vv.yh, vv.yl);
        }
        reinterpret_cast<__half*>(sbuf)[i * 32 + lane] = hv;
      }
    } else if constexpr (KIND == kS32) {
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) reinterpret_cast<uint32_t*>(sbuf)[i * 32 + lane] = r[i];
    } else {
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) h[i] = epi_wo<KIND>(__uint_as_float(r[i]), rc);
#pragma unroll
      for (int i = 0; i < 16; ++i) reinterpret_cast<__half*>(sbuf)[i * 32 + lane] = h[i];
    }
}

// store: the box in `sbuf`, transposed, as coalesced 16-byte stores of
// channels [nb, nb + 32) x tokens [m0 + 16c, m0 + 16c + 16).
template <int KIND>
__device__ __forceinline__ void epilogue_chunk_store(int c, int nb, int m0, int lane, const uint8_t* sbuf,
                                                     const GemmParams& p) {
  using T = KindTraits<KIND>;
    __syncwarp();
    {
      constexpr int kRowChunks = 32 * T::kOutBytes / 16;     // 16-byte chunks per box row
      constexpr int kPerLane = 16 * kRowChunks / 32;
#pragma unroll
      for (int j = 0; j < kPerLane; ++j) {
        const int idx = j * 32 + lane;
        const int row = idx / kRowChunks, ch = idx % kRowChunks;
        const int m = m0 + c * 16 + row;
        const int n = nb + ch * (16 / static_cast<int>(T::kOutBytes));
        const uint4 v = *reinterpret_cast<const uint4*>(sbuf + row * 32 * T::kOutBytes + ch * 16);
        if (m < p.M && n < p.N)  // N % 16 == 0: a 16-byte chunk is wholly in or out
          *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.Y) +
                                    (static_cast<int64_t>(m) * p.N + n) * T::kOutBytes) = v;
      }
    }
}

// The calling warp's chunks c_first, c_first + cs, ... < nchunk of one
// accumulator buffer (`tacc`: its 32 TMEM lanes). After the last TMEM read,
// `release()` runs (warp-uniform; the buffer may then be reused). Store boxes
// alternate between the two halves of `sb0`, `nst` counting the boxes used
// so far. Returns the new count. (Loading the next chunk from TMEM while the
// current one is converted measured slower: 36.6 against 33.8 us at
// M = 4096, N = 4608, K = 1536.)
template <int KIND, class Release>
__device__ __forceinline__ int epilogue_chunks(int c_first, int cs, int nchunk, uint32_t tacc, int lane,
                                               uint8_t* sb0, int nst, const RowConst<KIND>& rc,
                                               const float* sxs, int nb, int m0, const GemmParams& p,
                                               Release release) {
  using T = KindTraits<KIND>;
  if (c_first >= nchunk) {
    release();
    return nst;
  }
  for (int c = c_first; c < nchunk; c += cs) {
    uint8_t* sbuf = sb0 + (nst & 1) * T::kStageBuf;
    epilogue_chunk_compute<KIND>(c, tacc, lane, sbuf, rc, sxs);
    if (c + cs >= nchunk) release();
    epilogue_chunk_store<KIND>(c, nb, m0, lane, sbuf, p);
    ++nst;
  }
  return nst;
}

// ----------------------------------------------- fused activation quant ---
// "Results" (aria project page): W8A8 quantises the activations per token to
// 8 bits. In the fused form every CTA of the GEMM quantises a share of the
// token rows (one warp per row: absmax, s = absmax / 127 as an IEEE fp32
// quotient, codes rounded half-to-even -- the same steps and bits as
// row_quant_i8_kernel) into the workspace, publishes the stores to the
// async proxy, and meets the other CTAs at a grid-wide barrier; the MMA
// pipeline then loads the codes with TMA. The grid never exceeds the SMs
// and each CTA fills one SM, so all CTAs are resident together once the
// preceding kernel has finished. The barrier is a sense-reversal barrier:
// the last CTA to arrive resets the count to zero and advances the
// generation, so the workspace is ready for the next call. Waiting is
// bounded (kWaitLimitNs); on timeout the status word records it.
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __noinline__ bool grid_barrier(unsigned* gbar, unsigned ctas, volatile int* abort) {
  unsigned* count = gbar;
  unsigned* gen = gbar + 1;
  const unsigned g0 = ld_acquire_gpu(gen);
  __threadfence();
  if (atomicAdd(count, 1u) == ctas - 1) {
    atomicExch(count, 0u);
    __threadfence();
    st_release_gpu(gen, g0 + 1);
    return true;
  }
  const uint64_t t0 = globaltimer();
  while (ld_acquire_gpu(gen) == g0) {
    __nanosleep(64);  // fewer polls of the line the arrivals update
    if (globaltimer() - t0 > kWaitLimitNs) {
      atomicOr(&g_status, kStatusTimeout);
      atomicExch(&g_wait_site, 30u);
      *abort = 1;
      return false;
    }
  }
  return true;
}

// `wmax`: kThreads/32 floats of shared memory not in use at this point
template <int KIND>
__device__ __forceinline__ void fused_act_quant(const GemmParams& p, volatile int* abort,
                                                float* wmax) {
  constexpr int kWarps = KindTraits<KIND>::kThreads / 32;
  const unsigned ctas = gridDim.x * gridDim.y;
  const unsigned b = blockIdx.y * gridDim.x + blockIdx.x;
  const int rb0 = static_cast<int>(static_cast<int64_t>(p.M) * b / ctas);
  const int rb1 = static_cast<int>(static_cast<int64_t>(p.M) * (b + 1) / ctas);
  const int rows = rb1 - rb0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = p.K >> 3;  // 16-byte chunks per row
  // a CTA's few rows are spread over all its warps: wpr warps per row
  const int wpr = rows >= 12 ? 1 : rows >= 6 ? 2 : rows >= 3 ? 4 : rows == 2 ? 6 : 12;
  const int slots = kWarps / wpr;                   // rows quantised side by side
  const int slot = warp / wpr;
  const int tr = (warp % wpr) * 32 + lane, tpr = wpr * 32;
  for (int r0 = rb0; r0 < rb1; r0 += slots) {       // the same rounds in every warp
    const int r = r0 + slot;
    const bool live = slot < slots && r < rb1;
    const uint4* xr = reinterpret_cast<const uint4*>(p.xf16 + static_cast<int64_t>(live ? r : rb0) * p.K);
    float a = 0.0f;
    if (live)
      for (int c = tr; c < nch; c += tpr) a = fmaxf(a, absmax8(ld_dep_v4(xr + c)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) wmax[warp] = a;
    __syncthreads();
    if (live) {
      for (int w = slot * wpr; w < slot * wpr + wpr; ++w) a = fmaxf(a, wmax[w]);
      const float s = __fdiv_rn(a, 127.0f);
      uint2* qr = reinterpret_cast<uint2*>(p.xq_ws + static_cast<int64_t>(r) * p.K);
      for (int c = tr; c < nch; c += tpr) qr[c] = quant8_i8(ld_dep_v4(xr + c), s, a == 0.0f);
      if (tr == 0) p.sx_ws[r] = s;
    }
    __syncthreads();                                // wmax is reused by the next round
  }
  if (threadIdx.x == 0) ARIA_STAMP(13);
  // The codes are read by other CTAs' TMA loads (async proxy): each thread
  // orders its stores toward the async proxy, the CTA meets, and one thread
  // makes them visible at GPU scope (the fence is cumulative over the
  // barrier) and arrives at the grid barrier.
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __syncthreads();
  if (threadIdx.x == 0) {
    ARIA_STAMP(14);
    __threadfence();
    grid_barrier(p.gbar, ctas, abort);
    ARIA_STAMP(15);
  }
  __syncthreads();
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ------------------------------------------------------------------ kernel --
template <int KIND>
__global__ void __launch_bounds__(KindTraits<KIND>::kThreads, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmS,
                 const __grid_constant__ CUtensorMap tmX, const GemmParams p) {
  using T = KindTraits<KIND>;
  extern __shared__ uint8_t dyn_smem[];
  // 1024-byte alignment of the shared-window address (128-byte swizzle atoms)
  const uint32_t base_u32 = smem_u32(dyn_smem);
  uint8_t* smem = dyn_smem + (((base_u32 + 1023u) & ~1023u) - base_u32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t wlim = p.wait_ns ? p.wait_ns : kWaitLimitNs;
  const bool drop0 = !T::kDequant && p.drop_first_stage != 0;  // self-test hook
  if (threadIdx.x == 0) ARIA_STAMP(0);
  const bool split = p.splits > 1;
  const int rank = split ? static_cast<int>(cluster_ctarank()) : 0;
  const int tile0 = split ? static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.x);
  const int tstep = split ? static_cast<int>(gridDim.y) : static_cast<int>(gridDim.x);
  // units < 2^26 and rank < 8: the products fit in 32 bits
  const int u_begin = static_cast<int>(static_cast<unsigned>(p.units) * rank / static_cast<unsigned>(p.splits));
  const int u_end = static_cast<int>(static_cast<unsigned>(p.units) * (rank + 1) / static_cast<unsigned>(p.splits));
  const int nu = u_end - u_begin;
  const int nkb = nu * T::kKbPerUnit;

  uint8_t* raw = smem + p.off_raw;
  uint8_t* abuf = smem + p.off_a;
  uint8_t* xbuf = smem + p.off_x;
  uint8_t* stage = smem + p.off_stage;
  float* sxs = reinterpret_cast<float*>(smem + p.off_sxd);   // s_x of two m-tiles [2][kTileBnMax]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bar);
  // one stage = an A tile (weights, 128 rows x 128 B of K) and an X tile
  // (activations, BN rows x 128 B of K); one commit releases both
  uint64_t* raw_full = bars;
  uint64_t* raw_empty = raw_full + p.n_raw;
  uint64_t* st_full = raw_empty + p.n_raw;
  uint64_t* st_empty = st_full + p.n_a;
  uint64_t* acc_full = st_empty + p.n_a;  // [2]
  uint64_t* acc_empty = acc_full + 2;     // [2]
  uint64_t* mma_drain = acc_empty + 2;
  // single use: the CTA's last tile is complete. The dequant warps, which
  // leave their role early to help with that tile, wait on it rather than
  // on acc_full, whose parity could alias when they run several tiles ahead
  // of the MMA (short K, many tiles per CTA)
  uint64_t* acc_last = mma_drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_last + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // ---- prologue. Warp 0 initialises the barriers, one per lane; lane 0
  // takes the "full" barriers of the first weight loads and issues those
  // loads at once (they need nothing else), before the CTA-wide barrier that
  // also waits for the TMEM allocation.
  //
  // Programmatic dependent launch: this CTA may start while the preceding
  // kernel in the stream drains. Packed weights and their scales are inputs
  // that no kernel of this library writes while a following GEMM can already
  // run (the pack kernels do not allow an early start; the header states the
  // rule for callers), so the first ring of weight tiles is loaded before
  // the wait: the raw units of the first tile (q8/q4) or the weight half of
  // its first stages (W8A8, whose activation half follows after the wait on
  // the same barrier). Activations, their scales and the output wait for
  // the preceding kernel to complete.
  int issued_w = 0, issued_x = 0;  // kept for the teardown drain
  int pre = 0;                     // raw units / stages of the first tile issued before the wait
  if (warp == 0) {
    if (tile0 < p.tiles) pre = T::kDequant ? (nu < p.n_raw ? nu : p.n_raw) : (nkb < p.n_a ? nkb : p.n_a);
    uint64_t* pre_full = T::kDequant ? raw_full : st_full;  // arrival count 1 in both rings
    const int nbar = 2 * (p.n_raw + p.n_a) + 6;
    if (lane == 0) {
      for (int i = 0; i < pre; ++i) mbar_init(pre_full + i, 1);
      *abort_flag = 0;
    } else {
      for (int i = lane - 1; i < nbar; i += 31) {
        uint64_t* bar = bars + i;
        if (bar >= pre_full && bar < pre_full + pre) continue;  // lane 0's
        uint32_t cnt = 1;                                         // raw_full, st_empty, acc_full, drain, last
        if (i >= p.n_raw && i < 2 * p.n_raw)
          cnt = (KIND == kQ4 && p.tmem_a) ? 256 : 128;            // raw_empty: the dequant threads
        else if (i >= 2 * p.n_raw && i < 2 * p.n_raw + p.n_a)
          cnt = T::kDequant ? 129 : 1;                            // st_full: dequant threads + X producer
        else if (bar == acc_empty || bar == acc_empty + 1)
          cnt = T::kEpiWarps;
        mbar_init(bar, cnt);
      }
    }
    fence_mbar_init();
    if (lane == 0) {
      ARIA_STAMP(16);
      prefetch_tmap(&tmW);
      prefetch_tmap(&tmX);
      if constexpr (KIND == kQ4) prefetch_tmap(&tmS);
      if (pre > 0) {
        const int n0 = (tile0 % p.tiles_n) * kTileN;
        const uint64_t pol = policy_evict_first();
        for (int i = 0; i < pre; ++i) {
          if constexpr (T::kDequant) {
            const int u = u_begin + i;
            uint8_t* dst = raw + i * p.raw_stage;
            if constexpr (KIND == kQ8) {
              mbar_arrive_expect_tx(raw_full + i, kATile);
              tma_load_2d(&tmW, raw_full + i, dst, u * 128, n0, pol);
            } else {
              mbar_arrive_expect_tx(raw_full + i, kATile + kQ4ScaleTile);
              tma_load_2d(&tmW, raw_full + i, dst, u * 128, n0, pol);
              tma_load_2d(&tmS, raw_full + i, dst + kATile, u * 8, n0, pol);
            }
          } else {
            if (i == 0 && drop0) continue;  // self-test: this stage never fills
            mbar_arrive_expect_tx(st_full + i, kATile + p.x_stage);
            tma_load_2d(&tmW, st_full + i, abuf + i * kATile, (u_begin + i) * T::kWUnitX, n0, pol);
          }
        }
        for (int i = pre; i < nu && i < pre + kL2Ahead; ++i) {  // and the next units into L2
          tma_prefetch_2d(&tmW, (u_begin + i) * T::kWUnitX, n0);
          if constexpr (KIND == kQ4) tma_prefetch_2d(&tmS, (u_begin + i) * 8, n0);
        }
      }
    }
    issued_w = pre;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kAccCols);
    tmem_relinquish();
    if (lane == 0) ARIA_STAMP(18);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) ARIA_STAMP(19);
  const uint32_t tmem_base = *tmem_slot;
  if (threadIdx.x == 0) ARIA_STAMP(1);
  pdl_wait();
  pdl_launch_dependents();
  if constexpr (KIND == kW8A8) {
    if (p.xf16) fused_act_quant<KIND>(p, abort_flag, reinterpret_cast<float*>(smem + p.off_sxd));
  }
  if (threadIdx.x == 0) ARIA_STAMP(2);
  bool epi_ok = true;               // split-K: this CTA's accumulator is complete

  // Dequantisation of the raw weight ring into A stages by 128 threads, one
  // weight row each (t = row within the tile). `ngrp` groups of 128
  // threads share the work: group `grp` takes the K blocks kb with
  // kb % ngrp == grp (every raw stage holds an even number of K blocks).
  auto dequant_rows = [&](const int t, const int grp, const int ngrp) -> bool {
    int s = 0, sa = 0;  // raw ring slot, stage ring slot
    uint32_t rph = 0, aph = 0;
    bool ok = true;
    WaitClock wc_raw, wc_empty;  // trace builds: time waiting for weights / for a free stage
    for (int tile = tile0; tile < p.tiles && ok; tile += tstep) {
      for (int i = 0; i < nu && ok; ++i) {
        wc_raw.start();
        ok = mbar_wait_fast(raw_full + s, rph, abort_flag, 6, wlim);
        wc_raw.stop();
        if (!ok) break;
        if (t == 0 && grp == 0 && tile == tile0 && i == 0) ARIA_STAMP(12);
        const uint8_t* src = raw + s * p.raw_stage;
        uint4 v[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {  // the 16-byte chunks of this group's K blocks
          v[c] = make_uint4(0u, 0u, 0u, 0u);
          if (ngrp == 1 || (c / (8 / T::kKbPerUnit)) % 2 == grp)
            v[c] = *reinterpret_cast<const uint4*>(src + sw128(t, c));
        }
        uint4 sc = make_uint4(0, 0, 0, 0);
        if constexpr (KIND == kQ4) sc = *reinterpret_cast<const uint4*>(src + kATile + t * 16);
        // The slot's next writer is a TMA load (async proxy): order this
        // thread's generic-proxy reads of it before that write. Without
        // the proxy fence the release of the arrive alone let a refill land
        // before the reads of v[4..7] completed (measured: wrong second A
        // tile of a unit in about 1 of 3 launches at M = 4096).
        fence_proxy_async_smem();
        mbar_arrive(raw_empty + s);
        if (++s == p.n_raw) { s = 0; rph ^= 1u; }
#pragma unroll
        for (int h = 0; h < T::kKbPerUnit; ++h) {  // A tiles produced per raw stage
          if (ngrp == 2 && h % 2 != grp) {  // the other group's K block
            if (++sa == p.n_a) { sa = 0; aph ^= 1u; }
            continue;
          }
          wc_empty.start();
          ok = mbar_wait_fast(st_empty + sa, aph ^ 1, abort_flag, 7, wlim);
          wc_empty.stop();
          if (!ok) break;
          if (p.tmem_a) {
            // the MMA that read this slot has completed (its commit arrived)
            tc_fence_after();
            uint32_t o[32];  // TMEM column c = fp16 pair (k = 2c, 2c + 1) of this K block
            if constexpr (KIND == kQ8) {
#pragma unroll
              for (int cc = 0; cc < 4; ++cc) {
                const uint4 w = v[4 * h + cc];
                i8x4_to_h(w.x, o[8 * cc + 0], o[8 * cc + 1]);
                i8x4_to_h(w.y, o[8 * cc + 2], o[8 * cc + 3]);
                i8x4_to_h(w.z, o[8 * cc + 4], o[8 * cc + 5]);
                i8x4_to_h(w.w, o[8 * cc + 6], o[8 * cc + 7]);
              }
            } else {
              const uint32_t* scw = reinterpret_cast<const uint32_t*>(&sc);
#pragma unroll
              for (int g = 0; g < 2; ++g) {
                const int c = 2 * h + g;
                const uint32_t spair = scw[c >> 1];
                const uint32_t s2 = (c & 1) ? __byte_perm(spair, 0, 0x3232) : __byte_perm(spair, 0, 0x1010);
                const uint4 w = v[c];
                const uint4 q0 = nib8_to_h(w.x, s2), q1 = nib8_to_h(w.y, s2);
                const uint4 q2 = nib8_to_h(w.z, s2), q3 = nib8_to_h(w.w, s2);
                o[16 * g + 0] = q0.x; o[16 * g + 1] = q0.y; o[16 * g + 2] = q0.z; o[16 * g + 3] = q0.w;
                o[16 * g + 4] = q1.x; o[16 * g + 5] = q1.y; o[16 * g + 6] = q1.z; o[16 * g + 7] = q1.w;
                o[16 * g + 8] = q2.x; o[16 * g + 9] = q2.y; o[16 * g + 10] = q2.z; o[16 * g + 11] = q2.w;
                o[16 * g + 12] = q3.x; o[16 * g + 13] = q3.y; o[16 * g + 14] = q3.z; o[16 * g + 15] = q3.w;
              }
            }
            __syncwarp();  // tcgen05.st is warp-collective
            tmem_st32(tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) + kAccCols +
                          static_cast<uint32_t>(sa) * 32u,
                      o);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(st_full + sa);
            if (++sa == p.n_a) { sa = 0; aph ^= 1u; }
            continue;
          }
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
          mbar_arrive(st_full + sa);
          if (++sa == p.n_a) { sa = 0; aph ^= 1u; }
        }
      }
    }
    if (t == 0 && grp == 0) {
      ARIA_TRACE_VAL(23, wc_raw.total);
      ARIA_TRACE_VAL(17, wc_empty.total);
    }
    return ok;
  };

  // The producer and MMA roles run as whole converged warps: every lane waits,
  // one lane issues (TMA by lane 0, MMA and commit by elect.sync), so the
  // issue loops stay warp-uniform. Ring slots and phases advance
  // incrementally (no division by the runtime ring depth in the loops).
  if (warp == 0) {
    // ------------------------------------------------ weight tile producer
    const uint64_t pol = policy_evict_first();  // weights are read once per m-tile
    bool ok = true;
    WaitClock wc_pe;  // trace builds (W8A8, fp16): time waiting for free stages
    int s = 0;
    uint32_t ph = 0;
    for (int tile = tile0; tile < p.tiles && ok; tile += tstep) {
      const int n0 = (tile % p.tiles_n) * kTileN;
      if constexpr (T::kDequant) {
        for (int i = 0; i < nu; ++i) {
          if (tile == tile0 && i < pre) {  // issued before the dependency wait
            if (++s == p.n_raw) { s = 0; ph ^= 1u; }
            continue;
          }
          if (!(ok = mbar_wait_warp(raw_empty + s, ph ^ 1, abort_flag, 1, wlim))) break;
          if (lane == 0) {
            uint8_t* dst = raw + s * p.raw_stage;
            const int u = u_begin + i;
            if (i + kL2Ahead < nu) {  // keep the weight stream kL2Ahead units ahead in L2
              tma_prefetch_2d(&tmW, (u + kL2Ahead) * 128, n0);
              if constexpr (KIND == kQ4) tma_prefetch_2d(&tmS, (u + kL2Ahead) * 8, n0);
            }
            if constexpr (KIND == kQ8) {
              mbar_arrive_expect_tx(raw_full + s, kATile);
              tma_load_2d(&tmW, raw_full + s, dst, u * 128, n0, pol);
            } else {
              mbar_arrive_expect_tx(raw_full + s, kATile + kQ4ScaleTile);
              tma_load_2d(&tmW, raw_full + s, dst, u * 128, n0, pol);        // 256 k as bytes
              tma_load_2d(&tmS, raw_full + s, dst + kATile, u * 8, n0, pol);  // 8 group scales
            }
          }
          ++issued_w;
          if (++s == p.n_raw) { s = 0; ph ^= 1u; }
        }
      } else {
        const uint64_t polx = policy_evict_last();
        const int m0 = (tile / p.tiles_n) * p.BN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (tile == tile0 && kb < pre) {
            // the weight half went out before the dependency wait (the barrier
            // already expects both halves): add the activation half
            if (lane == 0 && !(kb == 0 && drop0))
              tma_load_2d(&tmX, st_full + s, xbuf + s * p.x_stage, (u_begin + kb) * T::kXElemsPerKb, m0,
                          polx);
            if (++s == p.n_a) { s = 0; ph ^= 1u; }
            continue;
          }
          wc_pe.start();
          ok = mbar_wait_warp(st_empty + s, ph ^ 1, abort_flag, 2, wlim);
          wc_pe.stop();
          if (!ok) break;
          if (lane == 0) {
            if (kb + kL2Ahead < nkb) tma_prefetch_2d(&tmW, (u_begin + kb + kL2Ahead) * T::kWUnitX, n0);
            mbar_arrive_expect_tx(st_full + s, kATile + p.x_stage);
            tma_load_2d(&tmW, st_full + s, abuf + s * kATile, (u_begin + kb) * T::kWUnitX, n0, pol);
            tma_load_2d(&tmX, st_full + s, xbuf + s * p.x_stage, (u_begin + kb) * T::kXElemsPerKb, m0,
                        polx);
          }
          ++issued_w;
          if (++s == p.n_a) { s = 0; ph ^= 1u; }
        }
      }
    }
    if constexpr (!T::kDequant) {
      if (lane == 0) ARIA_TRACE_VAL(17, wc_pe.total);
    }
  } else if (warp == 2 && T::kDequant) {
    // -------------------------------------------- activation tile producer
    const uint64_t pol = policy_evict_last();   // re-read by every weight tile
    const int kx0 = u_begin * T::kKbPerUnit;
    bool ok = true;
    int s = 0;
    uint32_t ph = 0;
    for (int tile = tile0; tile < p.tiles && ok; tile += tstep) {
      const int m0 = (tile / p.tiles_n) * p.BN;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!(ok = mbar_wait_warp(st_empty + s, ph ^ 1, abort_flag, 3, wlim))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(st_full + s, p.x_stage);
          tma_load_2d(&tmX, st_full + s, xbuf + s * p.x_stage, (kx0 + kb) * T::kXElemsPerKb, m0, pol);
        }
        ++issued_x;
        if (++s == p.n_a) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    const uint32_t idesc = T::kMmaF16 ? idesc_f16_f32(p.BN) : idesc_s8_s32(p.BN);
    int ti = 0, sa = 0;
    uint32_t ph = 0;
    bool ok = true;
    WaitClock wc_full;  // trace builds: time waiting for full stages
    for (int tile = tile0; tile < p.tiles && ok; tile += tstep, ++ti) {
      const int b = ti & 1;
      if (!(ok = mbar_wait_warp(acc_empty + b, ((ti >> 1) & 1) ^ 1, abort_flag, 9, wlim))) break;
      if (ti == 0 && lane == 0) ARIA_STAMP(3);
      tc_fence_after();
      const uint32_t dt = tmem_base + b * kAccCols;
      for (int kb = 0; kb < nkb; ++kb) {
        wc_full.start();
        ok = mbar_wait_warp(st_full + sa, ph, abort_flag, 4, wlim);
        wc_full.stop();
        if (!ok) break;
        if (kb == 0 && ti == 0 && lane == 0) ARIA_STAMP(4);
        tc_fence_after();
        const uint64_t bd = sdesc_sw128(smem_u32(xbuf + sa * p.x_stage));
        if (T::kDequant && p.tmem_a) {
          // A: this stage's 32 TMEM columns (8 per 16-wide K step)
          const uint32_t at = tmem_base + kAccCols + static_cast<uint32_t>(sa) * 32u;
#pragma unroll
          for (int j = 0; j < 4; ++j) umma_f16_ts_elect(dt, at + 8 * j, bd + 2 * j, idesc, (kb | j) != 0);
        } else {
          const uint64_t ad = sdesc_sw128(smem_u32(abuf + sa * kATile));
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // 4 x 32 bytes of K per 128-byte block
            if constexpr (T::kMmaF16)
              umma_f16_elect(dt, ad + 2 * j, bd + 2 * j, idesc, (kb | j) != 0);
            else
              umma_i8_elect(dt, ad + 2 * j, bd + 2 * j, idesc, (kb | j) != 0);
          }
        }
        umma_commit_elect(st_empty + sa);  // releases both tiles of the stage
        if (++sa == p.n_a) { sa = 0; ph ^= 1u; }
      }
      umma_commit_elect(acc_full + b);  // also fires when nothing was issued
      if (tile + tstep >= p.tiles) umma_commit_elect(acc_last);
      if (lane == 0) ARIA_STAMP(5);
    }
    if (lane == 0) ARIA_TRACE_VAL(22, wc_full.total);
  } else if (T::kDequant && warp >= 8) {
    // ------------------------------------------------------ dequantise
    if constexpr (T::kDequant) {
      const int t = threadIdx.x - 256;  // weight row within the tile
      const bool ok = dequant_rows(t, 0, (KIND == kQ4 && p.tmem_a) ? 2 : 1);
      // The CTA's last tile: these warps take its odd epilogue chunks, with
      // store boxes staged in the now idle raw-weight ring.
      if (ok && !split && tile0 < p.tiles) {
        const int ti = (p.tiles - tile0 + tstep - 1) / tstep - 1;
        const int tile = tile0 + ti * tstep;
        const int b = ti & 1;
        const int n0 = (tile % p.tiles_n) * kTileN;
        const int m0 = (tile / p.tiles_n) * p.BN;
        const RowConst<KIND> rc = row_const<KIND>(n0 + t, p);
        bool ok2 = mbar_wait(acc_last, 0, abort_flag, 10, wlim);
        ok2 = __all_sync(0xffffffffu, ok2);
        if (ok2) {
          tc_fence_after();
          const uint32_t tacc = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16) + b * kAccCols;
          uint8_t* sb0 = raw + (warp - 8) * 2 * T::kStageBuf;
          // the last tile's buffer is not reused: nothing to release
          epilogue_chunks<KIND>(1, p.helpers ? 3 : 2, p.BN / 16, tacc, lane, sb0, 0, rc, sxs,
                                n0 + (warp & 3) * 32, m0, p, [] {});
        }
      }
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- epilogue
    // kEpiWarps warps; warp e (0-based) reads TMEM lanes 32*(warp%4).. and
    // takes every (kEpiWarps/4)-th 16-column chunk starting at e/4.
    if constexpr (KIND == kQ4) {
      // one tile per CTA (A in tensor memory): these warps have nothing to
      // do until its accumulator is complete, so they dequantise half of its
      // K blocks beside warps 8..11 (q4 only: the q8 conversion is cheap
      // enough for one group, measured no faster with two)
      if (p.tmem_a) dequant_rows(threadIdx.x - 128, 1, 2);
    }
    const int e = warp - 4;
    const int nep = T::kEpiWarps * 32;
    const int te = threadIdx.x - 128;
    const int t = (warp & 3) * 32 + lane;  // weight row within the tile == TMEM lane
    const int cgrp = e >> 2, cstep = T::kEpiWarps >> 2;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    if (!split) {
      uint8_t* sbuf0 = stage + e * 2 * T::kStageBuf;
      const float alpha = p.steer ? steer_alpha(p) : 0.0f;
      // The channel constants and (W8A8) token scales of a tile are loaded
      // one tile ahead, so their latency hides behind the previous tile's
      // epilogue; the token scales alternate between two shared buffers.
      RowRaw rr;
      if (tile0 < p.tiles) {
        rr = row_raw<KIND>((tile0 % p.tiles_n) * kTileN + t, p);
        if constexpr (KIND == kW8A8) {
          const int m0f = (tile0 / p.tiles_n) * p.BN;
          if (te < p.BN) sxs[te] = (m0f + te < p.M) ? ld_dep_f32(p.sx + m0f + te) : 0.0f;
        }
      }
      int ti = 0, nst = 0;
      for (int tile = tile0; tile < p.tiles; tile += tstep, ++ti) {
        const int b = ti & 1;
        const int n0 = (tile % p.tiles_n) * kTileN;
        const int m0 = (tile / p.tiles_n) * p.BN;
        const RowConst<KIND> rc = row_const_from<KIND>(rr, n0 + t, p, alpha);
        const float* sxc = sxs + (ti & 1) * kTileBnMax;
        const int tnext = tile + tstep;
        float sx_next = 0.0f;
        if (tnext < p.tiles) {
          rr = row_raw<KIND>((tnext % p.tiles_n) * kTileN + t, p);
          if constexpr (KIND == kW8A8) {
            const int m0n = (tnext / p.tiles_n) * p.BN;
            if (te < p.BN && m0n + te < p.M) sx_next = ld_dep_f32(p.sx + m0n + te);
          }
        }
        // W8A8: this tile's token scales are in place, and every reader of
        // the other buffer (the previous tile) is done with it
        if constexpr (KIND == kW8A8) named_bar(1, nep);
        bool ok = mbar_wait(acc_full + b, (ti >> 1) & 1, abort_flag, 8, wlim);
        ok = __all_sync(0xffffffffu, ok);  // warp-uniform before .sync.aligned TMEM loads
        if (ok) {
          if (te == 0 && ti == 0) ARIA_STAMP(6);
          tc_fence_after();
          // the CTA's last tile: q8/q4's dequant warps have no work left and
          // take chunks too (see the end of the dequant role), and so do
          // warps 0..3 (see below)
          const int cs = tnext >= p.tiles ? (p.helpers ? 3 : (T::kDequant ? 2 : cstep)) : cstep;
          nst = epilogue_chunks<KIND>(cgrp, cs, p.BN / 16, tmem_base + lane_off + b * kAccCols, lane, sbuf0,
                                      nst, rc, sxc, n0 + (warp & 3) * 32, m0, p, [&] {
                                        // this warp's last TMEM read of buffer b: the
                                        // tile after next may reuse it
                                        tc_fence_before();
                                        __syncwarp();
                                        if (lane == 0) mbar_arrive(acc_empty + b);
                                      });
          if (te == 0) ARIA_STAMP(7);
        }
        // (on a failed wait, keep taking part in the named barriers of later tiles)
        if constexpr (KIND == kW8A8) {
          if (tnext < p.tiles && te < p.BN) sxs[((ti + 1) & 1) * kTileBnMax + te] = sx_next;
        }
      }
    }
  }

  // ---- the CTA's last tile: warps 0..3 have finished their roles (the
  // producers issued their last loads, the MMA warp its last commit) and take
  // every third epilogue chunk from chunk 2. Their store boxes, and for W8A8
  // their copy of the tile's token scales, sit in the activation ring, idle
  // once the tile's last MMA has completed (acc_last).
  if (warp < 4 && p.helpers && !split && tile0 < p.tiles) {
    const int ti = (p.tiles - tile0 + tstep - 1) / tstep - 1;
    const int tile = tile0 + ti * tstep;
    const int n0 = (tile % p.tiles_n) * kTileN;
    const int m0 = (tile / p.tiles_n) * p.BN;
    const int t = warp * 32 + lane;  // weight row within the tile == TMEM lane
    const RowConst<KIND> rc = row_const<KIND>(n0 + t, p);
    float* hsx = reinterpret_cast<float*>(xbuf + 8 * T::kStageBuf);
    bool ok = mbar_wait(acc_last, 0, abort_flag, 10, wlim);
    ok = __all_sync(0xffffffffu, ok);
    if constexpr (KIND == kW8A8) {
      if (ok)
        for (int j = threadIdx.x; j < p.BN; j += 128) hsx[j] = (m0 + j < p.M) ? ld_dep_f32(p.sx + m0 + j) : 0.0f;
      named_bar(2, 128);
    }
    if (ok) {
      tc_fence_after();
      epilogue_chunks<KIND>(2, 3, p.BN / 16,
                            tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + (ti & 1) * kAccCols, lane,
                            xbuf + warp * 2 * T::kStageBuf, 0, rc, hsx, n0 + warp * 32, m0, p, [] {});
    }
  }

  // ------------------------------------------- split-K: cluster reduction
  // One tile per CTA. Once its partial accumulator is complete every role
  // has finished, so all 12 warps take part: each writes a third of its
  // TMEM lane group's columns to red[m_local][128] (32-bit words, overlaying
  // the idle stage rings). After a cluster barrier, rank r reduces token rows
  // [BN*r/S, BN*(r+1)/S): each thread keeps one group of 4 channels, issues
  // the distributed-shared-memory loads of all S partials for two rows at
  // once, then sums them in rank order (deterministic) and applies the
  // epilogue.
  if (split) {
    epi_ok = mbar_wait_warp(acc_full, 0, abort_flag, 8, wlim);
    const int lg = warp & 3, wg = warp >> 2;  // TMEM lane group; third of the columns
    uint32_t* red = reinterpret_cast<uint32_t*>(smem);
    {
      const int t = lg * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(lg * 32) << 16;
      tc_fence_after();
      for (int c = wg; c < p.BN / 16; c += 3) {
        uint32_t r[16];
        tmem_ld16(tmem_base + lane_off + c * 16, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) red[(c * 16 + i) * 128 + t] = epi_ok ? r[i] : 0u;
      }
    }
    __syncwarp();
    cluster_sync();
    ARIA_STAMP(8);
    {
      constexpr int kWarps = KindTraits<KIND>::kThreads / 32;
      constexpr int kRows = 2;       // rows in flight per thread
      constexpr int kMaxSplits = 8;
      const int n0 = (tile0 % p.tiles_n) * kTileN;
      const int m0 = (tile0 / p.tiles_n) * p.BN;
      const int mb = p.BN * rank / p.splits, me = p.BN * (rank + 1) / p.splits;
      const int nl = lane * 4;
      const int n = n0 + nl;
      RowConst<KIND> rc[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) rc[j] = row_const<KIND>(n + j, p);
      const uint32_t red_u32 = smem_u32(smem);
      for (int ml0 = mb + warp; ml0 < me; ml0 += kRows * kWarps) {
        uint4 v[kMaxSplits][kRows];
#pragma unroll
        for (int q = 0; q < kMaxSplits; ++q) {
#pragma unroll
          for (int u = 0; u < kRows; ++u) {
            const int ml = ml0 + u * kWarps;
            v[q][u] = make_uint4(0u, 0u, 0u, 0u);
            if (q < p.splits && ml < me)
              v[q][u] = ld_dsmem_v4(mapa_shared(red_u32 + static_cast<uint32_t>((ml * 128 + nl) * 4), q));
          }
        }
        uint4 acc[kRows];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
          acc[u] = v[0][u];
#pragma unroll
          for (int q = 1; q < kMaxSplits; ++q) {
            if (q < p.splits) {
              acc[u].x = reduce_add<KIND>(acc[u].x, v[q][u].x);
              acc[u].y = reduce_add<KIND>(acc[u].y, v[q][u].y);
              acc[u].z = reduce_add<KIND>(acc[u].z, v[q][u].z);
              acc[u].w = reduce_add<KIND>(acc[u].w, v[q][u].w);
            }
          }
        }
        if (threadIdx.x == 0 && ml0 == mb) ARIA_STAMP(20);  // the first partials summed
        uint32_t rare_mask = 0;  // W8A8: elements to redo exactly (bit 4u+k)
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
          const int ml = ml0 + u * kWarps;
          const int m = m0 + ml;
          if (ml >= me || m >= p.M || n >= p.N) continue;  // N % 16 == 0: 4 columns in range
          const int64_t o = static_cast<int64_t>(m) * p.N + n;
          if constexpr (KIND == kS32) {
            *reinterpret_cast<uint4*>(reinterpret_cast<int32_t*>(p.Y) + o) = acc[u];
          } else {
            const uint32_t a4[4] = {acc[u].x, acc[u].y, acc[u].z, acc[u].w};
            __half h[4];
            if constexpr (KIND == kW8A8) {
              const float sxm = ld_dep_f32(p.sx + m);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                bool rare;
                if (!rc[k].has_bias && !rc[k].has_steer) {
                  const uint32_t pk = w8a8_plain_pair(static_cast<int32_t>(a4[k]), sxm, rc[k].sw_up, rc[k].sw_dn);
                  h[k] = __ushort_as_half(static_cast<unsigned short>(pk & 0xFFFFu));
                  rare = pair_split(pk) | w8a8_acc_big(static_cast<int32_t>(a4[k]));
                } else {
                  W8A8Val vv;
                  h[k] = w8a8_round(static_cast<int32_t>(a4[k]), sxm, rc[k], vv, rare);
                }
                rare_mask |= static_cast<uint32_t>(rare) << (4 * u + k);
              }
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k) h[k] = epi_wo<KIND>(__uint_as_float(a4[k]), rc[k]);
            }
            *reinterpret_cast<uint2*>(reinterpret_cast<__half*>(p.Y) + o) = *reinterpret_cast<uint2*>(h);
          }
        }
        if (threadIdx.x == 0 && ml0 == mb) ARIA_STAMP(21);  // their outputs stored
        if constexpr (KIND == kW8A8) {
          // rare elements: round exactly from the summed accumulator (picked
          // from registers by index: no second trip to the peers' shared
          // memory); these later stores of the same thread replace the
          // values written above
          while (rare_mask) {
            const int idx = __ffs(rare_mask) - 1;
            rare_mask &= rare_mask - 1;
            const int u = idx >> 2, k = idx & 3;
            const int ml = ml0 + u * kWarps;
            const int m = m0 + ml;
            uint32_t asel = 0u;
#pragma unroll
            for (int uu = 0; uu < kRows; ++uu) {
              if (uu == u) {
                const uint32_t c4[4] = {acc[uu].x, acc[uu].y, acc[uu].z, acc[uu].w};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  if (kk == k) asel = c4[kk];
              }
            }
            const int32_t a = static_cast<int32_t>(asel);
            const RowConst<kW8A8> rk = row_const<kW8A8>(n + k, p);
            reinterpret_cast<__half*>(p.Y)[static_cast<int64_t>(m) * p.N + n + k] =
                epi_w8a8(a, ld_dep_f32(p.sx + m), rk);
          }
        }
      }
    }
    ARIA_STAMP(9);
    __syncwarp();
    cluster_sync();
    ARIA_STAMP(10);
  }

  // ---------------------------------------------------------------- teardown
  const bool aborted = *abort_flag != 0;
  if (aborted && lane == 0) {
    // drain copies still in flight into this CTA's shared memory
    // (q8/q4 stage barriers also wait for dequant arrivals, so only the raw
    // ring and W8A8 stages are drained here; X loads of q8/q4 stages were
    // issued only after their stage was empty and complete on their own)
    if (warp == 0) {
      const int nring = T::kDequant ? p.n_raw : p.n_a;
      uint64_t* full = T::kDequant ? raw_full : st_full;
      for (int i = (issued_w > nring ? issued_w - nring : 0); i < issued_w; ++i)
        if (!(i == 0 && drop0))  // a withheld stage has nothing in flight
          mbar_wait_drain(full + (i % nring), (i / nring) & 1, wlim);
    } else if (warp == 2 && issued_x > 0) {
      const uint64_t t0 = globaltimer();  // X loads of q8/q4: allow 100 us to land
      while (globaltimer() - t0 < 100000ull) __nanosleep(1000);
    }
  }
  if (warp == 1 && __any_sync(0xffffffffu, aborted)) {
    // MMAs issued before the abort finish before TMEM is freed; the commit
    // comes from the lane that issued them (elect.sync, as in the issue loop)
    umma_commit_elect(mma_drain);
    mbar_wait_drain(mma_drain, 0, wlim);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kAccCols);
  }
  if (threadIdx.x == 0) ARIA_STAMP(11);
}

}  // namespace aria
