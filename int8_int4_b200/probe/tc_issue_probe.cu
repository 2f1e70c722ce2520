// tc_issue_probe.cu -- a standalone measurement, not part of libaria_q.so.
// Two rates the GEMM kernels' pipeline is built on, each from one CTA per SM:
//
//  mma   one converged warp issues 4 x `iters` tcgen05.mma (M = 128,
//        cta_group::1) back to back on operands already in shared / tensor
//        memory, for kind::f16 with A and B in shared memory (f16_ss),
//        kind::i8 likewise (i8_ss) and kind::f16 with A in tensor memory
//        (f16_ts), N swept; each form is its own template instance, so the
//        issue loop has no run-time dispatch; optionally a tcgen05.commit
//        after every 4 MMAs (one 128-byte K block, as in the kernels).
//        Prints SM cycles per MMA.
//  ring  one thread fills a ring of S stages with B TMA boxes of R rows x
//        128 bytes each (128-byte swizzle) from an L2-resident 32 MB tensor,
//        one thread waits for each stage and releases it (no other work).
//        Prints nanoseconds per stage on 148 SMs.
//
//   python -m int8_int4_b200.build --probe && ./int8_int4_b200/tc_issue_probe
#include <cstdio>
#include <vector>

#include "../csrc/ptx.cuh"

using namespace aria;

namespace {

enum Form { kF16SS = 0, kI8SS = 1, kF16TS = 2 };

template <int FORM>
__global__ void __launch_bounds__(128, 1) mma_rate(int n, int iters, int commit_per_kb, long long* out) {
  extern __shared__ uint8_t dyn[];
  const uint32_t base = smem_u32(dyn);
  uint8_t* sm = dyn + (((base + 1023u) & ~1023u) - base);  // 128-byte swizzle atoms: 1024-aligned
  uint8_t* a = sm;                                          // 128 rows x 128 B
  uint8_t* b = sm + 16384;                                  // up to 256 rows x 128 B
  __shared__ uint64_t done_bar, kb_bar;
  __shared__ uint32_t tslot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // operands: fp16 values in [0.5, 1) with random signs, or small int8 codes
  uint32_t* w = reinterpret_cast<uint32_t*>(sm);
  for (int i = threadIdx.x; i < (16384 + 32768) / 4; i += blockDim.x) {
    const uint32_t h = static_cast<uint32_t>(i + 1) * 2654435761u;
    const uint32_t lo = 0x3800u | (h & 0x3FFu) | (((h >> 10) & 1u) << 15);
    const uint32_t hi = 0x3800u | ((h >> 11) & 0x3FFu) | (((h >> 21) & 1u) << 15);
    w[i] = FORM == kI8SS ? (h & 0x0F0F0F0Fu) : (lo | (hi << 16));
  }
  if (threadIdx.x == 0) {
    mbar_init(&done_bar, 1);
    mbar_init(&kb_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tslot, 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();  // generic-proxy operand writes before the MMAs read them
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = tslot;
  if (FORM == kF16TS) {  // A in TMEM columns [256, 288): each warp its 32 lanes
    uint32_t r[32];
    for (int j = 0; j < 32; ++j) r[j] = 0x3C003C00u ^ static_cast<uint32_t>((lane * 7 + j) & 0x3FF);
    tmem_st32(tb + (static_cast<uint32_t>(warp * 32) << 16) + 256u, r);
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    const uint64_t ad = sdesc_sw128(smem_u32(a)), bd = sdesc_sw128(smem_u32(b));
    const uint32_t idesc =
        FORM == kI8SS ? idesc_s8_s32(static_cast<uint32_t>(n)) : idesc_f16_f32(static_cast<uint32_t>(n));
    const long long c0 = clock64();
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // 4 x 32 bytes of K: one 128-byte K block
        const uint32_t acc = (it | j) != 0;
        if constexpr (FORM == kF16SS)
          umma_f16_elect(tb, ad + 2 * j, bd + 2 * j, idesc, acc);
        else if constexpr (FORM == kI8SS)
          umma_i8_elect(tb, ad + 2 * j, bd + 2 * j, idesc, acc);
        else
          umma_f16_ts_elect(tb, tb + 256u + 8u * j, bd + 2 * j, idesc, acc);
      }
      if (commit_per_kb) umma_commit_elect(&kb_bar);
    }
    umma_commit_elect(&done_bar);
    const bool ok = mbar_wait_drain(&done_bar, 0, 2000000000ull);
    const long long c1 = clock64();
    if (lane == 0) {
      out[blockIdx.x * 2 + 0] = c1 - c0;
      out[blockIdx.x * 2 + 1] = ok ? 1 : 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tb, 512);
}

// Thread 0 fills, thread 32 drains; stage slots and phases advance by
// counters (no division in the loops).
__global__ void __launch_bounds__(64, 1) ring_rate(const __grid_constant__ CUtensorMap tm, uint32_t row_mask,
                                                   int R, int B, int S, int iters, long long* out) {
  extern __shared__ uint8_t dyn[];
  const uint32_t base = smem_u32(dyn);
  uint8_t* ring = dyn + (((base + 1023u) & ~1023u) - base);
  __shared__ uint64_t full[8], empty[8];
  __shared__ int abort_flag, issued, drained;
  const int box = R * 128, stage = box * B;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    abort_flag = 0;
    issued = 0;
    drained = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* ab = &abort_flag;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm);
    const uint64_t pol = policy_evict_last();
    uint32_t row = blockIdx.x * 7919u * 256u;
    int s = 0, i = 0;
    uint32_t ph = 0;
    for (; i < iters; ++i) {
      if (i >= S && !mbar_wait_fast(empty + s, ph ^ 1u, ab, 1, 1000000000ull)) break;
      mbar_arrive_expect_tx(full + s, static_cast<uint32_t>(stage));
      for (int j = 0; j < B; ++j) {
        tma_load_2d(&tm, full + s, ring + s * stage + j * box, 0, static_cast<int>(row & row_mask), pol);
        row += static_cast<uint32_t>(R);
      }
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    issued = i;
  } else if (threadIdx.x == 32) {
    const uint64_t g0 = globaltimer();
    int s = 0, i = 0;
    uint32_t ph = 0;
    for (; i < iters; ++i) {
      if (!mbar_wait_fast(full + s, ph, ab, 2, 1000000000ull)) break;
      mbar_arrive(empty + s);
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    out[blockIdx.x * 2 + 0] = static_cast<long long>(globaltimer() - g0);
    out[blockIdx.x * 2 + 1] = i;
    drained = i;
  }
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag)  // loads still in flight land before the CTA exits
    for (int i = drained; i < issued; ++i) mbar_wait_drain(full + (i % S), (i / S) & 1, 1000000000ull);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

template <int FORM>
bool run_mma(const char* name, long long* d_out, std::vector<long long>& h) {
  const int smem = 120 * 1024;  // one CTA per SM
  cudaFuncSetAttribute(mma_rate<FORM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const int iters = 2000;
  for (int commit : {0, 1})
    for (int n : {32, 64, 96, 128, 144, 160, 192, 224, 256}) {
      for (int rep = 0; rep < 2; ++rep) {  // the first launch warms up
        mma_rate<FORM><<<1, 128, smem>>>(n, iters, commit, d_out);
        const cudaError_t e = cudaDeviceSynchronize();
        if (e != cudaSuccess) {
          printf("CUDA error: %s\n", cudaGetErrorString(e));
          return false;
        }
      }
      cudaMemcpy(h.data(), d_out, 2 * sizeof(long long), cudaMemcpyDeviceToHost);
      printf("mma %s commit_per_kb=%d N=%d cycles_per_mma=%.1f nominal_N/2=%d%s\n", name, commit, n,
             static_cast<double>(h[0]) / (4.0 * iters), n / 2, h[1] == 1 ? "" : " TIMEOUT");
    }
  return true;
}

}  // namespace

int main() {
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
  long long* d_out = nullptr;
  if (cudaMalloc(&d_out, static_cast<size_t>(sms) * 2 * sizeof(long long)) != cudaSuccess) return 1;
  std::vector<long long> h(static_cast<size_t>(sms) * 2);
  if (!run_mma<kF16SS>("f16_ss", d_out, h) || !run_mma<kI8SS>("i8_ss", d_out, h) ||
      !run_mma<kF16TS>("f16_ts", d_out, h))
    return 1;

  void* fp = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return 1;
  const auto encode = reinterpret_cast<EncodeTiledFn>(fp);
  const int log_rows = 18;  // 32 MB of 128-byte rows, plus one box of slack
  const size_t rows = (size_t{1} << log_rows) + 256;
  uint8_t* src = nullptr;
  if (cudaMalloc(&src, rows * 128) != cudaSuccess) return 1;
  cudaMemset(src, 1, rows * 128);
  const int smem = 220 * 1024;
  cudaFuncSetAttribute(ring_rate, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  for (int R : {64, 128, 256}) {
    CUtensorMap tm;
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {128};
    cuuint32_t boxd[2] = {128, static_cast<cuuint32_t>(R)};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, src, dims, strides, boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return 1;
    for (int B : {1, 2})
      for (int S : {4, 8}) {
        const int stage = R * 128 * B;
        if (stage * S + 1024 > smem) continue;
        const int iters = 4000;
        for (int rep = 0; rep < 2; ++rep) {
          ring_rate<<<sms, 64, smem>>>(tm, (1u << log_rows) - 1u, R, B, S, iters, d_out);
          const cudaError_t e = cudaDeviceSynchronize();
          if (e != cudaSuccess) {
            printf("CUDA error: %s\n", cudaGetErrorString(e));
            return 1;
          }
        }
        cudaMemcpy(h.data(), d_out, h.size() * sizeof(long long), cudaMemcpyDeviceToHost);
        double tmax = 0;
        bool ok = true;
        for (int i = 0; i < sms; ++i) {
          tmax = static_cast<double>(h[i * 2]) > tmax ? static_cast<double>(h[i * 2]) : tmax;
          ok = ok && h[i * 2 + 1] == iters;
        }
        const double ns = tmax / iters;
        printf("ring box_rows=%d boxes_per_stage=%d stages=%d ns_per_stage=%.1f GBps_per_SM=%.1f%s\n", R, B, S, ns,
               stage / ns, ok ? "" : " INCOMPLETE");
      }
  }
  unsigned st = 0;
  cudaMemcpyFromSymbol(&st, g_status, sizeof(st));
  cudaFree(src);
  cudaFree(d_out);
  return st == 0 ? 0 : 2;
}
