/*
 * aria_q.h -- C ABI of libaria_q.so: quantized linear layers (q8 / q4
 * weight-only, W8A8) for NVIDIA B200 (sm_100a).
 *
 * Source of the method: "A Quantized Native Runtime for On-Device Semantic
 * Audio Generation" (aria project page). "What aria is": the diffusion
 * transformer's weights are packed from fp16 to 8 or 4 bits and the fp16
 * copy is released, so the packed form replaces the footprint. "Results":
 * four precisions -- fp16, q8, W8A8 (8-bit arithmetic on integer tensor
 * cores, the fastest GPU mode) and q4; q8 and W8A8 share one footprint.
 * "Steering is real": a direction vector is added at one transformer block,
 * and alpha = 0 removes it with bit-identical output. "Live steering while
 * streaming": the steering lives inside the captured CUDA graph, so its
 * strength can change from one step or chunk to the next.
 *
 * Formats (the pages give none; these are the library's fixed readings):
 *   Q8 / W8A8 weights: Wq int8 [N,K] row-major (K contiguous),
 *       scales fp32 [N]; s[n] = absmax_k|W[n,k]| / 127 (fp32 division),
 *       Wq = clamp(round_half_even(W / s), -127, 127); all-zero row -> s = 0.
 *   Q4 weights (group 32 along K): Wq uint8 [N,K/2]; byte k/2 holds k even in
 *       its low nibble and k odd in its high nibble, each as code+8 (offset
 *       binary); scales fp16 [N,K/32]; s16 = fp16_rn(absmax/7),
 *       code = clamp(round_half_even(W / float(s16)), -7, 7).
 *   Activations for W8A8: Xq int8 [M,K], s_x fp32 [M], the Q8 rule per token row.
 *   X, W, bias, Y: fp16 (IEEE binary16), row-major; Y is [M,N].
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are caller-owned device memory on the current
 *     CUDA device; the library keeps no pointer after the call returns.
 *   - Every device pointer must be 16-byte aligned (ARIA_ERR_MISALIGNED).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). All work is
 *     enqueued on it; calls return after launch, without synchronising.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns an error and launches nothing.
 *   - Kernels bound every wait. A wait that runs out (about 4 s) records
 *     ARIA_ERR_TIMEOUT in a device status word, and the kernel returns;
 *     aria_device_status() reports and clears it.
 *   - Non-finite inputs are outside the contract (not checked).
 *   - The library allocates no device memory, makes no host-device copies
 *     inside the entry points below, and is safe to call while a stream is
 *     being captured into a CUDA graph (aria_device_status excepted). The
 *     one entry point that needs scratch memory (aria_qgemm_w8a8_fused)
 *     takes it from the caller.
 */
#ifndef ARIA_Q_H
#define ARIA_Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ARIA_OK = 0,
    ARIA_ERR_INVALID_ARG = 1,  /* NULL pointer, non-positive or too-large size */
    ARIA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (group != 32, shape rule) */
    ARIA_ERR_MISALIGNED = 3,   /* a device pointer is not 16-byte aligned */
    ARIA_ERR_CUDA = 4,         /* a CUDA runtime call failed (see aria_last_error_message) */
    ARIA_ERR_TIMEOUT = 5       /* a kernel's bounded wait ran out (device status word) */
} aria_status;

typedef enum {
    ARIA_FMT_Q8 = 1,    /* 8-bit weights, fp16 activations (weight-only) */
    ARIA_FMT_Q4 = 2,    /* 4-bit group-32 weights, fp16 activations (weight-only) */
    ARIA_FMT_W8A8 = 3,  /* 8-bit weights (the Q8 pack) x per-token int8 activations */
    ARIA_FMT_F16 = 4    /* unquantised fp16 weights (the fp16 rung of the precision table) */
} aria_format;

/* Human-readable name of a status code (static string). */
const char *aria_status_string(aria_status s);

/* Text of the last error returned on the calling host thread ("" if none). */
const char *aria_last_error_message(void);

/*
 * aria_qpack_size -- bytes of the packed weights and of their scales.
 * ("What aria is": weights packed from fp16 to 8 or 4 bits.)
 *   fmt    ARIA_FMT_Q8 or ARIA_FMT_W8A8 (same pack), or ARIA_FMT_Q4. ARIA_FMT_F16
 *          weights are used unpacked: ARIA_ERR_UNSUPPORTED.
 *   group  0 for Q8 / W8A8 (per output channel); 32 for Q4.
 *   N, K   output and input features of the linear layer (W is [N,K]).
 *   wq_bytes, scale_bytes  host outputs: N*K and 4*N (Q8), N*K/2 and 2*N*K/32 (Q4).
 * Errors: INVALID_ARG (NULL outputs, N or K <= 0), UNSUPPORTED (group, K % 32 for Q4).
 */
aria_status aria_qpack_size(aria_format fmt, int group, int64_t N, int64_t K,
                            size_t *wq_bytes, size_t *scale_bytes);

/*
 * aria_qpack -- pack fp16 weights W [N,K] into the Q8 or Q4 format above.
 * ("What aria is": the fp16 copy is released once packed -- the caller may
 * free W after the stream reaches this call; the library never holds it.)
 *   W       device, fp16 [N,K] row-major.
 *   Wq      device output, int8 [N,K] (Q8, W8A8) or uint8 [N,K/2] (Q4).
 *   scales  device output, fp32 [N] (Q8, W8A8) or fp16 [N,K/32] (Q4).
 * Shape rules: N >= 1; K >= 16 and K % 16 == 0 (Q8); K % 32 == 0 (Q4).
 * Packed bytes are a pure function of W (bit-exact, deterministic).
 */
aria_status aria_qpack(aria_format fmt, int group, const void *W, int64_t N, int64_t K,
                       void *Wq, void *scales, void *stream);

/*
 * aria_act_quant -- per-token dynamic int8 quantisation of activations (the
 * "A8" of W8A8, "Results": 8-bit arithmetic on integer tensor cores).
 *   X   device, fp16 [M,K] row-major.
 *   Xq  device output, int8 [M,K]; sx device output, fp32 [M].
 *   s_x[m] = absmax_k |X[m,k]| / 127; Xq = clamp(rhe(X / s_x[m]), -127, 127).
 * Shape rules: M >= 1, K >= 16, K % 16 == 0. Bit-exact and deterministic.
 */
aria_status aria_act_quant(const void *X, int64_t M, int64_t K, int8_t *Xq, float *sx,
                           void *stream);

/*
 * aria_qgemm -- Y = X . dequant(W)^T with the fused epilogue
 *   Y[m,n] = fp16( main[m,n] + bias[n] + alpha * v[n] ).
 *   Q8:   main = s_w[n] * sum_k X[m,k] * Wq[n,k]            (fp16 tensor cores)
 *   Q4:   main = sum_k X[m,k] * fp16((code-8) * s16[n,k/32]) (fp16 tensor cores)
 *   W8A8: main = acc[m,n] * s_x[m] * s_w[n], acc = sum_k Xq*Wq exact int32
 *         (int8 tensor cores); the epilogue is evaluated in fp64 and rounded
 *         once to fp16.
 *   F16:  main = sum_k X[m,k] * W[n,k] on the unquantised fp16 weights
 *         (fp16 tensor cores; "Results": the fp16 column of the table).
 *   Weight-only and F16 results accumulate in fp32 and are rounded once to fp16.
 *   X       device: fp16 [M,K] (Q8, Q4, F16) or int8 [M,K] from aria_act_quant (W8A8).
 *   sx      device fp32 [M] (W8A8 only; must be NULL otherwise).
 *   Wq, scales  device, as produced by aria_qpack (W8A8 takes the Q8 pack);
 *           F16: Wq is the fp16 weight [N,K] itself and scales must be NULL.
 *   bias    device fp16 [N], or NULL for none.
 *   steer_vec device fp32 [N], or NULL. The steering add ("Steering is real")
 *           is skipped entirely when steer_vec == NULL or alpha == 0, so the
 *           output is then bit-identical to an unsteered call.
 *   Y       device output, fp16 [M,N] row-major. Must not alias any input.
 * Shape rules: M >= 1; N >= 16, N % 16 == 0; K >= 16, K % 16 == 0;
 *   Q4 additionally K % 256 == 0; group as in aria_qpack_size (0 for F16);
 *   W8A8 additionally K * 127^2 < 2^31 (K <= 133144), so that the exact
 *   int32 accumulators cannot wrap (ARIA_ERR_UNSUPPORTED otherwise).
 * Deterministic: the same inputs give the same bytes on every call.
 * Stream order: the kernel is launched with programmatic dependent launch,
 *   so it may start while the preceding kernel in `stream` finishes. X, sx,
 *   bias, steer_vec, a device alpha and Y are touched only after that kernel
 *   has completed; the first weight tiles (Wq, and the Q4 scales) are loaded
 *   before. Wq and scales must therefore be complete before the preceding
 *   kernel in the stream starts, or be written by a kernel that does not
 *   allow an early start of its successor (no griddepcontrol.launch_dependents
 *   / cudaTriggerProgrammaticLaunchCompletion before its last write) and
 *   whose threads make their stores visible at GPU scope and to the async
 *   proxy before they exit (__threadfence(); fence.proxy.async.global).
 *   aria_qpack's kernels do both, so pack-then-GEMM on one stream is safe.
 */
aria_status aria_qgemm(aria_format fmt, int group, int64_t M, int64_t N, int64_t K,
                       const void *X, const float *sx, const void *Wq, const void *scales,
                       const void *bias, const float *steer_vec, float alpha, void *Y,
                       void *stream);

/*
 * aria_qgemm_steer_dev -- aria_qgemm with the steering strength read from
 * device memory when the kernel runs ("Live steering while streaming": the
 * steering lives inside the captured graph, so control can change
 * mid-stream; "Run it": the steer spec names a step window, e.g. 0-7).
 * A CUDA graph captured once can then follow an alpha schedule: capture
 * step s's steered call with alpha_dev = &schedule[s], and rewrite the
 * schedule (e.g. with cudaMemcpyAsync) between replays; steps outside the
 * window hold 0.
 *   alpha_dev  device fp32 scalar, 4-byte aligned; read after the preceding
 *              kernel in `stream` has completed. Required when steer_vec is
 *              not NULL (ARIA_ERR_INVALID_ARG), ignored when it is NULL.
 *   Every other argument and rule as for aria_qgemm (alpha is *alpha_dev).
 *   A value of 0 at run time skips the add entirely, so that step's output
 *   is bit-identical to an unsteered call; a non-zero value gives the same
 *   bytes as aria_qgemm with that alpha.
 */
aria_status aria_qgemm_steer_dev(aria_format fmt, int group, int64_t M, int64_t N, int64_t K,
                                 const void *X, const float *sx, const void *Wq,
                                 const void *scales, const void *bias, const float *steer_vec,
                                 const float *alpha_dev, void *Y, void *stream);

/*
 * aria_w8a8_workspace_size -- bytes of the workspace aria_qgemm_w8a8_fused
 * needs for M tokens of K features: 256 + 4*M rounded up to 256 + M*K.
 * Errors: INVALID_ARG (NULL output, M or K outside [1, 2^31)).
 */
aria_status aria_w8a8_workspace_size(int64_t M, int64_t K, size_t *bytes);

/*
 * aria_qgemm_w8a8_fused -- the W8A8 linear from fp16 activations in one
 * launch: the per-token int8 quantisation of X (exactly aria_act_quant's
 * rule and bits) runs inside the GEMM kernel, then the integer-tensor-core
 * GEMM and the epilogue of aria_qgemm(ARIA_FMT_W8A8) ("Results": W8A8 is
 * 8-bit arithmetic on integer tensor cores; the activations are quantised
 * per token).
 *   X          device fp16 [M,K] row-major (not quantised).
 *   Wq, sw     device, the Q8 pack (int8 [N,K], fp32 [N]).
 *   bias, steer_vec, alpha  as for aria_qgemm; alpha_dev, if not NULL, a
 *              device fp32 scalar (4-byte aligned) used instead of alpha, as
 *              in aria_qgemm_steer_dev.
 *   Y          device output fp16 [M,N]: the same bytes as aria_act_quant
 *              followed by aria_qgemm(ARIA_FMT_W8A8).
 *   workspace  caller-owned device memory, 256-byte aligned, at least
 *              aria_w8a8_workspace_size(M, K) bytes (INVALID_ARG otherwise).
 *              Its first 256 bytes hold a grid barrier: bytes 0..3 (the
 *              arrival count) must be zero before the first call, and every
 *              successful call leaves them zero; bytes 4..7 count the calls
 *              (any starting value). After the call the workspace holds the
 *              token scales
 *              (fp32 [M] at byte 256) and the codes (int8 [M,K] at byte
 *              256 + 4*M rounded up to 256), as aria_act_quant would write
 *              them. Calls that share a workspace must not overlap on the
 *              GPU (one stream, or ordered by events).
 *   The kernel's CTAs meet at a grid-wide barrier after quantising their
 *   share of the rows; its wait is bounded: if it runs out, the device
 *   status word reports ARIA_ERR_TIMEOUT and the workspace's arrival count
 *   must be zeroed again before the next call.
 * Shape rules and stream order as for aria_qgemm(ARIA_FMT_W8A8).
 */
aria_status aria_qgemm_w8a8_fused(int64_t M, int64_t N, int64_t K, const void *X, const void *Wq,
                                  const float *sw, const void *bias, const float *steer_vec,
                                  float alpha, const float *alpha_dev, void *Y, void *workspace,
                                  size_t workspace_bytes, void *stream);

/*
 * aria_qgemm_w8a8_fused_noalloc -- aria_qgemm_w8a8_fused without a caller
 * workspace and without allocating anything. The paper has no counterpart:
 * this entry point exists for callers that must not allocate device memory
 * while they run -- a real-time audio render callback, where cudaMalloc can
 * block or synchronise the device and miss the deadline, or a host that
 * fixes the device memory budget at load time and forbids allocation
 * afterwards. Its scratch (the codes, the token scales and the grid barrier)
 * is a static device array of ARIA_NOALLOC_SCRATCH_BYTES (32 MiB) inside
 * the library, which every GPU that loads the library holds until the
 * process exits.
 *   Arguments and result as for aria_qgemm_w8a8_fused (no workspace).
 *   Size limit: 256 + 4*M rounded up to 256 + M*K must not exceed
 *   ARIA_NOALLOC_SCRATCH_BYTES; larger calls return ARIA_ERR_UNSUPPORTED and
 *   launch nothing (e.g. M = 4096 allows K up to 8176).
 *   The first call on a device looks up the scratch's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.
 *   Each call clears the scratch's barrier words on `stream` before its
 *   kernel (no allocation: a memset). All calls share the one scratch array,
 *   which keeps the last call's contents: calls that overlap on the GPU
 *   (different streams without ordering) race and give wrong results.
 *   Calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define ARIA_NOALLOC_SCRATCH_BYTES (32u << 20)
aria_status aria_qgemm_w8a8_fused_noalloc(int64_t M, int64_t N, int64_t K, const void *X,
                                          const void *Wq, const float *sw, const void *bias,
                                          const float *steer_vec, float alpha, const float *alpha_dev,
                                          void *Y, void *stream);

/*
 * aria_qgemm_s32 -- the W8A8 integer GEMM alone: C[m,n] = sum_k Xq[m,k]*Wq[n,k]
 * as exact int32 ("Results": 8-bit arithmetic on integer tensor cores). Runs
 * the same tensor-core mainloop as aria_qgemm(ARIA_FMT_W8A8) and stores the
 * raw accumulators, for bit-exact checks.
 *   Xq device int8 [M,K]; Wq device int8 [N,K]; C device output int32 [M,N].
 * Shape rules as for aria_qgemm, including K * 127^2 < 2^31 (ARIA_ERR_UNSUPPORTED).
 */
aria_status aria_qgemm_s32(int64_t M, int64_t N, int64_t K, const int8_t *Xq, const int8_t *Wq,
                           int32_t *C, void *stream);

/*
 * aria_selftest_bounded_wait -- failure-detection self-test (no counterpart
 * on the pages; the library's own fault path). Launches the W8A8 GEMM of
 * aria_qgemm(ARIA_FMT_W8A8) with every bounded wait limited to
 * wait_limit_us microseconds and with the first pipeline stage of each
 * CTA's first tile withheld, so that the waits on that stage run out. The
 * kernel then unwinds without hanging or faulting: the waiting roles give
 * up, the copies already in flight are drained, tensor memory is freed, and
 * the device status word records the timeout. aria_device_status() on the
 * same stream then returns ARIA_ERR_TIMEOUT (and clears it); Y is left
 * unspecified; the context stays usable for the next call.
 *   Xq, sx, Wq, sw, Y  as for aria_qgemm(ARIA_FMT_W8A8) (device, 16-byte aligned).
 *   wait_limit_us      1 .. 4000000 (INVALID_ARG otherwise).
 * Shape rules as for aria_qgemm(ARIA_FMT_W8A8).
 */
aria_status aria_selftest_bounded_wait(int64_t M, int64_t N, int64_t K, const int8_t *Xq,
                                       const float *sx, const int8_t *Wq, const float *sw,
                                       void *Y, uint32_t wait_limit_us, void *stream);

/*
 * aria_device_status -- synchronise `stream`, then read and clear the device
 * status word of the current device. Returns ARIA_ERR_TIMEOUT if any kernel
 * of this library gave up on a bounded wait since the last call, ARIA_ERR_CUDA
 * if the stream reports an error, else ARIA_OK. Not for use during capture.
 */
aria_status aria_device_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ARIA_Q_H */
