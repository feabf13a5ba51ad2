/*
 * attn.h -- C ABI of the B200 (sm_100a) exact-attention library.
 *
 * The library computes exact scaled-dot-product attention,
 *     O = softmax(scale * Q K^T) V,   LSE[i] = log sum_j exp(scale * q_i . k_j),
 * tile by tile with the online-softmax recurrence, so the N x N score and probability matrices
 * never reach HBM (the invariant of every FlashAttention version: "FlashAttention evolution"
 * article, section 1 "The Invariant and the Moving Bottleneck"; the per-row metadata beside O:
 * "Flash Attention" overview, section "The IO problem").
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - All tensors live in device memory owned by the caller. The library allocates nothing per call
 *    and keeps no pointer after a call returns. Work is enqueued on `stream` and runs
 *    asynchronously; no entry point synchronises the host.
 *  - bf16 tensors are dense and token-major:
 *        Q, O   [B, Nq, Hq, d]        K, V   [B, Nkv, Hkv, d]         LSE [B, Hq, Nq] (fp32)
 *    Decode: q, O [B, Hq, d]; caches [B, Nkv_cap, Hkv, d]; kv_lens int32 [B]; LSE [B, Hq].
 *  - Every pointer must be 16-byte aligned. d must be 32, 64, 128 or 256. Hq must be a multiple of
 *    Hkv; query head h reads kv head h / (Hq / Hkv) (contiguous groups).
 *  - Causal masking is bottom-right aligned: key j is visible to query i iff j <= i + Nkv - Nq.
 *    A query row that sees no key gets O = 0 and LSE = -inf.
 *  - Arithmetic: bf16 inputs, fp32 accumulation and softmax state, bf16 O, fp32 LSE in natural log.
 *  - Errors: argument errors are reported before anything is enqueued. Launch failures map to
 *    ATTN_ERR_CUDA. Kernel-side faults that the kernels detect themselves (a pipeline wait that
 *    gave up, an out-of-range decode length) are recorded in a device error word read by
 *    attn_get_last_error(). No entry point throws, aborts or traps.
 */
#ifndef EXACT_IO_AWARE_ATTN_H
#define EXACT_IO_AWARE_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null/misaligned pointer, non-positive size, Hq % Hkv != 0, ... */
  ATTN_ERR_UNSUPPORTED = 2, /* a head dim or GQA group the kernels are not built for */
  ATTN_ERR_WORKSPACE = 3,   /* decode workspace missing or smaller than attn_decode_workspace_bytes */
  ATTN_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed (launch, attribute, tensor map) */
  ATTN_ERR_TIMEOUT = 5      /* a kernel's bounded pipeline wait gave up (reported by attn_get_last_error) */
} attn_status_t;

/*
 * Prefill forward: O = softmax(scale * Q K^T) V and LSE, causal or not, with GQA.
 * ("FlashAttention evolution", sections 3-5: query-block parallelism, producer/consumer overlap,
 *  accumulators in tensor memory.)
 *
 *   q      [B, Nq, Hq, d]  bf16, read only
 *   k, v   [B, Nkv, Hkv, d] bf16, read only
 *   o      [B, Nq, Hq, d]  bf16, written
 *   lse    [B, Hq, Nq]     fp32, written (natural-log log-sum-exp of the scaled scores)
 *   B, Hq, Hkv, Nq, Nkv >= 1; d in {32, 64, 128, 256}; scale > 0 and finite (1/sqrt(d) usually);
 *   causal 0 or 1.
 * Returns ATTN_OK once the kernel is enqueued.
 *
 * Concurrency: the persistent kernel hands out its work from one of 256 claim counters in device
 * memory, assigned to launches round robin and returned to zero by each launch's last CTA. Launches
 * on one stream never overlap, and launches on different streams are safe as long as fewer than
 * 256 later prefill launches on that device start before an earlier one finishes (a launch held
 * back behind a cross-stream wait while 256 others run past it would share a counter). d = 256
 * launches clusters of two CTAs (2-SM tensor-core products) with a fixed share of the work per
 * cluster and uses no claim counter; it needs a device and context where clusters of two can be
 * resident (ATTN_ERR_CUDA otherwise).
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                       int Hkv, int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream);

/*
 * 8-bit inputs for attn_fwd_fp8, with incoherent processing (FP8 with incoherent processing:
 * "Flash Attention" overview, FA-3 paragraph; FlashAttention generation comparison record, FA-3
 * "Workarounds"). For each row of x (bf16 [B, N, H, d], d = 128), in fp32 and in this order:
 *   y = x * signs (elementwise; skipped, with the next two steps, when signs is NULL);
 *   fast Walsh-Hadamard butterflies (a, b) -> (a + b, a - b) for h = 1, 2, 4, ..., 64 on the pairs
 *   (j, j + h) inside blocks of 2h (the Sylvester Hadamard matrix); y *= fp32(1 / sqrt(d));
 * then amax[b, h] = max |y| over the head's rows and codes = e4m3(y * fp32(448 / amax[b, h]))
 * (round to nearest even, saturating at +-448; scale 1 when amax = 0). A rotation is orthogonal, so
 * rotating Q and K with the same signs leaves Q K^T unchanged while spreading outlier channels.
 *   x      bf16 [B, N, H, d], read only;  signs fp32 [d] of +1 / -1 (device) or NULL
 *   codes  uint8 (e4m3), written: [B, N, H, d], or [B, H, d, N] when transpose = 1 (the layout
 *          attn_fwd_fp8 takes V in; then N must be a multiple of 16)
 *   amax   fp32 [B, H], written (first zeroed on the stream, then raised by the kernels)
 *   B, N, H >= 1, B * H <= 65535; d = 128 (ATTN_ERR_UNSUPPORTED otherwise).
 */
attn_status_t attn_fp8_quantize(const void* x, const float* signs, void* codes, float* amax, int B, int N, int H,
                                int d, int transpose, cudaStream_t stream);

/*
 * Prefill forward on 8-bit operands: O = softmax(scale * Q' K'^T) V' and LSE, where Q', K', V' are
 * the values the codes stand for (code value * amax / 448 per batch and head). The products run on
 * the tensor cores in e4m3 (kind::f8f6f4) with fp32 accumulation; P is rounded to e4m3 before the PV
 * product; softmax state, row sums and LSE are fp32 as in attn_fwd.
 *   q8     uint8 [B, Nq, Hq, d] codes of Q (rotated), k8 uint8 [B, Nkv, Hkv, d] codes of K (rotated
 *          with the same signs), vt8 uint8 [B, Hkv, d, Nkv] codes of V, transposed
 *   amax_q fp32 [B, Hq], amax_k, amax_v fp32 [B, Hkv] as attn_fp8_quantize wrote them
 *   o      bf16 [B, Nq, Hq, d], lse fp32 [B, Hq, Nq], written
 *   d = 128 (ATTN_ERR_UNSUPPORTED otherwise); Nkv a multiple of 16 (ATTN_ERR_INVALID_ARG otherwise);
 *   everything else as attn_fwd.
 */
attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* amax_q, const float* amax_k,
                           const float* amax_v, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                           float scale, int causal, cudaStream_t stream);

/*
 * Backward pass: the gradients of a scalar loss L through O = softmax(scale * Q K^T) V, given
 * dO = dL/dO, recomputing S tile by tile instead of storing it (FlashAttention generation
 * comparison record, "Workarounds": recompute S in backward). With P = exp(scale * S - LSE):
 *   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
 *   dQ = scale * dS K,  dK = scale * dS^T Q  (dK, dV summed over the query heads of a GQA group).
 * Products on the tensor cores in bf16 with fp32 accumulation; P and dS are rounded to bf16 before
 * the products that take them; dQ is accumulated in fp32 in the workspace.
 *   q, o, dout  bf16 [B, Nq, Hq, d];  k, v bf16 [B, Nkv, Hkv, d];  lse fp32 [B, Hq, Nq] (from
 *               attn_fwd with the same q, k, v, scale and causal flag), all read only
 *   dq          bf16 [B, Nq, Hq, d];  dk, dv bf16 [B, Nkv, Hkv, d], written
 *   workspace   caller-owned, at least attn_bwd_workspace_bytes(B, Hq, Nq, d) bytes, 256-byte
 *               aligned, no initialisation needed (the call zeroes what it accumulates into)
 *   d = 128 (ATTN_ERR_UNSUPPORTED otherwise); everything else as attn_fwd.
 */
size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq, int d);
attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                       void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nkv, int d, float scale,
                       int causal, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Bytes of device workspace attn_decode_splitkv needs: the per-split partial outputs
 * (fp32 [B, Hq, n_splits, d]) and partial LSEs (fp32 [B, Hq, n_splits]), n_splits =
 * ceil(Nkv_cap / chunk). chunk = 0 selects the same automatic chunk attn_decode_splitkv uses.
 * Returns 0 for invalid arguments.
 */
size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int Nkv_cap, int chunk);

/* The KV chunk (tokens per split) chosen when chunk = 0 is passed. */
int attn_decode_default_chunk(int B, int Hkv, int Nkv_cap);

/*
 * Flash-Decoding split-KV forward for one query token per sequence, followed by the LSE-weighted
 * combine, both enqueued on `stream` ("FlashAttention evolution", section 6 "Flash-Decoding: A
 * Different Parallel Shape": partitions of the KV sequence each produce a partial max, sum and
 * weighted output; a final reduction merges them with the online-softmax identity).
 *
 *   q                [B, Hq, d] bf16
 *   k_cache, v_cache [B, Nkv_cap, Hkv, d] bf16; only tokens [0, kv_lens[b]) of sequence b are read
 *   kv_lens          int32 [B] in device memory, each in [0, Nkv_cap] (out-of-range values are
 *                    clamped and flagged in the device error word)
 *   o                [B, Hq, d] bf16, written;  lse [B, Hq] fp32, written (-inf when kv_lens[b] = 0)
 *   d in {32, 64, 128, 256}; Hq / Hkv in {1, 2, 4, 8}; chunk = tokens per split (multiple of 64)
 *                    or 0 (automatic: about eight splits per SM of the current device).
 *   workspace        caller-owned device memory of at least attn_decode_workspace_bytes(...) bytes;
 *                    fully overwritten before it is read, so it needs no initialisation.
 * Sizes the kernels cannot take (B or Hkv above 65535, more than 25600 splits per row) return
 * ATTN_ERR_UNSUPPORTED before either kernel is enqueued.
 */
attn_status_t attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* kv_lens, int Nkv_cap, void* o, float* lse, int B, int Hq,
                                  int Hkv, int d, float scale, int chunk, void* workspace,
                                  size_t workspace_bytes, cudaStream_t stream);

/*
 * Size of the fixed device array that attn_decode_splitkv_static keeps its partials in (48 MiB).
 * The array belongs to the library's device code: it is committed on a GPU when that code is first
 * loaded there (with CUDA's default lazy loading, the first call of any library entry point that
 * launches a kernel, or the address look-up below), and held until the process exits. Under memory
 * pressure that first load can fail and surfaces as ATTN_ERR_CUDA, so make one warm-up call at
 * start-up.
 */
#define ATTN_DECODE_STATIC_SCRATCH_BYTES (48u << 20)

/*
 * attn_decode_splitkv without a workspace argument, for callers that cannot allocate device
 * memory: a plugin running inside a host runtime that owns all device memory and offers it no
 * allocator, or a latency-critical loop that must not call cudaMalloc (it can synchronise the device
 * and can fail under memory pressure). The pages have no counterpart to this entry point; it only
 * changes where the per-split partials live.
 *
 * Arguments, result and arithmetic are those of attn_decode_splitkv. The caller still passes q, the
 * caches, kv_lens, o and lse. The partials go to one file-scope device array of
 * ATTN_DECODE_STATIC_SCRATCH_BYTES; nothing is allocated and no allocating routine is called.
 *  - Sizes whose partials (see attn_decode_workspace_bytes) exceed that array are rejected with
 *    ATTN_ERR_WORKSPACE before anything is enqueued; a larger chunk makes the partials smaller.
 *  - The first call on each device looks up the array's device address on the current device
 *    (cudaGetSymbolAddress), which also loads the library's device code there and commits the
 *    array, and caches it; make that first call at start-up, before any stream capture.
 *  - Every call shares the one array and it keeps the last call's partials. Calls that overlap on
 *    the GPU (on different streams, or from different host threads without ordering) race on it.
 */
attn_status_t attn_decode_splitkv_static(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* kv_lens, int Nkv_cap, void* o, float* lse, int B,
                                         int Hq, int Hkv, int d, float scale, int chunk, cudaStream_t stream);

/*
 * The combine step on its own: merges n_splits partial states per row with
 *     LSE = log sum_s exp(lse_s),   O = sum_s exp(lse_s - LSE) * o_s
 * ("FlashAttention evolution", section 6). Partials with lse_s = -inf contribute nothing; a row
 * whose partials are all -inf gets O = 0 and LSE = -inf.
 *
 *   part_o   fp32 [rows, n_splits, d] (each o_s already normalised by its own sum)
 *   part_lse fp32 [rows, n_splits]
 *   o        bf16 [rows, d], written;  lse fp32 [rows], written
 *   rows >= 1, 1 <= n_splits <= 25600, d in {32, 64, 128, 256}.
 */
attn_status_t attn_decode_combine(const float* part_o, const float* part_lse, int rows, int n_splits, int d,
                                  void* o, float* lse, cudaStream_t stream);

/*
 * Reads and clears the device error word (synchronises the calling thread with the device).
 * ATTN_OK if no kernel recorded a fault since the last call, ATTN_ERR_TIMEOUT if a bounded
 * pipeline wait gave up, ATTN_ERR_INVALID_ARG if a decode length was out of range, ATTN_ERR_CUDA
 * if the word could not be read or a kernel found its shared memory misaligned (and did nothing).
 */
attn_status_t attn_get_last_error(void);

/* Static, human-readable name of a status code. */
const char* attn_status_string(attn_status_t status);

/*
 * Name of the kernel(s) that `which` selects (0 = prefill forward, bf16 or 8-bit, 1 = decode split,
 * 2 = decode combine, 3 = backward), for recording which kernel a measurement ran (the evolution article's section 1.1
 * asks that a benchmark name its kernel). Returns NULL for an unknown index.
 */
const char* attn_kernel_name(int which);

/*
 * Test hook for the bounded waits: launches a one-CTA kernel that waits on an mbarrier nothing
 * ever completes, with the given limit in microseconds, then returns normally. Afterwards
 * attn_get_last_error() reports ATTN_ERR_TIMEOUT. Nothing faults or hangs.
 */
attn_status_t attn_selftest_bounded_wait(unsigned int limit_us, cudaStream_t stream);

/*
 * Test hook for the waits between the two CTAs of a cluster (the d = 256 prefill's CTA pairs):
 * launches one cluster of two CTAs; in each, one thread waits with the given limit (microseconds) on
 * an mbarrier of its own CTA. cross_arrive = 1: each CTA first arrives on the other's barrier through
 * its cluster address, both waits complete and attn_get_last_error() stays ATTN_OK; cross_arrive =
 * 0: nothing arrives, both waits run out and it reports ATTN_ERR_TIMEOUT. Nothing faults or hangs.
 * ATTN_ERR_INVALID_ARG for limit_us outside [1, 10^7] or cross_arrive other than 0 or 1.
 */
attn_status_t attn_selftest_pair_wait(unsigned int limit_us, int cross_arrive, cudaStream_t stream);

/*
 * Test hook for the FMA-pipe exponential (Cody-Waite range reduction and a degree-3 polynomial;
 * the "emulated exponentials" the FlashAttention generation comparison record describes for
 * FA-4). The prefill kernels can evaluate part of their exponentials with it (a build option, off
 * by default). Writes y[i] = 2^x[i] through that approximation for n device floats (x < 127.5;
 * inputs below -125 give 2^-125 times the polynomial's value at 0). Max relative error 7.5e-5 on
 * [-125, 127.5). x and y are 4-byte aligned device pointers, n >= 1; asynchronous on `stream`.
 */
attn_status_t attn_selftest_exp2_poly(const float* x, float* y, int n, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_IO_AWARE_ATTN_H */
