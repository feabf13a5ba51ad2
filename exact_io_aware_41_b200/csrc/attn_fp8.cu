// Incoherent processing and e4m3 quantization for the 8-bit prefill path.
//
// FP8 attention with incoherent processing ("Flash Attention" overview, FA-3 paragraph; the
// FlashAttention generation comparison record, FA-3 "Workarounds"): Q and K are multiplied by the
// same random orthogonal matrix before they are rounded to 8 bits. Q K^T is unchanged by it (for
// orthogonal M, (Q M)(K M)^T = Q K^T), while the rotation spreads a few large channels over all
// of them, so the 8-bit grid loses less to outliers. Here M = diag(s) H / sqrt(d), with s a caller-
// chosen sign vector and H the Sylvester Hadamard matrix (H_1 = [1], H_2n = [[H, H], [H, -H]]),
// applied with the fast Walsh-Hadamard transform.
//
// Every (batch, head) of a tensor gets its own scale: codes = e4m3(y * 448 / amax), amax = max |y|
// over the head's rows, so the head's largest value lands on the largest finite e4m3 value. The
// steps are fixed, in fp32, so that a checker following them gets the same codes bit for bit:
//   1. y = x * s (exact: s = +-1)            2. butterflies (a, b) -> (a + b, a - b), stages h = 1,
//   2, 4, ..., d/2, pairs (j, j + h) within blocks of 2h     3. y *= fp32(1 / sqrt(d))
//   4. amax per head; scale = 448 / amax (1 if amax = 0)     5. code = e4m3 RNE, saturating(y * scale)
// Without signs (V), steps 1-3 are skipped.
#include <cuda_bf16.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn {

constexpr int kF8D = 128;  // head dim of the 8-bit path
constexpr int kF8Rows = 128;  // rows (tokens) per block, one per thread

// Row n of head (b, h) of x [B, N, H, d] -> y (rotated when signs != null), fp32.
__device__ __forceinline__ void load_rotate_row(const __nv_bfloat16* __restrict__ x, const float* __restrict__ signs,
                                                size_t row_off, float* y) {
  const uint4* src = reinterpret_cast<const uint4*>(x + row_off);
#pragma unroll
  for (int u = 0; u < kF8D / 8; ++u) {
    const uint4 w = src[u];
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      y[8 * u + 2 * i] = __uint_as_float(ww[i] << 16);
      y[8 * u + 2 * i + 1] = __uint_as_float(ww[i] & 0xFFFF0000u);
    }
  }
  if (signs == nullptr) return;
#pragma unroll
  for (int e = 0; e < kF8D; ++e) y[e] *= signs[e];
#pragma unroll
  for (int h = 1; h < kF8D; h <<= 1) {
#pragma unroll
    for (int i = 0; i < kF8D; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float a = y[j], b = y[j + h];
        y[j] = __fadd_rn(a, b);
        y[j + h] = __fsub_rn(a, b);
      }
    }
  }
  const float inv_sqrt_d = 0.0883883461356163f;  // fp32(1 / sqrt(128))
#pragma unroll
  for (int e = 0; e < kF8D; ++e) y[e] = __fmul_rn(y[e], inv_sqrt_d);
}

// Pass 1: amax[b * H + h] = max |y| over the head's rows (amax zeroed before the launch).
__global__ void __launch_bounds__(kF8Rows)
    fp8_amax_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ signs, float* __restrict__ amax,
                    int N, int H) {
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int n = blockIdx.x * kF8Rows + threadIdx.x;
  float m = 0.f;
  if (n < N) {
    float y[kF8D];
    load_rotate_row(x, signs, ((size_t(b) * N + n) * H + h) * kF8D, y);
#pragma unroll
    for (int e = 0; e < kF8D; ++e) m = fmaxf(m, fabsf(y[e]));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wm[kF8Rows / 32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = wm[0];
    for (int w = 1; w < kF8Rows / 32; ++w) t = fmaxf(t, wm[w]);
    // non-negative floats order like their bit patterns
    atomicMax(reinterpret_cast<unsigned int*>(amax) + bh, __float_as_uint(t));
  }
}

// Pass 2: the codes, [B, N, H, d] or, transposed, [B, H, d, N] (then N % 16 == 0).
__global__ void __launch_bounds__(kF8Rows)
    fp8_quant_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ signs,
                     const float* __restrict__ amax, uint8_t* __restrict__ codes, int N, int H, int transpose) {
  const int bh = blockIdx.y, b = bh / H, h = bh % H;
  const int n0 = blockIdx.x * kF8Rows;
  const int n = n0 + threadIdx.x;
  const float am = amax[bh];
  const float sc = am > 0.f ? __fdiv_rn(448.0f, am) : 1.0f;
  uint32_t w[kF8D / 4];
  if (n < N) {
    float y[kF8D];
    load_rotate_row(x, signs, ((size_t(b) * N + n) * H + h) * kF8D, y);
#pragma unroll
    for (int i = 0; i < kF8D / 4; ++i)
      w[i] = pack_e4m3x4(__fmul_rn(y[4 * i], sc), __fmul_rn(y[4 * i + 1], sc), __fmul_rn(y[4 * i + 2], sc),
                         __fmul_rn(y[4 * i + 3], sc));
  }
  if (!transpose) {
    if (n < N) {
      uint4* dst = reinterpret_cast<uint4*>(codes + ((size_t(b) * N + n) * H + h) * kF8D);
#pragma unroll
      for (int u = 0; u < kF8D / 16; ++u) dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
    }
    return;
  }
  // transposed: stage the block's 128 x 128 codes as [e][n] in shared memory, then write whole rows
  __shared__ __align__(16) uint8_t tile[kF8D * kF8Rows];
  if (n < N) {
#pragma unroll
    for (int i = 0; i < kF8D / 4; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) tile[(4 * i + k) * kF8Rows + threadIdx.x] = uint8_t(w[i] >> (8 * k));
  }
  __syncthreads();
  const int valid = min(kF8Rows, N - n0);  // a multiple of 16
  const int e = threadIdx.x;                // one d row per thread
  const uint4* src = reinterpret_cast<const uint4*>(tile + e * kF8Rows);
  uint4* dst = reinterpret_cast<uint4*>(codes + ((size_t(b) * H + h) * kF8D + e) * N + n0);
  for (int u = 0; u < valid / 16; ++u) dst[u] = src[u];
}

attn_status_t fp8_quantize_dispatch(const void* x, const float* signs, void* codes, float* amax, int B, int N, int H,
                                    int transpose, cudaStream_t stream) {
  if (cudaMemsetAsync(amax, 0, size_t(B) * H * sizeof(float), stream) != cudaSuccess) return ATTN_ERR_CUDA;
  const dim3 grid((N + kF8Rows - 1) / kF8Rows, B * H);
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
  fp8_amax_kernel<<<grid, kF8Rows, 0, stream>>>(xb, signs, amax, N, H);
  fp8_quant_kernel<<<grid, kF8Rows, 0, stream>>>(xb, signs, amax, reinterpret_cast<uint8_t*>(codes), N, H,
                                                 transpose);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

}  // namespace attn
