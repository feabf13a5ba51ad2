// Flash-Decoding for sm_100a: single-query attention over a long KV cache, split along the KV
// sequence ("FlashAttention evolution" article, section 6 "Flash-Decoding: A Different Parallel
// Shape"). Each CTA owns (batch b, kv head g, KV partition s) and produces, for the G = Hq/Hkv query
// heads that share kv head g, a partial output normalised by its own sum and the partial
// log-sum-exp. A second kernel merges the partitions with the online-softmax identity.
//
// The split kernel is HBM-bound: every K/V byte is read once and serves G query heads. Inside a
// warp, LPT = d/8 lanes cover one token row with one 16-byte load each (coalesced: a warp load
// reads 32/LPT whole rows), U token rows are in flight per lane, and the next iteration's rows are
// loaded before the current ones are used. Dot products are reduced across the LPT lanes with a
// reduce-scatter butterfly, so that G*U partial sums cost G*U-1 shuffles instead of (G*U)*log2(LPT).
#include <cuda_bf16.h>
#include <math.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn {

constexpr float kDecodeTau = 8.0f;  // log2-units slack before the accumulators are rescaled
constexpr int kDecodeWarps = 4;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float* f) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <int D, int G>
struct DecCfg {
  static constexpr int LPT = D / 8;                       // lanes per token row
  static constexpr int R = 32 / LPT;                      // token rows per warp-wide load
  static constexpr int U0 = LPT / G;
  static constexpr int U = U0 < 1 ? 1 : (U0 > 4 ? 4 : U0);  // rows in flight per lane
  static constexpr int NV = G * U;                        // partial sums per lane before reduction
  static constexpr int TPI = U * R;                       // tokens per warp iteration
  static constexpr int LOG_LPT = (LPT == 8) ? 3 : (LPT == 16) ? 4 : 5;
  static constexpr int LOG_NV = (NV == 1) ? 0 : (NV == 2) ? 1 : (NV == 4) ? 2 : (NV == 8) ? 3 : (NV == 16) ? 4 : 5;
  static constexpr int LOG_G = (G == 1) ? 0 : (G == 2) ? 1 : (G == 4) ? 2 : 3;
  static constexpr int SH = LOG_LPT - LOG_NV;             // low lane bits that only duplicate a value
  static_assert(NV <= LPT, "one partial sum per lane group after the reduce-scatter");
};

// Eight query heads per kv head need 64 accumulator registers per lane: allow two CTAs per SM
// (up to 255 registers) there, four CTAs (128 registers, 16 warps per SM) otherwise.
template <int D, int G>
__global__ void __launch_bounds__(kDecodeWarps * 32, (G >= 8) ? 2 : 4)
    decode_split_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                        const __nv_bfloat16* __restrict__ vc, const int32_t* __restrict__ kv_lens, int Nkv_cap,
                        int Hkv, int chunk, int n_splits, float scale_log2, float* __restrict__ part_o,
                        float* __restrict__ part_lse) {
  using C = DecCfg<D, G>;
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = Hkv * G;

  int L = kv_lens[b];
  if (L < 0 || L > Nkv_cap) {
    if (threadIdx.x == 0 && s == 0 && g == 0) atomicOr(&g_error_word, kErrBadLengthBit);
    L = L < 0 ? 0 : Nkv_cap;
  }
  const int t_begin = s * chunk;
  const int t_end = min(L, t_begin + chunk);
  const size_t row0 = size_t(b) * Hq + size_t(g) * G;  // first query head row of this group
  if (t_begin >= t_end) {
    if (threadIdx.x < G) part_lse[(row0 + threadIdx.x) * n_splits + s] = -INFINITY;
    return;
  }

  // the group's query rows, pre-scaled by scale*log2(e) (scores come out in log2 units)
  __shared__ __align__(16) float sq[G][D];
  for (int i = threadIdx.x; i < G * D / 8; i += blockDim.x) {
    const int hh = i / (D / 8), e = (i % (D / 8)) * 8;
    float f[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(q + (row0 + hh) * D + e), f);
#pragma unroll
    for (int k = 0; k < 8; ++k) sq[hh][e + k] = f[k] * scale_log2;
  }
  __syncthreads();

  const int sub = lane % C::LPT;   // which 8 elements of d this lane covers
  const int r = lane / C::LPT;     // which token row of a warp-wide load
  const int e0 = sub * 8;
  const size_t tok_stride = size_t(Hkv) * D;  // elements between consecutive tokens
  const __nv_bfloat16* kbase = kc + (size_t(b) * Nkv_cap * Hkv + g) * D + e0;
  const __nv_bfloat16* vbase = vc + (size_t(b) * Nkv_cap * Hkv + g) * D + e0;

  // value index held by this lane after the reduce-scatter: vi = u*G + head
  const int vi = (lane % C::LPT) >> C::SH;
  const int my_head = vi % G;
  const int my_u = vi / G;

  float m_ref[G];  // per-head reference max (log2 units), uniform across the warp
  float acc[G][8];
  float l_lane = 0.f;  // partial sum of p for (my_head), over this lane's tokens
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    m_ref[hh] = -INFINITY;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[hh][i] = 0.f;
  }

  // Rows of a warp iteration: token tb + u*R + r for u < U. Loads past t_end are skipped (zeros).
  auto load_rows = [&](const __nv_bfloat16* base, int tb, uint4* dst) {
#pragma unroll
    for (int uu = 0; uu < C::U; ++uu) {
      const int t = tb + uu * C::R + r;
      dst[uu] = (t < t_end) ? __ldcs(reinterpret_cast<const uint4*>(base + size_t(t) * tok_stride))
                            : make_uint4(0, 0, 0, 0);
    }
  };

  const int stride = kDecodeWarps * C::TPI;
  int tb = t_begin + warp * C::TPI;
  uint4 kr[C::U], vr[C::U];
  if (tb < t_end) load_rows(kbase, tb, kr);
  for (; tb < t_end; tb += stride) {
    // V rows of this iteration are only needed after the softmax: issue them first
    load_rows(vbase, tb, vr);

    // ---- partial dot products: val[u*G + head] over this lane's 8 elements
    float val[C::NV];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float4 qa = *reinterpret_cast<const float4*>(&sq[hh][e0]);
      const float4 qb = *reinterpret_cast<const float4*>(&sq[hh][e0 + 4]);
      const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int uu = 0; uu < C::U; ++uu) {
        float kf[8];
        bf16x8_to_f32(kr[uu], kf);
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaf(qv[i], kf[i], a);
        val[uu * G + hh] = a;
      }
    }
    // the K registers are free again: start the next iteration's K rows now
    const int tn = tb + stride;
    if (tn < t_end) load_rows(kbase, tn, kr);

    // ---- reduce across the LPT lanes of a token row: reduce-scatter while >1 value, then all-reduce
    {
      int cnt = C::NV;
#pragma unroll
      for (int o = C::LPT / 2; o >= 1; o >>= 1) {
        if (cnt > 1) {
          const bool upper = (lane & o) != 0;
          const int half = cnt / 2;
#pragma unroll
          for (int i = 0; i < C::NV / 2; ++i) {
            if (i < half) {
              const float send = upper ? val[i] : val[i + half];
              const float keep = upper ? val[i + half] : val[i];
              val[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
          }
          cnt = half;
        } else {
          val[0] += __shfl_xor_sync(0xffffffffu, val[0], o);
        }
      }
    }
    // score (log2 units) of token (my_u, r) for my_head; invalid tokens are -inf
    const int my_t = tb + my_u * C::R + r;
    const float sc = (my_t < t_end) ? val[0] : -INFINITY;

    // ---- per-head max over the iteration's tokens: xor over the u and r lane bits
    float mx = sc;
#pragma unroll
    for (int o = 1 << (C::SH + C::LOG_G); o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float mxh[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) mxh[hh] = __shfl_sync(0xffffffffu, mx, hh << C::SH);

    // ---- conditional rescale (uniform across the warp)
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      if (mxh[hh] - m_ref[hh] > kDecodeTau) {
        const float alpha = ex2(m_ref[hh] - mxh[hh]);  // 0 on the first live iteration
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[hh][i] *= alpha;
        if (my_head == hh) l_lane *= alpha;
        m_ref[hh] = mxh[hh];
      }
    }
    float mref_mine = m_ref[0];
#pragma unroll
    for (int hh = 1; hh < G; ++hh)
      if (my_head == hh) mref_mine = m_ref[hh];
    const float p = (sc == -INFINITY) ? 0.f : ex2(sc - mref_mine);
    l_lane += p;

    // ---- acc[head] += p(token, head) * v(token)
#pragma unroll
    for (int uu = 0; uu < C::U; ++uu) {
      float vf[8];
      bf16x8_to_f32(vr[uu], vf);
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float pp = __shfl_sync(0xffffffffu, p, r * C::LPT + ((uu * G + hh) << C::SH));
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[hh][i] = fmaf(pp, vf[i], acc[hh][i]);
      }
    }
  }

  // ---- warp-level totals: acc over the R token rows, l over the distinct (u, r) lanes of a head
#pragma unroll
  for (int o = C::LPT; o < 32; o <<= 1)
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[hh][i] += __shfl_xor_sync(0xffffffffu, acc[hh][i], o);
#pragma unroll
  for (int o = 1 << (C::SH + C::LOG_G); o < 32; o <<= 1) l_lane += __shfl_xor_sync(0xffffffffu, l_lane, o);

  // ---- combine the warps of the CTA through shared memory
  __shared__ float sm_m[kDecodeWarps][G], sm_l[kDecodeWarps][G];
  __shared__ float sm_acc[kDecodeWarps][G][D];
  if (lane < G) {
    sm_m[warp][lane] = m_ref[0];
#pragma unroll
    for (int hh = 1; hh < G; ++hh)
      if (lane == hh) sm_m[warp][lane] = m_ref[hh];
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
    if (lane == (hh << C::SH)) sm_l[warp][hh] = l_lane;
  if (r == 0) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
#pragma unroll
      for (int i = 0; i < 8; ++i) sm_acc[warp][hh][e0 + i] = acc[hh][i];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int hh = idx / D, e = idx % D;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) m = fmaxf(m, sm_m[w][hh]);
    float lt = 0.f, ot = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecodeWarps; ++w) {
        const float f = ex2(sm_m[w][hh] - m);
        lt = fmaf(f, sm_l[w][hh], lt);
        ot = fmaf(f, sm_acc[w][hh][e], ot);
      }
    }
    const size_t row = row0 + hh;
    part_o[(row * n_splits + s) * D + e] = (lt > 0.f) ? ot / lt : 0.f;
    if (e == 0) part_lse[row * n_splits + s] = (lt > 0.f) ? (m * 0.6931471805599453f + logf(lt)) : -INFINITY;
  }
}

// One CTA per output row; each thread owns EPT consecutive elements of d. The partial LSEs are
// reduced first, the live splits are compacted into a list in shared memory, and the partial
// outputs are accumulated with four independent loads in flight per thread.
// LSE = log sum_s exp(lse_s), O = sum_s exp(lse_s - LSE) o_s.
template <int D>
struct CombCfg {
  static constexpr int NT = D <= 128 ? 32 : 64;  // threads per row
  static constexpr int EPT = D / NT;             // elements per thread (2 or 4)
};

template <int EPT>
struct VecF;
template <>
struct VecF<2> {
  using T = float2;
  static __device__ __forceinline__ void fma(float w, const float* src, float* acc) {
    const float2 v = *reinterpret_cast<const float2*>(src);
    acc[0] = fmaf(w, v.x, acc[0]);
    acc[1] = fmaf(w, v.y, acc[1]);
  }
};
template <>
struct VecF<4> {
  static __device__ __forceinline__ void fma(float w, const float* src, float* acc) {
    const float4 v = *reinterpret_cast<const float4*>(src);
    acc[0] = fmaf(w, v.x, acc[0]);
    acc[1] = fmaf(w, v.y, acc[1]);
    acc[2] = fmaf(w, v.z, acc[2]);
    acc[3] = fmaf(w, v.w, acc[3]);
  }
};

template <int D>
__global__ void __launch_bounds__(CombCfg<D>::NT)
    decode_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse, int rows,
                          int n_splits, __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  constexpr int NT = CombCfg<D>::NT, EPT = CombCfg<D>::EPT;
  extern __shared__ float s_w[];  // [n_splits] weights of the live splits, then their indices
  __shared__ float red[NT / 32];
  __shared__ int n_live;
  int* live = reinterpret_cast<int*>(s_w + n_splits);
  const int row = blockIdx.x;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const float* pl = part_lse + size_t(row) * n_splits;
  float mx = -INFINITY;
  for (int s = t; s < n_splits; s += NT) mx = fmaxf(mx, pl[s]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  if (t == 0) n_live = 0;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) mx = fmaxf(mx, red[w]);
  // weights and the compacted list of live splits (the order does not matter for the sums)
  for (int s = t; s < n_splits; s += NT) {
    const float ls = pl[s];
    if (ls != -INFINITY) {
      const int k = atomicAdd(&n_live, 1);
      live[k] = s;
      s_w[k] = expf(ls - mx);
    }
  }
  __syncthreads();
  const int nl = n_live;
  float acc[4][EPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < EPT; ++e) acc[i][e] = 0.f;
  float z = 0.f;
  const float* po = part_o + size_t(row) * n_splits * D + t * EPT;
  int k = 0;
  for (; k + 4 <= nl; k += 4) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float w = s_w[k + i];
      z += w;
      VecF<EPT>::fma(w, po + size_t(live[k + i]) * D, acc[i]);
    }
  }
  for (; k < nl; ++k) {
    const float w = s_w[k];
    z += w;
    VecF<EPT>::fma(w, po + size_t(live[k]) * D, acc[0]);
  }
  const float inv = (z > 0.f) ? 1.0f / z : 0.f;
  __nv_bfloat16* orow = o + size_t(row) * D + t * EPT;
#pragma unroll
  for (int e = 0; e < EPT; e += 2) {
    const float a0 = (acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e]);
    const float a1 = (acc[0][e + 1] + acc[1][e + 1]) + (acc[2][e + 1] + acc[3][e + 1]);
    *reinterpret_cast<uint32_t*>(orow + e) = pack_bf16x2(a0 * inv, a1 * inv);
  }
  if (t == 0) lse[row] = (z > 0.f) ? mx + logf(z) : -INFINITY;
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
int decode_default_chunk(int B, int Hkv, int Nkv_cap) {
  // aim for ~8 live CTAs per SM if every sequence were full, in multiples of 64 tokens, at most 1024
  const long long total = (long long)B * Hkv * Nkv_cap;
  long long c = total / (148LL * 8);
  c = (c + 63) / 64 * 64;
  if (c < 64) c = 64;
  if (c > 1024) c = 1024;
  return int(c);
}

size_t decode_workspace(int B, int Hq, int d, int Nkv_cap, int chunk) {
  const size_t n_splits = (size_t(Nkv_cap) + chunk - 1) / chunk;
  const size_t po = size_t(B) * Hq * n_splits * d * sizeof(float);
  const size_t pl = size_t(B) * Hq * n_splits * sizeof(float);
  return ((po + 255) / 256) * 256 + pl;
}

template <int D, int G>
static attn_status_t launch_split(const void* q, const void* kc, const void* vc, const int32_t* lens, int cap,
                                  int B, int Hkv, int chunk, int n_splits, float scale, float* po, float* pl,
                                  cudaStream_t stream) {
  dim3 grid(n_splits, Hkv, B);
  decode_split_kernel<D, G><<<grid, kDecodeWarps * 32, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(kc),
      reinterpret_cast<const __nv_bfloat16*>(vc), lens, cap, Hkv, chunk, n_splits,
      scale * 1.4426950408889634f, po, pl);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

template <int D>
static attn_status_t split_by_group(int G, const void* q, const void* kc, const void* vc, const int32_t* lens,
                                    int cap, int B, int Hkv, int chunk, int n_splits, float scale, float* po,
                                    float* pl, cudaStream_t st) {
  switch (G) {
    case 1: return launch_split<D, 1>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    case 2: return launch_split<D, 2>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    case 4: return launch_split<D, 4>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    case 8: return launch_split<D, 8>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

attn_status_t decode_split_dispatch(const void* q, const void* kc, const void* vc, const int32_t* lens, int cap,
                                    int B, int Hq, int Hkv, int d, float scale, int chunk, int n_splits,
                                    float* po, float* pl, cudaStream_t st) {
  const int G = Hq / Hkv;
  switch (d) {
    case 64: return split_by_group<64>(G, q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    case 128: return split_by_group<128>(G, q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    case 256: return split_by_group<256>(G, q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

attn_status_t decode_combine_dispatch(const float* po, const float* pl, int rows, int n_splits, int d, void* o,
                                      float* lse, cudaStream_t st) {
  const dim3 grid(rows);
  __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(o);
  const size_t sm = size_t(n_splits) * (sizeof(float) + sizeof(int));  // weights + live split list
  if (sm > 200 * 1024) return ATTN_ERR_UNSUPPORTED;
  switch (d) {
    case 64:
      if (sm > 48 * 1024) cudaFuncSetAttribute(decode_combine_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm));
      decode_combine_kernel<64><<<grid, CombCfg<64>::NT, sm, st>>>(po, pl, rows, n_splits, ob, lse);
      break;
    case 128:
      if (sm > 48 * 1024) cudaFuncSetAttribute(decode_combine_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm));
      decode_combine_kernel<128><<<grid, CombCfg<128>::NT, sm, st>>>(po, pl, rows, n_splits, ob, lse);
      break;
    case 256:
      if (sm > 48 * 1024) cudaFuncSetAttribute(decode_combine_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sm));
      decode_combine_kernel<256><<<grid, CombCfg<256>::NT, sm, st>>>(po, pl, rows, n_splits, ob, lse);
      break;
    default: return ATTN_ERR_UNSUPPORTED;
  }
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

}  // namespace attn
