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

// ============================================================================================
// Split kernel, tensor-core variant (d = 64 or 128).
//
// A producer warp streams the CTA's K and V rows for its kv head through a STAGES-deep
// shared-memory ring with TMA (tiles of TT tokens, 128-byte swizzle); the K/V rows are read from
// HBM exactly once and never pass through registers on their way in. Each of the NW consumer warps
// takes 16 tokens of every tile and does the two per-tile products on warp-level tensor cores
// (mma.sync m16n8k16, bf16 in, fp32 accumulate): S = Q K^T with the group's query heads as the 16
// rows (zero-padded past G), then O += P V with P taken straight from the S accumulators. The
// online softmax runs on the accumulator fragments: lane (g, t) owns head g's scores for four of the
// warp's tokens, so a row max is two shuffles. This keeps the per-token instruction count small
// enough for the kernel to stay bound by HBM bandwidth.
// ============================================================================================
template <int D>
struct DecTcCfg {
  static constexpr int NW = 4;                  // consumer warps
  static constexpr int TT = 16 * NW;            // tokens per tile
  static constexpr int STAGES = 3;
  // Rows of a tile are stored in chunks of CE elements along d: 64 elements (128 bytes) with the
  // 128-byte swizzle for d >= 64; d = 32 uses plain 64-byte rows (no swizzle).
  static constexpr int CE = D < 64 ? D : 64;
  static constexpr int ROWB = CE * 2;           // bytes per stored row of a chunk
  static constexpr bool SWIZZLE = (D >= 64);
  static constexpr int NCHUNK = D / CE;
  static constexpr int CHUNK_BYTES = TT * ROWB;
  static constexpr int TILE_BYTES = TT * D * 2;  // one K or V tile
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int THREADS = 32 * (NW + 1);
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 2 * STAGES * 8 + 16;
};

// Byte address of element (row, col) of a TT x D bf16 tile written by TMA. With the 128-byte
// swizzle (d >= 64): 64-column chunks of 128-byte rows, the 16-byte unit index XOR-ed with the row
// index mod 8. Without (d = 32): one chunk of plain 64-byte rows.
template <int D>
__device__ __forceinline__ uint32_t dec_sw128(uint32_t tile, int row, int col) {
  using C = DecTcCfg<D>;
  if constexpr (C::SWIZZLE) {
    const int chunk = col >> 6, unit = (col & 63) >> 3;
    return tile + chunk * C::CHUNK_BYTES + row * 128 + ((unit ^ (row & 7)) << 4) + ((col & 7) << 1);
  } else {
    return tile + row * C::ROWB + (col << 1);
  }
}

template <int D, int G>
__global__ void __launch_bounds__(DecTcCfg<D>::THREADS, 2)
    decode_split_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ kv_lens, int Nkv_cap,
                           int Hkv, int chunk, int n_splits, float scale_log2, float* __restrict__ part_o,
                           float* __restrict__ part_lse, unsigned long long timeout_ns) {
  using C = DecTcCfg<D>;
  static_assert(G <= 8, "query heads of a group fill at most the upper half of the 16 MMA rows");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + C::STAGES);
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = Hkv * G;
  const uint64_t T = timeout_ns;

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
  const int n_tiles = (t_end - t_begin + C::TT - 1) / C::TT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::NW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == C::NW) {
    // ================================ TMA producer ================================
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      int i = 0;
      for (; i < n_tiles; ++i) {
        const int st = i % C::STAGES;
        if (!mbar_wait(&empty[st], uint32_t(((i / C::STAGES) & 1) ^ 1), abort_flag, T)) break;
        mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
        uint8_t* kt = smem + st * C::STAGE_BYTES;
        const int tok = t_begin + i * C::TT;
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c) {
          tma_load_4d(kt + c * C::CHUNK_BYTES, &tmK, &full[st], c * C::CE, g, tok, b);
          tma_load_4d(kt + C::TILE_BYTES + c * C::CHUNK_BYTES, &tmV, &full[st], c * C::CE, g, tok, b);
        }
      }
      if (i < n_tiles) {
        // gave up: let the copies in flight land before the CTA exits
        for (int st = 0; st < C::STAGES; ++st) {
          const int fills = (i - st + C::STAGES - 1) / C::STAGES;
          if (fills > 0) mbar_wait(&full[st], (fills - 1) & 1, nullptr, 100000000ull);
        }
      }
    }
    return;  // the consumers' closing barrier below counts only the consumer warps
  }

  // ================================ consumer warps ================================
  const int gid = lane >> 2, tid = lane & 3;  // mma fragment coordinates
  // A fragments of Q (rows = query heads of the group, zero past G), one pair per 16-wide k-step
  uint32_t qa[D / 16][2];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    if (gid < G) {
      const __nv_bfloat16* qr = q + (row0 + gid) * D + kk * 16 + 2 * tid;
      qa[kk][0] = *reinterpret_cast<const uint32_t*>(qr);
      qa[kk][1] = *reinterpret_cast<const uint32_t*>(qr + 8);
    } else {
      qa[kk][0] = qa[kk][1] = 0u;
    }
  }
  float o[D / 8][4];  // O rows gid (and padding rows gid + 8), columns 8n + 2t, 8n + 2t + 1
#pragma unroll
  for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m_ref = -INFINITY;  // head gid's reference max (log2 units of the scaled scores)
  float l = 0.f;            // partial sum of p over this lane's tokens
  const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: which 8x8 matrix this lane addresses, and its row

  bool ok = true;
  for (int i = 0; i < n_tiles; ++i) {
    const int st = i % C::STAGES;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[st], uint32_t((i / C::STAGES) & 1), abort_flag, T))) {
      ok = false;
      break;
    }
    const uint32_t kt = smem_u32(smem + st * C::STAGE_BYTES);
    const uint32_t vt = kt + C::TILE_BYTES;
    const int my_tok0 = t_begin + i * C::TT + 16 * warp;  // this warp's tokens: my_tok0 .. my_tok0 + 15
    const int valid = t_end - my_tok0;                     // how many of them exist
    if (valid > 0) {
      // ---- S = Q K^T over 16 tokens (two 8-token column blocks)
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t b00, b01, b10, b11;
        ldsm_x4(dec_sw128<D>(kt, 16 * warp + 8 * (mi >> 1) + rr, kk * 16 + 8 * (mi & 1)), b00, b01, b10, b11);
        mma_bf16_16816(sacc[0], qa[kk][0], 0u, qa[kk][1], 0u, b00, b01);
        mma_bf16_16816(sacc[1], qa[kk][0], 0u, qa[kk][1], 0u, b10, b11);
      }
      // scores of head gid for tokens 2t, 2t+1, 8+2t, 9+2t (log2 units); tokens past t_end are -inf
      float x[4] = {sacc[0][0] * scale_log2, sacc[0][1] * scale_log2, sacc[1][0] * scale_log2,
                    sacc[1][1] * scale_log2};
      const int tk[4] = {2 * tid, 2 * tid + 1, 8 + 2 * tid, 9 + 2 * tid};
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (tk[k] >= valid) x[k] = -INFINITY;
        mx = fmaxf(mx, x[k]);
      }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));  // max over the warp's 16 tokens
      if (mx - m_ref > kDecodeTau) {                          // conditional rescale (first tile: always)
        const float alpha = ex2(m_ref - mx);
        l *= alpha;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          o[n][0] *= alpha;
          o[n][1] *= alpha;
        }
        m_ref = mx;
      }
      float pv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        pv[k] = (x[k] == -INFINITY) ? 0.f : ex2(x[k] - m_ref);
        l += pv[k];
      }
      const uint32_t pa0 = pack_bf16x2(pv[0], pv[1]);  // P[gid][tokens 2t, 2t+1]
      const uint32_t pa2 = pack_bf16x2(pv[2], pv[3]);  // P[gid][tokens 8+2t, 9+2t]
      // V rows past the end of the sequence may hold anything (0 * NaN would poison O): zero them
      if (valid < 16) {
        const int first = valid < 0 ? 0 : valid;
        // whole rows are zeroed, so the swizzle (a permutation inside a row) does not matter
        constexpr int UPR = C::ROWB / 16;  // 16-byte units per stored row of a chunk
        for (int idx = lane; idx < (16 - first) * (D / 8); idx += 32) {
          const int r = first + idx / (D / 8), unit = idx % (D / 8);
          const uint32_t a = vt + (unit / UPR) * C::CHUNK_BYTES + (16 * warp + r) * C::ROWB + ((unit % UPR) << 4);
          asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
        }
        __syncwarp();
      }
      // ---- O += P V (16-column blocks of d: one transposed ldmatrix, two MMAs)
#pragma unroll
      for (int db = 0; db < D / 16; ++db) {
        uint32_t v00, v01, v10, v11;
        ldsm_x4_t(dec_sw128<D>(vt, 16 * warp + 8 * (mi & 1) + rr, 16 * db + 8 * (mi >> 1)), v00, v01, v10, v11);
        mma_bf16_16816(o[2 * db], pa0, 0u, pa2, 0u, v00, v01);
        mma_bf16_16816(o[2 * db + 1], pa0, 0u, pa2, 0u, v10, v11);
      }
      if (valid < 16) fence_proxy_async_smem();  // the zeroing writes precede the next TMA into the stage
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---- merge the consumer warps (the ring is idle now: every tile has been consumed)
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  float* sm_m = reinterpret_cast<float*>(smem);   // [NW][G]
  float* sm_l = sm_m + C::NW * G;                 // [NW][G]
  float* sm_acc = sm_l + C::NW * G;               // [NW][G][D]
  asm volatile("bar.sync 1, %0;" ::"n"(C::NW * 32) : "memory");  // all consumers are done with the ring
  if (gid < G) {
    if (tid == 0) {
      sm_m[warp * G + gid] = ok ? m_ref : -INFINITY;
      sm_l[warp * G + gid] = l;
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      sm_acc[(warp * G + gid) * D + 8 * n + 2 * tid] = o[n][0];
      sm_acc[(warp * G + gid) * D + 8 * n + 2 * tid + 1] = o[n][1];
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(C::NW * 32) : "memory");
  for (int idx = threadIdx.x; idx < G * D; idx += C::NW * 32) {
    const int hh = idx / D, e = idx % D;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < C::NW; ++w) m = fmaxf(m, sm_m[w * G + hh]);
    float lt = 0.f, ot = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int w = 0; w < C::NW; ++w) {
        const float f = ex2(sm_m[w * G + hh] - m);
        lt = fmaf(f, sm_l[w * G + hh], lt);
        ot = fmaf(f, sm_acc[(w * G + hh) * D + e], ot);
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
  static constexpr int EPT = D / NT;             // elements per thread (1, 2 or 4)
};

template <int EPT>
struct VecF;
template <>
struct VecF<1> {
  static __device__ __forceinline__ void fma(float w, const float* src, float* acc) { acc[0] = fmaf(w, *src, acc[0]); }
};
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
  if constexpr (EPT == 1) {
    const float a0 = (acc[0][0] + acc[1][0]) + (acc[2][0] + acc[3][0]);
    orow[0] = __float2bfloat16_rn(a0 * inv);
  } else {
#pragma unroll
    for (int e = 0; e < EPT; e += 2) {
      const float a0 = (acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e]);
      const float a1 = (acc[0][e + 1] + acc[1][e + 1]) + (acc[2][e + 1] + acc[3][e + 1]);
      *reinterpret_cast<uint32_t*>(orow + e) = pack_bf16x2(a0 * inv, a1 * inv);
    }
  }
  if (t == 0) lse[row] = (z > 0.f) ? mx + logf(z) : -INFINITY;
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
int decode_default_chunk(int B, int Hkv, int Nkv_cap) {
  // aim for ~8 live CTAs per SM if every sequence were full, in multiples of 64 tokens, at most 2048
  const long long total = (long long)B * Hkv * Nkv_cap;
  int sms = sm_count();
  if (sms <= 0) sms = 148;  // no device visible: size for a B200
  long long c = total / (sms * 8LL);
  c = (c + 63) / 64 * 64;
  if (c < 64) c = 64;
  if (c > 2048) c = 2048;
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

template <int D, int G>
static attn_status_t launch_split_tc(const void* q, const void* kc, const void* vc, const int32_t* lens, int cap,
                                     int B, int Hkv, int chunk, int n_splits, float scale, float* po, float* pl,
                                     cudaStream_t stream) {
  using C = DecTcCfg<D>;
  CUtensorMap tmK, tmV;
  const unsigned swz = C::SWIZZLE ? 128u : 0u;
  if (!encode_tile_map(&tmK, kc, D, Hkv, cap, B, C::CE, C::TT, swz) ||
      !encode_tile_map(&tmV, vc, D, Hkv, cap, B, C::CE, C::TT, swz))
    return ATTN_ERR_CUDA;
  if (ensure_dyn_smem(reinterpret_cast<const void*>(decode_split_tc_kernel<D, G>), C::SMEM_BYTES) != cudaSuccess)
    return ATTN_ERR_CUDA;
  dim3 grid(n_splits, Hkv, B);
  decode_split_tc_kernel<D, G><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(
      tmK, tmV, reinterpret_cast<const __nv_bfloat16*>(q), lens, cap, Hkv, chunk, n_splits,
      scale * 1.4426950408889634f, po, pl, kWaitLimitNs);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

// d = 32, 64 and 128 use the tensor-core split kernel; d = 256 (whose O fragments would not fit the
// register budget) uses the CUDA-core one.
template <int D>
static attn_status_t split_by_group(int G, const void* q, const void* kc, const void* vc, const int32_t* lens,
                                    int cap, int B, int Hkv, int chunk, int n_splits, float scale, float* po,
                                    float* pl, cudaStream_t st) {
  if constexpr (D <= 128) {
    switch (G) {
      case 1: return launch_split_tc<D, 1>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
      case 2: return launch_split_tc<D, 2>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
      case 4: return launch_split_tc<D, 4>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
      case 8: return launch_split_tc<D, 8>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
      default: return ATTN_ERR_UNSUPPORTED;
    }
  } else {
    switch (G) {
      case 1: return launch_split<D, 1>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
      case 2: return launch_split<D, 2>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
      case 4: return launch_split<D, 4>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
      case 8: return launch_split<D, 8>(q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
      default: return ATTN_ERR_UNSUPPORTED;
    }
  }
}

attn_status_t decode_split_dispatch(const void* q, const void* kc, const void* vc, const int32_t* lens, int cap,
                                    int B, int Hq, int Hkv, int d, float scale, int chunk, int n_splits,
                                    float* po, float* pl, cudaStream_t st) {
  const int G = Hq / Hkv;
  switch (d) {
    case 32: return split_by_group<32>(G, q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    case 64: return split_by_group<64>(G, q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    case 128: return split_by_group<128>(G, q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    case 256: return split_by_group<256>(G, q, kc, vc, lens, cap, B, Hkv, chunk, n_splits, scale, po, pl, st);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

template <int D>
static attn_status_t launch_combine(const float* po, const float* pl, int rows, int n_splits, void* o, float* lse,
                                    cudaStream_t st) {
  const size_t sm = size_t(n_splits) * (sizeof(float) + sizeof(int));  // weights + live split list
  if (sm > 48 * 1024 &&
      ensure_dyn_smem(reinterpret_cast<const void*>(decode_combine_kernel<D>), int(sm)) != cudaSuccess)
    return ATTN_ERR_CUDA;
  decode_combine_kernel<D><<<dim3(rows), CombCfg<D>::NT, sm, st>>>(po, pl, rows, n_splits,
                                                                   reinterpret_cast<__nv_bfloat16*>(o), lse);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

attn_status_t decode_combine_dispatch(const float* po, const float* pl, int rows, int n_splits, int d, void* o,
                                      float* lse, cudaStream_t st) {
  if (!combine_fits(n_splits)) return ATTN_ERR_UNSUPPORTED;
  switch (d) {
    case 32: return launch_combine<32>(po, pl, rows, n_splits, o, lse, st);
    case 64: return launch_combine<64>(po, pl, rows, n_splits, o, lse, st);
    case 128: return launch_combine<128>(po, pl, rows, n_splits, o, lse, st);
    case 256: return launch_combine<256>(po, pl, rows, n_splits, o, lse, st);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace attn
