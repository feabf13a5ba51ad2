// Prefill forward for sm_100a: O = softmax(scale * Q K^T) V and LSE, tile by tile.
//
// Work decomposition (one CTA per unit): a unit is (batch b, query head h, block of NQT query
// tiles of 128 rows). Units are numbered so the block scheduler hands out the heaviest causal units
// first (longest-processing-time order). Query-block parallelism follows the "FlashAttention
// evolution" article, section 3; LPT ordering the FlashAttention generation comparison record,
// "Workarounds" (FA-4).
//
// Roles inside a CTA (warp specialisation, evolution article section 4, rebuilt on sm_100a):
//   warp 0        TMA producer: Q tiles once, then K_j, V_j into a STAGES-deep shared-memory ring
//   warp 1        MMA issuer (one thread): S = Q K^T and O += P V with tcgen05.mma, accumulators
//                 in tensor memory (evolution article section 5)
//   warp 2        tensor-memory allocator
//   warpgroups 1+ softmax: each thread owns one query row = one TMEM lane ("sliced-Q" ownership,
//                 section 3, so no cross-thread reduction). Reads S from TMEM, applies the mask,
//                 runs the online-softmax update, writes P (bf16) back over S for the PV MMA, and
//                 rescales O in TMEM only when its running max grew by more than TAU (conditional
//                 rescaling, section 5). At the end it divides by the row sum once (delayed
//                 normalisation, section 3) and writes O and LSE.
// With two query tiles per CTA (d <= 128) the two softmax warpgroups alternate with the tensor
// core: while one tile's softmax runs, the other tile's MMAs run ("overlaps multiple query tiles",
// section 5). With d = 256 one query tile alternates between two S buffers instead.
//
// S and P never leave the SM: S is fp32 in TMEM, P is bf16 written in place over S and read by
// the MMA straight from TMEM.
#include <cuda_bf16.h>
#include <math.h>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn {

// Running-max slack before O is rescaled, in log2 units: P entries stay <= 2^TAU.
constexpr float kRescaleTau = 8.0f;

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;                        // query rows per tile (TMEM lanes)
  static constexpr int NQT = (D <= 128) ? 2 : 1;        // query tiles per CTA
  static constexpr int BN = (D <= 128) ? 128 : 64;      // keys per K/V tile
  static constexpr int CHUNK = (D >= 64) ? 64 : 32;     // elements per swizzled smem row
  static constexpr int NCHUNK = D / CHUNK;              // swizzle chunks along d
  static constexpr int ROWB = CHUNK * 2;                // bytes per swizzled row (128 or 64)
  static constexpr uint32_t LAYOUT = (D >= 64) ? kLayoutSW128 : kLayoutSW64;
  static constexpr int KPC = CHUNK / 16;                // 16-wide MMA k-steps per chunk
  static constexpr int Q_CHUNK_BYTES = BM * ROWB;
  static constexpr int KV_CHUNK_BYTES = BN * ROWB;
  static constexpr int Q_TILE_BYTES = BM * D * 2;
  static constexpr int KV_TILE_BYTES = BN * D * 2;
  static constexpr int STAGES = (D == 128 || D == 256) ? 4 : 8;
  static constexpr int NSMWG = (NQT == 2) ? 2 : 1;      // softmax warpgroups
  static constexpr int THREADS = 128 * (1 + NSMWG);
  // TMEM columns (fp32 each): two S slots, then one O accumulator per query tile.
  static constexpr int S_COL0 = 0;
  static constexpr int S_COL1 = BN;
  static constexpr int O_COL0 = 2 * BN;
  static constexpr int O_COL1 = 2 * BN + D;
  static constexpr int TMEM_COLS = 512;
  static_assert(2 * BN + NQT * D <= TMEM_COLS, "tensor memory budget");
  static constexpr int NBARS = 1 + 2 * STAGES + 2 + 2 + NQT + 1;
  static constexpr int SMEM_DATA = NQT * Q_TILE_BYTES + STAGES * KV_TILE_BYTES;
  // Pad small-d configurations so only one CTA (and one 512-column TMEM allocation) fits per SM.
  static constexpr int SMEM_MIN = 120 * 1024;
  static constexpr int SMEM_BYTES_RAW = 1024 + SMEM_DATA + NBARS * 8 + 16;
  static constexpr int SMEM_BYTES = SMEM_BYTES_RAW > SMEM_MIN ? SMEM_BYTES_RAW : SMEM_MIN;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdArgs args) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::NQT * C::Q_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::STAGES * C::KV_TILE_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = q_full + 1;
  uint64_t* kv_empty = kv_full + C::STAGES;
  uint64_t* s_full = kv_empty + C::STAGES;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + C::NQT;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t T = args.timeout_ns;

  // ---- unit of work ------------------------------------------------------------------------
  const int BH = args.B * args.Hq;
  const int u = blockIdx.x;
  const int qblk = args.n_qblk - 1 - u / BH;  // heaviest causal blocks first
  const int bh = u % BH;
  const int b = bh / args.Hq;
  const int h = bh % args.Hq;
  const int g = h / args.group;
  const int q0 = qblk * C::NQT * C::BM;
  const int diag = args.Nkv - args.Nq;  // key j visible to query i iff j <= i + diag
  int kv_end = args.Nkv;
  if (args.causal) {
    const int q_last = min(q0 + C::NQT * C::BM, args.Nq) - 1;
    kv_end = min(args.Nkv, q_last + diag + 1);
  }
  const int n_tiles = kv_end > 0 ? (kv_end + C::BN - 1) / C::BN : 0;

  // ---- set-up --------------------------------------------------------------------------------
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    for (int i = 0; i < C::NQT; ++i) mbar_init(&o_done[i], 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if (warp == 2) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ================================ TMA producer ================================
    if (lane == 0 && n_tiles > 0) {
      int fills[C::STAGES];
#pragma unroll
      for (int s = 0; s < C::STAGES; ++s) fills[s] = 0;
      bool ok = true;
      mbar_arrive_expect_tx(q_full, C::NQT * C::Q_TILE_BYTES);
#pragma unroll
      for (int qt = 0; qt < C::NQT; ++qt)
#pragma unroll
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_4d(sQ + qt * C::Q_TILE_BYTES + c * C::Q_CHUNK_BYTES, &tmQ, q_full, c * C::CHUNK, h,
                      q0 + qt * C::BM, b);
      int pos = 0;
      for (int j = 0; j < n_tiles && ok; ++j) {
#pragma unroll
        for (int kv = 0; kv < 2; ++kv, ++pos) {
          const int s = pos % C::STAGES;
          const uint32_t ph = (pos / C::STAGES) & 1;
          if (!mbar_wait(&kv_empty[s], ph ^ 1, abort_flag, T)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[s], C::KV_TILE_BYTES);
          const CUtensorMap* m = kv ? &tmV : &tmK;
#pragma unroll
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_4d(sKV + s * C::KV_TILE_BYTES + c * C::KV_CHUNK_BYTES, m, &kv_full[s], c * C::CHUNK, g,
                        j * C::BN, b);
          ++fills[s];
        }
      }
      if (!ok) {
        // Give the copies already in flight a bounded chance to land before the CTA exits.
        mbar_wait(q_full, 0, nullptr, 100000000ull);
        for (int s = 0; s < C::STAGES; ++s)
          if (fills[s] > 0) mbar_wait(&kv_full[s], (fills[s] - 1) & 1, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================ MMA issuer ================================
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t sQ_addr = smem_u32(sQ);
      const uint32_t sKV_addr = smem_u32(sKV);
      // S[slot] = Q_qt K^T : A = Q tile (K-major), B = K tile (K-major), k-steps of 16 along d.
      auto issue_qk = [&](int qt, int s_col, int stage) {
        const uint32_t a0 = sQ_addr + qt * C::Q_TILE_BYTES;
        const uint32_t b0 = sKV_addr + stage * C::KV_TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = (kk / C::KPC) * C::Q_CHUNK_BYTES + (kk % C::KPC) * 32;
          const uint32_t bo = (kk / C::KPC) * C::KV_CHUNK_BYTES + (kk % C::KPC) * 32;
          umma_ss(tmem + s_col, smem_desc(a0 + ao, 16, 8 * C::ROWB, C::LAYOUT),
                  smem_desc(b0 + bo, 16, 8 * C::ROWB, C::LAYOUT), idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_qt += P V : A = P (bf16, in TMEM over S), B = V tile read MN-major (N = d), k-steps of 16 keys.
      auto issue_pv = [&](int o_col, int p_col, int stage, bool accumulate) {
        const uint32_t b0 = sKV_addr + stage * C::KV_TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          umma_ts(tmem + o_col, tmem + p_col + kk * 8,
                  smem_desc(b0 + kk * 16 * C::ROWB, C::KV_CHUNK_BYTES, 8 * C::ROWB, C::LAYOUT), idesc_pv,
                  (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      auto kv_slot = [&](int pos) { return pos % C::STAGES; };
      auto kv_phase = [&](int pos) { return uint32_t((pos / C::STAGES) & 1); };
      bool ok = mbar_wait(q_full, 0, abort_flag, T);
      tc_fence_after();
      if (C::NQT == 2) {
        // Ring order: K_0, V_0, K_1, V_1, ...  (K_j at position 2j, V_j at 2j + 1)
        if (ok) ok = mbar_wait(&kv_full[kv_slot(0)], kv_phase(0), abort_flag, T);
        if (ok) {
          tc_fence_after();
          issue_qk(0, C::S_COL0, kv_slot(0));
          umma_commit(&s_full[0]);
          issue_qk(1, C::S_COL1, kv_slot(0));
          umma_commit(&s_full[1]);
          umma_commit(&kv_empty[kv_slot(0)]);
        }
        for (int j = 0; j < n_tiles && ok; ++j) {
          const int pv_pos = 2 * j + 1, pk_pos = 2 * j + 2;
          const bool nxt = j + 1 < n_tiles;
          ok = mbar_wait(&kv_full[kv_slot(pv_pos)], kv_phase(pv_pos), abort_flag, T);
          if (ok && nxt) ok = mbar_wait(&kv_full[kv_slot(pk_pos)], kv_phase(pk_pos), abort_flag, T);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int qt = 0; qt < 2; ++qt) {
            const int s_col = qt ? C::S_COL1 : C::S_COL0;
            ok = mbar_wait(&p_full[qt], j & 1, abort_flag, T);
            if (!ok) break;
            tc_fence_after();
            issue_pv(qt ? C::O_COL1 : C::O_COL0, s_col, kv_slot(pv_pos), j > 0);
            umma_commit(&o_done[qt]);
            if (nxt) {
              issue_qk(qt, s_col, kv_slot(pk_pos));
              umma_commit(&s_full[qt]);
            }
          }
          if (!ok) break;
          umma_commit(&kv_empty[kv_slot(pv_pos)]);
          if (nxt) umma_commit(&kv_empty[kv_slot(pk_pos)]);
        }
      } else {
        // One query tile, S alternating between two slots: QK_0, QK_1, PV_0, QK_2, PV_1, QK_3, ...
        for (int j = 0; j < 2 && j < n_tiles && ok; ++j) {
          ok = mbar_wait(&kv_full[kv_slot(2 * j)], kv_phase(2 * j), abort_flag, T);
          if (!ok) break;
          tc_fence_after();
          issue_qk(0, j ? C::S_COL1 : C::S_COL0, kv_slot(2 * j));
          umma_commit(&s_full[j]);
          umma_commit(&kv_empty[kv_slot(2 * j)]);
        }
        for (int j = 0; j < n_tiles && ok; ++j) {
          const int slot = j & 1;
          const int s_col = slot ? C::S_COL1 : C::S_COL0;
          ok = mbar_wait(&kv_full[kv_slot(2 * j + 1)], kv_phase(2 * j + 1), abort_flag, T);
          if (ok) ok = mbar_wait(&p_full[slot], (j >> 1) & 1, abort_flag, T);
          if (!ok) break;
          tc_fence_after();
          issue_pv(C::O_COL0, s_col, kv_slot(2 * j + 1), j > 0);
          umma_commit(&o_done[0]);
          umma_commit(&kv_empty[kv_slot(2 * j + 1)]);
          if (j + 2 < n_tiles) {
            const int kp = 2 * (j + 2);
            ok = mbar_wait(&kv_full[kv_slot(kp)], kv_phase(kp), abort_flag, T);
            if (!ok) break;
            tc_fence_after();
            issue_qk(0, s_col, kv_slot(kp));
            umma_commit(&s_full[slot]);
            umma_commit(&kv_empty[kv_slot(kp)]);
          }
        }
      }
      if (!ok) {
        // Let the MMAs already issued finish before tensor memory is released.
        umma_commit(drain);
        mbar_wait(drain, 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================ softmax warpgroups ================================
    const int wg = (warp - 4) >> 2;
    const int wq = warp & 3;             // warp within its warpgroup: TMEM lanes 32*wq .. 32*wq+31
    const int row = wq * 32 + lane;      // query row within the tile = TMEM lane
    const int qt = (C::NQT == 2) ? wg : 0;
    const int q_first = q0 + qt * C::BM;
    const int q_row = q_first + row;
    const uint32_t lane_addr = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t o_col = qt ? C::O_COL1 : C::O_COL0;
    const float c = args.scale_log2;
    // last key visible to this row (any key index <= lim is visible); rows past Nq are padding
    const int lim = args.causal ? min(args.Nkv - 1, q_row + diag) : args.Nkv - 1;

    float m_ref = -INFINITY;  // reference max (raw-score units) of the exponentials in l and O
    float l = 0.f;            // running row sum of exp2(c * (s - m_ref))
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int slot = (C::NQT == 2) ? qt : (j & 1);
      const uint32_t ph = (C::NQT == 2) ? uint32_t(j & 1) : uint32_t((j >> 1) & 1);
      const uint32_t s_addr = lane_addr + (slot ? C::S_COL1 : C::S_COL0);
      if (!mbar_wait(&s_full[slot], ph, abort_flag, T)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t r[C::BN];
#pragma unroll
      for (int cc = 0; cc < C::BN / 32; ++cc) tmem_ld32(s_addr + cc * 32, r + cc * 32);
      tmem_ld_wait();
#pragma unroll
      for (int cc = 0; cc < C::BN / 32; ++cc) tmem_reg_fence32(r + cc * 32);

      const int kbase = j * C::BN;
      // warp-uniform: does any key of this tile fall outside some row's visible range?
      const bool need_mask = (kbase + C::BN > args.Nkv) || (args.causal && kbase + C::BN - 1 > q_first + diag);
      if (need_mask) {
#pragma unroll
        for (int i = 0; i < C::BN; ++i)
          if (kbase + i > lim) r[i] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < C::BN; ++i) mx = fmaxf(mx, __uint_as_float(r[i]));
      const float m_new = fmaxf(m_ref, mx);
      // true when the max moved by more than TAU (also on the first live tile: -inf -> finite)
      const bool need = (m_new - m_ref) * c > kRescaleTau;
      if (__any_sync(0xffffffffu, need)) {
        const float alpha = need ? ex2((m_ref - m_new) * c) : 1.0f;
        if (need) m_ref = m_new;
        l *= alpha;
        if (j > 0) {
          if (C::NQT == 1) {
            // PV_{j-1} must have landed in O before it is rescaled
            if (!mbar_wait(&o_done[0], (j - 1) & 1, abort_flag, T)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(lane_addr + o_col + cc * 32, o);
            tmem_ld_wait();
            tmem_reg_fence32(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(lane_addr + o_col + cc * 32, o);
          }
          tmem_st_wait();
        }
      }
      const float mc = (m_ref == -INFINITY) ? 0.f : m_ref * c;
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t p[C::BN / 2];
#pragma unroll
      for (int i = 0; i < C::BN / 2; ++i) {
        const float p0 = ex2(fmaf(__uint_as_float(r[2 * i]), c, -mc));
        const float p1 = ex2(fmaf(__uint_as_float(r[2 * i + 1]), c, -mc));
        rs0 += p0;
        rs1 += p1;
        p[i] = pack_bf16x2(p0, p1);
      }
      l += rs0 + rs1;
      // P overwrites the first BN/2 columns of this S slot (two bf16 per 32-bit column)
#pragma unroll
      for (int cc = 0; cc < C::BN / 64; ++cc) tmem_st32(s_addr + cc * 32, p + cc * 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[slot]);
    }

    // ---- epilogue: O = acc / l (once), LSE = scale * m_ref + ln l -------------------------------
    const bool valid = q_row < args.Nq;
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(args.o) +
                          ((size_t(b) * args.Nq + (valid ? q_row : 0)) * args.Hq + h) * D;
    if (n_tiles > 0 && ok) {
      ok = mbar_wait(&o_done[qt], (n_tiles - 1) & 1, abort_flag, T);
      tc_fence_after();
    }
    if (ok) {
      const float inv = (l > 0.f) ? 1.0f / l : 0.f;
      if (n_tiles > 0) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(lane_addr + o_col + cc * 32, o);
          tmem_ld_wait();
          tmem_reg_fence32(o);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
      } else if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
        for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
      }
      if (valid)
        args.lse[(size_t(b) * args.Hq + h) * args.Nq + q_row] =
            (l > 0.f) ? fmaf(m_ref, args.scale, logf(l)) : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
template <int D>
static attn_status_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                                int Hkv, int Nq, int Nkv, float scale, int causal, cudaStream_t stream) {
  using C = FwdCfg<D>;
  CUtensorMap tmQ, tmK, tmV;
  const uint32_t swz = (D >= 64) ? 128u : 64u;
  if (!encode_tile_map(&tmQ, q, D, Hq, Nq, B, C::CHUNK, C::BM, swz) ||
      !encode_tile_map(&tmK, k, D, Hkv, Nkv, B, C::CHUNK, C::BN, swz) ||
      !encode_tile_map(&tmV, v, D, Hkv, Nkv, B, C::CHUNK, C::BN, swz))
    return ATTN_ERR_CUDA;

  static bool attr_set = false;  // per template instance; the attribute is per-function and sticky
  if (!attr_set) {
    if (cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
      return ATTN_ERR_CUDA;
    attr_set = true;
  }
  FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nkv = Nkv;
  a.group = Hq / Hkv;
  a.n_qblk = (Nq + C::NQT * C::BM - 1) / (C::NQT * C::BM);
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = kWaitLimitNs;
  const long long units = (long long)a.n_qblk * B * Hq;
  if (units > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  attn_fwd_kernel<D><<<dim3(unsigned(units)), dim3(C::THREADS), C::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, a);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

attn_status_t fwd_dispatch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                           int Hkv, int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream) {
  switch (d) {
    case 32: return launch_fwd<32>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, stream);
    case 64: return launch_fwd<64>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, stream);
    case 128: return launch_fwd<128>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, stream);
    case 256: return launch_fwd<256>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, stream);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

}  // namespace attn
