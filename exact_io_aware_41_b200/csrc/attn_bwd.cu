// Backward pass for sm_100a (d = 128): dQ, dK, dV of O = softmax(scale * Q K^T) V, recomputing S tile
// by tile instead of storing it (the FlashAttention generation comparison record, "Workarounds":
// recompute S in backward). Per (batch, query head), with P = exp(scale * S - LSE):
//   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),  dQ = scale dS K,
//   dK = scale dS^T Q  (dK, dV of a kv head summed over the query heads of its group).
//
// One CTA per (key block of 128 keys, batch, kv head), heaviest key blocks first for causal masks.
// It loads its K and V tiles once and walks every query head of its group and every query tile
// that sees some of its keys. Per step (all products on tcgen05, accumulators in TMEM):
//   S^T = K Q^T      (M = keys, N = queries)           -> TMEM columns [0, 128)
//   dP^T = V dO^T                                      -> TMEM columns [128, 256)
//   elementwise warps (thread = key row): once S^T is in, P^T = exp2(S^T * scale * log2 e -
//   LSE * log2 e), masked, P^T (bf16) over S^T (each 32-query chunk's 16 packed columns at the start
//   of its own 32 score columns); once dP^T is in, dS^T = P^T * (dP^T - D), dS^T (bf16) over dP^T
//   and dS^T into shared memory
//   dV += P^T dO     (A = P^T in TMEM, B = dO read MN-major)   -> columns [256, 384), whole unit;
//                    issued as soon as P^T is in, so it runs while dS is formed
//   dQ  = dS K       (A = dS from shared memory, M-major; B = K read MN-major) -> columns [0, 128)
//   dK += dS^T Q     (A = dS^T in TMEM, B = Q read MN-major)   -> columns [384, 512), whole unit
//   a warpgroup of its own reads dQ out (thread = query row) while dK runs, stages it in the step's
//   Q / dO buffer, and the TMA unit adds it into an fp32 accumulator (cp.reduce.async.bulk.tensor
//   ... add); the boxes that go into the Q tile wait for dK, its last reader. Meanwhile the
//   elementwise warps go on to the next step.
// MMAs issued by one thread execute in issue order, so dQ may overwrite P^T's columns after the dV
// product that reads them, and the next step's dP^T may overwrite dS^T's after the dK product; the
// next step's S^T waits until dQ has been read out of its columns. Eight elementwise warps (two per
// TMEM lane quadrant, 64 of the 128 columns each) and four dQ warps (one per quadrant), next to the
// producer and MMA warps; Q, dO and their LSE' and D rows are double-buffered so the next step's
// loads overlap this one. The unit ends with dK (times scale) and dV converted to bf16 in the dS
// tile and written by TMA stores.
//
// A pre-pass writes D and LSE * log2 e per query row (padded to whole tiles; rows without keys or
// past Nq get LSE' = +inf, so their P is 0) and zeroes the dQ accumulator; a post-pass rounds
// scale * dQ to bf16.
#include <cuda_bf16.h>
#include <math.h>

#include <atomic>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn {

namespace bwd {
constexpr int D = 128;
constexpr int BM = 128;                       // query rows per step
constexpr int BN = 128;                       // keys per CTA
constexpr int CHUNK_BYTES = 128 * 128;        // 64-column chunk of a 128-row tile (128-byte rows)
constexpr int TILE_BYTES = 2 * CHUNK_BYTES;   // 128 x 128 bf16
constexpr int NSW = 8;                        // softmax / epilogue warps: two per TMEM lane quadrant
constexpr int CPW = 16 / NSW;                 // 32-column chunks of a 128-column tile per warp
constexpr int NDQ = 4;                        // dQ warps: one per TMEM lane quadrant
constexpr int THREADS = 128 + 32 * NSW + 32 * NDQ;
// register split (setmaxnreg) per warpgroup: control, elementwise (two warpgroups), dQ; the sum must
// fit in the launch allocation (THREADS x the kernel's register count, checked on the host)
constexpr int CTRL_REGS = 96;
constexpr int EW_REGS = 160;
constexpr int DQ_REGS = 96;
constexpr int TMEM_COLS = 512;
constexpr int S_COL = 0, DP_COL = 128, DV_COL = 256, DK_COL = 384;
// shared memory (tiles first, 1024-byte aligned): K, V, dS, then Q and dO of two stages; then the
// two stages' LSE' and D rows and the barriers. The whole budget (about 226 KB) leaves no room to
// pad for alignment, so the kernel checks that its dynamic shared memory starts on a 1024-byte
// boundary (it does when the kernel declares no static shared memory) and otherwise records an
// error and does nothing.
constexpr int OFF_K = 0, OFF_V = TILE_BYTES, OFF_DS = 2 * TILE_BYTES;
constexpr int OFF_Q0 = 3 * TILE_BYTES;        // stage s: Q at OFF_Q0 + 2s tiles, dO right after it
constexpr int OFF_LSE0 = 7 * TILE_BYTES;      // stage s: LSE' at OFF_LSE0 + s * 1024, D 512 bytes later
constexpr int OFF_BAR = OFF_LSE0 + 2 * 1024;
// kv_full, q_full[2], q_empty[2], s_full, p_full, dq_full, dq_free, dkv_full, dk_done[2], epi_full, epi_free,
// st_full, pt_full
constexpr int NBARS = 16;
constexpr int SMEM_BYTES = OFF_BAR + NBARS * 8 + 16;
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
}  // namespace bwd

struct BwdArgs {
  void* dk;
  void* dv;
  float* dq_acc;          // fp32 [B, Nq, Hq, d]
  const float* lse2;      // [B * Hq, Nq_pad]: LSE * log2 e (+inf: no keys or padding)
  const float* dd;        // [B * Hq, Nq_pad]: D
  int B, Hq, Hkv, Nq, Nkv, Nq_pad, group, n_kb;
  int causal;
  float scale_log2;
  float scale;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Adds a shared-memory box into global memory through the TMA unit (element-wise fp32 add at the
// destination), tracked by the issuing thread's bulk async-group.
__device__ __forceinline__ void tma_reduce_add_4d(const CUtensorMap* map, const void* smem_src, int c0, int c1, int c2,
                                                  int c3) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Stores a shared-memory box to global memory through the TMA unit (rows and columns outside the
// tensor are not written), tracked by the issuing thread's bulk async-group.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* smem_src, int c0, int c1, int c2,
                                             int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// First query tile whose rows see some key of block kb (causal: key j visible to row i iff
// j <= i + Nkv - Nq).
__device__ __forceinline__ int first_q_tile(const BwdArgs& a, int kb) {
  if (!a.causal) return 0;
  const int lo = kb * bwd::BN - (a.Nkv - a.Nq);  // smallest row that sees key kb * BN
  return lo <= 0 ? 0 : lo / bwd::BM;
}

__global__ void __launch_bounds__(bwd::THREADS, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const __grid_constant__ CUtensorMap tmDQ, const __grid_constant__ CUtensorMap tmDK,
                    const __grid_constant__ CUtensorMap tmDV, const BwdArgs args) {
  using namespace bwd;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(&g_error_word, kErrSmemAlignBit);
    return;  // every thread of the CTA takes this branch: nothing was started
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;   // [2]
  uint64_t* q_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* dq_full = bars + 7;
  uint64_t* dq_free = bars + 8;
  uint64_t* dkv_full = bars + 9;
  uint64_t* dk_done = bars + 10;  // [2] step t's dK product (the last reader of its Q tile) is done: slot
                                  // t & 1, one phase per two steps
  uint64_t* epi_full = bars + 12; // one phase per dK / dV tile: staged in shared memory by every warp
  uint64_t* epi_free = bars + 13; // one phase per dK / dV tile: the TMA unit has read it
  uint64_t* st_full = bars + 14;  // one phase per step: S^T is in (s_full: dP^T too)
  uint64_t* pt_full = bars + 15;  // one phase per step: P^T is in (p_full: dS^T too)
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t T = args.timeout_ns;
  // unit: key block kb (heaviest first), batch b, kv head g
  const int per_kb = args.B * args.Hkv;
  const int kb = blockIdx.x / per_kb;
  const int b = (blockIdx.x % per_kb) / args.Hkv;
  const int g = blockIdx.x % args.Hkv;
  const int n_qt = (args.Nq + BM - 1) / BM;
  const int qt0 = first_q_tile(args, kb);
  const int steps_per_head = qt0 < n_qt ? n_qt - qt0 : 0;
  const int n_steps = steps_per_head * args.group;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], NDQ);  // the dQ warps release a stage (its space stages dQ last)
    }
    mbar_init(s_full, 1);
    mbar_init(st_full, 1);
    mbar_init(pt_full, NSW);  // one arrival per elementwise warp
    mbar_init(p_full, NSW);   // one arrival per softmax warp
    mbar_init(dq_full, 1);
    mbar_init(dq_free, NDQ);  // one arrival per dQ warp
    mbar_init(dkv_full, 1);
    mbar_init(&dk_done[0], 1);
    mbar_init(&dk_done[1], 1);
    mbar_init(epi_full, NSW);  // one arrival per elementwise warp
    mbar_init(epi_free, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  auto step_coords = [&](int t, int& h, int& qt) {
    h = g * args.group + t / steps_per_head;
    qt = qt0 + t % steps_per_head;
  };

  if (warp == 0) {
    // ================================ TMA producer ================================
    regs_dec<CTRL_REGS>();
    if (lane == 0 && n_steps > 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      prefetch_tensormap(&tmDO);
      mbar_arrive_expect_tx(kv_full, 2 * TILE_BYTES);
      for (int c = 0; c < 2; ++c) {
        tma_load_4d(smem + OFF_K + c * CHUNK_BYTES, &tmK, kv_full, c * 64, g, kb * BN, b);
        tma_load_4d(smem + OFF_V + c * CHUNK_BYTES, &tmV, kv_full, c * 64, g, kb * BN, b);
      }
      int t = 0;
      for (; t < n_steps; ++t) {
        const int st = t & 1;
        // the stage's previous contents (step t - 2) are no longer read by any MMA
        if (t >= 2 && !mbar_wait(&q_empty[st], uint32_t(((t - 2) >> 1) & 1), abort_flag, T)) break;
        int h, qt;
        step_coords(t, h, qt);
        uint8_t* sq = smem + OFF_Q0 + 2 * st * TILE_BYTES;
        mbar_arrive_expect_tx(&q_full[st], 2 * TILE_BYTES + 2 * BM * 4);
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(sq + c * CHUNK_BYTES, &tmQ, &q_full[st], c * 64, h, qt * BM, b);
          tma_load_4d(sq + TILE_BYTES + c * CHUNK_BYTES, &tmDO, &q_full[st], c * 64, h, qt * BM, b);
        }
        const size_t row = size_t(b * args.Hq + h) * args.Nq_pad + size_t(qt) * BM;
        bulk_load(smem + OFF_LSE0 + st * 1024, args.lse2 + row, BM * 4, &q_full[st]);
        bulk_load(smem + OFF_LSE0 + st * 1024 + 512, args.dd + row, BM * 4, &q_full[st]);
      }
      // copies in flight land before the CTA exits (bounded)
      mbar_wait(kv_full, 0, nullptr, 100000000ull);
      for (int u = t - 2; u < t; ++u)
        if (u >= 0) mbar_wait(&q_full[u & 1], uint32_t((u >> 1) & 1), nullptr, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================ MMA issuer ================================
    regs_dec<CTRL_REGS>();
    if (lane == 0 && n_steps > 0) {
      // K-major reads of K, V, Q, dO (rows of d) and MN-major reads of Q, dO, K and the dS tile
      const uint64_t dK_k = smem_desc(smem_u32(smem + OFF_K), 16, 1024, kLayoutSW128);
      const uint64_t dV_k = smem_desc(smem_u32(smem + OFF_V), 16, 1024, kLayoutSW128);
      const uint64_t dK_mn = smem_desc(smem_u32(smem + OFF_K), CHUNK_BYTES, 1024, kLayoutSW128);
      const uint64_t dDS_mn = smem_desc(smem_u32(smem + OFF_DS), CHUNK_BYTES, 1024, kLayoutSW128);
      constexpr uint32_t idesc_kk = idesc_bf16_f32(128, 128, 0, 0);    // A, B K-major
      constexpr uint32_t idesc_tmn = idesc_bf16_f32(128, 128, 0, 1);   // A from TMEM, B MN-major
      constexpr uint32_t idesc_mnmn = idesc_bf16_f32(128, 128, 1, 1);  // A, B MN-major
      bool ok = mbar_wait(kv_full, 0, abort_flag, T);
      for (int t = 0; t < n_steps && ok; ++t) {
        const int st = t & 1;
        const uint32_t sq = smem_u32(smem + OFF_Q0 + 2 * st * TILE_BYTES);
        const uint64_t dQ_k = smem_desc(sq, 16, 1024, kLayoutSW128);
        const uint64_t dDO_k = smem_desc(sq + TILE_BYTES, 16, 1024, kLayoutSW128);
        const uint64_t dQ_mn = smem_desc(sq, CHUNK_BYTES, 1024, kLayoutSW128);
        const uint64_t dDO_mn = smem_desc(sq + TILE_BYTES, CHUNK_BYTES, 1024, kLayoutSW128);
        ok = mbar_wait(&q_full[st], uint32_t((t >> 1) & 1), abort_flag, T);
        if (!ok) break;
        tc_fence_after();
        // S^T = K Q^T into [0, 128), once the previous step's dQ (there) has been read out
        if (t > 0) {
          ok = mbar_wait(dq_free, uint32_t((t - 1) & 1), abort_flag, T);
          if (!ok) break;
          tc_fence_after();
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * CHUNK_BYTES + (kk % 4) * 32) >> 4;
          umma_ss(tmem + S_COL, dK_k + off, dQ_k + off, idesc_kk, kk > 0 ? 1u : 0u);
        }
        umma_commit(st_full);  // the elementwise warps start on P while dP^T runs
        // dP^T = V dO^T into [128, 256): dS^T of the previous step there was read by its dK product,
        // issued earlier by this thread
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * CHUNK_BYTES + (kk % 4) * 32) >> 4;
          umma_ss(tmem + DP_COL, dV_k + off, dDO_k + off, idesc_kk, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
        // over the step's 128 queries (k-steps of 16): dV += P^T dO as soon as P^T is in (it runs
        // while the elementwise warps form dS), then dQ = dS K into [0, 128) (after the dV product
        // has read P^T there), whose read-out overlaps dK += dS^T Q.
        // A = P^T / dS^T: queries 16kk .. 16kk+15 are columns 8 (kk % 2) .. of chunk kk / 2, which
        // starts at column 32 (kk / 2)
        ok = mbar_wait(pt_full, uint32_t(t & 1), abort_flag, T);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          umma_ts(tmem + DV_COL, tmem + S_COL + 32 * (kk / 2) + 8 * (kk % 2),
                  dDO_mn + uint64_t((kk * 16 * 128) >> 4), idesc_tmn, (t > 0 || kk > 0) ? 1u : 0u);
        ok = mbar_wait(p_full, uint32_t(t & 1), abort_flag, T);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ss(tmem + S_COL, dDS_mn + uint64_t((kk * 16 * 128) >> 4), dK_mn + uint64_t((kk * 16 * 128) >> 4),
                  idesc_mnmn, kk > 0 ? 1u : 0u);
        umma_commit(dq_full);
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          umma_ts(tmem + DK_COL, tmem + DP_COL + 32 * (kk / 2) + 8 * (kk % 2),
                  dQ_mn + uint64_t((kk * 16 * 128) >> 4), idesc_tmn, (t > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&dk_done[t & 1]);
        if (t == n_steps - 1) umma_commit(dkv_full);
      }
      if (!ok) {
        // a wait gave up: let the MMAs already issued finish before tensor memory is released
        // (dkv_full has not been committed on this path, so its first phase is the drain)
        umma_commit(dkv_full);
        mbar_wait(dkv_full, 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    regs_dec<CTRL_REGS>();
  } else if (warp >= 4 + NSW) {
    // ================================ dQ warps ================================
    // Per step, thread = query row q0 + row: once the dQ product is done, read it from TMEM (columns
    // 64..127 first, staged at once into the step's dO tile, read last by dV, done; then 0..63, after
    // which the columns are released) and stage it as four 32 x 32 fp32 boxes (128-byte rows,
    // swizzled like the tensor map): box c of this warp at c * 16 KB + wq * 4 KB, so boxes 0 and 1
    // land in the Q tile, which they may overwrite once dK (its last reader) is done. The TMA unit
    // adds the boxes into the fp32 accumulator; once it has read them the buffer goes back to the
    // producer.
    regs_dec<DQ_REGS>();
    const int wq = warp & 3;
    const uint32_t lane_addr = tmem + (uint32_t(wq * 32) << 16);
    auto wait_warp = [&](uint64_t* bar, uint32_t ph) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, ph, abort_flag, T));
    };
    auto stage_box = [&](uint8_t* box, const uint32_t* o) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t a = smem_u32(box) + lane * 128 + ((u ^ (lane & 7)) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(o[4 * u]), "r"(o[4 * u + 1]),
                     "r"(o[4 * u + 2]), "r"(o[4 * u + 3])
                     : "memory");
      }
    };
    for (int t = 0; t < n_steps; ++t) {
      int h, qt;
      step_coords(t, h, qt);
      const int row0 = qt * BM + wq * 32;  // first query row of this warp's boxes
      uint8_t* buf = smem + OFF_Q0 + 2 * (t & 1) * TILE_BYTES + wq * 4096;
      if (!wait_warp(dq_full, uint32_t(t & 1))) break;
      tc_fence_after();
      {
        uint32_t o[2][32];
        tmem_ld32(lane_addr + S_COL + 64, o[0]);
        tmem_ld32(lane_addr + S_COL + 96, o[1]);
        tmem_ld_wait();
        tmem_reg_fence32(o[0]);
        tmem_reg_fence32(o[1]);
        stage_box(buf + 2 * 16384, o[0]);
        stage_box(buf + 3 * 16384, o[1]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && row0 < args.Nq) {  // rows past Nq are clipped by the TMA unit
        tma_reduce_add_4d(&tmDQ, buf + 2 * 16384, 64, h, row0, b);
        tma_reduce_add_4d(&tmDQ, buf + 3 * 16384, 96, h, row0, b);
      }
      uint32_t o[2][32];
      tmem_ld32(lane_addr + S_COL, o[0]);
      tmem_ld32(lane_addr + S_COL + 32, o[1]);
      tmem_ld_wait();
      tmem_reg_fence32(o[0]);
      tmem_reg_fence32(o[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free);
      // the Q tile may take the boxes once dK (its last reader) is done. Step t's dK completes slot
      // t & 1; the slot's next phase needs step t + 2's dK, which runs only after this warp has
      // released step t + 1's columns, so this wait cannot miss its phase
      if (!wait_warp(&dk_done[t & 1], uint32_t((t >> 1) & 1))) break;
      stage_box(buf, o[0]);
      stage_box(buf + 16384, o[1]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (row0 < args.Nq) {
          tma_reduce_add_4d(&tmDQ, buf, 0, h, row0, b);
          tma_reduce_add_4d(&tmDQ, buf + 16384, 32, h, row0, b);
        }
        bulk_commit_group();
        bulk_wait_group_read0();  // the TMA unit has read the boxes: the buffer may be refilled
        mbar_arrive(&q_empty[t & 1]);
      }
      __syncwarp();
    }
    // The additions still in flight complete with the kernel; the CTA may exit once the TMA unit has
    // read their shared-memory sources (done after every step; here for a step left by an error).
    if (lane == 0) {
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  } else {
    // ========================= softmax / dK dV epilogue warps =========================
    regs_inc<EW_REGS>();
    const int wq = warp & 3;
    const int cw = (warp - 4) >> 2;   // which CPW x 32 of the 128 columns this warp covers
    const int row = wq * 32 + lane;   // TMEM lane: key row (softmax, dK dV) or query row (dQ)
    const uint32_t lane_addr = tmem + (uint32_t(wq * 32) << 16);
    const float c = args.scale_log2;
    const int key = kb * BN + row;
    const bool key_ok = key < args.Nkv;
    const int diag = args.Nkv - args.Nq;
    auto wait_warp = [&](uint64_t* bar, uint32_t ph) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, ph, abort_flag, T));
    };
    bool ok = true;
    for (int t = 0; t < n_steps && ok; ++t) {
      int h, qt;
      step_coords(t, h, qt);
      const float* s_lse = reinterpret_cast<const float*>(smem + OFF_LSE0 + (t & 1) * 1024);
      const float* s_dd = s_lse + 128;
      const int q0 = qt * BM;
      // P first, from S^T alone (its product is done before dP^T's), kept in fp32 for dS
      if (!wait_warp(st_full, uint32_t(t & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float pf[CPW][32];
#pragma unroll
      for (int cx = 0; cx < CPW; ++cx) {  // 32 query columns at a time, this warp's CPW x 32
        const int cc = CPW * cw + cx;
        uint32_t sv[32];
        tmem_ld32(lane_addr + S_COL + cc * 32, sv);
        tmem_ld_wait();
        tmem_reg_fence32(sv);
        // warp-uniform: does some (key, query) of this 32 x 32 block fall outside the mask? (rows
        // past Nq need no test: their LSE' is +inf, so P = 0)
        const int qf = q0 + cc * 32;
        const bool need_mask = (kb * BN + BN > args.Nkv) || (args.causal && kb * BN + BN - 1 > qf + diag);
        uint32_t pk[16];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 l4 = *reinterpret_cast<const float4*>(s_lse + cc * 32 + 4 * i4);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
          // pairs of query columns on the packed FMA pipe (the same roundings as the scalar forms)
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int u = 2 * h2, qi = cc * 32 + 4 * i4 + u;
            const float2 x = ffma2(make_float2(__uint_as_float(sv[4 * i4 + u]), __uint_as_float(sv[4 * i4 + u + 1])),
                                   make_float2(c, c), make_float2(-lv[u], -lv[u + 1]));
            float2 p = make_float2(ex2(x.x), ex2(x.y));
            if (need_mask) {
              if (!(key_ok && (!args.causal || key <= q0 + qi + diag))) p.x = 0.f;
              if (!(key_ok && (!args.causal || key <= q0 + qi + 1 + diag))) p.y = 0.f;
            }
            pf[cx][4 * i4 + u] = p.x;
            pf[cx][4 * i4 + u + 1] = p.y;
            pk[2 * i4 + h2] = pack_bf16x2(p.x, p.y);
          }
        }
        // P^T over S^T, bf16 pairs: the chunk's 16 columns go to the first 16 of its own 32 score
        // columns (just read), so no warp writes where the other still reads
        tmem_st16(lane_addr + S_COL + cc * 32, pk);
      }
      // P^T is in tensor memory: the dV product may start
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pt_full);
      // then dS = P (dP - D), once dP^T is in
      if (!wait_warp(s_full, uint32_t(t & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cx = 0; cx < CPW; ++cx) {
        const int cc = CPW * cw + cx;
        uint32_t dpv[32];
        tmem_ld32(lane_addr + DP_COL + cc * 32, dpv);
        tmem_ld_wait();
        tmem_reg_fence32(dpv);
        uint32_t dk2[16];
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 d4 = *reinterpret_cast<const float4*>(s_dd + cc * 32 + 4 * i4);
          const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int u = 2 * h2;
            const float2 ds = fmul2(make_float2(pf[cx][4 * i4 + u], pf[cx][4 * i4 + u + 1]),
                                    fadd2(make_float2(__uint_as_float(dpv[4 * i4 + u]), __uint_as_float(dpv[4 * i4 + u + 1])),
                                          make_float2(-dv4[u], -dv4[u + 1])));
            dk2[2 * i4 + h2] = pack_bf16x2(ds.x, ds.y);
          }
        }
        // dS^T over dP^T, as P^T over S^T
        tmem_st16(lane_addr + DP_COL + cc * 32, dk2);
        // dS^T row into the shared tile [key][query] (128-byte swizzled, 64-query chunks): the A
        // operand of dQ = dS K, read M-major
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int qcol = cc * 32 + u * 8;
          const int chunk = qcol >> 6, unit = (qcol & 63) >> 3;
          const uint32_t addr =
              smem_u32(smem + OFF_DS) + chunk * CHUNK_BYTES + row * 128 + ((unit ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dk2[4 * u]), "r"(dk2[4 * u + 1]),
                       "r"(dk2[4 * u + 2]), "r"(dk2[4 * u + 3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();  // the dS tile is read by the MMA (async proxy)
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // dK (times scale) and dV of this key block, bf16, this warp's 64 of the d columns
    if (key_ok && n_steps == 0) {
      for (int which = 0; which < 2; ++which) {
        uint4* dz = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(which ? args.dv : args.dk) +
                                             ((size_t(b) * args.Nkv + key) * args.Hkv + g) * D + 32 * CPW * cw);
        for (int v4 = 0; v4 < 4 * CPW; ++v4) dz[v4] = make_uint4(0, 0, 0, 0);
      }
    }
    if (n_steps > 0 && ok && wait_warp(dkv_full, 0)) {
      tc_fence_after();
      // Staged in the dS tile (free: every MMA is done), 128-byte swizzled like the tensor maps
      // (this warp's 64 columns are box cw), and written by TMA stores, dK first; the tile is
      // reused for dV once the TMA unit has read it.
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const float mul = which == 0 ? args.scale : 1.0f;
#pragma unroll 1
        for (int cx = 0; cx < CPW; ++cx) {
          uint32_t o[32];
          tmem_ld32(lane_addr + (which == 0 ? DK_COL : DV_COL) + (CPW * cw + cx) * 32, o);
          tmem_ld_wait();
          tmem_reg_fence32(o);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * mul, __uint_as_float(o[2 * i + 1]) * mul);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            const int unit = cx * 4 + v4;  // 16-byte unit of the row's 128 bytes
            const uint32_t addr = smem_u32(smem + OFF_DS) + cw * CHUNK_BYTES + row * 128 + ((unit ^ (row & 7)) << 4);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * v4]), "r"(pk[4 * v4 + 1]),
                         "r"(pk[4 * v4 + 2]), "r"(pk[4 * v4 + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(epi_full);
        if (warp == 4 && lane == 0) {
          // every warp's rows are in: store the tile, and free it once the TMA unit has read it
          if (mbar_wait(epi_full, uint32_t(which), abort_flag, T)) {
            const CUtensorMap* m = which == 0 ? &tmDK : &tmDV;
            tma_store_4d(m, smem + OFF_DS, 0, g, kb * BN, b);
            tma_store_4d(m, smem + OFF_DS + CHUNK_BYTES, 64, g, kb * BN, b);
            bulk_commit_group();
            bulk_wait_group_read0();
            mbar_arrive(epi_free);
          }
        }
        if (!wait_warp(epi_free, uint32_t(which))) break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// D_i = sum_e dO_ie O_ie and LSE'_i = LSE_i * log2 e (+inf when the row has no key) per (b, i, h) row,
// and the row of the fp32 dQ accumulator zeroed. Rows are taken in memory order, 16 lanes per row
// (16 bytes of O, of dO and 32 bytes of the accumulator each), so every access is coalesced; the
// 16-lane partial sums are combined by shuffles. The padding entries of the LSE' / D rows (whole
// tiles) get +inf and 0.
__global__ void __launch_bounds__(256)
    attn_bwd_pre_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                        const float* __restrict__ lse, float* __restrict__ lse2, float* __restrict__ dd,
                        float* __restrict__ acc, int B, int Nq, int Hq, int Nq_pad) {
  const long long rows = (long long)B * Nq * Hq;
  const int lane = threadIdx.x & 31, seg = lane & 15;
  const long long warp_g = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long n_warps = (gridDim.x * (long long)blockDim.x) >> 5;
  for (long long r = 2 * warp_g + (lane >> 4); r - (lane >> 4) < rows; r += 2 * n_warps) {
    const bool valid = r < rows;
    float dsum = 0.f;
    if (valid) {
      const uint4 a = reinterpret_cast<const uint4*>(o + r * bwd::D)[seg];
      const uint4 c = reinterpret_cast<const uint4*>(dout + r * bwd::D)[seg];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        dsum = fmaf(__uint_as_float(wa[k] << 16), __uint_as_float(wc[k] << 16), dsum);
        dsum = fmaf(__uint_as_float(wa[k] & 0xFFFF0000u), __uint_as_float(wc[k] & 0xFFFF0000u), dsum);
      }
      float4* z = reinterpret_cast<float4*>(acc + r * bwd::D) + 2 * seg;
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, off);
    if (valid && seg == 0) {
      const int h = int(r % Hq);
      const long long bi = r / Hq;
      const int i = int(bi % Nq), b = int(bi / Nq);
      const size_t bh = size_t(b) * Hq + h;
      const float L = lse[bh * Nq + i];
      lse2[bh * Nq_pad + i] = (L == -INFINITY) ? INFINITY : L * 1.4426950408889634f;
      dd[bh * Nq_pad + i] = dsum;
    }
  }
  // padding entries i in [Nq, Nq_pad) of every (b, h) row
  const int pad = Nq_pad - Nq;
  const long long n_pad = (long long)B * Hq * pad;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n_pad; e += gridDim.x * (long long)blockDim.x) {
    const long long bh = e / pad;
    const int i = Nq + int(e % pad);
    lse2[bh * Nq_pad + i] = INFINITY;
    dd[bh * Nq_pad + i] = 0.f;
  }
}

// dQ = scale * accumulator, bf16
__global__ void attn_bwd_post_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq, size_t n4,
                                     float scale) {
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(acc)[i];
    uint2 w;
    w.x = pack_bf16x2(v.x * scale, v.y * scale);
    w.y = pack_bf16x2(v.z * scale, v.w * scale);
    reinterpret_cast<uint2*>(dq)[i] = w;
  }
}

size_t bwd_workspace(int B, int Hq, int Nq, int d) {
  const size_t nq_pad = (size_t(Nq) + 127) / 128 * 128;
  const size_t acc = size_t(B) * Nq * Hq * d * sizeof(float);
  return ((acc + 255) / 256) * 256 + 2 * size_t(B) * Hq * nq_pad * sizeof(float);
}

attn_status_t bwd_dispatch(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nkv,
                           float scale, int causal, void* workspace, cudaStream_t stream) {
  using namespace bwd;
  const int Nq_pad = (Nq + 127) / 128 * 128;
  const size_t acc_bytes = size_t(B) * Nq * Hq * D * sizeof(float);
  float* acc = static_cast<float*>(workspace);
  float* lse2 = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((acc_bytes + 255) / 256) * 256);
  float* dd = lse2 + size_t(B) * Hq * Nq_pad;
  CUtensorMap tmQ, tmK, tmV, tmDO;
  if (!encode_tile_map(&tmQ, q, D, Hq, Nq, B, 64, BM, 128) || !encode_tile_map(&tmK, k, D, Hkv, Nkv, B, 64, BN, 128) ||
      !encode_tile_map(&tmV, v, D, Hkv, Nkv, B, 64, BN, 128) ||
      !encode_tile_map(&tmDO, dout, D, Hq, Nq, B, 64, BM, 128))
    return ATTN_ERR_CUDA;
  // dK and dV are written by TMA stores of 64-column boxes of a key block
  CUtensorMap tmDK, tmDV;
  if (!encode_tile_map(&tmDK, dk, D, Hkv, Nkv, B, 64, BN, 128) || !encode_tile_map(&tmDV, dv, D, Hkv, Nkv, B, 64, BN, 128))
    return ATTN_ERR_CUDA;
  CUtensorMap tmDQ;
  {
    const long long dims[4] = {D, Hq, Nq, B};
    const int box[4] = {32, 1, 32, 1};
    if (!encode_map(&tmDQ, acc, 4, dims, box, 128)) return ATTN_ERR_CUDA;
  }
  if (ensure_dyn_smem(reinterpret_cast<const void*>(attn_bwd_kernel), SMEM_BYTES) != cudaSuccess) return ATTN_ERR_CUDA;
  {
    // setmaxnreg.inc waits until the registers it asks for are free in the CTA's launch allocation,
    // so a split whose total exceeds that allocation would never proceed: refuse to launch it
    static std::atomic<int> regs_ok{0};  // 0 unknown, 1 fits, 2 does not (same binary on every device)
    int st = regs_ok.load(std::memory_order_relaxed);
    if (st == 0) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, attn_bwd_kernel) != cudaSuccess) return ATTN_ERR_CUDA;
      const long long need = 128LL * (CTRL_REGS + 2 * EW_REGS + DQ_REGS);
      st = (long long)fa.numRegs * THREADS >= need ? 1 : 2;
      regs_ok.store(st, std::memory_order_relaxed);
    }
    if (st != 1) return ATTN_ERR_UNSUPPORTED;
  }
  {
    // the row pass: rows are 16-lane groups, two per warp; about 16 warps per SM in flight
    const long long rows = (long long)B * Nq * Hq;
    const int n_sm = sm_count();
    if (n_sm <= 0) return ATTN_ERR_CUDA;
    const long long want = (rows + 15) / 16;  // blocks of 8 warps, 16 rows per block and iteration
    const long long cap = (long long)n_sm * 8;
    attn_bwd_pre_kernel<<<dim3(unsigned(want < cap ? want : cap)), 256, 0, stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(o), reinterpret_cast<const __nv_bfloat16*>(dout), lse, lse2, dd, acc, B,
        Nq, Hq, Nq_pad);
  }
  BwdArgs a;
  a.dk = dk;
  a.dv = dv;
  a.dq_acc = acc;
  a.lse2 = lse2;
  a.dd = dd;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.Nq = Nq;
  a.Nkv = Nkv;
  a.Nq_pad = Nq_pad;
  a.group = Hq / Hkv;
  a.n_kb = (Nkv + BN - 1) / BN;
  a.causal = causal;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.scale = scale;
  a.timeout_ns = kWaitLimitNs;
  const long long grid = (long long)a.n_kb * B * Hkv;
  if (grid > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  attn_bwd_kernel<<<dim3(unsigned(grid)), THREADS, SMEM_BYTES, stream>>>(tmQ, tmK, tmV, tmDO, tmDQ, tmDK, tmDV, a);
  const size_t n4 = size_t(B) * Nq * Hq * D / 4;
  attn_bwd_post_kernel<<<dim3(unsigned(n4 / 256 + 1 < 8192 ? n4 / 256 + 1 : 8192)), 256, 0, stream>>>(
      acc, reinterpret_cast<__nv_bfloat16*>(dq), n4, scale);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

}  // namespace attn
