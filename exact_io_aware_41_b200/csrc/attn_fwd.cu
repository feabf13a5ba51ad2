// Prefill forward for sm_100a: O = softmax(scale * Q K^T) V and LSE, tile by tile.
//
// Work decomposition: a unit is (batch b, query head h, block of NQT query tiles of 128 rows; at
// d = 256 one tile in each CTA of a pair). The grid is persistent (one CTA per SM); each CTA claims
// units from a per-launch atomic counter (CTA pairs take fixed shares instead). Units are numbered
// by L2 head group and, inside a group, heaviest first (longest-processing-time order for causal
// masks). Query-block parallelism follows the "FlashAttention evolution" article,
// section 3; LPT ordering the FlashAttention generation comparison record, "Workarounds" (FA-4).
//
// Roles inside a CTA (warp specialisation, evolution article section 4, rebuilt on sm_100a):
//   warp 0        TMA producer: claims units, loads each unit's Q tiles once, then K_j, V_j into a
//                 STAGES-deep shared-memory ring
//   warp 1        MMA issuer (one thread): S = Q K^T and O += P V with tcgen05.mma, accumulators
//                 in tensor memory (evolution article section 5)
//   warp 2        tensor-memory allocator
//   warpgroups 1+ softmax: each thread owns one query row = one TMEM lane ("sliced-Q" ownership,
//                 section 3, so no cross-thread reduction). Reads S from TMEM, applies the mask,
//                 runs the online-softmax update, writes P (bf16) to TMEM for the PV MMA, and
//                 rescales O in TMEM only when its running max grew by more than TAU (conditional
//                 rescaling, section 5). At the end it divides by the row sum once (delayed
//                 normalisation, section 3) and writes O and LSE.
// With two query tiles per CTA (d <= 128) the two softmax warpgroups alternate with the tensor
// core: while one tile's softmax runs, the other tile's MMAs run ("overlaps multiple query tiles",
// section 5). With d = 256 the O accumulator takes half of tensor memory, so each CTA holds one
// query tile, which alternates between two S buffers instead; two CTAs form a pair (a cluster of
// two) that runs 2-SM MMAs (M = 256) over 256 query rows, each CTA loading half of every K/V tile
// (the evolution article's 2-CTA MMA, section 5).
//
// S and P never leave the SM: S is fp32 in TMEM, P is bf16 in TMEM, read by the MMA straight from
// there. At d = 128 and 256 P is written in place over S, so the next S = Q K^T into that slot
// waits for the PV that reads P. At d <= 64 the O accumulators are narrow enough to leave TMEM
// columns for P buffers of its own: the next S of a tile is computed as soon as the softmax has
// read the current one, overlapping that tile's own softmax.
#include <cuda_bf16.h>
#include <math.h>

#include <atomic>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn {

// K/V bytes of a whole launch below which all heads form one L2 group (see launch_fwd).
#ifndef ATTN_L2_ONE_GROUP_MB
#define ATTN_L2_ONE_GROUP_MB 96
#endif
constexpr double kL2OneGroupBytes = ATTN_L2_ONE_GROUP_MB * 1.0e6;

// Running-max slack before O is rescaled, in log2 units: P entries stay <= 2^TAU.
constexpr float kRescaleTau = 8.0f;

// Columns (per 128 keys) whose exponential is evaluated on the FMA pipe instead of the exp unit, in
// tiles without masked keys, per head dim. Every tile needs BM x BN exponentials whatever d is, so
// the exp unit bounds the softmax; moving part of them to the FMA pipe relieves it only when the
// FMA pipe has room and enough independent pairs are in flight. Measured on B200 it did not pay at
// any head dim, so the product builds use none; the variant is built and checked by the tests.
#ifndef ATTN_EMU_COLS_D32
#define ATTN_EMU_COLS_D32 0
#endif
#ifndef ATTN_EMU_COLS_D64
#define ATTN_EMU_COLS_D64 0
#endif
#ifndef ATTN_EMU_COLS_D128
#define ATTN_EMU_COLS_D128 0
#endif
#ifndef ATTN_EMU_COLS_D256
#define ATTN_EMU_COLS_D256 0
#endif

// F8: Q and K are e4m3 codes (rotated), V is given transposed (e4m3 [d, keys] per head), and the
// products run as kind::f8f6f4 MMAs with 32-element k-steps; P is packed four e4m3 per TMEM column.
// PAIR (used at d = 256): a cluster of two CTAs works on 256 query rows, 128 per CTA, with 2-SM MMAs
// (cta_group::2, M = 256). Each CTA holds half of every K tile (its 64 of the tile's 128 keys) and
// half of every V tile (its 128 of the d columns), so 128-key tiles fit a 5-stage ring and the QK
// products run at N = 128 (a 64-key N = 64 product costs ~52 cycles per k-step against 32 for its
// FLOPs; N = 128 runs at the full rate). The same configuration builds at d = 128 (one query tile per
// CTA, two S slots) but measured slower there than two query tiles per CTA: with half the FLOPs per
// key tile, the single softmax warpgroup per CTA sets the pace.
template <int D, bool F8 = false, bool PAIR = false>
struct FwdCfg {
  static_assert(!F8 || D == 128, "the 8-bit path is built for d = 128");
  static_assert(!PAIR || (D >= 128 && !F8), "CTA pairs are built for bf16 at d = 128 and 256");
  static_assert(PAIR || D <= 128, "d = 256 runs on CTA pairs");
  static constexpr int EB = F8 ? 1 : 2;                 // bytes per element of Q, K, V
  static constexpr int BM = 128;                        // query rows per tile (TMEM lanes)
  static constexpr int NQT = (D <= 128 && !PAIR) ? 2 : 1;  // query tiles per CTA
  static constexpr int BN = (D <= 128 || PAIR) ? 128 : 64;  // keys per K/V tile
  static constexpr int CTAS = PAIR ? 2 : 1;             // CTAs per unit
  static constexpr int UNIT_ROWS = NQT * BM * CTAS;     // query rows per unit
  // d <= 64: P lives in tensor-memory buffers of its own instead of over S, so a tile's next
  // S = Q K^T is computed while the softmax still works on the current one (the two O accumulators
  // leave room for the buffers). d = 128 has no room for them and writes P over S.
  static constexpr bool SEP_P = (NQT == 2) && (D < 128);
  static constexpr int CHUNK = (D * EB >= 128) ? 128 / EB : D;  // elements per swizzled smem row
  static constexpr int NCHUNK = D / CHUNK;              // swizzle chunks along d
  static constexpr int ROWB = CHUNK * EB;               // bytes per swizzled row (128 or 64)
  static constexpr uint32_t LAYOUT = (ROWB == 128) ? kLayoutSW128 : kLayoutSW64;
  static constexpr int KSTEP = 32 / EB;                 // elements per MMA k-step (32 bytes)
  static constexpr int KPC = CHUNK / KSTEP;             // MMA k-steps per chunk
  static constexpr int Q_CHUNK_BYTES = BM * ROWB;
  static constexpr int K_ROWS = BN / CTAS;              // keys of a K tile held by one CTA
  static constexpr int V_COLS = D / CTAS;               // d columns of a V tile held by one CTA
  static constexpr int K_CHUNK_BYTES = K_ROWS * ROWB;   // one swizzle chunk (CHUNK of d) of the K part
  static constexpr int V_CHUNK_BYTES = BN * ROWB;       // one swizzle chunk of the V part (all BN keys)
  static constexpr int Q_TILE_BYTES = BM * D * EB;
  static constexpr int KV_TILE_BYTES = BN * D * EB / CTAS;  // one ring stage: this CTA's K or V part
  static_assert(!F8 || BN * EB == 128, "a transposed V tile row (BN keys) is one 128-byte swizzled row");
  static constexpr int STAGES = (D == 256) ? 5 : (KV_TILE_BYTES >= 32768) ? 4 : 8;
  static constexpr int P_ARRIVALS = 4 * CTAS;           // p_full: one arrival per softmax warp of the unit
  static constexpr int NSMWG = (NQT == 2) ? 2 : 1;      // softmax warpgroups
  static constexpr int THREADS = 128 * (1 + NSMWG);
  // register split (setmaxnreg) with two softmax warpgroups: control warpgroup, softmax warpgroups;
  // the sum must fit in the launch allocation (THREADS x the kernel's register count, checked on the
  // host before the first launch)
  static constexpr bool SPLIT_REGS = (NQT == 2);
  static constexpr int CTRL_REGS = 104;
  static constexpr int SM_REGS = 192;
  static constexpr int EMU_COLS = F8 ? 0 : D == 32 ? ATTN_EMU_COLS_D32 : D == 64 ? ATTN_EMU_COLS_D64
                                  : D == 128 ? ATTN_EMU_COLS_D128 : ATTN_EMU_COLS_D256;
  static_assert(EMU_COLS % 8 == 0 && EMU_COLS >= 0 && EMU_COLS <= 128, "emulated column count");
  static constexpr int PPC = 4 / EB;                    // P values per 32-bit TMEM column (2 bf16, 4 e4m3)
  static constexpr int HALF_PAIRS = BN / 2 / PPC;       // TMEM columns of P per half tile
  // TMEM columns (fp32 each): two S slots, then one O accumulator per query tile.
  static constexpr int S_COL0 = 0;
  static constexpr int S_COL1 = BN;
  static constexpr int O_COL0 = 2 * BN;
  static constexpr int O_COL1 = 2 * BN + D;
  // separate P buffers (bf16 pairs: BN / 2 columns each), after the O accumulators
  static constexpr int P_COL0 = 2 * BN + NQT * D;
  static constexpr int P_COL1 = P_COL0 + BN / 2;
  static constexpr int TMEM_COLS = 512;
  static_assert(2 * BN + NQT * D + (SEP_P ? NQT * BN / 2 : 0) <= TMEM_COLS, "tensor memory budget");
  // q_full, q_empty, kv_full[S], kv_empty[S], s_full[2], p_full[2], o_done, o_final[2], drain,
  // s_free[2], p_free[2], sched_full[SCHED], sched_empty[SCHED]
  static constexpr int SCHED = 4;  // units the producer may claim ahead of the consumers
  static constexpr int NBARS = 2 + 2 * STAGES + 2 + 2 + 1 + 2 + 1 + 2 + 2 + 2 * SCHED;
  static constexpr int SCHED_CONSUMERS = 1 + 4 * NSMWG;  // MMA thread + one arrival per softmax warp
  static constexpr int SMEM_DATA = NQT * Q_TILE_BYTES + STAGES * KV_TILE_BYTES;
  // Pad small-d configurations so only one CTA (and one 512-column TMEM allocation) fits per SM.
  static constexpr int SMEM_MIN = 120 * 1024;
  static constexpr int SMEM_BYTES_RAW = 1024 + SMEM_DATA + NBARS * 8 + 16 + SCHED * 4;
  static constexpr int SMEM_BYTES = SMEM_BYTES_RAW > SMEM_MIN ? SMEM_BYTES_RAW : SMEM_MIN;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Signals an mbarrier once per warp after the warp's tcgen05.st have completed: each lane waits
// for its own stores and fences them, the warp syncs, and one lane arrives (barrier count = 4 warps).
__device__ __forceinline__ void warp_publish_tmem_stores(uint64_t* bar, int lane) {
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
}

// Dynamic unit scheduling: a launch claims units from one slot of these counters (next unit, CTAs
// finished). The host gives each launch the next of kSchedSlots slots; the last CTA of a launch to
// finish returns the slot to zero, so launches that follow each other never see a live counter.
constexpr int kSchedSlots = 256;
__device__ unsigned int g_sched_next[kSchedSlots];
__device__ unsigned int g_sched_done[kSchedSlots];
// The slots are shared by every variant of the kernel (head dims, 8-bit), so one launch counter
// serves them all: two launches in flight on different streams never get the same slot, whatever
// variants they are (up to kSchedSlots launches in flight).
static std::atomic<unsigned> g_fwd_launch_count{0};

// Units in issue order: heads grouped so a group's K/V fit comfortably in L2 (group size chosen on
// the host) and, inside a group, heaviest first (every head's last query block, then the one
// before, ...), the longest-processing-time order for causal masks.
struct Unit {
  int b, h, q0;
  int n_tiles;   // K/V tiles the unit streams (the last query tile's count)
  int n_tile0;   // K/V tiles the first query tile needs (fewer when the last one is above its diagonal)
};

template <int D, bool PAIR>
__device__ __forceinline__ Unit unit_at(const FwdArgs& a, int lin) {
  using C = FwdCfg<D, false, PAIR>;
  const int BH = a.B * a.Hq;
  const int per_group = a.heads_per_group * a.n_qblk;
  const int grp = lin / per_group;
  const int r_in = lin % per_group;
  const int gh = min(a.heads_per_group, BH - grp * a.heads_per_group);  // heads in this group
  const int bh = grp * a.heads_per_group + r_in % gh;
  const int qblk = a.n_qblk - 1 - r_in / gh;
  Unit u;
  u.b = bh / a.Hq;
  u.h = bh % a.Hq;
  u.q0 = qblk * C::UNIT_ROWS;
  int kv_end = a.Nkv;
  if (a.causal) {
    const int q_last = min(u.q0 + C::UNIT_ROWS, a.Nq) - 1;
    kv_end = min(a.Nkv, q_last + (a.Nkv - a.Nq) + 1);
  }
  u.n_tiles = kv_end > 0 ? (kv_end + C::BN - 1) / C::BN : 0;
  u.n_tile0 = u.n_tiles;
  if (C::NQT == 2 && a.causal) {
    const int end0 = min(a.Nkv, min(u.q0 + C::BM, a.Nq) - 1 + (a.Nkv - a.Nq) + 1);
    u.n_tile0 = end0 > 0 ? (end0 + C::BN - 1) / C::BN : 0;
  }
  return u;
}

template <int D, bool F8, bool PAIR>
__global__ void __launch_bounds__(FwdCfg<D, F8, PAIR>::THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdArgs args) {
  using C = FwdCfg<D, F8, PAIR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::NQT * C::Q_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::STAGES * C::KV_TILE_BYTES);
  uint64_t* q_full = bars;                  // one phase per unit: Q tiles landed
  uint64_t* q_empty = q_full + 1;           // one phase per unit: every MMA reading Q is done
  uint64_t* kv_full = q_empty + 1;
  uint64_t* kv_empty = kv_full + C::STAGES;
  uint64_t* s_full = kv_empty + C::STAGES;  // [slot]: S = Q K^T landed in TMEM
  uint64_t* p_full = s_full + 2;            // [slot]: P (bf16) of that slot is in TMEM
  uint64_t* o_done = p_full + 2;            // one phase per PV (single-tile path: O rescale needs PV_{j-1})
  uint64_t* o_final = o_done + 1;           // [tile] one phase per unit: every MMA of the unit is done
  uint64_t* drain = o_final + 2;            // error path: MMAs in flight have finished
  uint64_t* s_free = drain + 1;             // [tile] separate P: the softmax has read S (one phase per S)
  uint64_t* p_free = s_free + 2;            // [tile] separate P: the PV reading the P buffer is done
  uint64_t* sched_full = p_free + 2;        // [SCHED] the producer wrote the k-th unit index
  uint64_t* sched_empty = sched_full + C::SCHED;  // [SCHED] every role read it
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sched_empty + C::SCHED);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* sched_unit = reinterpret_cast<volatile int*>(tmem_holder + 2);  // [SCHED]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint64_t T = args.timeout_ns;
  const int total_units = args.B * args.Hq * args.n_qblk;
  const int diag = args.Nkv - args.Nq;  // key j visible to query i iff j <= i + diag
  // CTA pair: rank 0 (the leader) issues the MMAs of both; barriers that the MMAs, the TMA copies
  // of both CTAs or the softmax warps of both CTAs feed live in the leader's shared memory
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;

  // ---- set-up --------------------------------------------------------------------------------
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], C::P_ARRIVALS);  // one arrival per softmax warp (of both CTAs of a pair)
      mbar_init(&o_final[i], 1);
      mbar_init(&s_free[i], 4);  // one arrival per softmax warp of the tile
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    for (int i = 0; i < C::SCHED; ++i) {
      mbar_init(&sched_full[i], 1);
      mbar_init(&sched_empty[i], C::SCHED_CONSUMERS);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  if (warp == 2) {
    if (PAIR) {
      tmem_alloc_pair(tmem_holder, C::TMEM_COLS);  // the same columns in both CTAs
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // a pair: the peer's barriers are initialised before any remote arrival or copy can reach them
  if (PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // With two softmax warpgroups the 128 control threads give registers to the 256 softmax threads:
  // 128 * 104 + 256 * 192 = 62464 <= 384 * 168 (the launch allocation). Each role changes its budget
  // at the top of its own branch so the new limit covers all of that role's code.
  constexpr bool kSplitRegs = C::SPLIT_REGS;

  // ---- MMA issue helpers ------------------------------------------------------------------------
  // bf16: V is read MN-major (rows of d); 8-bit: V is given transposed and read K-major like K
  // (a pair's MMAs have M = 256: 128 rows in each CTA; each CTA's shared memory holds half of B's N)
  constexpr int MMA_M = 128 * C::CTAS;
  constexpr uint32_t idesc_qk = F8 ? idesc_e4m3_f32(128, C::BN, 0, 0) : idesc_bf16_f32(MMA_M, C::BN, 0, 0);
  constexpr uint32_t idesc_pv = F8 ? idesc_e4m3_f32(128, D, 0, 0) : idesc_bf16_f32(MMA_M, D, 0, 1);
  // Only the start-address field (bits 0-13, 16-byte units) differs between the descriptors of one
  // operand, so each base descriptor is built once and the k-step offsets are added to it.
  // Shared-memory addresses stay below 2^18, so the field never carries into its neighbour.
  const uint64_t dQ = smem_desc(smem_u32(sQ), 16, 8 * C::ROWB, C::LAYOUT);
  const uint64_t dK = smem_desc(smem_u32(sKV), 16, 8 * C::ROWB, C::LAYOUT);
  const uint64_t dV = F8 ? smem_desc(smem_u32(sKV), 16, 8 * C::ROWB, C::LAYOUT)
                        : smem_desc(smem_u32(sKV), C::V_CHUNK_BYTES, 8 * C::ROWB, C::LAYOUT);
  // S[slot] = Q_qt K^T : A = Q tile (K-major), B = K tile (K-major), k-steps of 16 along d.
  auto issue_qk = [&](int qt, int s_col, int stage) {
    const uint64_t a0 = dQ + uint64_t((qt * C::Q_TILE_BYTES) >> 4);
    const uint64_t b0 = dK + uint64_t((stage * C::KV_TILE_BYTES) >> 4);
#pragma unroll
    for (int kk = 0; kk < D / C::KSTEP; ++kk) {
      const uint32_t ao = (kk / C::KPC) * C::Q_CHUNK_BYTES + (kk % C::KPC) * 32;
      const uint32_t bo = (kk / C::KPC) * C::K_CHUNK_BYTES + (kk % C::KPC) * 32;
      if (PAIR)
        umma_ss_pair(tmem + s_col, a0 + (ao >> 4), b0 + (bo >> 4), idesc_qk, kk > 0 ? 1u : 0u);
      else if (F8)
        umma_ss_f8(tmem + s_col, a0 + (ao >> 4), b0 + (bo >> 4), idesc_qk, kk > 0 ? 1u : 0u);
      else
        umma_ss(tmem + s_col, a0 + (ao >> 4), b0 + (bo >> 4), idesc_qk, kk > 0 ? 1u : 0u);
    }
  };
  // O += P V over the tile's keys: A = P (bf16, in TMEM over S), B = V tile read MN-major (N = d),
  // k-steps of 16 keys.
  auto issue_pv = [&](int o_col, int p_col, int stage, bool accumulate) {
    const uint64_t b0 = dV + uint64_t((stage * C::KV_TILE_BYTES) >> 4);
#pragma unroll
    for (int kk = 0; kk < C::BN / C::KSTEP; ++kk) {
      // A = P: KSTEP keys = 8 TMEM columns in both forms; B: the next KSTEP rows of V (MN-major) or
      // the next 32 bytes of each transposed-V row (K-major)
      if (PAIR)
        umma_ts_pair(tmem + o_col, tmem + p_col + kk * 8, b0 + uint64_t((kk * 16 * C::ROWB) >> 4), idesc_pv,
                     (accumulate || kk > 0) ? 1u : 0u);
      else if (F8)
        umma_ts_f8(tmem + o_col, tmem + p_col + kk * 8, b0 + uint64_t((kk * 32) >> 4), idesc_pv,
                   (accumulate || kk > 0) ? 1u : 0u);
      else
        umma_ts(tmem + o_col, tmem + p_col + kk * 8, b0 + uint64_t((kk * 16 * C::ROWB) >> 4), idesc_pv,
                (accumulate || kk > 0) ? 1u : 0u);
    }
  };
  // K/V ring positions run on across units; inside a unit K_j is at base + 2j, V_j at base + 2j + 1.
  auto kv_slot = [](int pos) { return pos % C::STAGES; };
  auto kv_phase = [](int pos) { return uint32_t((pos / C::STAGES) & 1); };

  // The k-th unit of this CTA as handed out by the producer (-1: no more units or a wait gave up).
  // Every consumer role reads the slot and then arrives once (one thread for the MMA warp, lane 0
  // of each softmax warp after the warp has read it).
  auto next_unit = [&](int k, bool whole_warp) -> int {
    const int slot = k % C::SCHED;
    const uint32_t ph = uint32_t((k / C::SCHED) & 1);
    bool seen = mbar_wait(&sched_full[slot], ph, abort_flag, T);
    if (whole_warp) seen = __all_sync(0xffffffffu, seen);
    if (!seen) return -1;
    const int lin = sched_unit[slot];
    if (whole_warp) __syncwarp();
    if (!whole_warp || lane == 0) mbar_arrive(&sched_empty[slot]);
    return lin;
  };
  // A pair's units are fixed instead: cluster p of P takes units p, p + P, p + 2P, ... in issue
  // order, and every role of both CTAs walks the same list.
  auto pair_unit = [&](int k) -> int {
    const long long lin = (long long)(blockIdx.x / 2) + (long long)k * (gridDim.x / 2);
    return lin < total_units ? int(lin) : -1;
  };
  // MMA completion: to this CTA's barrier, or to the barrier at the same offset in both CTAs of a pair
  auto commit = [&](uint64_t* bar) {
    if (PAIR)
      umma_commit_pair(bar);
    else
      umma_commit(bar);
  };
  // waits on phases that the other CTA of a pair may complete (acquire at cluster scope)
  auto wait_x = [&](uint64_t* bar, uint32_t ph) -> bool {
    return PAIR ? mbar_wait_cluster(bar, ph, abort_flag, T) : mbar_wait(bar, ph, abort_flag, T);
  };

  if (warp == 0) {
    // ================================ TMA producer ================================
    if (kSplitRegs) regs_dec<C::CTRL_REGS>();
    if (lane == 0) {
      bool ok = true;
      int pos = 0;  // next ring position
      int qc = 0;   // units loaded so far (phase of q_full / q_empty)
      for (int k = 0; ok; ++k) {
        int lin;
        if (PAIR) {
          lin = pair_unit(k);
        } else {
          // claim the next unit (longest first) and hand it to the other roles
          const int slot = k % C::SCHED;
          if (!mbar_wait(&sched_empty[slot], uint32_t(((k / C::SCHED) & 1) ^ 1), abort_flag, T)) {
            ok = false;
            break;
          }
          const unsigned claimed = atomicAdd(&g_sched_next[args.sched_slot], 1u);
          lin = claimed < unsigned(total_units) ? int(claimed) : -1;
          sched_unit[slot] = lin;
          mbar_arrive(&sched_full[slot]);
        }
        if (lin < 0) break;
        const Unit un = unit_at<D, PAIR>(args, lin);
        if (un.n_tiles == 0) continue;
        const int g = un.h / args.group;
        // Q of the previous unit must be consumed by all its QK MMAs before it is overwritten
        if (qc > 0 && !wait_x(q_empty, (qc - 1) & 1)) {
          ok = false;
          break;
        }
        if (PAIR) {
          // each CTA loads its own 128 rows; the leader's q_full counts the bytes of both (the leader
          // arrives on its own barrier, so the plain CTA-scope form suffices: a cluster-scope release
          // costs ~1,000 cycles on this path)
          if (rank == 0) mbar_arrive_expect_tx(q_full, C::CTAS * C::Q_TILE_BYTES);
          const uint32_t bar_l = mapa_shared(q_full, 0);
#pragma unroll
          for (int c = 0; c < C::NCHUNK; ++c)
            tma_load_4d_pair(sQ + c * C::Q_CHUNK_BYTES, &tmQ, bar_l, c * C::CHUNK, un.h, un.q0 + int(rank) * C::BM,
                             un.b);
        } else {
          mbar_arrive_expect_tx(q_full, C::NQT * C::Q_TILE_BYTES);
#pragma unroll
          for (int qt = 0; qt < C::NQT; ++qt)
#pragma unroll
            for (int c = 0; c < C::NCHUNK; ++c)
              tma_load_4d(sQ + qt * C::Q_TILE_BYTES + c * C::Q_CHUNK_BYTES, &tmQ, q_full, c * C::CHUNK, un.h,
                          un.q0 + qt * C::BM, un.b);
        }
        ++qc;
        for (int j = 0; j < un.n_tiles && ok; ++j) {
#pragma unroll
          for (int kv = 0; kv < 2; ++kv, ++pos) {
            const int s = kv_slot(pos);
            if (!wait_x(&kv_empty[s], kv_phase(pos) ^ 1)) {
              ok = false;
              break;
            }
            if (PAIR) {
              // K part: this CTA's 64 keys of the tile, all of d; V part: all keys, this CTA's half of d.
              // The leader's kv_full counts the bytes of both CTAs.
              if (rank == 0) mbar_arrive_expect_tx(&kv_full[s], C::CTAS * C::KV_TILE_BYTES);
              const uint32_t bar_l = mapa_shared(&kv_full[s], 0);
              uint8_t* dst = sKV + s * C::KV_TILE_BYTES;
              if (kv == 0) {
#pragma unroll
                for (int c = 0; c < C::NCHUNK; ++c)
                  tma_load_4d_pair(dst + c * C::K_CHUNK_BYTES, &tmK, bar_l, c * C::CHUNK, g,
                                   j * C::BN + int(rank) * C::K_ROWS, un.b);
              } else {
#pragma unroll
                for (int c = 0; c < C::V_COLS / C::CHUNK; ++c)
                  tma_load_4d_pair(dst + c * C::V_CHUNK_BYTES, &tmV, bar_l, int(rank) * C::V_COLS + c * C::CHUNK, g,
                                   j * C::BN, un.b);
              }
              continue;
            }
            mbar_arrive_expect_tx(&kv_full[s], C::KV_TILE_BYTES);
            const CUtensorMap* m = kv ? &tmV : &tmK;
            if (F8 && kv) {
              // transposed V [B, Hkv, d, Nkv]: keys j*BN .. j*BN+BN-1 of all d rows, one box
              tma_load_4d(sKV + s * C::KV_TILE_BYTES, m, &kv_full[s], j * C::BN, 0, g, un.b);
            } else {
#pragma unroll
              for (int c = 0; c < C::NCHUNK; ++c)
                tma_load_4d(sKV + s * C::KV_TILE_BYTES + c * C::K_CHUNK_BYTES, m, &kv_full[s], c * C::CHUNK, g,
                            j * C::BN, un.b);
            }
          }
        }
      }
      if (!ok && rank == 0) {
        // Give the copies already in flight a bounded chance to land before the CTA exits (a pair's
        // copies, the peer's included, complete on the leader's barriers).
        if (qc > 0) mbar_wait(q_full, (qc - 1) & 1, nullptr, 100000000ull);
        // ring positions [0, pos) were issued; slot s holds the fills at positions s, s + STAGES, ...
        for (int s = 0; s < C::STAGES; ++s) {
          const int fills = (pos - s + C::STAGES - 1) / C::STAGES;
          if (fills > 0) mbar_wait(&kv_full[s], (fills - 1) & 1, nullptr, 100000000ull);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ================================ MMA issuer ================================
    if (kSplitRegs) regs_dec<C::CTRL_REGS>();
    if (lane == 0 && rank == 0) {  // a pair: the leader issues for both CTAs
      // K/V tiles and Q arrive by TMA (complete_tx on the mbarrier): the MMAs may read them once the
      // barrier phase is observed. P is written to TMEM by the softmax threads' tcgen05.st, so
      // observing p_full is followed by tcgen05.fence::after_thread_sync before the PV MMAs.
      bool ok = true;
      int pos = 0;    // ring position of the next K/V tile to consume
      int qc = 0;     // units issued (phase of q_full)
      int pc[2] = {0, 0};  // P tiles consumed per slot (phase of p_full)
      int qk_cnt[2] = {0, 0};  // separate P: S tiles issued per query tile (phase of s_free)
      int t_run = 0;  // single-tile path: S tiles issued so far (slot = t_run & 1)
      for (int k = 0; ok; ++k) {
        const int lin = PAIR ? pair_unit(k) : next_unit(k, false);
        if (lin < 0) break;
        const Unit un = unit_at<D, PAIR>(args, lin);
        const int n = un.n_tiles;
        if (n == 0) continue;
        ok = wait_x(q_full, qc & 1);
        ++qc;
        const int base = pos;  // K_j at base + 2j, V_j at base + 2j + 1
        if (C::SEP_P) {
          // Two query tiles, P in buffers of its own. QK(t, j+1) may overwrite S once the softmax has
          // read S(t, j) (s_free); PV(t, j) reads P(t, j) once it is in place (p_full) and frees the
          // buffer when done (p_free):  QK(0,0) QK(1,0) | QK(0,1) QK(1,1) PV(0,0) PV(1,0) | ...
          const int nt[2] = {un.n_tile0, n};
          auto qk_into = [&](int qt, int jj, int stage) -> bool {
            if (qk_cnt[qt] > 0) {
              if (!wait_x(&s_free[qt], uint32_t((qk_cnt[qt] - 1) & 1))) return false;
              tc_fence_after();
            }
            issue_qk(qt, qt ? C::S_COL1 : C::S_COL0, stage);
            commit(&s_full[qt]);
            if (qt == 1 && jj == n - 1) commit(q_empty);  // the unit's last QK: Q may be reloaded
            ++qk_cnt[qt];
            return true;
          };
          if (ok) ok = wait_x(&kv_full[kv_slot(base)], kv_phase(base));
#pragma unroll
          for (int qt = 0; qt < 2; ++qt)
            if (ok && nt[qt] > 0) ok = qk_into(qt, 0, kv_slot(base));
          if (ok) commit(&kv_empty[kv_slot(base)]);
          for (int j = 0; j < n && ok; ++j) {
            const int pv_pos = base + 2 * j + 1, pk_pos = base + 2 * j + 2;
            const bool nxt = j + 1 < n;
            ok = wait_x(&kv_full[kv_slot(pv_pos)], kv_phase(pv_pos));
            if (ok && nxt) ok = wait_x(&kv_full[kv_slot(pk_pos)], kv_phase(pk_pos));
#pragma unroll
            for (int qt = 0; qt < 2; ++qt)
              if (ok && j + 1 < nt[qt]) ok = qk_into(qt, j + 1, kv_slot(pk_pos));
#pragma unroll
            for (int qt = 0; qt < 2; ++qt) {
              if (!ok || j >= nt[qt]) continue;
              ok = wait_x(&p_full[qt], pc[qt] & 1);
              if (!ok) break;
              ++pc[qt];
              tc_fence_after();
              issue_pv(qt ? C::O_COL1 : C::O_COL0, qt ? C::P_COL1 : C::P_COL0, kv_slot(pv_pos), j > 0);
              commit(&p_free[qt]);
              if (qt == 0 && j == nt[0] - 1 && nt[0] < n) commit(&o_final[0]);  // see below
            }
            if (!ok) break;
            commit(&kv_empty[kv_slot(pv_pos)]);
            if (nxt) commit(&kv_empty[kv_slot(pk_pos)]);
          }
          pos = base + 2 * n;
        } else if (C::NQT == 2) {
          // Two query tiles, one S slot each: QK(0,0) QK(1,0) | PV(0,j) QK(0,j+1) PV(1,j) QK(1,j+1) | ...
          if (ok) ok = wait_x(&kv_full[kv_slot(base)], kv_phase(base));
          // a causal unit's first query tile may need one K/V tile fewer than the second
          const int nt[2] = {un.n_tile0, n};
          if (ok) {
#pragma unroll
            for (int qt = 0; qt < 2; ++qt) {
              if (nt[qt] == 0) continue;
              issue_qk(qt, qt ? C::S_COL1 : C::S_COL0, kv_slot(base));
              commit(&s_full[qt]);
              if (qt == 1 && n == 1) commit(q_empty);  // the unit's last QK: Q may be reloaded
            }
            commit(&kv_empty[kv_slot(base)]);
          }
          for (int j = 0; j < n && ok; ++j) {
            const int pv_pos = base + 2 * j + 1, pk_pos = base + 2 * j + 2;
            const bool nxt = j + 1 < n;
            ok = wait_x(&kv_full[kv_slot(pv_pos)], kv_phase(pv_pos));
            if (ok && nxt) ok = wait_x(&kv_full[kv_slot(pk_pos)], kv_phase(pk_pos));
#pragma unroll
            for (int qt = 0; qt < 2; ++qt) {
              if (!ok) break;
              if (j >= nt[qt]) continue;
              const int s_col = qt ? C::S_COL1 : C::S_COL0;
              ok = wait_x(&p_full[qt], pc[qt] & 1);
              if (!ok) break;
              ++pc[qt];
              tc_fence_after();
              issue_pv(qt ? C::O_COL1 : C::O_COL0, s_col, kv_slot(pv_pos), j > 0);
              if (qt == 0 && j == nt[0] - 1 && nt[0] < n) commit(&o_final[0]);  // see below
              // P of this tile is consumed by the PV MMAs above before this QK overwrites the slot:
              // MMAs issued by one thread execute in issue order.
              if (j + 1 < nt[qt]) {
                issue_qk(qt, s_col, kv_slot(pk_pos));
                commit(&s_full[qt]);
                if (qt == 1 && j + 2 == n) commit(q_empty);  // the unit's last QK
              }
            }
            if (!ok) break;
            commit(&kv_empty[kv_slot(pv_pos)]);
            if (nxt) commit(&kv_empty[kv_slot(pk_pos)]);
          }
          pos = base + 2 * n;
        } else {
          // One query tile, S alternating between two slots: QK_0, QK_1, PV_0, QK_2, PV_1, QK_3, ...
          const int t0 = t_run;
          for (int j = 0; j < 2 && j < n && ok; ++j) {
            ok = wait_x(&kv_full[kv_slot(base + 2 * j)], kv_phase(base + 2 * j));
            if (!ok) break;
            issue_qk(0, ((t0 + j) & 1) ? C::S_COL1 : C::S_COL0, kv_slot(base + 2 * j));
            commit(&s_full[(t0 + j) & 1]);
            if (j == n - 1) commit(q_empty);  // the unit's last QK: Q may be reloaded
            commit(&kv_empty[kv_slot(base + 2 * j)]);
          }
          for (int j = 0; j < n && ok; ++j) {
            const int t = t0 + j;
            const int slot = t & 1;
            const int s_col = slot ? C::S_COL1 : C::S_COL0;
            ok = wait_x(&kv_full[kv_slot(base + 2 * j + 1)], kv_phase(base + 2 * j + 1));
            if (ok) ok = wait_x(&p_full[slot], (t >> 1) & 1);
            if (!ok) break;
            tc_fence_after();
            issue_pv(C::O_COL0, s_col, kv_slot(base + 2 * j + 1), j > 0);
            commit(o_done);
            commit(&kv_empty[kv_slot(base + 2 * j + 1)]);
            if (j + 2 < n) {
              const int kp = base + 2 * (j + 2);
              ok = wait_x(&kv_full[kv_slot(kp)], kv_phase(kp));
              if (!ok) break;
              issue_qk(0, s_col, kv_slot(kp));
              commit(&s_full[slot]);
              if (j + 3 == n) commit(q_empty);  // the unit's last QK
              commit(&kv_empty[kv_slot(kp)]);
            }
          }
          t_run = t0 + n;
          pos = base + 2 * n;
        }
        if (!ok) break;
        // O may be read once every MMA writing it is done (one o_final phase per tile and unit with
        // keys for that tile), here after the unit's last PV. When tile 0 needs fewer K/V tiles
        // (causal) its phase came right after its own last PV instead, so its epilogue runs during
        // tile 1's last step. A tile without keys gets no phase: its warpgroup takes no part in the
        // unit, so phases committed for it could run two ahead of its waits, which a parity wait
        // cannot tell apart. (Q was released after the unit's last QK, so the next unit's Q load
        // overlaps the last PVs and the epilogues.)
        if (C::NQT == 1 || un.n_tile0 == n) commit(&o_final[0]);
        if (C::NQT == 2) commit(&o_final[1]);
      }
      if (!ok) {
        // Let the MMAs already issued finish before tensor memory is released.
        commit(drain);
        mbar_wait(drain, 0, nullptr, 100000000ull);
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    if (kSplitRegs) regs_dec<C::CTRL_REGS>();
  } else {
    // ================================ softmax warpgroups ================================
    if (kSplitRegs) regs_inc<C::SM_REGS>();
    const int wg = (warp - 4) >> 2;
    const int wq = warp & 3;             // warp within its warpgroup: TMEM lanes 32*wq .. 32*wq+31
    const int row = wq * 32 + lane;      // query row within the tile = TMEM lane
    const int qt = (C::NQT == 2) ? wg : 0;
    const uint32_t lane_addr = tmem + (uint32_t(wq * 32) << 16);
    const uint32_t o_col = qt ? C::O_COL1 : C::O_COL0;
    float c = args.scale_log2;  // log2-domain factor on the raw scores (8-bit: times both dequantizations)
    float sc_nat = args.scale;  // the same in natural-log units, for the LSE
    float o_mul = 1.0f;         // epilogue factor on O (8-bit: V's dequantization)
    // every lane waits; the warp continues only if all of them saw the phase (tcgen05.ld/st below are
    // warp-collective, so a partial give-up must not split the warp)
    auto wait_warp = [&](uint64_t* bar, uint32_t ph) -> bool { return __all_sync(0xffffffffu, wait_x(bar, ph)); };
    // P of this warp's 32 rows is in TMEM: tell the MMA thread (a pair's is in the leader)
    auto publish_p = [&](uint64_t* bar) {
      if (PAIR) {
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(bar, 0));
      } else {
        warp_publish_tmem_stores(bar, lane);
      }
    };

    bool ok = true;
    int sc = 0;     // S tiles consumed by this warpgroup (two tiles: phase of s_full[qt])
    int t_run = 0;  // single-tile path: S tiles consumed so far (slot = t_run & 1)
    int uc = 0;     // units with keys finished (phase of o_final)
    int pt = 0;     // separate P: P tiles this warpgroup has published (phase of p_free[qt])
    for (int k = 0; ok; ++k) {
      const int lin = PAIR ? pair_unit(k) : next_unit(k, true);
      if (lin < 0) break;
      const Unit un = unit_at<D, PAIR>(args, lin);
      if (F8) {
        // codes decode as value = code * amax / 448 per (batch, head)
        const int g = un.h / args.group;
        const float dq = args.amax_q[un.b * args.Hq + un.h] / 448.0f;
        const float dk = args.amax_k[un.b * args.Hkv + g] / 448.0f;
        c = args.scale_log2 * dq * dk;
        sc_nat = args.scale * dq * dk;
        o_mul = args.amax_v[un.b * args.Hkv + g] / 448.0f;
      }
      const int q_first = un.q0 + (qt + int(rank)) * C::BM;  // (a pair: NQT = 1, rank 1 takes the second 128 rows)
      const int q_row = q_first + row;
      // last key visible to this row (any key index <= lim is visible); rows past Nq are padding
      const int lim = args.causal ? min(args.Nkv - 1, q_row + diag) : args.Nkv - 1;
      float m_ref = -INFINITY;  // reference max (raw-score units) of the exponentials in l and O
      float l = 0.f;            // running row sum of exp2(c * (s - m_ref))

      const int my_tiles = (qt == 0) ? un.n_tile0 : un.n_tiles;
      for (int j = 0; j < my_tiles; ++j) {
        // two query tiles: one S slot per tile; one query tile: S alternates between the two slots
        const int slot = (C::NQT == 2) ? qt : (t_run & 1);
        const uint32_t ph = (C::NQT == 2) ? uint32_t(sc & 1) : uint32_t((t_run >> 1) & 1);
        if (!wait_warp(&s_full[slot], ph)) {
          ok = false;
          break;
        }
        ++sc;
        ++t_run;
        tc_fence_after();
        const uint32_t s_addr = lane_addr + (slot ? C::S_COL1 : C::S_COL0);
        // where P goes: a buffer of its own, or over S
        const uint32_t p_addr = C::SEP_P ? lane_addr + (slot ? C::P_COL1 : C::P_COL0) : s_addr;
        // separate P: the previous PV of this tile (it reads the P buffer and adds into O) is done
        auto wait_prev_pv = [&]() -> bool {
          if (!C::SEP_P || pt == 0) return true;
          if (!wait_warp(&p_free[slot], uint32_t((pt - 1) & 1))) return false;
          tc_fence_after();
          return true;
        };

        // ---- S -> P: mask, running max with conditional O rescale, exponentials, row sum ----
        uint32_t r[C::BN];
#pragma unroll
        for (int cc = 0; cc < C::BN / 32; ++cc) tmem_ld32(s_addr + cc * 32, r + cc * 32);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < C::BN / 32; ++cc) tmem_reg_fence32(r + cc * 32);
        if (C::SEP_P) {
          // S is in registers: the next QK of this tile may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_free[slot]);
        }

        const int kbase = j * C::BN;
        // warp-uniform: does any key of this tile fall outside some row's visible range?
        const bool need_mask =
            (kbase + C::BN > args.Nkv) || (args.causal && kbase + C::BN - 1 > q_first + diag);
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < C::BN; ++i)
            if (kbase + i > lim) r[i] = __float_as_uint(-INFINITY);
        }
        // row max: a balanced tree of 3-input max (depth 5 for 128 keys; eight chains of 3-input
        // max would be depth 9, and the first exponential waits for this max)
        float mx;
        {
          float t[C::BN];
#pragma unroll
          for (int i = 0; i < C::BN; ++i) t[i] = __uint_as_float(r[i]);
          int m = C::BN;  // values left: t[0 .. m)
#pragma unroll
          for (int lvl = 0; lvl < 6; ++lvl) {  // 128 -> 44 -> 16 -> 6 -> 2 -> 1
            if (m <= 1) break;
            if (m == 2) {
              t[0] = fmaxf(t[0], t[1]);
              m = 1;
              break;
            }
            const int n3 = m / 3, rem = m - 3 * n3;
#pragma unroll
            for (int i = 0; i < C::BN / 3 + 1; ++i)
              if (i < n3) t[i] = fmax3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
#pragma unroll
            for (int i = 0; i < 2; ++i)
              if (i < rem) t[n3 + i] = t[3 * n3 + i];
            m = n3 + rem;
          }
          mx = t[0];
        }
        const float m_new = fmaxf(m_ref, mx);
        // true when the max moved by more than TAU (also on the first live tile: -inf -> finite)
        const bool need = (m_new - m_ref) * c > kRescaleTau;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2((m_ref - m_new) * c) : 1.0f;
          if (need) m_ref = m_new;
          l *= alpha;
          if (j > 0) {
            if (C::NQT == 1) {
              // PV of the previous tile must have landed in O before it is rescaled. (With two query
              // tiles and P over S, S_j is committed after PV_{j-1} of the same tile, so it has
              // landed already; with separate P it is waited for here.)
              if (!wait_warp(o_done, uint32_t((t_run - 2) & 1))) {
                ok = false;
                break;
              }
              tc_fence_after();
            } else if (!wait_prev_pv()) {
              ok = false;
              break;
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
        // P = 2^(c*s - c*m_ref) as bf16 over the first BN/2 columns of the slot (two per 32-bit
        // column; the S values it replaces are already in registers). Pairs go through the packed
        // FMA pipe; the exponential uses the exp unit (MUFU.EX2) or, for the last kEmuCols columns
        // of tiles without masked keys, the FMA-pipe polynomial (EMU_COLS).
        const float mc = (m_ref == -INFINITY) ? 0.f : m_ref * c;
        const float2 c2 = make_float2(c, c);
        const float2 nmc2 = make_float2(-mc, -mc);
        float2 acc4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
        constexpr int EMU_FROM = (C::BN - C::EMU_COLS * C::BN / 128) / 2;  // first emulated pair
        const bool emu = C::EMU_COLS > 0 && !need_mask;
        if (!wait_prev_pv()) {  // the P buffer is free again
          ok = false;
          break;
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t p[C::HALF_PAIRS];
          if constexpr (F8) {
            // four keys per TMEM column, e4m3 (P <= 2^TAU stays far below the e4m3 limit of 448)
#pragma unroll
            for (int i2 = 0; i2 < C::HALF_PAIRS; ++i2) {
              const int k0 = 4 * (half * C::HALF_PAIRS + i2);
              const float2 x0 =
                  ffma2(make_float2(__uint_as_float(r[k0]), __uint_as_float(r[k0 + 1])), c2, nmc2);
              const float2 x1 =
                  ffma2(make_float2(__uint_as_float(r[k0 + 2]), __uint_as_float(r[k0 + 3])), c2, nmc2);
              const float2 e0 = make_float2(ex2(x0.x), ex2(x0.y));
              const float2 e1 = make_float2(ex2(x1.x), ex2(x1.y));
              acc4[(2 * i2) & 3] = fadd2(acc4[(2 * i2) & 3], e0);
              acc4[(2 * i2 + 1) & 3] = fadd2(acc4[(2 * i2 + 1) & 3], e1);
              p[i2] = pack_e4m3x4(e0.x, e0.y, e1.x, e1.y);
            }
          } else {
#pragma unroll
            for (int i2 = 0; i2 < C::HALF_PAIRS; ++i2) {
              const int i = half * C::HALF_PAIRS + i2;
              const float2 x =
                  ffma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), c2, nmc2);
              float2 e;
              if (i >= EMU_FROM && emu) {
                e = exp2_poly2(x);
              } else {
                e.x = ex2(x.x);
                e.y = ex2(x.y);
              }
              acc4[i & 3] = fadd2(acc4[i & 3], e);
              p[i2] = pack_bf16x2(e.x, e.y);
            }
          }
          if (C::HALF_PAIRS == 32)
            tmem_st32(p_addr + half * C::HALF_PAIRS, p);
          else
            tmem_st16(p_addr + half * C::HALF_PAIRS, p);
        }
        publish_p(&p_full[slot]);
        ++pt;
        const float2 s01 = fadd2(acc4[0], acc4[1]);
        const float2 s23 = fadd2(acc4[2], acc4[3]);
        const float2 s = fadd2(s01, s23);
        l += s.x + s.y;
      }
      if (!ok) break;

      // ---- epilogue: O = acc / l (once), LSE = scale * m_ref + ln l -------------------------------
      const bool valid = q_row < args.Nq;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(args.o) +
                            ((size_t(un.b) * args.Nq + (valid ? q_row : 0)) * args.Hq + un.h) * D;
      if (un.n_tiles > 0 && my_tiles == 0) {
        // this tile saw no key: O = 0 (no MMA wrote its accumulator, and no o_final phase was
        // committed for it)
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow);
          for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
        }
      } else if (un.n_tiles > 0) {
        if (!wait_warp(&o_final[qt], uint32_t(uc & 1))) {
          ok = false;
          break;
        }
        ++uc;
        tc_fence_after();
        const float inv = (l > 0.f) ? o_mul / l : 0.f;
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
            if (D >= 128 && (reinterpret_cast<uintptr_t>(args.o) & 31) == 0) {
              // 32-byte stores, one full sector per lane: the row-per-thread layout makes every store
              // instruction touch 32 rows, and halving their number shortens the epilogue (causal
              // N2048: +2 %); d = 64 measured slightly slower with them
#pragma unroll
              for (int v8 = 0; v8 < 2; ++v8)
                asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(orow + cc * 32 + v8 * 16),
                             "r"(pk[8 * v8]), "r"(pk[8 * v8 + 1]), "r"(pk[8 * v8 + 2]), "r"(pk[8 * v8 + 3]),
                             "r"(pk[8 * v8 + 4]), "r"(pk[8 * v8 + 5]), "r"(pk[8 * v8 + 6]), "r"(pk[8 * v8 + 7])
                             : "memory");
            } else {
              uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4)
                dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
            }
          }
        }
        // O of this tile was read (tcgen05.wait::ld above) before any P of the next unit is
        // published, so the next unit's first PV cannot overwrite it early.
      } else if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
        for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
      }
      if (valid)
        args.lse[(size_t(un.b) * args.Hq + un.h) * args.Nq + q_row] =
            (l > 0.f) ? fmaf(m_ref, sc_nat, logf(l)) : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  // a pair: neither CTA frees its tensor memory or exits while the leader's MMAs or the other CTA's
  // barrier arrivals and copies may still reach it
  if (PAIR) cluster_sync();
  if (warp == 2) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem, C::TMEM_COLS);
    else
      tmem_dealloc(tmem, C::TMEM_COLS);
  }
  // The last CTA to finish returns the scheduling slot to zero (all CTAs have stopped claiming).
  if (!PAIR && threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&g_sched_done[args.sched_slot], 1u) == gridDim.x - 1) {
      atomicExch(&g_sched_next[args.sched_slot], 0u);
      atomicExch(&g_sched_done[args.sched_slot], 0u);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
// F8: q and k are e4m3 codes [B, N, H, d], v is the transposed code tensor [B, Hkv, d, Nkv] and
// amax_* the per-(batch, head) dequantization maxima; otherwise bf16 tensors and null amax.
template <int D, bool F8, bool PAIR = false>
static attn_status_t launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                                int Hkv, int Nq, int Nkv, float scale, int causal, const float* amax_q,
                                const float* amax_k, const float* amax_v, cudaStream_t stream) {
  using C = FwdCfg<D, F8, PAIR>;
  auto kernel = attn_fwd_kernel<D, F8, PAIR>;
  CUtensorMap tmQ, tmK, tmV;
  const uint32_t swz = C::ROWB == 128 ? 128u : 64u;
  if (F8) {
    const long long dq[4] = {D, Hq, Nq, B}, dk[4] = {D, Hkv, Nkv, B}, dvt[4] = {Nkv, D, Hkv, B};
    const int bq[4] = {C::CHUNK, 1, C::BM, 1}, bk[4] = {C::CHUNK, 1, C::BN, 1}, bv[4] = {C::BN, D, 1, 1};
    if (!encode_map(&tmQ, q, 1, dq, bq, swz) || !encode_map(&tmK, k, 1, dk, bk, swz) ||
        !encode_map(&tmV, v, 1, dvt, bv, swz))
      return ATTN_ERR_CUDA;
  } else if (!encode_tile_map(&tmQ, q, D, Hq, Nq, B, C::CHUNK, C::BM, swz) ||
             !encode_tile_map(&tmK, k, D, Hkv, Nkv, B, C::CHUNK, C::K_ROWS, swz) ||
             !encode_tile_map(&tmV, v, D, Hkv, Nkv, B, C::CHUNK, C::BN, swz)) {
    return ATTN_ERR_CUDA;
  }

  if (ensure_dyn_smem(reinterpret_cast<const void*>(kernel), C::SMEM_BYTES) != cudaSuccess)
    return ATTN_ERR_CUDA;
  // setmaxnreg.inc waits until the registers it asks for are free in the CTA's launch allocation,
  // so a split whose total exceeds that allocation would never proceed: refuse to launch it.
  if (C::SPLIT_REGS) {
    static std::atomic<int> regs_ok{0};  // 0 unknown, 1 fits, 2 does not (same binary on every device)
    int st = regs_ok.load(std::memory_order_relaxed);
    if (st == 0) {
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return ATTN_ERR_CUDA;
      const long long pool = (long long)fa.numRegs * C::THREADS;
      const long long need = 128LL * C::CTRL_REGS + 128LL * C::NSMWG * C::SM_REGS;
      st = pool >= need ? 1 : 2;
      regs_ok.store(st, std::memory_order_relaxed);
    }
    if (st != 1) return ATTN_ERR_UNSUPPORTED;
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
  a.n_qblk = (Nq + C::UNIT_ROWS - 1) / C::UNIT_ROWS;
  a.causal = causal;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = kWaitLimitNs;
  a.amax_q = amax_q;
  a.amax_k = amax_k;
  a.amax_v = amax_v;
  // heads per L2 group: K/V of one kv head is read by every query head of its group and block; keep
  // a group's K/V within ~48 MB of the 126 MB L2. Causal launches whose K/V fits in L2 comfortably
  // use one group: longest-first then runs over every unit, so no group's long units start near the
  // end of the launch.
  {
    const double kv_bytes_per_head = 2.0 * Nkv * D * C::EB / double(Hq / Hkv);
    const double kv_bytes_total = 2.0 * Nkv * D * C::EB * double(B) * Hkv;
    long long gh = (causal && kv_bytes_total <= kL2OneGroupBytes) ? (long long)B * Hq
                                                                  : (long long)(48.0e6 / kv_bytes_per_head);
    if (gh < 1) gh = 1;
    if (gh > (long long)B * Hq) gh = (long long)B * Hq;
    a.heads_per_group = int(gh);
  }
  const long long units = (long long)a.n_qblk * B * Hq;
  if (units > 0x7FFFFFFFll) return ATTN_ERR_UNSUPPORTED;
  const int sms = sm_count();
  if (sms <= 0) return ATTN_ERR_CUDA;
  if (PAIR) {
    // persistent grid of CTA pairs: as many pairs as fit on the device at once (one CTA per SM), each
    // walking its fixed share of the units
    const int pairs = max_pairs(reinterpret_cast<const void*>(kernel), C::THREADS, C::SMEM_BYTES);
    if (pairs <= 0) return ATTN_ERR_CUDA;
    const long long n_pairs = units < pairs ? units : pairs;
    a.sched_slot = 0;
    cudaLaunchConfig_t lc = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    lc.gridDim = dim3(unsigned(2 * n_pairs));
    lc.blockDim = dim3(C::THREADS);
    lc.dynamicSmemBytes = C::SMEM_BYTES;
    lc.stream = stream;
    lc.attrs = at;
    lc.numAttrs = 1;
    if (cudaLaunchKernelEx(&lc, kernel, tmQ, tmK, tmV, a) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_CUDA;
    }
    return ATTN_OK;
  }
  // persistent grid: one CTA per SM (each holds all 512 TMEM columns), walking the units in order
  const unsigned grid = unsigned(units < sms ? units : sms);
  a.sched_slot = int(g_fwd_launch_count.fetch_add(1) % kSchedSlots);
  kernel<<<dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, stream>>>(tmQ, tmK, tmV, a);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

attn_status_t fwd_dispatch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                           int Hkv, int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream) {
  switch (d) {
    case 32: return launch_fwd<32, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, nullptr, nullptr, nullptr, stream);
    case 64: return launch_fwd<64, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, nullptr, nullptr, nullptr, stream);
    case 128: return launch_fwd<128, false, false>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, nullptr, nullptr, nullptr, stream);
    case 256: return launch_fwd<256, false, true>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, nullptr, nullptr, nullptr, stream);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

attn_status_t fwd_fp8_dispatch(const void* q8, const void* k8, const void* vt8, const float* amax_q,
                               const float* amax_k, const float* amax_v, void* o, float* lse, int B, int Hq, int Hkv,
                               int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream) {
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  return launch_fwd<128, true>(q8, k8, vt8, o, lse, B, Hq, Hkv, Nq, Nkv, scale, causal, amax_q, amax_k, amax_v,
                               stream);
}

}  // namespace attn
