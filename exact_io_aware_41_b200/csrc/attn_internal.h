// Declarations shared by the library's translation units (not part of the public ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "attn.h"

namespace attn {

// Bits of the device error word (g_error_word).
enum : unsigned int {
  kErrBadLengthBit = 2u,  // a decode length outside [0, Nkv_cap] was clamped
  kErrSmemAlignBit = 4u,  // a kernel found its dynamic shared memory off its required alignment
};

// Wall-time limit of every pipeline wait inside a kernel. Far above any legitimate wait (a whole
// 8k x 8k head takes well under a millisecond), so reaching it means the pipeline is broken.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

struct FwdArgs {
  void* o;
  float* lse;
  int B, Hq, Hkv, Nq, Nkv;
  int group;   // Hq / Hkv
  int n_qblk;  // query blocks of NQT*128 rows per (b, h)
  int heads_per_group;  // query heads per L2 group of units
  int sched_slot;       // which unit-claim counter this launch uses
  int causal;
  float scale;       // natural-log scale on Q K^T
  float scale_log2;  // scale * log2(e)
  unsigned long long timeout_ns;
  const float* amax_q;  // 8-bit path: per-(batch, head) maxima the codes were scaled by; else null
  const float* amax_k;
  const float* amax_v;
};

bool is_aligned16(const void* p);

// Devices the per-device host tables cover (device ordinals 0 .. kMaxDevices-1).
constexpr int kMaxDevices = 128;

// Streaming multiprocessors of the current device (-1 on error), looked up once per device.
int sm_count();
// Clusters of two CTAs of `func` (threads, dynamic shared memory as given) resident on the current
// device at once; cached per device for the last kernel asked about. -1 on error.
int max_pairs(const void* func, int threads, int smem_bytes);

// A 4-d TMA map over a token-major bf16 tensor [outer, rows, heads, d] (d innermost), with a box
// of `box_cols` elements of d x 1 head x `box_rows` tokens x 1 batch; swizzle_bytes is 128, 64 or 0
// (none). Maps are cached per (pointer, shape, box, swizzle): a map holds only the address and the
// geometry, so a cached copy is valid wherever the same key comes back. Returns false on failure.
bool encode_tile_map(CUtensorMap* map, const void* base, int d, int heads, int rows, int outer, int box_cols,
                     int box_rows, unsigned swizzle_bytes);

// The general form: a 4-d tensor of elem_bytes-sized elements (1: 8-bit codes, 2: bf16, 4: fp32) with dense
// strides, dims[0] innermost, box[] elements per dimension; cached like encode_tile_map.
bool encode_map(CUtensorMap* map, const void* base, int elem_bytes, const long long* dims, const int* box,
                unsigned swizzle_bytes);

// Opts `func` into `bytes` of dynamic shared memory on the current device. The attribute belongs to
// the function on one device, so it is set once per (function, device) and again only when a
// larger size is asked for; safe to call from several host threads.
cudaError_t ensure_dyn_smem(const void* func, int bytes);

// Largest dynamic shared memory the decode combine kernel takes (its per-split weights and live
// split list, 8 bytes per split).
constexpr size_t kCombineSmemMax = 200 * 1024;
inline bool combine_fits(long long n_splits) {
  return n_splits >= 1 && size_t(n_splits) * (sizeof(float) + sizeof(int)) <= kCombineSmemMax;
}

attn_status_t fwd_dispatch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                           int Hkv, int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream);
attn_status_t fwd_fp8_dispatch(const void* q8, const void* k8, const void* vt8, const float* amax_q,
                               const float* amax_k, const float* amax_v, void* o, float* lse, int B, int Hq, int Hkv,
                               int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream);

attn_status_t fp8_quantize_dispatch(const void* x, const float* signs, void* codes, float* amax, int B, int N, int H,
                                    int transpose, cudaStream_t stream);

size_t bwd_workspace(int B, int Hq, int Nq, int d);
attn_status_t bwd_dispatch(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nkv,
                           float scale, int causal, void* workspace, cudaStream_t stream);

int decode_default_chunk(int B, int Hkv, int Nkv_cap);
size_t decode_workspace(int B, int Hq, int d, int Nkv_cap, int chunk);
attn_status_t decode_split_dispatch(const void* q, const void* kc, const void* vc, const int32_t* lens, int cap,
                                    int B, int Hq, int Hkv, int d, float scale, int chunk, int n_splits,
                                    float* po, float* pl, cudaStream_t st);
attn_status_t decode_combine_dispatch(const float* po, const float* pl, int rows, int n_splits, int d, void* o,
                                      float* lse, cudaStream_t st);

}  // namespace attn
