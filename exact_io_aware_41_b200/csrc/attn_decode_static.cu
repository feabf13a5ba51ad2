// Split-KV decode for callers that cannot allocate device memory.
//
// attn_decode_splitkv needs a caller-provided workspace for the per-split partial outputs and
// log-sum-exps. Some callers have no way to provide one: a plugin loaded into a host runtime that
// owns every device allocation and exposes no allocator, or a latency-critical serving loop that
// must not call cudaMalloc (which can synchronise the device and can fail under memory pressure).
// This entry point keeps those partials in a fixed, file-scope device array instead and allocates
// nothing. The array is part of the library image: every GPU that loads the library holds it until
// the process exits.
#include <mutex>

#include "attn_internal.h"

namespace attn {
namespace {

static_assert(ATTN_DECODE_STATIC_SCRATCH_BYTES % 256 == 0, "scratch size");

// The partials of the most recent call. Device code could name it directly; host code must not
// pass its name to a kernel (on the host it is only a stand-in), so set-up below asks the runtime
// for its device address once per device.
static __device__ __align__(256) unsigned char g_decode_scratch[ATTN_DECODE_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up on the first call per device).
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace attn

using namespace attn;

extern "C" attn_status_t attn_decode_splitkv_static(const void* q, const void* k_cache, const void* v_cache,
                                                     const int32_t* kv_lens, int Nkv_cap, void* o, float* lse, int B,
                                                     int Hq, int Hkv, int d, float scale, int chunk,
                                                     cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !kv_lens || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!is_aligned16(q) || !is_aligned16(k_cache) || !is_aligned16(v_cache) || !is_aligned16(o) ||
      !is_aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(kv_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nkv_cap < 1 || Hq % Hkv != 0 || chunk < 0 || (chunk % 64) != 0)
    return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if ((d != 32 && d != 64 && d != 128 && d != 256) || (G != 1 && G != 2 && G != 4 && G != 8))
    return ATTN_ERR_UNSUPPORTED;
  if (chunk == 0) chunk = decode_default_chunk(B, Hkv, Nkv_cap);
  // every size check comes before the split kernel is enqueued, so a refused call leaves nothing behind
  if (Hkv > 65535 || B > 65535 || !combine_fits((Nkv_cap + (long long)chunk - 1) / chunk))
    return ATTN_ERR_UNSUPPORTED;
  // The partials must fit the fixed array; a larger chunk makes them smaller.
  if (decode_workspace(B, Hq, d, Nkv_cap, chunk) > size_t(ATTN_DECODE_STATIC_SCRATCH_BYTES))
    return ATTN_ERR_WORKSPACE;

  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return ATTN_ERR_CUDA;
  const long long n_splits = (Nkv_cap + (long long)chunk - 1) / chunk;
  float* po = static_cast<float*>(scratch);
  const size_t po_bytes = size_t(B) * Hq * n_splits * d * sizeof(float);
  float* pl = reinterpret_cast<float*>(static_cast<char*>(scratch) + ((po_bytes + 255) / 256) * 256);
  // Nothing in the array has to start at zero: the split kernel writes every partial LSE
  // (-inf for empty splits) and every partial output the combine kernel reads.
  attn_status_t st = decode_split_dispatch(q, k_cache, v_cache, kv_lens, Nkv_cap, B, Hq, Hkv, d, scale, chunk,
                                           int(n_splits), po, pl, stream);
  if (st != ATTN_OK) return st;
  return decode_combine_dispatch(po, pl, B * Hq, int(n_splits), d, o, lse, stream);
}
