// The C ABI (include/attn.h): argument checks, TMA descriptors, launches, the device error word.
#include <cudaTypedefs.h>
#include <math.h>
#include <atomic>
#include <mutex>

#include "attn_internal.h"
#include "sm100_ptx.cuh"

namespace attn {

// One CTA waits on a barrier that is initialised for one arrival and never receives it.
__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);
  __syncthreads();
}

// A cluster of two CTAs: each CTA's thread 0 waits (bounded, cluster-scope acquire) on its own
// mbarrier, after arriving on the other CTA's through its shared::cluster address when cross_arrive
// is set (the hand-off the prefill's CTA pairs use); without it nothing completes either barrier and
// both waits run out. Both CTAs meet at the cluster barrier before exiting.
__global__ void pair_wait_selftest_kernel(unsigned long long limit_ns, int cross_arrive) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  cluster_sync();
  if (threadIdx.x == 0) {
    if (cross_arrive) mbar_arrive_cluster(mapa_shared(&bar, rank ^ 1u));
    mbar_wait_cluster(&bar, 0, &abort_flag, limit_ns);
  }
  __syncthreads();
  cluster_sync();
}

// 2^x through the FMA-pipe polynomial (exp2_poly2), two values per thread, for checking it against
// the exact function.
__global__ void exp2_poly_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int pairs = (n + 1) / 2;
  for (int p = blockIdx.x * blockDim.x + threadIdx.x; p < pairs; p += gridDim.x * blockDim.x) {
    const int i = 2 * p;
    const bool two = i + 1 < n;
    const float2 r = exp2_poly2(make_float2(x[i], two ? x[i + 1] : 0.f));
    y[i] = r.x;
    if (two) y[i + 1] = r.y;
  }
}

// ---- driver entry point for cuTensorMapEncodeTiled (no link-time dependency on libcuda) ----
static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A 4-d tiled TMA map: dims[0] innermost (contiguous), dims[i] elements of elem_bytes each, dense
// strides; box[] elements per dimension; swizzle 128, 64 or 0 bytes.
static bool encode_map_uncached(CUtensorMap* map, const void* base, int elem_bytes, const long long* dims,
                                const int* box, unsigned swizzle_bytes) {
  auto fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t gd[4] = {cuuint64_t(dims[0]), cuuint64_t(dims[1]), cuuint64_t(dims[2]), cuuint64_t(dims[3])};
  const cuuint64_t gs[3] = {gd[0] * elem_bytes, gd[0] * gd[1] * elem_bytes, gd[0] * gd[1] * gd[2] * elem_bytes};
  const cuuint32_t bx[4] = {cuuint32_t(box[0]), cuuint32_t(box[1]), cuuint32_t(box[2]), cuuint32_t(box[3])};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUtensorMapDataType dt = elem_bytes == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                   : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUresult r = fn(map, dt, 4, const_cast<void*>(base), gd, gs, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {
// Recently encoded tensor maps, replaced round robin. Every field that enters the encoding is part
// of the key, so a hit returns exactly the map the encoder would produce.
struct MapKey {
  const void* base;
  int elem_bytes;
  long long dims[4];
  int box[4];
  unsigned swizzle;
  bool operator==(const MapKey& o) const {
    if (base != o.base || elem_bytes != o.elem_bytes || swizzle != o.swizzle) return false;
    for (int i = 0; i < 4; ++i)
      if (dims[i] != o.dims[i] || box[i] != o.box[i]) return false;
    return true;
  }
};
constexpr int kMapCacheSize = 64;
struct MapCache {
  std::mutex mu;
  MapKey key[kMapCacheSize];
  CUtensorMap map[kMapCacheSize];
  bool used[kMapCacheSize] = {};
  int next = 0;
};
MapCache& map_cache() {
  static MapCache c;
  return c;
}
}  // namespace

bool encode_map(CUtensorMap* map, const void* base, int elem_bytes, const long long* dims, const int* box,
                unsigned swizzle_bytes) {
  MapKey k{base, elem_bytes, {dims[0], dims[1], dims[2], dims[3]}, {box[0], box[1], box[2], box[3]}, swizzle_bytes};
  MapCache& c = map_cache();
  std::lock_guard<std::mutex> lock(c.mu);
  for (int i = 0; i < kMapCacheSize; ++i) {
    if (c.used[i] && c.key[i] == k) {
      *map = c.map[i];
      return true;
    }
  }
  if (!encode_map_uncached(map, base, elem_bytes, dims, box, swizzle_bytes)) return false;
  const int slot = c.next;
  c.next = (c.next + 1) % kMapCacheSize;
  c.key[slot] = k;
  c.map[slot] = *map;
  c.used[slot] = true;
  return true;
}

bool encode_tile_map(CUtensorMap* map, const void* base, int d, int heads, int rows, int outer, int box_cols,
                     int box_rows, unsigned swizzle_bytes) {
  const long long dims[4] = {d, heads, rows, outer};
  const int box[4] = {box_cols, 1, box_rows, 1};
  return encode_map(map, base, 2, dims, box, swizzle_bytes);
}

namespace {
std::mutex g_attr_mu;
// (function, device) -> dynamic shared memory bytes the function has been opted into
struct AttrEntry {
  const void* func;
  int dev;
  int bytes;
};
AttrEntry g_attr[512];
int g_attr_n = 0;
std::atomic<int> g_sm_count[kMaxDevices];
}  // namespace

cudaError_t ensure_dyn_smem(const void* func, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  int i = 0;
  for (; i < g_attr_n; ++i)
    if (g_attr[i].func == func && g_attr[i].dev == dev) break;
  if (i < g_attr_n && g_attr[i].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (i == g_attr_n) {
    if (g_attr_n == int(sizeof(g_attr) / sizeof(g_attr[0]))) return cudaSuccess;  // table full: set every time
    g_attr[g_attr_n++] = AttrEntry{func, dev, bytes};
  } else {
    g_attr[i].bytes = bytes;
  }
  return cudaSuccess;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < kMaxDevices) {
    const int cached = g_sm_count[dev].load(std::memory_order_relaxed);
    if (cached > 0) return cached;
  }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

namespace {
// per device: the kernel the pair count was taken for, and the count
struct PairEntry {
  std::atomic<const void*> func{nullptr};
  std::atomic<int> pairs{0};
};
PairEntry g_pairs[kMaxDevices];
}  // namespace

int max_pairs(const void* func, int threads, int smem_bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  const bool cacheable = dev >= 0 && dev < kMaxDevices;
  if (cacheable && g_pairs[dev].func.load(std::memory_order_acquire) == func) {
    const int cached = g_pairs[dev].pairs.load(std::memory_order_relaxed);
    if (cached > 0) return cached;
  }
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.gridDim = dim3(2);
  lc.blockDim = dim3(threads);
  lc.dynamicSmemBytes = smem_bytes;
  lc.attrs = at;
  lc.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, func, &lc) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  if (n <= 0) return -1;
  if (cacheable) {
    g_pairs[dev].pairs.store(n, std::memory_order_relaxed);
    g_pairs[dev].func.store(func, std::memory_order_release);
  }
  return n;
}

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace attn

using namespace attn;

extern "C" {

attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                       int Nq, int Nkv, int d, float scale, int causal, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!is_aligned16(q) || !is_aligned16(k) || !is_aligned16(v) || !is_aligned16(o) || !is_aligned16(lse))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  if (d != 32 && d != 64 && d != 128 && d != 256) return ATTN_ERR_UNSUPPORTED;
  return fwd_dispatch(q, k, v, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, causal, stream);
}

attn_status_t attn_fp8_quantize(const void* x, const float* signs, void* codes, float* amax, int B, int N, int H,
                                int d, int transpose, cudaStream_t stream) {
  if (!x || !codes || !amax) return ATTN_ERR_INVALID_ARG;
  if (!is_aligned16(x) || !is_aligned16(codes) || (reinterpret_cast<uintptr_t>(amax) & 3u) ||
      (reinterpret_cast<uintptr_t>(signs) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1 || (transpose != 0 && transpose != 1)) return ATTN_ERR_INVALID_ARG;
  if (transpose && (N % 16) != 0) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * H > 65535) return ATTN_ERR_UNSUPPORTED;  // grid y
  return fp8_quantize_dispatch(x, signs, codes, amax, B, N, H, transpose, stream);
}

attn_status_t attn_fwd_fp8(const void* q8, const void* k8, const void* vt8, const float* amax_q, const float* amax_k,
                           const float* amax_v, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nkv, int d,
                           float scale, int causal, cudaStream_t stream) {
  if (!q8 || !k8 || !vt8 || !amax_q || !amax_k || !amax_v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!is_aligned16(q8) || !is_aligned16(k8) || !is_aligned16(vt8) || !is_aligned16(o) || !is_aligned16(lse) ||
      ((reinterpret_cast<uintptr_t>(amax_q) | reinterpret_cast<uintptr_t>(amax_k) |
        reinterpret_cast<uintptr_t>(amax_v)) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  if (Nkv % 16 != 0) return ATTN_ERR_INVALID_ARG;  // rows of the transposed V start on 16-byte boundaries
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  return fwd_fp8_dispatch(q8, k8, vt8, amax_q, amax_k, amax_v, o, lse, B, Hq, Hkv, Nq, Nkv, d, scale, causal, stream);
}

size_t attn_bwd_workspace_bytes(int B, int Hq, int Nq, int d) {
  if (B < 1 || Hq < 1 || Nq < 1 || d < 1) return 0;
  return bwd_workspace(B, Hq, Nq, d);
}

attn_status_t attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                       void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Nq, int Nkv, int d, float scale,
                       int causal, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, dout, dq, dk, dv};
  for (const void* p : ptrs)
    if (!is_aligned16(p)) return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(lse) & 3u) return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nkv < 1 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) ||
      workspace_bytes < bwd_workspace(B, Hq, Nq, d))
    return ATTN_ERR_WORKSPACE;
  return bwd_dispatch(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Nq, Nkv, scale, causal, workspace, stream);
}

int attn_decode_default_chunk(int B, int Hkv, int Nkv_cap) {
  if (B < 1 || Hkv < 1 || Nkv_cap < 1) return 0;
  return decode_default_chunk(B, Hkv, Nkv_cap);
}

size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int Nkv_cap, int chunk) {
  if (B < 1 || Hq < 1 || Hkv < 1 || d < 1 || Nkv_cap < 1 || chunk < 0 || Hq % Hkv) return 0;
  if (chunk == 0) chunk = decode_default_chunk(B, Hkv, Nkv_cap);
  return decode_workspace(B, Hq, d, Nkv_cap, chunk);
}

attn_status_t attn_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens,
                                  int Nkv_cap, void* o, float* lse, int B, int Hq, int Hkv, int d, float scale,
                                  int chunk, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !k_cache || !v_cache || !kv_lens || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!is_aligned16(q) || !is_aligned16(k_cache) || !is_aligned16(v_cache) || !is_aligned16(o) || !is_aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(kv_lens) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nkv_cap < 1 || Hq % Hkv != 0 || chunk < 0 || (chunk % 64) != 0)
    return ATTN_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return ATTN_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if ((d != 32 && d != 64 && d != 128 && d != 256) || (G != 1 && G != 2 && G != 4 && G != 8))
    return ATTN_ERR_UNSUPPORTED;
  if (chunk == 0) chunk = decode_default_chunk(B, Hkv, Nkv_cap);
  const long long n_splits = (Nkv_cap + (long long)chunk - 1) / chunk;
  // every size check comes before the split kernel is enqueued, so a refused call leaves nothing behind
  if (Hkv > 65535 || B > 65535 || !combine_fits(n_splits)) return ATTN_ERR_UNSUPPORTED;
  const size_t need = decode_workspace(B, Hq, d, Nkv_cap, chunk);
  if (workspace == nullptr || !is_aligned16(workspace) || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  float* po = static_cast<float*>(workspace);
  const size_t po_bytes = size_t(B) * Hq * n_splits * d * sizeof(float);
  float* pl = reinterpret_cast<float*>(static_cast<char*>(workspace) + ((po_bytes + 255) / 256) * 256);
  attn_status_t st =
      decode_split_dispatch(q, k_cache, v_cache, kv_lens, Nkv_cap, B, Hq, Hkv, d, scale, chunk, int(n_splits), po,
                            pl, stream);
  if (st != ATTN_OK) return st;
  return decode_combine_dispatch(po, pl, B * Hq, int(n_splits), d, o, lse, stream);
}

attn_status_t attn_decode_combine(const float* part_o, const float* part_lse, int rows, int n_splits, int d,
                                  void* o, float* lse, cudaStream_t stream) {
  if (!part_o || !part_lse || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!is_aligned16(part_o) || !is_aligned16(o) || (reinterpret_cast<uintptr_t>(part_lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return ATTN_ERR_INVALID_ARG;
  if (rows < 1 || n_splits < 1) return ATTN_ERR_INVALID_ARG;
  if ((d != 32 && d != 64 && d != 128 && d != 256) || !combine_fits(n_splits)) return ATTN_ERR_UNSUPPORTED;
  return decode_combine_dispatch(part_o, part_lse, rows, n_splits, d, o, lse, stream);
}

attn_status_t attn_get_last_error(void) {
  unsigned int word = 0;
  const unsigned int zero = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return ATTN_ERR_CUDA;
  if (word & kErrTimeoutBit) return ATTN_ERR_TIMEOUT;
  if (word & kErrSmemAlignBit) return ATTN_ERR_CUDA;
  if (word & kErrBadLengthBit) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

const char* attn_status_string(attn_status_t s) {
  switch (s) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case ATTN_ERR_WORKSPACE: return "decode workspace missing or too small";
    case ATTN_ERR_CUDA: return "CUDA call failed";
    case ATTN_ERR_TIMEOUT: return "a kernel pipeline wait timed out";
  }
  return "unknown status";
}

const char* attn_kernel_name(int which) {
  switch (which) {
    case 0: return "attn::attn_fwd_kernel<D, F8, PAIR>";
    case 1: return "attn::decode_split_tc_kernel<D,G> (d <= 128), attn::decode_split_kernel<D,G> (d = 256)";
    case 2: return "attn::decode_combine_kernel<D>";
    case 3: return "attn::attn_bwd_pre_kernel, attn::attn_bwd_kernel, attn::attn_bwd_post_kernel";
  }
  return nullptr;
}

attn_status_t attn_selftest_bounded_wait(unsigned int limit_us, cudaStream_t stream) {
  if (limit_us == 0 || limit_us > 10000000u) return ATTN_ERR_INVALID_ARG;
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(1000ull * limit_us);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

attn_status_t attn_selftest_pair_wait(unsigned int limit_us, int cross_arrive, cudaStream_t stream) {
  if (limit_us == 0 || limit_us > 10000000u || (cross_arrive != 0 && cross_arrive != 1)) return ATTN_ERR_INVALID_ARG;
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  lc.gridDim = dim3(2);
  lc.blockDim = dim3(32);
  lc.stream = stream;
  lc.attrs = at;
  lc.numAttrs = 1;
  if (cudaLaunchKernelEx(&lc, pair_wait_selftest_kernel, 1000ull * limit_us, cross_arrive) != cudaSuccess) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

attn_status_t attn_selftest_exp2_poly(const float* x, float* y, int n, cudaStream_t stream) {
  if (!x || !y || n < 1) return ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 3u) || (reinterpret_cast<uintptr_t>(y) & 3u)) return ATTN_ERR_INVALID_ARG;
  const long long pairs = (n + 1ll) / 2;
  const int grid = int(pairs / 256 + 1 < 4096 ? pairs / 256 + 1 : 4096);
  exp2_poly_selftest_kernel<<<grid, 256, 0, stream>>>(x, y, n);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : (cudaGetLastError(), ATTN_ERR_CUDA);
}

}  // extern "C"
