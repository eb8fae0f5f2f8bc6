// kmip_abi.cu -- the C ABI of libkmip (declared in include/kmip.h): argument
// checks, the per-device status word, the library's scratch pool and kernel
// dispatch.
#include <math.h>

#include <mutex>

#include "kmip_internal.h"

#if defined(__GNUC__)
#define KMIP_EXPORT extern "C" __attribute__((visibility("default")))
#else
#define KMIP_EXPORT extern "C"
#endif

namespace kmip {

// Per-device status word: the first device-side error since the last
// kmip_get_status() call (0 = none).
__device__ int g_status;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
cudaMemPool_t g_pool[kMaxDevices] = {};
uint64_t g_pool_keep[kMaxDevices] = {};

}  // namespace

// Device address of g_status on the current device (resolved once per device).
int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

namespace {

bool supported_d(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

}  // namespace

kmip_status_t check_common(int64_t N, int H, int d, int k, float scale, kmip_dtype_t dtype) {
  if (N < 0 || N > INT32_MAX || H < 1 || k < 1 || !(scale > 0.f) || !isfinite(scale))
    return KMIP_ERR_INVALID_ARG;
  if (dtype != KMIP_BF16 && dtype != KMIP_F32) return KMIP_ERR_INVALID_ARG;
  if (H > 64 || k > 64 || !supported_d(d)) return KMIP_ERR_UNSUPPORTED;
  if ((int64_t)N * H * (int64_t)(d > k ? d : k) > ((int64_t)1 << 40))
    return KMIP_ERR_UNSUPPORTED;
  return KMIP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The library's own stream-ordered memory pool on the current device.  It
// keeps, between calls, the most memory it has held (its release threshold
// follows its largest reservation), so a loop of calls maps device memory
// once instead of on every call, and it leaves the device's default pool,
// which other code in the process may use, alone.
cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return cudaErrorInvalidDevice;
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_pool[dev]) {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.handleTypes = cudaMemHandleTypeNone;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      const cudaError_t e = cudaMemPoolCreate(&g_pool[dev], &props);
      if (e != cudaSuccess) {
        g_pool[dev] = nullptr;
        cudaGetLastError();
        return e;
      }
    }
    pool = g_pool[dev];
  }
  const cudaError_t e = cudaMallocFromPoolAsync(p, bytes, pool, stream);
  if (e == cudaSuccess) {
    // keep all that the pool holds now: trimming to the request alone would
    // still return the last, partly used block of the pool's reservation
    std::lock_guard<std::mutex> lock(g_mu);
    uint64_t r = 0;
    if (cudaMemPoolGetAttribute(pool, cudaMemPoolAttrReservedMemCurrent, &r) == cudaSuccess &&
        r > g_pool_keep[dev] &&
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &r) == cudaSuccess)
      g_pool_keep[dev] = r;
    cudaGetLastError();
  }
  return e;
}

// Reserved and high-water bytes of the library's pool on the current device
// (zeros before its first allocation).
cudaError_t scratch_usage(uint64_t* reserved, uint64_t* used_high, bool reset_high) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  uint64_t r = 0, h = 0;
  cudaMemPool_t pool = g_pool[dev];
  if (pool) {
    if (reset_high) {
      uint64_t zero = 0;
      if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &zero) != cudaSuccess)
        return cudaGetLastError();
    }
    if (cudaMemPoolGetAttribute(pool, cudaMemPoolAttrReservedMemCurrent, &r) != cudaSuccess ||
        cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &h) != cudaSuccess)
      return cudaGetLastError();
  }
  if (reserved) *reserved = r;
  if (used_high) *used_high = h;
  return cudaSuccess;
}

// Trim the library's pool on the current device and reset what it keeps.
cudaError_t scratch_trim() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaMemPool_t pool = g_pool[dev];
  if (!pool) return cudaSuccess;
  uint64_t zero = 0;
  cudaError_t e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &zero);
  if (e == cudaSuccess) e = cudaMemPoolTrimTo(pool, 0);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e;
  }
  g_pool_keep[dev] = 0;
  return cudaSuccess;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_sm_count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

}  // namespace kmip

using namespace kmip;

namespace {

// The forward of kmip_attn_fwd and kmip_attn_fwd_diag (lse_all = nullptr:
// no all-key diagnostics).
kmip_status_t attn_fwd_impl(const void* Q, const void* K, const void* V,
                            const int32_t* graph_offsets, int64_t N, int H, int d, int k,
                            float scale, void* out, int32_t* idx, float* lse, float* lse_all,
                            kmip_stream_t stream_, int num_graphs, kmip_dtype_t dtype) {
  kmip_status_t st = check_common(N, H, d, k, scale, dtype);
  if (st != KMIP_OK) return st;
  if (graph_offsets && num_graphs < 1) return KMIP_ERR_INVALID_ARG;
  if (N == 0) return KMIP_OK;
  if (!Q || !K || !V || !out || !idx || !lse) return KMIP_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out))
    return KMIP_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  int* status = status_ptr();
  if (!status) return KMIP_ERR_CUDA;

  const bool tc = dtype == KMIP_BF16 && fwd_tc_supported(d, k);
  const int qpi = tc ? kTcQueries : kSimtQueries;
  const int G = graph_offsets ? num_graphs : 1;
  const int64_t max_items = max_work_items(N, G, qpi);
  if (max_items * H > INT32_MAX) return KMIP_ERR_UNSUPPORTED;

  // Work-list scratch: [count (16 B)] [items], stream-ordered.
  void* scratch = nullptr;
  const size_t bytes = 16 + sizeof(WorkItem) * (size_t)max_items;
  if (scratch_alloc(&scratch, bytes, stream) != cudaSuccess) {
    cudaGetLastError();
    return KMIP_ERR_CUDA;
  }
  int* count = static_cast<int*>(scratch);
  WorkItem* items = reinterpret_cast<WorkItem*>(static_cast<char*>(scratch) + 16);

  cudaError_t e = launch_worklist(graph_offsets, G, (int)N, qpi, items, count, (int)max_items,
                                  status, stream);
  if (e == cudaSuccess) {
    FwdArgs a{Q, K, V, (int)N, H, d, k, scale, out, idx, lse, items, count, (int)max_items, status,
              lse_all};
    e = tc ? launch_fwd_tc(a, stream) : launch_fwd_simt(dtype, a, stream);
  }
  cudaError_t ef = cudaFreeAsync(scratch, stream);
  if (e != cudaSuccess || ef != cudaSuccess) {
    cudaGetLastError();
    return KMIP_ERR_CUDA;
  }
  return KMIP_OK;
}

}  // namespace

KMIP_EXPORT kmip_status_t kmip_attn_fwd(const void* Q, const void* K, const void* V,
                                        const int32_t* graph_offsets, int64_t N, int H, int d,
                                        int k, float scale, void* out, int32_t* idx, float* lse,
                                        kmip_stream_t stream, int num_graphs,
                                        kmip_dtype_t dtype) {
  return attn_fwd_impl(Q, K, V, graph_offsets, N, H, d, k, scale, out, idx, lse, nullptr,
                       stream, num_graphs, dtype);
}

KMIP_EXPORT kmip_status_t kmip_attn_fwd_diag(const void* Q, const void* K, const void* V,
                                             const int32_t* graph_offsets, int64_t N, int H,
                                             int d, int k, float scale, void* out, int32_t* idx,
                                             float* lse, float* lse_all, kmip_stream_t stream,
                                             int num_graphs, kmip_dtype_t dtype) {
  if (N > 0 && !lse_all) return KMIP_ERR_INVALID_ARG;
  return attn_fwd_impl(Q, K, V, graph_offsets, N, H, d, k, scale, out, idx, lse, lse_all,
                       stream, num_graphs, dtype);
}

namespace {

kmip_status_t attn_bwd_impl(const void* dOut, const void* Q, const void* K, const void* V,
                            const int32_t* idx, const float* lse, float* dQ, float* dK,
                            float* dV, kmip_stream_t stream_, int64_t N, int H, int d, int k,
                            float scale, kmip_dtype_t dtype, bool deterministic) {
  kmip_status_t st = check_common(N, H, d, k, scale, dtype);
  if (st != KMIP_OK) return st;
  if (N == 0) return KMIP_OK;
  if (!dOut || !Q || !K || !V || !idx || !lse || !dQ || !dK || !dV) return KMIP_ERR_INVALID_ARG;
  if (!aligned16(dOut) || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dQ) ||
      !aligned16(dK) || !aligned16(dV))
    return KMIP_ERR_INVALID_ARG;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  int* status = status_ptr();
  if (!status) return KMIP_ERR_CUDA;
  BwdArgs a{dOut, Q, K, V, idx, lse, dQ, dK, dV, (int)N, H, d, k, scale, status};
  cudaError_t e;
  if (deterministic) {
    e = launch_bwd_deterministic(dtype, a, stream);
    if (e == cudaErrorNotSupported) {
      cudaGetLastError();
      return KMIP_ERR_UNSUPPORTED;
    }
  } else {
    const size_t bytes = sizeof(float) * (size_t)N * H * d;
    e = cudaMemsetAsync(dK, 0, bytes, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dV, 0, bytes, stream);
    if (e == cudaSuccess) e = launch_bwd(dtype, a, stream);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return KMIP_ERR_CUDA;
  }
  return KMIP_OK;
}

}  // namespace

KMIP_EXPORT kmip_status_t kmip_attn_bwd(const void* dOut, const void* Q, const void* K,
                                        const void* V, const int32_t* idx, const float* lse,
                                        float* dQ, float* dK, float* dV, kmip_stream_t stream,
                                        int64_t N, int H, int d, int k, float scale,
                                        kmip_dtype_t dtype) {
  return attn_bwd_impl(dOut, Q, K, V, idx, lse, dQ, dK, dV, stream, N, H, d, k, scale, dtype,
                       false);
}

KMIP_EXPORT kmip_status_t kmip_attn_bwd_deterministic(const void* dOut, const void* Q,
                                                      const void* K, const void* V,
                                                      const int32_t* idx, const float* lse,
                                                      float* dQ, float* dK, float* dV,
                                                      kmip_stream_t stream, int64_t N, int H,
                                                      int d, int k, float scale,
                                                      kmip_dtype_t dtype) {
  return attn_bwd_impl(dOut, Q, K, V, idx, lse, dQ, dK, dV, stream, N, H, d, k, scale, dtype,
                       true);
}

KMIP_EXPORT kmip_status_t kmip_attn_gather(const void* Q, const void* K, const void* V,
                                           const int32_t* idx, int64_t N, int H, int d, int k,
                                           float scale, void* out, float* lse,
                                           kmip_stream_t stream_, kmip_dtype_t dtype) {
  kmip_status_t st = check_common(N, H, d, k, scale, dtype);
  if (st != KMIP_OK) return st;
  if (N == 0) return KMIP_OK;
  if (!Q || !K || !V || !idx || !out || !lse) return KMIP_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out))
    return KMIP_ERR_INVALID_ARG;
  int* status = status_ptr();
  if (!status) return KMIP_ERR_CUDA;
  GatherArgs a{Q, K, V, idx, (int)N, H, d, k, scale, out, lse, status};
  if (launch_gather(dtype, a, static_cast<cudaStream_t>(stream_)) != cudaSuccess) {
    cudaGetLastError();
    return KMIP_ERR_CUDA;
  }
  return KMIP_OK;
}

KMIP_EXPORT kmip_status_t kmip_get_status(kmip_stream_t stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return KMIP_ERR_CUDA;
  }
  int* status = status_ptr();
  if (!status) return KMIP_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return KMIP_ERR_CUDA;
  if (h != 0) {
    const int zero = 0;
    if (cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return KMIP_ERR_CUDA;
  }
  return static_cast<kmip_status_t>(h);
}

KMIP_EXPORT kmip_status_t kmip_scratch_usage(uint64_t* reserved, uint64_t* used_high,
                                             int reset_high) {
  return kmip::scratch_usage(reserved, used_high, reset_high != 0) == cudaSuccess ? KMIP_OK
                                                                                  : KMIP_ERR_CUDA;
}

KMIP_EXPORT kmip_status_t kmip_scratch_trim(void) {
  return kmip::scratch_trim() == cudaSuccess ? KMIP_OK : KMIP_ERR_CUDA;
}

KMIP_EXPORT const char* kmip_error_string(kmip_status_t s) {
  switch (s) {
    case KMIP_OK: return "KMIP_OK: success";
    case KMIP_ERR_INVALID_ARG: return "KMIP_ERR_INVALID_ARG: invalid argument";
    case KMIP_ERR_UNSUPPORTED: return "KMIP_ERR_UNSUPPORTED: shape outside the supported set";
    case KMIP_ERR_CUDA: return "KMIP_ERR_CUDA: CUDA runtime error";
    case KMIP_ERR_BAD_OFFSETS: return "KMIP_ERR_BAD_OFFSETS: malformed graph_offsets";
    case KMIP_ERR_TIMEOUT: return "KMIP_ERR_TIMEOUT: a device pipeline wait ran out";
    case KMIP_ERR_BAD_INDEX: return "KMIP_ERR_BAD_INDEX: idx entry outside [-1, N)";
    case KMIP_ERR_SCRATCH_LIMIT:
      return "KMIP_ERR_SCRATCH_LIMIT: work list exceeds the no-allocation entry point's fixed array";
  }
  return "KMIP_ERR_UNKNOWN: unknown status code";
}

KMIP_EXPORT int kmip_fwd_path(int d, int k, kmip_dtype_t dtype) {
  if (check_common(1, 1, d, k, 1.0f, dtype) != KMIP_OK) return -1;
  return dtype == KMIP_BF16 && fwd_tc_supported(d, k) ? 1 : 0;
}

KMIP_EXPORT int kmip_version(void) { return 200; }
