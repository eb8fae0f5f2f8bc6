// kmip_noalloc.cu -- a forward entry point that allocates no device memory.
//
// kmip_attn_fwd takes its work list from the library's stream-ordered memory
// pool on every call.  Some callers cannot allow that: a framework whose own pool
// has reserved the GPU's memory up front, a process on a driver or
// virtualised device without stream-ordered memory pools, or a latency-
// critical loop that must not enter the allocator after start-up.
// kmip_attn_fwd_noalloc runs the same kernels with the work list placed in a
// fixed array in the library's own device image instead.
//
// That array is a file-scope __device__ variable: every GPU that loads the
// library holds it (kNoAllocBytes) until the process exits.  Its host-side
// name is only a stand-in for the symbol, so the device address is looked up
// with cudaGetSymbolAddress, once per device, with that device current, on
// the first call that runs on it.
//
// The array is shared by every call on a device and keeps the last call's
// contents.  Nothing in it needs to start at zero: the work-list kernel
// writes the item count and every item the forward kernel later reads.  Two
// calls whose work overlaps on the GPU (different streams, or host threads
// racing) would overwrite each other's work list; such calls must be ordered.
#include <mutex>

#include "kmip_internal.h"

#if defined(__GNUC__)
#define KMIP_EXPORT extern "C" __attribute__((visibility("default")))
#else
#define KMIP_EXPORT extern "C"
#endif

namespace kmip {
namespace {

// Largest work list this entry point accepts, in items.  One item covers up
// to 128 (fp32 path) or 256 (tensor-core path) consecutive queries of one
// graph and is shared by all heads, so a call needs at most
// ceil(N / 128 or 256) + num_graphs items.
constexpr int kNoAllocMaxItems = 65536;
constexpr size_t kNoAllocHeader = 256;  // item count, padded to keep items aligned
constexpr size_t kNoAllocBytes = kNoAllocHeader + sizeof(WorkItem) * kNoAllocMaxItems;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char* g_scratch_dev[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.
unsigned char* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_dev[dev]) {
    unsigned char* p = nullptr;
    if (cudaGetSymbolAddress((void**)&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_dev[dev] = p;
  }
  return g_scratch_dev[dev];
}

}  // namespace
}  // namespace kmip

using namespace kmip;

KMIP_EXPORT kmip_status_t kmip_attn_fwd_noalloc(const void* Q, const void* K, const void* V,
                                                const int32_t* graph_offsets, int64_t N, int H,
                                                int d, int k, float scale, void* out,
                                                int32_t* idx, float* lse, kmip_stream_t stream_,
                                                int num_graphs, kmip_dtype_t dtype) {
  kmip_status_t st = check_common(N, H, d, k, scale, dtype);
  if (st != KMIP_OK) return st;
  if (graph_offsets && num_graphs < 1) return KMIP_ERR_INVALID_ARG;
  if (N == 0) return KMIP_OK;
  if (!Q || !K || !V || !out || !idx || !lse) return KMIP_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out))
    return KMIP_ERR_INVALID_ARG;

  const bool tc = dtype == KMIP_BF16 && fwd_tc_supported(d, k);
  const int qpi = tc ? kTcQueries : kSimtQueries;
  const int G = graph_offsets ? num_graphs : 1;
  const int64_t max_items = max_work_items(N, G, qpi);
  if (max_items > kNoAllocMaxItems) return KMIP_ERR_SCRATCH_LIMIT;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  int* status = status_ptr();
  unsigned char* scratch = scratch_address();
  if (!status || !scratch) return KMIP_ERR_CUDA;
  int* count = reinterpret_cast<int*>(scratch);
  WorkItem* items = reinterpret_cast<WorkItem*>(scratch + kNoAllocHeader);

  cudaError_t e = launch_worklist(graph_offsets, G, (int)N, qpi, items, count, (int)max_items,
                                  status, stream);
  if (e == cudaSuccess) {
    FwdArgs a{Q, K, V, (int)N, H, d, k, scale, out, idx, lse, items, count, (int)max_items, status};
    e = tc ? launch_fwd_tc(a, stream) : launch_fwd_simt(dtype, a, stream);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return KMIP_ERR_CUDA;
  }
  return KMIP_OK;
}
