// kmip_internal.h -- host-side launchers shared between the C ABI
// (kmip_abi.cu) and the kernel translation units.  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kmip_common.cuh"

namespace kmip {

struct FwdArgs {
  const void* Q;
  const void* K;
  const void* V;
  int N, H, d, k;
  float scale;
  void* out;
  int32_t* idx;
  float* lse;
  const WorkItem* items;  // work list (device)
  const int* count;       // number of items (device)
  int max_items;          // host-side upper bound on *count
  int* status;            // device status word
  float* lse_all = nullptr;  // [N, H] log-sum-exp over every key, or nullptr
};

// Buffers of the deterministic backward (all device, E = N H k entries):
// per kept key its (p, scale dS) coefficients, its (key, head) bucket as a
// sort key (sentinel for padding) and its position in idx; per bucket the
// number of kept keys that point to it.
struct DetBuffers {
  float2* coef = nullptr;
  uint32_t* keys = nullptr;
  uint32_t* vals = nullptr;
  int* count = nullptr;
  uint32_t sentinel = 0;
};

struct BwdArgs {
  const void* dO;
  const void* Q;
  const void* K;
  const void* V;
  const int32_t* idx;
  const float* lse;
  float* dQ;
  float* dK;
  float* dV;
  int N, H, d, k;
  float scale;
  int* status;
  DetBuffers det = {};  // keys != nullptr: write coefficients instead of scattering
};

struct GatherArgs {
  const void* Q;
  const void* K;
  const void* V;
  const int32_t* idx;
  int N, H, d, k;
  float scale;
  void* out;
  float* lse;
  int* status;
};

// Queries per work item of each forward kernel (the tensor-core forward
// takes two 128-row Q tiles per item).
constexpr int kSimtQueries = 128;
constexpr int kTcQueries = 256;

// Upper bound on the number of work items for N nodes in G graphs.
inline int64_t max_work_items(int64_t N, int64_t G, int queries_per_item) {
  return (N + queries_per_item - 1) / queries_per_item + G;
}

cudaError_t launch_worklist(const int32_t* offsets, int G, int N, int queries_per_item,
                            WorkItem* items, int* count, int max_items, int* status,
                            cudaStream_t stream);

cudaError_t launch_fwd_simt(kmip_dtype_t dtype, const FwdArgs& a, cudaStream_t stream);

// tcgen05 forward (bf16).  Returns cudaErrorNotSupported when the shape is
// not covered by the tensor-core kernel.
cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t stream);
bool fwd_tc_supported(int d, int k);

cudaError_t launch_bwd(kmip_dtype_t dtype, const BwdArgs& a, cudaStream_t stream);

// Softmax and V gather over given key sets (kmip_gather.cu).
cudaError_t launch_gather(kmip_dtype_t dtype, const GatherArgs& a, cudaStream_t stream);

// Deterministic backward: coefficients, a stable sort of the kept keys by
// (key, head) and an in-order reduction per key (kmip_bwd_det.cu).  Takes
// its scratch from the library's pool (scratch_alloc).
cudaError_t launch_bwd_deterministic(kmip_dtype_t dtype, const BwdArgs& a, cudaStream_t stream);

int device_sm_count();

// Stream-ordered allocation from the library's own memory pool on the
// current device (kmip_abi.cu); free with cudaFreeAsync on the same stream.
cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t stream);
cudaError_t scratch_usage(uint64_t* reserved, uint64_t* used_high, bool reset_high);
cudaError_t scratch_trim();

// Per-device status word address (nullptr if it cannot be resolved).
int* status_ptr();

// Shared argument checks of the entry points (no device access).
kmip_status_t check_common(int64_t N, int H, int d, int k, float scale, kmip_dtype_t dtype);
bool aligned16(const void* p);

}  // namespace kmip
