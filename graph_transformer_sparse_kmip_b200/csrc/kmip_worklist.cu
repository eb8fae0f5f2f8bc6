// kmip_worklist.cu -- segment work list for the forward kernels.
//
// Batched small graphs form a block-diagonal node set (the GraphGPS
// experiments on batched small-graph datasets, k-Maximum Inner Product
// Attention for Graph Transformers ..., Tables 8 and 9): a query only scores
// keys of its own graph.  This kernel validates graph_offsets and cuts each
// graph into items of `queries_per_item` consecutive queries, each carrying
// its graph's key range, so the forward kernels never touch a key tile
// outside a query's graph.
#include "kmip_internal.h"

namespace kmip {
namespace {

constexpr int kThreads = 1024;

// Block-wide exclusive scan of one int per thread; returns the block total.
__device__ int block_exclusive_scan(int v, int* excl, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  int base = warp ? warp_sums[warp - 1] : 0;
  *excl = base + x - v;
  int total = warp_sums[31];
  __syncthreads();  // warp_sums is reused by the next call
  return total;
}

__global__ void __launch_bounds__(kThreads)
worklist_kernel(const int32_t* __restrict__ offsets, int G, int N, int qpi,
                WorkItem* __restrict__ items, int* __restrict__ count, int max_items,
                int* status) {
  __shared__ int warp_sums[32];
  // 1. validate: o[0] = 0, o[G] = N, non-decreasing.
  int bad = 0;
  if (offsets) {
    if (threadIdx.x == 0) bad = (offsets[0] != 0) || (offsets[G] != N);
    for (int g = threadIdx.x; g < G; g += kThreads)
      bad |= offsets[g + 1] < offsets[g];
  }
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0) {
      *count = 0;
      record_status(status, KMIP_ERR_BAD_OFFSETS);
    }
    return;
  }
  // 2. items of each graph, placed by an exclusive scan of per-graph counts.
  int carry = 0;
  for (int g0 = 0; g0 < G; g0 += kThreads) {
    int g = g0 + threadIdx.x;
    int j0 = 0, j1 = 0, nb = 0;
    if (g < G) {
      j0 = offsets ? offsets[g] : 0;
      j1 = offsets ? offsets[g + 1] : N;
      nb = (j1 - j0 + qpi - 1) / qpi;
    }
    int excl;
    int total = block_exclusive_scan(nb, &excl, warp_sums);
    for (int b = 0; b < nb; ++b) {
      int t = carry + excl + b;
      if (t < max_items) {
        int q0 = j0 + b * qpi;
        items[t] = WorkItem{q0, min(q0 + qpi, j1), j0, j1};
      }
    }
    carry += total;
  }
  if (threadIdx.x == 0) *count = min(carry, max_items);
}

}  // namespace

cudaError_t launch_worklist(const int32_t* offsets, int G, int N, int queries_per_item,
                            WorkItem* items, int* count, int max_items, int* status,
                            cudaStream_t stream) {
  worklist_kernel<<<1, kThreads, 0, stream>>>(offsets, offsets ? G : 1, N, queries_per_item,
                                              items, count, max_items, status);
  return cudaGetLastError();
}

}  // namespace kmip
