// kmip_gather.cu -- attention over given key sets (the softmax and V-gather
// stage of k-MIP attention on its own).
//
// k-Maximum Inner Product Attention for Graph Transformers ... (Abstract):
// once a query's k keys are chosen, the layer is ordinary softmax attention
// over them.  kmip_attn_gather takes the chosen sets (idx, as kmip_attn_fwd
// writes them) and computes, per (query, head),
//   s_j = q . k_j,  lse = log sum_j exp(scale s_j),  out = sum_j p_j V_j
// for a caller that keeps a selection across steps, and as the gather stage
// measured by itself.  One warp per (query, head); lanes split the d columns
// in 16-byte slices, 32 / (d / slice) kept rows per warp instruction, with
// coalesced 16-byte loads of the K and V rows.
#include <math.h>

#include "kmip_internal.h"

namespace kmip {
namespace {

constexpr int kWarps = 8;

template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
gather_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
              const int32_t* __restrict__ idx, int N, int H, int k, float scale,
              T* __restrict__ out, float* __restrict__ lse, int* status) {
  using VT = Vec<T>;
  constexpr int VN = VT::N;
  constexpr int LPR = D / VN;
  constexpr int RPP = 32 / LPR;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rs = lane / LPR, cs = (lane % LPR) * VN;
  const int64_t HD = (int64_t)H * D;
  const int64_t pairs = (int64_t)N * H;
  const int npass = (k + RPP - 1) / RPP;
  for (int64_t pr = (int64_t)blockIdx.x * kWarps + warp; pr < pairs;
       pr += (int64_t)gridDim.x * kWarps) {
    const int64_t base = pr * D;
    const int64_t hoff = base % HD;
    float q[VN];
    VT::load(Q + base + cs, q);
    const int32_t* ir = idx + pr * k;
    // online softmax over the kept keys: running max m, sum l, output o
    float m = -INFINITY, l = 0.f, o[VN];
#pragma unroll
    for (int u = 0; u < VN; ++u) o[u] = 0.f;
    for (int ps = 0; ps < npass; ++ps) {
      const int t = ps * RPP + rs;
      int j = t < k ? ir[t] : -1;
      if (j >= N || j < -1) {
        record_status(status, KMIP_ERR_BAD_INDEX);
        j = -1;
      }
      float s = 0.f, vv[VN];
#pragma unroll
      for (int u = 0; u < VN; ++u) vv[u] = 0.f;
      if (j >= 0) {
        float kv[VN];
        VT::load(K + (int64_t)j * HD + hoff + cs, kv);
        VT::load(V + (int64_t)j * HD + hoff + cs, vv);
#pragma unroll
        for (int u = 0; u < VN; ++u) s = fmaf(q[u], kv[u], s);
      }
#pragma unroll
      for (int o2 = 1; o2 < LPR; o2 <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o2);
      const float z = j >= 0 ? scale * s : -INFINITY;
      // this lane group's row joins the group's running softmax
      const float mn = fmaxf(m, z);
      if (mn > -INFINITY) {
        const float a = expf(m - mn), b = expf(z - mn);
        l = l * a + b;
#pragma unroll
        for (int u = 0; u < VN; ++u) o[u] = fmaf(o[u], a, b * vv[u]);
        m = mn;
      }
    }
    // combine the RPP lane groups (fixed shuffle tree)
#pragma unroll
    for (int o2 = LPR; o2 < 32; o2 <<= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o2);
      const float l2 = __shfl_xor_sync(0xffffffffu, l, o2);
      const float mn = fmaxf(m, m2);
      const float a = mn > -INFINITY ? expf(m - mn) : 0.f;
      const float b = mn > -INFINITY ? expf(m2 - mn) : 0.f;
#pragma unroll
      for (int u = 0; u < VN; ++u) {
        const float other = __shfl_xor_sync(0xffffffffu, o[u], o2);
        o[u] = o[u] * a + other * b;
      }
      l = l * a + l2 * b;
      m = mn;
    }
    if (rs == 0) {
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float r[VN];
#pragma unroll
      for (int u = 0; u < VN; ++u) r[u] = o[u] * inv;
      VT::store(out + base + cs, r);
      if (lane == 0) lse[pr] = l > 0.f ? m + logf(l) : -INFINITY;
    }
  }
}

template <typename T, int D>
cudaError_t launch_typed(const GatherArgs& a, cudaStream_t stream) {
  const int64_t pairs = (int64_t)a.N * a.H;
  int64_t blocks = (pairs + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)device_sm_count() * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  gather_kernel<T, D><<<(int)blocks, kWarps * 32, 0, stream>>>(
      static_cast<const T*>(a.Q), static_cast<const T*>(a.K), static_cast<const T*>(a.V), a.idx,
      a.N, a.H, a.k, a.scale, static_cast<T*>(a.out), a.lse, a.status);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const GatherArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 16: return launch_typed<T, 16>(a, stream);
    case 32: return launch_typed<T, 32>(a, stream);
    case 64: return launch_typed<T, 64>(a, stream);
    case 128: return launch_typed<T, 128>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_gather(kmip_dtype_t dtype, const GatherArgs& a, cudaStream_t stream) {
  if (dtype == KMIP_BF16) return launch_t<__nv_bfloat16>(a, stream);
  if (dtype == KMIP_F32) return launch_t<float>(a, stream);
  return cudaErrorNotSupported;
}

}  // namespace kmip
