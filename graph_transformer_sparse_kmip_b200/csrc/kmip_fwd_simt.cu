// kmip_fwd_simt.cu -- forward k-MIP attention with fp32 FMA scoring.
//
// This is the path for fp32 inputs (scores by fp32 fused multiply-add, so
// the selection sees true fp32 inner products; tensor-core tf32 would round
// the inputs) and the reference-shaped path every other kernel is tested
// beside.  One thread owns one (query, head): it streams its graph's key
// tiles through shared memory, keeps a running top-k in shared memory with
// a register threshold (the k-th best score so far; a key is inserted only
// if it beats it), then applies the softmax over the kept scores and sums
// the kept V rows (k-Maximum Inner Product Attention for Graph Transformers
// ..., Abstract: top-k selection by inner product, then attention over the
// selected keys).
#include <math.h>

#include "kmip_internal.h"

namespace kmip {
namespace {

constexpr int kThreads = kSimtQueries;  // one query row per thread
constexpr int kKeyTile = 64;

// Sorted insertion (larger score first; an equal score stays behind the
// entries already present, which have smaller node indices because keys are
// visited in increasing index order).  Lists are column-major in shared
// memory: entry t of thread x lives at [t * kThreads + x].
__device__ __forceinline__ void topk_insert(float* ls, int* li, int& cnt, int k, float s, int j,
                                            float& thr) {
  int pos = cnt < k ? cnt++ : k - 1;
  const int x = threadIdx.x;
  while (pos > 0 && ls[(pos - 1) * kThreads + x] < s) {
    ls[pos * kThreads + x] = ls[(pos - 1) * kThreads + x];
    li[pos * kThreads + x] = li[(pos - 1) * kThreads + x];
    --pos;
  }
  ls[pos * kThreads + x] = s;
  li[pos * kThreads + x] = j;
  if (cnt == k) thr = ls[(k - 1) * kThreads + x];
}

template <typename T, int D, int KCAP, bool DIAG>
__global__ void __launch_bounds__(kThreads)
fwd_simt_kernel(const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
                const WorkItem* __restrict__ items, const int* __restrict__ count_ptr, int H,
                int k, float scale, T* __restrict__ out, int32_t* __restrict__ idx,
                float* __restrict__ lse, float* __restrict__ lse_all) {
  using VT = Vec<T>;
  constexpr int VN = VT::N;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* Ks = reinterpret_cast<float*>(smem_raw);          // [kKeyTile][D]
  float* ls = Ks + kKeyTile * D;                           // [KCAP][kThreads]
  int* li = reinterpret_cast<int*>(ls + KCAP * kThreads);  // [KCAP][kThreads]

  const int count = *count_ptr;
  const int64_t HD = (int64_t)H * D;
  for (int64_t w = blockIdx.x; w < (int64_t)H * count; w += gridDim.x) {
    const int h = (int)(w / count);
    const WorkItem it = items[w % count];
    const int i = it.q0 + threadIdx.x;
    const bool active = i < it.q1;

    float q[D];
    if (active) {
#pragma unroll
      for (int c = 0; c < D; c += VN) VT::load(Q + i * HD + h * D + c, q + c);
    }
    float thr = -INFINITY;
    int cnt = 0;
    // all-key diagnostics: running maximum and sum of exp2(c2 (s - max))
    const float c2 = scale * 1.4426950408889634f;
    float dmax = -INFINITY, dsum = 0.f;

    for (int jt = it.j0; jt < it.j1; jt += kKeyTile) {
      const int nt = min(kKeyTile, it.j1 - jt);
      __syncthreads();  // previous tile fully consumed
      for (int e = threadIdx.x; e < kKeyTile * (D / VN); e += kThreads) {
        const int r = e / (D / VN), c = (e % (D / VN)) * VN;
        float f[VN];
        if (r < nt) {
          VT::load(K + (int64_t)(jt + r) * HD + h * D + c, f);
        } else {
#pragma unroll
          for (int t = 0; t < VN; ++t) f[t] = 0.f;
        }
#pragma unroll
        for (int t = 0; t < VN; ++t) Ks[r * D + c + t] = f[t];
      }
      __syncthreads();
      if (active) {
        for (int r = 0; r < nt; ++r) {
          const float4* kr = reinterpret_cast<const float4*>(Ks + r * D);
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int c = 0; c < D / 4; c += 2) {
            float4 x = kr[c];
            a0 = fmaf(q[4 * c + 0], x.x, a0);
            a0 = fmaf(q[4 * c + 1], x.y, a0);
            a0 = fmaf(q[4 * c + 2], x.z, a0);
            a0 = fmaf(q[4 * c + 3], x.w, a0);
            float4 y = kr[c + 1];
            a1 = fmaf(q[4 * c + 4], y.x, a1);
            a1 = fmaf(q[4 * c + 5], y.y, a1);
            a1 = fmaf(q[4 * c + 6], y.z, a1);
            a1 = fmaf(q[4 * c + 7], y.w, a1);
          }
          const float s = a0 + a1;
          if (s > thr) topk_insert(ls, li, cnt, k, s, jt + r, thr);
          if constexpr (DIAG) {
            if (s > dmax) {
              dsum = dsum * exp2f((dmax - s) * c2) + 1.f;
              dmax = s;
            } else {
              dsum += exp2f((s - dmax) * c2);
            }
          }
        }
      }
    }

    if (active) {
      // Softmax over the kept scaled scores and the weighted sum of V rows.
      const int x = threadIdx.x;
      const int64_t row = (int64_t)i * H + h;
      const float m = scale * ls[x];
      float sum = 0.f;
      for (int t = 0; t < cnt; ++t) sum += expf(scale * ls[t * kThreads + x] - m);
      const float L = m + logf(sum);
      float o[D];
#pragma unroll
      for (int c = 0; c < D; ++c) o[c] = 0.f;
      for (int t = 0; t < cnt; ++t) {
        const float p = expf(scale * ls[t * kThreads + x] - L);
        const int j = li[t * kThreads + x];
#ifdef KMIP_DEBUG_BOUNDS
        if (j < it.j0 || j >= it.j1) continue;  // cannot happen: keys come from [j0, j1)
#endif
#pragma unroll
        for (int c = 0; c < D; c += VN) {
          float f[VN];
          VT::load(V + (int64_t)j * HD + h * D + c, f);
#pragma unroll
          for (int u = 0; u < VN; ++u) o[c + u] = fmaf(p, f[u], o[c + u]);
        }
      }
#pragma unroll
      for (int c = 0; c < D; c += VN) VT::store(out + row * D + c, o + c);
      for (int t = 0; t < k; ++t) idx[row * k + t] = t < cnt ? li[t * kThreads + x] : -1;
      lse[row] = L;
      if constexpr (DIAG) lse_all[row] = (dmax * c2 + log2f(dsum)) * 0.6931471805599453f;
    }
  }
}

template <typename T, int D, int KCAP, bool DIAG>
cudaError_t launch_diag(const FwdArgs& a, cudaStream_t stream) {
  auto kern = fwd_simt_kernel<T, D, KCAP, DIAG>;
  const size_t smem = sizeof(float) * (kKeyTile * D + 2 * KCAP * kThreads);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)a.H * a.max_items;
  const int grid = (int)(blocks < 65535 * 16 ? blocks : 65535 * 16);
  kern<<<grid, kThreads, smem, stream>>>(
      static_cast<const T*>(a.Q), static_cast<const T*>(a.K), static_cast<const T*>(a.V), a.items,
      a.count, a.H, a.k, a.scale, static_cast<T*>(a.out), a.idx, a.lse, a.lse_all);
  return cudaGetLastError();
}

template <typename T, int D, int KCAP>
cudaError_t launch_typed(const FwdArgs& a, cudaStream_t stream) {
  if (a.lse_all) return launch_diag<T, D, KCAP, true>(a, stream);
  return launch_diag<T, D, KCAP, false>(a, stream);
}

template <typename T, int D>
cudaError_t launch_d(const FwdArgs& a, cudaStream_t stream) {
  if (a.k <= 16) return launch_typed<T, D, 16>(a, stream);
  if (a.k <= 32) return launch_typed<T, D, 32>(a, stream);
  return launch_typed<T, D, 64>(a, stream);
}

template <typename T>
cudaError_t launch_t(const FwdArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 16: return launch_d<T, 16>(a, stream);
    case 32: return launch_d<T, 32>(a, stream);
    case 64: return launch_d<T, 64>(a, stream);
    case 128: return launch_d<T, 128>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_fwd_simt(kmip_dtype_t dtype, const FwdArgs& a, cudaStream_t stream) {
  if (dtype == KMIP_BF16) return launch_t<__nv_bfloat16>(a, stream);
  if (dtype == KMIP_F32) return launch_t<float>(a, stream);
  return cudaErrorNotSupported;
}

}  // namespace kmip
