// kmip_bwd.cu -- backward pass of k-MIP attention through the kept keys.
//
// The pages time a "training setting" (k-Maximum Inner Product Attention for
// Graph Transformers ..., Tables 10-12 and 16) without spelling out the
// gradient; differentiating the forward with the selection held fixed gives,
// for query i, head h and kept keys j:
//   p_j  = exp(scale s_j - lse),  dP_j = dO . V_j,  D = sum_j p_j dP_j,
//   dS_j = p_j (dP_j - D),        dQ_i = scale sum_j dS_j K_j,
//   dK_j += scale dS_j Q_i,       dV_j += p_j dO_i.
//
// p_j is taken as exp(scale s_j - lse) over the sum of those terms, the
// softmax of the scores as this kernel recomputes them: lse (from the
// forward) only shifts the exponent, and the forward's scores may differ from
// these in the last bits (another summation order), which would leave the
// p_j summing to 1 only up to rounding; when one key takes nearly all the
// weight, dS_j = p_j (dP_j - D) cancels and that mismatch, not the
// arithmetic of this kernel, would set its error.
//
// One warp per (query, head).  The d columns are split into 16-byte slices
// (8 bf16 or 4 fp32 values per lane), so one warp instruction touches
// 32 / (d / slice) kept rows at once with coalesced 16-byte loads.  Pass 1
// recomputes s_j and dP_j for every kept key, pass 2 forms dS_j, accumulates
// dQ in registers and scatters dK/dV rows with vector fp32 reductions
// (red.global.add.v4.f32), one 16-byte reduction per lane per row.
#include <math.h>

#include "kmip_internal.h"

namespace kmip {
namespace {

constexpr int kWarps = 8;
constexpr int kKmax = 64;

// DET: instead of scattering into dK/dV, write for every kept key its
// coefficients (p_j, scale dS_j), its (key, head) bucket as a sort key and
// its position in idx as the sort value, and count the bucket's entries;
// the deterministic reduction (kmip_bwd_det.cu) sums them per key.
template <typename T, int D, bool DET>
__global__ void __launch_bounds__(kWarps * 32)
bwd_kernel(const T* __restrict__ dO, const T* __restrict__ Q, const T* __restrict__ K,
           const T* __restrict__ V, const int32_t* __restrict__ idx,
           const float* __restrict__ lse, float* __restrict__ dQ, float* __restrict__ dK,
           float* __restrict__ dV, int N, int H, int k, float scale, int* status,
           DetBuffers det) {
  using VT = Vec<T>;
  constexpr int VN = VT::N;         // elements per lane slice
  constexpr int LPR = D / VN;       // lanes per row
  constexpr int RPP = 32 / LPR;     // rows per pass
  static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "bad slice split");
  __shared__ float sp[kWarps][kKmax];
  __shared__ float sdp[kWarps][kKmax];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rs = lane / LPR, cs = (lane % LPR) * VN;
  const int64_t HD = (int64_t)H * D;
  const int64_t pairs = (int64_t)N * H;
  const int npass = (k + RPP - 1) / RPP;

  for (int64_t pr = (int64_t)blockIdx.x * kWarps + warp; pr < pairs;
       pr += (int64_t)gridDim.x * kWarps) {
    const int64_t base = pr * D;  // row (i, h) of [N, H, d]
    float q[VN], go[VN];
    VT::load(Q + base + cs, q);
    VT::load(dO + base + cs, go);
    const float L = lse[pr];
    const int32_t* ir = idx + pr * k;

    // Pass 1: p_j and dP_j of every kept key.
    float Dsum = 0.f, Psum = 0.f;
    for (int ps = 0; ps < npass; ++ps) {
      const int t = ps * RPP + rs;
      int j = t < k ? ir[t] : -1;
      if (j >= N || j < -1) {
        record_status(status, KMIP_ERR_BAD_INDEX);
        j = -1;
      }
      float s = 0.f, dp = 0.f;
      if (j >= 0) {
        float kv[VN], vv[VN];
        VT::load(K + (int64_t)j * HD + (base % HD) + cs, kv);
        VT::load(V + (int64_t)j * HD + (base % HD) + cs, vv);
#pragma unroll
        for (int u = 0; u < VN; ++u) {
          s = fmaf(q[u], kv[u], s);
          dp = fmaf(go[u], vv[u], dp);
        }
      }
#pragma unroll
      for (int o = 1; o < LPR; o <<= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, o);
        dp += __shfl_xor_sync(0xffffffffu, dp, o);
      }
      const float p = j >= 0 ? expf(scale * s - L) : 0.f;
      if (t < k && (lane % LPR) == 0) {
        sp[warp][t] = p;
        sdp[warp][t] = dp;
        if constexpr (DET) {
          const int64_t e = pr * k + t;
          const uint32_t b = j >= 0 ? (uint32_t)((int64_t)j * H + pr % H) : det.sentinel;
          det.keys[e] = b;
          det.vals[e] = (uint32_t)e;
          if (j >= 0) atomicAdd(det.count + b, 1);
        }
      }
      Dsum = fmaf(p, dp, Dsum);  // identical in the LPR lanes of a row
      Psum += p;
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
      Dsum += __shfl_xor_sync(0xffffffffu, Dsum, o);
      Psum += __shfl_xor_sync(0xffffffffu, Psum, o);
    }
    const float inv = Psum > 0.f ? 1.f / Psum : 0.f;
    Dsum *= inv;
    __syncwarp();

    // Pass 2: dS_j, dQ accumulation, dK/dV scatter.
    float dq[VN];
#pragma unroll
    for (int u = 0; u < VN; ++u) dq[u] = 0.f;
    for (int ps = 0; ps < npass; ++ps) {
      const int t = ps * RPP + rs;
      int j = t < k ? ir[t] : -1;
      if (j >= N || j < -1) j = -1;
      if (j >= 0) {
        const float p = sp[warp][t] * inv;
        const float ds = p * (sdp[warp][t] - Dsum);
        const int64_t kb = (int64_t)j * HD + (base % HD) + cs;
        float kv[VN];
        VT::load(K + kb, kv);
#pragma unroll
        for (int u = 0; u < VN; ++u) dq[u] = fmaf(ds, kv[u], dq[u]);
        const float a = scale * ds;
        if constexpr (DET) {
          if ((lane % LPR) == 0) det.coef[pr * k + t] = make_float2(p, a);
        } else {
#pragma unroll
          for (int u = 0; u < VN; u += 4) {
            red_add_v4(dK + kb + u, a * q[u], a * q[u + 1], a * q[u + 2], a * q[u + 3]);
            red_add_v4(dV + kb + u, p * go[u], p * go[u + 1], p * go[u + 2], p * go[u + 3]);
          }
        }
      }
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
      for (int u = 0; u < VN; ++u) dq[u] += __shfl_xor_sync(0xffffffffu, dq[u], o);
    }
    if (rs == 0) {
      float r[VN];
#pragma unroll
      for (int u = 0; u < VN; ++u) r[u] = scale * dq[u];
#pragma unroll
      for (int u = 0; u < VN; u += 4)
        *reinterpret_cast<float4*>(dQ + base + cs + u) = make_float4(r[u], r[u + 1], r[u + 2], r[u + 3]);
    }
    __syncwarp();  // sp/sdp reused by the next pair
  }
}

template <typename T, int D>
cudaError_t launch_typed(const BwdArgs& a, cudaStream_t stream) {
  const int64_t pairs = (int64_t)a.N * a.H;
  int64_t blocks = (pairs + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)device_sm_count() * 16;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (a.det.keys)
    bwd_kernel<T, D, true><<<(int)blocks, kWarps * 32, 0, stream>>>(
        static_cast<const T*>(a.dO), static_cast<const T*>(a.Q), static_cast<const T*>(a.K),
        static_cast<const T*>(a.V), a.idx, a.lse, a.dQ, a.dK, a.dV, a.N, a.H, a.k, a.scale,
        a.status, a.det);
  else
    bwd_kernel<T, D, false><<<(int)blocks, kWarps * 32, 0, stream>>>(
        static_cast<const T*>(a.dO), static_cast<const T*>(a.Q), static_cast<const T*>(a.K),
        static_cast<const T*>(a.V), a.idx, a.lse, a.dQ, a.dK, a.dV, a.N, a.H, a.k, a.scale,
        a.status, a.det);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const BwdArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 16: return launch_typed<T, 16>(a, stream);
    case 32: return launch_typed<T, 32>(a, stream);
    case 64: return launch_typed<T, 64>(a, stream);
    case 128: return launch_typed<T, 128>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_bwd(kmip_dtype_t dtype, const BwdArgs& a, cudaStream_t stream) {
  if (a.k > kKmax) return cudaErrorNotSupported;
  if (dtype == KMIP_BF16) return launch_t<__nv_bfloat16>(a, stream);
  if (dtype == KMIP_F32) return launch_t<float>(a, stream);
  return cudaErrorNotSupported;
}

}  // namespace kmip
