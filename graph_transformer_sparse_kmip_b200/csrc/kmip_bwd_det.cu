// kmip_bwd_det.cu -- deterministic backward of k-MIP attention.
//
// The backward of kmip_bwd.cu scatters dK_j += scale dS_j Q_i and
// dV_j += p_j dO_i with fp32 atomics, so the order of the additions (and the
// last bits of dK, dV) changes from run to run.  This variant gathers
// instead of scattering, with no atomics on the values:
//   1. the backward kernel in its coefficient mode computes p_j, dS_j and dQ
//      per (query, head) as before, and writes for every kept key e its
//      coefficients (p_j, scale dS_j), its bucket b = key * H + head as a sort
//      key and e itself as the value; padding slots get a sentinel bucket;
//   2. a stable least-significant-digit radix sort (8-bit digits) orders the
//      (bucket, e) pairs by bucket, keeping the e order inside a bucket;
//   3. an exclusive scan of the per-bucket counts gives each bucket's range;
//   4. one warp per bucket (key j, head h) sums a scale dS Q_i and p dO_i over
//      its range in that order and writes dK[j, h], dV[j, h] once.
// Every sum is taken in an order fixed by the data alone, so dK and dV are
// bitwise reproducible.  The radix sort's ranks are counted per warp with
// match_any and combined in warp order, which keeps it stable.
#include "kmip_internal.h"

namespace kmip {
namespace {

constexpr int kSortThreads = 512;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortItems = 8;                      // elements per thread per tile
constexpr int kTile = kSortThreads * kSortItems;   // 4096
constexpr int kRadixBits = 8;
constexpr int kRadix = 1 << kRadixBits;

constexpr int kScanThreads = 1024;
constexpr int kScanItems = 4;
constexpr int kScanBlock = kScanThreads * kScanItems;  // 4096

// Per-tile digit histogram, stored digit-major: hist[digit * tiles + tile],
// so an exclusive scan of hist gives every (digit, tile) its first output
// slot with tiles in order inside each digit (what keeps the sort stable).
__global__ void __launch_bounds__(kSortThreads)
radix_hist_kernel(const uint32_t* __restrict__ keys, int64_t n, int shift, int tiles,
                  uint32_t* __restrict__ hist) {
  __shared__ uint32_t cnt[kRadix];
  for (int d = threadIdx.x; d < kRadix; d += kSortThreads) cnt[d] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kTile;
  for (int it = 0; it < kSortItems; ++it) {
    const int64_t i = base + it * kSortThreads + threadIdx.x;
    if (i < n) atomicAdd(&cnt[(keys[i] >> shift) & (kRadix - 1)], 1u);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < kRadix; d += kSortThreads)
    hist[(int64_t)d * tiles + blockIdx.x] = cnt[d];
}

// Block-wide exclusive scan of kScanBlock values (4 per thread).
__device__ uint32_t block_scan(uint32_t (&v)[kScanItems], uint32_t* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t local = 0;
#pragma unroll
  for (int u = 0; u < kScanItems; ++u) {
    const uint32_t x = v[u];
    v[u] = local;
    local += x;
  }
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const uint32_t before = (warp ? warp_sums[warp - 1] : 0u) + incl - local;
#pragma unroll
  for (int u = 0; u < kScanItems; ++u) v[u] += before;
  const uint32_t total = warp_sums[31];
  __syncthreads();
  return total;
}

// Exclusive scan of x[0, n) in place, in blocks; block totals to sums.
__global__ void __launch_bounds__(kScanThreads)
scan_blocks_kernel(uint32_t* __restrict__ x, int64_t n, uint32_t* __restrict__ sums) {
  __shared__ uint32_t warp_sums[32];
  const int64_t base = (int64_t)blockIdx.x * kScanBlock + (int64_t)threadIdx.x * kScanItems;
  uint32_t v[kScanItems];
#pragma unroll
  for (int u = 0; u < kScanItems; ++u) v[u] = base + u < n ? x[base + u] : 0u;
  const uint32_t total = block_scan(v, warp_sums);
#pragma unroll
  for (int u = 0; u < kScanItems; ++u)
    if (base + u < n) x[base + u] = v[u];
  if (threadIdx.x == 0 && sums) sums[blockIdx.x] = total;
}

__global__ void __launch_bounds__(kScanThreads)
scan_add_kernel(uint32_t* __restrict__ x, int64_t n, const uint32_t* __restrict__ sums) {
  const int64_t base = (int64_t)blockIdx.x * kScanBlock + (int64_t)threadIdx.x * kScanItems;
  const uint32_t add = sums[blockIdx.x];
#pragma unroll
  for (int u = 0; u < kScanItems; ++u)
    if (base + u < n) x[base + u] += add;
}

// Exclusive scan of up to kScanBlock^2 values: per-block scans, a scan of
// the block totals in one block, then the totals added back.
cudaError_t exclusive_scan(uint32_t* x, int64_t n, uint32_t* sums, cudaStream_t stream) {
  const int64_t blocks = (n + kScanBlock - 1) / kScanBlock;
  if (blocks > kScanBlock) return cudaErrorNotSupported;
  scan_blocks_kernel<<<(int)blocks, kScanThreads, 0, stream>>>(x, n, sums);
  if (blocks > 1) {
    scan_blocks_kernel<<<1, kScanThreads, 0, stream>>>(sums, blocks, nullptr);
    scan_add_kernel<<<(int)blocks, kScanThreads, 0, stream>>>(x, n, sums);
  }
  return cudaGetLastError();
}

// Stable scatter of one radix pass.  Warp w of a tile takes the tile's
// elements [256 w, 256 w + 256) in 8 rounds of 32 consecutive ones; an
// element's rank among equal digits is the count in earlier rounds of its
// warp plus the lanes before it with the same digit (match_any), then the
// counts of the earlier warps of the tile are added.
__global__ void __launch_bounds__(kSortThreads)
radix_scatter_kernel(const uint32_t* __restrict__ keys_in, const uint32_t* __restrict__ vals_in,
                     uint32_t* __restrict__ keys_out, uint32_t* __restrict__ vals_out,
                     int64_t n, int shift, int tiles, const uint32_t* __restrict__ offs) {
  __shared__ uint32_t wcount[kSortWarps][kRadix];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < kSortWarps * kRadix; i += kSortThreads) (&wcount[0][0])[i] = 0;
  __syncthreads();
  const int64_t base = (int64_t)blockIdx.x * kTile + warp * (kTile / kSortWarps);
  uint32_t key[kSortItems], val[kSortItems], rank[kSortItems];
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * 32 + lane;
    const bool in = i < n;
    key[r] = in ? keys_in[i] : 0u;
    val[r] = in ? vals_in[i] : 0u;
    const uint32_t d = in ? (key[r] >> shift) & (kRadix - 1) : (uint32_t)kRadix;
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    rank[r] = in ? wcount[warp][d] + __popc(peers & lt) : 0u;
    __syncwarp();
    if (in && (peers & lt) == 0) wcount[warp][d] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int d = threadIdx.x; d < kRadix; d += kSortThreads) {
    uint32_t run = 0;
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t c = wcount[w][d];
      wcount[w][d] = run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * 32 + lane;
    if (i < n) {
      const uint32_t d = (key[r] >> shift) & (kRadix - 1);
      const uint32_t o = offs[(int64_t)d * tiles + blockIdx.x] + wcount[warp][d] + rank[r];
      keys_out[o] = key[r];
      vals_out[o] = val[r];
    }
  }
}

// One warp per bucket b = (key j, head h): dK[j, h] = sum a_e Q[i_e, h],
// dV[j, h] = sum p_e dO[i_e, h] over the bucket's entries in sorted (= idx)
// order.  Lanes split the d columns in 16-byte slices; entry t of the bucket
// goes to lane group t % RPP, and the groups' partial sums are combined by a
// fixed shuffle tree.
template <typename T, int D>
__global__ void __launch_bounds__(256)
gather_reduce_kernel(const T* __restrict__ Q, const T* __restrict__ dO,
                     const uint32_t* __restrict__ vals, const uint32_t* __restrict__ start,
                     const float2* __restrict__ coef, float* __restrict__ dK,
                     float* __restrict__ dV, int64_t buckets, int H, int k) {
  using VT = Vec<T>;
  constexpr int VN = VT::N;
  constexpr int LPR = D / VN;
  constexpr int RPP = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int rs = lane / LPR, cs = (lane % LPR) * VN;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t b = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); b < buckets;
       b += warps) {
    const uint32_t lo = start[b], hi = start[b + 1];
    float ak[VN], av[VN];
#pragma unroll
    for (int u = 0; u < VN; ++u) ak[u] = av[u] = 0.f;
    for (uint32_t p0 = lo; p0 < hi; p0 += RPP) {
      const uint32_t pos = p0 + rs;
      if (pos < hi) {
        const uint32_t e = vals[pos];
#ifdef KMIP_DEBUG_BOUNDS
        if ((int64_t)(e / (uint32_t)k) >= buckets) continue;  // not a (query, head) of [N, H]
#endif
        const float2 c = coef[e];
        const int64_t row = (int64_t)(e / (uint32_t)k) * D;  // (query, head) row of [N, H, d]
        float q[VN], g[VN];
        VT::load(Q + row + cs, q);
        VT::load(dO + row + cs, g);
#pragma unroll
        for (int u = 0; u < VN; ++u) {
          ak[u] = fmaf(c.y, q[u], ak[u]);
          av[u] = fmaf(c.x, g[u], av[u]);
        }
      }
    }
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) {
#pragma unroll
      for (int u = 0; u < VN; ++u) {
        ak[u] += __shfl_xor_sync(0xffffffffu, ak[u], o);
        av[u] += __shfl_xor_sync(0xffffffffu, av[u], o);
      }
    }
    if (rs == 0) {
      float* kr = dK + b * D + cs;
      float* vr = dV + b * D + cs;
#pragma unroll
      for (int u = 0; u < VN; u += 4) {
        *reinterpret_cast<float4*>(kr + u) = make_float4(ak[u], ak[u + 1], ak[u + 2], ak[u + 3]);
        *reinterpret_cast<float4*>(vr + u) = make_float4(av[u], av[u + 1], av[u + 2], av[u + 3]);
      }
    }
  }
}

template <typename T>
cudaError_t launch_reduce(const BwdArgs& a, const uint32_t* vals, const uint32_t* start,
                          const float2* coef, cudaStream_t stream) {
  const int64_t buckets = (int64_t)a.N * a.H;
  int64_t blocks = (buckets + 7) / 8;
  const int64_t cap = (int64_t)device_sm_count() * 16;
  if (blocks > cap) blocks = cap;
  const T* Q = static_cast<const T*>(a.Q);
  const T* dO = static_cast<const T*>(a.dO);
#define KMIP_REDUCE(DD)                                                                    \
  gather_reduce_kernel<T, DD><<<(int)blocks, 256, 0, stream>>>(Q, dO, vals, start, coef, \
                                                               a.dK, a.dV, buckets, a.H, a.k)
  switch (a.d) {
    case 16: KMIP_REDUCE(16); break;
    case 32: KMIP_REDUCE(32); break;
    case 64: KMIP_REDUCE(64); break;
    case 128: KMIP_REDUCE(128); break;
    default: return cudaErrorNotSupported;
  }
#undef KMIP_REDUCE
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_deterministic(kmip_dtype_t dtype, const BwdArgs& a_in, cudaStream_t stream) {
  const int64_t E = (int64_t)a_in.N * a_in.H * a_in.k;
  const int64_t NB = (int64_t)a_in.N * a_in.H;
  if (E >= ((int64_t)1 << 32) - 1 || NB + 1 >= ((int64_t)1 << 32)) return cudaErrorNotSupported;
  const int64_t tiles = (E + kTile - 1) / kTile;
  const int64_t hist_n = (int64_t)kRadix * tiles;
  const int64_t scan_max = (int64_t)kScanBlock * kScanBlock;
  if (hist_n > scan_max || NB + 1 > scan_max) return cudaErrorNotSupported;
  int passes = 0;
  for (uint64_t s = (uint64_t)NB; s; s >>= kRadixBits) ++passes;  // digits of the sentinel NB
  if (passes == 0) passes = 1;

  // scratch: coef [E] float2 | keys, vals [E] x2 | count/start [NB+1] | hist | block sums
  const int64_t sums_n = kScanBlock;
  size_t bytes = 0;
  auto take = [&](size_t b) {
    const size_t o = bytes;
    bytes += (b + 255) & ~size_t(255);
    return o;
  };
  const size_t o_coef = take(sizeof(float2) * E), o_k0 = take(4 * E), o_v0 = take(4 * E),
               o_k1 = take(4 * E), o_v1 = take(4 * E), o_cnt = take(4 * (NB + 1)),
               o_hist = take(4 * hist_n), o_sums = take(4 * sums_n);
  char* scratch = nullptr;
  if (scratch_alloc(reinterpret_cast<void**>(&scratch), bytes, stream) != cudaSuccess)
    return cudaErrorMemoryAllocation;
  float2* coef = reinterpret_cast<float2*>(scratch + o_coef);
  uint32_t* keys[2] = {reinterpret_cast<uint32_t*>(scratch + o_k0),
                       reinterpret_cast<uint32_t*>(scratch + o_k1)};
  uint32_t* vals[2] = {reinterpret_cast<uint32_t*>(scratch + o_v0),
                       reinterpret_cast<uint32_t*>(scratch + o_v1)};
  uint32_t* cnt = reinterpret_cast<uint32_t*>(scratch + o_cnt);
  uint32_t* hist = reinterpret_cast<uint32_t*>(scratch + o_hist);
  uint32_t* sums = reinterpret_cast<uint32_t*>(scratch + o_sums);

  cudaError_t e = cudaMemsetAsync(cnt, 0, 4 * (NB + 1), stream);
  BwdArgs a = a_in;
  a.det.coef = coef;
  a.det.keys = keys[0];
  a.det.vals = vals[0];
  a.det.count = reinterpret_cast<int*>(cnt);
  a.det.sentinel = (uint32_t)NB;
  if (e == cudaSuccess) e = launch_bwd(dtype, a, stream);
  int cur = 0;
  for (int ps = 0; ps < passes && e == cudaSuccess; ++ps) {
    const int shift = ps * kRadixBits;
    radix_hist_kernel<<<(int)tiles, kSortThreads, 0, stream>>>(keys[cur], E, shift, (int)tiles,
                                                                 hist);
    e = exclusive_scan(hist, hist_n, sums, stream);
    if (e != cudaSuccess) break;
    radix_scatter_kernel<<<(int)tiles, kSortThreads, 0, stream>>>(
        keys[cur], vals[cur], keys[cur ^ 1], vals[cur ^ 1], E, shift, (int)tiles, hist);
    e = cudaGetLastError();
    cur ^= 1;
  }
  // bucket ranges: exclusive scan of the counts (NB + 1 entries, the last one 0)
  if (e == cudaSuccess) e = exclusive_scan(cnt, NB + 1, sums, stream);
  if (e == cudaSuccess) {
    e = dtype == KMIP_BF16
            ? launch_reduce<__nv_bfloat16>(a_in, vals[cur], cnt, coef, stream)
            : launch_reduce<float>(a_in, vals[cur], cnt, coef, stream);
  }
  const cudaError_t ef = cudaFreeAsync(scratch, stream);
  return e != cudaSuccess ? e : ef;
}

}  // namespace kmip
