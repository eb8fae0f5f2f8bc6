// kmip_fwd_tc.cu -- fused k-MIP attention forward on the sm_100a tensor cores.
//
// k-Maximum Inner Product Attention for Graph Transformers ... (Abstract):
// every query keeps the k keys of its graph with the largest inner product
// and attends over them only; the N x N score matrix is never stored, so
// memory stays linear in N.  Here the scores of a 256-query x 128-key tile
// are dense contractions on the tensor cores (tcgen05, fp32 accumulators in
// tensor memory), and the running top-k filter reads them straight out of
// tensor memory.
//
// Persistent CTAs, one per SM, walk the work list (256 queries of one graph,
// one head per item).  Warp roles:
//   warp 0       TMA producer: the item's two 128-row Q tiles once, then the
//                graph's K tiles (128 keys each) through a shared-memory ring.
//   warps 1, 2   MMA issuers, one thread each, alternating K tiles: S = Q K^T
//                for both Q tiles into the warp's own TMEM accumulator (2 x
//                128 lanes x 128 fp32 columns).  One thread issuing every MMA,
//                commit and wait cannot keep the tensor pipe busy when d is
//                small (a tile is only 2 d/16 instructions); two can.
//   warps 3..10  epilogue, one thread per query row: it copies the tile's 128
//                scores of its row to registers and releases the accumulator
//                at once.  The per-score filter has no branch: a three-input-
//                max tree gives each 16-column group's maximum, and a group
//                whose maximum beats the row's threshold (its k-th best score
//                so far) sets a bit in a candidate mask.  The warp walks the
//                union of flagged groups and queues each flagged lane's whole
//                group in shared memory.  Queues are drained by all lanes
//                together (one entry per lane per round) into the row's sorted
//                list, held in registers while the drain runs (a branch-free
//                compare-exchange chain for k <= 16; binary search and shift in
//                shared memory for larger k).  The first tile of an item, where
//                the threshold starts at -inf, is queued and drained 32 scores
//                at a time straight from tensor memory.  After the last key
//                tile: the softmax over the kept scores, lse, and the weighted
//                sum of the kept V rows (16-byte loads).
// Keys outside the query's graph are never loaded (the key range comes from
// the work item); the last tile of a graph masks its tail columns.
//
// Every pipeline wait is bounded (kmip_sm100.cuh); on a timeout the CTA
// raises its abort flag, records KMIP_ERR_TIMEOUT, lets in-flight copies and
// MMAs drain (again bounded), frees its tensor memory and returns.
#include <cuda.h>
#include <math.h>

#include <mutex>

#include "kmip_internal.h"
#include "kmip_sm100.cuh"

namespace kmip {
namespace {

using namespace sm100;

constexpr int kBM = 128;           // rows of one Q tile (TMEM lanes)
constexpr int kMT = 2;             // Q tiles per work item
constexpr int kBN = 128;           // keys per K tile (MMA N)
constexpr int kNB = 2;             // accumulator buffers, one per MMA warp
constexpr int kMmaWarps = kNB;
constexpr int kEpiWarps = 8;       // 4 lane quarters x 2 Q tiles
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kFirstEpiWarp = 1 + kMmaWarps;
constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);
constexpr int kRegK = 16;          // lists up to this k live in registers during a drain
constexpr uint32_t kTmemCols = kNB * kMT * kBN;  // 512
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s
constexpr size_t kSmemBudget = 227 * 1024;
constexpr size_t kMinSmem = 120 * 1024;  // keeps one CTA (one TMEM owner) per SM

static_assert(kTcQueries == kBM * kMT, "work item size");
static_assert(kTmemCols == 512, "tensor memory budget");

template <int D, int KCAP>
struct Cfg {
  static constexpr int kRegionElems = D < 64 ? D : 64;        // K columns per swizzle region
  static constexpr int kRegions = D / kRegionElems;           // 1, or 2 for d = 128
  static constexpr int kRowBytes = kRegionElems * 2;          // 32, 64 or 128 B
  static constexpr uint32_t kLayout = kRowBytes == 32 ? 6u : (kRowBytes == 64 ? 4u : 2u);
  static constexpr uint32_t kSbo = 8 * kRowBytes;             // 8-row core group stride
  static constexpr int kRegionBytes = 128 * kRowBytes;        // one region of a 128-row box
  static constexpr int kBoxBytes = kRegions * kRegionBytes;   // a 128-row box, all of d
  static constexpr int kQBytes = kMT * kBoxBytes;             // the item's Q tiles
  static constexpr int kStageBytes = kBoxBytes;               // one K tile (128 keys)
  static constexpr int kListBytes = 2 * KCAP * kEpiThreads * 4;
  static constexpr int kBarBytes = 1024;
  static constexpr int kBase = kQBytes + kListBytes + kBarBytes + 1024;  // + slack
  // Candidate queue: 32 entries per row where three ring stages still fit, else 16.
  static constexpr int kQueue =
      (int)((kSmemBudget - kBase - 32 * 8 * kEpiThreads) / kStageBytes) >= 3 ? 32 : 16;
  static constexpr int kFixed = kBase + kQueue * 8 * kEpiThreads;
  static constexpr int kStagesFit = (int)((kSmemBudget - kFixed) / kStageBytes);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr size_t kSmem = (size_t)kFixed + (size_t)kStages * kStageBytes;
  static constexpr size_t kSmemLaunch = kSmem > kMinSmem ? kSmem : kMinSmem;
  static constexpr bool kFits = kStages >= 2 && kSmem <= kSmemBudget;
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN);
  // Start-address offset (16-byte units) of K step kk (16 bf16 columns).
  static constexpr uint32_t step_off(int kk) {
    return (uint32_t)(((kk * 16 / kRegionElems) * kRegionBytes + (kk * 16 % kRegionElems) * 2) >> 4);
  }
};

struct TcParams {
  const __nv_bfloat16* V;
  const WorkItem* items;
  const int* count;
  int H, k;
  float scale;
  __nv_bfloat16* out;
  int32_t* idx;
  float* lse;
  int* status;
  uint64_t timeout_ns;
};

// Maximum of 16 scores with three-input max.
__device__ __forceinline__ float max16(const float* x) {
  const float a = fmax3(x[0], x[1], x[2]), b = fmax3(x[3], x[4], x[5]);
  const float c = fmax3(x[6], x[7], x[8]), d = fmax3(x[9], x[10], x[11]);
  const float e = fmax3(x[12], x[13], x[14]);
  return fmax3(fmax3(a, b, c), fmax3(d, e, x[15]), -INFINITY);
}

// Top-k state of one query row.  The sorted list (larger score
// first, equal scores by smaller key index) and the FIFO candidate queue live
// column-major in shared memory (slot t at [t * kEpiThreads]).  For
// KCAP == kRegK the list always has kRegK slots: the first kRegK - k hold +inf
// sentinels, the k real entries follow, so the k-th best is always the last
// slot; otherwise the k real entries are slots 0 .. k-1.  thr is the k-th best
// score (a key must beat it to enter).
template <int KCAP>
struct RowState {
  float* ls;
  int* li;
  float* qs;
  int* qj;
  float thr;
  int qn;

  __device__ __forceinline__ int first_slot(int k) const { return KCAP == kRegK ? kRegK - k : 0; }

  __device__ __forceinline__ void reset(int k) {
    constexpr int S = kEpiThreads;
    if (KCAP == kRegK) {
#pragma unroll
      for (int t = 0; t < kRegK; ++t) {
        ls[t * S] = t < kRegK - k ? INFINITY : -INFINITY;
        li[t * S] = -1;
      }
    } else {
      for (int t = 0; t < k; ++t) {
        ls[t * S] = -INFINITY;
        li[t * S] = -1;
      }
    }
    thr = -INFINITY;
    qn = 0;
  }

  // All lanes of the warp empty their queues together, oldest entry first.
  // in_regs: the list is held in registers while draining (use where few
  // other registers are live).
  __device__ __forceinline__ void drain(int k, bool in_regs);
};

// Drain with the list in registers: a branch-free compare-exchange chain per
// round (k <= kRegK lists; the k-th best is the last of kRegK slots).
// Returns the new threshold.  Out of line so that its code exists once.
__device__ __noinline__ float drain_regs(float* ls, int* li, const float* qs, const int* qj,
                                         int qn, float thr) {
  constexpr int S = kEpiThreads;
  const int rounds = __reduce_max_sync(0xffffffffu, qn);
  if (rounds == 0) return thr;
  float L[kRegK];
  int J[kRegK];
#pragma unroll
  for (int t = 0; t < kRegK; ++t) {
    L[t] = ls[t * S];
    J[t] = li[t * S];
  }
  for (int r = 0; r < rounds; ++r) {
    float s = -INFINITY;
    int j = -1;
    if (r < qn) {
      s = qs[r * S];
      j = qj[r * S];
    }
    if (!(s > thr)) s = -INFINITY;  // no-op pass
    if (!__any_sync(0xffffffffu, s > thr)) continue;  // nothing enters this round
    // Compare-exchange chain: the larger value stays, the smaller moves on.
#pragma unroll
    for (int t = 0; t < kRegK; ++t) {
      const bool c = s > L[t];
      const float hi = fmaxf(L[t], s), lo = fminf(L[t], s);
      const int jk = c ? j : J[t], jm = c ? J[t] : j;
      L[t] = hi;
      s = lo;
      J[t] = jk;
      j = jm;
    }
    thr = L[kRegK - 1];
  }
#pragma unroll
  for (int t = 0; t < kRegK; ++t) {
    ls[t * S] = L[t];
    li[t * S] = J[t];
  }
  __syncwarp();
  return thr;
}

// Drain by binary search and shift in shared memory over the k real entries
// starting at slot `first` (keys arrive in increasing index order, so an
// equal score stays behind).  Returns the new threshold.  Out of line.
__device__ __noinline__ float drain_smem(float* ls, int* li, const float* qs, const int* qj,
                                         int qn, float thr, int k, int first) {
  constexpr int S = kEpiThreads;
  const int rounds = __reduce_max_sync(0xffffffffu, qn);
  float* L = ls + first * S;
  int* J = li + first * S;
  for (int r = 0; r < rounds; ++r) {
    if (r < qn) {
      const float s = qs[r * S];
      if (s > thr) {
        const int jn = qj[r * S];
        int lo = 0, hi = k - 1;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (L[mid * S] < s) hi = mid; else lo = mid + 1;
        }
        for (int e = k - 1; e > lo; --e) {
          L[e * S] = L[(e - 1) * S];
          J[e * S] = J[(e - 1) * S];
        }
        L[lo * S] = s;
        J[lo * S] = jn;
        thr = L[(k - 1) * S];
      }
    }
  }
  __syncwarp();
  return thr;
}

template <int KCAP>
__device__ __forceinline__ void RowState<KCAP>::drain(int k, bool in_regs) {
  if (KCAP == kRegK && in_regs)
    thr = drain_regs(ls, li, qs, qj, qn, thr);
  else
    thr = drain_smem(ls, li, qs, qj, qn, thr, k, first_slot(k));
  qn = 0;
}

// Queue the scores of a 16-score group (keys jb .. jb+15) that beat the
// row's threshold, when `on`.  Branch-free: every score is written at the
// queue tail and the tail only advances past qualifying ones (a later score
// overwrites a rejected one).  The caller guarantees room for 16 more
// entries, so every store stays inside the queue.
template <int KCAP>
__device__ __forceinline__ void append_group(RowState<KCAP>& R, const float* v, int jb, bool on) {
  constexpr int S = kEpiThreads;
  if (on) {
    const float t = R.thr;
    int n = R.qn;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      R.qs[n * S] = v[u];
      R.qj[n * S] = jb + u;
      n += v[u] > t ? 1 : 0;
    }
    R.qn = n;
  }
}

template <int D, int KCAP>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const TcParams p) {
  using C = Cfg<D, KCAP>;
  constexpr int kStages = C::kStages;
  constexpr int S = kEpiThreads;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment of the swizzled tiles.
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_smem = base;
  unsigned char* k_smem = q_smem + C::kQBytes;
  float* ls = reinterpret_cast<float*>(k_smem + kStages * C::kStageBytes);
  int* li = reinterpret_cast<int*>(ls + KCAP * S);
  float* qs = reinterpret_cast<float*>(li + KCAP * S);
  int* qj = reinterpret_cast<int*>(qs + C::kQueue * S);
  uint64_t* bars = reinterpret_cast<uint64_t*>(qj + C::kQueue * S);
  uint64_t* full = bars;                  // [kStages]  K tile landed
  uint64_t* empty = full + kStages;       // [kStages]  K tile consumed by the MMAs
  uint64_t* tfull = empty + kStages;      // [kNB]      accumulator ready
  uint64_t* tempty = tfull + kNB;         // [kNB]      accumulator copied out
  uint64_t* qfull = tempty + kNB;         // Q tile landed
  uint64_t* qempty = qfull + 1;           // Q tile no longer read (both MMA warps)
  uint64_t* mdone = qempty + 1;           // every MMA of this CTA finished
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(full + s), 1);
      mbar_init(smem_addr(empty + s), 1);
    }
    for (int b = 0; b < kNB; ++b) {
      mbar_init(smem_addr(tfull + b), 1);
      mbar_init(smem_addr(tempty + b), kEpiWarps);
    }
    mbar_init(smem_addr(qfull), 1);
    mbar_init(smem_addr(qempty), kMmaWarps);
    mbar_init(smem_addr(mdone), kMmaWarps);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_holder), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  const int count = *p.count;
  const int64_t total = (int64_t)p.H * count;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kn = 0, qn = 0;  // K tiles and Q tiles issued
      bool ok = true;
      for (int64_t w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const int h = (int)(w / count);
        const WorkItem it = p.items[w % count];
        if (!mbar_wait(smem_addr(qempty), (qn & 1) ^ 1, abort_flag, p.timeout_ns)) break;
        mbar_arrive_expect_tx(smem_addr(qfull), C::kQBytes);
        for (int mt = 0; mt < kMT; ++mt)
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_2d(smem_addr(q_smem + mt * C::kBoxBytes + r * C::kRegionBytes), &tmQ,
                        smem_addr(qfull), h * D + r * C::kRegionElems, it.q0 + mt * kBM);
        ++qn;
        const int ntiles = (it.j1 - it.j0 + kBN - 1) / kBN;
        for (int t = 0; t < ntiles; ++t, ++kn) {
          const int s = (int)(kn % kStages);
          const uint32_t ph = (kn / kStages) & 1;
          if (!mbar_wait(smem_addr(empty + s), ph ^ 1, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(smem_addr(full + s), C::kStageBytes);
          for (int r = 0; r < C::kRegions; ++r)
            tma_load_2d(smem_addr(k_smem + s * C::kStageBytes + r * C::kRegionBytes), &tmK,
                        smem_addr(full + s), h * D + r * C::kRegionElems, it.j0 + t * kBN);
        }
      }
      // Drain: every copy this thread issued has landed before the CTA exits.
      for (int s = 0; s < kStages; ++s) {
        const uint32_t issued = kn > (uint32_t)s ? (kn - 1 - s) / kStages + 1 : 0;
        if (issued) {
          const uint64_t t0 = global_ns();
          while (!mbar_try_wait(smem_addr(full + s), (issued - 1) & 1) &&
                 global_ns() - t0 < p.timeout_ns) {
          }
        }
      }
      if (qn) {
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(smem_addr(qfull), (qn - 1) & 1) && global_ns() - t0 < p.timeout_ns) {
        }
      }
    }
  } else if (warp < kFirstEpiWarp) {
    // ------------------------------------------------- MMA (two warps)
    const int m = warp - 1;  // this warp's accumulator buffer and tile parity
    if (lane == 0) {
      const uint64_t qdesc = smem_desc(smem_addr(q_smem), C::kSbo, C::kLayout);
      const uint64_t kdesc0 = smem_desc(smem_addr(k_smem), C::kSbo, C::kLayout);
      const uint32_t dcol = tmem + m * (kMT * kBN);
      uint32_t tn = 0, qn = 0;  // K tiles (all, both parities), items
      bool ok = true;
      for (int64_t w = blockIdx.x; w < total && ok; w += gridDim.x) {
        const WorkItem it = p.items[w % count];
        const int mts = (it.q1 - it.q0) > kBM ? 2 : 1;  // Q tiles with rows
        if (!mbar_wait(smem_addr(qfull), qn & 1, abort_flag, p.timeout_ns)) break;
        ++qn;
        tc_fence_after();
        const int ntiles = (it.j1 - it.j0 + kBN - 1) / kBN;
        for (int t = 0; t < ntiles; ++t, ++tn) {
          if ((int)(tn % kNB) != m) continue;
          const int s = (int)(tn % kStages);
          const uint32_t ph = (tn / kStages) & 1;
          const uint32_t use = tn / kNB;
          if (!mbar_wait(smem_addr(tempty + m), (use & 1) ^ 1, abort_flag, p.timeout_ns) ||
              !mbar_wait(smem_addr(full + s), ph, abort_flag, p.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kdesc = kdesc0 + (uint64_t)((s * C::kStageBytes) >> 4);
          for (int mt = 0; mt < mts; ++mt) {
            const uint64_t qd = qdesc + (uint64_t)((mt * C::kBoxBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_bf16(dcol + mt * kBN, qd + C::step_off(kk), kdesc + C::step_off(kk), C::kIdesc,
                       kk > 0);
          }
          mma_commit(smem_addr(empty + s));
          mma_commit(smem_addr(tfull + m));
        }
        if (ok) mma_commit(smem_addr(qempty));
      }
      mma_commit(smem_addr(mdone));
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(smem_addr(mdone), 0) && global_ns() - t0 < p.timeout_ns) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - kFirstEpiWarp;     // 0..7
    const int mt = ew >> 2;                  // Q tile of this warp
    const int quarter = warp & 3;            // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;     // row within the Q tile
    const int et = ew * 32 + lane;           // shared-memory column of this thread
    RowState<KCAP> R{ls + et, li + et, qs + et, qj + et, -INFINITY, 0};
    const int64_t HD = (int64_t)p.H * D;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    uint32_t tn = 0;
    bool ok = true;
    for (int64_t w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const int h = (int)(w / count);
      const WorkItem it = p.items[w % count];
      const bool tile_on = mt == 0 || (it.q1 - it.q0) > kBM;  // warp-uniform
      const int i = it.q0 + mt * kBM + row;
      R.reset(p.k);
      const int ntiles = (it.j1 - it.j0 + kBN - 1) / kBN;
      for (int t = 0; t < ntiles; ++t, ++tn) {
        const int b = (int)(tn % kNB);
        const uint32_t use = tn / kNB;
        const bool got = __all_sync(
            0xffffffffu, mbar_wait(smem_addr(tfull + b), use & 1, abort_flag, p.timeout_ns));
        if (!got) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem + lane_base + b * (kMT * kBN) + mt * kBN;
        const int jt = it.j0 + t * kBN;            // key of column 0
        const int valid = min(kBN, it.j1 - jt);
        if (!tile_on) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_addr(tempty + b));
          continue;
        }
        if (t == 0) {
          // The threshold starts at -inf, so the first tile holds a large share
          // of a row's candidates: queue and drain it straight from tensor
          // memory, then release the accumulator.
#pragma unroll 1
          for (int c = 0; c < kBN / 32; ++c) {
            float v[32];
            tmem_ld32(ta + c * 32, v);
            tmem_ld_wait(v);
            constexpr int QB = C::kQueue < 32 ? C::kQueue : 32;  // queue batch
#pragma unroll
            for (int sb = 0; sb < 32; sb += QB) {
#pragma unroll
              for (int u = 0; u < QB; ++u) {
                R.qs[u * S] = c * 32 + sb + u < valid ? v[sb + u] : -INFINITY;
                R.qj[u * S] = jt + c * 32 + sb + u;
              }
              R.qn = QB;
              R.drain(p.k, true);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_addr(tempty + b));
          continue;
        }
        // Copy the row's 128 scores to registers.
        float vt[kBN / 32][32];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(ta + c * 32, vt[c]);
        tmem_ld_wait_all();
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) reg_fence(vt[c]);
        if (valid < kBN) {
#pragma unroll
          for (int c = 0; c < kBN / 32; ++c)
#pragma unroll
            for (int u = 0; u < 32; ++u)
              if (c * 32 + u >= valid) vt[c][u] = -INFINITY;
        }
        uint32_t mask = 0;
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          if (max16(vt[c]) > R.thr) mask |= 1u << (2 * c);
          if (max16(vt[c] + 16) > R.thr) mask |= 1u << (2 * c + 1);
        }
        const uint32_t todo = __reduce_or_sync(0xffffffffu, mask);
        const bool roomy = !__any_sync(0xffffffffu, R.qn + 16 * __popc(mask) > C::kQueue);
        if (roomy) {
          // Common case: every lane has room for all its flagged groups, so
          // release the accumulator now and queue from registers.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_addr(tempty + b));
#pragma unroll
          for (int gi = 0; gi < kBN / 16; ++gi)
            if (todo & (1u << gi))  // warp-uniform
              append_group(R, vt[gi >> 1] + (gi & 1) * 16, jt + gi * 16, (mask >> gi) & 1u);
          __syncwarp();
        } else {
          // Rare: a queue could overflow.  Keep the accumulator, re-read each
          // flagged group from tensor memory, drain between groups as needed.
#pragma unroll 1
          for (int gi = 0; gi < kBN / 16; ++gi) {
            if (todo & (1u << gi)) {
              if (__any_sync(0xffffffffu, R.qn > C::kQueue - 16)) R.drain(p.k, false);
              float g[16];
              tmem_ld16(ta + gi * 16, g);
              tmem_ld_wait(g);
#pragma unroll
              for (int u = 0; u < 16; ++u)
                if (gi * 16 + u >= valid) g[u] = -INFINITY;
              append_group(R, g, jt + gi * 16, (mask >> gi) & 1u);
              __syncwarp();
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_addr(tempty + b));
        }
        if (todo) {
          // Insert once half the lanes have queued groups, or before a queue
          // could overflow during the next tile.
          if (__popc(__ballot_sync(0xffffffffu, R.qn > 0)) >= 16 ||
              __any_sync(0xffffffffu, 2 * R.qn > C::kQueue))
            R.drain(p.k, true);
        }
      }
      if (!ok) break;
      R.drain(p.k, true);
      if (tile_on && i < it.q1) {
        const float* L = R.ls + R.first_slot(p.k) * S;
        const int* J = R.li + R.first_slot(p.k) * S;
        int cnt = 0;
        while (cnt < p.k && J[cnt * S] >= 0) ++cnt;
        // Softmax over the kept scaled scores, lse, weighted sum of V rows.
        const int64_t rowg = (int64_t)i * p.H + h;
        const float mx = p.scale * L[0];
        float sum = 0.f;
        for (int t = 0; t < cnt; ++t) sum += expf(p.scale * L[t * S] - mx);
        const float lse_v = mx + logf(sum);
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          constexpr int CW = D < 32 ? D : 32;
          float o[CW];
#pragma unroll
          for (int u = 0; u < CW; ++u) o[u] = 0.f;
          for (int t = 0; t < cnt; ++t) {
            const float pw = expf(p.scale * L[t * S] - lse_v);
            const __nv_bfloat16* vr = p.V + (int64_t)J[t * S] * HD + h * D + c0;
#pragma unroll
            for (int u = 0; u < CW; u += 8) {
              float f[8];
              Vec<__nv_bfloat16>::load(vr + u, f);
#pragma unroll
              for (int e = 0; e < 8; ++e) o[u + e] = fmaf(pw, f[e], o[u + e]);
            }
          }
#pragma unroll
          for (int u = 0; u < CW; u += 8) Vec<__nv_bfloat16>::store(p.out + rowg * D + c0 + u, o + u);
        }
        for (int t = 0; t < p.k; ++t) p.idx[rowg * p.k + t] = t < cnt ? J[t * S] : -1;
        p.lse[rowg] = lse_v;
      }
    }
  }

  // --------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) record_status(p.status, KMIP_ERR_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// [N rows, H*d columns] bf16, box = (region width, 128 rows), swizzled.
template <int D>
bool make_map(CUtensorMap* m, const void* ptr, int N, int H) {
  using C = Cfg<D, kRegK>;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)H * D, (cuuint64_t)N};
  const cuuint64_t strides[1] = {(cuuint64_t)H * D * 2};
  const cuuint32_t box[2] = {(cuuint32_t)C::kRegionElems, 128u};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = C::kRowBytes == 32   ? CU_TENSOR_MAP_SWIZZLE_32B
                                : C::kRowBytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                     : CU_TENSOR_MAP_SWIZZLE_128B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int KCAP>
cudaError_t launch_cfg(const FwdArgs& a, cudaStream_t stream) {
  using C = Cfg<D, KCAP>;
  static_assert(C::kFits, "shared memory budget");
  CUtensorMap mq, mk;
  if (!make_map<D>(&mq, a.Q, a.N, a.H) || !make_map<D>(&mk, a.K, a.N, a.H))
    return cudaErrorInvalidValue;
  auto kern = fwd_tc_kernel<D, KCAP>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemLaunch);
  if (e != cudaSuccess) return e;
  const int64_t units = (int64_t)a.H * a.max_items;
  const int sms = device_sm_count();
  const int grid = (int)(units < sms ? units : sms);
  TcParams p{static_cast<const __nv_bfloat16*>(a.V), a.items, a.count, a.H, a.k, a.scale,
             static_cast<__nv_bfloat16*>(a.out), a.idx, a.lse, a.status, kTimeoutNs};
  kern<<<grid, kThreads, C::kSmemLaunch, stream>>>(mq, mk, p);
  return cudaGetLastError();
}

template <int D, int KCAP>
cudaError_t launch_k(const FwdArgs& a, cudaStream_t stream) {
  if constexpr (Cfg<D, KCAP>::kFits) return launch_cfg<D, KCAP>(a, stream);
  return cudaErrorNotSupported;
}

template <int D>
cudaError_t launch_d(const FwdArgs& a, cudaStream_t stream) {
  if (a.k <= kRegK) return launch_k<D, kRegK>(a, stream);
  if (a.k <= 32) return launch_k<D, 32>(a, stream);
  return launch_k<D, 64>(a, stream);
}

}  // namespace

template <int D>
bool fits_d(int k) {
  if (k <= kRegK) return Cfg<D, kRegK>::kFits;
  if (k <= 32) return Cfg<D, 32>::kFits;
  return Cfg<D, 64>::kFits;
}

// Shapes whose lists, queues, Q tile and at least two K stages fit in shared
// memory (d = 128 does not); other shapes run the fp32-FMA forward.
bool fwd_tc_supported(int d, int k) {
  if (k < 1 || k > 64) return false;
  switch (d) {
    case 16: return fits_d<16>(k);
    case 32: return fits_d<32>(k);
    case 64: return fits_d<64>(k);
    case 128: return fits_d<128>(k);
    default: return false;
  }
}

cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t stream) {
  if (!fwd_tc_supported(a.d, a.k)) return cudaErrorNotSupported;
  switch (a.d) {
    case 16: return launch_d<16>(a, stream);
    case 32: return launch_d<32>(a, stream);
    case 64: return launch_d<64>(a, stream);
    case 128: return launch_d<128>(a, stream);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace kmip
