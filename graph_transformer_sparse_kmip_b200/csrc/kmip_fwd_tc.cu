// kmip_fwd_tc.cu -- fused k-MIP attention forward on the sm_100a tensor cores.
//
// k-Maximum Inner Product Attention for Graph Transformers ... (Abstract):
// every query keeps the k keys of its graph with the largest inner product
// and attends over them only; the N x N score matrix is never stored, so
// memory stays linear in N.  Here the scores of a 256-query x 128-key tile
// are dense contractions on the tensor cores (tcgen05, fp32 accumulators in
// tensor memory), and a running top-k filter reads them straight out of
// tensor memory.
//
// Persistent CTAs, one per SM, walk the work list (256 queries of one graph,
// one head per item).  Warp roles:
//   warp 0        TMA producer: the item's two 128-row Q tiles once, then the
//                 graph's K tiles (128 keys each) through a shared-memory ring.
//   warps 1, 2    MMA issuers, one thread each, alternating K tiles: S = Q K^T
//                 for both Q tiles into the warp's own TMEM accumulator (2 x
//                 128 lanes x 128 fp32 columns).  One thread issuing every MMA,
//                 commit and wait cannot keep the tensor pipe busy when d is
//                 small (a tile is only 2 d/16 instructions); two can.
//   warp 3        spare (completes the first warpgroup).
//   warps 4..11   filters, one thread per query row.  A filter copies its
//                 row's 128 scores of the tile to registers and hands the
//                 accumulator back at once.  The per-score test has
//                 no branch: a three-input-max tree gives each 16-column
//                 group's maximum, and a group whose maximum beats the row's
//                 threshold (a lower bound of its k-th best score so far) is
//                 stored whole, as a 16-score "record", in one of two record
//                 buffers of the warp's rows.  A full buffer (or, once enough
//                 rows hold records, a buffer whose twin is free) is handed
//                 to the warp's insert warp, and the filter goes on with the
//                 other buffer; it waits for an insertion only when both of
//                 its buffers are full.
//   warps 12..19  inserters, one per filter warp and one thread per row: they
//                 take the handed-over buffers in order, insert every
//                 recorded score that beats the row's threshold into the
//                 row's top-k (k <= 16: a sorted list held in registers for
//                 the whole item, each candidate placed in one step of
//                 independent compares;
//                 larger k: a four-ary heap in shared memory with the worst
//                 entry at the root; 32, 48 or 64 slots), publish the new
//                 threshold, which the filter reads every tile, and after an
//                 item's last batch compute the softmax over the kept scores,
//                 lse, and the weighted sum of the kept V rows (16-byte loads)
//                 while the filters already work on the next item.
// The warpgroups rebalance their registers at the start (setmaxnreg): the
// producer/MMA warpgroup and the inserters give some up, and the filters,
// which hold a tile's scores, take them (32 / 160 / 64 per thread: the split
// the filters and inserters compile into without spilling scores).
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
constexpr int kRows = kBM * kMT;   // query rows per work item
constexpr int kBN = 128;           // keys per K tile (MMA N)
constexpr int kNB = 2;             // accumulator buffers, one per MMA warp
constexpr int kMmaWarps = kNB;
constexpr int kFilterWarps = 8;    // 4 lane quarters x 2 Q tiles
constexpr int kInsertWarps = kFilterWarps;
constexpr int kFirstFilterWarp = 4;   // warps 0..3: producer, MMA x2, spare (one warpgroup)
constexpr int kFirstInsertWarp = kFirstFilterWarp + kFilterWarps;
constexpr int kThreads = 32 * (kFirstInsertWarp + kInsertWarps);
constexpr int kRegK = 16;          // lists up to this k are insert-sorted in registers
constexpr int kHandLanes = 16;      // rows holding records that hand a batch over early
constexpr uint32_t kTmemCols = kNB * kMT * kBN;  // 512
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s
constexpr size_t kSmemBudget = 227 * 1024;
constexpr size_t kMinSmem = 120 * 1024;  // keeps one CTA (one TMEM owner) per SM
// Registers per thread: at launch, and after the warpgroups rebalance them
// (producer/MMA warpgroup and inserters give some up, filters take them).
constexpr int kLaunchRegs = 96;
constexpr int kRegsCtl = 32, kRegsFilter = 160, kRegsInsert = 64;
static_assert(kThreads % 128 == 0, "whole warpgroups");
static_assert(128 * kRegsCtl + 32 * kFilterWarps * kRegsFilter + 32 * kInsertWarps * kRegsInsert <=
                  kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");

static_assert(kTcQueries == kRows, "work item size");
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
  // list slots per row: KCAP + 1 for the register-list path (+1: banks); for
  // the heap, 3 slots of lead so that each node's four children are one
  // aligned 16-byte quad, rounded up to a multiple of 4 (16-byte rows)
  static constexpr int kListStride = KCAP == kRegK ? KCAP + 1 : KCAP + 4;
  static constexpr int kListBytes = 2 * kListStride * kRows * 4;
  // One record buffer: per row r records of 16 scores (+4 floats: banks),
  // their first keys, and the row's record count.
  static constexpr int rec_stride(int r) { return r * 16 + 4; }
  static constexpr int buf_bytes(int r) { return kRows * (rec_stride(r) + r + 1) * 4; }
  static constexpr int kMiscBytes = kRows * 8 + 2 * kFilterWarps * 4;  // thresholds, batch flags
  static constexpr int kBarBytes = 1024;
  static constexpr int kBase = kQBytes + kListBytes + kMiscBytes + kBarBytes + 1024;  // + align
  static constexpr int stages_for(int r) {
    return ((int)kSmemBudget - kBase - 2 * buf_bytes(r)) / kStageBytes;
  }
  // Records per row and buffer: the most that leave four ring stages (else two).
  static constexpr int kRec = stages_for(4) >= 4   ? 4
                              : stages_for(3) >= 4 ? 3
                              : stages_for(2) >= 4 ? 2
                              : stages_for(2) >= 2 ? 2
                                                   : 1;
  static constexpr int kRecStride = rec_stride(kRec);
  static constexpr int kStagesFit = stages_for(kRec);
  static constexpr int kStages = kStagesFit > 8 ? 8 : kStagesFit;
  static constexpr bool kFits = kStages >= 2;
  // Byte offsets from the 1024-aligned base.
  static constexpr int kOffK = kQBytes;                                  // K ring
  static constexpr int kOffLs = kOffK + kStages * kStageBytes;           // list scores [rows][LS]
  static constexpr int kOffLi = kOffLs + kListStride * kRows * 4;        // list keys [rows][LS]
  static constexpr int kOffRs = kOffLi + kListStride * kRows * 4;        // [2][rows][kRecStride]
  static constexpr int kOffRj = kOffRs + 2 * kRows * kRecStride * 4;     // [2][kRec][rows]
  static constexpr int kOffRn = kOffRj + 2 * kRec * kRows * 4;           // [2][rows]
  static constexpr int kOffThr = kOffRn + 2 * kRows * 4;                 // [rows] (thr, item)
  static constexpr int kOffFlag = kOffThr + kRows * 8;                   // [2][filter warps]
  static constexpr int kOffBars = kOffFlag + 2 * kFilterWarps * 4;
  static constexpr size_t kSmem = (size_t)kOffBars + kBarBytes + 1024;
  static constexpr size_t kSmemLaunch = kSmem > kMinSmem ? kSmem : kMinSmem;
  static_assert(!kFits || kSmem <= kSmemBudget, "shared-memory layout");
  static_assert(!kFits || (kOffRs % 16 == 0 && (kRecStride * 4) % 16 == 0),
                "records are written as float4");
  static_assert(kOffBars % 8 == 0, "mbarrier alignment");
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN);
  // Start-address offset (16-byte units) of K step kk (16 bf16 columns).
  static constexpr uint32_t step_off(int kk) {
    return (uint32_t)(((kk * 16 / kRegionElems) * kRegionBytes + (kk * 16 % kRegionElems) * 2) >> 4);
  }
};

struct TcParams {
  const __nv_bfloat16* V;
  float* lse_all;  // with the all-key diagnostics: log-sum-exp over every key
  float c2;        // scale * log2(e)
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

// A row's top-k list is its line of shared memory: scores ls[..] and keys
// li[..].  For KCAP == kRegK it is a sorted list of kRegK slots, larger score
// first, kept in the insert thread's registers during an item and written
// here for the softmax and gather: the first kRegK - k slots hold +inf
// sentinels and the k real entries follow, so the k-th best is always the
// last slot.  For larger KCAP the k entries, from slot 3 of the line on,
// form a four-ary heap with the worst entry at the root: entry a is worse
// than entry b when a's score is smaller, or equal with a larger key; the
// root's score is the row's threshold.  Unused entries hold -inf and key -1.
template <int KCAP>
__device__ __forceinline__ int first_slot(int k) {
  return KCAP == kRegK ? kRegK - k : 0;
}

template <int KCAP>
__device__ __forceinline__ void list_reset(float* ls, int* li, int k) {
  if (KCAP == kRegK) {
#pragma unroll
    for (int t = 0; t < kRegK; ++t) {
      ls[t] = t < kRegK - k ? INFINITY : -INFINITY;
      li[t] = -1;
    }
  } else {
    for (int t = 0; t < k; ++t) {
      ls[t] = -INFINITY;
      li[t] = -1;
    }
  }
}

// (sa, ja) is worse than (sb, jb): smaller score, or equal score and larger
// key.  Padding entries (-inf, -1) are worse than every real entry.
__device__ __forceinline__ bool worse(float sa, int ja, float sb, int jb) {
  return sa < sb || (sa == sb && ja > jb);
}

// Four-ary heap (children of p: 4p+1 .. 4p+4).  H + 1 and J + 1 are 16-byte
// aligned, so each node's children are read as one float4 and one int4;
// children at or past n count as +inf (never the worst).  Put (s, j) at
// slot `pos` and sift it down to where all its children are no worse.
__device__ __forceinline__ void heap4_sift(float* H, int* J, int n, int pos, float s, int j) {
  for (;;) {
    const int c0 = 4 * pos + 1;
    if (c0 >= n) break;
    const float4 cs = *reinterpret_cast<const float4*>(H + c0);
    const int4 cj = *reinterpret_cast<const int4*>(J + c0);
    int c = c0;
    float ws = cs.x;
    int wj = cj.x;
    if (c0 + 1 < n && worse(cs.y, cj.y, ws, wj)) { c = c0 + 1; ws = cs.y; wj = cj.y; }
    if (c0 + 2 < n && worse(cs.z, cj.z, ws, wj)) { c = c0 + 2; ws = cs.z; wj = cj.z; }
    if (c0 + 3 < n && worse(cs.w, cj.w, ws, wj)) { c = c0 + 3; ws = cs.w; wj = cj.w; }
    if (!worse(ws, wj, s, j)) break;
    H[pos] = ws;
    J[pos] = wj;
    pos = c;
  }
  H[pos] = s;
  J[pos] = j;
}

// Heap of n entries -> sorted list, best first (heap sort: the worst entry
// is moved to the back, then the next worst, ...).
__device__ __forceinline__ void heap_to_sorted(float* H, int* J, int n) {
  for (int end = n - 1; end > 0; --end) {
    const float s = H[end];
    const int j = J[end];
    H[end] = H[0];
    J[end] = J[0];
    heap4_sift(H, J, end, 0, s, j);
  }
}

// Bit 16 r + u is set when score u of record r beats thr.
template <int NREC>
__device__ __forceinline__ uint64_t record_bits(const float* rs, int rn, float thr) {
  static_assert(NREC <= 4, "64-bit record mask");
  uint64_t m = 0;
#pragma unroll
  for (int r = 0; r < NREC; ++r) {
    if (r < rn) {
      const float4* src = reinterpret_cast<const float4*>(rs + r * 16);
      uint32_t b = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 x = src[q];
        b |= (x.x > thr ? 1u : 0u) << (4 * q);
        b |= (x.y > thr ? 1u : 0u) << (4 * q + 1);
        b |= (x.z > thr ? 1u : 0u) << (4 * q + 2);
        b |= (x.w > thr ? 1u : 0u) << (4 * q + 3);
      }
      m |= (uint64_t)b << (16 * r);
    }
  }
  return m;
}

// Next recorded score (in key order) that still beats thr; false when none
// is left.  rj: the row's record keys, record r at rj[r * kRows].
__device__ __forceinline__ bool next_candidate(uint64_t& m, const float* rs, const int* rj,
                                               float thr, float& s, int& j) {
  while (m) {
    const int b = __ffsll((long long)m) - 1;
    m &= m - 1;
    const float x = rs[b];  // record b >> 4, column b & 15
    if (x > thr) {
      s = x;
      j = rj[(b >> 4) * kRows] + (b & 15);
      return true;
    }
  }
  return false;
}

// Insertion for k <= kRegK: the insert warp keeps the row's list in
// registers for the whole item and takes one candidate per lane per round.
// A candidate beats the last slot (the k-th best); every slot compares
// itself and its neighbour with the candidate at once and keeps its entry,
// takes the candidate or takes its neighbour's entry, so a round is a fixed,
// short run of independent compares and selects instead of a chain of
// compare-and-swap steps (which measured 6-12% slower overall).  Records are
// visited in key order, so an equal score stays ahead of the candidate.
// Returns the new threshold.
template <int NREC>
__device__ __forceinline__ float insert_in_regs(float (&L)[kRegK], int (&J)[kRegK], const float* rs,
                                                const int* rj, int rn, float thr) {
  uint64_t m = record_bits<NREC>(rs, rn, thr);
  while (__any_sync(0xffffffffu, m != 0)) {
    float s = -INFINITY;
    int j = -1;
    const bool have = next_candidate(m, rs, rj, thr, s, j);
    if (!__any_sync(0xffffffffu, have)) break;
    if (have) {
      // The candidate goes in after every entry scoring at least as much
      // (an equal score came from an earlier key); the entries behind it
      // move down one slot and the last one drops out.  Every slot is
      // decided at once from its own comparison and its neighbour's.
      bool bt = false;  // the candidate beats the last slot
#pragma unroll
      for (int t = kRegK - 1; t >= 1; --t) {
        const bool bp = L[t - 1] >= s;
        const float nl = bt ? L[t] : (bp ? s : L[t - 1]);
        const int nj = bt ? J[t] : (bp ? j : J[t - 1]);
        L[t] = nl;
        J[t] = nj;
        bt = bp;
      }
      if (!bt) {
        L[0] = s;
        J[0] = j;
      }
    }
    thr = L[kRegK - 1];
  }
  return thr;
}

// Insertion for larger k: every recorded score that still beats the root of
// the row's heap replaces the root and sifts down (log4 k levels in shared
// memory, one 16-byte load of scores and one of keys per level, whatever the
// candidate's rank; a four-ary heap measured 1-5% faster for the whole
// kernel than a binary one at k = 45 and 64).  Returns the new threshold.
template <int NREC>
__device__ __forceinline__ float insert_heap(float* H, int* J, const float* rs, const int* rj,
                                             int rn, float thr, int k) {
  uint64_t m = record_bits<NREC>(rs, rn, thr);
  float s;
  int jn;
  while (next_candidate(m, rs, rj, thr, s, jn)) {
    heap4_sift(H, J, k, 0, s, jn);
    thr = H[0];
  }
  __syncwarp();
  return thr;
}

template <int D, int KCAP, bool DIAG>
__global__ void __launch_bounds__(kThreads, 1)
fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const TcParams p) {
  using C = Cfg<D, KCAP>;
  constexpr int kStages = C::kStages;
  constexpr int LS = C::kListStride, RS = C::kRecStride, NR = C::kRec;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte alignment of the swizzled tiles.
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* q_smem = base;
  unsigned char* k_smem = base + C::kOffK;
  float* ls = reinterpret_cast<float*>(base + C::kOffLs);
  int* li = reinterpret_cast<int*>(base + C::kOffLi);
  float* rec_s = reinterpret_cast<float*>(base + C::kOffRs);
  int* rec_j = reinterpret_cast<int*>(base + C::kOffRj);
  int* rec_n = reinterpret_cast<int*>(base + C::kOffRn);
  float* thr_row = reinterpret_cast<float*>(base + C::kOffThr);
  int* bflag = reinterpret_cast<int*>(base + C::kOffFlag);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::kOffBars);
  uint64_t* full = bars;                  // [kStages]  K tile landed
  uint64_t* empty = full + kStages;       // [kStages]  K tile consumed by the MMAs
  uint64_t* tfull = empty + kStages;      // [kNB]      accumulator ready
  uint64_t* tempty = tfull + kNB;         // [kNB]      accumulator copied out
  uint64_t* qfull = tempty + kNB;         // Q tile landed
  uint64_t* qempty = qfull + 1;           // Q tile no longer read (both MMA warps)
  uint64_t* mdone = qempty + 1;           // every MMA of this CTA finished
  uint64_t* rfull = mdone + 1;            // [filter warps][2] record buffer handed over
  uint64_t* rempty = rfull + 2 * kFilterWarps;  // [filter warps][2] record buffer inserted
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(rempty + 2 * kFilterWarps);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  static_assert((2 * kStages + 2 * kNB + 3 + 4 * kFilterWarps) * 8 + 8 <= C::kBarBytes,
                "barrier space");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(full + s), 1);
      mbar_init(smem_addr(empty + s), 1);
    }
    for (int b = 0; b < kNB; ++b) {
      mbar_init(smem_addr(tfull + b), 1);
      mbar_init(smem_addr(tempty + b), kFilterWarps);
    }
    mbar_init(smem_addr(qfull), 1);
    mbar_init(smem_addr(qempty), kMmaWarps);
    mbar_init(smem_addr(mdone), kMmaWarps);
    for (int b = 0; b < 2 * kFilterWarps; ++b) {
      mbar_init(smem_addr(rfull + b), 1);
      mbar_init(smem_addr(rempty + b), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  // Published thresholds start as (-inf, item 0); items count from 1, so a
  // value left in shared memory by an earlier kernel is never taken.
  for (int r = threadIdx.x; r < kRows; r += blockDim.x)
    reinterpret_cast<unsigned long long*>(thr_row)[r] = __float_as_uint(-INFINITY);
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

  if (warp < kFirstFilterWarp) {
   reg_dealloc<kRegsCtl>();
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
  } else if (warp <= kMmaWarps) {
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
   }  // warp 3: spare
  } else if (warp < kFirstInsertWarp) {
    reg_alloc<kRegsFilter>();
    // ------------------------------------------------------------- filters
    const int f = warp - kFirstFilterWarp;   // 0..7
    const int mt = f >> 2;                   // Q tile of this warp
    const int quarter = warp & 3;            // TMEM lanes this warp may read
    const int et = f * 32 + lane;            // this row's line in the item's row arrays
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    uint64_t* my_full = rfull + 2 * f;
    uint64_t* my_empty = rempty + 2 * f;
    float thr = -INFINITY;                   // lower bound of the row's k-th best score
    int rn = 0;                              // records of this row in the current buffer
    int cb = 0;                              // buffer being filled
    uint32_t handed0 = 0, handed1 = 0;       // batches handed over from each buffer
    int item = 0;                            // items started by this warp
    uint32_t tn = 0;
    bool ok = true;
    // Hand accumulator buffer b back to the MMA warps.
    auto release = [&](int b) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(tempty + b));
    };
    // When `on`, queue the 16 scores v (keys jb .. jb+15) as the row's next
    // record (needs rn < NR).
    auto push_if = [&](bool on, const float* v, int jb) {
      const uint32_t d = smem_addr(rec_s + (cb * kRows + et) * RS + rn * 16);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_shared_v4_if(on, d + 16 * q, v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
      st_shared_b32_if(on, smem_addr(rec_j + (cb * NR + rn) * kRows + et), jb);
      rn += on ? 1 : 0;
    };
    // Hand the current buffer to the insert warp (flags 1: the item's last
    // batch) and switch to the other one once its previous batch has been
    // inserted.
    auto hand_over = [&](int flags) {
      rec_n[cb * kRows + et] = rn;
      if (lane == 0) bflag[cb * kFilterWarps + f] = flags;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(my_full + cb));
      if (cb) ++handed1; else ++handed0;
      cb ^= 1;
      rn = 0;
      const uint32_t used = cb ? handed1 : handed0;
      if (used > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(smem_addr(my_empty + cb), (used - 1) & 1,
                                               abort_flag, p.timeout_ns)))
          ok = false;
      }
    };
    // The buffer not being filled holds no batch waiting to be inserted.
    auto other_free = [&]() -> bool {
      const uint32_t used = cb ? handed0 : handed1;
      return used == 0 ||
             __any_sync(0xffffffffu, mbar_test_wait(smem_addr(my_empty + (cb ^ 1)), (used - 1) & 1));
    };
    for (int64_t w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const WorkItem it = p.items[w % count];
      const bool tile_on = mt == 0 || (it.q1 - it.q0) > kBM;  // warp-uniform
      ++item;
      thr = -INFINITY;
      // all-key diagnostics: running maximum and sum of exp2(c2 (s - max))
      float dmax = -INFINITY, dsum = 0.f;
      const int ntiles = (it.j1 - it.j0 + kBN - 1) / kBN;
      for (int t = 0; t < ntiles; ++t, ++tn) {
        const int b = (int)(tn % kNB);
        const uint32_t use = tn / kNB;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(smem_addr(tfull + b), use & 1, abort_flag, p.timeout_ns))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (!tile_on) {
          release(b);
          continue;
        }
        {
          // The threshold the insert warp reached for this row, if it is
          // working on this item already.
          const unsigned long long tv =
              *reinterpret_cast<volatile unsigned long long*>(thr_row + 2 * et);
          if ((int)(tv >> 32) == item) thr = fmaxf(thr, __uint_as_float((unsigned)tv));
        }
        const uint32_t ta = tmem + lane_base + b * (kMT * kBN) + mt * kBN;
        const int jt = it.j0 + t * kBN;            // key of column 0
        const int valid = min(kBN, it.j1 - jt);
        // The row's 128 scores in registers; the accumulator goes back to
        // the MMA warps at once.
        float v[kBN / 32][32];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(ta + c * 32, v[c]);
        tmem_ld_wait_all();
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) reg_fence(v[c]);
        release(b);
        if (valid < kBN) {
#pragma unroll
          for (int c = 0; c < kBN / 32; ++c)
#pragma unroll
            for (int u = 0; u < 32; ++u)
              if (c * 32 + u >= valid) v[c][u] = -INFINITY;
        }
        float gm[kBN / 16];  // maxima of the eight 16-key groups
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          gm[2 * c] = max16(v[c]);
          gm[2 * c + 1] = max16(v[c] + 16);
        }
        uint32_t mask = 0;
#pragma unroll
        for (int g = 0; g < kBN / 16; ++g) mask |= (gm[g] > thr ? 1u : 0u) << g;
        if constexpr (DIAG) {
          // Softmax normaliser over every key of the graph (online: the sum
          // is rescaled whenever the running maximum rises).
          const float tm = fmax3(fmax3(gm[0], gm[1], gm[2]), fmax3(gm[3], gm[4], gm[5]),
                                 fmaxf(gm[6], gm[7]));
          if (tm > dmax) {
            dsum *= exp2f((dmax - tm) * p.c2);
            dmax = tm;
          }
          if (dmax > -INFINITY) {
            const float off = dmax * p.c2;
#pragma unroll
            for (int c = 0; c < kBN / 32; ++c)
#pragma unroll
              for (int u = 0; u < 32; ++u) dsum += exp2f(fmaf(v[c][u], p.c2, -off));
          }
        }
        const uint32_t todo = __reduce_or_sync(0xffffffffu, mask);
        if (todo) {
          // Only the groups that some lane keeps issue their (predicated)
          // stores: in the steady state a few of the eight.  The branch on
          // a group's bit is warp-uniform and the loop is unrolled, so the
          // scores stay statically indexed registers.
          if (!__any_sync(0xffffffffu, rn + __popc(mask) > NR)) {
#pragma unroll
            for (int g = 0; g < kBN / 16; ++g)
              if (todo & (1u << g)) push_if((mask >> g) & 1u, v[g >> 1] + (g & 1) * 16, jt + g * 16);
          } else {
            // some lane runs out of records within this tile: hand batches
            // over between groups
#pragma unroll
            for (int g = 0; g < kBN / 16; ++g) {
              if (todo & (1u << g)) {
                const bool on = (mask >> g) & 1u;
                if (__any_sync(0xffffffffu, on && rn == NR)) hand_over(0);
                push_if(on, v[g >> 1] + (g & 1) * 16, jt + g * 16);
              }
            }
          }
          // Hand a batch over early once enough rows hold records and the
          // insert warp has nothing else queued.
          if (ok && __popc(__ballot_sync(0xffffffffu, rn > 0)) >= kHandLanes && other_free())
            hand_over(0);
        }
        if (!ok) break;
      }
      if (!ok) break;
      if constexpr (DIAG) {
        const int i = it.q0 + mt * kBM + quarter * 32 + lane;
        if (tile_on && i < it.q1)
          p.lse_all[(int64_t)i * p.H + (int)(w / count)] = (dmax * p.c2 + log2f(dsum)) * 0.6931471805599453f;
      }
      hand_over(1);  // the item's last batch
    }
  } else {
    reg_dealloc<kRegsInsert>();
    // ----------------------------------------------------------- inserters
    const int f = warp - kFirstInsertWarp;             // paired filter warp f
    const int mt = f >> 2;
    const int quarter = (f + kFirstFilterWarp) & 3;    // that filter's lane quarter
    const int row = quarter * 32 + lane;               // row within the Q tile
    const int et = f * 32 + lane;
    float* L = ls + et * LS;
    int* J = li + et * LS;
    uint64_t* my_full = rfull + 2 * f;
    uint64_t* my_empty = rempty + 2 * f;
    const int64_t HD = (int64_t)p.H * D;
    int cb = 0;
    uint32_t taken0 = 0, taken1 = 0;  // batches taken from each buffer
    int item_no = 0;
    bool ok = true;
    for (int64_t w = blockIdx.x; w < total && ok; w += gridDim.x) {
      const int h = (int)(w / count);
      const WorkItem it = p.items[w % count];
      const bool tile_on = mt == 0 || (it.q1 - it.q0) > kBM;
      const int i = it.q0 + mt * kBM + row;
      float RL[kRegK];
      int RJ[kRegK];
      if constexpr (KCAP == kRegK) {
#pragma unroll
        for (int t = 0; t < kRegK; ++t) {
          RL[t] = t < kRegK - p.k ? INFINITY : -INFINITY;
          RJ[t] = -1;
        }
      } else {
        list_reset<KCAP>(L + 3, J + 3, p.k);
      }
      float thr = -INFINITY;
      ++item_no;
      for (;;) {
        const uint32_t tk = cb ? taken1 : taken0;
        if (!__all_sync(0xffffffffu,
                        mbar_wait(smem_addr(my_full + cb), tk & 1, abort_flag, p.timeout_ns))) {
          ok = false;
          break;
        }
        const int rn = rec_n[cb * kRows + et];
        const int flags = bflag[cb * kFilterWarps + f];
        const float* rs = rec_s + (cb * kRows + et) * RS;
        const int* rj = rec_j + cb * NR * kRows + et;
        if constexpr (KCAP == kRegK)
          thr = insert_in_regs<NR>(RL, RJ, rs, rj, rn, thr);
        else
          thr = insert_heap<NR>(L + 3, J + 3, rs, rj, rn, thr, p.k);
        {
          // Publish the row's threshold with the item it belongs to, in one
          // 8-byte store, for the filter to raise its own.
          *reinterpret_cast<volatile unsigned long long*>(thr_row + 2 * et) =
              ((unsigned long long)(unsigned)item_no << 32) | __float_as_uint(thr);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(my_empty + cb));
        if (cb) ++taken1; else ++taken0;
        cb ^= 1;
        if (flags & 1) break;
      }
      if (!ok) break;
      if constexpr (KCAP == kRegK) {
#pragma unroll
        for (int t = 0; t < kRegK; ++t) {
          L[t] = RL[t];
          J[t] = RJ[t];
        }
      }
      if (tile_on && i < it.q1) {
        if (KCAP != kRegK) heap_to_sorted(L + 3, J + 3, p.k);
        const float* Lf = L + (KCAP == kRegK ? first_slot<KCAP>(p.k) : 3);
        const int* Jf = J + (KCAP == kRegK ? first_slot<KCAP>(p.k) : 3);
        int cnt = 0;
        while (cnt < p.k && Jf[cnt] >= 0) ++cnt;
        // Softmax over the kept scaled scores, lse, weighted sum of V rows.
        const int64_t rowg = (int64_t)i * p.H + h;
        const float mx = p.scale * Lf[0];
        float sum = 0.f;
        for (int t = 0; t < cnt; ++t) sum += expf(p.scale * Lf[t] - mx);
        const float lse_v = mx + logf(sum);
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          constexpr int CW = D < 32 ? D : 32;
          float o[CW];
#pragma unroll
          for (int u = 0; u < CW; ++u) o[u] = 0.f;
          for (int t = 0; t < cnt; ++t) {
#ifdef KMIP_DEBUG_BOUNDS
            if (Jf[t] < it.j0 || Jf[t] >= it.j1) {
              record_status(p.status, KMIP_ERR_BAD_INDEX);
              continue;
            }
#endif
            const float pw = expf(p.scale * Lf[t] - lse_v);
            const __nv_bfloat16* vr = p.V + (int64_t)Jf[t] * HD + h * D + c0;
#pragma unroll
            for (int u = 0; u < CW; u += 8) {
              float fv[8];
              Vec<__nv_bfloat16>::load(vr + u, fv);
#pragma unroll
              for (int e = 0; e < 8; ++e) o[u + e] = fmaf(pw, fv[e], o[u + e]);
            }
          }
#pragma unroll
          for (int u = 0; u < CW; u += 8) Vec<__nv_bfloat16>::store(p.out + rowg * D + c0 + u, o + u);
        }
        for (int t = 0; t < p.k; ++t) p.idx[rowg * p.k + t] = t < cnt ? Jf[t] : -1;
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

template <int D, int KCAP, bool DIAG>
cudaError_t launch_cfg(const FwdArgs& a, cudaStream_t stream) {
  using C = Cfg<D, KCAP>;
  static_assert(C::kFits, "shared memory budget");
  CUtensorMap mq, mk;
  if (!make_map<D>(&mq, a.Q, a.N, a.H) || !make_map<D>(&mk, a.K, a.N, a.H))
    return cudaErrorInvalidValue;
  auto kern = fwd_tc_kernel<D, KCAP, DIAG>;
  // The warpgroups' register split draws on the launch allocation: refuse
  // to launch a build whose kernel was given fewer registers.
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return cudaErrorInvalidDeviceFunction;
  if (fa.numRegs < kLaunchRegs) return cudaErrorNotSupported;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmemLaunch);
  if (e != cudaSuccess) return e;
  const int64_t units = (int64_t)a.H * a.max_items;
  const int sms = device_sm_count();
  const int grid = (int)(units < sms ? units : sms);
  TcParams p{static_cast<const __nv_bfloat16*>(a.V), a.lse_all, a.scale * 1.4426950408889634f,
             a.items, a.count, a.H, a.k, a.scale,
             static_cast<__nv_bfloat16*>(a.out), a.idx, a.lse, a.status, kTimeoutNs};
  kern<<<grid, kThreads, C::kSmemLaunch, stream>>>(mq, mk, p);
  return cudaGetLastError();
}

template <int D, int KCAP>
cudaError_t launch_k(const FwdArgs& a, cudaStream_t stream) {
  if constexpr (Cfg<D, KCAP>::kFits) {
    if (a.lse_all) return launch_cfg<D, KCAP, true>(a, stream);
    return launch_cfg<D, KCAP, false>(a, stream);
  }
  return cudaErrorNotSupported;
}

template <int D>
cudaError_t launch_d(const FwdArgs& a, cudaStream_t stream) {
  if (a.k <= kRegK) return launch_k<D, kRegK>(a, stream);
  if (a.k <= 32) return launch_k<D, 32>(a, stream);
  if (a.k <= 48) return launch_k<D, 48>(a, stream);
  return launch_k<D, 64>(a, stream);
}

}  // namespace

template <int D>
bool fits_d(int k) {
  if (k <= kRegK) return Cfg<D, kRegK>::kFits;
  if (k <= 32) return Cfg<D, 32>::kFits;
  if (k <= 48) return Cfg<D, 48>::kFits;
  return Cfg<D, 64>::kFits;
}

// Shapes whose lists, record buffers, Q tiles and at least two K stages fit
// in shared memory; other shapes run the fp32-FMA forward.
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
