/*
 * kmip.h -- C ABI of libkmip: k-Maximum-Inner-Product (k-MIP) attention for
 * graph transformers on NVIDIA B200 (sm_100a).
 *
 * The operation (k-Maximum Inner Product Attention for Graph Transformers
 * and the Expressive Power of GraphGPS, Abstract: each query attends only to
 * the keys whose inner product with it is among the k largest, and the
 * scores are computed without ever storing them all, so memory grows
 * linearly with the node count): for query node i of graph g and head h,
 *
 *   s_j  = Q[i,h,:] . K[j,h,:]          for every node j of graph g
 *   S    = the k_eff = min(k, n_g) keys with the largest s_j
 *          (larger s first; equal s -> smaller node index first)
 *   lse  = log sum_{j in S} exp(scale * s_j)          (natural log)
 *   p_j  = exp(scale * s_j - lse)
 *   out  = sum_{j in S} p_j V[j,h,:]
 *
 * and its backward pass through the selected scores (the pages time a
 * "training setting", Tables 10-12 and 16; the selection is piecewise
 * constant and gets no gradient):
 *
 *   dP_j = dOut . V_j,  D = sum_j p_j dP_j,  dS_j = p_j (dP_j - D)
 *   dQ_i = scale sum_j dS_j K_j,  dK_j += scale dS_j Q_i,  dV_j += p_j dOut_i
 *
 * Graphs: a batch of graphs is a block-diagonal node set.  Graph g owns the
 * contiguous node range [graph_offsets[g], graph_offsets[g+1]); a query only
 * ever selects keys of its own graph.  Every node of the graph, including
 * the query node itself, is a candidate key.
 *
 * Memory: the N x N score matrix is never materialised; scores live in
 * tensor memory / registers only.  The library's own device memory is a
 * work list of O(N / q + G) 16-byte items per forward call (q = 256 queries
 * per item on the tensor-core path, 128 otherwise; the same items serve
 * every head), and the deterministic backward's sort scratch.  Both are
 * stream-ordered allocations from a memory pool the library creates on each
 * device it is called on (cudaMemPoolCreate; the device's default pool is
 * not touched), released on the same stream.  The pool keeps, between
 * calls, the most memory it has reserved so far (about the largest scratch
 * taken from it), so a loop of calls maps device memory only once.
 *
 * Conventions common to every call:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device
 *     (the device of `stream`), owned by the caller; the library keeps no
 *     pointer after a call returns.
 *   - Q, K, V, dOut, out are [N, H, d] row-major (node-major, heads
 *     interleaved: the layout a Linear of width H*d produces), of the element
 *     type `dtype`, 16-byte aligned.  idx is [N, H, k] int32, lse is [N, H]
 *     fp32; dQ, dK, dV are [N, H, d] fp32.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream).
 *     A non-OK status returned by a call means nothing was enqueued.
 *   - Errors found on the device (malformed graph_offsets, an index out of
 *     range, a pipeline wait that ran out) are recorded in a per-device
 *     status word and reported by kmip_get_status(); outputs of the affected
 *     work are left untouched.
 *   - Supported: N in [0, 2^31 - 1]; 1 <= H <= 64; d in {16, 32, 64, 128};
 *     1 <= k <= 64; scale finite and > 0.
 */
#ifndef KMIP_H
#define KMIP_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream (a cudaStream_t); NULL means the legacy default stream. */
typedef void* kmip_stream_t;

typedef enum {
  KMIP_BF16 = 0, /* bfloat16 inputs; scores accumulated in fp32 */
  KMIP_F32 = 1   /* fp32 inputs; scores by fp32 fused multiply-add */
} kmip_dtype_t;

typedef enum {
  KMIP_OK = 0,
  KMIP_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad scale */
  KMIP_ERR_UNSUPPORTED = 2, /* d, k or H outside the supported set */
  KMIP_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  KMIP_ERR_BAD_OFFSETS = 4, /* device: graph_offsets not 0 = o_0 <= ... <= o_G = N */
  KMIP_ERR_TIMEOUT = 5,     /* device: a pipeline wait ran out (kernel gave up) */
  KMIP_ERR_BAD_INDEX = 6,   /* device: idx entry outside [-1, N) in the backward */
  KMIP_ERR_SCRATCH_LIMIT = 7 /* kmip_attn_fwd_noalloc: work list larger than its fixed array */
} kmip_status_t;

/*
 * Forward pass.
 *   Q, K, V        [N, H, d] of `dtype` (device).
 *   graph_offsets  int32 [num_graphs + 1] (device): offsets[0] = 0,
 *                  offsets[num_graphs] = N, non-decreasing (empty graphs are
 *                  allowed).  NULL means one graph of N nodes (num_graphs is
 *                  then ignored).  Checked on the device: a malformed array
 *                  records KMIP_ERR_BAD_OFFSETS and no output is written.
 *   N, H, d, k     sizes; scale multiplies the scores inside the softmax
 *                  (selection uses the unscaled scores; equivalent for scale > 0).
 *   out            [N, H, d] of `dtype` (device), overwritten.
 *   idx            [N, H, k] int32 (device), overwritten: the kept keys as
 *                  global node indices, larger score first, padded with -1
 *                  when the graph has fewer than k nodes.
 *   lse            [N, H] fp32 (device), overwritten: log-sum-exp of the
 *                  scaled kept scores (needed by the backward).
 * bf16 inputs run on the tcgen05 tensor-core path (scores exact products,
 * fp32 accumulation); fp32 inputs run an fp32 FMA path.
 * Returns KMIP_OK, KMIP_ERR_INVALID_ARG, KMIP_ERR_UNSUPPORTED or KMIP_ERR_CUDA.
 */
kmip_status_t kmip_attn_fwd(const void* Q, const void* K, const void* V,
                            const int32_t* graph_offsets, int64_t N, int H, int d, int k,
                            float scale, void* out, int32_t* idx, float* lse,
                            kmip_stream_t stream, int num_graphs, kmip_dtype_t dtype);

/*
 * Forward pass that allocates no device memory.  (No counterpart in the
 * pages: this is an interface variant for callers, not part of the method.)
 *
 * Same arguments, outputs and results as kmip_attn_fwd.  kmip_attn_fwd
 * takes its work list from the library's memory pool on each call; this
 * variant is for callers that cannot let a library allocate: a framework
 * whose own memory pool already holds the GPU's memory, a driver or
 * virtualised device without stream-ordered memory pools, or a loop that
 * must not enter the allocator once it is running.  The work list lives in a
 * fixed device array inside the library (about 1 MiB, held on every GPU that
 * loads the library until the process exits); no cudaMalloc, cudaFree or
 * allocating library routine is called.
 *
 * Limit: ceil(N / 256) + num_graphs <= 65536 work items for bf16 inputs on
 * the tensor-core path, ceil(N / 128) + num_graphs <= 65536 otherwise
 * (num_graphs counts as 1 when graph_offsets is NULL); larger calls return
 * KMIP_ERR_SCRATCH_LIMIT with nothing enqueued.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and so should come before any stream capture.
 * Every call on a device shares the one array and it keeps the last call's
 * contents; nothing in it needs to be zero, since each call writes the whole
 * work list it reads.  Calls whose work overlaps on the GPU (on different
 * streams, or from host threads that do not order them) race on the array
 * and must be serialised by the caller.
 */
kmip_status_t kmip_attn_fwd_noalloc(const void* Q, const void* K, const void* V,
                                    const int32_t* graph_offsets, int64_t N, int H, int d,
                                    int k, float scale, void* out, int32_t* idx, float* lse,
                                    kmip_stream_t stream, int num_graphs, kmip_dtype_t dtype);

/*
 * Forward pass with the all-key diagnostics (k-Maximum Inner Product
 * Attention for Graph Transformers ..., Figure 8: how far k-MIP attention is
 * from full softmax attention).  Same arguments and results as
 * kmip_attn_fwd, plus
 *   lse_all        [N, H] fp32 (device), overwritten: the log-sum-exp of the
 *                  scaled scores over EVERY key of the query's graph, i.e.
 *                  the normaliser of full softmax attention.
 * exp(lse - lse_all) is the share of the full softmax weight that the k kept
 * keys carry (1 when k covers the graph).  The scores are the same ones the
 * selection uses; the sum is accumulated in fp32 with one exp2 per score, so
 * this call is slower than kmip_attn_fwd.  lse_all may not be NULL when
 * N > 0 (KMIP_ERR_INVALID_ARG).
 */
kmip_status_t kmip_attn_fwd_diag(const void* Q, const void* K, const void* V,
                                 const int32_t* graph_offsets, int64_t N, int H, int d, int k,
                                 float scale, void* out, int32_t* idx, float* lse,
                                 float* lse_all, kmip_stream_t stream, int num_graphs,
                                 kmip_dtype_t dtype);

/*
 * Attention over given key sets: the softmax and V-gather stage of the
 * forward on its own (k-Maximum Inner Product Attention for Graph
 * Transformers ..., Abstract: once a query's k keys are chosen the layer is
 * softmax attention over them).  For a caller that keeps a selection across
 * calls, and the gather stage measured by itself.
 *   Q, K, V        [N, H, d] of `dtype` (device).
 *   idx            [N, H, k] int32 (device): the kept keys of each (query,
 *                  head), -1 = padding (as kmip_attn_fwd writes it).  The
 *                  scores of the kept keys are recomputed from Q and K.
 *   out            [N, H, d] of `dtype` (device), overwritten.
 *   lse            [N, H] fp32 (device), overwritten (-inf for a row whose
 *                  entries are all -1).
 * An idx entry outside [-1, N) records KMIP_ERR_BAD_INDEX on the device and
 * is skipped.  Returns KMIP_OK, KMIP_ERR_INVALID_ARG, KMIP_ERR_UNSUPPORTED or
 * KMIP_ERR_CUDA.
 */
kmip_status_t kmip_attn_gather(const void* Q, const void* K, const void* V, const int32_t* idx,
                               int64_t N, int H, int d, int k, float scale, void* out,
                               float* lse, kmip_stream_t stream, kmip_dtype_t dtype);

/*
 * Backward pass.
 *   dOut           [N, H, d] of `dtype` (device): gradient of the loss w.r.t. out.
 *   Q, K, V        the forward's inputs; idx, lse the forward's outputs.
 *   dQ, dK, dV     [N, H, d] fp32 (device), overwritten (the library zeroes
 *                  dK and dV itself before scattering into them).
 * dK and dV are accumulated with fp32 atomics, so their bits may differ from
 * run to run in the last places; dQ is deterministic.  An idx entry outside
 * [-1, N) records KMIP_ERR_BAD_INDEX on the device and is skipped.
 * Returns KMIP_OK, KMIP_ERR_INVALID_ARG, KMIP_ERR_UNSUPPORTED or KMIP_ERR_CUDA.
 */
kmip_status_t kmip_attn_bwd(const void* dOut, const void* Q, const void* K, const void* V,
                            const int32_t* idx, const float* lse, float* dQ, float* dK,
                            float* dV, kmip_stream_t stream, int64_t N, int H, int d, int k,
                            float scale, kmip_dtype_t dtype);

/*
 * Backward pass with bitwise reproducible gradients.  Same arguments and
 * results as kmip_attn_bwd, computed without atomic additions: the kept keys
 * are sorted by (key, head) with a stable radix sort, and each key's dK and
 * dV rows are summed by one warp over its queries in the order of their
 * positions in idx, so repeated calls on the same inputs return identical
 * bits.  Takes O(N H k) scratch (about 28 bytes per kept key plus 4 per
 * (node, head)) from the library's memory pool (see Memory above) and
 * releases it on the same stream.  Returns KMIP_ERR_UNSUPPORTED when
 * N H k >= 2^32 - 1 or the sort's scans would exceed 2^24 entries
 * (N H k > about 2.7e8); otherwise as kmip_attn_bwd.
 */
kmip_status_t kmip_attn_bwd_deterministic(const void* dOut, const void* Q, const void* K,
                                          const void* V, const int32_t* idx, const float* lse,
                                          float* dQ, float* dK, float* dV, kmip_stream_t stream,
                                          int64_t N, int H, int d, int k, float scale,
                                          kmip_dtype_t dtype);

/*
 * Synchronises `stream`, then returns and clears the current device's status
 * word (the first device-side error recorded since the last call), or
 * KMIP_ERR_CUDA if the synchronisation itself failed.
 */
kmip_status_t kmip_get_status(kmip_stream_t stream);

/*
 * Which forward kernel kmip_attn_fwd runs for these sizes: 1 = the tcgen05
 * tensor-core kernel (bf16 inputs whose top-k lists, record buffers, Q tiles
 * and two K stages fit in shared memory: d = 16 or 32 with any k <= 64,
 * d = 64 with k <= 48, d = 128 with k <= 16), 0 = the fp32-FMA kernel (fp32
 * inputs and the other bf16 shapes), -1 = unsupported arguments.  Pure host
 * logic; touches no device.
 */
int kmip_fwd_path(int d, int k, kmip_dtype_t dtype);

/*
 * The library's scratch memory on the current device (see Memory above):
 * *reserved = device memory the library's pool holds now (in use or kept
 * for the next call), *used_high = the most it had in use at once since the
 * pool was created or since the last call with reset_high != 0 (which
 * restarts that count from what is in use now).  Both are 0 before the
 * first allocating call on the device.  Either pointer may be NULL.
 * Returns KMIP_OK, or KMIP_ERR_CUDA if the pool could not be queried.
 */
kmip_status_t kmip_scratch_usage(uint64_t* reserved, uint64_t* used_high, int reset_high);

/*
 * Returns the memory the library's pool on the current device keeps but
 * does not use to the device (cudaMemPoolTrimTo), and lets the pool keep
 * nothing between calls until the next allocating call raises that again.
 * Call it once the streams that ran library calls on the device have been
 * synchronised: scratch still in use by queued work is not returned.
 * Returns KMIP_OK (also when the pool does not exist yet) or KMIP_ERR_CUDA.
 */
kmip_status_t kmip_scratch_trim(void);

/* Static, human-readable name of a status code (never NULL). */
const char* kmip_error_string(kmip_status_t status);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
int kmip_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KMIP_H */
