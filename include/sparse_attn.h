/*
 * sparse_attn.h — C ABI of the B200 (sm_100a) block-sparse attention library.
 *
 * Two calls make up the path:
 *
 *   sparse_attn_plan  — stage 1 of the two-stage filter in the SpargeAttn abstract
 *                       ("rapidly and accurately predict the attention map"):
 *                       mean-pool Q and K over 64-token blocks, softmax of the
 *                       pooled scores, and per query block keep the fewest key
 *                       blocks whose cumulative attention energy reaches tau —
 *                       the per-row dynamic threshold of the DynSparse article
 *                       ("Training-free sparse attention based on cumulative
 *                       energy filtering", method paragraph).
 *   sparse_attn_fwd   — stage 2: FlashAttention-style forward over the kept
 *                       blocks only, plus the online-softmax-aware filter of the
 *                       SpargeAttn abstract (second stage): skip P.V of a block
 *                       whose rows all satisfy rowmax(S_blk) - running_max < lambda.
 *
 * Conventions shared by every call:
 *   - Q, K, V, O are bf16, row-major [B, H, N, d] (d contiguous), device memory,
 *     16-byte aligned. d is 64 or 128. block must be 64.
 *   - Nb = ceil(N / 64) blocks per head; the last block may be ragged.
 *   - A query tile is 128 rows = two 64-row query blocks of one (b, h), paired by
 *     sparse_attn_plan (or (2t, 2t+1) without a plan order); Tq = ceil(Nb / 2)
 *     tiles per head, B*H*Tq tiles in all.
 *   - All pointers are owned by the caller. The library allocates no memory and
 *     keeps no state across calls except one device-side error word per GPU.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every call is asynchronous on that stream; results are ready when it is.
 *   - Argument errors are detected on the host before anything is launched and
 *     return a status; nothing is written then. A failed launch returns
 *     SA_ERR_CUDA. Device-side checks (a wait that timed out, an index out of
 *     range) never trap: the kernel stops its tile, records a code in the
 *     device error word and returns; read it with sparse_attn_device_error.
 */
#ifndef SPARSE_ATTN_H
#define SPARSE_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SA_OK = 0,
  SA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, tau outside (0,1], NaN, misaligned pointer */
  SA_ERR_UNSUPPORTED = 2,  /* d not in {64,128}, block != 64, Nb > 4096, B*H > 65535 */
  SA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than sparse_attn_plan_workspace_size */
  SA_ERR_CUDA = 4,         /* a CUDA runtime/driver call or a launch failed */
  SA_ERR_DEVICE_CHECK = 5  /* the device error word was set (see sparse_attn_device_error) */
} sa_status;

typedef struct {
  int32_t B;     /* batch */
  int32_t H;     /* heads */
  int32_t N;     /* tokens per head, >= 1 */
  int32_t d;     /* head dim, 64 or 128 */
  int32_t block; /* mask block size, must be 64 */
} sa_shape;

/* Bytes of device workspace sparse_attn_plan needs for shape s: pooled Q and K
 * (fp32 [B,H,Nb,d] each), an 8-byte sort key and a ceil(Nb/32)-word kept-set
 * bitset per query block, above about 1,200 blocks per head (where the pairing's
 * copy of the bitsets no longer fits in shared memory) that copy, and the pooled
 * scores of as many 128-query-block strips (128 rows of ceil(Nb/32)*32 floats) as
 * fit in 64 MiB, at least one (the plan computes and selects the strips batch by
 * batch); each region 256-byte aligned. 0 if the shape is invalid. */
size_t sparse_attn_plan_workspace_size(sa_shape s);

/* Number of 128-row query tiles, B*H*ceil(Nb/2); `work` holds two entries per
 * tile. 0 if the shape is invalid. */
int64_t sparse_attn_num_tiles(sa_shape s);

/* Stage 1: block mask from mean-pooled Q and K.
 *
 *   Q, K      device bf16 [B,H,N,d]
 *   tau       recall threshold in (0, 1]: per query block i, the kept set is the
 *             shortest prefix of key blocks sorted by pooled probability
 *             (descending, ties to the lower index) whose sum reaches tau times
 *             the row sum. tau = 1 keeps every block with a finite pooled score.
 *   scale     softmax scale of the pooled scores (use the attention's, 1/sqrt(d))
 *   causal    nonzero: key block j > i is excluded from row i's softmax
 *   mask      out, device uint8 [B,H,Nb,Nb]: 1 = kept
 *   count     out, device int32 [B,H,Nb]: kept blocks per query block (>= 1)
 *   idx       out, device int32 [B,H,Nb,Nb] or NULL: kept key blocks in ascending
 *             order in the first count[..] entries of each row; the rest of the
 *             row is left untouched
 *   work      out, device int32 [2 * sparse_attn_num_tiles(s)] or NULL: the query
 *             tiles in execution order, two global query-block ids per tile
 *             ((b*H + h)*Nb + i; the second is -1 when a head has an odd block
 *             count). Every query block appears exactly once. Within a head,
 *             blocks are paired so that the two kept sets overlap (sorted by two
 *             MinHash signatures of the kept set, then, in up to six rounds, blocks
 *             that pick each other as the best match among the 32 unpaired blocks
 *             within 16 places in that order are paired, the rest in order), and
 *             the head's tiles are ranked by decreasing union size (longest
 *             first). Heads are taken in
 *             ascending (b,h) order in groups of G consecutive heads, G being the
 *             most heads whose K and V together fit in 64 MB (at least 1); within a
 *             group the tiles are interleaved by rank (rank 0 of every head of the
 *             group, then rank 1, ...), so the longest tiles of all of the group's
 *             heads start first. Deterministic for a given mask.
 *   workspace device scratch of at least sparse_attn_plan_workspace_size(s) bytes,
 *             256-byte aligned; its contents on entry do not matter
 */
sa_status sparse_attn_plan(const void* Q, const void* K, sa_shape s, float tau, float scale,
                           int32_t causal, uint8_t* mask, int32_t* count, int32_t* idx,
                           int32_t* work, void* workspace, size_t workspace_bytes, void* stream);

/* sparse_attn_plan with one recall threshold per head: head (b, h) keeps, per
 * query block, the shortest prefix of its sorted pooled probabilities reaching
 * tau[b*H + h] times the row sum. This is the per-head, per-call threshold of an
 * SNR-guided sparsity schedule (iCATS abstract: the sparsity follows the
 * denoising timestep). tau is a DEVICE array of B*H floats, 4-byte aligned, read
 * on the stream. A value outside (0, 1] (NaN included) cannot be checked on the
 * host: that head then keeps every block with a finite score (as tau = 1), and
 * bit 2 of the device error word is set. All other arguments, outputs and
 * errors are those of sparse_attn_plan. */
sa_status sparse_attn_plan_heads(const void* Q, const void* K, sa_shape s, const float* tau, float scale,
                                 int32_t causal, uint8_t* mask, int32_t* count, int32_t* idx,
                                 int32_t* work, void* workspace, size_t workspace_bytes, void* stream);

/* Stage 2: sparse attention over the kept blocks, with the lambda P.V filter.
 *
 *   Q, K, V   device bf16 [B,H,N,d]
 *   mask      device uint8 [B,H,Nb,Nb] (nonzero = kept), e.g. from sparse_attn_plan;
 *             with causal, entries j > i are ignored
 *   work      device int32 [2 * num_tiles]: query-block pairs from sparse_attn_plan, or
 *             NULL for the natural pairs (2t, 2t+1) of each head. Each entry must be
 *             a global query-block id < B*H*Nb (or -1 as the second of a pair), both
 *             of a pair in one head, every block exactly once; a tile whose entry is
 *             out of range is skipped and sets the device error word.
 *   lambda    threshold in natural-log units of the scaled scores. For each query
 *             block and kept key block (ascending order), the block's P.V is skipped
 *             when every row that sees a key of the block has
 *             rowmax(S_blk) - m < lambda (m = running max before the block); the
 *             block still updates the running max and the softmax denominator.
 *             -INFINITY turns the filter off. NaN is rejected.
 *   scale     softmax scale (1/sqrt(d) for standard attention), finite, > 0
 *   causal    nonzero: key token s is visible to query token t only if s <= t
 *   O         out, device bf16 [B,H,N,d]. A row with no visible key is written as 0.
 *   stats     device int64[4] or NULL; zeroed, then filled with: kept (query block,
 *             key block) pairs visited, pairs whose P.V was skipped by lambda,
 *             128x64 score tiles computed, 128x64 P.V tiles computed
 *
 * If a bounded device wait gives up (a pipeline stalled for seconds; this does
 * not happen in a healthy run), the tile stops, records the timeout in the
 * device error word and leaves its rows of O unwritten: O is undefined for
 * those rows. A caller that needs to know checks sparse_attn_device_error after
 * the stream has finished.
 */
sa_status sparse_attn_fwd(const void* Q, const void* K, const void* V, sa_shape s,
                          const uint8_t* mask, const int32_t* work, float lambda, float scale,
                          int32_t causal, void* O, int64_t* stats, void* stream);

/* Stage 2 with the in-operator cumulative-energy P.V filter instead of the lambda
 * test (DynSparse article: keep a fixed recall of the attention energy, with a
 * threshold that follows the cumulative energy the FlashAttention operator
 * already holds; the formula below is this library's reading of it).
 *
 *   recall    in (0, 1]. Per row r, l_r is the running softmax sum (the energy of
 *             the keys seen so far) and sk_r the part of it whose P.V was skipped,
 *             both relative to the running max. For each query block and kept key
 *             block (ascending order), with e_r the block's energy in row r and
 *             alpha_r the rescale to the new running max, the block's P.V is
 *             skipped when every row that sees a key of the block has
 *             sk_r*alpha_r + e_r <= (1 - recall) * (l_r*alpha_r + e_r); the
 *             block always enters l, and enters sk only when skipped. Every row
 *             then keeps at least the fraction `recall` of the energy of the
 *             blocks it visits. recall = 1 skips only blocks of zero energy.
 *             NaN or a value outside (0, 1] is rejected.
 *   stats     as sparse_attn_fwd; entry 1 counts the pairs skipped by this test.
 *
 * All other arguments, outputs and errors are those of sparse_attn_fwd. */
sa_status sparse_attn_fwd_recall(const void* Q, const void* K, const void* V, sa_shape s,
                                 const uint8_t* mask, const int32_t* work, float recall, float scale,
                                 int32_t causal, void* O, int64_t* stats, void* stream);

/* P.V filter selectors of sparse_attn_fwd_decisions. */
typedef enum {
  SA_FILTER_LAMBDA = 0,  /* the lambda test of sparse_attn_fwd; value = lambda (-INFINITY = off) */
  SA_FILTER_RECALL = 1   /* the cumulative-energy test of sparse_attn_fwd_recall; value = recall */
} sa_filter;

/* Stage 2 that also records the P.V filter's decisions, for verification: the
 * filters decide in fp32 on the GPU, so a decision may flip against an fp64
 * re-computation where the test's margin is within rounding of zero; with the
 * decisions recorded, a checker can replay exactly the skips the kernel took.
 * The same kernels, tile order and arithmetic as sparse_attn_fwd (filter =
 * SA_FILTER_LAMBDA) or sparse_attn_fwd_recall (SA_FILTER_RECALL); the only
 * extra work is one byte written per visited pair.
 *
 *   filter     SA_FILTER_LAMBDA or SA_FILTER_RECALL (else SA_ERR_INVALID_ARG)
 *   value      lambda or recall, checked as by the call it selects
 *   decisions  out, device uint8 [B,H,Nb,Nb], not NULL: for every query block i
 *              and kept, visible key block j the kernel visits, 1 if the pair's
 *              P.V was skipped, else 0. Entries of other pairs are not written
 *              (fill the buffer first if they are read).
 *
 * All other arguments, outputs and errors are those of sparse_attn_fwd. */
sa_status sparse_attn_fwd_decisions(const void* Q, const void* K, const void* V, sa_shape s,
                                    const uint8_t* mask, const int32_t* work, int32_t filter, float value,
                                    float scale, int32_t causal, void* O, int64_t* stats, uint8_t* decisions,
                                    void* stream);

/* End to end from host buffers: copy Q, K, V to the device, sparse_attn_plan +
 * the forward, copy O back, all on the caller's streams. The B*H heads are
 * independent, so the call pipelines them over `chunks` consecutive groups of
 * heads: group g's host-to-device copy runs on copy_in_stream, its plan and
 * forward on `stream`, and its device-to-host copy on copy_out_stream, so the
 * copies of one group overlap the work of the others in both directions of the
 * host link.
 *
 *   Qh, Kh, Vh  host bf16 [B,H,N,d]; pinned (page-locked) memory makes the copies
 *               asynchronous DMA, pageable memory works but serialises them
 *   tau         one recall threshold for every head, as sparse_attn_plan
 *   tau_heads   NULL, or a DEVICE array of B*H thresholds (4-byte aligned) that
 *               replaces tau, as sparse_attn_plan_heads (tau is then ignored)
 *   filter, value  the P.V filter, as sparse_attn_fwd_decisions (SA_FILTER_RECALL
 *               takes bf16 scores: it cannot be combined with either score flag)
 *   scale, causal  as sparse_attn_fwd
 *   flags       0, SA_HOST_FP8_SCORES: scores on FP8 codes of Q and K
 *               (sparse_attn_plan_q8 + sparse_attn_fwd_q8), or SA_HOST_INT8_SCORES:
 *               on INT8 codes (sparse_attn_plan_i8 + sparse_attn_fwd_i8); d must be
 *               128 for either, and the two flags cannot be combined
 *   Oh          out, host bf16 [B,H,N,d]; complete once `stream` is
 *   workspace   device memory of at least sparse_attn_host_workspace_size(s,
 *               chunks, flags) bytes, 256-byte aligned: the device copies of Q, K,
 *               V, O, the plan's outputs and scratch. The call waits (on the
 *               device) for earlier work on `stream` before overwriting it.
 *   chunks      number of head groups, >= 1 (values above B*H act as B*H)
 *   stream      the compute stream; when it completes, so has everything the call
 *               enqueued, the last copy back included
 *   copy_in_stream, copy_out_stream  streams for the two copy directions, or NULL
 *               to put that direction on `stream` (no overlap)
 *
 * The call enqueues and returns; synchronise `stream` before reading Oh, then
 * check sparse_attn_device_error if device-side failures matter (see
 * sparse_attn_fwd). Errors: those of sparse_attn_plan and sparse_attn_fwd, and
 * SA_ERR_WORKSPACE for a missing, misaligned or short workspace. */
#define SA_HOST_FP8_SCORES 1
#define SA_HOST_INT8_SCORES 2
size_t sparse_attn_host_workspace_size(sa_shape s, int32_t chunks, int32_t flags);
sa_status sparse_attn_host(const void* Qh, const void* Kh, const void* Vh, sa_shape s, float tau,
                           const float* tau_heads, int32_t filter, float value, float scale,
                           int32_t causal, int32_t flags,
                           void* Oh, void* workspace, size_t workspace_bytes, int32_t chunks,
                           void* stream, void* copy_in_stream, void* copy_out_stream);

/* Quantized scores (SpargeAttn: "sparse and quantized"; the quantization scheme
 * is this library's own, the pages give none). sparse_attn_plan that also writes
 * FP8 E4M3 copies of Q and K from the same pass over them:
 *
 *   Q8, K8          out, device uint8 [B,H,N,d] (16-byte aligned): E4M3 codes
 *   qscale, kscale  out, device float [B,H,Nb]: one scale per 64-token block
 *
 * For each (b, h, block) of Q and of K: amax = max |x| over the block, scale =
 * amax / 448 and code = x * (448 / amax) rounded to the nearest E4M3 value (ties
 * to even, saturating at 448), both in fp32; an all-zero block gets scale 1 and
 * codes 0. code * scale is the dequantized value. d must be 128, else
 * SA_ERR_UNSUPPORTED. Other arguments, outputs and errors: as sparse_attn_plan. */
sa_status sparse_attn_plan_q8(const void* Q, const void* K, sa_shape s, float tau, float scale,
                              int32_t causal, uint8_t* mask, int32_t* count, int32_t* idx,
                              int32_t* work, void* Q8, void* K8, float* qscale, float* kscale,
                              void* workspace, size_t workspace_bytes, void* stream);

/* sparse_attn_fwd with the scores taken on the FP8 codes of sparse_attn_plan_q8:
 * S = (Q8 K8^T) * qscale[query block] * kscale[key block] by tcgen05.mma
 * kind::f8f6f4 (fp32 accumulate); the softmax, the lambda filter, P.V (bf16 P, bf16
 * V) and O are those of sparse_attn_fwd. d must be 128. Other arguments and
 * errors: as sparse_attn_fwd. */
sa_status sparse_attn_fwd_q8(const void* Q8, const void* K8, const float* qscale, const float* kscale,
                             const void* V, sa_shape s, const uint8_t* mask, const int32_t* work,
                             float lambda, float scale, int32_t causal, void* O, int64_t* stats,
                             void* stream);

/* INT8 scores: the same two calls as sparse_attn_plan_q8 / sparse_attn_fwd_q8 with
 * signed INT8 codes instead of FP8 E4M3 (this library's second quantization
 * scheme; the pages give none). For each (b, h, 64-token block) of Q and of K:
 * amax = max |x| over the block, scale = amax / 127 and code = x * (127 / amax)
 * rounded to the nearest integer, ties to even (|code| <= 127, so -128 never
 * occurs), both in fp32; an all-zero block gets scale 1 and codes 0. The forward
 * takes S = (Q8 K8^T) * qscale[query block] * kscale[key block] by tcgen05.mma
 * kind::i8 (exact s32 accumulation). INT8 keeps 7 significant bits per operand
 * where E4M3 keeps 4, so the scores are about 16 times closer to the bf16 ones.
 * Q8, K8 hold int8_t values; other arguments, outputs and errors: as the q8 calls. */
sa_status sparse_attn_plan_i8(const void* Q, const void* K, sa_shape s, float tau, float scale,
                              int32_t causal, uint8_t* mask, int32_t* count, int32_t* idx,
                              int32_t* work, void* Q8, void* K8, float* qscale, float* kscale,
                              void* workspace, size_t workspace_bytes, void* stream);
sa_status sparse_attn_fwd_i8(const void* Q8, const void* K8, const float* qscale, const float* kscale,
                             const void* V, sa_shape s, const uint8_t* mask, const int32_t* work,
                             float lambda, float scale, int32_t causal, void* O, int64_t* stats,
                             void* stream);

/* Interaction clustering (iCATS abstract: query and key tokens clustered by
 * their dot-product interaction, the objective written as a quadratic form; the
 * formula is this library's reading of it). Replacing a token x of X by a
 * centroid c changes its score with every token y of Y by (x - c).y; the sum of
 * the squares is (x - c)^T G (x - c), G = sum_y y y^T. Per (b, h): k-means of
 * X's tokens under that distance, C = ceil(N/64) clusters initialised to the
 * 64-token block means, `iters` Lloyd iterations (assign each token to the
 * nearest centroid, fp32, ties to the lowest cluster index; move each centroid
 * to the mean of its tokens, an empty cluster keeping its centroid). Then the
 * tokens are ordered by cluster, in token order within a cluster, clusters
 * packed back to back (no padding: a cluster's tail shares a block with the
 * next one's head).
 *
 *   X, Y       device bf16 [B,H,N,d]: the side to cluster and the other side
 *              (queries are clustered with Y = K, keys with Y = Q)
 *   iters      0..64; 0 leaves every token in its block (perm = identity)
 *   assign     out, device int32 [B,H,N] or NULL: each token's cluster
 *   perm       out, device int32 [B,H,N]: perm[b,h,p] = the token at position p
 *   centroids  out, device fp32 [B,H,C,d] or NULL: the means of the final clusters
 *   workspace  device scratch of sparse_attn_cluster_workspace_size(s) bytes,
 *              256-byte aligned
 * Errors: as sparse_attn_plan (misaligned or NULL X, Y or perm, iters outside
 * 0..64: SA_ERR_INVALID_ARG; workspace: SA_ERR_WORKSPACE). A token whose every
 * distance is NaN goes to cluster 0 and sets bit 2 of the device error word. */
size_t sparse_attn_cluster_workspace_size(sa_shape s);
sa_status sparse_attn_cluster(const void* X, const void* Y, sa_shape s, int32_t iters, int32_t* assign,
                              int32_t* perm, float* centroids, void* workspace, size_t workspace_bytes,
                              void* stream);

/* Moves the rows of a bf16 [B,H,N,d] tensor by a per-head permutation (e.g.
 * sparse_attn_cluster's perm): inverse = 0 gathers dst[b,h,p] = src[b,h,perm[p]],
 * inverse != 0 scatters dst[b,h,perm[p]] = src[b,h,p]. src and dst must differ,
 * 16-byte aligned; perm 4-byte aligned and, per head, a permutation of 0..N-1
 * (an entry outside 0..N-1 moves nothing and sets bit 1 of the device error
 * word). */
sa_status sparse_attn_permute_rows(const void* src, const int32_t* perm, sa_shape s, int32_t inverse, void* dst,
                                   void* stream);

/* sparse_attn_plan without a workspace, for callers that cannot allocate device
 * memory (a runtime that reserves its whole memory budget up front, a plugin
 * whose host owns the allocator, a latency-critical path that must not call
 * cudaMalloc). The paper has no counterpart: this is a deployment variant.
 *
 * Same arguments, outputs and errors as sparse_attn_plan, minus the workspace,
 * and the same results. Its scratch goes to a fixed 32 MiB device array inside
 * the library, held by every GPU that loads the library until the process exits:
 * the regions sparse_attn_plan_workspace_size counts, with as many score strips as
 * the array leaves room for. The call fits when the other regions and one strip
 * fit in 32 MiB (e.g. H=24, d=128 up to N = 74,432) and returns SA_ERR_WORKSPACE
 * (nothing launched) otherwise. It calls no allocator. The first call on a device looks up the
 * array's device address and caches it; make that first call before any stream
 * capture on the device. All calls share the array (it keeps the last call's
 * contents, and nothing in it needs to start at zero), so calls that overlap on
 * the GPU race: keep them ordered on one stream. */
sa_status sparse_attn_plan_noalloc(const void* Q, const void* K, sa_shape s, float tau, float scale,
                                   int32_t causal, uint8_t* mask, int32_t* count, int32_t* idx,
                                   int32_t* work, void* stream);

/* Diagnostic of the device-side failure path (no counterpart in the paper; it
 * tests this library's own safeguards). Launches one warp on `stream` that
 * waits on a barrier nothing completes, through the bounded wait every pipeline
 * of this library uses, with a limit of limit_us microseconds instead of the
 * usual 4 s. The wait gives up, records bit 0 (a wait timed out) in the device
 * error word and the kernel returns normally, so the context stays usable; read
 * the word with sparse_attn_device_error. limit_us must be in [1, 4000000],
 * else SA_ERR_INVALID_ARG and nothing is launched. A failed launch returns
 * SA_ERR_CUDA. */
sa_status sparse_attn_selftest_wait_timeout(uint32_t limit_us, void* stream);

/* Human-readable name of a status code (static string). */
const char* sparse_attn_status_string(sa_status st);

/* Reads the device error word of the current GPU (after synchronising `stream`),
 * stores it in *code (0 = no device-side check fired; bit 0 = a pipeline wait
 * timed out, bit 1 = an index was out of range, bit 2 = a value read from
 * device memory was invalid, e.g. a per-head tau outside (0, 1]) and clears
 * it. Returns SA_OK, or SA_ERR_CUDA if the copy failed. */
sa_status sparse_attn_device_error(void* stream, int32_t* code);

#ifdef __cplusplus
}
#endif

#endif /* SPARSE_ATTN_H */
