/*
 * mcs.h - C ABI of the MC-Sparse token-sparse attention library for NVIDIA B200 (sm_100a).
 *
 * The method is MC-Sparse (meta-cached sparse attention for diffusion transformers), as
 * described on the pages "MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다" (cited below
 * as P4) and "MC-Sparse: 解构并弥合 Diffusion Transformers 中的稠密-稀疏注意力差距" (P1):
 *
 *   anchor step  (P4, section 무엇과 다른가): run dense attention, build the query groups G,
 *                select the KV tokens S by exact probabilities, record R = O_full - O_sparse;
 *   reuse step   (same section):  O_hat_t = SparseAttn(Q_t, K_t, V_t; G, S) + R.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Tensors are DEVICE pointers to contiguous row-major arrays, each 16-byte aligned:
 *      Q, K, V, O, O_full, R, out : bf16 [B, H, N, d]
 *      perm                       : int32 [B, H, N]  (group g of head (b,h) is
 *                                   perm[b,h, g*C : (g+1)*C], ascending query ids)
 *      idx                        : int32 [B, H, N/C, k] (ascending key ids per group)
 *      lse                        : fp32 [B, H, N] (natural-log log-sum-exp of scale*q.k)
 *  - d is 64 or 128; C (the query tile / group size) is 64 or 128 and must divide N;
 *    1 <= k <= N.  shape.scale <= 0 selects 1/sqrt(d).
 *  - The caller owns every buffer.  The library never allocates device memory; calls that
 *    need scratch take a caller-provided workspace (`ws`, `ws_bytes`, 256-byte aligned) whose
 *    size mcs_workspace_size() reports.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only enqueues
 *    work and returns; results are ready when the stream reaches them.
 *  - Argument errors are reported before anything is enqueued.  Errors found by kernels
 *    (an index outside [0, N), a bounded wait that gave up) set a device status word that
 *    mcs_sync_status() reads and clears.  No kernel traps.
 *  - Outputs are deterministic: the same inputs give bit-identical results.
 */
#ifndef MCS_H_
#define MCS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MCS_OK = 0,
  MCS_ERR_INVALID_ARG = 1,        /* null pointer, B/H/N < 1, C or k out of range        */
  MCS_ERR_SHAPE = 2,              /* d not in {64,128}, C not in {64,128}, N % C != 0,    */
                                  /* B*H > 65535, N > 2^24 or B*H*N > 2^32 - 1           */
  MCS_ERR_DTYPE_ALIGN = 3,        /* a tensor or the workspace is misaligned             */
  MCS_ERR_UNSUPPORTED_ARCH = 4,   /* current device is not compute capability 10.0        */
  MCS_ERR_CUDA = 5,               /* a CUDA runtime call or kernel launch failed          */
  MCS_ERR_BAD_INDEX = 6,          /* a kernel met perm/idx entries outside [0, N)         */
  MCS_ERR_TIMEOUT = 7,            /* a kernel's bounded wait expired                      */
  MCS_ERR_WORKSPACE = 8           /* ws is NULL or ws_bytes < mcs_workspace_size()        */
} mcs_status;

typedef struct {
  int B, H, N, d;
  float scale; /* softmax scale; <= 0 means 1/sqrt(d) */
} mcs_shape;

/* Library ABI version (this header: 1). */
int mcs_abi_version(void);

/* Human-readable name of a status code (static string). */
const char* mcs_status_string(mcs_status s);

/* Bytes of workspace that mcs_group, mcs_select and mcs_anchor need for this shape, group
 * size C and selection size k (the maximum over the three).  Returns 0 for invalid shapes. */
size_t mcs_workspace_size(mcs_shape s, int C, int k);

/* Dense attention (P4, section 무엇과 다른가: the anchor step runs dense attention; P4,
 * section 전제와 한계: dense attention is the speed baseline).
 *   O[b,h,i,:] = sum_j softmax_j(scale * q_i . k_j) v_j
 *   lse[b,h,i] = log sum_j exp(scale * q_i . k_j)   (pass 1 of the exact selection)
 * O may be NULL (LSE only); lse may be NULL.  Any N >= 1 (no C constraint). */
mcs_status mcs_dense_attn(mcs_shape s, const void* Q, const void* K, const void* V, void* O, float* lse,
                          void* stream);

/* Tile-aligned query grouping by median-split PDDP (P4, section 어떻게 쓰나): writes perm,
 * a partition of each head's N queries into N/C groups of exactly C, by recursive
 * principal-direction splits at the median, all nodes of one depth (all heads) batched
 * ("Fast PDDP").  Readings fixed where the page is silent: centered data, 20 power-
 * iteration steps from 1/sqrt(d), sign making the largest-magnitude component positive,
 * left child = floor(m/2)*C smallest projections (ties to the lower query id). */
mcs_status mcs_group(mcs_shape s, const void* Q, int C, int32_t* perm, void* ws, size_t ws_bytes,
                     void* stream);

/* Exact two-pass KV selection (P4, sections 어떻게 쓰나 and 어떻게 동작하나; P1, section
 * 集成接口): for each group g, score_g[j] = sum_{i in g} exp(scale*q_i.k_j - lse_i) (exact
 * softmax probabilities summed over the group), idx[g,:] = the k keys of largest score, ties
 * to the lower key id, stored ascending.  lse = NULL runs pass 1 (mcs_dense_attn without O)
 * into the workspace first. */
mcs_status mcs_select(mcs_shape s, const void* Q, const void* K, const int32_t* perm, int C, int k,
                      const float* lse, int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/* Reuse step (P4, section 무엇과 다른가; token-level gather: section 어떻게 쓰나):
 *   out[q] = sum_{j in idx[g]} softmax_j(scale * q . k_j) v_j + R[q]   for q in group g,
 * with the softmax renormalised over the k selected keys.  R may be NULL (no residual).
 * out must not alias Q, K, V or R. */
mcs_status mcs_sparse_attn(mcs_shape s, const void* Q, const void* K, const void* V, const int32_t* perm,
                           int C, const int32_t* idx, int k, const void* R, void* out, void* stream);

/* Device staging bytes that mcs_sparse_attn_host needs: two slots of Q, K, V and out for
 * min(heads_per_chunk, B*H) heads each, 2 * 4 * that * N * d * 2 bytes.  0 for an invalid shape
 * or heads_per_chunk < 1. */
size_t mcs_host_staging_size(mcs_shape s, int heads_per_chunk);

/* The reuse step of mcs_sparse_attn with Q, K, V and out in HOST memory (an addition of this
 * library; the pages only say the cached metadata may be offloaded to CPU memory, section
 * 어떻게 쓰나): hQ, hK, hV, hOut are [B,H,N,d] bf16 host buffers (page-locked for the copies to
 * overlap; pageable memory works but serialises them), perm, idx and R (nullable) are the
 * device-resident cached metadata as for mcs_sparse_attn.  The B*H heads go through in chunks
 * of heads_per_chunk: the host-to-device copies of chunk c+1 and the device-to-host copy of
 * chunk c-1 run on two side streams while chunk c's kernel runs on `stream`, through two slots
 * of `staging` (device, 256-byte aligned, at least mcs_host_staging_size bytes).  Results are
 * bit-identical to mcs_sparse_attn.  Asynchronous like every call here: the caller keeps the
 * host buffers alive and reads hOut only after synchronising `stream`, on which all later work
 * is ordered after the last output copy.  The two side streams and their events are created
 * on the first call on a device and kept until the process exits; calls from several threads
 * take turns while enqueuing.  Errors as mcs_sparse_attn; heads_per_chunk < 1 is
 * MCS_ERR_INVALID_ARG; a missing or small staging buffer MCS_ERR_WORKSPACE. */
mcs_status mcs_sparse_attn_host(mcs_shape s, const void* hQ, const void* hK, const void* hV, const int32_t* perm,
                                int C, const int32_t* idx, int k, const void* R, void* hOut, int heads_per_chunk,
                                void* staging, size_t staging_bytes, void* stream);

/* Residual record of the anchor step (P4, section 무엇과 다른가: R = O_full - O_sparse):
 * R[q] = O_full[q] - SparseAttn(Q, K, V; perm, idx)[q].  R must not alias the inputs. */
mcs_status mcs_residual(mcs_shape s, const void* Q, const void* K, const void* V, const int32_t* perm,
                        int C, const int32_t* idx, int k, const void* O_full, void* R, void* stream);

/* Whole anchor step: O_full and lse (dense), perm (mcs_group), idx (mcs_select with that
 * lse) and R (mcs_residual), enqueued in that order on `stream`. */
mcs_status mcs_anchor(mcs_shape s, const void* Q, const void* K, const void* V, int C, int k, void* O_full,
                      int32_t* perm, int32_t* idx, void* R, void* ws, size_t ws_bytes, void* stream);

/* Same selection as mcs_select, for callers that cannot allocate device memory at all, so
 * cannot provide a workspace: for example code running inside an engine or framework that
 * owns every byte of device memory through its own pool, or a latency-critical loop whose
 * policy forbids any allocation (and the implicit synchronisation cudaMalloc/cudaFree bring).
 * The pages describe no such entry point; it is an addition of this library.
 *   - The per-block score scratch is a fixed 16 MiB array compiled into the library (every
 *     GPU that loads the library keeps it until the process exits).  Problems with
 *     round_up(N, 64) > 2,097,152 are rejected with MCS_ERR_WORKSPACE.
 *   - lse must be given (pass 1, e.g. from mcs_dense_attn); NULL is MCS_ERR_INVALID_ARG.
 *   - The first call on a device looks up the array's device address (once per device, with
 *     that device current); make that first call before any stream capture.
 *   - All calls share the one array: calls whose executions overlap on the GPU (other
 *     streams, other threads) race and give wrong results.  Each call writes every score it
 *     reads, so nothing carried over from an earlier call affects the result.
 *   - Nothing is allocated or freed: no cudaMalloc/cudaFree, no allocating library call. */
mcs_status mcs_select_noalloc(mcs_shape s, const void* Q, const void* K, const int32_t* perm, int C, int k,
                              const float* lse, int32_t* idx, void* stream);

/* ---- Selection variants of the controlled oracle comparison (P4, section 어떻게 동작하나:
 * block oracle, token oracle, per-query oracle, all by exact dense attention probabilities,
 * against vanilla block-sparse attention, which scores blocks from mean-pooled queries and
 * keys; P4, section 무엇인가).  They serve the error-decomposition study at equal density; the
 * token oracle is mcs_select with contiguous query blocks (perm = the identity). */

/* KV-block selection per query group, emitted as token indices so that mcs_sparse_attn runs it
 * unchanged: idx[b,h,g, i*BK + r] = blk_i*BK + r for the kb chosen blocks blk_0 < blk_1 < ...
 * (k = kb*BK ascending key ids per group).  Block j covers keys [j*BK, (j+1)*BK).
 *   method 0 (block oracle): block score = sum over the block's keys of score_g[j], the exact
 *            group score of mcs_select; lse = NULL runs pass 1 into the workspace first.
 *   method 1 (vanilla BSA): block score = qbar_g . kbar_j, the mean of the group's queries
 *            against the mean of the block's keys (fp32; lse is ignored).
 * kb largest scores, ties to the lower block.  Requires BK a multiple of 16 with 64 <= BK,
 * N % BK == 0, N/BK <= 4096 and 1 <= kb <= N/BK; the workspace of mcs_workspace_size(s, C,
 * kb*BK).  Errors as mcs_select. */
mcs_status mcs_select_blocks(mcs_shape s, const void* Q, const void* K, const int32_t* perm, int C, int BK,
                             int kb, int method, const float* lse, int32_t* idx, void* ws, size_t ws_bytes,
                             void* stream);

/* Workspace bytes of mcs_perquery_attn (the logits of the queries in flight, N floats each);
 * 0 for an invalid shape. */
size_t mcs_perquery_workspace_size(mcs_shape s);

/* Per-query oracle: every query attends to its own k keys of largest logit (equivalently of
 * largest exact probability), ties to the lower key id, softmax renormalised over that set:
 *   out[b,h,i,:] = sum_{j in S_i} exp(l_ij - m_i) v_j / sum_{j in S_i} exp(l_ij - m_i),
 *   l_ij = scale * q_i . k_j,  S_i = top-k of l_i.,  m_i = max_j l_ij.
 * An analysis variant on CUDA cores (O(N^2 d) per head).  Requires N % 16 == 0 and
 * 1 <= k <= N; ws of mcs_perquery_workspace_size(s) bytes. */
mcs_status mcs_perquery_attn(mcs_shape s, const void* Q, const void* K, const void* V, int k, void* out, void* ws,
                             size_t ws_bytes, void* stream);

/* Failure-path hook of the attention kernels (those of mcs_dense_attn, mcs_sparse_attn,
 * mcs_residual, mcs_sparse_attn_host and the dense and residual launches of mcs_anchor), for
 * tests and diagnosis; the pages have no counterpart.  For every such kernel enqueued after
 * this call, process-wide:
 *   - ns bounds any single wait inside the kernel, in nanoseconds (0 restores the default of
 *     2 s, far above any legitimate wait);
 *   - hold, if not NULL, is a device pointer to a uint32 flag that the kernel waits for (until
 *     it is nonzero, within that bound) before issuing any tensor-core work.
 * A kernel whose wait runs out abandons the rest of its work (its outputs are then undefined),
 * lets the copies and tensor-core operations it already issued finish, releases its tensor
 * memory and returns; mcs_sync_status() then reports MCS_ERR_TIMEOUT, and calls made after
 * the hook is reset (ns = 0, hold = NULL) run normally.  A flag that nothing sets makes every
 * launch take that path.  The selection and grouping kernels keep the fixed 2 s bound and
 * ignore the flag (their top-k step needs every thread of a CTA to reach the same decision).
 * Returns the previous bound. */
uint64_t mcs_set_attn_wait_limit(uint64_t ns, const uint32_t* hold);

/* ---- Grouping-cost baseline (P4, section 전제와 한계 sets Fast PDDP's grouping cost against a
 * k-means clustering; the pages give no algorithm for an equal-size k-means, so this one is a
 * reading).  Not part of the hot path: it exists to time Fast PDDP against.
 * Equal-size groups of exactly C queries per head: G = N/C centroids start as the means of the
 * contiguous query blocks [g*C, (g+1)*C); `iters` Lloyd steps send every query to its nearest
 * centroid (squared Euclidean distance, ties to the lower centroid) and move every centroid to
 * the mean of its queries (an empty cluster keeps its centroid); then clusters 0, 1, ..., G-1 in
 * turn take the C not yet taken queries nearest to their centroid (ties to the lower query id).
 * perm as for mcs_group (group g is cluster g's queries, ascending).  All in fp64, no fused
 * multiply-adds.  ws of mcs_kmeans_workspace_size bytes (256-byte aligned; it holds the G x N
 * distance matrix of every head); 0 <= iters <= 1000. */
size_t mcs_kmeans_workspace_size(mcs_shape s, int C);
mcs_status mcs_group_kmeans(mcs_shape s, const void* Q, int C, int iters, int32_t* perm, void* ws, size_t ws_bytes,
                            void* stream);

/* Synchronise `stream`, then read and clear the device status word of the current device:
 * MCS_OK, MCS_ERR_BAD_INDEX, MCS_ERR_TIMEOUT, or MCS_ERR_CUDA if the stream reports an error.
 * There is one word per device, shared by the library's kernels on every stream: with calls
 * in flight on several streams, a status may come from any of them (and reading clears it for
 * all), so synchronise the streams that matter before attributing it. */
mcs_status mcs_sync_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MCS_H_ */
