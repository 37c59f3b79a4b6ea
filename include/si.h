/*
 * si.h -- C ABI of the streaming top-k indexer for NVIDIA B200 (sm_100a).
 *
 * The operation (StreamIndex: Memory-Bounded Compressed Sparse Attention via
 * Streaming Top-k, arXiv 2605.02568v1, Abstract): the lightning indexer of
 * Compressed Sparse Attention scores every compressed key for each query and
 * keeps the top-k keys per query, without materialising the [B,S,H_I,T] fp32
 * score tensor.  The Abstract gives no formula for the score (only that it is
 * learned and taken over the compressed keys); this library computes
 *
 *     score[b,t,s] = sum_h w[b,t,h] * max(0, sum_d q[b,t,h,d] * kc[b,s,d])
 *
 * over the keys visible to query t, key s being visible iff (s+1)*m <= t+1
 * and s < T, i.e. s < V_t = min(T, floor((t+1)/m)).  Each output row holds
 * min(k, V_t) keys ordered by score descending and, for equal scores, by key
 * index ascending, followed by padding (index -1, score -infinity).
 *
 * Conventions for every entry point:
 *  - All tensors are dense, contiguous and row-major, in device memory
 *    unless stated otherwise.  q: bf16 [B,S,H_I,d_I]; w: fp32 [B,S,H_I];
 *    kc: bf16 [B,T,d_I]; out_idx: int32 [B,S,k]; out_score: fp32 [B,S,k].
 *  - q, w and kc must be 16-byte aligned; out_idx and out_score 4-byte
 *    aligned.  The workspace must be 16-byte aligned.
 *  - Supported: H_I in {8,16,32,64}; d_I in {64,128}; 1 <= k <= 2048;
 *    m >= 1; B, S >= 1; T >= 0; S*H_I < 2^31; T < 2^31; B < 2^31.
 *  - The caller owns every buffer; the library never allocates or frees
 *    device memory.  Work is enqueued on `stream` (NULL = legacy default
 *    stream) without any host synchronisation; results are ready when the
 *    stream reaches that point.  Calls are reentrant; concurrent calls need
 *    separate workspaces and outputs.  Results are deterministic.
 *  - Argument errors are reported before anything is enqueued.  Errors of
 *    the device (a bounded wait that expired) are recorded in the workspace
 *    and read with si_check_device_status().
 */
#ifndef STREAMING_TOP_INDEXER_SI_H_
#define STREAMING_TOP_INDEXER_SI_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SI_API __attribute__((visibility("default")))
#else
#define SI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so callers need no CUDA header. */
typedef struct CUstream_st* si_stream_t;

typedef enum {
    SI_OK = 0,
    SI_ERR_INVALID_ARG = 1,        /* null pointer or out-of-range size */
    SI_ERR_UNSUPPORTED = 2,        /* H_I, d_I or k outside the supported set */
    SI_ERR_MISALIGNED = 3,         /* a pointer breaks the alignment rules */
    SI_ERR_WORKSPACE_TOO_SMALL = 4,
    SI_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
    SI_ERR_TIMEOUT = 6             /* a device-side wait expired (kernel aborted) */
} si_status;

/* Bytes of workspace si_indexer_topk needs for these sizes (host arithmetic
 * only, no CUDA call).  At least 256.  It is O(number of SMs x top-k pool),
 * independent of S and T, never O(S*T).  Returns 0 for unsupported sizes. */
SI_API size_t si_workspace_bytes(int64_t B, int64_t S, int64_t T, int H_I, int d_I, int m, int k);

/* The indexer step: top-k keys and scores of every query row.
 * Enqueues: a 256-byte reset of the workspace header, then the fused scoring,
 * selection and row-sort kernel.  The separate per-row sort is added only
 * where si_select_sorts_rows() is 0.  Writes every element of out_idx and
 * out_score, padding included. */
SI_API si_status si_indexer_topk(const void* q, const float* w, const void* kc,
                          int64_t B, int64_t S, int64_t T, int H_I, int d_I, int m, int k,
                          int32_t* out_idx, float* out_score,
                          void* workspace, size_t workspace_bytes, si_stream_t stream);

/* si_indexer_topk for the query rows [t_begin, t_end) of every batch only.
 * The method selects each query row's keys on its own (StreamIndex:
 * Memory-Bounded Compressed Sparse Attention via Streaming Top-k, Abstract),
 * so rows can be computed in windows.  This lets a caller overlap the
 * host-to-device copy of later rows, and the copy back of earlier results,
 * with the computation of a window.
 *   q, w, out_idx, out_score: the WHOLE [B,S,...] tensors (same layout and
 *     alignment rules as si_indexer_topk); only the window's rows of q and w
 *     are read and only the window's rows of the outputs are written.
 *   kc: the whole [B,T,d_I] tensor (keys are visible by the absolute row t).
 *   t_begin: a multiple of 256; t_end: a multiple of 256, or S;
 *     0 <= t_begin <= t_end <= S (else SI_ERR_INVALID_ARG, nothing enqueued).
 *   workspace: as si_indexer_topk.  Its header (device error word) is NOT
 *     reset: reset it once with si_reset_device_status before a sequence of
 *     windows, and si_check_device_status afterwards reports a failure of
 *     any of them.  Windows enqueued on different streams with one
 *     workspace race.
 * Result rows are identical to those of si_indexer_topk. */
SI_API si_status si_indexer_topk_rows(const void* q, const float* w, const void* kc,
                               int64_t B, int64_t S, int64_t T, int H_I, int d_I, int m, int k,
                               int64_t t_begin, int64_t t_end,
                               int32_t* out_idx, float* out_score,
                               void* workspace, size_t workspace_bytes, si_stream_t stream);

/* si_indexer_topk on HOST inputs and outputs, copies included (the call a
 * user with host data makes).  Rows are computed in windows with
 * si_indexer_topk_rows (rows select their keys independently: StreamIndex:
 * Memory-Bounded Compressed Sparse Attention via Streaming Top-k, Abstract),
 * last rows first.  While one window is computed on `stream`, the q and w rows
 * of the next are copied in and the results of the previous one copied out,
 * on two copy streams the library keeps per device.
 *   q_h, w_h, kc_h: host q bf16 [B,S,H_I,d_I], w fp32 [B,S,H_I], kc bf16
 *     [B,T,d_I]; idx_h, score_h: host outputs [B,S,k].  Page-locked host
 *     memory lets the copies overlap the computation; pageable memory gives
 *     the same results with serialised copies.
 *   q_d, w_d, kc_d, idx_d, score_d: caller-owned device buffers of the same
 *     shapes (the rules of si_indexer_topk apply to them); workspace as for
 *     si_indexer_topk (its header is reset by this call).
 *   chunks: number of row windows, 0 for the default min(32, max(1, S/2048));
 *     windows hold a multiple of 256 rows (see si_host_window_rows).
 *   The current device must be the one that owns `stream` and the buffers.
 * Arguments are checked before anything is enqueued (the codes of
 * si_indexer_topk, SI_ERR_INVALID_ARG for a null host pointer or chunks < 0).
 * Everything is asynchronous: the host outputs are complete once `stream` is
 * synchronised.  A later call, or other work on `stream`, may reuse the
 * buffers: the copies in wait for the work queued on `stream` before. */
SI_API si_status si_indexer_topk_host(const void* q_h, const float* w_h, const void* kc_h,
                               int64_t B, int64_t S, int64_t T, int H_I, int d_I, int m, int k,
                               int32_t* idx_h, float* score_h,
                               void* q_d, float* w_d, void* kc_d, int32_t* idx_d, float* score_d,
                               void* workspace, size_t workspace_bytes, int chunks, si_stream_t stream);

/* Rows per window of si_indexer_topk_host for `chunks` windows: ceil(S /
 * chunks) rounded down to a multiple of 256, at least 256 (0 for S <= 0);
 * the last window ends at S. */
SI_API int64_t si_host_window_rows(int64_t S, int chunks);

/* First stage of si_indexer_topk alone: the fused scoring + selection kernel.
 * Does not reset the workspace header.  Where si_select_sorts_rows() is 1
 * for these sizes, the kernel also sorts each row at the end of its work
 * unit, and the rows are final.  Otherwise each row's top-k set is left
 * unordered (padding at the tail) for si_sort_topk.  Exposed so that the
 * stages can be timed separately: si_indexer_topk is the header reset, then
 * this, then si_sort_topk only where the kernel leaves rows unordered. */
SI_API si_status si_select_topk(const void* q, const float* w, const void* kc,
                         int64_t B, int64_t S, int64_t T, int H_I, int d_I, int m, int k,
                         int32_t* out_idx, float* out_score,
                         void* workspace, size_t workspace_bytes, si_stream_t stream);

/* Second stage: orders each of the `rows` rows of k (index, score) pairs by
 * score descending, then index ascending, padding last (in place).  Also a
 * general utility for rows in any order. */
SI_API si_status si_sort_topk(int32_t* out_idx, float* out_score, int64_t rows, int k,
                       si_stream_t stream);

/* The materialise path, for small problems: writes score[b,t,s] for every
 * visible key into out_scores, fp32 [B,S,T] (entries of invisible keys are
 * left untouched), through the same TMA + tcgen05 pipeline as the streaming
 * path.  Same argument rules as si_indexer_topk; needs a workspace of at
 * least 256 bytes. */
SI_API si_status si_indexer_scores(const void* q, const float* w, const void* kc,
                            int64_t B, int64_t S, int64_t T, int H_I, int d_I, int m,
                            float* out_scores, void* workspace, size_t workspace_bytes,
                            si_stream_t stream);

/* Clears the device error word in the workspace header (a 256-byte
 * asynchronous memset on `stream`), as si_indexer_topk does at its start.
 * SI_ERR_INVALID_ARG for a null workspace, SI_ERR_MISALIGNED unless it is
 * 16-byte aligned, SI_ERR_CUDA if the memset cannot be enqueued.  The paper
 * has no counterpart; it serves sequences of si_indexer_topk_rows calls. */
SI_API si_status si_reset_device_status(void* workspace, si_stream_t stream);

/* Synchronises `stream`, then returns SI_OK or the device error recorded in
 * the workspace header by the last call that used it (SI_ERR_TIMEOUT), or
 * SI_ERR_CUDA if reading it failed. */
SI_API si_status si_check_device_status(const void* workspace, si_stream_t stream);

/* Self-test of the device-side bounded wait: launches a one-block kernel that
 * waits on a barrier nobody arrives at, with a limit of limit_ns; the wait
 * gives up and records SI_ERR_TIMEOUT in the workspace header, which
 * si_check_device_status() then returns.  No fault, trap or hang. */
SI_API si_status si_selftest_timeout(void* workspace, size_t workspace_bytes, uint64_t limit_ns,
                              si_stream_t stream);

/* si_indexer_topk without a caller-supplied workspace, for callers that
 * cannot allocate device memory themselves (for instance a plugin inside a
 * host application that owns all device memory, or a serving loop whose
 * memory plan is fixed after start-up).  The paper has no counterpart; this
 * is a packaging variant of the same computation and results.
 *
 * Scratch: a fixed 1 MiB array in device memory, one per device, that every
 * device which loads this library keeps until the process exits.  The call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 * The first call on a device looks up that array's device address (with the
 * device current) and remembers it; that first call on a device should come
 * before any stream capture.  All calls on a device share the
 * array, which keeps the last call's contents; the call clears what must
 * start at zero.  Calls whose work overlaps on the GPU (different streams,
 * no ordering between them) race on the shared array: order them.
 *
 * Limit: configurations whose si_workspace_bytes() exceeds 1 MiB return
 * SI_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.  Those are exactly
 * the ones whose candidate pools do not fit in shared memory.  The first
 * refused k for each (H_I, d_I) is:
 *     H_I=64: d_I=128 k >= 1089; d_I=64 none (every k up to 2048 runs)
 *     H_I=32: d_I=128 k >= 465;  d_I=64 k >= 1185
 *     H_I=16: d_I=128 k >= 161;  d_I=64 k >= 481
 *     H_I=8:  d_I=128 every k;   d_I=64 k >= 193
 * So the array only ever holds the device error word.  Everything else is
 * as si_indexer_topk.  out_status, if not NULL,
 * is a device word that receives the device status of the call (0, or
 * SI_ERR_TIMEOUT) once the stream reaches the end of the call. */
SI_API si_status si_indexer_topk_noalloc(const void* q, const float* w, const void* kc,
                                         int64_t B, int64_t S, int64_t T, int H_I, int d_I, int m, int k,
                                         int32_t* out_idx, float* out_score, uint32_t* out_status,
                                         si_stream_t stream);

/* 1 if the select kernel writes rows already sorted for these sizes: every
 * k <= 1024.  The kernel's unit-end sort covers 128*E keys, with E the
 * smallest power of two such that 128*E >= k.  For larger k the separate
 * row sort is faster.  Otherwise 0, and si_indexer_topk adds the si_sort_topk
 * pass.
 * Host arithmetic only.  Returns 0 for unsupported sizes. */
SI_API int si_select_sorts_rows(int H_I, int d_I, int k);

/* Process-wide switch for later calls.  Nonzero (the default): the select
 * kernel sorts rows where it can.  Zero: it always leaves rows unordered,
 * and si_indexer_topk sorts them with the separate row-sort kernel.  Both give
 * identical results; the switch exists to time the two designs. */
SI_API void si_set_sort_in_select(int enable);

/* The sparse attention stage of CSA, over the keys the indexer selected
 * (StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
 * Top-k, Abstract: the attention reads only the selected compressed keys; the
 * Abstract gives no formula, and this is the plainest reading):
 *
 *     out[b,t,h,:] = sum_j softmax_j(scale * q[b,t,h,:] . K[b,j,:]) V[b,j,:]
 *     lse[b,t,h]   = log sum_j exp(scale * q[b,t,h,:] . K[b,j,:])
 *
 * with j over the entries idx[b,t,0..k) in [0, T); other entries (the
 * indexer's -1 padding) are skipped.  A row with no such entry gives
 * out = 0 and lse = -infinity.  K and V are shared by all heads.
 *   q:      bf16 [B,S,H_a,d]   (H_a = 128: one head per MMA row)
 *   kcache: bf16 [B,T,d]       compressed keys;  vcache: bf16 [B,T,d_v]
 *   idx:    int32 [B,S,k]      e.g. si_indexer_topk's out_idx
 *   out:    bf16 [B,S,H_a,d_v];  lse: fp32 [B,S,H_a]
 *   status: a device word, set to 0 by the call and to SI_ERR_TIMEOUT if a
 *           bounded device wait expired (read it after the stream reaches
 *           the end of the call).
 * Supported: H_a = 128; d, d_v in {64, 128}; 1 <= k <= 2048;
 * B*S*128 < 2^31; B*T < 2^31.  q, kcache, vcache and out 16-byte aligned;
 * idx, lse and status 4-byte aligned.  Allocates nothing; asynchronous on
 * `stream`.  Arithmetic: bf16 products, fp32 accumulation, softmax weights
 * rounded to bf16 for the P.V product (sums in fp32), bf16 output. */
SI_API si_status si_sparse_attention(const void* q, const void* kcache, const void* vcache, const int32_t* idx,
                                     int64_t B, int64_t S, int64_t T, int H_a, int d, int d_v, int k,
                                     float scale, void* out, float* lse, uint32_t* status, si_stream_t stream);

/* Design parameters of the select kernel, process-wide, for later calls and
 * si_workspace_bytes (0 keeps a default).  They are the counterparts of the
 * driver parameters the pages sweep (StreamIndex: Memory-Bounded Compressed
 * Sparse Attention via Streaming Top-k, Abstract: chunk size, key-tile size):
 *   pool_entries  candidates a query's pool holds between partition-merges
 *                 (default: as many as shared memory allows, at least
 *                 max(k+288, min(2k, k+768)); else 4k in the workspace).  It
 *                 is raised to k + 4*(32*check_tiles+1) + 28 if smaller.  It
 *                 stays in shared memory when it fits, else goes to the workspace;
 *   cut_slack     entries above k an intermediate merge may keep (default 256);
 *   check_tiles   128-key tiles streamed between two checks of the pools'
 *                 fill (default 2).
 * Results do not depend on them: every setting returns the exact top-k.
 * Returns SI_ERR_INVALID_ARG (and changes nothing) for pool_entries outside
 * [0, 65504], cut_slack outside [0, 4096] or check_tiles outside [0, 16].
 * The workspace size depends on pool_entries: size it after the call. */
SI_API si_status si_set_tuning(int pool_entries, int cut_slack, int check_tiles);

/* The indexer's inputs from hidden states, with given weights (the paper has
 * the indexer score queries against keys compressed at ratio m with a
 * learned projection, StreamIndex: Memory-Bounded Compressed Sparse
 * Attention via Streaming Top-k, Abstract, and gives neither the
 * projections nor the compressor; this is the plainest reading):
 *     q[b,t,h,:] = x[b,t,:] . W_q[h*d_I + (0..d_I), :]^T   bf16 [B,S,H_I,d_I]
 *     w[b,t,h]   = x[b,t,:] . W_w[h, :]^T                   fp32 [B,S,H_I]
 *     kc[b,s,:]  = (1/m) sum_{j<m} x[b,s*m+j,:] . W_k^T    bf16 [B,T,d_I], T = floor(S/m)
 *   x:   bf16 [B,S,d_model];  W_q: bf16 [H_I*d_I, d_model];  W_w: bf16
 *   [H_I, d_model];  W_k: bf16 [d_I, d_model] (the [out, in] layout).
 *   Each output is one tcgen05 GEMM with fp32 accumulation; the key
 *   compressor reads a group of m tokens as one row (the mean pooling is
 *   part of the contraction).
 *   status: a device word, set to 0 by the call and to SI_ERR_TIMEOUT if a
 *   bounded device wait expired.
 * Supported: d_model a multiple of 64; H_I a multiple of 4; d_I and H_I*d_I
 * multiples of 8; B*S < 2^31.  All pointers 16-byte aligned (status 4).
 * Allocates nothing; asynchronous on `stream`. */
SI_API si_status si_indexer_inputs(const void* x, const void* w_q, const void* w_w, const void* w_k,
                                   int64_t B, int64_t S, int d_model, int H_I, int d_I, int m,
                                   void* q, float* w, void* kc, uint32_t* status, si_stream_t stream);

/* Device-side wait limit, in nanoseconds, used by later calls (default 2 s). */
SI_API void si_set_timeout_ns(uint64_t ns);

/* Human-readable name of a status code. */
SI_API const char* si_status_string(si_status s);

/* Library version string. */
SI_API const char* si_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STREAMING_TOP_INDEXER_SI_H_ */
