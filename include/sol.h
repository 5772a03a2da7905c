/*
 * sol.h -- C ABI of libsol.so: Sol block-sparse attention forward on B200 (sm_100a).
 *
 * The forward pass has three stages, each one entry point, enqueued in order
 * on one CUDA stream (or ordered by the caller):
 *
 *   sol_pool      block centroids of Q, K, V (+ optional log-mass bias)
 *   sol_route     block scores, per-row mean + tau*std threshold, CSR lists
 *                 of exact key blocks
 *   sol_attn_fwd  exact attention over the listed key blocks, one centroid
 *                 term per unlisted block, merged in one fp32 online softmax
 *
 * Method sources (web pages; no code or equations are published):
 *   - Star7 README "MiniMax H3 Activation Chunk & Attention Acceleration",
 *     section 工作原理 > Sol: Q64/K64 blocks, tau = 1.0 threshold routing;
 *     selected K/V blocks exact, unselected blocks contribute through their
 *     K/V centroids, both merged in the same FP32 online softmax; the
 *     audio-range KV sink is kept and prefix query rows attend densely.
 *   - thakicloud "MiniMax-H3 ComfyUI accel stack", section 이 기술은 무엇인가:
 *     tau counts standard deviations above the mean block score; strided
 *     views of the fused QKV projection are passed without copies.
 *   - Spark-H3 news page (comfyui-wiki), section "Spark-Attn이 바꾸는 것",
 *     Spark-Reweight bullet and compressed-branch figure caption: the
 *     log-mass bias restoring E[exp(x)] over exp(E[x]), scored against one
 *     anchor per head, the mean video query.
 *   - Star7 README, section 环境与分发: a native library that takes only
 *     tensor addresses, shapes and the current CUDA stream, and refuses a
 *     mismatched architecture naming required and detected capability.
 *
 * Conventions (all entry points):
 *   - Every buffer is owned by the caller.  The library never allocates
 *     device memory and never synchronises, except sol_last_device_status.
 *   - Argument errors are reported synchronously, before anything is
 *     enqueued.  Launch failures map to SOL_ERR_CUDA.  The first call on a
 *     device checks that it is compute capability 10.0 (B200, sm_100a) and
 *     returns SOL_ERR_UNSUPPORTED otherwise; sol_last_error_text() then
 *     names the detected capability.
 *   - Tensors are bf16 with the head dimension contiguous.  Q, K, V share
 *     one set of element strides (in_stride_*), so strided views into a
 *     fused QKV buffer are accepted; O has its own (out_stride_*).  Base
 *     addresses must be 16-byte aligned and every stride a multiple of 8
 *     elements.
 *   - B == 0 or N == 0 is a valid empty problem: nothing is enqueued.
 *   - Heads are independent in every stage, so a call may cover any run of
 *     heads [h0, h0 + Hg) of a larger tensor: set H = Hg, keep the strides,
 *     and offset each base pointer by h0 * in_stride_h (O by h0 *
 *     out_stride_h) elements.  Workspace, CSR and LSE then hold those Hg
 *     heads only (CSR rows in (b, h - h0, i) order), and every output equals
 *     that head's slice of the whole call bit for bit.  This is how one call
 *     is split over GPUs (each takes H / G heads, no collective).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).
 */
#ifndef SOL_H_
#define SOL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SOL_OK = 0,
  SOL_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, stride, alignment or tau */
  SOL_ERR_UNSUPPORTED = 2,   /* wrong GPU architecture, head dim or block size */
  SOL_ERR_WORKSPACE = 3,     /* workspace smaller than sol_workspace_bytes() */
  SOL_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  SOL_ERR_TIMEOUT = 5        /* a kernel's bounded wait expired (device status) */
} sol_status;

typedef struct {
  int32_t B, N, H, D;        /* batch, rows of the packed sequence, heads, head dim (64 or 128) */
  int32_t q_block, k_block;  /* rows per query / key block; the GPU path takes 64 and 64 */
  float tau;                 /* threshold in std units above the row mean; finite or -INFINITY
                                (-INFINITY makes every block exact) */
  float scale;               /* softmax and score scale; 0 selects 1/sqrt(D) */
  int32_t prefix_len;        /* rows [0, prefix_len) are the packed text/audio prefix:
                                key blocks holding any of them are always exact (KV sink),
                                query blocks holding any of them attend densely */
  int32_t log_mass_bias;     /* centroid terms of unselected key blocks (Spark-H3 news page,
                                Spark-Reweight bullet); a = anchor = mean of the query rows
                                >= prefix_len (all rows when prefix_len = N):
                                0: logit s*q.kbar_j + log n_j, value vbar_j (block means);
                                1: plus bias_j = log mean_t exp(s*a.k_t) - s*a.kbar_j;
                                2: anchor-weighted summaries: with w_t = softmax over the
                                   block's rows of s*a.k_t, key ktil_j = sum_t w_t k_t, value
                                   vtil_j = sum_t w_t v_t, logit s*q.ktil_j + log n_j + bias_j,
                                   bias_j = log mean_t exp(s*a.k_t) - s*a.ktil_j.
                                Routing always scores the block means.  Other values:
                                SOL_ERR_INVALID_ARG. */
  int64_t in_stride_b, in_stride_n, in_stride_h;    /* element strides of Q, K, V */
  int64_t out_stride_b, out_stride_n, out_stride_h; /* element strides of O */
  int32_t routing;           /* 0: Sol threshold routing (tau), q_block = 64, a centroid term per
                                unselected key block (Star7 README 工作原理 > Sol);
                                1: Top-K routing, the SLA variant (Star7 README 工作原理 > SLA):
                                q_block = 128, each 128-row query block keeps the
                                k = round(topk_ratio * ceil(N/64)) key blocks with the largest
                                scores (equal scores: lower index first), query blocks holding
                                prefix rows keep every key block, unselected blocks are
                                dropped; tau is unused and log_mass_bias must be 0;
                                2: Top-K with the compressed branch (the Spark-H3
                                configuration): as 0 with the threshold test replaced by
                                membership in the row's k highest scores (q_block = 64, sink
                                and dense prefix rows kept, centroid terms and every
                                log_mass_bias mode apply; tau is unused).
                                Other values: SOL_ERR_INVALID_ARG. */
  float topk_ratio;          /* routing 1, 2: fraction of key blocks kept, in (0, 1];
                                k = floor(topk_ratio * n_kb + 0.5) in double precision from this
                                float (nearest, halves up), clamped to [1, n_kb]. */
  int32_t qk_int8;           /* 1: INT8 QK with per-block residual keys (thakicloud "MiniMax-H3
                                ComfyUI accel stack", section 실제 실험 결과, closing accuracy
                                paragraph): every exact logit is
                                s*(q.kmean16_j + sigma_q sigma_j (q_code . r_code)), where
                                kmean16_j is key block j's mean rounded to bf16, r = k - kmean16_j
                                is quantized to INT8 with one scale sigma_j = max|r| / 127 per
                                block, and each query row with its own sigma_q = max|q| / 127
                                (codes rint(x / sigma), ties to even, in fp32).  The tensor cores
                                run QK^T as an INT8 product; centroid terms and routing are
                                unchanged.  Needs D = 128.  0: bf16 QK. */
} sol_params;

/* Bytes of device workspace that sol_pool / sol_route / sol_attn_fwd share for
 * one problem of this shape (centroids, bias, routing mask, row counts).
 * Returns 0 for an invalid or empty problem. */
size_t sol_workspace_bytes(const sol_params* p);

/* Byte offsets, from the workspace base, of the pooled quantities that
 * sol_pool / sol_route leave in the workspace, for inspection and tests:
 *   offsets[0] qbar   fp32 [B, H, nqb, D]     offsets[1] kbar   fp32 [B, H, nkb, D]
 *   offsets[2] kbar   bf16 [B, H, nkb, D]     offsets[3] vbar   bf16 [B, H, nkb, D]
 *              (the centroid key/value the attention uses: ktil_j / vtil_j when
 *              log_mass_bias = 2, the block means otherwise)
 *   offsets[4] centroid-logit offset fp32 [B, H, nkb] = log n_j (+ bias_j)
 *   offsets[5] anchor fp32 [B, H, D] (log_mass_bias 1 or 2 only)
 *   offsets[6] exact-block bitmap uint32 [B*H*nqb, ceil(nkb/32)]
 *   offsets[7] row counts int32 [B*H*nqb]
 * with nqb = nkb = ceil(N/64).  With qk_int8 the workspace also holds the
 * residual key codes int8 [B, H, N, D], their scales fp32 [B, H, nkb] and the
 * bf16 block means [B, H, nkb, D] (written by sol_pool).  Returns SOL_ERR_INVALID_ARG for a bad p or
 * a NULL offsets array. */
sol_status sol_workspace_offsets(const sol_params* p, int64_t offsets[8]);

/* Byte offsets, from the workspace base, of what sol_pool writes for INT8 QK
 * (qk_int8 = 1), for inspection and tests:
 *   offsets[0] residual key codes int8 [B, H, N, D]  (codes of rows >= N are not written)
 *   offsets[1] residual scales fp32 [B, H, nkb]
 *   offsets[2] block means rounded to bf16 [B, H, nkb, D]
 * Returns SOL_ERR_INVALID_ARG for a bad p, qk_int8 = 0 or a NULL offsets array. */
sol_status sol_workspace_int8_offsets(const sol_params* p, int64_t offsets[3]);

/* Worst-case number of CSR column entries: B*H*ceil(N/64)*ceil(N/64) (64-row query-block rows). */
int64_t sol_col_capacity(const sol_params* p);

/* sol_pool: block centroids (Star7 README 工作原理 > Sol; Spark-H3 news page,
 * Spark-Reweight bullet).
 *   q, k, v  [B, N, H, D] bf16 device pointers, strides p->in_stride_*.
 *   ws       device workspace of ws_bytes >= sol_workspace_bytes(p) bytes,
 *            256-byte aligned.  Receives, per (b, h, block): qbar, kbar as
 *            fp32, kbar and vbar as bf16, the valid row count n_j, and the
 *            centroid-logit offset log n_j (+ bias_j when log_mass_bias).
 * Means are over each block's valid rows, accumulated in fp32.  With
 * log_mass_bias = 2 the bf16 key/value centroids are the anchor-weighted
 * summaries, computed in one pass over K and V after the anchor.  With
 * qk_int8 a further pass quantizes each key block's residual from its bf16
 * mean. */
sol_status sol_pool(const sol_params* p, const void* q, const void* k, const void* v,
                    void* ws, size_t ws_bytes, void* stream);

/* sol_route: block scores and CSR lists of exact key blocks (thakicloud blog,
 * 이 기술은 무엇인가; Star7 README 工作原理 > Sol, and 工作原理 > SLA for
 * routing 1).
 *   ws       workspace filled by sol_pool for the same p.
 *   row_ptr  int32 [B*H*ceil(N/64) + 1] device, written: exclusive scan
 *            of the per-row counts in (b, h, i) order; row_ptr[last] = nnz.
 *            Rows are 64-row query blocks for either routing (with routing 1
 *            the two halves of a 128-row block carry the same list).
 *   col_idx  int32 device, capacity sol_col_capacity(p); row r's exact key
 *            blocks, ascending, at [row_ptr[r], row_ptr[r+1]).
 * Routing 0: S_ij = s * qbar_i . kbar_j to fp32 accuracy (for D = 128 from
 * bf16 hi/lo terms on the tensor cores, within 4e-6 * |qbar_i||kbar_j| s of
 * the fp32 dot product); block j is exact for row i
 * iff S_ij > mean_j S_ij + tau * std_j S_ij (population std over all key
 * blocks), or j is a sink block, or i is a dense (prefix) query block.
 * Routing 1: qbar_i over 128 rows; row i keeps its k largest S_ij (equal
 * scores: lower j first), or every block if it holds prefix rows. */
sol_status sol_route(const sol_params* p, void* ws, size_t ws_bytes,
                     int32_t* row_ptr, int32_t* col_idx, void* stream);

/* sol_attn_fwd: exact + centroid attention (Star7 README 工作原理 > Sol).
 *   q, k, v  as for sol_pool; ws, row_ptr, col_idx as filled by sol_pool
 *            and sol_route for the same p (the caller may substitute its own
 *            CSR lists with the same layout, e.g. to replay a mask).
 *   o        [B, N, H, D] bf16 device, strides p->out_stride_*; written.
 *   lse      optional fp32 [B, H, N] device (natural-log normaliser); NULL
 *            to skip.
 * Row r of query block i: logits s*q_r.k_t over the rows t of the listed
 * key blocks, and s*q_r.kbar_j + log n_j (+ bias_j) with value vbar_j for
 * each unlisted key block j; one fp32 online softmax over all of them.
 * Keys at rows >= N are masked; O rows >= N are not written. */
sol_status sol_attn_fwd(const sol_params* p, const void* q, const void* k, const void* v,
                        const void* ws, size_t ws_bytes, const int32_t* row_ptr,
                        const int32_t* col_idx, void* o, float* lse, void* stream);

/* sol_route_static: the routing of sol_route without any caller-provided
 * scratch, for callers that cannot allocate device memory (a host framework
 * that owns every device allocation through a fixed-budget pool, or a code
 * path that must not allocate).  The pages describe no such entry point; it
 * has no counterpart in the method's sources.
 *   ws       the workspace sol_pool filled for the same p; only its pooled
 *            part is read, so ws_bytes may be as small as offsets[6] of
 *            sol_workspace_offsets (the bitmap offset).
 *   row_ptr, col_idx  outputs exactly as for sol_route (identical values).
 * The bitmap and row counts live in one fixed 8 MiB device array inside the
 * library, held by every GPU that loads it until the process exits; problems
 * needing more than 8 MiB (B*H*ceil(N/64) rows x (ceil(N/64/32) words + 1
 * count) x 4 bytes, bitmap rounded up to 256 bytes) are rejected with
 * SOL_ERR_UNSUPPORTED.  The library allocates nothing.  All calls share the
 * array: calls that overlap on the GPU race on it.  The first call on a
 * device looks up the array's device address; make it before any stream
 * capture. */
sol_status sol_route_static(const sol_params* p, const void* ws, size_t ws_bytes,
                            int32_t* row_ptr, int32_t* col_idx, void* stream);

/* sol_forward_host: pool + route + attention on HOST buffers, pipelined.
 *   q, k, v  host pointers [B, N, H, D] bf16 with p's in_stride_*; o a host
 *            pointer with p's out_stride_* (written: every row < N of every
 *            head).  Pinned (page-locked) memory lets the copies overlap the
 *            kernels; pageable memory works but the copies then serialise.
 *   heads_per_chunk  heads per pipeline chunk; 0 picks 4 (a chunk is also
 *            capped at H).  Must be >= 0.
 *   staging  device buffer of staging_bytes >= sol_host_staging_bytes(p,
 *            heads_per_chunk), 256-byte aligned, owned by the caller; two
 *            chunk slots of compact Q, K, V, O plus each chunk's workspace
 *            and CSR.
 * Heads are split into chunks; chunk c+1's host-to-device copy (an internal
 * copy-in stream), chunk c's kernels (on `stream`) and chunk c-1's O copy
 * back (an internal copy-out stream) overlap.  The output equals that of
 * sol_pool + sol_route + sol_attn_fwd on the whole problem bit for bit.
 * `stream` is ordered after all of it: synchronise it (or wait on an event
 * recorded on it) before reading o or reusing staging.  On first use per
 * device the library creates two non-blocking streams and seven events,
 * kept until exit; calls from several host threads enqueue one at a time.
 * The pages describe no such entry point: it serves the end-to-end path of
 * a caller whose tensors live in host memory. */
sol_status sol_forward_host(const sol_params* p, const void* q, const void* k, const void* v, void* o,
                            int32_t heads_per_chunk, void* staging, size_t staging_bytes, void* stream);

/* Bytes of device staging sol_forward_host needs for p and heads_per_chunk
 * (0 for an invalid or empty problem or a negative heads_per_chunk). */
size_t sol_host_staging_bytes(const sol_params* p, int32_t heads_per_chunk);

/* Synchronises `stream`, then reports and clears the device-side status word
 * that kernels set when a bounded wait expires (SOL_ERR_TIMEOUT) or a CSR
 * entry is out of range (SOL_ERR_INVALID_ARG). */
sol_status sol_last_device_status(void* stream);

/* ---- Adaptive partition (optional; Spark-H3 news page, Spark-Reblock
 * bullet, and its workflow paragraph: reblock_layout=q_reuse_k) ----------
 * sol_reblock computes, per (b, h), an order of the rows in which every 64
 * consecutive rows are one adaptive block: the key rows past the prefix
 * blocks (which stay in place) are whitened by the Cholesky factor of the
 * video queries' second moment (mean q q^T + 1e-4 trace / D * I), so that
 * the plain cosine of the unit vectors is the Mahalanobis cosine, and split
 * recursively along each group's principal axis (4 power steps on its
 * covariance from its first row minus its mean) at the size-balanced rank
 * 64 * ceil(ceil(n / 64) / 2), lowest projections left, ties to the lower
 * row; every group keeps ascending row order.  Queries reuse the keys' order.
 * perm[(b*H + h)*N + pos] (int32, device, caller-owned) = the original row
 * at position pos.  Fields used: B, N, H, D, prefix_len, in_stride_*; the
 * other fields must still pass the common validation.  The workspace (device,
 * 256-byte aligned, >= sol_reblock_workspace_bytes, which may be 0 when
 * every row is a prefix-block row) holds fp32 whitened keys, partial
 * moments (reused for the levels' Gram partials), the factor, the split
 * scratch, the split axes and the group means (about 1.22 GB at B=1, H=56,
 * N=32768, D=128); it may be reused once the stream has passed the call.
 *
 * A reblocked forward pass: sol_reblock; sol_gather_rows of q, k and v into
 * head-major copies [B, H, N, D] (in_stride_* describe the source); the
 * usual sol_pool / sol_route / sol_attn_fwd on the copies (strides
 * b = H*N*D, n = D, h = N*D); sol_scatter_rows of the head-major output
 * into o (out_stride_* describe the destination).  A perm entry outside
 * [0, N) is skipped and reported as SOL_ERR_INVALID_ARG through the device
 * status word.  All three enqueue on `stream` and return before the work
 * runs. */
size_t sol_reblock_workspace_bytes(const sol_params* p);
sol_status sol_reblock(const sol_params* p, const void* q, const void* k, void* ws, size_t ws_bytes,
                       int32_t* perm, void* stream);
/* perm must hold, for each (b, h), a permutation of 0 .. N-1 (as sol_reblock
 * writes it).  Only the range of each entry is checked (an entry outside
 * [0, N) is skipped and reported); a repeated entry is not detected, and a
 * scatter through it then writes some rows twice and leaves others as they
 * were.
 * xp[b, h, pos, :] = x[b, perm[b, h, pos], h, :]  (x strided by in_stride_*) */
sol_status sol_gather_rows(const sol_params* p, const int32_t* perm, const void* x, void* xp, void* stream);
/* x[b, perm[b, h, pos], h, :] = xp[b, h, pos, :]  (x strided by out_stride_*) */
sol_status sol_scatter_rows(const sol_params* p, const int32_t* perm, const void* xp, void* x, void* stream);

/* Fault injection for testing the bounded waits (the device-side failure
 * path).  Only a library built with SOL_FAULT_TEST (libsol_fault.so, whose
 * waits expire after 2^16 polls instead of 2^22) acts on it: from the next
 * sol_attn_fwd on, every CTA's softmax withholds its "P ready" arrive of
 * step `step` (0-based S tile; -1 restores normal operation), so the MMA
 * warp's bounded wait expires.  That launch then stops issuing, drains its
 * copies and MMAs, frees its tensor memory, writes no output and leaves
 * SOL_ERR_TIMEOUT in the device status word; the context stays usable.
 * Synchronous (a symbol copy), not for use while kernels run.  Returns
 * SOL_ERR_INVALID_ARG for step < -1; the product library returns
 * SOL_ERR_UNSUPPORTED and changes nothing. */
sol_status sol_debug_drop_arrive(int32_t step);

/* Static, human-readable name of a status code. */
const char* sol_status_string(sol_status s);

/* Text of the last error raised on this thread (argument or CUDA detail);
 * empty string if none. */
const char* sol_last_error_text(void);

#ifdef __cplusplus
}
#endif

#endif /* SOL_H_ */
