/*
 * xattn.h -- C ABI of the XAttention prefill hot path on NVIDIA B200 (sm_100a).
 *
 * The three calls below are the three steps of "XAttention: Block Sparse
 * Attention with Antidiagonal Scoring":
 *   xattn_score        strided antidiagonal scoring and block probabilities
 *                      (§2.1 Importance Prediction; §2.2; Algorithm 1)
 *   xattn_select       find_blocks threshold selection per query-block row
 *                      (§2.2 Threshold Block Selection, the find_blocks formula)
 *   xattn_sparse_attn  attention over the selected blocks only
 *                      (§1 step 3, "Block Sparse Attention")
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller. The library
 *   never allocates or frees them. Scratch space ("workspace") is also passed
 *   in by the caller, sized by the *_workspace_bytes() query.
 * - Q, K, V, O are contiguous [batch, heads, L, d] arrays. Q and O have hq
 *   heads; K and V have hkv heads. hq must be a multiple of hkv, and query
 *   head h reads KV head h / (hq / hkv) (grouped-query attention).
 * - NB = ceil(L / B) query blocks and key blocks. r = B / S reshaped rows per
 *   block. L must be a multiple of S (INVALID_ARG otherwise) but need not be a
 *   multiple of B: the last block then holds the L - (NB-1)*B remaining tokens
 *   (fewer reshaped rows and columns). Algorithm 1 only walks floor(L/B) whole
 *   blocks; this extension keeps every definition below and applies it to the
 *   tokens that exist: softmax rows run over the L/S reshaped columns, a block
 *   probability divides by its block's own number of reshaped rows (so rows of
 *   P still sum to 1), and attention has no query or key past L.
 * - Every call is asynchronous on the given CUDA stream (a cudaStream_t passed
 *   as void*; NULL means the legacy default stream). No call synchronises the
 *   device, except xattn_get_device_status.
 * - Arguments are checked on the host before anything is launched. A failed
 *   check returns a negative xattn_status and launches nothing.
 * - Device-side faults that a kernel can detect on its own (a pipeline wait
 *   that exceeded its time limit, a device-resident tau out of range) are
 *   recorded in a per-device status word that xattn_get_device_status reads
 *   and clears. Kernels never trap.
 *
 * Two further calls run the pages' ablation variants through the same
 * kernels: xattn_score_pattern (diagonal / random sampling instead of the
 * antidiagonal) and xattn_select_topk / xattn_select_topratio (fixed budgets
 * instead of the threshold).
 *
 * The remaining calls have no counterpart in the paper; each is documented
 * where it is declared:
 *   xattn_score_select         scoring and find_blocks in one call (P kept on chip)
 *   xattn_score_partials       the scoring GEMM alone (its partial sums, no P)
 *   xattn_sparse_attn_noalloc  the attention without a workspace
 *   xattn_check_lists          validation of block lists made by the caller
 *   xattn_prefill_host         the whole step on HOST buffers (the one call
 *                              whose tensors may live in host memory)
 *   xattn_prefill_varlen       the whole step on packed variable-length sequences
 *
 * Data types: XATTN_BF16 runs the tensor-core (tcgen05) kernels and needs
 * d = 128 and B = 128. XATTN_F32 runs plain FP32 CUDA-core kernels for small
 * problems and needs d in {32, 64, 128} and B <= 256.
 */
#ifndef XATTN_H_
#define XATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  XATTN_OK = 0,
  XATTN_ERR_INVALID_ARG = -1, /* bad shape, pointer, tau or stride */
  XATTN_ERR_UNSUPPORTED = -2, /* valid, but outside what the kernels handle */
  XATTN_ERR_CUDA = -3,        /* a CUDA runtime call failed */
  XATTN_ERR_WORKSPACE = -4,   /* workspace pointer NULL or too small */
  XATTN_ERR_TIMEOUT = -5      /* a kernel's bounded wait ran out (device status) */
} xattn_status;

typedef enum { XATTN_F32 = 0, XATTN_BF16 = 1 } xattn_dtype;

/* Problem shape. causal != 0 selects causal attention. dtype is an xattn_dtype. */
typedef struct {
  int batch, hq, hkv, L, d, B, S, causal, dtype;
} xattn_shape;

/* Largest hq accepted (the per-head tau vector travels as a kernel argument). */
#define XATTN_MAX_HEADS 256
/* Largest NB = ceil(L / B) accepted by xattn_select and xattn_score. */
#define XATTN_MAX_BLOCKS 4096

/*
 * Bytes of workspace xattn_score needs: one fp32 partial log-sum-exp per
 * (reshaped query row, allowed key block). Causal: batch*hq*r*NB*(NB+1)/2
 * floats; non-causal: batch*hq*(L/S)*NB floats. Returns 0 for an invalid shape.
 */
size_t xattn_score_workspace_bytes(const xattn_shape* shape);

/*
 * Block probabilities P (§2.2; Algorithm 1's A_approx, block-summed).
 *
 * For each (batch, query head h, query block b), the reshaped queries are
 * rows [Q[bB+tS+S-1], ..., Q[bB+tS]] (t = 0..r-1, joined along features),
 * and the reshaped keys are rows [K[cS], ..., K[cS+S-1]]. Let
 * x = Q_r K_r^T / sqrt(d*S). With causal != 0, reshaped column c is visible
 * to global reshaped row rho only when c <= rho. A = row softmax of x.
 * Then P[b, j] = (1/r_b) * (sum of A over the sub-block (b, j)), where r_b = r
 * for a whole block and the number of reshaped rows of a short last block, so
 * every row of P sums to 1. Causal rows are 0 for j > b.
 *
 * Q: [batch, hq, L, d], K: [batch, hkv, L, d], both of type shape->dtype and
 *    16-byte aligned.
 * probs: out, fp32 [batch, hq, NB, NB], fully written.
 * ws / ws_bytes: workspace of at least xattn_score_workspace_bytes(shape),
 *          4-byte aligned (every CUDA allocation is).
 * Errors: INVALID_ARG (NULL pointer, bad shape, misaligned ws), UNSUPPORTED
 * (dtype limits, NB > XATTN_MAX_BLOCKS), WORKSPACE, CUDA.
 */
int xattn_score(const void* Q, const void* K, const xattn_shape* shape, float* probs,
                void* ws, size_t ws_bytes, void* stream);

/*
 * find_blocks (§2.2): for every row (batch, h, b) of P, the smallest set of
 * allowed key blocks whose probabilities sum to at least tau[h]. Blocks are
 * ranked by probability (descending), ties by block index (ascending). The
 * allowed blocks are 0..b when causal, all NB otherwise. If tau[h] >= 1, or the
 * row's allowed sum never reaches tau[h], every allowed block is selected.
 * Sums are accumulated in fp64.
 *
 * probs: fp32 [batch, hq, NB, NB], device.
 * tau:   DEVICE pointer to hq floats (per-head thresholds, read by the kernels
 *        when they run, so a captured CUDA graph picks up new values written
 *        there). Each must lie in (0, 1]. A value outside (or NaN) cannot be
 *        seen on the host: the kernels select nothing in that head's rows
 *        (counts 0, mask words 0) and record the fault, which the next
 *        xattn_get_device_status returns as XATTN_ERR_INVALID_ARG.
 * mask:   out, uint32 [batch, hq, NB, ceil(NB/32)]; bit (j % 32) of word j / 32
 *         is set iff block j is selected. Fully written.
 * counts: out, int32 [batch, hq, NB], the number of selected blocks.
 * idx:    out, int32 [batch, hq, NB, NB]; the first counts[...] entries of a
 *         row are the selected block indices in ascending order. The rest of
 *         the row is left unwritten.
 * Errors (returned): INVALID_ARG (NULL pointer, bad shape), UNSUPPORTED, CUDA.
 */
int xattn_select(const float* probs, const float* tau, const xattn_shape* shape,
                 uint32_t* mask, int32_t* counts, int32_t* idx, void* stream);

/*
 * xattn_score and xattn_select in one call: the scoring GEMM, then one kernel
 * that reduces each query block's partials to its row of P and runs
 * find_blocks on it straight from on-chip memory, so P makes no round trip
 * through HBM (§2.2: block scores, then the threshold selection).
 *
 * tau:   DEVICE pointer to hq floats in (0, 1], read and checked by the
 *        kernels as for xattn_select.
 * probs: out, optional (may be NULL): fp32 [batch, hq, NB, NB], bit-identical
 *        to xattn_score's output when given.
 * mask, counts, idx: out, as for xattn_select, and bit-identical to
 *        xattn_select run on xattn_score's P.
 * ws / ws_bytes: the scoring workspace (xattn_score_workspace_bytes), 4-byte
 *          aligned.
 * Errors: as for xattn_score and xattn_select.
 */
int xattn_score_select(const void* Q, const void* K, const xattn_shape* shape, const float* tau,
                       float* probs, uint32_t* mask, int32_t* counts, int32_t* idx, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * Scoring with another sampling pattern inside each S x S tile: the
 * sparsity-pattern ablation of "XAttention: Block Sparse Attention with
 * Antidiagonal Scoring" (chapterpal page, Knowl 9; §3.4 Ablation Study)
 * compares the antidiagonal with diagonal and random sampling.
 *
 * perm: HOST pointer to S int32 values, a permutation of 0..S-1. Feature
 *       chunk i of a reshaped row pairs query token rho*S + perm[i] with key
 *       token c*S + i, so the score of tile (rho, c) is the sum of q.k over
 *       the cells (perm[i], i). perm[i] = S-1-i is the antidiagonal (equal to
 *       xattn_score), perm[i] = i the main diagonal; a random pattern is a
 *       permutation the caller draws. INVALID_ARG if perm is NULL or not a
 *       permutation.
 * Everything else (scale, causal mask, softmax, block sums, probs, workspace,
 * errors) is as for xattn_score.
 */
int xattn_score_pattern(const void* Q, const void* K, const xattn_shape* shape,
                        const int32_t* perm, float* probs, void* ws, size_t ws_bytes,
                        void* stream);

/*
 * The first stage of xattn_score alone: the strided antidiagonal product
 * (§2.1, Algorithm 1's Q_r K_r^T with the 1/sqrt(d*S) scale and the causal
 * mask), reduced within each key block and written to the workspace. It is
 * the tensor-core GEMM of the path by itself, for timing it on its own, and
 * for callers that reduce the sums themselves.
 *
 * For each (batch, query head) bh, reshaped query row rho (0 <= rho < L/S) and
 * allowed key block j (j <= rho / r when causal, all NB otherwise; r = B/S):
 *   L[bh, rho, j] = log2 sum over the visible reshaped columns c of block j of
 *                   2^(x[rho, c] * log2(e)),  x = Q_r K_r^T / sqrt(d*S)
 * (fp32; a column c of block j is visible when c < L/S and, causal, c <= rho).
 * Layout in ws (fp32): head bh starts at bh * H floats, H = r*NB*(NB+1)/2
 * (causal) or (L/S)*NB; within a head, the row of rho starts at
 * r*b*(b+1)/2 + t*(b+1) (causal, b = rho / r, t = rho % r) or rho*NB, and
 * holds the row's allowed blocks j = 0, 1, ... in order. P follows as
 * P[b, j] = (1/r_b) sum over the block's rows rho of 2^(L[rho, j] - LSE[rho]),
 * LSE[rho] = log2 sum_j 2^L[rho, j].
 *
 * ws / ws_bytes: as for xattn_score (the sums occupy its first bytes).
 * Errors: as for xattn_score.
 */
int xattn_score_partials(const void* Q, const void* K, const xattn_shape* shape, void* ws,
                         size_t ws_bytes, void* stream);

/*
 * Fixed-budget selection, the Top-K and Top-Ratio strategies of the
 * selection-strategy ablation (chapterpal page, Knowl 9; §3.4 Ablation Study).
 * A row's allowed blocks (0..b when causal, all NB otherwise; n of them) are
 * ranked as in xattn_select (probability descending, index ascending) and the
 * first k are kept:
 *   xattn_select_topk:     k = min(k[h], n). k: HOST pointer to hq int32
 *                          values, each >= 1 (a token budget K is K / B blocks).
 *   xattn_select_topratio: k = ratio[h] * n rounded to the nearest integer
 *                          (halves up), at least 1 and at most n. ratio: HOST
 *                          pointer to hq floats in (0, 1]. The product is
 *                          formed exactly, so the count is exact.
 * Outputs (mask, counts, idx) have the layout of xattn_select. INVALID_ARG for
 * a NULL pointer or a k / ratio out of range.
 */
int xattn_select_topk(const float* probs, const int32_t* k, const xattn_shape* shape,
                      uint32_t* mask, int32_t* counts, int32_t* idx, void* stream);
int xattn_select_topratio(const float* probs, const float* ratio, const xattn_shape* shape,
                          uint32_t* mask, int32_t* counts, int32_t* idx, void* stream);

/*
 * Bytes of workspace xattn_sparse_attn needs (the work schedule:
 * 8 * (batch*hq*NB + 32) bytes). Returns 0 for an invalid shape.
 */
size_t xattn_attn_workspace_bytes(const xattn_shape* shape);

/*
 * Block-sparse attention. For each query q in query block b of head h:
 *   O[q] = sum_k softmax_k(Q[q] . K[k] / sqrt(d)) V[k]
 * over the keys k of the blocks idx[batch, h, b, 0 .. counts[batch, h, b]-1]
 * (KV head h / (hq/hkv)). With causal != 0, keys k > q are dropped, and listed
 * blocks j > b are skipped. A row with no visible key gets O = 0 and
 * lse = -inf.
 *
 * Q, K, V: as for xattn_score (16-byte aligned); O: out, same type as Q,
 *          [batch, hq, L, d].
 * counts, idx: as written by xattn_select (device).
 * lse: out, optional (may be NULL), fp32 [batch, hq, L], natural-log
 *      log-sum-exp of each row's scaled logits.
 * ws / ws_bytes: at least xattn_attn_workspace_bytes(shape).
 * The work units (batch, h, b) run on persistent CTAs, longest list first,
 * dealt in serpentine rounds; when the lists average at least 48 blocks the
 * order is grouped by KV head first (one head's K/V at a time stays in L2).
 * The order changes only the speed: every unit's output is the same.
 * Every call is capturable in a CUDA graph.
 */
int xattn_sparse_attn(const void* Q, const void* K, const void* V, const xattn_shape* shape,
                      const int32_t* counts, const int32_t* idx, void* O, float* lse,
                      void* ws, size_t ws_bytes, void* stream);

/* Largest batch*hq*NB accepted by xattn_sparse_attn_noalloc (bf16 calls; the
 * fp32 kernel uses no scratch and has no such limit). */
#define XATTN_NOALLOC_MAX_UNITS (1 << 18)

/*
 * xattn_sparse_attn without a workspace: the same attention, and for the same
 * inputs the same outputs, but the call allocates nothing and takes no
 * workspace. This entry point has no counterpart in the paper. It is for
 * callers that cannot call cudaMalloc: a host program whose device memory all
 * belongs to another allocator, or a serving loop that may not allocate once
 * running (an allocation can synchronise the device or fail under memory
 * pressure).
 *
 * The work order lives in a __device__ array of the library, sized for
 * XATTN_NOALLOC_MAX_UNITS work units (2 MiB). Each GPU that loads the library
 * holds it until the process exits. A bf16 call returns XATTN_ERR_WORKSPACE
 * when batch*hq*NB exceeds that limit (the fp32 path uses no scratch).
 *
 * The first call on a device (and the first after the device's context has
 * changed, e.g. after cudaDeviceReset) looks up the array's device address
 * (cudaGetSymbolAddress) and caches it for that context; make that first call
 * before any stream capture. All calls on a device share the array and it
 * keeps the last call's contents. Calls whose kernels overlap on the GPU (for
 * example on two unordered streams) race on it, so order such calls on one
 * stream.
 * Arguments and other errors are as for xattn_sparse_attn.
 */
int xattn_sparse_attn_noalloc(const void* Q, const void* K, const void* V,
                              const xattn_shape* shape, const int32_t* counts,
                              const int32_t* idx, void* O, float* lse, void* stream);

/*
 * Validates block lists made outside xattn_select before they go to
 * xattn_sparse_attn. That call trusts the layout xattn_select writes: each
 * counts[batch, h, b] is in [0, NB], and the first counts[batch, h, b]
 * entries of idx[batch, h, b, :] are strictly ascending block indices in
 * [0, NB) (causal rows may end in blocks above the diagonal; the attention
 * drops those). A list that breaks it gives wrong rows but no out-of-bounds
 * access. This entry point has no counterpart in the paper.
 *
 * counts, idx: device, [batch, hq, NB] and [batch, hq, NB, NB] int32 (entries
 *              past a row's count are not read).
 * bad_rows: device, one int32; the call sets it to the number of rows that
 *           break the layout (0 for valid lists). Read it after the stream
 *           has reached it. Owned by the caller.
 * Returns XATTN_ERR_INVALID_ARG for a bad shape or a NULL pointer, else the
 * launch status. Capturable in a CUDA graph.
 */
int xattn_check_lists(const int32_t* counts, const int32_t* idx, const xattn_shape* shape,
                      int32_t* bad_rows, void* stream);

/*
 * Workspace bytes of xattn_prefill_host for a shape and a chunk size (see
 * below). Returns 0 for an invalid shape or chunk size.
 */
size_t xattn_prefill_host_workspace_bytes(const xattn_shape* shape, int kv_heads_per_chunk);

/*
 * The whole prefill step of one layer -- xattn_score_select (threshold tau),
 * then xattn_sparse_attn -- on Q, K, V held in HOST memory, writing O (and
 * lse) back to host memory. Results are bit-identical to those two calls on
 * device copies of the same tensors. This entry point has no counterpart in
 * the paper: it is the step as a host program sees it, with the
 * host<->device copies overlapped with the compute.
 * Every step of the method is independent across KV heads, so the call cuts
 * the layer into chunks of kv_heads_per_chunk KV heads (with their hq/hkv
 * query heads each) per batch entry; 0 means 1, and a last chunk of a batch
 * entry may be smaller when hkv is not a multiple. Each chunk goes through a
 * ring of two device slots: copy in on one internal stream, compute on
 * `stream`, copy out on a second internal stream, so chunk c+1 is copied in
 * and chunk c-1 copied out while chunk c is computed.
 * Q, K, V: [batch, heads, L, d] contiguous, as for xattn_sparse_attn, in host
 *          memory (page-locked, e.g. from cudaHostAlloc, for the copies to
 *          overlap; pageable memory gives the same results more slowly) or
 *          device memory. Not modified.
 * tau:     HOST pointer to hq floats in (0, 1], checked before anything is
 *          launched (INVALID_ARG) and passed to the kernels by value: this
 *          host-facing call takes its thresholds from the host.
 * O:       out, [batch, hq, L, d] of the same type, host or device memory.
 * lse:     out, optional (may be NULL), fp32 [batch, hq, L], as for
 *          xattn_sparse_attn.
 * ws / ws_bytes: DEVICE workspace of at least
 *          xattn_prefill_host_workspace_bytes(shape, kv_heads_per_chunk)
 *          bytes, 256-byte aligned; it holds the two slots and the scratch of
 *          both steps (WORKSPACE otherwise).
 * Ordering: the call is asynchronous on `stream` like every other call: the
 * copies start after the work queued on `stream` before the call, and work
 * queued on `stream` after it starts once O and lse are in place. The host
 * buffers must stay valid and unchanged until then. The call creates, and
 * releases, its two copy streams and its events on each call.
 * Errors: INVALID_ARG (NULL pointer, bad shape or tau, kv_heads_per_chunk < 0
 * or > hkv), UNSUPPORTED and CUDA as for the two steps, WORKSPACE. A failure
 * part-way through leaves O partly written.
 */
int xattn_prefill_host(const void* Q, const void* K, const void* V, const xattn_shape* shape,
                       const float* tau, void* O, float* lse, int kv_heads_per_chunk, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * Workspace bytes of xattn_prefill_varlen for these lengths: the scratch of
 * the longest sequence, once for each concurrent lane (one lane per non-empty
 * sequence, at most four). Returns 0 when the lengths or the shape are
 * invalid.
 */
size_t xattn_prefill_varlen_workspace_bytes(const xattn_shape* shape, int nseq,
                                            const int32_t* seqlens);

/*
 * The whole prefill step -- xattn_score_select (threshold tau), then
 * xattn_sparse_attn -- on a batch of nseq sequences of different lengths.
 * Sequence i has L_i = seqlens[i] tokens (HOST array; 0 skips a sequence;
 * otherwise a multiple of S, and not necessarily of B: a short last block is
 * handled as for a fixed-length batch). Results are bit-identical to the two
 * calls run on sequence i alone as a batch-1 problem.
 * Layout: the sequences are packed one after another. Sequence i of Q is a
 * contiguous [hq, L_i, d] array starting T_i * hq * d elements into Q, with
 * T_i = L_0 + ... + L_{i-1}; K and V hold [hkv, L_i, d] arrays at T_i * hkv *
 * d; O is laid out like Q, and lse (optional, may be NULL) holds [hq, L_i]
 * fp32 arrays at T_i * hq. All DEVICE pointers, 16-byte aligned for bf16.
 * shape: hq, hkv, d, B, S, causal and dtype apply to every sequence; its
 * batch and L are ignored.
 * tau: HOST pointer to hq floats in (0, 1], checked before anything is
 *      launched and passed to the kernels by value.
 * ws / ws_bytes: DEVICE workspace of at least
 *          xattn_prefill_varlen_workspace_bytes(shape, nseq, seqlens) bytes,
 *          256-byte aligned.
 * The sequences are dealt round-robin over up to four lanes that run
 * concurrently (a short sequence's kernels leave most SMs free): lane 0 is
 * `stream`, the others are streams the call creates, forked off `stream` with
 * an event and joined back into it, so the call is ordered on `stream` like
 * any other. Each lane has its own part of the workspace.
 * Errors: INVALID_ARG (NULL pointer, nseq < 1, a negative length, no
 * non-empty sequence, a length that is not a multiple of S, bad tau),
 * UNSUPPORTED (dtype limits, a sequence with more than XATTN_MAX_BLOCKS
 * blocks, more than 2^31 - 1 query rows in all), WORKSPACE, CUDA. Every
 * argument is checked before the first launch.
 * This entry point has no counterpart in the paper.
 */
int xattn_prefill_varlen(const void* Q, const void* K, const void* V, const xattn_shape* shape,
                         int nseq, const int32_t* seqlens, const float* tau, void* O,
                         float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word. Returns XATTN_OK, XATTN_ERR_TIMEOUT if a kernel gave up a bounded
 * wait since the last call, XATTN_ERR_INVALID_ARG if a selection kernel met a
 * device-resident tau outside (0, 1], or XATTN_ERR_CUDA if the stream reports
 * an error. When several faults happened, the last one recorded is returned.
 */
int xattn_get_device_status(void* stream);

/*
 * Self-test of the failure detection: launches one small kernel whose
 * bounded pipeline wait (the same wait every kernel of the library uses) runs
 * out after its time limit (about 2 s), because nothing ever completes the
 * barrier it waits on. The kernel records the time-out in the device status
 * word and returns normally, so the next xattn_get_device_status on the stream
 * returns XATTN_ERR_TIMEOUT and clears it, and the context stays usable. No
 * fault, trap or unbounded wait is involved. Returns XATTN_OK once launched.
 */
int xattn_selftest_timeout(void* stream);

/* Static, human-readable text for an xattn_status value. */
const char* xattn_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* XATTN_H_ */
