/*
 * libhils: HiLS-Attention forward pass (and its backward) on NVIDIA B200 (sm_100a). C ABI.
 *
 * The method is Hierarchical Landmark Sparse attention, from "Hierarchical Sparse
 * Attention Done Right: Toward Infinite Context Modeling" (arXiv 2607.02980). The
 * citations below name the page (picx.dev summary, or the rcap.io post) and the
 * section or equation on it.
 *
 * Stages, one entry point each:
 *   hils_summarize       landmark chunk summaries k'_c, b'_c         (summary, Methodology 1, Eq. 8)
 *   hils_select          chunk scores s^_{i,c} and top-K selection   (summary, Eq. 7 and Methodology 2;
 *                                                                     post, pseudocode figure)
 *   hils_attend_prefill  hierarchical softmax over the selected chunks plus the sliding
 *   hils_attend_decode   window, for every position of a sequence, or for one new token
 *                        per sequence against a KV cache            (summary, Methodology 2, Eq. 10;
 *                                                                     post, pseudocode figure)
 *   hils_decode          one decode step: hils_select then hils_attend_decode, chained
 *   hils_summarize_append  decode-time summary of the chunk each newest token completed
 *   hils_attend_prefill_backward, hils_select_backward, hils_summarize_backward
 *                        gradients for a fixed selection            (Eq. 10, Eq. 7, Eq. 8)
 *
 * Conventions shared by every call
 * --------------------------------
 * Tensors. A 4-D tensor [B, H, T, d] is described by hils_ctensor/hils_tensor:
 *   element (b, h, t, x) is at ptr + b*sb + h*sh + t*st + x, with strides counted in
 *   elements of params->dtype. The head dimension x is contiguous (stride 1).
 *   ptr must be 16-byte aligned, and sb, sh, st times the element size must be
 *   multiples of 16 bytes (HILS_ERR_ALIGNMENT otherwise).
 *   Plain arrays (Bsum, idx, score, nsel, lse, qpos, cache_len) are dense row-major
 *   with the shape given beside them.
 * Memory. Every pointer is device memory that the caller allocates and owns. The
 *   library allocates nothing, frees nothing and never synchronises: each call
 *   enqueues its kernels on `stream` and returns.
 * Workspace. Calls that need scratch memory take (workspace, ws_bytes). Query the
 *   size with hils_workspace_bytes(). The workspace carries arrival counters that
 *   every call leaves at zero; zero a new workspace once before its first use (for
 *   example with hils_workspace_init). Calls that share a workspace must not
 *   overlap in time on the device.
 * Errors. A call validates its arguments before launching anything and returns a
 *   hils_status. HILS_ERR_CUDA means a launch failed; hils_last_cuda_error() then
 *   gives the CUDA error text for the calling thread. No exception crosses the ABI.
 * Threads. Calls keep no global state and may be made from several host threads.
 *
 * Stated readings of the method (the pages leave these open):
 *   - Every dot product is multiplied by scale = 1/sqrt(d); the entropy bias b'_c
 *     is added unscaled (Eq. 7).
 *   - Chunk c holds tokens [c*S, (c+1)*S). It is eligible for the query at position
 *     t when c < floor(t / S): only complete chunks strictly before the query's own.
 *   - The sliding window is the W most recent tokens including the query's own,
 *     [max(0, t-W+1), t]. It joins the selected chunks under one normaliser
 *     Z^_i = sum_{c selected} exp(s^_{i,c}) + sum_{j in window} exp(scale q_i.k_j),
 *     and a token that lies both in a selected chunk and in the window enters
 *     through both terms.
 *   - Queries with fewer than K eligible chunks keep all of them; the rest of their
 *     selection row is padding (idx -1, score -inf). A query with no selected chunk
 *     and an empty window gets o = 0 and lse = -inf.
 *   - Grouped-query attention (summary page, Methodology 3, GQA adaptation): with
 *     Hk = params->H_kv key-value heads, the H query heads form groups of G = H / Hk
 *     consecutive heads, query head h reading key-value head h / G. Landmark queries,
 *     summaries and chunk scores stay per query head; the heads of a group keep the
 *     same chunks, the K chunks with the largest maximum over the group of s^_{h,i,c}
 *     (equal maxima to the lower chunk index), and each head weights them with its own
 *     s^_{h,i,c} in Eq. 10. K, V, the KV cache, idx and nsel then have Hk heads; Q,
 *     Q_cal, LQ, Ksum, Bsum, score, O and lse keep H. H_kv = 0 or H is multi-head
 *     attention (G = 1).
 */
#ifndef HILS_H
#define HILS_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { HILS_F32 = 0, HILS_BF16 = 1 } hils_dtype;

typedef enum {
    HILS_OK = 0,
    HILS_ERR_INVALID_ARG = 1,  /* null pointer, negative size, inconsistent shape */
    HILS_ERR_UNSUPPORTED = 2,  /* d not in {64,128}, S != 64, K > 32, unknown flags, H / H_kv > 8,
                                  hils_select_backward over too many chunks */
    HILS_ERR_ALIGNMENT = 3,    /* pointer or stride not 16-byte aligned */
    HILS_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required */
    HILS_ERR_CUDA = 5          /* a kernel launch failed; see hils_last_cuda_error() */
} hils_status;

/* Read-only / writable strided view of a [B, H, T, d] tensor (strides in elements). */
typedef struct {
    const void *ptr;
    int64_t sb, sh, st;
} hils_ctensor;

typedef struct {
    void *ptr;
    int64_t sb, sh, st;
} hils_tensor;

/* Flags (hils_params.flags).
 *   HILS_FLAG_EXCLUDE_WINDOW_CHUNKS: the window-exclusion variant. A chunk that lies
 *     wholly inside the query's window [max(0, t-W+1), t] is not eligible for
 *     selection (the window already attends its tokens exactly), so no token is
 *     counted twice except in the chunk holding the window's first token when the
 *     window starts inside a chunk (that chunk stays eligible, or its earlier tokens
 *     would be reached by neither term). The pages' normaliser over the selected chunks
 *     and the window (summary page, Methodology 2) does not say whether a token may be
 *     counted in both; without the flag it may (the default). Only hils_select and
 *     hils_decode read the flag; summaries and the attend calls are unchanged. */
#define HILS_FLAG_EXCLUDE_WINDOW_CHUNKS 1u
/*   HILS_FLAG_DIAG_EXPIRE_WAITS: diagnostic, for tests of the failure path. The
 *     tensor-core kernels of hils_select (bf16, d = 128, many queries), of
 *     hils_attend_prefill and of hils_attend_prefill_backward (bf16, d = 128) bound every
 *     wait on work in progress (copies, tensor-core operations, other warps' hand-offs)
 *     by a time limit of the GPU's global timer (0.1 s). With this flag every such wait expires at its first check,
 *     whether or not its phase has completed. The kernel then sets the call's status word (the
 *     first 4 bytes of its workspace, bit 0), stops issuing work, waits (bounded by the
 *     normal limit) for the copies and operations it already started, releases its
 *     tensor memory and returns without writing the outputs of unfinished work. Other
 *     calls and other kernels ignore the flag. */
#define HILS_FLAG_DIAG_EXPIRE_WAITS 0x80000000u

/* Problem description shared by every call.
 *   B      batch (sequences), H query heads,
 *   d      head dimension: 64 or 128,
 *   S      chunk size: 64,
 *   K      chunks kept per query (top-K): 0..32,
 *   W      sliding-window length in tokens: >= 0,
 *   dtype  element type of every Q/K/V/LQ/Ksum/O tensor,
 *   scale  softmax scale; 0 selects (float)(1/sqrt(d)),
 *   flags  0, or HILS_FLAG_EXCLUDE_WINDOW_CHUNKS and HILS_FLAG_DIAG_EXPIRE_WAITS (above);
 *          other bits are rejected,
 *   H_kv   key-value heads: 0 (= H) or a divisor of H with H / H_kv <= 8; groups of
 *          G = H / H_kv query heads share a key-value head and their chunk selection
 *          (see above). */
typedef struct {
    int B, H, d, S, K, W;
    hils_dtype dtype;
    float scale;
    uint32_t flags;
    int H_kv;
} hils_params;

/* Which call a workspace size is asked for. */
typedef enum {
    HILS_CALL_SELECT = 0,
    HILS_CALL_ATTEND_PREFILL = 1,
    HILS_CALL_ATTEND_DECODE = 2,
    HILS_CALL_DECODE = 3,
    HILS_CALL_ATTEND_BACKWARD = 4
} hils_call;

/* Landmark chunk summaries (summary page, Methodology 1, Eq. 8).
 * For every complete chunk c < C = floor(N / S) of every (b, h), h a query head:
 *   l_j = scale * q'_c . k_j for the S keys of the chunk, p = softmax(l),
 *   k'_c = sum_j p_j k_j,   b'_c = -sum_j p_j log p_j.
 *   K     [B, Hk, N, d] keys of the sequence (only the first C*S positions are read;
 *         query head h reads key-value head h / G)
 *   N     number of tokens
 *   LQ    [B, H, C, d]  landmark query q'_c of each chunk
 *   Ksum  [B, H, C, d]  out: k'_c in dtype (float32 sums rounded to nearest-even)
 *   Bsum  [B, H, C]     out: b'_c, float32, dense
 * Returns HILS_OK, or an error before any launch. */
int hils_summarize(const hils_params *p, hils_ctensor K, int N, hils_ctensor LQ,
                   hils_tensor Ksum, float *Bsum, cudaStream_t stream);

/* Decode-time summary of the chunk each sequence's newest token completed (the same
 * Eq. 8 arithmetic, and the same bits, as hils_summarize): for every b whose
 * cache_len[b] is a positive multiple of S with cache_len[b] / S <= C, chunk
 * c = cache_len[b] / S - 1 of every head h is summarised into Ksum[b, h, c] and
 * Bsum[b, h, c]; every other entry of Ksum and Bsum, and every other sequence, is left
 * as it was. Run after appending a token and before the next decode step's selection:
 * the chunk becomes eligible for the query at position cache_len[b].
 *   K          [B, Hk, T, d] the KV cache's keys, T >= cache_len[b]
 *   cache_len  [B] int32, device
 *   LQ         [B, H, C, d] landmark queries
 *   Ksum, Bsum [B, H, C, d] / [B, H, C] the summary table (capacity C chunks)
 * Returns HILS_OK, or an error before any launch. */
int hils_summarize_append(const hils_params *p, hils_ctensor K, const int32_t *cache_len, hils_ctensor LQ,
                          hils_tensor Ksum, float *Bsum, int C, cudaStream_t stream);

/* Chunk scores and top-K (summary page, Eq. 7 and Methodology 2; post, pseudocode).
 * For every query i at position t_i, every eligible chunk c < min(floor(t_i/S), C) gets
 *   s^_{i,c} = scale * (q~_i . k'_c) + b'_c,
 * and the K chunks with the largest s^ are kept; equal scores go to the lower chunk
 * index. The ranking is exact: it equals the ranking of the float64 value
 * (sum_x q~_x k'_x) * scale + b'_c (products and sums in x order, each rounded to
 * float64) computed from the stored inputs.
 *   Qcal  [B, H, Lq, d]  calibrated scoring query q~_i
 *   Lq    queries per (b, h)
 *   qpos  [B, Lq] int32 position t of each query, or NULL for t = i (prefill)
 *   Ksum  [B, H, C, d]  summary keys k'_c;  Bsum [B, H, C] float32 entropy biases b'_c
 *   C     number of summarised chunks
 *   idx   [B, Hk, Lq, K] int32 out: kept chunks in ascending chunk index, -1 padding
 *         (with G > 1: the group's chunks, ranked by the maximum over its heads of the
 *         exact value below)
 *   score [B, H, Lq, K] float32 out: s^_{i,c} of each kept chunk for each query head
 *         (float32 evaluation, within 2^-9 * scale * |q~| |k'_c| + 2^-20 |s^| of the
 *         exact value), -inf padding
 *   nsel  [B, Hk, Lq] int32 out: number of kept chunks, min(K, eligible)
 *   workspace, ws_bytes: scratch of hils_workspace_bytes(p, HILS_CALL_SELECT, Lq, C) bytes
 *         (at least 256), zeroed before first use. Its first 32-bit word is a status
 *         word: the paths with bounded waits (the tensor-core path for bf16, d = 128 and
 *         many queries; the bf16 decode-shaped screen, whose rows arrive by TMA) set it
 *         nonzero if a wait on their own asynchronous copies or matrix operations ever
 *         expires, and then write no output for the affected queries. */
int hils_select(const hils_params *p, hils_ctensor Qcal, int Lq, const int32_t *qpos,
                hils_ctensor Ksum, const float *Bsum, int C,
                int32_t *idx, float *score, int32_t *nsel,
                void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Hierarchical softmax for every position of a sequence (summary page, Methodology 2,
 * Eq. 10; post, pseudocode). Query i sits at t = i and attends to
 *   - each kept chunk c with weight exp(s^_{i,c}) / Z^_i on the chunk's own softmax
 *     output sum_{j in c} softmax_j(scale q_i.k_j) v_j, and
 *   - each window token j in [max(0, i-W+1), i] with weight exp(scale q_i.k_j) / Z^_i.
 *   Q [B, H, N, d];  K, V [B, Hk, N, d] (query head h reads key-value head h / G)
 *   idx, score, nsel: as written by hils_select ([B, Hk, N, K], [B, H, N, K],
 *         [B, Hk, N]): each row's first nsel entries are
 *         distinct chunks in ascending chunk index (score is used as the chunk's
 *         log-mass; passing exact log Z_{i,c} instead gives exact block-sparse attention)
 *   O    [B, H, N, d]  out, dtype (float32 result rounded to nearest-even)
 *   lse  [B, H, N] float32 out: log Z^_i, or NULL
 *   workspace, ws_bytes: hils_workspace_bytes(p, HILS_CALL_ATTEND_PREFILL, N, C) bytes,
 *         zeroed before first use. Its first 32-bit word is a status word: the bf16,
 *         d = 128 path (tensor cores, bounded waits) sets it nonzero if a wait on its own
 *         asynchronous copies or matrix operations ever expires, and then writes no output
 *         for the affected tile. */
int hils_attend_prefill(const hils_params *p, hils_ctensor Q, hils_ctensor K, hils_ctensor V,
                        int N, const int32_t *idx, const float *score, const int32_t *nsel,
                        hils_tensor O, float *lse, void *workspace, size_t ws_bytes,
                        cudaStream_t stream);

/* Hierarchical softmax for one new token per sequence against its KV cache (same
 * passages). Sequence b holds cache_len[b] tokens and its query sits at
 * t = cache_len[b] - 1 (the query's own key and value are the last cache entries).
 *   Q      [B, H, 1, d]
 *   Kc, Vc [B, Hk, Lmax, d] KV cache; positions >= cache_len[b] are never read
 *   cache_len [B] int32 on the device
 *   idx, nsel [B, Hk, 1, K] / [B, Hk, 1] and score [B, H, 1, K] from hils_select with
 *          qpos = cache_len - 1
 *   O      [B, H, 1, d] out;  lse [B, H] float32 out, or NULL
 *   workspace, ws_bytes: hils_workspace_bytes(p, HILS_CALL_ATTEND_DECODE, 1, 0). */
int hils_attend_decode(const hils_params *p, hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc,
                       const int32_t *cache_len,
                       const int32_t *idx, const float *score, const int32_t *nsel,
                       hils_tensor O, float *lse, void *workspace, size_t ws_bytes,
                       cudaStream_t stream);

/* One decode step: hils_select with qpos = cache_len - 1 (Lq = 1), then
 * hils_attend_decode on its outputs, enqueued as one chain on `stream` (the same
 * passages as the two calls). Results are those of the two calls made in turn: the
 * same kept chunks and scores (idx, score, nsel), and O and lse within rounding of
 * hils_attend_decode's.
 * Inside the chain the attend's window tiles need not wait for the select: its first
 * kernel starts only after all earlier work on the stream, so the window overlaps the
 * chunk selection.
 *   Qcal [B, H, 1, d]; Ksum [B, H, C, d]; Bsum [B, H, C]; C summarised chunks
 *   Q, Kc, Vc, cache_len, O, lse: as for hils_attend_decode
 *   idx [B, Hk, 1, K], score [B, H, 1, K], nsel [B, Hk, 1]: out
 *   workspace, ws_bytes: hils_workspace_bytes(p, HILS_CALL_DECODE, 1, C) bytes, zeroed
 *         before first use (the select part first, then the attend part). */
int hils_decode(const hils_params *p, hils_ctensor Qcal, hils_ctensor Ksum, const float *Bsum, int C,
                hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc, const int32_t *cache_len,
                int32_t *idx, float *score, int32_t *nsel, hils_tensor O, float *lse,
                void *workspace, size_t ws_bytes, cudaStream_t stream);

/* hils_attend_decode without a workspace argument: the library keeps the scratch
 * memory itself, in one fixed 4 MiB array of device global memory that every GPU
 * loading this library holds until the process exits. The paper has no counterpart;
 * this entry point exists for callers that cannot allocate device memory: a plug-in
 * that is handed only raw pointers and a stream by a host application owning every
 * allocation, or code running where device allocation is forbidden or would break a
 * fixed memory budget.
 *   Arguments, layouts and results are those of hils_attend_decode.
 *   Capacity: (B*H) * (K + ceil(W/64)) * (d+1) floats plus 256-byte-rounded counters
 *   must fit in 4 MiB (hils_workspace_bytes(p, HILS_CALL_ATTEND_DECODE, 1, 0) <=
 *   4194304); larger problems return HILS_ERR_WORKSPACE before anything is launched.
 *   Set-up: the first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before any
 *   stream capture. Each call then zeroes the array's counters on `stream`
 *   (cudaMemsetAsync) and launches; nothing is allocated or freed.
 *   All calls share the one array and it keeps the last call's contents: calls whose
 *   work overlaps on the GPU (other streams, other host threads) race on it. */
int hils_attend_decode_noalloc(const hils_params *p, hils_ctensor Q, hils_ctensor Kc, hils_ctensor Vc,
                               const int32_t *cache_len,
                               const int32_t *idx, const float *score, const int32_t *nsel,
                               hils_tensor O, float *lse, cudaStream_t stream);

/* Backward pass for a fixed selection (summary page, Methodology 1-2, Eq. 7, 8, 10;
 * top-K is piecewise constant, so no gradient flows through the choice of chunks).
 * Gradients are float32, dense and row-major, in the shapes of their tensors. Three
 * calls, in this order, give every gradient of sum(O * dO):
 *   hils_attend_prefill_backward -> dQ, dK and dV (token terms), dscore
 *   hils_select_backward         -> dQcal, dKsum, dBsum
 *   hils_summarize_backward      -> dLQ, and the summaries' share of dK
 * Arrays marked "accumulated" are added to with atomic adds (in no fixed order): zero
 * them before the first call. Queries are prefill positions t = i. */

/* Eq. 10 backward. Inputs as hils_attend_prefill (idx, score, nsel from hils_select),
 * with its outputs O [B,H,N,d] (dtype) and lse [B,H,N], and dO [B,H,N,d] float32.
 *   dQ     [B, H, N, d]   out (written)
 *   dK, dV [B, Hk, N, d]  accumulated
 *   dscore [B, H, N, K]   out: the gradient of each kept chunk's score, 0 padding
 *   workspace, ws_bytes: hils_workspace_bytes(p, HILS_CALL_ATTEND_BACKWARD, N, 0) bytes
 *         (the inverted index of the selection, D_i = dO_i . o_i, and for bf16 with
 *         d = 128 per-entry records and bf16 copies of dO and Q), no initialisation
 *         needed. Its first 32-bit word is a status word that each call clears: the bf16,
 *         d = 128 path (tensor cores, bounded waits) sets it nonzero if a wait on its own
 *         asynchronous copies or matrix operations ever expires, and then adds nothing
 *         more for the affected work item. */
int hils_attend_prefill_backward(const hils_params *p, hils_ctensor Q, hils_ctensor K, hils_ctensor V, int N,
                                 const int32_t *idx, const float *score, const int32_t *nsel,
                                 hils_ctensor O, const float *lse, const float *dO,
                                 float *dQ, float *dK, float *dV, float *dscore, void *workspace,
                                 size_t ws_bytes, cudaStream_t stream);

/* Eq. 7 backward: dQcal [B,H,Lq,d] (written) = scale sum_k dscore_k k'_{idx_k};
 * dKsum [B,H,C,d] += scale dscore q~ and dBsum [B,H,C] += dscore (accumulated).
 * Returns HILS_ERR_UNSUPPORTED when C is too large for one CTA's sort of its kept entries
 * in shared memory (8 C bytes plus 2 K KB within 200 KB: C up to about 21,000 at K = 16). */
int hils_select_backward(const hils_params *p, hils_ctensor Qcal, int Lq, hils_ctensor Ksum, int C,
                         const int32_t *idx, const int32_t *nsel, const float *dscore,
                         float *dQcal, float *dKsum, float *dBsum, cudaStream_t stream);

/* Eq. 8 backward for the C = floor(N / S) complete chunks: dLQ [B,H,C,d] (written),
 * dK [B,Hk,N,d] (accumulated) from dKsum [B,H,C,d] and dBsum [B,H,C]. */
int hils_summarize_backward(const hils_params *p, hils_ctensor K, int N, hils_ctensor LQ,
                            const float *dKsum, const float *dBsum, float *dK, float *dLQ, cudaStream_t stream);

/* Diagnostic (no counterpart on the pages): evaluates the two FMA-pipe helpers that the
 * tensor-core prefill attend uses instead of MUFU instructions, element by element:
 *   exp2_out[i]  = 2^x[i]  (a fitted degree-5 polynomial; relative error <= 2.4e-7 for
 *                  x in [-125, 127]; x below -125 gives 2^-125)
 *   recip_out[i] = 1/z[i]  (an integer seed and two Newton steps; relative error
 *                  <= 7e-6 for normal positive z)
 * x, z, exp2_out, recip_out: device arrays of n floats. Returns HILS_ERR_INVALID_ARG
 * for n < 0 or a null pointer with n > 0. */
int hils_selftest_fast_math(const float *x, const float *z, int n, float *exp2_out, float *recip_out,
                            cudaStream_t stream);

/* Bytes of workspace a call needs for these sizes (Lq = queries per (b, h); C =
 * summarised chunks). Returns 0 for invalid parameters. */
size_t hils_workspace_bytes(const hils_params *p, int call, int Lq, int C);

/* Zeroes a workspace on `stream` (cudaMemsetAsync); needed once after allocation. */
int hils_workspace_init(void *workspace, size_t ws_bytes, cudaStream_t stream);

/* Static description of a status code. */
const char *hils_status_string(int status);

/* CUDA error text of the calling thread's last HILS_ERR_CUDA ("" if none). */
const char *hils_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* HILS_H */
