/*
 * hsa.h -- C ABI of the B200 (sm_100a) Hierarchical Sparse Attention (HSA) library, libhsa_b200.so.
 *
 * The operation is the one described on the explainer page of "Every Token Counts: Generalizing 16M
 * Ultra-Long Context in Large Language Models", section "How It Works (Technically)":
 *   Step 1  the history is cut into chunks of 64 tokens; chunk c holds tokens 64c .. 64c+63 and
 *           owns one landmark vector L[c];
 *   Step 2  each query token t scores every chunk that has ended at or before t,
 *           s[t,c] = scale * Q[t].L[c], and keeps the top-K chunks I_t;
 *   Step 3  inside each selected chunk it runs ordinary softmax attention,
 *           O[t,c] = softmax(scale * Q[t] K_c^T) V_c, separately per chunk;
 *   Step 4  it blends the chunk outputs by the softmax of their retrieval scores,
 *           w = softmax(s[t, I_t]),  out[t] = sum_{c in I_t} w_c O[t,c].
 * and the per-token procedure of section "The algorithm, simplified" (stable sort of the scores in
 * descending order, first top_k kept).
 *
 * Readings of points the page leaves open, used by every entry point below:
 *   - causal rule: chunk c is admissible for token t iff 64c + 63 <= t, so a token sees
 *     n_t = (t + 1) / 64 chunks (the token that completes a chunk may retrieve it);
 *   - a token with n_t = 0 gets out = 0, sel_idx = -1, sel_w = 0 in every slot;
 *   - n_t < topk: all n_t chunks are selected and the fusion softmax runs over those only;
 *     the remaining slots hold sel_idx = -1, sel_w = 0;
 *   - ties: equal scores keep ascending chunk order (lower chunk index wins);
 *   - one query serves both as retrieval query and attention query; one scale serves both
 *     (scale <= 0 selects 1/sqrt(D)); no query-key normalisation and no positional encoding
 *     are applied (inputs are used as given). The *_ex entry points at the end add a separate
 *     retrieval query, query-key normalisation and grouped key/value heads;
 *   - selection itself carries no gradient; the landmarks receive gradient through the selected
 *     scores only (Step 4: w multiplies the output, so the loss reaches s).
 *
 * Conventions shared by all entry points:
 *   - Tensor arguments are DEVICE pointers owned by the caller, contiguous, row-major in the
 *     shapes given, 16-byte aligned. bf16 values are passed as raw 16-bit patterns (hsa_bf16).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy default
 *     stream). Validation is done on the host before any launch; an invalid call launches
 *     nothing and returns a negative status. No call synchronises the stream.
 *   - Scratch memory is caller-provided: query its size with the matching *_workspace_size
 *     function and pass at least that many bytes, 256-byte aligned. The library allocates no
 *     device memory. Workspace contents on entry are irrelevant; they are clobbered.
 *   - Every device-side wait of the kernels is bounded. A wait that runs out (a stalled pipeline:
 *     never expected, but possible on a faulty device) sets a status flag that lives in the first
 *     bytes of the call's workspace and lets the kernel unwind; the call itself has already
 *     returned (calls are asynchronous). hsa_workspace_status() reads that flag.
 *   - Supported now: D in {64, 128}, chunk == 64, 1 <= topk <= 64 (the per-token procedure's default is
 *     64; the "Build Your Own" recipe gives 16-64). Anything else returns HSA_ERR_UNSUPPORTED.
 *   - Every output element is written (including padding and all-zero rows).
 *   - Inputs must be finite; NaN/Inf inputs give unspecified results.
 *   - On any non-OK status, hsa_last_error() returns a message for the calling thread.
 */
#ifndef HSA_B200_H
#define HSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t hsa_bf16; /* raw bfloat16 bit pattern */

typedef enum {
    HSA_OK = 0,
    HSA_ERR_INVALID_ARG = -1, /* null pointer, bad size, misalignment */
    HSA_ERR_UNSUPPORTED = -2, /* valid HSA call outside what the kernels implement (D, chunk, topk) */
    HSA_ERR_WORKSPACE = -3,   /* workspace missing, misaligned or smaller than *_workspace_size */
    HSA_ERR_CUDA = -4,        /* a CUDA runtime call failed; hsa_last_error() holds its text */
    HSA_ERR_TIMEOUT = -5      /* a bounded device-side wait ran out (see hsa_workspace_status) */
} hsa_status;

/* Message describing the last non-OK status returned on the calling thread ("" if none). */
const char *hsa_last_error(void);

/* Device-side status of the last hsa_forward / hsa_backward / hsa_decode call that used `workspace`
 * (the pointer passed to that call). Synchronizes `stream` (cudaStream_t, NULL = legacy default
 * stream), then reads the flag stored in the first 4 bytes of the workspace.
 * Returns HSA_OK, HSA_ERR_TIMEOUT if a bounded device wait of that call ran out (its outputs are
 * then unspecified), HSA_ERR_INVALID_ARG for a NULL workspace, or HSA_ERR_CUDA. */
hsa_status hsa_workspace_status(const void *workspace, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Prefill forward (Steps 1-4 for every token of a sequence).
 *
 *   Q, K, V  [B, H, T, D] bf16      queries, keys, values
 *   L        [B, H, T/64, D] bf16   one landmark per complete chunk (a trailing partial chunk has
 *                                   no landmark and is never selected)
 *   out      [B, H, T, D] bf16      required; rounded to nearest-even from fp32
 *   sel_idx  [B, H, T, topk] int32  optional (NULL): selected chunk ids, by score descending then
 *                                   chunk ascending; -1 padding
 *   sel_w    [B, H, T, topk] fp32   optional (NULL): fusion weights in the same order; 0 padding
 * Scores and softmaxes are computed in fp32 from bf16 inputs. Requires 1 <= T, B*H*T*topk < 2^31.
 * ------------------------------------------------------------------------------------------- */
size_t hsa_forward_workspace_size(int B, int H, int T, int D, int chunk, int topk);

hsa_status hsa_forward(const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V, const hsa_bf16 *L, int B, int H,
                       int T, int D, int chunk, int topk, float scale, hsa_bf16 *out, int32_t *sel_idx,
                       float *sel_w, void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Decode: one new query token per sequence against a cached history (Steps 2-4 with the query
 * at the last cached position, so it sees n = cache_len[b] / 64 complete chunks).
 *
 *   q          [B, H, D] bf16
 *   Kc, Vc     [B, H, Tmax, D] bf16     key / value cache
 *   Lc         [B, H, Tmax/64, D] bf16  landmark cache
 *   cache_len  [B] int64, DEVICE        tokens held by each sequence, 0 <= cache_len[b] <= Tmax
 *   out        [B, H, D] bf16           required
 *   sel_idx    [B, H, topk] int32       optional; sel_w [B, H, topk] fp32 optional
 * The landmark scan is split over chunk ranges (split-over-chunks); each range keeps its exact
 * top-K and the ranges are merged exactly, so the result equals a single global top-K.
 * ------------------------------------------------------------------------------------------- */
size_t hsa_decode_workspace_size(int B, int H, int64_t Tmax, int D, int chunk, int topk);

hsa_status hsa_decode(const hsa_bf16 *q, const hsa_bf16 *Kc, const hsa_bf16 *Vc, const hsa_bf16 *Lc,
                      const int64_t *cache_len, int64_t Tmax, int B, int H, int D, int chunk, int topk,
                      float scale, hsa_bf16 *out, int32_t *sel_idx, float *sel_w, void *workspace,
                      size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Decode without any allocation. The pages have no counterpart: this is an interface addition.
 *
 * Same operation, arguments and results as hsa_decode, minus the workspace. It is for callers that
 * cannot allocate device memory when they run a decode step: an engine that has given all of HBM
 * to its KV-cache pool and allows no allocation while serving, a plain C caller without a caching
 * allocator for whom cudaMalloc / cudaFree per step would synchronise the device, or a thread that
 * must not take the driver's allocation locks. The call allocates nothing (no cudaMalloc, no
 * cudaFree, no allocating library routine). Its scratch lives in one fixed device array of
 * HSA_DECODE_NOALLOC_SCRATCH_BYTES inside the library; every GPU that loads the library holds that
 * array until the process exits.
 *   - The first call on a device looks up the array's device address (with that device current)
 *     and caches it; make that first call before any stream capture on that device.
 *   - A call whose scratch would exceed the array (it grows with B*H*topk*(D + scan ranges)) is
 *     rejected on the host with HSA_ERR_UNSUPPORTED and a message; use hsa_decode then.
 *   - Every call shares the one array, which keeps the last call's contents; the parts that must
 *     start at zero are cleared by each call on its stream. Calls that overlap on the GPU (issued on
 *     streams not ordered with each other, or from several threads at once) race on the array and
 *     give wrong results: order them, e.g. on a single stream.
 * ------------------------------------------------------------------------------------------- */
#define HSA_DECODE_NOALLOC_SCRATCH_BYTES (4u * 1024u * 1024u)

hsa_status hsa_decode_noalloc(const hsa_bf16 *q, const hsa_bf16 *Kc, const hsa_bf16 *Vc, const hsa_bf16 *Lc,
                              const int64_t *cache_len, int64_t Tmax, int B, int H, int D, int chunk, int topk,
                              float scale, hsa_bf16 *out, int32_t *sel_idx, float *sel_w, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Backward of hsa_forward for the selection the forward made.
 *
 *   Q, K, V, L, out as in hsa_forward (out = the forward's output); dout [B, H, T, D] bf16
 *   sel_idx [B, H, T, topk] int32, sel_w [B, H, T, topk] fp32: the forward's selection (required)
 *   dQ, dK, dV [B, H, T, D] fp32, dL [B, H, T/64, D] fp32: overwritten (zeroed by the call)
 * Chain rule through Step 3 (per-chunk softmax) and Step 4 (fusion softmax over the selected
 * scores); the discrete selection is treated as constant.
 * ------------------------------------------------------------------------------------------- */
size_t hsa_backward_workspace_size(int B, int H, int T, int D, int chunk, int topk);

hsa_status hsa_backward(const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V, const hsa_bf16 *L,
                        const hsa_bf16 *out, const hsa_bf16 *dout, const int32_t *sel_idx, const float *sel_w,
                        int B, int H, int T, int D, int chunk, int topk, float scale, float *dQ, float *dK,
                        float *dV, float *dL, void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Extended entry points: a separate retrieval query, query-key normalisation, grouped key heads.
 *
 * Same operation, shapes, layouts, ownership, workspace rules, error behaviour and outputs as the
 * calls above, with three additions. Each is off when its argument takes the value shown in brackets,
 * and then the result is that of the plain call.
 *
 *   Qs / qs [NULL]   separate retrieval query, shaped like Q / q. Explainer of "Every Token Counts",
 *                    "How It Works (Technically)" Steps 2-3 and the per-token procedure in "The
 *                    algorithm, simplified": the query that scores the landmarks (q_slc) and the query
 *                    that attends inside the selected chunks (q_attn) are separate projections. Qs gives
 *                    the Step 2 scores, the top-K and the Step 4 fusion weights; Q attends in Step 3.
 *   flags & HSA_QK_NORM [0]   query-key normalisation (Step 3: the in-chunk logits are
 *                    norm(q_attn) . norm(K_c)^T * scale, norm = L2 normalisation, as in the
 *                    procedure's l2norm calls). Reading: norm(x) = x / max(||x||_2, 1e-6) per row; the
 *                    retrieval scores (Step 2) are not normalised. The prefill forward and backward
 *                    normalise Q and K into bf16 copies in the workspace; the decode normalises in fp32
 *                    on the fly.
 *   Hkv [H]          grouped heads ("How to Improve It" #2: several query heads per key/value head):
 *                    K, V, L (Kc, Vc, Lc) have Hkv heads, H a multiple of Hkv, and query head h uses
 *                    head h / (H / Hkv). Each query head still selects its own chunks.
 *                    Shapes: K, V [B, Hkv, T, D], L [B, Hkv, T/64, D]; dK, dV, dL likewise.
 *   Tq [1] (decode)  several query tokens per sequence and head in one decode step (verifying drafted
 *                    tokens, or decoding a few tokens at once): q, qs, out [B, H, Tq, D], sel_idx and
 *                    sel_w [B, H, Tq, topk], 1 <= Tq <= 64. The Tq tokens are the LAST Tq tokens of the
 *                    cache (their K, V and any completed landmark already in it): token i sits at
 *                    position cache_len[b] - Tq + i and sees the chunks that have ended at or before it,
 *                    the prefill's causal rule (so the result equals the forward's last Tq rows).
 *                    Tq > 1 requires topk <= 32. Every query row is scored on the tensor cores together
 *                    with the other rows that share its key head (up to 16 per pass over the landmarks).
 *
 * Unknown flag bits give HSA_ERR_INVALID_ARG. hsa_backward_ex writes dQ (the attention query's
 * gradient, taken back through the normalisation when it is on) and, when Qs is given, dQs (the
 * retrieval query's gradient) -- both fp32 [B, H, T, D] and overwritten; without Qs, dQ holds both
 * parts and dQs must be NULL. The *_ex_workspace_size functions take the same Hkv and flags.
 * -------------------------------------------------------------------------------------------*/
#define HSA_QK_NORM 1u

size_t hsa_forward_ex_workspace_size(int B, int H, int Hkv, int T, int D, int chunk, int topk, unsigned flags);

hsa_status hsa_forward_ex(const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V,
                          const hsa_bf16 *L, int B, int H, int Hkv, int T, int D, int chunk, int topk, float scale,
                          unsigned flags, hsa_bf16 *out, int32_t *sel_idx, float *sel_w, void *workspace,
                          size_t workspace_bytes, void *stream);

size_t hsa_decode_ex_workspace_size(int B, int H, int Hkv, int Tq, int64_t Tmax, int D, int chunk, int topk,
                                    unsigned flags);

hsa_status hsa_decode_ex(const hsa_bf16 *qs, const hsa_bf16 *q, const hsa_bf16 *Kc, const hsa_bf16 *Vc,
                         const hsa_bf16 *Lc, const int64_t *cache_len, int64_t Tmax, int B, int H, int Hkv, int Tq,
                         int D, int chunk, int topk, float scale, unsigned flags, hsa_bf16 *out, int32_t *sel_idx,
                         float *sel_w, void *workspace, size_t workspace_bytes, void *stream);

size_t hsa_backward_ex_workspace_size(int B, int H, int Hkv, int T, int D, int chunk, int topk, unsigned flags);

hsa_status hsa_backward_ex(const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V,
                           const hsa_bf16 *L, const hsa_bf16 *out, const hsa_bf16 *dout, const int32_t *sel_idx,
                           const float *sel_w, int B, int H, int Hkv, int T, int D, int chunk, int topk, float scale,
                           unsigned flags, float *dQ, float *dK, float *dV, float *dL, float *dQs, void *workspace,
                           size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Variable-length batches in the packed, token-major layout (no counterpart on the pages: the
 * layout model code holds between layers). Same operation, options, rules and errors as the *_ex
 * calls, per sequence:
 *   cu_seqlens  [B + 1] int32, DEVICE: sequence b holds tokens cu_seqlens[b] .. cu_seqlens[b+1] - 1
 *               (cu_seqlens[0] = 0, non-decreasing, every length <= max_seqlen; not checked)
 *   Q, Qs, out, dout [total, H, D] bf16;  K, V [total, Hkv, D] bf16  (total = cu_seqlens[B])
 *   L           [total_chunks, Hkv, D] bf16: sequence b's floor(len_b / 64) landmarks one after another,
 *               in sequence order (total_chunks = the sum of those counts)
 *   sel_idx, sel_w [total, H, topk]: chunk ids within the token's own sequence (0 .. len_b/64 - 1)
 *   dQ, dQs [total, H, D], dK, dV [total, Hkv, D], dL [total_chunks, Hkv, D] fp32 (overwritten)
 * A fixed-length batch in [B, T, H, D] layout is the case cu_seqlens[b] = b * T.
 * The library moves the rows to a head-major batch padded to max_seqlen in the workspace (streaming
 * copies), runs the batched kernels with each sequence's length (padded rows select nothing and cost no
 * attention work) and moves the results back. The *_varlen_workspace_size functions size the
 * workspace for max_seqlen, with room for a separate retrieval query.
 * ------------------------------------------------------------------------------------------- */
size_t hsa_forward_varlen_workspace_size(int B, int H, int Hkv, int max_seqlen, int D, int chunk, int topk,
                                         unsigned flags);

hsa_status hsa_forward_varlen(const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V,
                              const hsa_bf16 *L, const int32_t *cu_seqlens, int B, int max_seqlen, int H, int Hkv,
                              int D, int chunk, int topk, float scale, unsigned flags, hsa_bf16 *out,
                              int32_t *sel_idx, float *sel_w, void *workspace, size_t workspace_bytes, void *stream);

size_t hsa_backward_varlen_workspace_size(int B, int H, int Hkv, int max_seqlen, int D, int chunk, int topk,
                                          unsigned flags);

hsa_status hsa_backward_varlen(const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V,
                               const hsa_bf16 *L, const hsa_bf16 *out, const hsa_bf16 *dout, const int32_t *sel_idx,
                               const float *sel_w, const int32_t *cu_seqlens, int B, int max_seqlen, int H, int Hkv,
                               int D, int chunk, int topk, float scale, unsigned flags, float *dQ, float *dK, float *dV,
                               float *dL, float *dQs, void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Self-test of the bounded device waits (no counterpart on the pages; failure detection).
 *
 * Every kernel waits on mbarriers with a bounded number of probes; a wait that runs out records the
 * failure in the status flag of the call's workspace, lets the kernel unwind (its copies finish, its
 * TMEM is freed) and returns, so hsa_workspace_status() reports HSA_ERR_TIMEOUT instead of the device
 * hanging. In a healthy run no wait runs out, so this call makes one run out on purpose: it clears the
 * flag at the start of `workspace` (>= 256 bytes, 256-byte aligned, device memory), then launches one
 * warp on `stream` that allocates TMEM, waits with the kernels' own helper -- but at most `probes`
 * probes, 1 <= probes <= 2^20 -- on an mbarrier whose only expected arrival is never made, records the
 * timeout as the kernels do, frees its TMEM and exits. Nothing faults; the context stays usable; the next
 * operator call on the same workspace clears the flag again. Returns HSA_ERR_WORKSPACE or
 * HSA_ERR_INVALID_ARG (host checks, nothing launched) or HSA_ERR_CUDA.
 * ------------------------------------------------------------------------------------------- */
hsa_status hsa_selftest_bounded_wait(void *workspace, size_t workspace_bytes, unsigned probes, void *stream);

/* ---------------------------------------------------------------------------------------------
 * Measurement hooks (no counterpart on the pages; used to time each kernel live).
 *
 * hsa_profile_enable(1) starts recording a pair of CUDA events around every kernel launch and
 * memset the library issues, on the stream it is issued on (0 stops recording); either call
 * discards earlier records. hsa_profile_summary() waits for the recorded events and writes one line
 * per launch site, "name,launches,total_ms\n", into buf (truncated to cap - 1 bytes, NUL-terminated);
 * it returns the full text length, or -1 if an event query failed. Host-side only; thread-safe.
 * ------------------------------------------------------------------------------------------- */
int hsa_profile_enable(int on);
int hsa_profile_summary(char *buf, size_t cap);

#ifdef __cplusplus
}
#endif

#endif /* HSA_B200_H */
