// launch.h -- internal interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include <cuda.h>

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace hsa {

struct DecodeArgs {
    const uint16_t *qs;  // retrieval query (scan); q attends
    const uint16_t *q, *Kc, *Vc, *Lc;
    const int64_t *cache_len;
    int64_t Tmax, Nmax;
    int B, H, D, K;
    int Hkv;           // key/value/landmark heads (H a multiple; query head h reads h / (H / Hkv))
    int Tq;            // query tokens per sequence and head (q, out: [B, H, Tq, D]); 0 means 1
    float scale;
    uint16_t *out;
    int32_t *sel_idx;  // [B*H*Tq, K] (caller's or workspace)
    float *sel_w;      // [B*H*Tq, K]
    uint64_t *cand;    // [B*H*Tq, nsplit, K]
    unsigned *counters;  // [2, B*H*Tq]
    float *partial;    // [B*H*Tq, K, D]
    bool qk_norm;      // Step 3 attends with q / max(|q|, eps) and k / max(|k|, eps)
    int32_t *err;      // [1] or NULL: set when a bounded device wait ran out (grouped scan)
};
int decode_split_size(int64_t Nmax, int K, int BH);
size_t decode_scan_smem(int split, int nsplit, int K);
// How a decode call splits the landmark scan: ranges of `split` landmarks, `nsplit` of them; grouped:
// one CTA per (range, key head) scores all query heads of the group and a merge kernel follows.
struct DecodePlan {
    int split, nsplit;
    int row_groups;  // grouped: CTAs per (range, key head), 16 query rows each
    bool grouped;
};
DecodePlan decode_plan(int64_t Nmax, int K, int B, int H, int Hkv, int Tq);
size_t decode_plan_smem(const DecodePlan &p, int K);  // the largest dynamic shared memory of its kernels
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);

// Chunk-major work list entry: one tile (forward: <= 128 pairs) or work unit (backward: <= kBwdUnitPairs)
// of (token, slot) pairs of one chunk.
struct PairTile {
    int32_t chunk;  // flat (b*H + h) * N + c
    int32_t start;  // first pair (offset into the pair arrays)
    int32_t count;  // pairs in this tile
    int32_t pad;
};
// The work list is sized for tiles of at least kPairTile pairs (every chunk adds one partial tile), which
// covers both the forward's tiles and the backward's units.
constexpr int kPairTile = 64;

struct ForwardArgs {
    const uint16_t *Qs;  // retrieval queries (scores, fusion weights); Q attends
    const uint16_t *Q, *K, *V, *L;
    int B, H, T, D, N, topk;
    int Hkv;  // key/value/landmark heads: K, V [B, Hkv, T, D], L [B, Hkv, N, D]
    // optional: sequences padded to T; sequence b has cu_seqlens[b+1] - cu_seqlens[b] valid tokens, and
    // the rows past them select nothing (output 0, selection -1 / 0)
    const int32_t *cu_seqlens;
    float scale;
    uint16_t *out;
    int32_t *sel_idx;  // [B*H*T, topk] (caller's or workspace)
    float *sel_w;
    // workspace
    float *o_acc;          // [B*H*T, D] fp32 accumulator
    // chunk ids are flat over the QUERY heads, (b*H + h) * N + c; a kernel that reads K, V or L for a
    // chunk id uses key head (chunk id / N) / (H / Hkv)
    int32_t *chunk_count;  // [B*H*N]
    int32_t *chunk_off;    // [B*H*N + 1]
    int32_t *tile_off;     // [B*H*N + 1]
    int32_t *chunk_cursor; // [B*H*N]
    int32_t *pair_row;     // [B*H*T*topk] flat token row (b*H + h)*T + t
    float *pair_w;         // [B*H*T*topk]
    PairTile *tiles;       // [max_tiles]
    int32_t *num_tiles;    // [1]
    int32_t *err;          // [1] set when a bounded device wait ran out
    int max_tiles;
    // query-key normalisation: Q and K are normalised into these bf16 workspace copies first
    bool qk_norm;
    uint16_t *Qn, *Kn;     // [B*H*T, D] and [B*Hkv*T, D]
};
size_t forward_max_tiles(int B, int H, int T, int topk);
// Step 2 scores + top-K + fusion weights on the tcgen05 tensor cores (score_tc.cu).
cudaError_t launch_score_tc(const ForwardArgs &a, cudaStream_t s);
// K <= 16: the persistent scoring kernel (score_wide.cu); cudaErrorInvalidValue for larger K.
cudaError_t launch_score_wide(const ForwardArgs &a, cudaStream_t s);
// Step 3 + blend on the tcgen05 tensor cores (attn_tc.cu); tiles of up to 128 pairs.
cudaError_t launch_attn_tc(const ForwardArgs &a, cudaStream_t s);
cudaError_t launch_forward(const ForwardArgs &a, cudaStream_t s);
// Chunk-major dispatch shared by the forward and the backward: per-chunk pair counts, offsets, the
// tile work list, and the (token row, weight[, slot]) pair arrays. The lists are per query head even
// when query heads share key heads: a tile's pairs then all write accumulator rows of one query head,
// which keeps the rows that the concurrent tiles reduce into within L2.
// Zeroes the error flag and the dispatch's chunk counts and cursors: one memset when the workspace
// holds them in that order with at most alignment padding between them, else three.
cudaError_t zero_dispatch_state(int32_t *err, int32_t *chunk_count, int32_t *chunk_cursor, size_t chunks,
                                cudaStream_t s);

// Launches kern as a programmatic dependent of the previous kernel in stream s (kern must call
// pdl_wait() first; see common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

cudaError_t launch_dispatch(const int32_t *sel_idx, const float *sel_w, int B, int H, int T, int N, int topk,
                            int32_t *chunk_count, int32_t *chunk_off, int32_t *tile_off, int32_t *chunk_cursor,
                            int32_t *pair_row,
                            float *pair_w, int32_t *pair_slot, PairTile *tiles, int32_t *num_tiles, int max_tiles,
                            int tile_pairs, bool counts_ready, cudaStream_t s, const int32_t *cu_seqlens = nullptr);

struct BackwardArgs {
    const uint16_t *Qs;  // separate retrieval queries, or NULL when Q retrieves too
    float *dQs;          // their gradient (the ds L_c terms), with Qs
    float *ds_pair;      // [B*H*T, topk] workspace: ds per (token, slot), with Qs
    const uint16_t *Q, *K, *V, *L, *out, *dout;
    const int32_t *sel_idx;
    const float *sel_w;
    int B, H, T, D, N, topk;
    int Hkv;  // key/value/landmark heads: K, V, dK, dV [B, Hkv, T, D], L, dL [B, Hkv, N, D]
    float scale;
    float *dQ, *dK, *dV, *dL;
    // workspace (shares the dispatch layout of the forward)
    float *delta;          // [B*H*T]  dO . O
    int32_t *chunk_count, *chunk_off, *tile_off, *chunk_cursor, *pair_row;
    float *pair_w;
    int32_t *pair_slot;    // [B*H*T*topk] slot j of each pair (unused by the forward)
    PairTile *tiles;
    int32_t *num_tiles;
    int32_t *err;          // [1] set when a bounded device wait ran out
    int max_tiles;
    // query-key normalisation: Q and K are normalised into these bf16 workspace copies, the kernels
    // run on them (with the raw Q as retrieval query when there is no Qs), and dQ / dK go back
    // through the normalisation at the end
    bool qk_norm;
    uint16_t *Qn, *Kn;     // [B*H*T, D] and [B*Hkv*T, D]
};
cudaError_t launch_backward(const BackwardArgs &a, cudaStream_t s);
// Gradients on the tcgen05 tensor cores (bwd_tc.cu), head dims 64 and 128; work units of up to 1024 pairs.
constexpr int kBwdUnitPairs = 1024;
cudaError_t launch_backward_tc(const BackwardArgs &a, cudaStream_t s);

// 2-D bf16 tensor map over a [rows, D] row-major tensor: boxes of 64 columns x box_rows rows,
// 128-byte swizzle (attn_tc.cu). False if the driver entry point is missing or the encoding fails.
bool make_tmap_bf16(CUtensorMap *m, const void *base, uint64_t rows, int D, int box_rows);

// Query-key normalisation (qknorm.cu), y = x / max(|x|_2, 1e-6) per row of D elements.
// Rows X0 -> Y0 and X1 -> Y1 in one launch (bf16 in, bf16 out, round to nearest even).
cudaError_t launch_l2norm_rows(const uint16_t *X0, uint16_t *Y0, size_t R0, const uint16_t *X1, uint16_t *Y1,
                               size_t R1, int D, cudaStream_t s);
// In place, per row: dX <- dX taken back through that normalisation of X (fp32 gradients).
cudaError_t launch_l2norm_grad_rows(const uint16_t *X, float *dX, size_t rows, int D, cudaStream_t s);
constexpr float kQkNormEps = 1e-6f;

// Variable-length batches (varlen.cu). cuN[b] = the packed landmark row of sequence b's first chunk.
cudaError_t launch_chunk_offsets(const int32_t *cu, int B, int32_t *cuN, cudaStream_t s);
// Rows between the packed token-major layout [total, Hs, row] (sequence b at rows cu[b] ..) and the
// head-major batch [B, Hs, Tp, row]; with fill_pad, pack fills the batch rows past a sequence's end
// with `fill` (the rows no kernel reads are left alone otherwise).
cudaError_t launch_varlen_rows(const void *src, void *dst, const int32_t *cu, int B, int Hs, int Tp, int row_bytes,
                               bool pack, bool fill_pad, uint32_t fill, cudaStream_t s);

// Message returned by hsa_last_error() on the calling thread.
void set_last_error(const char *msg);

}  // namespace hsa
