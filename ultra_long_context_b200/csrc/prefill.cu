// prefill.cu -- HSA forward for every token of a sequence (prefill).
//
// Explainer page of "Every Token Counts", "How It Works (Technically)", Steps 2-4. HSA is built
// like a mixture of experts whose experts are chunks of the history ("How It Works", opening
// paragraphs), and the kernels follow that shape:
//
//   score_topk (score_tc.cu)  Step 2: S = scale * Q L^T on the tensor cores, causal over completed
//                       chunks, per-token top-K (score descending, ties to the lower chunk) and the
//                       fusion softmax (Step 4 weights). Scores never reach HBM.
//   count / scan /      "Router" bookkeeping (this file): histogram of selected chunks, exclusive
//   tiles / scatter     scan, tile list, and a scatter of (token, weight) pairs into chunk-major
//                       lists cut into tiles of up to 128 pairs (64 for the backward).
//   chunk_attn (attn_tc.cu)  Step 3 + Step 4 blend: per tile, S = Q K_c^T on the tensor cores,
//                       exact softmax over the chunk's 64 keys, O = P V_c, scaled by the pair's
//                       fusion weight and added into an fp32 accumulator row of the token.
//   finalize_kernel     fp32 accumulator -> bf16 output (round to nearest even).
#include "common.cuh"
#include "launch.h"
#include "profile.h"

namespace hsa {

// ------------------------------------------------------------------------------------------------
// Dispatch: chunk-major pair lists
// ------------------------------------------------------------------------------------------------
constexpr int kDispatchRows = 256;
constexpr int kSmemHistMax = 8192;  // chunks per (b, h) histogrammed in shared memory

__global__ void __launch_bounds__(kDispatchRows) count_kernel(const int32_t *__restrict__ sel_idx, int T, int N,
                                                              int K, int32_t *__restrict__ chunk_count) {
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ int s_hist[];
    const int bh = blockIdx.y;
    const bool use_smem = N <= kSmemHistMax;
    if (use_smem) {
        for (int i = threadIdx.x; i < N; i += blockDim.x) s_hist[i] = 0;
        __syncthreads();
    }
    // the block's rows are contiguous in [B, H, T, K]: one flat, coalesced range of entries
    const int t0 = blockIdx.x * kDispatchRows;
    const int nent = max(0, min(kDispatchRows, T - t0)) * K;
    const int32_t *si = sel_idx + ((size_t)bh * T + t0) * K;
    for (int eb = 0; eb < nent; eb += 8 * kDispatchRows) {  // 8 loads in flight per thread
        int cb[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int e = eb + k * kDispatchRows + threadIdx.x;
            cb[k] = e < nent ? si[e] : -1;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int c = cb[k];
            if (c < 0 || c >= N) continue;  // -1 = empty slot (or past the block's rows); ids past N are ignored
            if (use_smem) atomicAdd(&s_hist[c], 1);
            else atomicAdd(&chunk_count[(size_t)bh * N + c], 1);
        }
    }
    if (use_smem) {
        __syncthreads();
        for (int i = threadIdx.x; i < N; i += blockDim.x)
            if (s_hist[i]) atomicAdd(&chunk_count[(size_t)bh * N + i], s_hist[i]);
    }
}

// Block-wide exclusive scan helper (1024 threads): returns the exclusive prefix of v and the total.
__device__ inline int block_exclusive_scan(int v, int *s_warp, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarp ? s_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += x;
        }
        if (lane < nwarp) s_warp[lane] = wi - w;
        if (lane == 31) s_warp[32] = wi;
    }
    __syncthreads();
    const int res = s_warp[warp] + incl - v;
    total = s_warp[32];
    __syncthreads();
    return res;
}

// One CTA: exclusive offsets of every chunk's pair list and of its tiles (<= tp pairs each). Rounds
// of 8192 counts, 8 contiguous ones per thread loaded and stored as vectors where they are whole (the
// tables are 256-byte aligned), each round's block scan carried into the next.
constexpr int kScanPer = 8;

__global__ void __launch_bounds__(1024) scan_kernel(const int32_t *__restrict__ chunk_count, int M,
                                                    int32_t *__restrict__ chunk_off, int32_t *__restrict__ tile_off,
                                                    int32_t *__restrict__ num_tiles, int max_tiles, int tp) {
    pdl_launch_dependents();
    pdl_wait();
    __shared__ int s_warp[33];
    int carry = 0, tcarry = 0;
    for (int base = 0; base < M; base += (int)blockDim.x * kScanPer) {
        const int lo = base + (int)threadIdx.x * kScanPer;
        int c[kScanPer];
        if (lo + kScanPer <= M) {  // lo is a multiple of 8 ints: 32-byte aligned in the 256-aligned table
            const int4 a = reinterpret_cast<const int4 *>(chunk_count + lo)[0];
            const int4 b = reinterpret_cast<const int4 *>(chunk_count + lo)[1];
            c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w;
            c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
        } else {
#pragma unroll
            for (int k = 0; k < kScanPer; ++k) c[k] = lo + k < M ? chunk_count[lo + k] : 0;
        }
        int sum = 0, tsum = 0;
#pragma unroll
        for (int k = 0; k < kScanPer; ++k) {
            sum += c[k];
            tsum += (c[k] + tp - 1) / tp;
        }
        int total, ttotal;
        int off = block_exclusive_scan(sum, s_warp, total) + carry;
        int toff = block_exclusive_scan(tsum, s_warp, ttotal) + tcarry;
        int o[kScanPer], to[kScanPer];
#pragma unroll
        for (int k = 0; k < kScanPer; ++k) {
            o[k] = off;
            to[k] = toff;
            off += c[k];
            toff += (c[k] + tp - 1) / tp;
        }
        if (lo + kScanPer <= M) {
            reinterpret_cast<int4 *>(chunk_off + lo)[0] = make_int4(o[0], o[1], o[2], o[3]);
            reinterpret_cast<int4 *>(chunk_off + lo)[1] = make_int4(o[4], o[5], o[6], o[7]);
            reinterpret_cast<int4 *>(tile_off + lo)[0] = make_int4(to[0], to[1], to[2], to[3]);
            reinterpret_cast<int4 *>(tile_off + lo)[1] = make_int4(to[4], to[5], to[6], to[7]);
        } else {
#pragma unroll
            for (int k = 0; k < kScanPer; ++k)
                if (lo + k < M) {
                    chunk_off[lo + k] = o[k];
                    tile_off[lo + k] = to[k];
                }
        }
        carry += total;
        tcarry += ttotal;
    }
    if (threadIdx.x == 0) {
        chunk_off[M] = carry;
        tile_off[M] = tcarry;
        num_tiles[0] = min(tcarry, max_tiles);
    }
}

// One warp per chunk writes that chunk's tiles into the work list.
__global__ void __launch_bounds__(256) tile_list_kernel(const int32_t *__restrict__ chunk_count,
                                                        const int32_t *__restrict__ chunk_off,
                                                        const int32_t *__restrict__ tile_off, int M,
                                                        PairTile *__restrict__ tiles, int max_tiles, int tp) {
    pdl_launch_dependents();
    pdl_wait();
    const int i = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (i >= M) return;
    const int n = chunk_count[i], base = tile_off[i], off = chunk_off[i];
    for (int k = lane; k * tp < n; k += 32) {
        if (base + k >= max_tiles) break;
        PairTile pt;
        pt.chunk = i;
        pt.start = off + k * tp;
        pt.count = min(tp, n - k * tp);
        pt.pad = 0;
        tiles[base + k] = pt;
    }
}

__global__ void __launch_bounds__(kDispatchRows) scatter_kernel(const int32_t *__restrict__ sel_idx,
                                                                const float *__restrict__ sel_w, int T, int N, int K,
                                                                const int32_t *__restrict__ chunk_off,
                                                                int32_t *__restrict__ chunk_cursor,
                                                                int32_t *__restrict__ pair_row,
                                                                float *__restrict__ pair_w,
                                                                int32_t *__restrict__ pair_slot,
                                                                const int32_t *__restrict__ cu_seqlens, int H) {
    // no early release of the dependent: the persistent attention kernel would take SMs from this one
    pdl_wait();
    extern __shared__ int s_mem[];
    const int bh = blockIdx.y;
    const int Tv = cu_seqlens ? min(T, cu_seqlens[bh / H + 1] - cu_seqlens[bh / H]) : T;
    if ((int)(blockIdx.x * kDispatchRows) >= Tv) return;
    const bool use_smem = N <= kSmemHistMax / 2;
    int *s_cnt = s_mem, *s_base = s_mem + (use_smem ? N : 0);
    const int t = blockIdx.x * kDispatchRows + threadIdx.x;
    const int32_t *si = sel_idx + ((size_t)bh * T + (t < T ? t : 0)) * K;
    if (use_smem) {
        for (int i = threadIdx.x; i < N; i += blockDim.x) s_cnt[i] = 0;
        __syncthreads();
        if (t < Tv)
            for (int j = 0; j < K; ++j)
                if (si[j] >= 0 && si[j] < N) atomicAdd(&s_cnt[si[j]], 1);
        __syncthreads();
        for (int i = threadIdx.x; i < N; i += blockDim.x) {
            const int c = s_cnt[i];
            s_base[i] = c ? atomicAdd(&chunk_cursor[(size_t)bh * N + i], c) : 0;
            s_cnt[i] = 0;
        }
        __syncthreads();
    }
    if (t >= Tv) return;
    const size_t row = (size_t)bh * T + t;
    for (int j = 0; j < K; ++j) {
        const int c = si[j];
        if (c < 0 || c >= N) continue;
        const size_t ch = (size_t)bh * N + c;
        const int local = use_smem ? s_base[c] + atomicAdd(&s_cnt[c], 1) : atomicAdd(&chunk_cursor[ch], 1);
        const int pos = chunk_off[ch] + local;
        pair_row[pos] = (int32_t)row;
        pair_w[pos] = sel_w[row * K + j];
        if (pair_slot) pair_slot[pos] = j;
    }
}

// Scatter as a block-level counting sort: the block's (token, slot) entries are ranked by chunk in
// shared memory first, so each chunk's run of entries from this block is written to consecutive
// pair-list positions (coalesced stores instead of one scattered store per entry). The block's entries
// are contiguous in [B, H, T, K]: they are read as one flat, coalesced range, with a batch of loads
// in flight per thread (a load per iteration would leave every thread waiting on memory latency),
// and the shared-memory atomic that counts an entry also returns its rank within its chunk, so one
// pass both counts and ranks. Used when the chunk count per (b, h) fits the shared-memory tables
// (N <= kSortedScatterMaxN).
constexpr int kSortedScatterMaxN = 2048;
constexpr int kRankBits = 14;  // rank of an entry within its chunk (< kDispatchRows * 64 entries per block)
constexpr int kScatterBatch = 8;  // entries per thread whose loads are in flight together

__global__ void __launch_bounds__(kDispatchRows) scatter_sorted_kernel(
    const int32_t *__restrict__ sel_idx, const float *__restrict__ sel_w, int T, int N, int K,
    const int32_t *__restrict__ chunk_off, int32_t *__restrict__ chunk_cursor, int32_t *__restrict__ pair_row,
    float *__restrict__ pair_w, int32_t *__restrict__ pair_slot, const int32_t *__restrict__ cu_seqlens, int H) {
    // no early release of the dependent: the persistent attention kernel would take SMs from this one
    pdl_wait();
    extern __shared__ int s_mem[];
    const int nent_max = kDispatchRows * K;
    int *s_cnt = s_mem;                  // [N] entries per chunk in this block
    int *s_scan = s_cnt + N;             // [N] exclusive scan of s_cnt
    int *s_gbase = s_scan + N;           // [N] global position of this block's run for the chunk
    int *s_tmp = s_gbase + N;            // [rows * K] (c << kRankBits) | rank, in entry order; -1: empty slot
    int *s_key = s_tmp + nent_max;       // [rows * K] (c << kRankBits) | entry, sorted by chunk
    float *s_wt = reinterpret_cast<float *>(s_key + nent_max);
    __shared__ int s_warp[33];
    const int bh = blockIdx.y, tid = threadIdx.x;
    const int t0 = blockIdx.x * kDispatchRows;
    const int Tv = cu_seqlens ? min(T, cu_seqlens[bh / H + 1] - cu_seqlens[bh / H]) : T;  // rows past it: none
    if (t0 >= Tv) return;
    const int nent = min(kDispatchRows, Tv - t0) * K;
    const size_t e0 = ((size_t)bh * T + t0) * K;  // the block's first entry in [B, H, T, K]
    for (int i = tid; i < N; i += blockDim.x) s_cnt[i] = 0;
    __syncthreads();
    // count and rank; kScatterBatch loads in flight per thread before their atomics
    for (int eb = 0; eb < nent; eb += kScatterBatch * kDispatchRows) {
        int cb[kScatterBatch];
#pragma unroll
        for (int k = 0; k < kScatterBatch; ++k) {
            const int e = eb + k * kDispatchRows + tid;
            cb[k] = e < nent ? sel_idx[e0 + e] : -1;
        }
#pragma unroll
        for (int k = 0; k < kScatterBatch; ++k) {
            const int e = eb + k * kDispatchRows + tid, c = cb[k];
            if (e < nent) s_tmp[e] = (c >= 0 && c < N) ? (c << kRankBits) | atomicAdd(&s_cnt[c], 1) : -1;
        }
    }
    __syncthreads();
    // this block's run of each chunk in the global lists: the atomics (chunks tid + 256 k) go out
    // before the block scan and are used after it
    int gpos[kSortedScatterMaxN / kDispatchRows];
#pragma unroll
    for (int k = 0; k < kSortedScatterMaxN / kDispatchRows; ++k) {
        const int i = tid + k * kDispatchRows;
        const int cnt = i < N ? s_cnt[i] : 0;
        gpos[k] = cnt ? atomicAdd(&chunk_cursor[(size_t)bh * N + i], cnt) + chunk_off[(size_t)bh * N + i] : 0;
    }
    // block exclusive scan of the N counts (contiguous segment per thread)
    const int per = (N + blockDim.x - 1) / blockDim.x;
    const int lo = min(N, tid * per), hi = min(N, lo + per);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += s_cnt[i];
    int total;
    int off = block_exclusive_scan(sum, s_warp, total);
    for (int i = lo; i < hi; ++i) {
        s_scan[i] = off;
        off += s_cnt[i];
    }
#pragma unroll
    for (int k = 0; k < kSortedScatterMaxN / kDispatchRows; ++k) {
        const int i = tid + k * kDispatchRows;
        if (i < N) s_gbase[i] = gpos[k];
    }
    __syncthreads();
    for (int eb = 0; eb < nent; eb += kScatterBatch * kDispatchRows) {
        int vb[kScatterBatch];
        float wb[kScatterBatch];
#pragma unroll
        for (int k = 0; k < kScatterBatch; ++k) {
            const int e = eb + k * kDispatchRows + tid;
            vb[k] = e < nent ? s_tmp[e] : -1;
            wb[k] = e < nent ? sel_w[e0 + e] : 0.0f;
        }
#pragma unroll
        for (int k = 0; k < kScatterBatch; ++k) {
            const int v = vb[k];
            if (v < 0) continue;
            const int c = v >> kRankBits;
            const int p = s_scan[c] + (v & ((1 << kRankBits) - 1));
            s_key[p] = (c << kRankBits) | (eb + k * kDispatchRows + tid);
            s_wt[p] = wb[k];
        }
    }
    __syncthreads();
    for (int i = tid; i < total; i += blockDim.x) {
        const int key = s_key[i];
        const int c = key >> kRankBits, e = key & ((1 << kRankBits) - 1);
        const int pos = s_gbase[c] + (i - s_scan[c]);
        pair_row[pos] = (int32_t)((size_t)bh * T + t0 + e / K);
        pair_w[pos] = s_wt[i];
        if (pair_slot) pair_slot[pos] = e % K;
    }
}

// o_acc -> out (bf16, round to nearest even), 8 elements per thread; grid (ceil(T*D/8/256), B*H). With
// cu_seqlens (sequences padded to T), the rows past a sequence's end are skipped: the caller never reads
// them.
__global__ void finalize_kernel(const float *__restrict__ o_acc, uint16_t *__restrict__ out,
                                const int32_t *__restrict__ cu_seqlens, int T, int H, int D) {
    pdl_launch_dependents();
    pdl_wait();
    const int bh = blockIdx.y;
    const int Tv = cu_seqlens ? min(T, cu_seqlens[bh / H + 1] - cu_seqlens[bh / H]) : T;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;  // 8-element unit within this (b, h)
    if (j >= Tv * (D / 8)) return;
    const size_t i = (size_t)bh * T * (D / 8) + j;
    const float4 a = reinterpret_cast<const float4 *>(o_acc)[2 * i];
    const float4 b = reinterpret_cast<const float4 *>(o_acc)[2 * i + 1];
    uint4 r;
    r.x = pack_bf16x2(a.x, a.y);
    r.y = pack_bf16x2(a.z, a.w);
    r.z = pack_bf16x2(b.x, b.y);
    r.w = pack_bf16x2(b.z, b.w);
    reinterpret_cast<uint4 *>(out)[i] = r;
}

// ------------------------------------------------------------------------------------------------
cudaError_t zero_dispatch_state(int32_t *err, int32_t *chunk_count, int32_t *chunk_cursor, size_t chunks,
                                cudaStream_t s) {
    const char *e0 = reinterpret_cast<const char *>(err);
    const char *c0 = reinterpret_cast<const char *>(chunk_count), *c1 = c0 + chunks * sizeof(int32_t);
    const char *u0 = reinterpret_cast<const char *>(chunk_cursor), *u1 = u0 + chunks * sizeof(int32_t);
    if (err && c0 >= e0 + sizeof(int32_t) && c0 - e0 <= 256 && u0 >= c1 && u0 - c1 <= 256)
        return cudaMemsetAsync(err, 0, (size_t)(u1 - e0), s);
    cudaError_t e = chunks ? cudaMemsetAsync(chunk_count, 0, chunks * sizeof(int32_t), s) : cudaSuccess;
    if (e == cudaSuccess && chunks) e = cudaMemsetAsync(chunk_cursor, 0, chunks * sizeof(int32_t), s);
    if (e == cudaSuccess && err) e = cudaMemsetAsync(err, 0, sizeof(int32_t), s);
    return e;
}

size_t forward_max_tiles(int B, int H, int T, int topk) {
    const size_t pairs = (size_t)B * H * T * topk;
    const size_t chunks = (size_t)B * H * (T / kChunk);
    return pairs / kPairTile + chunks + 1;
}

cudaError_t launch_dispatch(const int32_t *sel_idx, const float *sel_w, int B, int H, int T, int N, int topk,
                            int32_t *chunk_count, int32_t *chunk_off, int32_t *tile_off, int32_t *chunk_cursor,
                            int32_t *pair_row,
                            float *pair_w, int32_t *pair_slot, PairTile *tiles, int32_t *num_tiles, int max_tiles,
                            int tile_pairs, bool counts_ready, cudaStream_t s, const int32_t *cu_seqlens) {
    const int BH = B * H, M = BH * N;
    dim3 dgrid((T + kDispatchRows - 1) / kDispatchRows, BH);
    const size_t hsmem = N <= kSmemHistMax ? (size_t)N * sizeof(int) : 0;
    if (hsmem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsmem);
        if (e != cudaSuccess) return e;
    }
    if (!counts_ready) {  // the forward's score kernel has counted them already
        HSA_PROF("dispatch_count", s);
        cudaError_t e = launch_pdl(count_kernel, dgrid, dim3(kDispatchRows), hsmem, s, sel_idx, T, N, topk, chunk_count);
        if (e != cudaSuccess) return e;
    }
    {
        HSA_PROF("dispatch_scan", s);
        cudaError_t e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, s, chunk_count, M, chunk_off, tile_off,
                                   num_tiles, max_tiles, tile_pairs);
        if (e != cudaSuccess) return e;
    }
    {
        HSA_PROF("dispatch_tiles", s);
        cudaError_t e = launch_pdl(tile_list_kernel, dim3((M + 7) / 8), dim3(256), 0, s, chunk_count, chunk_off,
                                   tile_off, M, tiles, max_tiles, tile_pairs);
        if (e != cudaSuccess) return e;
    }
    if (N <= kSortedScatterMaxN && topk <= 64) {  // ranks and entries fit kRankBits
        const size_t ssmem = 3 * (size_t)N * sizeof(int) + (size_t)kDispatchRows * topk * 3 * sizeof(int);
        cudaError_t e = cudaFuncSetAttribute(scatter_sorted_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)ssmem);
        if (e != cudaSuccess) return e;
        HSA_PROF("dispatch_scatter", s);
        e = launch_pdl(scatter_sorted_kernel, dgrid, dim3(kDispatchRows), ssmem, s, sel_idx, sel_w, T, N, topk,
                       chunk_off, chunk_cursor, pair_row, pair_w, pair_slot, cu_seqlens, H);
        if (e != cudaSuccess) return e;
    } else {
        const size_t ssmem = N <= kSmemHistMax / 2 ? 2 * (size_t)N * sizeof(int) : 0;
        if (ssmem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
            if (e != cudaSuccess) return e;
        }
        HSA_PROF("dispatch_scatter", s);
        cudaError_t e = launch_pdl(scatter_kernel, dgrid, dim3(kDispatchRows), ssmem, s, sel_idx, sel_w, T, N, topk,
                                   chunk_off, chunk_cursor, pair_row, pair_w, pair_slot, cu_seqlens, H);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t launch_forward(const ForwardArgs &a0, cudaStream_t s) {
    ForwardArgs a = a0;
    if (a.Hkv <= 0) a.Hkv = a.H;
    if (a.H % a.Hkv != 0) return cudaErrorInvalidValue;
    if (a0.qk_norm) {  // Step 3 attends with the normalised query and keys; Qs (the raw Q unless
                       // separate) still scores the landmarks
        cudaError_t e = launch_l2norm_rows(a0.Q, a0.Qn, (size_t)a.B * a.H * a.T, a0.K, a0.Kn,
                                           (size_t)a.B * a.Hkv * a.T, a.D, s);
        if (e != cudaSuccess) return e;
        a.Q = a0.Qn;
        a.K = a0.Kn;
    }
    const int BH = a.B * a.H;
    const size_t chunks = (size_t)BH * a.N;
    cudaError_t e;
    {
        HSA_PROF("memset", s);
        // o_acc is zeroed by the score kernel, tile by tile
        e = zero_dispatch_state(a.err, a.chunk_count, a.chunk_cursor, chunks, s);
    }
    if (e != cudaSuccess) return e;
    e = a.topk <= 16 ? launch_score_wide(a, s) : launch_score_tc(a, s);
    if (e != cudaSuccess) return e;
    if (a.N == 0) {
        HSA_PROF("finalize", s);
        finalize_kernel<<<dim3((unsigned)(((size_t)a.T * a.D / 8 + 255) / 256), BH), 256, 0, s>>>(
            a.o_acc, a.out, a.cu_seqlens, a.T, a.H, a.D);
        return cudaGetLastError();
    }
    e = launch_dispatch(a.sel_idx, a.sel_w, a.B, a.H, a.T, a.N, a.topk, a.chunk_count, a.chunk_off, a.tile_off,
                        a.chunk_cursor, a.pair_row, a.pair_w, nullptr, a.tiles, a.num_tiles, a.max_tiles, 128, true, s,
                        a.cu_seqlens);
    if (e != cudaSuccess) return e;
    e = launch_attn_tc(a, s);
    if (e != cudaSuccess) return e;
    {
        HSA_PROF("finalize", s);
        e = launch_pdl(finalize_kernel, dim3((unsigned)(((size_t)a.T * a.D / 8 + 255) / 256), BH), dim3(256), 0, s,
                       a.o_acc, a.out, a.cu_seqlens, a.T, a.H, a.D);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

}  // namespace hsa
