// prefill.cu -- HSA forward for every token of a sequence (prefill).
//
// Explainer page of "Every Token Counts", "How It Works (Technically)", Steps 2-4. HSA is built
// like a mixture of experts whose experts are chunks of the history ("How It Works", opening
// paragraphs), and the kernels follow that shape:
//
//   score_topk_kernel   Step 2: S = scale * Q L^T on the tensor cores for a 128-token tile
//                       against 64-landmark blocks, causal over completed chunks, with a running
//                       per-token top-K (score descending, ties to the lower chunk) and the fusion
//                       softmax (Step 4 weights) in the epilogue. Scores never reach HBM.
//   count / scan /      "Router" bookkeeping: histogram of selected chunks, exclusive scan, and a
//   scatter kernels     scatter of (token, weight) pairs into chunk-major lists cut into tiles of
//                       up to 64 pairs.
//   chunk_attn_kernel   Step 3 + Step 4 blend: per tile, the chunk's 64 keys/values and the tile's
//                       gathered queries in shared memory; S = Q K_c^T, exact softmax over the 64
//                       keys, O = P V_c, scaled by the pair's fusion weight and added into an fp32
//                       accumulator row of the token.
//   finalize_kernel     fp32 accumulator -> bf16 output (round to nearest even).
#include "common.cuh"
#include "launch.h"
#include "profile.h"

namespace hsa {

// ------------------------------------------------------------------------------------------------
// Step 2: scores + per-token top-K + fusion weights
// ------------------------------------------------------------------------------------------------
constexpr int kScoreRows = 128;   // query rows per CTA (one per thread in the top-K epilogue)
constexpr int kScoreCols = 64;    // landmarks per block
constexpr int kScoreThreads = 128;

template <int D>
struct ScoreSmem {
    static constexpr int SD = D + 8;  // padded row stride (bf16 elements): conflict-free ldmatrix
    static constexpr int SS = kScoreCols + 1;
    static constexpr size_t q_bytes = (size_t)kScoreRows * SD * 2;
    static constexpr size_t l_bytes = (size_t)kScoreCols * SD * 2;
    static constexpr size_t s_bytes = (size_t)kScoreRows * SS * 4;
    static constexpr int SJ = 68;  // bytes per row of candidate column ids (17 words: conflict-free)
    static constexpr size_t j_bytes = (size_t)kScoreRows * SJ;
    static constexpr size_t total = q_bytes + 2 * l_bytes + s_bytes + j_bytes;
};

// K is the compile-time length of the running list (8, 16 or 32); the first kout <= K entries
// are the requested top-kout (a prefix of a longer sorted top list is the shorter top list).
template <int D, int K>
__global__ void __launch_bounds__(kScoreThreads) score_topk_kernel(const uint16_t *__restrict__ Q,
                                                                   const uint16_t *__restrict__ L, int T, int N,
                                                                   float scale, int kout,
                                                                   int32_t *__restrict__ sel_idx,
                                                                   float *__restrict__ sel_w) {
    using SM = ScoreSmem<D>;
    constexpr int SD = SM::SD, SS = SM::SS;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint16_t *sQ = reinterpret_cast<uint16_t *>(smem_raw);
    uint16_t *sL = reinterpret_cast<uint16_t *>(smem_raw + SM::q_bytes);
    float *sS = reinterpret_cast<float *>(smem_raw + SM::q_bytes + 2 * SM::l_bytes);
    uint8_t *sJ = smem_raw + SM::q_bytes + 2 * SM::l_bytes + SM::s_bytes;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ntile = (T + kScoreRows - 1) / kScoreRows;
    const int tile = ntile - 1 - blockIdx.x;  // longest rows first
    const int bh = blockIdx.y;
    const int t0 = tile * kScoreRows;
    const int t_last = min(T - 1, t0 + kScoreRows - 1);
    const int n_max = min(N, (t_last + 1) / kChunk);
    const int nblk = (n_max + kScoreCols - 1) / kScoreCols;

    const uint16_t *Qbh = Q + (size_t)bh * T * D;
    const uint16_t *Lbh = L + (size_t)bh * N * D;
    constexpr int VPR = D / 8;  // 16-byte vectors per row

    auto load_L = [&](int blk, int buf) {
        uint16_t *dst = sL + (size_t)buf * kScoreCols * SD;
        for (int i = tid; i < kScoreCols * VPR; i += kScoreThreads) {
            const int r = i / VPR, v = i % VPR;
            const int c = blk * kScoreCols + r;
            const bool ok = c < n_max;
            cp_async16(dst + r * SD + v * 8, ok ? (const void *)(Lbh + (size_t)c * D + v * 8) : (const void *)Lbh,
                       ok ? 16 : 0);
        }
    };

    if (nblk > 0) {
        for (int i = tid; i < kScoreRows * VPR; i += kScoreThreads) {
            const int r = i / VPR, v = i % VPR;
            const int t = t0 + r;
            const bool ok = t < T;
            cp_async16(sQ + r * SD + v * 8, ok ? (const void *)(Qbh + (size_t)t * D + v * 8) : (const void *)Qbh,
                       ok ? 16 : 0);
        }
        load_L(0, 0);
    }
    cp_async_commit();

    // per-thread (= per-row) running top-K, sorted by score descending; equal scores keep the
    // earlier (lower) chunk first because chunks are visited in increasing order
    float ls[K];
    int li[K];
#pragma unroll
    for (int i = 0; i < K; ++i) { ls[i] = -INFINITY; li[i] = -1; }
    const int my_t = t0 + tid;
    const int my_n = my_t < T ? min(N, (my_t + 1) / kChunk) : 0;

    for (int blk = 0; blk < nblk; ++blk) {
        if (blk + 1 < nblk) {
            load_L(blk + 1, (blk + 1) & 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint16_t *sLb = sL + (size_t)(blk & 1) * kScoreCols * SD;
        float acc[2][8][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[mt][nt][r] = 0.0f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
                ldmatrix_x4(a[mt][0], a[mt][1], a[mt][2], a[mt][3],
                            sQ + (warp * 32 + mt * 16 + (lane & 15)) * SD + ks * 16 + (lane >> 4) * 8);
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(b0, b1, b2, b3,
                            sLb + (np * 16 + (lane & 7) + (lane >> 4) * 8) * SD + ks * 16 + ((lane >> 3) & 1) * 8);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    mma_bf16_16816(acc[mt][2 * np], a[mt], b0, b1);
                    mma_bf16_16816(acc[mt][2 * np + 1], a[mt], b2, b3);
                }
            }
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int row = warp * 32 + mt * 16 + (lane >> 2) + (r >= 2 ? 8 : 0);
                    const int col = nt * 8 + (lane & 3) * 2 + (r & 1);
                    sS[row * SS + col] = acc[mt][nt][r] * scale;
                }
        __syncthreads();
        // per-row top-K update in two phases, so that a warp does not serialise on every column in
        // which any of its 32 rows inserts: (1) compact, in place, the columns that beat the row's
        // current K-th score (branch-light); (2) insert only those candidates.
        const int cbase = blk * kScoreCols;
        const int ncol = min(kScoreCols, my_n - cbase);
        float *row = sS + tid * SS;
        uint8_t *rj = sJ + tid * SM::SJ;
        const float tau = ls[K - 1];
        int nc = 0;
        for (int j = 0; j < ncol; ++j) {
            const float s = row[j];
            if (s > tau) {  // nc <= j: the slot written was already read
                row[nc] = s;
                rj[nc] = (uint8_t)j;
                ++nc;
            }
        }
        for (int i = 0; i < nc; ++i) {
            const float s = row[i];
            if (s > ls[K - 1]) {
                const int c = cbase + rj[i];
#pragma unroll
                for (int q = K - 1; q > 0; --q) {
                    const bool prev_lt = ls[q - 1] < s;
                    const bool cur_lt = ls[q] < s;
                    const float ns = prev_lt ? ls[q - 1] : (cur_lt ? s : ls[q]);
                    const int ni = prev_lt ? li[q - 1] : (cur_lt ? c : li[q]);
                    ls[q] = ns;
                    li[q] = ni;
                }
                if (ls[0] < s) { ls[0] = s; li[0] = c; }
            }
        }
    }
    if (my_t >= T) return;
    // Step 4 weights: softmax over the kept scores (fp32, max-subtracted)
    float e[K];
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < K; ++i) {
        e[i] = (i < kout && li[i] >= 0) ? expf(ls[i] - ls[0]) : 0.0f;
        z += e[i];
    }
    const float inv = z > 0.0f ? 1.0f / z : 0.0f;
    const size_t row = (size_t)bh * T + my_t;
#pragma unroll
    for (int i = 0; i < K; ++i) {
        if (i < kout) {
            sel_idx[row * kout + i] = li[i];
            sel_w[row * kout + i] = e[i] * inv;
        }
    }
}

// ------------------------------------------------------------------------------------------------
// Dispatch: chunk-major pair lists
// ------------------------------------------------------------------------------------------------
constexpr int kDispatchRows = 256;
constexpr int kSmemHistMax = 8192;  // chunks per (b, h) histogrammed in shared memory

__global__ void __launch_bounds__(kDispatchRows) count_kernel(const int32_t *__restrict__ sel_idx, int T, int N,
                                                              int K, int32_t *__restrict__ chunk_count) {
    extern __shared__ int s_hist[];
    const int bh = blockIdx.y;
    const bool use_smem = N <= kSmemHistMax;
    if (use_smem) {
        for (int i = threadIdx.x; i < N; i += blockDim.x) s_hist[i] = 0;
        __syncthreads();
    }
    const int t = blockIdx.x * kDispatchRows + threadIdx.x;
    if (t < T) {
        const int32_t *si = sel_idx + ((size_t)bh * T + t) * K;
        for (int j = 0; j < K; ++j) {
            const int c = si[j];
            if (c < 0 || c >= N) continue;  // -1 = empty slot; ids past N are ignored
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

// One CTA: exclusive offsets of every chunk's pair list and of its tiles (<= kPairTile pairs each).
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t *__restrict__ chunk_count, int M,
                                                    int32_t *__restrict__ chunk_off, int32_t *__restrict__ tile_off,
                                                    int32_t *__restrict__ num_tiles, int max_tiles, int tp) {
    __shared__ int s_warp[33];
    const int per = (M + blockDim.x - 1) / blockDim.x;
    const int lo = min(M, (int)threadIdx.x * per), hi = min(M, lo + per);
    int sum = 0, tsum = 0;
    for (int i = lo; i < hi; ++i) {
        const int c = chunk_count[i];
        sum += c;
        tsum += (c + tp - 1) / tp;
    }
    int total, ttotal;
    int off = block_exclusive_scan(sum, s_warp, total);
    int toff = block_exclusive_scan(tsum, s_warp, ttotal);
    for (int i = lo; i < hi; ++i) {
        const int c = chunk_count[i];
        chunk_off[i] = off;
        tile_off[i] = toff;
        off += c;
        toff += (c + tp - 1) / tp;
    }
    if (threadIdx.x == 0) {
        chunk_off[M] = total;
        tile_off[M] = ttotal;
        num_tiles[0] = min(ttotal, max_tiles);
    }
}

// One warp per chunk writes that chunk's tiles into the work list.
__global__ void __launch_bounds__(256) tile_list_kernel(const int32_t *__restrict__ chunk_count,
                                                        const int32_t *__restrict__ chunk_off,
                                                        const int32_t *__restrict__ tile_off, int M,
                                                        PairTile *__restrict__ tiles, int max_tiles, int tp) {
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
                                                                int32_t *__restrict__ pair_slot) {
    extern __shared__ int s_mem[];
    const int bh = blockIdx.y;
    const bool use_smem = N <= kSmemHistMax / 2;
    int *s_cnt = s_mem, *s_base = s_mem + (use_smem ? N : 0);
    const int t = blockIdx.x * kDispatchRows + threadIdx.x;
    const int32_t *si = sel_idx + ((size_t)bh * T + (t < T ? t : 0)) * K;
    if (use_smem) {
        for (int i = threadIdx.x; i < N; i += blockDim.x) s_cnt[i] = 0;
        __syncthreads();
        if (t < T)
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
    if (t >= T) return;
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
// pair-list positions (coalesced stores instead of one scattered store per entry). Used when the
// chunk count per (b, h) fits the shared-memory tables (N <= kSortedScatterMaxN).
constexpr int kSortedScatterMaxN = 2048;

__global__ void __launch_bounds__(kDispatchRows) scatter_sorted_kernel(
    const int32_t *__restrict__ sel_idx, const float *__restrict__ sel_w, int T, int N, int K,
    const int32_t *__restrict__ chunk_off, int32_t *__restrict__ chunk_cursor, int32_t *__restrict__ pair_row,
    float *__restrict__ pair_w, int32_t *__restrict__ pair_slot) {
    extern __shared__ int s_mem[];
    int *s_cnt = s_mem;                  // [N] entries per chunk in this block
    int *s_scan = s_cnt + N;             // [N] exclusive scan of s_cnt
    int *s_gbase = s_scan + N;           // [N] global position of this block's run for the chunk
    int *s_cur = s_gbase + N;            // [N] ranks handed out so far
    int *s_key = s_cur + N;              // [rows * K] (c << 14) | (t_local << 6) | slot, sorted by chunk
    float *s_wt = reinterpret_cast<float *>(s_key + kDispatchRows * K);
    __shared__ int s_warp[33];
    const int bh = blockIdx.y, tid = threadIdx.x;
    const int t0 = blockIdx.x * kDispatchRows;
    const int t = t0 + tid;
    for (int i = tid; i < N; i += blockDim.x) { s_cnt[i] = 0; s_cur[i] = 0; }
    __syncthreads();
    const int32_t *si = sel_idx + ((size_t)bh * T + (t < T ? t : 0)) * K;
    if (t < T)
        for (int j = 0; j < K; ++j) {
            const int c = si[j];
            if (c >= 0 && c < N) atomicAdd(&s_cnt[c], 1);
        }
    __syncthreads();
    // block exclusive scan of the N counts (contiguous segment per thread)
    const int per = (N + blockDim.x - 1) / blockDim.x;
    const int lo = min(N, tid * per), hi = min(N, lo + per);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += s_cnt[i];
    int total;
    int off = block_exclusive_scan(sum, s_warp, total);
    for (int i = lo; i < hi; ++i) {
        const int cnt = s_cnt[i];
        s_scan[i] = off;
        s_gbase[i] = cnt ? chunk_off[(size_t)bh * N + i] + atomicAdd(&chunk_cursor[(size_t)bh * N + i], cnt) : 0;
        off += cnt;
    }
    __syncthreads();
    if (t < T)
        for (int j = 0; j < K; ++j) {
            const int c = si[j];
            if (c < 0 || c >= N) continue;
            const int p = s_scan[c] + atomicAdd(&s_cur[c], 1);
            s_key[p] = (c << 14) | (tid << 6) | j;
            s_wt[p] = sel_w[((size_t)bh * T + t) * K + j];
        }
    __syncthreads();
    for (int i = tid; i < total; i += blockDim.x) {
        const int key = s_key[i];
        const int c = key >> 14, tl = (key >> 6) & 0xff, j = key & 63;
        const int pos = s_gbase[c] + (i - s_scan[c]);
        pair_row[pos] = (int32_t)((size_t)bh * T + t0 + tl);
        pair_w[pos] = s_wt[i];
        if (pair_slot) pair_slot[pos] = j;
    }
}

// ------------------------------------------------------------------------------------------------
// Step 3 + Step 4 blend, chunk-major
// ------------------------------------------------------------------------------------------------
constexpr int kAttnThreads = 128;  // 4 warps x 16 pairs = kPairTile

template <int D>
__global__ void __launch_bounds__(kAttnThreads) chunk_attn_kernel(
    const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K, const uint16_t *__restrict__ V, int T, int N,
    float scale, const PairTile *__restrict__ tiles, const int32_t *__restrict__ num_tiles,
    const int32_t *__restrict__ pair_row, const float *__restrict__ pair_w, float *__restrict__ o_acc) {
    constexpr int SD = D + 8, VPR = D / 8;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint16_t *sK = reinterpret_cast<uint16_t *>(smem_raw);
    uint16_t *sV = sK + kChunk * SD;
    uint16_t *sQ = sV + kChunk * SD;
    __shared__ int s_row[kPairTile];
    __shared__ float s_w[kPairTile];

    if ((int)blockIdx.x >= num_tiles[0]) return;
    const PairTile pt = tiles[blockIdx.x];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = pt.chunk / N, c = pt.chunk % N;
    const uint16_t *Kc = K + ((size_t)bh * T + (size_t)c * kChunk) * D;
    const uint16_t *Vc = V + ((size_t)bh * T + (size_t)c * kChunk) * D;
    if (tid < kPairTile) {
        const bool ok = tid < pt.count;
        s_row[tid] = ok ? pair_row[pt.start + tid] : -1;
        s_w[tid] = ok ? pair_w[pt.start + tid] : 0.0f;
    }
    __syncthreads();
    for (int i = tid; i < kChunk * VPR; i += kAttnThreads) {
        const int r = i / VPR, v = i % VPR;
        cp_async16(sK + r * SD + v * 8, Kc + (size_t)r * D + v * 8, 16);
        const int row = s_row[r];
        cp_async16(sQ + r * SD + v * 8, row >= 0 ? (const void *)(Q + (size_t)row * D + v * 8) : (const void *)Q,
                   row >= 0 ? 16 : 0);
    }
    cp_async_commit();
    for (int i = tid; i < kChunk * VPR; i += kAttnThreads) {
        const int r = i / VPR, v = i % VPR;
        cp_async16(sV + r * SD + v * 8, Vc + (size_t)r * D + v * 8, 16);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    // S = Q_w K_c^T : 16 pairs x 64 keys per warp
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) s[nt][r] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a[0], a[1], a[2], a[3], sQ + (warp * 16 + (lane & 15)) * SD + ks * 16 + (lane >> 4) * 8);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3,
                        sK + (np * 16 + (lane & 7) + (lane >> 4) * 8) * SD + ks * 16 + ((lane >> 3) & 1) * 8);
            mma_bf16_16816(s[2 * np], a, b0, b1);
            mma_bf16_16816(s[2 * np + 1], a, b2, b3);
        }
    }
    // exact softmax over the chunk's 64 keys (rows g and g+8 of this warp's 16)
    const float sl2 = scale * 1.4426950408889634f;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    float sum0 = 0.0f, sum1 = 0.0f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        s[nt][0] = exp2f((s[nt][0] - mx0) * sl2);
        s[nt][1] = exp2f((s[nt][1] - mx0) * sl2);
        s[nt][2] = exp2f((s[nt][2] - mx1) * sl2);
        s[nt][3] = exp2f((s[nt][3] - mx1) * sl2);
        sum0 += s[nt][0] + s[nt][1];
        sum1 += s[nt][2] + s[nt][3];
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
        sum0 += __shfl_xor_sync(0xffffffffu, sum0, o);
        sum1 += __shfl_xor_sync(0xffffffffu, sum1, o);
    }
    cp_async_wait<0>();
    __syncthreads();

    // O = P V_c : 16 pairs x D
    float o[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) o[nt][r] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < kChunk / 16; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
        a[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
        a[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        a[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(b0, b1, b2, b3,
                              sV + (kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * SD + np * 16 + (lane >> 4) * 8);
            mma_bf16_16816(o[2 * np], a, b0, b1);
            mma_bf16_16816(o[2 * np + 1], a, b2, b3);
        }
    }
    // epilogue: w_pair / rowsum, fp32 vector reduction into the token's accumulator row
    const int p0 = warp * 16 + (lane >> 2), p1 = p0 + 8;
    const int row0 = s_row[p0], row1 = s_row[p1];
    const float f0 = row0 >= 0 ? s_w[p0] / sum0 : 0.0f;
    const float f1 = row1 >= 0 ? s_w[p1] / sum1 : 0.0f;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
        const int col = nt * 8 + (lane & 3) * 2;
        if (row0 >= 0) red_add_v2(o_acc + (size_t)row0 * D + col, o[nt][0] * f0, o[nt][1] * f0);
        if (row1 >= 0) red_add_v2(o_acc + (size_t)row1 * D + col, o[nt][2] * f1, o[nt][3] * f1);
    }
}

__global__ void finalize_kernel(const float *__restrict__ o_acc, uint16_t *__restrict__ out, size_t n8) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n8) return;
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
size_t forward_max_tiles(int B, int H, int T, int topk) {
    const size_t pairs = (size_t)B * H * T * topk;
    const size_t chunks = (size_t)B * H * (T / kChunk);
    return pairs / kPairTile + chunks + 1;
}

template <int D, int K>
static cudaError_t launch_score(const ForwardArgs &a, cudaStream_t s) {
    const size_t smem = ScoreSmem<D>::total;
    cudaError_t e = cudaFuncSetAttribute(score_topk_kernel<D, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.T + kScoreRows - 1) / kScoreRows, a.B * a.H);
    HSA_PROF("score_topk", s);
    score_topk_kernel<D, K><<<grid, kScoreThreads, smem, s>>>(a.Q, a.L, a.T, a.N, a.scale, a.topk, a.sel_idx,
                                                              a.sel_w);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_score_d(const ForwardArgs &a, cudaStream_t s) {
    if (a.topk <= 8) return launch_score<D, 8>(a, s);
    if (a.topk <= 16) return launch_score<D, 16>(a, s);
    return launch_score<D, 32>(a, s);
}

cudaError_t launch_dispatch(const int32_t *sel_idx, const float *sel_w, int B, int H, int T, int N, int topk,
                            int32_t *chunk_count, int32_t *chunk_off, int32_t *tile_off, int32_t *chunk_cursor,
                            int32_t *pair_row,
                            float *pair_w, int32_t *pair_slot, PairTile *tiles, int32_t *num_tiles, int max_tiles,
                            int tile_pairs, cudaStream_t s) {
    const int BH = B * H;
    dim3 dgrid((T + kDispatchRows - 1) / kDispatchRows, BH);
    const size_t hsmem = N <= kSmemHistMax ? (size_t)N * sizeof(int) : 0;
    if (hsmem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsmem);
        if (e != cudaSuccess) return e;
    }
    {
        HSA_PROF("dispatch_count", s);
        count_kernel<<<dgrid, kDispatchRows, hsmem, s>>>(sel_idx, T, N, topk, chunk_count);
    }
    {
        HSA_PROF("dispatch_scan", s);
        scan_kernel<<<1, 1024, 0, s>>>(chunk_count, BH * N, chunk_off, tile_off, num_tiles, max_tiles, tile_pairs);
    }
    {
        HSA_PROF("dispatch_tiles", s);
        tile_list_kernel<<<(BH * N + 7) / 8, 256, 0, s>>>(chunk_count, chunk_off, tile_off, BH * N, tiles,
                                                          max_tiles, tile_pairs);
    }
    if (N <= kSortedScatterMaxN) {
        const size_t ssmem = 4 * (size_t)N * sizeof(int) + (size_t)kDispatchRows * topk * (sizeof(int) + sizeof(float));
        cudaError_t e = cudaFuncSetAttribute(scatter_sorted_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)ssmem);
        if (e != cudaSuccess) return e;
        HSA_PROF("dispatch_scatter", s);
        scatter_sorted_kernel<<<dgrid, kDispatchRows, ssmem, s>>>(sel_idx, sel_w, T, N, topk, chunk_off, chunk_cursor,
                                                                  pair_row, pair_w, pair_slot);
    } else {
        const size_t ssmem = N <= kSmemHistMax / 2 ? 2 * (size_t)N * sizeof(int) : 0;
        if (ssmem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
            if (e != cudaSuccess) return e;
        }
        HSA_PROF("dispatch_scatter", s);
        scatter_kernel<<<dgrid, kDispatchRows, ssmem, s>>>(sel_idx, sel_w, T, N, topk, chunk_off, chunk_cursor,
                                                           pair_row, pair_w, pair_slot);
    }
    return cudaGetLastError();
}

cudaError_t launch_forward(const ForwardArgs &a, cudaStream_t s) {
    const int BH = a.B * a.H;
    const size_t rows = (size_t)BH * a.T;
    cudaError_t e;
    {
        HSA_PROF("memset", s);
        e = cudaMemsetAsync(a.o_acc, 0, rows * a.D * sizeof(float), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.chunk_count, 0, (size_t)BH * a.N * sizeof(int32_t), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.chunk_cursor, 0, (size_t)BH * a.N * sizeof(int32_t), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.err, 0, sizeof(int32_t), s);
    }
    if (e != cudaSuccess) return e;
    e = a.D == 128 ? launch_score_d<128>(a, s) : launch_score_d<64>(a, s);
    if (e != cudaSuccess) return e;
    if (a.N == 0) {
        const size_t n8 = rows * a.D / 8;
        HSA_PROF("finalize", s);
        finalize_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(a.o_acc, a.out, n8);
        return cudaGetLastError();
    }
    e = launch_dispatch(a.sel_idx, a.sel_w, a.B, a.H, a.T, a.N, a.topk, a.chunk_count, a.chunk_off, a.tile_off,
                        a.chunk_cursor, a.pair_row, a.pair_w, nullptr, a.tiles, a.num_tiles, a.max_tiles, 128, s);
    if (e != cudaSuccess) return e;
    e = launch_attn_tc(a, s);
    if (e != cudaSuccess) return e;
    const size_t n8 = rows * a.D / 8;
    {
        HSA_PROF("finalize", s);
        finalize_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(a.o_acc, a.out, n8);
    }
    return cudaGetLastError();
}

}  // namespace hsa
