// score_tc.cu -- Step 2 (retrieval scores + top-K) and the Step 4 fusion weights of the HSA forward,
// on the 5th-generation tensor cores.
//
// Explainer page of "Every Token Counts", "How It Works (Technically)", Step 2: each token t scores
// every chunk that has ended at or before it, s[t,c] = scale * Q[t].L[c], and keeps the top-K; the
// per-token procedure ("The algorithm, simplified") sorts the scores in descending order, stably,
// so equal scores keep the lower chunk first. Step 4: w = softmax of the kept scores.
//
// One CTA per (128-token tile, batch*head); thread = token row = TMEM lane. The design aims at many
// resident warps (the selection is latency-bound per thread): a CTA holds 128 TMEM columns and about
// 50 KB of shared memory, so four CTAs (16 selecting warps) share an SM.
//   * The Q tile lives in TMEM: each selecting thread loads its own row and writes it to its lane
//     (tcgen05.st, two bf16 per column), and the MMA reads it as the A operand.
//   * Warp 4 is the producer (the warp runs it, one elected lane issues): 32-landmark blocks arrive by
//     TMA in the 128-byte-swizzled
//     layout (three stages), and it issues S_blk = Q L_blk^T (M = 128, N = 32, fp32) into one of the
//     TMEM score buffers. Full/empty mbarriers link it to warps 0-3, which run decoupled.
//   * Scores are compared unscaled (the scale is positive, so the order is the same); it enters the
//     fusion weights only. For each 32-landmark block a thread stores its row's 32 scores to a
//     per-thread column of shared memory at fixed offsets and sets one bit per candidate, so the
//     per-score cost is a store, a compare and an OR; only the set bits are visited afterwards.
//   * Pass 1 keeps, per row, the K largest score VALUES in a sorted register list: the candidates
//     are the scores above the current K-th value, each inserted with
//     new[i] = max(old[i], min(old[i-1], x)), which touches every slot independently (no dependent
//     chain). The first block seeds the list through a bitonic sorting network on its 32 values
//     instead. The K-th value tau results.
//   * Pass 2 recomputes the same blocks (bit-identical: same operands, same instruction sequence);
//     the candidates are the scores >= tau, visited in chunk order, and it keeps every one above tau
//     plus the lowest-index ones equal to tau until K are kept -- exactly the stable-sort rule. A
//     kept chunk's output slot is known when it is taken (the number of kept values above it, ties
//     in chunk order), so only its chunk id is stored; its value is the slot's entry of the sorted
//     list.
//   * At the end each row computes the fusion weights w = softmax over the kept values (fp32,
//     max-subtracted), and the tile's rows, contiguous in [B, H, T, K], are written by coalesced
//     stores through shared memory.
//   * Two pieces of the dispatch ride along, on memory bandwidth this ALU-bound kernel leaves idle:
//     the tile's rows of the fp32 output accumulator are zeroed, and the number of selected pairs per
//     chunk is counted in a shared-memory histogram and added into the dispatch's chunk counts.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "launch.h"
#include "profile.h"
#include "tc.cuh"

namespace hsa {

constexpr int kStRows = 128;                   // tokens per CTA (MMA M)
constexpr int kStCols = 32;                    // landmarks per block (MMA N)
constexpr int kStConsumers = 128;              // warps 0-3
constexpr int kStThreads = kStConsumers + 32;  // + producer warp
constexpr int kStLStages = 3;                  // landmark blocks in shared memory
constexpr uint32_t kStTmemCols = 128;          // Q (D/2 columns) + score buffers
constexpr int kStMaxCtasPerSm = 4;             // kStTmemCols x 4 = all 512 TMEM columns
constexpr int kStHistMax = 1024;               // chunks per (b, h) counted in shared memory

template <int D, int K>
struct StSmem {
    static constexpr int KH = D / 64;
    static constexpr uint32_t QCOLS = D / 2;                          // TMEM columns of the Q tile
    static constexpr int NB = (int)(kStTmemCols - QCOLS) / kStCols;   // TMEM score buffers
    static constexpr uint32_t LH = kStCols * 128;                     // one 64-column half of a block
    static constexpr uint32_t LB = KH * LH;                           // one landmark stage
    static constexpr uint32_t STAGE = 128 * (K + 1) * 8;              // output staging: idx + w, padded rows
    // region U holds the landmark stages during the loop and the output staging at the end
    static constexpr uint32_t U = kStLStages * LB > STAGE ? kStLStages * LB : STAGE;
    // [128][36] fp32: a block's scores, one padded row per thread (16-byte stores without bank
    // conflicts); [K+1][128] int32: the chunk of each output slot.
    static constexpr uint32_t CV = U;
    static constexpr uint32_t CC = CV + 128 * 36 * 4;
    static constexpr uint32_t HIST = CC + (K + 1) * 128 * 4;  // int[kStHistMax]: selected pairs per chunk
    static constexpr uint32_t BAR = HIST + kStHistMax * 4;  // q_ready, full_l[3], empty_l[3], full_s[NB], empty_s[NB]
    static constexpr int NBAR = 1 + 2 * kStLStages + 2 * NB;
    static constexpr uint32_t TMEM = BAR + NBAR * 8;
    static constexpr uint32_t BYTES = TMEM + 8;
    // padded so that at most four CTAs share an SM and their TMEM allocations always fit
    static constexpr size_t MIN_DYN = 228 * 1024 / (kStMaxCtasPerSm + 1) + 1024;
    static constexpr size_t DYN = BYTES + 1024 > MIN_DYN ? BYTES + 1024 : MIN_DYN;
    static_assert(NB >= 2, "need two score buffers");
};

template <int D, int K>
__global__ void __launch_bounds__(kStThreads) score_topk_tc_kernel(const uint16_t *__restrict__ Q, int T, int N,
                                                                   int Gh, int H, const int32_t *__restrict__ cu_seqlens,
                                                                   float scale, int kout,
                                                                   int32_t *__restrict__ sel_idx,
                                                                   float *__restrict__ sel_w, float *__restrict__ o_acc,
                                                                   int32_t *__restrict__ chunk_count,
                                                                   int32_t *__restrict__ err,
                                                                   const __grid_constant__ CUtensorMap tmL) {
    using SM = StSmem<D, K>;
    constexpr int NB = SM::NB;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    unsigned char *s = smem_raw + (sb - raw);
    const uint32_t q_ready = sb + SM::BAR;
    auto full_l = [&](int i) { return sb + SM::BAR + 8u * (1 + i); };
    auto empty_l = [&](int i) { return sb + SM::BAR + 8u * (1 + kStLStages + i); };
    auto full_s = [&](int i) { return sb + SM::BAR + 8u * (1 + 2 * kStLStages + i); };
    auto empty_s = [&](int i) { return sb + SM::BAR + 8u * (1 + 2 * kStLStages + NB + i); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntile = (T + kStRows - 1) / kStRows;
    const int tile = ntile - 1 - blockIdx.x;  // longest rows first
    const int bh = blockIdx.y, kvh = bh / Gh;  // Gh query heads share a landmark head
    const int t0 = tile * kStRows;
    const int nrows = min(kStRows, T - t0);
    // valid tokens of this sequence: all T, or its length when the batch holds sequences padded to T
    const int Tv = cu_seqlens ? min(T, cu_seqlens[bh / H + 1] - cu_seqlens[bh / H]) : T;
    const int t_last = min(t0 + nrows - 1, Tv - 1);
    const int n_max = t_last >= 0 ? min(N, (t_last + 1) / kChunk) : 0;
    const int nblk = (n_max + kStCols - 1) / kStCols;
    const size_t out0 = ((size_t)bh * T + t0) * kout;  // the tile's rows are contiguous

    // rows past the sequence's end (padded batches) are never read: no accumulator, no selection written
    const int nv = max(0, min(nrows, Tv - t0));
    {  // this tile's rows of the fp32 output accumulator start at zero (the chunk attention adds into them)
        float4 *acc = reinterpret_cast<float4 *>(o_acc + ((size_t)bh * T + t0) * D);
        for (int i = tid; i < nv * (D / 4); i += kStThreads) acc[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    }
    if (nblk == 0) {  // no token of this tile has a complete chunk
        for (int i = tid; i < nv * kout; i += kStThreads) {
            sel_idx[out0 + i] = -1;
            sel_w[out0 + i] = 0.0f;
        }
        return;
    }
    int *s_hist = reinterpret_cast<int *>(s + SM::HIST);  // pairs per chunk of this tile (n_max <= N)
    const bool hist_smem = n_max <= kStHistMax;
    if (hist_smem)
        for (int i = tid; i < n_max; i += kStThreads) s_hist[i] = 0;  // ordered by the __syncthreads below

    if (warp == 0) tc::tmem_alloc(sb + SM::TMEM, kStTmemCols);
    if (tid == kStConsumers) {
        tc::mbar_init(q_ready, kStConsumers / 32);
        for (int i = 0; i < kStLStages; ++i) {
            tc::mbar_init(full_l(i), 1);
            tc::mbar_init(empty_l(i), 1);
        }
        for (int i = 0; i < NB; ++i) {
            tc::mbar_init(full_s(i), 1);
            tc::mbar_init(empty_s(i), kStConsumers / 32);
        }
        tc::fence_mbar_init();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<uint32_t *>(s + SM::TMEM);
    const int G = 2 * nblk;  // blocks visited: pass 1, then pass 2
    bool ok = true;

    if (warp == kStConsumers / 32) {
        // ---------------- producer: the whole warp runs it, one elected lane issues (tc::*_w) ----------------
        {
            auto load_l = [&](int h) {  // landmark block h % nblk into stage h % 3
                const int st = h % kStLStages;
                const uint32_t dst = sb + st * SM::LB;
                tc::mbar_arrive_expect_tx_w(full_l(st), SM::LB);
#pragma unroll
                for (int k = 0; k < SM::KH; ++k)
                    tc::tma_load_2d_w(dst + k * SM::LH, &tmL, k * 64, kvh * N + (h % nblk) * kStCols, full_l(st));
            };
            int nload = 0, nmma = 0;
            for (; nload < kStLStages && nload < G; ++nload) load_l(nload);
            ok = tc::mbar_wait(q_ready, 0);
            constexpr uint32_t idesc = tc::idesc_bf16(kStRows, kStCols, 0, 0);
            for (int g = 0; ok && g < G; ++g) {
                const int st = g % kStLStages, buf = g % NB;
                if (!tc::mbar_wait(full_l(st), (uint32_t)(g / kStLStages) & 1u) ||
                    (g >= NB && !tc::mbar_wait(empty_s(buf), (uint32_t)(g / NB - 1) & 1u))) {
                    ok = false;
                    break;
                }
                tc::fence_after();
                const uint32_t lb = sb + st * SM::LB;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks)  // K step of 16: 8 TMEM columns of Q, 32 B of a swizzled row
                    tc::mma_bf16_ts_w(tmem + SM::QCOLS + buf * kStCols, tmem + ks * 8,
                                    tc::desc_kmajor(lb + (ks >> 2) * SM::LH + (ks & 3) * 32), idesc, ks > 0 ? 1u : 0u);
                tc::commit_w(full_s(buf));
                tc::commit_w(empty_l(st));
                nmma = g + 1;
                if (g + kStLStages < G) {  // refill this stage once MMA(g) has read it
                    if (!tc::mbar_wait(empty_l(st), (uint32_t)(g / kStLStages) & 1u)) {
                        ok = false;
                        break;
                    }
                    load_l(nload++);
                }
            }
            if (!ok) {  // let every copy and MMA this CTA started finish before its memory goes away
                atomicOr(err, 1);
                for (int h = nmma; h < nload; ++h) tc::mbar_wait(full_l(h % kStLStages), (uint32_t)(h / kStLStages) & 1u);
                if (nmma > 0) tc::mbar_wait(full_s((nmma - 1) % NB), (uint32_t)((nmma - 1) / NB) & 1u);
            }
        }
        __syncwarp();
    } else {
        // ---------------- selecting warps: one token row per thread ----------------
        const int my_t = t0 + tid;
        const int my_n = my_t < Tv ? min(N, (my_t + 1) / kChunk) : 0;
        const int k_keep = min(kout, my_n);
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

        {  // this row of Q into TMEM lane tid, columns [0, D/2)
            const uint4 *src = reinterpret_cast<const uint4 *>(Q + ((size_t)bh * T + (my_t < T ? my_t : t0)) * D);
#pragma unroll
            for (int h = 0; h < D / 64; ++h) {
                uint32_t r[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    uint4 u = make_uint4(0u, 0u, 0u, 0u);
                    if (my_t < T) u = __ldg(src + h * 8 + i);
                    r[4 * i] = u.x;
                    r[4 * i + 1] = u.y;
                    r[4 * i + 2] = u.z;
                    r[4 * i + 3] = u.w;
                }
                tc::tmem_st32(tmem + lane_off + h * 32, r);
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(q_ready);
        }

        // Scores are compared unscaled (scale > 0 keeps their order); the scale enters the weights only.
        float *cv = reinterpret_cast<float *>(s + SM::CV) + tid * 36;  // this thread's row: a block's scores
        int *cc = reinterpret_cast<int *>(s + SM::CC) + tid;      // chunk of each output slot
        float ls[K];  // pass 1: the K largest score values of this row, descending
#pragma unroll
        for (int i = 0; i < K; ++i) ls[i] = -INFINITY;
        float tau = -INFINITY;
        int need_eq = 0;
        uint64_t used = 0;  // pass 2: output slots filled

        for (int g = 0; g < G; ++g) {
            const int buf = g % NB;
            if (!__all_sync(~0u, tc::mbar_wait(full_s(buf), (uint32_t)(g / NB) & 1u))) {
                ok = false;
                break;
            }
            tc::fence_after();
            float v[32];
            tc::tmem_ld32(tmem + lane_off + SM::QCOLS + buf * kStCols, v);
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(empty_s(buf));  // the scores are in registers now

            if (g == nblk) {
                // end of pass 1: tau = the k_keep-th largest value; ties at tau go lowest chunk first
                tau = k_keep > 0 ? -INFINITY : INFINITY;
                int gt = 0;
#pragma unroll
                for (int i = 0; i < K; ++i)
                    if (i < k_keep) tau = ls[i];
#pragma unroll
                for (int i = 0; i < K; ++i) gt += (i < k_keep && ls[i] > tau) ? 1 : 0;
                need_eq = k_keep - gt;
            }
            const int b = g % nblk;
            const int ncol = min(kStCols, my_n - b * kStCols);
            const uint32_t valid = ncol >= 32 ? 0xffffffffu : (ncol > 0 ? (1u << ncol) - 1u : 0u);
            if (g == 0) {
                // the first block seeds the list: its K largest of 32 values by a bitonic sorting
                // network in registers (240 compare-exchanges, each a min and a max), where inserting
                // all 32 one by one costs 32 passes over the list and a loop step each
                float a[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) a[i] = v[i];
                if (ncol < 32) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) a[i] = i < ncol ? a[i] : -INFINITY;
                }
#pragma unroll
                for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
                    for (int jj = k >> 1; jj > 0; jj >>= 1)
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int l = i ^ jj;
                            if (l > i) {  // descending where bit k of i is clear (k = 32: the whole list)
                                const float hi = fmaxf(a[i], a[l]), lo = fminf(a[i], a[l]);
                                const bool desc = (i & k) == 0;
                                a[i] = desc ? hi : lo;
                                a[l] = desc ? lo : hi;
                            }
                        }
#pragma unroll
                for (int i = 0; i < K; ++i) ls[i] = i < 32 ? a[i] : -INFINITY;
                continue;  // nothing else of the loop body applies to pass 1's first block
            }
            // every score of the block to this thread's column; one bit per candidate
            // the mask is built in four independent parts (no 32-long dependency chain through one register)
            uint32_t mp[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int i = 0; i < 8; ++i)
                reinterpret_cast<float4 *>(cv)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            if (g < nblk) {  // warp-uniform
                const float thr = ls[K - 1];
#pragma unroll
                for (int i = 0; i < 32; ++i) mp[i & 3] |= v[i] > thr ? 1u << i : 0u;
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) mp[i & 3] |= v[i] >= tau ? 1u << i : 0u;
            }
            uint32_t m = ((mp[0] | mp[1]) | (mp[2] | mp[3])) & valid;
            if (g < nblk) {  // pass 1: insert the candidates that still beat the K-th value
                while (m) {
                    const int i = __ffs(m) - 1;
                    m &= m - 1;
                    const float x = cv[i];
                    if (x > ls[K - 1]) {
#pragma unroll
                        for (int j = K - 1; j > 0; --j) ls[j] = fmaxf(ls[j], fminf(ls[j - 1], x));
                        ls[0] = fmaxf(ls[0], x);
                    }
                }
            } else {  // pass 2: take every score > tau and the lowest chunks at tau, in chunk order
                while (m) {
                    const int i = __ffs(m) - 1;
                    m &= m - 1;
                    const float x = cv[i];
                    const bool eq = !(x > tau);
                    if (eq && need_eq <= 0) continue;
                    need_eq -= eq ? 1 : 0;
                    // output slot: after the kept values above x, ties in chunk order
                    // ls[jj] - x is positive exactly when ls[jj] > x (no flush to zero here); times +inf it
                    // saturates to 1, and to 0 when it is zero (the NaN saturates to 0) or negative.
                    // Entries past k_keep are <= tau <= x and add nothing. This runs on the FMA pipe,
                    // which the kernel leaves idle, instead of the ALU pipe that bounds it.
                    float lq[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int jj = 0; jj < K; ++jj) lq[jj & 3] += __saturatef((ls[jj] - x) * INFINITY);
                    const int lo = (int)((lq[0] + lq[1]) + (lq[2] + lq[3]));
                    const uint64_t freeb = ~used & (~0ull << lo);
                    const int slot = __ffsll((long long)freeb) - 1;
                    if (slot < 0 || slot >= k_keep) continue;  // only if pass 2 disagreed with pass 1
                    used |= 1ull << slot;
                    cc[128 * slot] = b * kStCols + i;
                }
            }
        }

        // weights from the sorted values, and the tile's rows staged in shared memory (the landmark
        // stages are free: every MMA has completed)
        asm volatile("bar.sync 1, %0;" ::"n"(kStConsumers) : "memory");
        // rows of kout + 1 entries: a row per thread without shared-memory bank conflicts
        int32_t *st_idx = reinterpret_cast<int32_t *>(s);
        float *st_w = reinterpret_cast<float *>(s) + kStRows * (kout + 1);
        if (tid < nrows) {
            const float top = ls[0];
            float z = 0.0f;
#pragma unroll
            for (int i = 0; i < K; ++i) z += i < k_keep ? expf((ls[i] - top) * scale) : 0.0f;
            const float rz = 1.0f / z;
#pragma unroll
            for (int i = 0; i < K; ++i) {
                if (i >= kout) break;
                const bool u = (used >> i) & 1ull;
                const int c = u ? cc[128 * i] : -1;
                st_idx[tid * (kout + 1) + i] = c;
                st_w[tid * (kout + 1) + i] = u ? expf((ls[i] - top) * scale) * rz : 0.0f;
                if (u) {
                    if (hist_smem) atomicAdd(&s_hist[c], 1);
                    else atomicAdd(&chunk_count[(size_t)bh * N + c], 1);
                }
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kStConsumers) : "memory");
        for (int i = tid; i < nv * kout; i += kStConsumers) {
            const int rr = i / kout, j = i - rr * kout;
            sel_idx[out0 + i] = st_idx[rr * (kout + 1) + j];
            sel_w[out0 + i] = st_w[rr * (kout + 1) + j];
        }
        if (hist_smem)  // the tile's per-chunk counts into the dispatch's histogram
            for (int i = tid; i < n_max; i += kStConsumers)
                if (s_hist[i]) atomicAdd(&chunk_count[(size_t)bh * N + i], s_hist[i]);
        if (!ok && lane == 0) atomicOr(err, 1);
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, kStTmemCols);
    }
}

template <int D, int K>
static cudaError_t launch_st(const ForwardArgs &a, const CUtensorMap &tl, cudaStream_t s) {
    const size_t smem = StSmem<D, K>::DYN;
    cudaError_t e = cudaFuncSetAttribute(score_topk_tc_kernel<D, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.T + kStRows - 1) / kStRows, a.B * a.H);
    HSA_PROF("score_topk", s);
    score_topk_tc_kernel<D, K><<<grid, kStThreads, smem, s>>>(a.Qs, a.T, a.N, a.H / a.Hkv, a.H, a.cu_seqlens,
                                                              a.scale, a.topk,
                                                              a.sel_idx, a.sel_w, a.o_acc, a.chunk_count, a.err, tl);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_st_d(const ForwardArgs &a, cudaStream_t s) {
    CUtensorMap tl;
    // with no complete chunk the landmark tensor may be empty: point the map at Q (never read)
    if (!make_tmap_bf16(&tl, a.N > 0 ? (const void *)a.L : (const void *)a.Q,
                 a.N > 0 ? (uint64_t)a.B * a.Hkv * a.N : (uint64_t)a.B * a.H * a.T, D, kStCols))
        return cudaErrorInvalidValue;
    if (a.topk <= 8) return launch_st<D, 8>(a, tl, s);
    if (a.topk <= 16) return launch_st<D, 16>(a, tl, s);
    if (a.topk <= 32) return launch_st<D, 32>(a, tl, s);
    return launch_st<D, 64>(a, tl, s);
}

cudaError_t launch_score_tc(const ForwardArgs &a, cudaStream_t s) {
    return a.D == 128 ? launch_st_d<128>(a, s) : launch_st_d<64>(a, s);
}

}  // namespace hsa
