// score_wide.cu -- Step 2 (retrieval scores + top-K) and the Step 4 fusion weights of the HSA forward
// for K <= 16, as a persistent kernel on the 5th-generation tensor cores.
//
// Explainer page of "Every Token Counts", "How It Works (Technically)", Step 2: each token t scores
// every chunk that has ended at or before it, s[t,c] = scale * Q[t].L[c], and keeps the top-K; the
// per-token procedure ("The algorithm, simplified") sorts the scores in descending order, stably,
// so equal scores keep the lower chunk first. Step 4: w = softmax of the kept scores.
//
// Work item: 256 consecutive token rows of one (batch, head), as two 128-row tiles that share every
// landmark block. One CTA per SM walks its items: items are ordered longest rows first and dealt to
// the CTAs in snake order (CTA c takes items c, 2G - 1 - c, 2G + c, ...), which evens out their cost.
// In a padded batch (per-sequence lengths) only the items with a row inside their sequence exist.
//   * Warp 16 (loader): TMA copies of each item's two Q tiles into a staging area and of 64-landmark
//     blocks (128-byte swizzle) through a four-stage ring. An item's blocks go through the ring twice
//     (two passes over the row); the next item's Q tiles are copied between the two.
//   * Warp 17 (MMA): S_blk = Q L_blk^T (M = 128, N = 64, fp32) for each tile into one of the tile's two
//     TMEM score buffers. Q is the A operand from TMEM (two bf16 per column), double-buffered by item;
//     the selectors' copies of it are counted in shared memory and the MMA warp waits on the count.
//   * Warps 0-15 (selectors): warp w serves tile w / 8, column half (w / 4) % 2 of every block and the
//     32 rows (w % 4) * 32 .. + 31 (= its TMEM lanes): two threads per token row, one per half.
//       - Each thread copies its half of the row of Q from the staging into TMEM: the next item's while
//         this one runs.
//       - Pass 1 keeps 2K group maxima per row, K per half: group j of a half holds its columns j,
//         j + K, ... of every block (one max per score). They are maxima of disjoint sets of scores, so
//         the K-th largest of all 2K, tau0, has K different chunks at or above it: the row's K-th largest
//         score is at least tau0, and no score below tau0 can be kept. Each half sorts its maxima, the
//         pair swaps them, and tau0 = min_j max(A[j], B[K-1-j]).
//       - Pass 2 (the same products, recomputed: bit-identical) stages each block's scores in shared
//         memory, marks the scores >= tau0 on the FMA pipe, and makes exact 64-bit keys -- ordered
//         score, then lower chunk first -- for those only. Each half keeps its K largest keys (on
//         i.i.d. scores about 1.3 K reach tau0 per row; a half with more keeps its K largest, one by
//         one; ties stay exact: the keys are unique).
//       - Each half sorts its keys (bitonic network in registers), the pair swaps them, and a bitonic
//         merge step gives the row's K largest in order; each thread writes half of the output slots.
//         Scores are compared unscaled (the scale is positive, so the order is the same); the scale
//         enters the fusion weights only.
//   * Warp 18 zeroes the item's rows of the fp32 output accumulator (the chunk attention adds into
//     them) and adds each finished item's pair counts per chunk, which the selectors gather in a
//     per-tile shared-memory histogram, into the dispatch's counts.
// The two warps of a row range meet on their own named barrier; the other hand-offs are mbarriers, each
// waited at every one of its phases in turn, and every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "launch.h"
#include "profile.h"
#include "tc.cuh"

namespace hsa {

constexpr int kSwRows = 128;    // rows per tile (MMA M)
constexpr int kSwItem = 256;    // rows per work item (two tiles)
constexpr int kSwCols = 64;     // landmarks per block (MMA N)
constexpr int kSwStages = 4;    // landmark blocks in shared memory
constexpr int kSwLoaderWarp = 16;  // warps 0-15 select
constexpr int kSwMmaWarp = 17;
constexpr int kSwZeroWarp = 18;
constexpr int kSwThreads = 32 * (kSwZeroWarp + 1);  // 608
constexpr int kSwMaxSeqs = 256;    // padded batches: sequences ordered in shared memory (else every item is dealt)
constexpr int kSwMaxLevels = 1024; // 256-row levels counted in shared memory (T <= 262144)
constexpr int kSwSlot = 32;     // key slot stride: slot j of a lane at [j * 32] of its half's slots
constexpr int kSwHist = 1024;   // chunks per (b, h) counted in shared memory (per tile, two buffers)

template <int D, int K>
struct SwSmem {
    static constexpr int KH = D / 64;                   // 64-column halves of a row
    static constexpr int NG = 2 * K;                    // pass-1 groups and key slots per row (K per half)
    static constexpr uint32_t LH = kSwCols * 128;       // one half of a landmark block: [64 rows][128 B]
    static constexpr uint32_t LB = KH * LH;             // one landmark stage
    static constexpr uint32_t QH = kSwRows * 128;       // one half of a Q tile: [128 rows][128 B]
    static constexpr uint32_t QT = KH * QH;             // one Q tile
    static constexpr uint32_t LST = 0;                  // landmark stages
    static constexpr uint32_t QST = LST + kSwStages * LB;  // Q staging: two tiles
    // u64 keys [pair][half][K][32 lanes]; a pair is the two warps (one per column half) that share 32
    // rows, and its region also holds the swapped group maxima before pass 2
    static constexpr uint32_t PAIR = 2 * K * kSwSlot * 8;
    static constexpr uint32_t CAND = QST + 2 * QT;
    static constexpr uint32_t HIST = CAND + 8 * PAIR;   // int[tile][2 buffers][kSwHist]
    static constexpr uint32_t HIST_BYTES = 4 * kSwHist * 4;
    // l_full[4], l_empty[4], q_sfull[2], q_sempty[2], two unused slots, s_full[2][2], s_empty[2][2],
    // h_full[2][2], h_free[2][2]
    // pass 2's score scratch of each tile, float [32][256 threads]: a tile's Q staging (32 KB at
    // D = 128) is free between the copy of the next item's Q and the end of that tile's pass 2; at
    // D = 64 it is too small and the scratch has its own region
    static constexpr uint32_t SCR_TILE = 32 * 256 * 4;
    static constexpr bool SCR_IN_Q = QT >= SCR_TILE;
    static constexpr uint32_t SCR = SCR_IN_Q ? QST : HIST + HIST_BYTES;
    static constexpr uint32_t SCR_STRIDE = SCR_IN_Q ? QT : SCR_TILE;  // tile u at SCR + u * SCR_STRIDE
    static constexpr uint32_t BAR = SCR_IN_Q ? HIST + HIST_BYTES : SCR + 2 * SCR_TILE;
    // + h_full[tile][buffer], h_free[tile][buffer]
    static constexpr int NBAR = 2 * kSwStages + 6 + 8 + 8;
    static constexpr uint32_t QCNT = BAR + NBAR * 8;     // unsigned[2]: warps' Q copies into TMEM, per tile
    static constexpr uint32_t TMEM = QCNT + 8;
    static constexpr uint32_t SEQ = TMEM + 16;                       // int[kSwMaxSeqs]: sequences by length
    static constexpr uint32_t CUM = SEQ + kSwMaxSeqs * 4;             // int[kSwMaxLevels + 1]: items before a level
    static constexpr uint32_t BYTES = CUM + (kSwMaxLevels + 1) * 4;
    static constexpr size_t DYN = BYTES + 1024;
    static_assert(DYN <= 227 * 1024, "shared memory budget");
    // TMEM columns: Q [item parity][tile] (D/2 each), then S [tile][buffer] (64 each)
    static constexpr uint32_t QC = D / 2;
    static constexpr uint32_t SBASE = 4 * QC;
    static constexpr uint32_t NCOLS = 512;
    static_assert(SBASE + 4 * kSwCols <= NCOLS, "TMEM budget");
};

// The k-th work item of this CTA: rows [t0, t0 + 256) of (batch, head) bh, or none.
struct SwItem {
    int bh, t0;
    bool valid;
};
__device__ __forceinline__ SwItem sw_item(int k, int G, int c, int P, int BH) {
    const int pos = (k & 1) ? G - 1 - c : c;  // snake order over the CTAs
    const long long i = (long long)k * G + pos;
    SwItem it{0, 0, false};
    if (i < (long long)P * BH) {
        const int level = (int)(i / BH);
        it.bh = (int)(i % BH);
        it.t0 = (P - 1 - level) * kSwItem;  // longest rows first
        it.valid = true;
    }
    return it;
}

// The k-th work item of this CTA in a padded batch: only the (sequence, head, 256-row block) items with a
// row inside their sequence exist. s_cum[L] counts the items of the levels before level L (level 0 =
// the longest rows) and s_seq lists the sequences by length, longest first, so the sequences that reach
// a level are a prefix of it; within a level the items go by that order, then by head.
__device__ __forceinline__ SwItem sw_item_seq(int k, int G, int c, int P, int H, const int *s_cum,
                                              const int *s_seq) {
    const int pos = (k & 1) ? G - 1 - c : c;
    const long long i = (long long)k * G + pos;
    SwItem it{0, 0, false};
    if (i >= s_cum[P]) return it;
    int lo = 0, hi = P;  // s_cum[lo] <= i < s_cum[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_cum[mid] <= i) lo = mid;
        else hi = mid;
    }
    const int o = (int)(i - s_cum[lo]);
    it.bh = s_seq[o / H] * H + o % H;
    it.t0 = (P - 1 - lo) * kSwItem;
    it.valid = true;
    return it;
}

// Chunks that the last valid row of [r0, r0 + n) sees (0 when no row of it is valid).
__device__ __forceinline__ int sw_nmax(int r0, int n, int Tv, int N) {
    const int tl = min(r0 + n - 1, Tv - 1);
    return tl >= r0 ? min(N, (tl + 1) / kChunk) : 0;
}

// This half's key slots once more than K keys have reached tau0: the K largest so far are kept (slot j
// at buf[j * kSwSlot]); kmin is the smallest of them and kslot its slot (kmin 0: not yet computed -- valid
// keys are never 0). Rare: only rows whose half has more than K scores at or above tau0.
struct SwHalf {
    int cnt;
    uint64_t kmin;
    int kslot;
};
template <int K>
__device__ __noinline__ SwHalf sw_keep_slow(const float *v, int sw, uint32_t m, int c0, uint64_t *buf, SwHalf h) {
    // v: this thread's 128-byte scratch row, 16-byte chunk q at chunk q ^ sw
    if (h.cnt == K && h.kmin == 0ull) {  // filled to exactly K by the fast path: the minimum is not known yet
        h.kmin = buf[0];
        h.kslot = 0;
        for (int j = 1; j < K; ++j) {
            const uint64_t x = buf[j * kSwSlot];
            if (x < h.kmin) {
                h.kmin = x;
                h.kslot = j;
            }
        }
    }
    while (m) {
        const int i = __ffs(m) - 1;
        m &= m - 1;
        const uint64_t key = make_key(v[(((i >> 2) ^ sw) << 2) + (i & 3)], (uint32_t)(c0 + i));
        if (h.cnt < K) {
            buf[h.cnt * kSwSlot] = key;
            if (++h.cnt < K) continue;
        } else {
            if (key <= h.kmin) continue;
            buf[h.kslot * kSwSlot] = key;
        }
        h.kmin = buf[0];  // the full slots' minimum
        h.kslot = 0;
        for (int j = 1; j < K; ++j) {
            const uint64_t x = buf[j * kSwSlot];
            if (x < h.kmin) {
                h.kmin = x;
                h.kslot = j;
            }
        }
    }
    return h;
}

// Named barrier over n threads that also ANDs a predicate across them.
__device__ __forceinline__ bool bar_and(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0u;
}

template <int D, int K>
__global__ void __launch_bounds__(kSwThreads, 1) score_topk_wide_kernel(
    int T, int N, int Gh, int H, int BH, const int32_t *__restrict__ cu_seqlens, float scale, int kout,
    int32_t *__restrict__ sel_idx, float *__restrict__ sel_w, float *__restrict__ o_acc,
    int32_t *__restrict__ chunk_count, int32_t *__restrict__ err, const __grid_constant__ CUtensorMap tmQ,
    const __grid_constant__ CUtensorMap tmL) {
    pdl_launch_dependents();  // the dispatch's scan may be scheduled (it waits for this grid)
    using SM = SwSmem<D, K>;
    constexpr int KH = SM::KH;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    unsigned char *s = smem_raw + (sb - raw);
    auto bar = [&](int i) { return sb + SM::BAR + 8u * (uint32_t)i; };
    auto l_full = [&](int st) { return bar(st); };
    auto l_empty = [&](int st) { return bar(kSwStages + st); };
    auto q_sfull = [&](int u) { return bar(2 * kSwStages + u); };
    auto q_sempty = [&](int u) { return bar(2 * kSwStages + 2 + u); };
    // the selectors' copies of an item's Q into TMEM are counted in q_cnt[tile] (8 per item), not on an
    // mbarrier: the MMA warp waits only for items whose tile has products, and a phase-parity wait that
    // skips items can pass two phases early; a count cannot
    unsigned *q_cnt = reinterpret_cast<unsigned *>(s + SM::QCNT);
    auto s_full = [&](int u, int b) { return bar(2 * kSwStages + 6 + 2 * u + b); };
    auto s_empty = [&](int u, int b) { return bar(2 * kSwStages + 10 + 2 * u + b); };
    auto h_full = [&](int u, int b) { return bar(2 * kSwStages + 14 + 2 * u + b); };
    auto h_free = [&](int u, int b) { return bar(2 * kSwStages + 18 + 2 * u + b); };
    // pair counts per chunk of an item, per tile, double-buffered by item: the selectors add, the zero
    // warp adds the buffer into the dispatch's counts and clears it
    auto hist = [&](int u, int b) { return reinterpret_cast<int *>(s + SM::HIST) + (2 * u + b) * kSwHist; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x, cta = blockIdx.x;
    const int P = (T + kSwItem - 1) / kSwItem;
    auto seq_len = [&](int bh) { return cu_seqlens ? min(T, cu_seqlens[bh / H + 1] - cu_seqlens[bh / H]) : T; };
    // padded batches: deal only the items with a row inside their sequence (tables built below)
    const int nseq = BH / H;
    const bool by_seq = cu_seqlens != nullptr && nseq <= kSwMaxSeqs && P <= kSwMaxLevels;
    int *s_seq = reinterpret_cast<int *>(s + SM::SEQ);
    int *s_cum = reinterpret_cast<int *>(s + SM::CUM);
    auto item_of = [&](int k) {
        return by_seq ? sw_item_seq(k, G, cta, P, H, s_cum, s_seq) : sw_item(k, G, cta, P, BH);
    };

    for (int i = tid; i < 4 * kSwHist; i += kSwThreads) hist(0, 0)[i] = 0;
    if (by_seq) {
        auto len = [&](int b) { return max(0, min(T, cu_seqlens[b + 1] - cu_seqlens[b])); };
        for (int b = tid; b < nseq; b += kSwThreads) {  // rank by length, longest first (ties: lower index)
            const int lb = len(b);
            int rank = 0;
            for (int b2 = 0; b2 < nseq; ++b2) {
                const int l2 = len(b2);
                rank += (l2 > lb || (l2 == lb && b2 < b)) ? 1 : 0;
            }
            s_seq[rank] = b;
        }
        for (int L = tid; L < P; L += kSwThreads) {  // sequences with a row at or past the level's first row
            const int t0 = (P - 1 - L) * kSwItem;
            int n = 0;
            for (int b2 = 0; b2 < nseq; ++b2) n += len(b2) > t0 ? 1 : 0;
            s_cum[L + 1] = n * H;
        }
        __syncthreads();
        if (warp == 0) {  // prefix sum over the levels: lane l sums its consecutive run, then a warp scan
            const int per = (P + 31) / 32, l0 = lane * per;
            int run = 0;
            for (int L = l0; L < min(P, l0 + per); ++L) run += s_cum[L + 1];
            int incl = run;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int x = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += x;
            }
            int acc = incl - run;  // items of the levels before this lane's run
            if (lane == 0) s_cum[0] = 0;
            for (int L = l0; L < min(P, l0 + per); ++L) {
                acc += s_cum[L + 1];
                s_cum[L + 1] = acc;
            }
        }
    }
    if (warp == kSwMmaWarp) tc::tmem_alloc(sb + SM::TMEM, SM::NCOLS);
    if (tid == 0) {
        for (int i = 0; i < kSwStages; ++i) {
            tc::mbar_init(l_full(i), 1);
            tc::mbar_init(l_empty(i), 1);
        }
        for (int u = 0; u < 2; ++u) {
            tc::mbar_init(q_sfull(u), 1);
            tc::mbar_init(q_sempty(u), 8);
            q_cnt[u] = 0u;
            for (int b = 0; b < 2; ++b) {
                tc::mbar_init(s_full(u, b), 1);
                tc::mbar_init(s_empty(u, b), 8);
                tc::mbar_init(h_full(u, b), 8);
                tc::mbar_init(h_free(u, b), 1);
            }
        }
        tc::fence_mbar_init();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<uint32_t *>(s + SM::TMEM);
    bool ok = true;

    if (warp == kSwLoaderWarp) {
        // ---------------- loader: the whole warp runs it, one elected lane issues (tc::*_w) ----------------
        uint32_t h = 0;     // landmark blocks issued
        int nq = 0;         // Q items issued
        auto load_q = [&](const SwItem &it) {
            for (int u = 0; u < 2 && ok; ++u) {
                if (nq >= 1) ok = tc::mbar_wait(q_sempty(u), (uint32_t)(nq - 1) & 1u);  // the previous item copied
                if (!ok) break;
                tc::mbar_arrive_expect_tx_w(q_sfull(u), SM::QT);
#pragma unroll
                for (int k = 0; k < KH; ++k)
                    tc::tma_load_2d_w(sb + SM::QST + u * SM::QT + k * SM::QH, &tmQ, k * 64,
                                      it.bh * T + it.t0 + u * kSwRows, q_sfull(u));
            }
            ++nq;
        };
        auto load_l = [&](int kvh, int blk) {
            const int st = (int)(h % kSwStages);
            if (h >= kSwStages) ok = ok && tc::mbar_wait(l_empty(st), (uint32_t)(h / kSwStages - 1) & 1u);
            if (!ok) return;
            tc::mbar_arrive_expect_tx_w(l_full(st), SM::LB);
#pragma unroll
            for (int k = 0; k < KH; ++k)
                tc::tma_load_2d_w(sb + SM::LST + st * SM::LB + k * SM::LH, &tmL, k * 64, kvh * N + blk * kSwCols,
                                  l_full(st));
            ++h;
        };
        SwItem it = item_of(0);
        if (it.valid) load_q(it);
        for (int k = 0; it.valid && ok; ++k) {
            const int nblk = (sw_nmax(it.t0, kSwItem, seq_len(it.bh), N) + kSwCols - 1) / kSwCols;
            const int kvh = it.bh / Gh;
            for (int b = 0; b < nblk && ok; ++b) load_l(kvh, b);  // pass 1
            const SwItem nx = item_of(k + 1);
            if (nx.valid && ok) load_q(nx);
            for (int b = 0; b < nblk && ok; ++b) load_l(kvh, b);  // pass 2
            it = nx;
        }
        if (!ok) {  // every copy this CTA started lands before its shared memory goes away
            for (uint32_t i = (h > kSwStages ? h - kSwStages : 0); i < h; ++i)
                tc::mbar_wait(l_full((int)(i % kSwStages)), (uint32_t)(i / kSwStages) & 1u);
            if (nq > 0)
                for (int u = 0; u < 2; ++u) tc::mbar_wait(q_sfull(u), (uint32_t)(nq - 1) & 1u);
        }
        __syncwarp();
    } else if (warp == kSwMmaWarp) {
        // ---------------- MMA issuer: the whole warp runs it, one elected lane issues ----------------
        constexpr uint32_t idesc = tc::idesc_bf16(kSwRows, kSwCols, 0, 0);
        uint32_t h = 0, g[2] = {0, 0};
        SwItem it = item_of(0);
        for (int k = 0; it.valid && ok; ++k) {
            const int Tv = seq_len(it.bh);
            const int nb0 = (sw_nmax(it.t0, kSwRows, Tv, N) + kSwCols - 1) / kSwCols;
            const int nb1 = (sw_nmax(it.t0 + kSwRows, kSwRows, Tv, N) + kSwCols - 1) / kSwCols;
            const int nblk = max(nb0, nb1);
            // the item's Q in TMEM, for the tiles that have products: all 8 warps of the tile have copied
            // items 0 .. k (bounded wait on the count, acquire)
            for (int u = 0; u < 2 && ok; ++u) {
                if ((u ? nb1 : nb0) == 0) continue;
                const unsigned target = 8u * (unsigned)(k + 1);
                uint32_t probe = 0;
                for (;;) {
                    unsigned c;
                    asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(c) : "r"(smem_u32(&q_cnt[u])) : "memory");
                    if (c >= target) break;
                    if (++probe > (1u << 24)) {
                        ok = false;
                        break;
                    }
                    __nanosleep(32);
                }
            }
            tc::fence_after();
            for (int pass = 0; pass < 2 && ok; ++pass) {
                for (int b = 0; b < nblk && ok; ++b) {
                    const int st = (int)(h % kSwStages);
                    ok = tc::mbar_wait(l_full(st), (uint32_t)(h / kSwStages) & 1u);
                    if (!ok) break;
                    tc::fence_after();
                    const uint32_t lb = sb + SM::LST + st * SM::LB;
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        if (b >= (u ? nb1 : nb0)) continue;
                        const int buf = (int)(g[u] & 1u);
                        if (g[u] >= 2 && !tc::mbar_wait(s_empty(u, buf), ((g[u] >> 1) - 1) & 1u)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after();
                        const uint32_t dq = tmem + (uint32_t)((2 * (k & 1) + u) * SM::QC);
                        const uint32_t ds = tmem + SM::SBASE + (uint32_t)((2 * u + buf) * kSwCols);
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks)  // K step of 16: 8 TMEM columns of Q, 32 B of a swizzled row
                            tc::mma_bf16_ts_w(ds, dq + ks * 8, tc::desc_kmajor(lb + (ks >> 2) * SM::LH + (ks & 3) * 32),
                                              idesc, ks > 0 ? 1u : 0u);
                        tc::commit_w(s_full(u, buf));
                        ++g[u];
                    }
                    tc::commit_w(l_empty(st));
                    ++h;
                }
            }
            it = item_of(k + 1);
        }
        if (!ok) {  // the products in flight complete before TMEM is released
            for (int u = 0; u < 2; ++u)
                if (g[u] > 0) tc::mbar_wait(s_full(u, (int)((g[u] - 1) & 1u)), ((g[u] - 1) >> 1) & 1u);
        }
        // the last stage release has landed before the CTA's shared memory goes away
        if (h > 0) tc::mbar_wait(l_empty((int)((h - 1) % kSwStages)), ((h - 1) / kSwStages) & 1u);
        __syncwarp();
    } else if (warp == kSwZeroWarp) {
        // ---------------- the items' rows of the fp32 output accumulator start at zero ----------------
        // it also adds each finished item's per-chunk pair counts into the dispatch's counts, one item
        // behind the zeroing
        auto flush = [&](int kk, const SwItem &f) {
            const int nmax = min(kSwHist, sw_nmax(f.t0, kSwItem, seq_len(f.bh), N));
            for (int u = 0; u < 2 && ok; ++u) {
                ok = tc::mbar_wait(h_full(u, kk & 1), (uint32_t)(kk >> 1) & 1u);
                if (!ok) break;
                int *hb = hist(u, kk & 1);
                for (int i = lane; i < nmax; i += 32) {
                    const int x = hb[i];
                    if (x) {
                        atomicAdd(&chunk_count[(size_t)f.bh * N + i], x);
                        hb[i] = 0;
                    }
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(h_free(u, kk & 1));
            }
        };
        SwItem it = item_of(0), prev{0, 0, false};
        int k = 0;
        for (; it.valid && ok; ++k) {
            const int nv = max(0, min(kSwItem, min(T, seq_len(it.bh)) - it.t0));
            float4 *acc = reinterpret_cast<float4 *>(o_acc + ((size_t)it.bh * T + it.t0) * D);
            for (int i = lane; i < nv * (D / 4); i += 32) acc[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (k > 0) flush(k - 1, prev);
            prev = it;
            it = item_of(k + 1);
        }
        if (ok && k > 0) flush(k - 1, prev);
    } else {
        // ---------------- selectors: tile u, column half hf of each block, one token row per thread pair ----------------
        const int u = warp >> 3, hf = (warp >> 2) & 1, r = (warp & 3) * 32 + lane;
        const int pair = u * 4 + (warp & 3);
        const int bar_pair = 1 + pair;  // named barrier of the two warps of this row range (64 threads)
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        // the pair's region: this half's K key slots (slot j at [j * 32]) and the partner's; before pass
        // 2 the same bytes hold the swapped, sorted group maxima (float, j at [j * 32]). Only the pair
        // touches its region, so two named-barrier steps of the pair order every access.
        unsigned char *preg = s + SM::CAND + pair * SM::PAIR;
        uint64_t *kb = reinterpret_cast<uint64_t *>(preg) + hf * K * kSwSlot + lane;
        const uint64_t *kb_o = reinterpret_cast<const uint64_t *>(preg) + (hf ^ 1) * K * kSwSlot + lane;
        float *gx = reinterpret_cast<float *>(preg) + hf * K * kSwSlot + lane;
        const float *gx_o = reinterpret_cast<const float *>(preg) + (hf ^ 1) * K * kSwSlot + lane;
        uint32_t gs = 0;  // score blocks taken so far
        // this thread's half of the row of Q of item kk from the staging into TMEM (item parity kk & 1)
        auto copy_q = [&](int kk, bool release) -> bool {
            if (!__all_sync(0xffffffffu, tc::mbar_wait(q_sfull(u), (uint32_t)kk & 1u))) return false;
            const unsigned char *src = s + SM::QST + u * SM::QT;
            const uint32_t tq = tmem + lane_off + (uint32_t)((2 * (kk & 1) + u) * SM::QC);
            if constexpr (D == 128) {  // the 64-column half hf: 8 chunks of 16 B, 32 TMEM columns
                uint32_t q32[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(src + hf * SM::QH + tc::sw128(r, i));
                    q32[4 * i] = x.x;
                    q32[4 * i + 1] = x.y;
                    q32[4 * i + 2] = x.z;
                    q32[4 * i + 3] = x.w;
                }
                tc::tmem_st32(tq + hf * 32, q32);
            } else {  // chunks 4 hf .. 4 hf + 3 of the one half: 16 TMEM columns
                uint32_t q16[16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 x = *reinterpret_cast<const uint4 *>(src + tc::sw128(r, 4 * hf + i));
                    q16[4 * i] = x.x;
                    q16[4 * i + 1] = x.y;
                    q16[4 * i + 2] = x.z;
                    q16[4 * i + 3] = x.w;
                }
                tc::tmem_st16(tq + hf * 16, q16);
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) {
                asm volatile("red.release.cta.shared::cta.add.u32 [%0], 1;" ::"r"(smem_u32(&q_cnt[u])) : "memory");
                if (release) tc::mbar_arrive(q_sempty(u));
            }
            return true;
        };
        auto get_block = [&](float (&v)[32]) -> bool {
            const int buf = (int)(gs & 1u);
            if (!__all_sync(0xffffffffu, tc::mbar_wait(s_full(u, buf), (gs >> 1) & 1u))) return false;
            tc::fence_after();
            tc::tmem_ld32(tmem + lane_off + SM::SBASE + (uint32_t)((2 * u + buf) * kSwCols + 32 * hf), v);
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(s_empty(u, buf));  // the scores are in registers now
            ++gs;
            return true;
        };

        SwItem it = item_of(0);
        if (it.valid) ok = copy_q(0, true);
        // this thread's scores in its tile's scratch: one 128-byte row, its 16-byte chunks XOR-swizzled by
        // (row % 8) so that a warp's 16-byte stores do not conflict; column i at scr_at(i)
        const int tt = tid & 255;
        unsigned char *scr = s + SM::SCR + u * SM::SCR_STRIDE + tt * 128;
        auto scr_at = [&](int i) { return reinterpret_cast<float *>(scr + (((i >> 2) ^ (tt & 7)) << 4)) + (i & 3); };
        // every barrier of an item is reached whatever happened: a failed wait skips the remaining waits
        // of the item, and at its end the selectors agree on the outcome and stop together
        for (int k = 0; it.valid; ++k) {
            const int Tv = seq_len(it.bh);
            const int t = it.t0 + u * kSwRows + r;
            const int my_n = t < Tv ? min(N, (t + 1) / kChunk) : 0;
            const int k_keep = min(kout, my_n);
            const int nbu = (sw_nmax(it.t0 + u * kSwRows, kSwRows, Tv, N) + kSwCols - 1) / kSwCols;
            // a tile with no row inside its sequence (padded batches) skips the sorting networks; it still
            // takes part in every hand-off and barrier of the item (the condition is the same for the pair)
            const bool live = it.t0 + u * kSwRows < min(T, Tv);
            float v[32];

            // pass 1: this half's K group maxima; group j takes columns j, j + K, .. of the half
            float gm[K];
#pragma unroll
            for (int j = 0; j < K; ++j) gm[j] = -INFINITY;
            for (int b = 0; b < nbu && ok; ++b) {
                if (!get_block(v)) {
                    ok = false;
                    break;
                }
                const int valid = my_n - b * kSwCols - 32 * hf;
                if (valid < 32) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = i < valid ? v[i] : -INFINITY;
                }
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    float m = v[j];
#pragma unroll
                    for (int q = 1; q < 32 / K; ++q) m = fmaxf(m, v[j + q * K]);
                    gm[j] = fmaxf(gm[j], m);
                }
            }
            // tau0 = the K-th largest of the row's 2K group maxima: both halves sort theirs (descending
            // bitonic network), swap them through shared memory, and the K largest of the union are
            // max(A[j], B[K-1-j]) (a bitonic merge step), whose minimum is tau0. With n <= K every score
            // is kept.
            if (live) {
#pragma unroll
                for (int kk = 2; kk <= K; kk <<= 1)
#pragma unroll
                    for (int jj = kk >> 1; jj > 0; jj >>= 1)
#pragma unroll
                        for (int i = 0; i < K; ++i) {
                            const int l = i ^ jj;
                            if (l > i) {
                                const float hi = fmaxf(gm[i], gm[l]), lo = fminf(gm[i], gm[l]);
                                const bool desc = (i & kk) == 0;
                                gm[i] = desc ? hi : lo;
                                gm[l] = desc ? lo : hi;
                            }
                        }
            }
#pragma unroll
            for (int j = 0; j < K; ++j) gx[j * kSwSlot] = gm[j];
            asm volatile("bar.sync %0, 64;" ::"r"(bar_pair) : "memory");
            float tmin = INFINITY;
#pragma unroll
            for (int j = 0; j < K; ++j) tmin = fminf(tmin, fmaxf(gm[j], gx_o[(K - 1 - j) * kSwSlot]));
            const float tau0 = my_n > K ? tmin : -INFINITY;
            // the next item's Q into TMEM, while this one's second pass runs
            const SwItem nx = item_of(k + 1);
            if (ok && nx.valid && !copy_q(k + 1, false)) ok = false;
            // the partner has read these maxima before the key slots reuse them (pass 2's scratch is this
            // thread's own part of the staging: the 16-byte chunks of its own row of Q, just copied)
            asm volatile("bar.sync %0, 64;" ::"r"(bar_pair) : "memory");

            // pass 2: this half's K largest keys among the scores >= tau0
            SwHalf hs{0, 0ull, 0};
            for (int b = 0; b < nbu && ok; ++b) {
                if (!get_block(v)) {
                    ok = false;
                    break;
                }
                const int valid = my_n - b * kSwCols - 32 * hf;
                // the scores to the scratch (a key is made only for the candidates, read back from there)
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<float4 *>(scr + ((q ^ (tt & 7)) << 4)) =
                        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                // one bit per candidate (v >= tau0), built on the FMA pipe: (tau0 - v) * inf saturates to 1
                // exactly when tau0 > v (0 * inf is NaN, which saturates to 0: ties are candidates), and
                // the bits are summed as exact integers in two floats
                float mf[2] = {65535.0f, 65535.0f};
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    mf[i >> 4] = fmaf(-__saturatef((tau0 - v[i]) * INFINITY), (float)(1u << (i & 15)), mf[i >> 4]);
                uint32_t m = (uint32_t)mf[0] | ((uint32_t)mf[1] << 16);
                m &= valid >= 32 ? 0xffffffffu : (valid > 0 ? (1u << valid) - 1u : 0u);
                if (m == 0u) continue;
                const int c0 = b * kSwCols + 32 * hf;
                if (hs.cnt + __popc(m) <= K) {
                    int pos = hs.cnt;
                    while (m) {
                        const int i = __ffs(m) - 1;
                        m &= m - 1;
                        kb[(pos++) * kSwSlot] = make_key(*scr_at(i), (uint32_t)(c0 + i));
                    }
                    hs.cnt = pos;
                } else {
                    hs = sw_keep_slow<K>(reinterpret_cast<const float *>(scr), tt & 7, m, c0, kb, hs);
                }
            }

            // the staging (pass 2's scratch) may take the item after next's Q now: the scratch stores are
            // ordered before the copy engine's writes
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && nx.valid) tc::mbar_arrive(q_sempty(u));
            // the row's selection: each half sorts its keys, the halves swap them, and the K largest of
            // the union come out of one bitonic merge (both threads of the row hold all K)
            uint64_t a[K];
#pragma unroll
            for (int j = 0; j < K; ++j) a[j] = j < hs.cnt ? kb[j * kSwSlot] : 0ull;
            if (live) {
#pragma unroll
                for (int kk = 2; kk <= K; kk <<= 1)
#pragma unroll
                    for (int jj = kk >> 1; jj > 0; jj >>= 1)
#pragma unroll
                        for (int i = 0; i < K; ++i) {
                            const int l = i ^ jj;
                            if (l > i) {
                                const uint64_t hi = a[i] > a[l] ? a[i] : a[l], lo = a[i] > a[l] ? a[l] : a[i];
                                const bool desc = (i & kk) == 0;
                                a[i] = desc ? hi : lo;
                                a[l] = desc ? lo : hi;
                            }
                        }
#pragma unroll
                for (int j = 0; j < K; ++j) kb[j * kSwSlot] = a[j];
            }
            asm volatile("bar.sync %0, 64;" ::"r"(bar_pair) : "memory");
            if (live) {
#pragma unroll
                for (int j = 0; j < K; ++j) {
                    const uint64_t o = kb_o[(K - 1 - j) * kSwSlot];
                    a[j] = a[j] > o ? a[j] : o;
                }
#pragma unroll
                for (int jj = K >> 1; jj > 0; jj >>= 1)
#pragma unroll
                    for (int i = 0; i < K; ++i) {
                        const int l = i ^ jj;
                        if (l > i) {
                            const uint64_t hi = a[i] > a[l] ? a[i] : a[l], lo = a[i] > a[l] ? a[l] : a[i];
                            a[i] = hi;
                            a[l] = lo;
                        }
                    }
            }
            // the item's histogram buffer was added in by the zero warp two items ago
            int *hb = hist(u, k & 1);
            if (ok && k >= 2 && !__all_sync(0xffffffffu, tc::mbar_wait(h_free(u, k & 1), (uint32_t)((k >> 1) - 1) & 1u)))
                ok = false;
            if (ok && t < min(T, Tv)) {
                // fusion weights (Step 4): softmax of the kept scores, fp32, max-subtracted; this thread
                // writes slots K/2 hf .. K/2 hf + K/2 - 1
                const float top = k_keep > 0 ? key_score(a[0]) : 0.0f;
                float e[K];
                float z = 0.0f;
#pragma unroll
                for (int i = 0; i < K; ++i) {
                    e[i] = i < k_keep ? expf((key_score(a[i]) - top) * scale) : 0.0f;
                    z += e[i];
                }
                const float rz = k_keep > 0 ? 1.0f / z : 0.0f;
                int32_t *oi = sel_idx + ((size_t)it.bh * T + t) * kout;
                float *ow = sel_w + ((size_t)it.bh * T + t) * kout;
                int ci[K / 2];
                float wi[K / 2];
#pragma unroll
                for (int i = 0; i < K / 2; ++i) {
                    const int sl = hf * (K / 2) + i;
                    const bool kept = sl < k_keep;
                    // both candidates by a static index (a run-time index would put a and e in local memory)
                    const uint64_t ak = hf ? a[K / 2 + i] : a[i];
                    const float ek = hf ? e[K / 2 + i] : e[i];
                    ci[i] = kept ? key_index(ak) : -1;
                    wi[i] = kept ? ek * rz : 0.0f;
                    if (kept) {
                        if (ci[i] < kSwHist) atomicAdd(&hb[ci[i]], 1);
                        else atomicAdd(&chunk_count[(size_t)it.bh * N + ci[i]], 1);
                    }
                }
                if (kout == K) {  // rows of K entries: 16-byte stores
#pragma unroll
                    for (int i = 0; i < K / 8; ++i) {
                        reinterpret_cast<int4 *>(oi + hf * (K / 2))[i] =
                            make_int4(ci[4 * i], ci[4 * i + 1], ci[4 * i + 2], ci[4 * i + 3]);
                        reinterpret_cast<float4 *>(ow + hf * (K / 2))[i] =
                            make_float4(wi[4 * i], wi[4 * i + 1], wi[4 * i + 2], wi[4 * i + 3]);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < K / 2; ++i) {
                        const int sl = hf * (K / 2) + i;
                        if (sl < kout) {
                            oi[sl] = ci[i];
                            ow[sl] = wi[i];
                        }
                    }
                }
            }
            // this warp's counts are in: the zero warp may add the buffer once all 8 warps of the tile are
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(h_full(u, k & 1));
            // the pair agrees on the outcome and stops together (its named barriers stay matched)
            ok = bar_and(bar_pair, 64, ok);
            if (!ok) break;
            it = nx;
        }
    }
    if (!ok) atomicOr(err, 1);
    tc::fence_before();
    __syncthreads();
    if (warp == kSwMmaWarp) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, SM::NCOLS);
    }
}

template <int D, int K>
static cudaError_t launch_sw(const ForwardArgs &a, const CUtensorMap &tq, const CUtensorMap &tl, cudaStream_t s) {
    const size_t smem = SwSmem<D, K>::DYN;
    cudaError_t e = cudaFuncSetAttribute(score_topk_wide_kernel<D, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int BH = a.B * a.H;
    const long long items = (long long)((a.T + kSwItem - 1) / kSwItem) * BH;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = items < sms ? (int)items : sms;
    if (grid <= 0) return cudaSuccess;
    HSA_PROF("score_topk", s);
    score_topk_wide_kernel<D, K><<<grid, kSwThreads, smem, s>>>(a.T, a.N, a.H / a.Hkv, a.H, BH, a.cu_seqlens,
                                                                a.scale, a.topk, a.sel_idx, a.sel_w, a.o_acc,
                                                                a.chunk_count, a.err, tq, tl);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_sw_d(const ForwardArgs &a, cudaStream_t s) {
    CUtensorMap tq, tl;
    if (!make_tmap_bf16(&tq, a.Qs, (uint64_t)a.B * a.H * a.T, D, kSwRows)) return cudaErrorInvalidValue;
    // with no complete chunk the landmark tensor may be empty: point the map at Q (never read)
    if (!make_tmap_bf16(&tl, a.N > 0 ? (const void *)a.L : (const void *)a.Qs,
                        a.N > 0 ? (uint64_t)a.B * a.Hkv * a.N : (uint64_t)a.B * a.H * a.T, D, kSwCols))
        return cudaErrorInvalidValue;
    if (a.topk <= 8) return launch_sw<D, 8>(a, tq, tl, s);
    return launch_sw<D, 16>(a, tq, tl, s);
}

cudaError_t launch_score_wide(const ForwardArgs &a, cudaStream_t s) {
    if (a.topk > 16) return cudaErrorInvalidValue;
    return a.D == 128 ? launch_sw_d<128>(a, s) : launch_sw_d<64>(a, s);
}

}  // namespace hsa
