// decode.cu -- HSA decode: one query token per sequence against a long KV/landmark cache.
//
// Explainer page of "Every Token Counts", "How It Works (Technically)": the token scores every
// complete chunk's landmark (Step 2), keeps the top-K, attends inside each kept chunk (Step 3) and
// blends by the softmax of the kept scores (Step 4). With a 1M-16M token cache the landmark scan is
// the whole cost (hundreds of MiB streamed per step), so it is split over chunk ranges:
//
//   decode_scan_kernel     grid (splits, B*H). Streams its range of landmarks with 16-byte
//                          coalesced loads (D/8 lanes per landmark), keeps the exact top-K of the
//                          range (block radix select on unique 64-bit keys), writes K candidates.
//                          The last CTA of each (b, h) to finish (atomic ticket, no waiting) merges
//                          the candidates of all ranges exactly and writes sel_idx / sel_w.
//   decode_attend_kernel   grid (K, B*H*Tq). One CTA per selected chunk: 64 logits, softmax, P.V_c;
//                          the last CTA of each query row blends the K chunk outputs and writes out.
//
// When several query rows read the same landmarks (grouped key/value heads, several query tokens per
// step) and K <= 32, the scan is the grouped one instead:
//   decode_scan_group_kernel  grid (ranges, B*Hkv, row groups of 16). Bulk-copied landmark sub-blocks,
//                          tensor-core scores for 16 rows at a time, one selector warp per row keeping
//                          a running exact top K; writes K candidates per row and range.
//   decode_merge_kernel    grid (B*H*Tq). The exact merge of one row's range candidates.
#include "common.cuh"
#include "launch.h"
#include "profile.h"
#include "tc.cuh"

namespace hsa {

constexpr int kDecodeThreads = 256;

// The rank select below does O(n) dependent shared-memory compares per key: faster than the radix
// select for a few dozen keys (the filtered merge), slower for hundreds (measured on B200).
constexpr int kRankSelectMax = 128;

// Top K of n <= 2 * blockDim keys (nonzero keys unique; 0 = empty), written to out[0..K) in descending
// order with 0 in the slots nothing fills; returns K (the caller treats 0 as empty). A nonzero key's
// rank is the number of keys above it, which for unique keys is its position in the descending order:
// selection and sort in one pass, O(n) compares per key.
__device__ inline int block_topk_rank(const uint64_t *keys, int n, int K, uint64_t *out) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    for (int i = tid; i < K; i += nthr) out[i] = 0ull;
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = tid + h * nthr;
        if (i < n) {
            const uint64_t k = keys[i];
            int rank = 0;
            for (int j = 0; j < n; ++j) rank += keys[j] > k ? 1 : 0;
            if (k != 0ull && rank < K) out[rank] = k;
        }
    }
    __syncthreads();
    return K;
}

// Compacts, in place and in order-free fashion, the keys[0..n) that are >= tau to the front; returns
// their number. Rounds of 4 x blockDim keys are read whole before any slot is written, and the kept
// count never passes the end of what has been read, so no unread key is overwritten. Uses misc[5].
__device__ inline int compact_at_least(uint64_t *keys, int n, uint64_t tau, int *misc) {
    const int tid = threadIdx.x, lane = tid & 31;
    if (tid == 0) misc[5] = 0;
    __syncthreads();
    constexpr int PER = 4;
    const int round = PER * (int)blockDim.x;
    for (int r0 = 0; r0 < n; r0 += round) {
        uint64_t mine[PER];
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const int i = r0 + r * (int)blockDim.x + tid;
            mine[r] = i < n ? keys[i] : 0ull;
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < PER; ++r) {
            const bool keep = mine[r] != 0ull && mine[r] >= tau;
            const unsigned bal = __ballot_sync(0xffffffffu, keep);
            int pos0 = 0;
            if (lane == 0 && bal) pos0 = atomicAdd(&misc[5], __popc(bal));
            pos0 = __shfl_sync(0xffffffffu, pos0, 0);
            if (keep) keys[pos0 + __popc(bal & ((1u << lane) - 1u))] = mine[r];
        }
        __syncthreads();
    }
    const int kept = misc[5];
    __syncthreads();
    return kept;
}

// Exact merge of the per-range candidates of one (b, h): all[r * K + j] holds range r's top K in
// descending order (0 = empty). Writes the head's selection (sel_idx_h[0..K), descending score, -1
// padding) and its fusion weights (Step 4, softmax of the kept scores; 0 padding). Block-wide; keys
// holds at least nsplit * K entries, topk and sorted 64 each, hist 256, misc 8.
__device__ void merge_ranges(const uint64_t *all, int nsplit, int K, uint64_t *keys, uint64_t *topk,
                             uint64_t *sorted, uint32_t *hist, int *misc, int32_t *sel_idx_h, float *sel_w_h) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ncand = nsplit * K;
#pragma unroll 8
    for (int i = tid; i < ncand; i += kDecodeThreads)
        keys[i] = __ldcg(reinterpret_cast<const unsigned long long *>(all) + i);
    __syncthreads();
    // Each range contributed its top K in descending order. The K-th largest of the range maxima, tau,
    // has K ranges with a key at or above it, so no candidate below tau can be in the top K.
    int nmerge = ncand;
    if (nsplit > K && nsplit <= 2 * kDecodeThreads) {
        unsigned long long *tau_s = reinterpret_cast<unsigned long long *>(topk);  // scratch until selection
        if (tid == 0) *tau_s = 0ull;  // stays 0 (keep every nonzero key) if fewer than K maxima are nonzero
        __syncthreads();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = tid + h * kDecodeThreads;
            if (r < nsplit) {
                const uint64_t mr = keys[r * K];
                int rank = 0;
                for (int q = 0; q < nsplit; ++q) rank += keys[q * K] > mr ? 1 : 0;
                if (rank == K - 1 && mr != 0ull) *tau_s = mr;  // unique nonzero keys: at most one range
            }
        }
        __syncthreads();
        const uint64_t tau = *tau_s;
        nmerge = compact_at_least(keys, ncand, tau == 0ull ? 1ull : tau, misc);
    }
    int m;
    if (nmerge <= kRankSelectMax) {
        m = block_topk_rank(keys, nmerge, K, sorted);
    } else {
        m = block_topk_u64(keys, nmerge, K, topk, hist, misc);
        block_sort_desc_small(topk, m, sorted);  // empty (0) keys sort last
    }
    if (warp == 0) {
        // fusion weights (Step 4): softmax over the kept scores, fp32, max-subtracted
        const uint64_t k0 = lane < m ? sorted[lane] : 0ull;
        const uint64_t k1 = lane + 32 < m ? sorted[lane + 32] : 0ull;
        const float top = m > 0 && sorted[0] ? key_score(sorted[0]) : 0.0f;
        const float e0 = k0 ? expf(key_score(k0) - top) : 0.0f;
        const float e1 = k1 ? expf(key_score(k1) - top) : 0.0f;
        const float z = warp_sum(e0 + e1);
        for (int j = lane; j < K; j += 32) {
            const uint64_t kk = j < 32 ? k0 : k1;
            const float e = j < 32 ? e0 : e1;
            sel_idx_h[j] = kk ? key_index(kk) : -1;
            sel_w_h[j] = kk ? e / z : 0.0f;
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kDecodeThreads, 4) decode_scan_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ Lc, const int64_t *__restrict__ cache_len, int H,
    int Gh, int64_t Nmax, int split, int nsplit, int K, float scale, uint64_t *__restrict__ cand, unsigned *counters,
    int32_t *__restrict__ sel_idx, float *__restrict__ sel_w) {
    constexpr int LPL = D / 8;              // lanes per landmark (one 16-byte vector each)
    constexpr int LPW = 32 / LPL;           // landmarks per warp-wide load
    constexpr int UNROLL = 8;               // independent loads in flight per lane
    constexpr int WARP_SPAN = UNROLL * LPW; // consecutive landmarks per warp per batch
    constexpr int NWARP = kDecodeThreads / 32;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int cap = max(split, nsplit * K);
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);
    uint64_t *topk = keys + cap;            // 64
    uint64_t *sorted = topk + 64;           // 64
    uint32_t *hist = reinterpret_cast<uint32_t *>(sorted + 64);
    int *misc = reinterpret_cast<int *>(hist + 256);  // 8 ints

    // the attend kernel may be scheduled now: it waits (griddepcontrol.wait) for this grid to complete
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int sp = blockIdx.x, bh = blockIdx.y, b = bh / H, kvh = bh / Gh;  // Gh query heads per landmark head
    int64_t nb = cache_len[b] / kChunk;
    nb = nb < 0 ? 0 : (nb > Nmax ? Nmax : nb);
    const int64_t c0 = (int64_t)sp * split;
    const int64_t c1 = min(c0 + (int64_t)split, nb);
    const int nloc = c1 > c0 ? (int)(c1 - c0) : 0;

    const int g = lane / LPL, sub = lane % LPL;
    float qr[8];
    {
        const uint4 v = *reinterpret_cast<const uint4 *>(q + (size_t)bh * D + sub * 8);
        qr[0] = bf16_lo(v.x) * scale; qr[1] = bf16_hi(v.x) * scale;
        qr[2] = bf16_lo(v.y) * scale; qr[3] = bf16_hi(v.y) * scale;
        qr[4] = bf16_lo(v.z) * scale; qr[5] = bf16_hi(v.z) * scale;
        qr[6] = bf16_lo(v.w) * scale; qr[7] = bf16_hi(v.w) * scale;
    }
    const uint16_t *Lbh = Lc + (size_t)kvh * Nmax * D;
    float gm[UNROLL];  // running maximum score of each of this lane group's UNROLL landmark streams
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) gm[u] = -INFINITY;
    for (int64_t base = c0 + (int64_t)warp * WARP_SPAN; base < c1; base += (int64_t)NWARP * WARP_SPAN) {
        uint4 v[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t c = base + u * LPW + g;
            v[u] = c < c1 ? ld_stream16(Lbh + c * D + sub * 8) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            float p = dot8(v[u], qr);
#pragma unroll
            for (int o = LPL / 2; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            const int64_t c = base + u * LPW + g;
            if (c < c1) gm[u] = fmaxf(gm[u], p);
            if (sub == 0 && c < c1) keys[c - c0] = make_key(p, (uint32_t)c);
        }
    }
    __syncthreads();
    // Exact pre-filter before the selection. Each lane group kept, during the stream, the maximum score
    // of each of its UNROLL landmark streams: NG disjoint groups of the range. The K largest group maxima
    // are K different landmarks, so the range's K-th largest score is at least the K-th largest group
    // maximum, tau, and no key below tau can be in the range's top K. The keys >= tau are compacted in
    // place (in rounds that are read whole before any of their slots is written), and the selection
    // runs over those only.
    constexpr int NG = NWARP * LPW * UNROLL;  // 128 (D = 128) or 256 (D = 64) groups
    int nkeys = nloc;
    if (nloc >= 4 * K && K <= NG) {
        float *gmax = reinterpret_cast<float *>(topk);  // scratch until the selection (topk, sorted: 1 KB)
        if (sub == 0) {
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) gmax[(warp * LPW + g) * UNROLL + u] = gm[u];
        }
        __syncthreads();
        for (int i = tid; i < NG; i += kDecodeThreads) {  // rank of each group maximum; ties by position
            const float x = gmax[i];
            int rank = 0;
            for (int jj = 0; jj < NG; ++jj) {
                const float y = gmax[jj];
                rank += (y > x || (y == x && jj < i)) ? 1 : 0;
            }
            if (rank == K - 1) misc[6] = __float_as_int(x);
        }
        __syncthreads();
        const float tau = __int_as_float(misc[6]);
        __syncthreads();  // gmax (topk) is free again
        nkeys = compact_at_least(keys, nloc, make_key(tau, 0xffffffffu), misc);
    }
    // the range's top K, in descending order (the merge reads each range's maximum at its head)
    int cnt;
    if (nkeys <= kRankSelectMax) {
        cnt = block_topk_rank(keys, nkeys, K, sorted);
    } else {
        cnt = block_topk_u64(keys, nkeys, K, topk, hist, misc);
        block_sort_desc_small(topk, cnt, sorted);
    }
    uint64_t *my_cand = cand + ((size_t)bh * nsplit + sp) * K;
    for (int j = tid; j < K; j += kDecodeThreads) my_cand[j] = j < cnt ? sorted[j] : 0ull;

    // ---- last CTA of this (b, h) merges all ranges (ticket taken after a release fence) ----
    __threadfence();
    __syncthreads();
    if (tid == 0) misc[4] = (atomicAdd(&counters[bh], 1u) == (unsigned)(nsplit - 1));
    __syncthreads();
    if (!misc[4]) return;
    __threadfence();
    merge_ranges(cand + (size_t)bh * nsplit * K, nsplit, K, keys, topk, sorted, hist, misc,
                 sel_idx + (size_t)bh * K, sel_w + (size_t)bh * K);
    if (tid == 0) counters[bh] = 0u;
}

// ------------------------------------------------------------------------------------------------
// Grouped heads (G query heads per landmark head): one CTA scores a landmark range for all G heads of
// the group, so the range leaves HBM (and L2) once instead of G times.
// ------------------------------------------------------------------------------------------------

// Sorts the warp's 32 keys (one per lane) into descending order across the lanes (bitonic network:
// 15 compare-exchange stages between lanes l and l ^ j).
__device__ inline uint64_t warp_sort_desc(uint64_t x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const uint64_t y = __shfl_xor_sync(0xffffffffu, x, j);
            const bool desc = (lane & k) == 0;  // k = 32: every lane, the whole warp descending
            const bool lower = (lane & j) == 0;
            x = (lower == desc) ? (x > y ? x : y) : (x < y ? x : y);
        }
    return x;
}

// The 32 largest of two descending 32-key lists (one key per lane), descending. The elementwise maximum
// of one list and the other reversed holds exactly those 32 keys as a bitonic sequence, which five
// half-cleaner stages sort.
__device__ inline uint64_t warp_merge_desc(uint64_t a, uint64_t b) {
    const int lane = threadIdx.x & 31;
    const uint64_t r = __shfl_sync(0xffffffffu, b, 31 - lane);
    uint64_t m = a > r ? a : r;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const uint64_t y = __shfl_xor_sync(0xffffffffu, m, j);
        m = (lane & j) == 0 ? (m > y ? m : y) : (m < y ? m : y);
    }
    return m;
}

// Running exact top K (K <= 32) of one row's scores, kept by one warp across the sub-blocks of a range:
// lane l < K holds the l-th largest key so far (0 = empty). A score at or above the current K-th kept
// score (ties included: the lower chunk may still win on the key) is staged; every 32 staged keys are
// sorted and merged in, and the threshold rises with the K-th kept key.
struct WarpTopK {
    uint64_t best = 0ull;
    float thr = -INFINITY;
    int ns = 0;  // staged keys (warp-uniform)

    __device__ void feed(const float *sc, int n, int64_t c0, int K, uint64_t *stage) {
        const int lane = threadIdx.x & 31;
        for (int r = 0; r < n; r += 32) {
            const int i = r + lane;
            const bool cand = i < n && sc[i] >= thr;
            const unsigned bal = __ballot_sync(0xffffffffu, cand);
            if (bal == 0u) continue;
            if (cand) stage[ns + __popc(bal & ((1u << lane) - 1u))] = make_key(sc[i], (uint32_t)(c0 + i));
            ns += __popc(bal);
            __syncwarp();
            if (ns >= 32) {
                best = warp_merge_desc(best, warp_sort_desc(stage[lane]));
                const uint64_t rest = lane + 32 < ns ? stage[lane + 32] : 0ull;
                __syncwarp();
                if (lane + 32 < ns) stage[lane] = rest;
                __syncwarp();
                ns -= 32;
                const uint64_t kth = __shfl_sync(0xffffffffu, best, K - 1);  // 0 until K keys are kept
                if (kth != 0ull) thr = fmaxf(thr, key_score(kth));
            }
        }
    }
    __device__ uint64_t finish(int K, const uint64_t *stage) {
        const int lane = threadIdx.x & 31;
        if (ns > 0) best = warp_merge_desc(best, warp_sort_desc(lane < ns ? stage[lane] : 0ull));
        ns = 0;
        return lane < K ? best : 0ull;
    }
};

constexpr int kDecodeGroupThreads = 768;  // warps 0-7 score the sub-blocks, warps 8-23 select (one row each)
constexpr int kGsScorers = 8;
constexpr int kGsSelectors = 16;
constexpr int kGsSub = 128;                // landmarks per sub-block (one bulk copy)
constexpr int kGsStages = 4;               // sub-blocks in flight
constexpr int kGsBufs = 4;                 // score buffers: the scorers may run this many sub-blocks ahead

template <int D>
struct GsSmem {
    static constexpr uint32_t STAGE = kGsSub * D * 2;                 // bf16 rows, 64-column boxes, 128 B swizzle
    static constexpr uint32_t SC = kGsStages * STAGE;                       // [kGsBufs][16][kGsSub + 8] fp32
    static constexpr uint32_t STG = SC + kGsBufs * 16 * (kGsSub + 8) * 4;   // [16 rows][64] staged keys
    // full[kGsStages] (copies landed), empty[kGsStages] (scorers read them), ready / free[kGsBufs] (scores)
    static constexpr uint32_t BAR = STG + 16 * 64 * 8;
    static constexpr uint32_t BYTES = BAR + (2 * kGsStages + 2 * kGsBufs) * 8;
    static constexpr size_t DYN = BYTES + 1024;                       // + alignment of the stages
};

// grid (nsplit, B*Hkv, ceil(R / 16)): the landmark range sp of key head kvh, for 16 of its R = Gh * Tq
// query rows (Gh query heads, Tq query tokens each; row r = g * Tq + i is token i of head g, and the
// rows of a key head are consecutive in q). Token i sits at position cache_len - Tq + i and sees the
// chunks that have ended at or before it.
// The range streams through shared memory in sub-blocks of 128 landmarks by bulk tensor copies (four in
// flight, so no register holds a load). Scorer warps turn each sub-block into scores: the scores of a
// tile of 8 landmarks for the 16 rows are one m16n8k16 tensor-core product per 16 columns of D (M = 16
// is below the tcgen05 tile, so the warp-level MMA). The reduction index is permuted alike in both
// operands so that each lane reads whole 16-byte chunks: lane (g, t4) takes columns 32 s + 8 t4 .. + 7
// of head rows g, g + 8 and of landmark g of the tile, and k-steps 2 s, 2 s + 1 take the two halves of
// that chunk. Selector warps (one per row) fold each sub-block's scores into the rows' running top K
// while the scorers work on the next ones (kGsBufs score buffers; mbarriers hand them over, every
// wait bounded).
template <int D>
__global__ void __launch_bounds__(kDecodeGroupThreads, 1) decode_scan_group_kernel(
    const uint16_t *__restrict__ q, const __grid_constant__ CUtensorMap tmL, const int64_t *__restrict__ cache_len,
    int Hkv, int R, int Tq, int64_t Nmax, int split, int nsplit, int K, float scale, uint64_t *__restrict__ cand,
    int32_t *__restrict__ err) {
    using SM = GsSmem<D>;
    constexpr int S = D / 32;  // 16-byte chunks per lane per row
    constexpr int LD = kGsSub + 8;  // score row stride (fewer bank conflicts on the fragment stores)
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sb - raw);
    float *sc = reinterpret_cast<float *>(smem + SM::SC);
    uint64_t *stage = reinterpret_cast<uint64_t *>(smem + SM::STG);
    auto full = [&](int st) { return sb + SM::BAR + 8u * st; };
    auto empty = [&](int st) { return sb + SM::BAR + 8u * (kGsStages + st); };
    auto ready = [&](int bf) { return sb + SM::BAR + 8u * (2 * kGsStages + bf); };
    auto freeb = [&](int bf) { return sb + SM::BAR + 8u * (2 * kGsStages + kGsBufs + bf); };

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t4 = lane & 3;
    const int sp = blockIdx.x, kvh = blockIdx.y, b = kvh / Hkv, r0 = blockIdx.z * 16;
    const int rows = min(16, R - r0);
    const int64_t len = cache_len[b];
    auto n_of = [&](int r) {  // chunks seen by row r: its token sits at len - Tq + r % Tq
        int64_t n = (len - Tq + r % Tq + 1) / kChunk;
        return n < 0 ? (int64_t)0 : (n > Nmax ? Nmax : n);
    };
    const int64_t nb = n_of(Tq - 1);  // the last token sees the most
    const int64_t c0 = (int64_t)sp * split;
    const int64_t c1 = min(c0 + (int64_t)split, nb);
    const int nloc = c1 > c0 ? (int)(c1 - c0) : 0;
    const int nsub = (nloc + kGsSub - 1) / kGsSub;
    const size_t q0 = (size_t)kvh * R + r0;  // q row of this CTA's first row

    if (tid == 0) {
        for (int st = 0; st < kGsStages; ++st) {
            tc::mbar_init(full(st), 1);
            tc::mbar_init(empty(st), kGsScorers);
        }
        for (int bf = 0; bf < kGsBufs; ++bf) {
            tc::mbar_init(ready(bf), kGsScorers);
            tc::mbar_init(freeb(bf), kGsSelectors);
        }
        tc::fence_mbar_init();
    }
    __syncthreads();
    auto load = [&](int i) {  // sub-block i into stage i % kGsStages
        const int st = i % kGsStages;
        tc::mbar_arrive_expect_tx(full(st), SM::STAGE);
#pragma unroll
        for (int h = 0; h < D / 64; ++h)
            tc::tma_load_2d(sb + st * SM::STAGE + h * kGsSub * 128, &tmL, h * 64,
                            (int)(kvh * Nmax + c0 + (int64_t)i * kGsSub), full(st));
    };
    int issued = 0;
    if (tid == 0)
        for (; issued < kGsStages && issued < nsub; ++issued) load(issued);
    bool ok = true;

    if (warp < kGsScorers) {
        // ---------------- scorers ----------------
        uint32_t a[S][2][4];
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const uint4 qa = g < rows ? *reinterpret_cast<const uint4 *>(q + (q0 + g) * D + 32 * s + 8 * t4)
                                      : make_uint4(0u, 0u, 0u, 0u);
            const uint4 qb = g + 8 < rows ? *reinterpret_cast<const uint4 *>(q + (q0 + g + 8) * D + 32 * s + 8 * t4)
                                          : make_uint4(0u, 0u, 0u, 0u);
            a[s][0][0] = qa.x; a[s][0][1] = qb.x; a[s][0][2] = qa.y; a[s][0][3] = qb.y;
            a[s][1][0] = qa.z; a[s][1][1] = qb.z; a[s][1][2] = qa.w; a[s][1][3] = qb.w;
        }
        for (int i = 0; i < nsub && ok; ++i) {
            const int st = i % kGsStages, bf = i % kGsBufs;
            ok = __all_sync(0xffffffffu,
                            tc::mbar_wait(full(st), (uint32_t)(i / kGsStages) & 1u) &&
                                (i < kGsBufs || tc::mbar_wait(freeb(bf), (uint32_t)((i / kGsBufs) - 1) & 1u)));
            if (!ok) break;  // (the scores of sub-block i - kGsBufs have been consumed)
            const int nt = min(kGsSub, nloc - i * kGsSub);
            const uint32_t stg = sb + st * SM::STAGE;
            float *scb = sc + bf * 16 * LD;  // buffer bf
            for (int tile = warp; tile * 8 < nt; tile += kGsScorers) {
                float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const int jj = (4 * s + t4) & 7;  // 16-byte chunk within the 64-column box
                    uint4 v;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                 : "r"(stg + ((4 * s + t4) >> 3) * kGsSub * 128 + tc::sw128(tile * 8 + g, jj)));
                    mma_bf16_16816(acc, a[s][0], v.x, v.y);
                    mma_bf16_16816(acc, a[s][1], v.z, v.w);
                }
                const int i0 = tile * 8 + 2 * t4;  // acc: rows g (0, 1) and g + 8 (2, 3), landmarks i0, i0 + 1
                if (g < rows) {
                    if (i0 < nt) scb[g * LD + i0] = acc[0] * scale;
                    if (i0 + 1 < nt) scb[g * LD + i0 + 1] = acc[1] * scale;
                }
                if (g + 8 < rows) {
                    if (i0 < nt) scb[(g + 8) * LD + i0] = acc[2] * scale;
                    if (i0 + 1 < nt) scb[(g + 8) * LD + i0 + 1] = acc[3] * scale;
                }
            }
            __syncwarp();
            if (lane == 0) {
                tc::mbar_arrive(ready(bf));  // this warp's scores of sub-block i are written
                tc::mbar_arrive(empty(st));  // and its reads of the stage are done
            }
            if (warp == 0) {  // refill the stage once every scorer has read it (lane 0; the warp waits)
                bool w_ok = true;
                if (lane == 0 && issued < nsub) {
                    w_ok = tc::mbar_wait(empty(st), (uint32_t)(i / kGsStages) & 1u);
                    if (w_ok) {
                        tc::fence_proxy_async_smem();
                        load(issued++);
                    }
                }
                ok = __all_sync(0xffffffffu, w_ok);
                if (!ok) break;
            }
        }
    } else {
        // ---------------- selectors: one row each ----------------
        const int r = warp - kGsScorers;
        WarpTopK sel;
        const int64_t lim = r < rows ? min(c1, n_of(r0 + r)) : c0;
        for (int i = 0; i < nsub && ok; ++i) {
            const int bf = i % kGsBufs;
            ok = __all_sync(0xffffffffu, tc::mbar_wait(ready(bf), (uint32_t)(i / kGsBufs) & 1u));
            if (!ok) break;
            const int nt = min(kGsSub, nloc - i * kGsSub);
            const int64_t base = c0 + (int64_t)i * kGsSub;
            const int64_t nr = min((int64_t)nt, lim - base);
            if (nr > 0) sel.feed(sc + (bf * 16 + r) * LD, (int)nr, base, K, stage + r * 64);  // buffer bf
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(freeb(bf));
        }
        if (r < rows) {
            const uint64_t best = sel.finish(K, stage + r * 64);
            if (lane < K) cand[((q0 + r) * nsplit + sp) * K + lane] = best;
        }
    }
    if (!ok) {  // a wait ran out: report it, and wait (bounded) for the copies this CTA issued
        if (err && lane == 0) atomicOr(err, 1);
        if (tid == 0)
            for (int i = issued > kGsStages ? issued - kGsStages : 0; i < issued; ++i)
                tc::mbar_wait(full(i % kGsStages), (uint32_t)(i / kGsStages) & 1u);
    }
}

// grid (B*H): the exact merge of one query head's range candidates. Launched as a programmatic
// dependent of the grouped scan; waits for that grid before reading its candidates.
__global__ void __launch_bounds__(kDecodeThreads) decode_merge_kernel(const uint64_t *__restrict__ cand, int nsplit,
                                                                      int K, int32_t *__restrict__ sel_idx,
                                                                      float *__restrict__ sel_w) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int cap = nsplit * K;
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);
    uint64_t *topk = keys + cap;
    uint64_t *sorted = topk + 64;
    uint32_t *hist = reinterpret_cast<uint32_t *>(sorted + 64);
    int *misc = reinterpret_cast<int *>(hist + 256);
    const size_t bh = blockIdx.x;
    merge_ranges(cand + bh * nsplit * K, nsplit, K, keys, topk, sorted, hist, misc, sel_idx + bh * K, sel_w + bh * K);
}

// QKN: query-key normalisation, the logits use q / max(|q|, eps) and k / max(|k|, eps) (fp32, on the fly).
template <int D, bool QKN>
__global__ void __launch_bounds__(kDecodeThreads) decode_attend_kernel(
    const uint16_t *__restrict__ q, const uint16_t *__restrict__ Kc, const uint16_t *__restrict__ Vc, int64_t Tmax,
    int Gh, int Tq, int K, float scale, const int32_t *__restrict__ sel_idx, const float *__restrict__ sel_w,
    float *__restrict__ partial, unsigned *counters, uint16_t *__restrict__ out) {
    constexpr int LPL = D / 8, LPW = 32 / LPL, NWARP = kDecodeThreads / 32;
    constexpr int GROUPS = kDecodeThreads / LPL;  // key groups for the P.V pass
    constexpr int KEYS_PER_GROUP = kChunk / GROUPS;
    __shared__ float s_p[kChunk];
    __shared__ float s_red[GROUPS][D];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int j = blockIdx.x, bh = blockIdx.y;
    // launched early (programmatic dependent launch): wait until the scan grid has completed and its
    // selection is visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int c = sel_idx[(size_t)bh * K + j];
    float *my_part = partial + ((size_t)bh * K + j) * D;
    if (c >= 0) {
        const int g = lane / LPL, sub = lane % LPL;
        float qr[8];
        const uint4 qv = *reinterpret_cast<const uint4 *>(q + (size_t)bh * D + sub * 8);
        qr[0] = bf16_lo(qv.x) * scale; qr[1] = bf16_hi(qv.x) * scale;
        qr[2] = bf16_lo(qv.y) * scale; qr[3] = bf16_hi(qv.y) * scale;
        qr[4] = bf16_lo(qv.z) * scale; qr[5] = bf16_hi(qv.z) * scale;
        qr[6] = bf16_lo(qv.w) * scale; qr[7] = bf16_hi(qv.w) * scale;
        if constexpr (QKN) {  // |scale q|^2 over the row's LPL lanes -> q / max(|q|, eps), times scale
            float n2 = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) n2 = fmaf(qr[e], qr[e], n2);
#pragma unroll
            for (int o = LPL / 2; o > 0; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
            const float rq = rsqrtf(fmaxf(n2, kQkNormEps * kQkNormEps * scale * scale)) * scale;
#pragma unroll
            for (int e = 0; e < 8; ++e) qr[e] *= rq;
        }
        const size_t row0 = ((size_t)(bh / Tq / Gh) * Tmax + (size_t)c * kChunk);  // the key head's cache
        constexpr int ROUNDS = kChunk / (NWARP * LPW);
        const int sl = tid % LPL, grp = tid / LPL;
        // issue every K and V load of this thread up front so both overlap the logit math
        uint4 kv[ROUNDS], vv[KEYS_PER_GROUP];
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r)
            kv[r] = *reinterpret_cast<const uint4 *>(Kc + (row0 + (r * NWARP + warp) * LPW + g) * D + sub * 8);
#pragma unroll
        for (int i = 0; i < KEYS_PER_GROUP; ++i)
            vv[i] = *reinterpret_cast<const uint4 *>(Vc + (row0 + grp * KEYS_PER_GROUP + i) * D + sl * 8);
        // Step 3 logits: a_u = scale * q . K_c[u] (with QKN: scale * norm(q) . norm(K_c[u]))
#pragma unroll
        for (int r = 0; r < ROUNDS; ++r) {
            float p = dot8(kv[r], qr);
#pragma unroll
            for (int o = LPL / 2; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
            if constexpr (QKN) {
                const uint32_t w[4] = {kv[r].x, kv[r].y, kv[r].z, kv[r].w};
                float k2 = 0.0f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    k2 = fmaf(bf16_lo(w[e]), bf16_lo(w[e]), k2);
                    k2 = fmaf(bf16_hi(w[e]), bf16_hi(w[e]), k2);
                }
#pragma unroll
                for (int o = LPL / 2; o > 0; o >>= 1) k2 += __shfl_xor_sync(0xffffffffu, k2, o);
                p *= rsqrtf(fmaxf(k2, kQkNormEps * kQkNormEps));
            }
            if (sub == 0) s_p[(r * NWARP + warp) * LPW + g] = p;
        }
        __syncthreads();
        if (warp == 0) {
            const float a0 = s_p[lane], a1 = s_p[lane + 32];
            float mx = fmaxf(a0, a1);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const float e0 = expf(a0 - mx), e1 = expf(a1 - mx);
            const float z = warp_sum(e0 + e1);
            s_p[lane] = e0 / z;
            s_p[lane + 32] = e1 / z;
        }
        __syncthreads();
        // O_c = P . V_c
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < KEYS_PER_GROUP; ++i) {
            const float p = s_p[grp * KEYS_PER_GROUP + i];
            acc[0] = fmaf(p, bf16_lo(vv[i].x), acc[0]); acc[1] = fmaf(p, bf16_hi(vv[i].x), acc[1]);
            acc[2] = fmaf(p, bf16_lo(vv[i].y), acc[2]); acc[3] = fmaf(p, bf16_hi(vv[i].y), acc[3]);
            acc[4] = fmaf(p, bf16_lo(vv[i].z), acc[4]); acc[5] = fmaf(p, bf16_hi(vv[i].z), acc[5]);
            acc[6] = fmaf(p, bf16_lo(vv[i].w), acc[6]); acc[7] = fmaf(p, bf16_hi(vv[i].w), acc[7]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) s_red[grp][sl * 8 + e] = acc[e];
        __syncthreads();
        for (int d = tid; d < D; d += kDecodeThreads) {
            float s = 0.0f;
#pragma unroll 8
            for (int gg = 0; gg < GROUPS; ++gg) s += s_red[gg][d];
            my_part[d] = s;
        }
    }
    // ---- last CTA of this (b, h) blends the K chunk outputs (Step 4) ----
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&counters[bh], 1u) == (unsigned)(K - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int d = tid; d < D; d += kDecodeThreads) {
        float o = 0.0f;
        for (int jj = 0; jj < K; ++jj) {
            if (sel_idx[(size_t)bh * K + jj] < 0) continue;
            o = fmaf(sel_w[(size_t)bh * K + jj], __ldcg(partial + ((size_t)bh * K + jj) * D + d), o);
        }
        out[(size_t)bh * D + d] = (uint16_t)(pack_bf16x2(o, 0.0f) & 0xffffu);
    }
    if (tid == 0) counters[bh] = 0u;
}

// Landmarks per scan range. The scan is HBM-bound and every range costs the same, so the ranges are
// sized for a single wave of CTAs: B*H*ranges <= kDecodeWaveCtas (148 SMs x 4 resident CTAs of
// 256 threads: the scan's launch bound holds it to 64 registers, without spills). A range keeps at least 256 landmarks and at most
// 6144 (its keys live in shared memory), and ranges*K <= 8192 (the merge holds all candidates).
constexpr int64_t kDecodeSms = 148;
constexpr int64_t kDecodeWaveCtas = kDecodeSms * 4;

int decode_split_size(int64_t Nmax, int K, int BH) {
    if (Nmax <= 0) return 1;
    int64_t ns = BH > 0 ? kDecodeWaveCtas / BH : 1;
    ns = ns < 1 ? 1 : ns;
    const int64_t by_min = (Nmax + 255) / 256;
    ns = ns < by_min ? ns : by_min;
    if ((Nmax + ns - 1) / ns > 6144) ns = (Nmax + 6143) / 6144;
    const int64_t merge_cap = 8192 / K > 0 ? 8192 / K : 1;
    ns = ns < merge_cap ? ns : merge_cap;
    ns = ns < 1 ? 1 : ns;
    return (int)((Nmax + ns - 1) / ns);
}

size_t decode_scan_smem(int split, int nsplit, int K) {
    const size_t cap = (size_t)(split > nsplit * K ? split : nsplit * K);
    return (cap + 128) * sizeof(uint64_t) + 256 * sizeof(uint32_t) + 8 * sizeof(int);
}


DecodePlan decode_plan(int64_t Nmax, int K, int B, int H, int Hkv, int Tq) {
    DecodePlan p{};
    const int Gh = Hkv > 0 ? H / Hkv : 1;
    const int R = Gh * (Tq > 0 ? Tq : 1);  // query rows per key head
    p.row_groups = (R + 15) / 16;
    if (R >= 2 && K <= 32 && Nmax <= 0) {  // no chunk at all: one empty range
        p.grouped = true;
        p.split = 64;
        p.nsplit = 1;
        return p;
    }
    if (R >= 2 && K <= 32) {
        // one CTA per SM in a single wave, >= 256 landmarks per range; the merge keeps every candidate in
        // shared memory (ranges * K <= 8192, ranges <= 512)
        int64_t ns = (int64_t)kDecodeSms / ((int64_t)B * Hkv * p.row_groups);
        ns = ns < 1 ? 1 : ns;
        const int64_t by_min = (Nmax + 255) / 256;
        ns = ns < by_min ? ns : by_min;
        const int64_t cap = (8192 / K < 512) ? 8192 / K : 512;
        ns = ns < cap ? ns : cap;
        int64_t split = (Nmax + ns - 1) / ns;
        split = (split + kGsSub - 1) / kGsSub * kGsSub;  // whole sub-blocks
        p.grouped = true;
        p.split = (int)split;
        p.nsplit = (int)((Nmax + split - 1) / split);
        return p;
    }
    p.split = decode_split_size(Nmax, K, B * H);
    const int64_t ns = (Nmax + p.split - 1) / p.split;
    p.nsplit = ns > 0 ? (int)ns : 1;
    return p;
}

size_t decode_plan_smem(const DecodePlan &p, int K) {
    if (!p.grouped) return decode_scan_smem(p.split, p.nsplit, K);
    const size_t merge = ((size_t)p.nsplit * K + 128) * sizeof(uint64_t) + 256 * sizeof(uint32_t) + 8 * sizeof(int);
    const size_t scan = GsSmem<128>::DYN;
    return merge > scan ? merge : scan;
}

// The attend kernel is launched as a programmatic dependent of the scan, so that its launch overlaps
// the scan's tail; it waits for the scan grid's completion before reading the selection.
template <int D>
static cudaError_t launch_attend(const DecodeArgs &a, dim3 grid, cudaStream_t s) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    auto kern = a.qk_norm ? decode_attend_kernel<D, true> : decode_attend_kernel<D, false>;
    return cudaLaunchKernelEx(&cfg, kern, a.q, a.Kc, a.Vc, a.Tmax, a.H / a.Hkv, a.Tq, a.K, a.scale,
                              (const int32_t *)a.sel_idx,
                              (const float *)a.sel_w, a.partial, a.counters + (size_t)a.B * a.H * a.Tq, a.out);
}

template <int D>
static cudaError_t launch_decode_grouped(const DecodeArgs &a, const DecodePlan &pl, cudaStream_t s) {
    const int R = a.H / a.Hkv * a.Tq, rows_q = a.B * a.H * a.Tq;
    const size_t gsmem = GsSmem<D>::DYN;
    cudaError_t e = cudaFuncSetAttribute(decode_scan_group_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)gsmem);
    if (e != cudaSuccess) return e;
    CUtensorMap tm;  // landmark rows [B*Hkv*Nmax, D]; boxes of kGsSub rows (with no chunk: never read)
    const uint64_t lrows = (uint64_t)a.B * a.Hkv * a.Nmax;
    if (!make_tmap_bf16(&tm, lrows > 0 ? (const void *)a.Lc : (const void *)a.q, lrows > 0 ? lrows : 1, D, kGsSub))
        return cudaErrorInvalidValue;
    {
        HSA_PROF("decode_scan", s);
        decode_scan_group_kernel<D><<<dim3(pl.nsplit, a.B * a.Hkv, pl.row_groups), kDecodeGroupThreads, gsmem, s>>>(
            a.qs, tm, a.cache_len, a.Hkv, R, a.Tq, a.Nmax, pl.split, pl.nsplit, a.K, a.scale, a.cand, a.err);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    const size_t msmem = ((size_t)pl.nsplit * a.K + 128) * sizeof(uint64_t) + 256 * sizeof(uint32_t) + 8 * sizeof(int);
    e = cudaFuncSetAttribute(decode_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(rows_q);
    cfg.blockDim = dim3(kDecodeThreads);
    cfg.dynamicSmemBytes = msmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    {
        HSA_PROF("decode_merge", s);
        e = cudaLaunchKernelEx(&cfg, decode_merge_kernel, (const uint64_t *)a.cand, pl.nsplit, a.K, a.sel_idx, a.sel_w);
    }
    if (e != cudaSuccess) return e;
    HSA_PROF("decode_attend", s);
    return launch_attend<D>(a, dim3(a.K, rows_q), s);
}

// The per-call reset: the ticket counters and the error flag. Both workspace layouts put the counters
// right after the flag, so one memset covers both (one graph node less per decode step).
static cudaError_t zero_decode_state(const DecodeArgs &a, size_t rows, cudaStream_t s) {
    char *f = reinterpret_cast<char *>(a.err), *c = reinterpret_cast<char *>(a.counters);
    const size_t cb = 2 * rows * sizeof(unsigned);
    if (f && c > f && (size_t)(c - f) <= 4096) return cudaMemsetAsync(f, 0, (size_t)(c - f) + cb, s);
    cudaError_t e = cudaMemsetAsync(c, 0, cb, s);
    if (e == cudaSuccess && f) e = cudaMemsetAsync(f, 0, sizeof(int32_t), s);
    return e;
}

cudaError_t launch_decode(const DecodeArgs &a0, cudaStream_t s) {
    DecodeArgs a = a0;
    if (a.Hkv <= 0) a.Hkv = a.H;
    if (a.Tq <= 0) a.Tq = 1;
    if (a.H % a.Hkv != 0) return cudaErrorInvalidValue;
    const DecodePlan pl = decode_plan(a.Nmax, a.K, a.B, a.H, a.Hkv, a.Tq);
    if (pl.grouped) {
        cudaError_t e;
        {
            HSA_PROF("memset", s);
            e = zero_decode_state(a, (size_t)a.B * a.H * a.Tq, s);
        }
        if (e != cudaSuccess) return e;
        e = a.D == 128 ? launch_decode_grouped<128>(a, pl, s) : launch_decode_grouped<64>(a, pl, s);
        return e != cudaSuccess ? e : cudaGetLastError();
    }
    if (a.Tq != 1) return cudaErrorInvalidValue;  // several query tokens need the grouped scan (K <= 32)
    const int split = decode_split_size(a.Nmax, a.K, a.B * a.H);
    const int nsplit = (int)((a.Nmax + split - 1) / split) > 0 ? (int)((a.Nmax + split - 1) / split) : 1;
    const size_t smem = decode_scan_smem(split, nsplit, a.K);
    const int BH = a.B * a.H;
    cudaError_t e;
    {
        HSA_PROF("memset", s);
        e = zero_decode_state(a, (size_t)BH, s);
    }
    if (e != cudaSuccess) return e;
    dim3 g1(nsplit, BH), g2(a.K, BH);
    if (a.D == 128) {
        e = cudaFuncSetAttribute(decode_scan_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        {
            HSA_PROF("decode_scan", s);
            decode_scan_kernel<128><<<g1, kDecodeThreads, smem, s>>>(a.qs, a.Lc, a.cache_len, a.H, a.H / a.Hkv, a.Nmax, split,
                                                                     nsplit, a.K, a.scale, a.cand, a.counters,
                                                                     a.sel_idx, a.sel_w);
        }
        HSA_PROF("decode_attend", s);
        e = launch_attend<128>(a, g2, s);
    } else {
        e = cudaFuncSetAttribute(decode_scan_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        {
            HSA_PROF("decode_scan", s);
            decode_scan_kernel<64><<<g1, kDecodeThreads, smem, s>>>(a.qs, a.Lc, a.cache_len, a.H, a.H / a.Hkv, a.Nmax, split,
                                                                    nsplit, a.K, a.scale, a.cand, a.counters,
                                                                    a.sel_idx, a.sel_w);
        }
        HSA_PROF("decode_attend", s);
        e = launch_attend<64>(a, g2, s);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace hsa
