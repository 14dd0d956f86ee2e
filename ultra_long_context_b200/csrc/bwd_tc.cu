// bwd_tc.cu -- gradients of the HSA forward on the 5th-generation tensor cores (head dims 64 and 128).
//
// Explainer page of "Every Token Counts", "How It Works (Technically)", Step 4: the fusion weight
// w = softmax(s over the selected chunks) multiplies the chunk output, so the loss gradient reaches
// the retrieval scores and through them the landmarks; the discrete top-K choice is held fixed.
// Per (token t, selected chunk c) pair with weight w, P = softmax(scale q K_c^T), O_c = P V_c:
//   dP' = dO V_c^T,  g = rowsum(P * dP'),  ds = w (g - delta_t)  with delta_t = dO . O_t
//   dS  = w P * (dP' - g)
//   dQ_t += scale (dS K_c + ds L_c),  dK_c += scale dS^T q,  dV_c += (w P)^T dO,  dL_c += scale ds q
//
// Work unit: up to 1024 pairs of one chunk (the chunk-major pair lists of the forward's dispatch),
// processed as tiles of 128 pairs. Persistent kernel, one CTA per SM, units round-robin.
//   * S = Q K^T and dP' = dO V^T (M = 128 pairs, N = 64 keys) into double-buffered TMEM;
//   * dQ = dS K (M = 128 pairs, N = D) into TMEM, then reduced into the tokens' fp32 rows (plus the
//     rank-one ds L term) -- the only per-pair reduction;
//   * dK^T += Q^T dS and dV^T += dO^T (w P) (M = D, N = 64 keys, K = the tile's pairs) accumulate in
//     TMEM over all tiles of the unit and are added into dK, dV once per unit.
// Every operand is read from shared memory in the layout it was written in: the gathered Q / dO tiles
// and K / V are 128-byte-swizzled rows that serve as K-major operands (for S, dP') and as MN-major
// operands (Q^T and dO^T for dK^T, dV^T; K for dQ); w P and dS are [pair][key] swizzled rows that
// serve as the K-major A operand of dQ and the MN-major B operand of dK^T / dV^T.
// Warps: 0-3 compute (one thread per pair row: softmax, g, ds, dS, w P), 4-11 epilogue (two
// warpgroups: one half of the dQ columns each, and the unit's dV or dK), 12-15 loaders (cp.async
// gathers of Q and dO rows, TMA tiles of K and V; dL from a tile's Q rows before its stage is
// reloaded), 16 MMA issuer.
// Head dim 64 uses the same layout: a Q or dO tile keeps two 64-column halves, the second zero (set
// once), so dK^T and dV^T stay M = 128 products whose rows 64-127 come out zero and are not read.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "launch.h"
#include "profile.h"
#include "tc.cuh"

namespace hsa {

constexpr int kBtTile = 128;                      // pairs per tile (MMA M)
static_assert(kBwdUnitPairs % 128 == 0, "units are whole 128-pair tiles");
constexpr int kBtEpiWarp0 = 4;                    // warps 4-11
constexpr int kBtLoaderWarp0 = 12;                // warps 12-15
constexpr int kBtMmaWarp = 16;
constexpr int kBtThreads = 32 * (kBtMmaWarp + 1);  // 544

struct BtSmem {  // head dims 64 and 128 (64: the second half of a Q / dO tile holds zeros)
    static constexpr uint32_t HALF = 16384;            // [128 rows][128 B]: 64 columns of a Q / dO tile
    static constexpr uint32_t QD = 4 * HALF;           // Q tile (two halves) + dO tile (two halves)
    static constexpr uint32_t KH = 8192;               // [64 rows][128 B]: 64 columns of K or V
    static constexpr uint32_t STG = 0;                 // Q / dO stages [2]
    static constexpr uint32_t KO = STG + 2 * QD;       // K (two halves)
    static constexpr uint32_t VO = KO + 2 * KH;        // V (two halves)
    static constexpr uint32_t WP = VO + 2 * KH;        // w P  [128 pairs][64 keys] bf16, swizzled
    static constexpr uint32_t DS = WP + 16384;         // dS   [128 pairs][64 keys] bf16, swizzled
    static constexpr uint32_t SLAB = 16;               // dQ epilogue columns per pass
    static constexpr uint32_t OUT_ROW = SLAB * 4 + 16; // fp32 staging row + pad
    static constexpr uint32_t OUT = DS + 16384;        // per epilogue warp: [32 rows][OUT_ROW]
    static constexpr uint32_t ROW = OUT + 8 * 32 * OUT_ROW;  // int[2][128]: token rows of a stage
    static constexpr uint32_t W = ROW + 1024;          // float[2][128]: fusion weights
    static constexpr uint32_t DEL = W + 1024;          // float[2][128]: delta of the pair's token
    static constexpr uint32_t LROW = DEL + 1024;       // float[4][128]: a unit's landmark row (fp32), slot k % 4
    static constexpr uint32_t EROW = LROW + 2048;      // int[4][128]: token rows for the dQ epilogue
    static constexpr uint32_t EDS = EROW + 2048;       // float[4][128]: ds (dQ epilogue and dL)
    static constexpr uint32_t SDL = EDS + 2048;        // float[4][128]: the unit's dL per compute warp
    static constexpr uint32_t SSLOT = SDL + 2048;      // int[2][128]: slot of each pair (separate Qs only)
    static constexpr uint32_t BAR = SSLOT + 1024;
    static constexpr int NBAR = 22;
    static constexpr uint32_t TMEM = BAR + NBAR * 8;
    static constexpr uint32_t BYTES = TMEM + 16;
    static constexpr size_t DYN = BYTES + 1024;
    static_assert(DYN <= 227 * 1024, "shared memory budget");
    // TMEM columns
    static constexpr uint32_t S_COL = 0;     // S: 64 (P, fp32, is written back over S)
    static constexpr uint32_t DP_COL = 64;   // dP': 64
    static constexpr uint32_t DQ_COL = 128;  // dQ buffers [2] x 128
    static constexpr uint32_t DV_COL = 384;  // dV^T: 64 (lane = d)
    static constexpr uint32_t DK_COL = 448;  // dK^T: 64 (lane = d)
};

// mbarrier slots. Phases: qd_* and dq_* per tile pair (j / 2), e_ready per 4 tiles (j / 4), s_* and
// ds_* per tile (j), kv_* and acc_* per unit (k).
enum {
    kBQdFull = 0,          // [2] loaders (128 arrivals, after their Q / dO copies have landed)
    kBQdEmpty = 2,         // [2] commit after the last MMA that reads the stage
    kBKvFull = 4,          // loader thread 0 (arrive + K, V bytes)
    kBKvEmpty = 5,         // commit after the unit's last MMA
    kBSFull = 6,           // commit after S and dP'
    kBSEmpty = 7,          // compute warps (128) once P / dP' are consumed
    kBDsFull = 8,          // compute warps (128) once w P and dS are in shared memory
    kBDsEmpty = 9,         // commit after dQ, dK^T, dV^T
    kBDqFull = 10,         // [2] commit after dQ into TMEM buffer j % 2
    kBDqEmpty = 12,        // [2] epilogue warps (256) once that buffer is read
    kBAccFull = 14,        // commit after the unit's last dK^T / dV^T
    kBAccEmpty = 15,       // epilogue warps (256) once dK^T / dV^T are read
    kBEReady = 16,         // [4] compute warps (128): rows and ds of tile j for the dQ epilogue (slot j % 4)
};

// Walks this CTA's units and their 128-pair tiles in order.
struct BtCursor {
    const PairTile *units;
    int first, stride, mine;  // unit blockIdx.x + k * stride, k < mine
    int k = 0, i = 0, nt = 0, j = 0;
    PairTile u{0, 0, 0, 0};
    __device__ void load() {
        if (k < mine) {
            u = units[first + (size_t)k * stride];
            nt = (u.count + kBtTile - 1) / kBtTile;
        }
    }
    __device__ bool done() const { return k >= mine; }
    __device__ bool first_tile() const { return i == 0; }
    __device__ bool last_tile() const { return i == nt - 1; }
    __device__ void next() {
        ++j;
        if (++i == nt) {
            i = 0;
            ++k;
            load();
        }
    }
};

template <int D, bool QSLC>
__global__ void __launch_bounds__(kBtThreads, 1) chunk_bwd_tc_kernel(
    const uint16_t *__restrict__ Q, const uint16_t *__restrict__ L, const uint16_t *__restrict__ dout,
    const float *__restrict__ delta, int T, int N, float scale, const PairTile *__restrict__ units,
    const int32_t *__restrict__ num_units, const int32_t *__restrict__ pair_row, const float *__restrict__ pair_w,
    float *__restrict__ dQ, float *__restrict__ dK, float *__restrict__ dV, float *__restrict__ dL,
    int32_t *__restrict__ err, const uint16_t *__restrict__ Qs, const int32_t *__restrict__ pair_slot,
    float *__restrict__ ds_pair, int Kslots, int Gh, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV) {
    // QSLC: separate retrieval queries Qs. dL takes ds times the retrieval query (read from global
    // memory), dQ leaves out the ds L_c term, and ds goes to ds_pair[token row, slot].
    using SM = BtSmem;
    static_assert(D == 64 || D == 128, "head dims 64 and 128");
    constexpr int KHALVES = D / 64;  // 64-column halves of a K / V tile
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;  // 1 KB aligned (swizzle atoms)
    unsigned char *s = smem_raw + (sb - raw);
    int *s_row = reinterpret_cast<int *>(s + SM::ROW);
    float *s_w = reinterpret_cast<float *>(s + SM::W);
    float *s_del = reinterpret_cast<float *>(s + SM::DEL);
    float *s_L = reinterpret_cast<float *>(s + SM::LROW);
    int *e_row = reinterpret_cast<int *>(s + SM::EROW);
    float *e_ds = reinterpret_cast<float *>(s + SM::EDS);
    float *s_dl = reinterpret_cast<float *>(s + SM::SDL);
    int *s_slot = reinterpret_cast<int *>(s + SM::SSLOT);
    auto bar = [&](int i) { return sb + SM::BAR + 8u * (uint32_t)i; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid < 4 * D) s_dl[tid] = 0.0f;  // ordered before use by the __syncthreads below
    if constexpr (D == 64) {  // the zero halves of both stages' Q and dO tiles (never written again)
        for (int i = tid; i < 4 * (int)SM::HALF / 16; i += kBtThreads) {
            const int h = i / (SM::HALF / 16), o = i % (SM::HALF / 16);  // h: stage 0/1, tile Q/dO
            *reinterpret_cast<uint4 *>(s + SM::STG + (h >> 1) * SM::QD + (2 * (h & 1) + 1) * SM::HALF + 16 * o) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        tc::fence_proxy_async_smem();  // generic-proxy stores -> tensor core reads
    }
    const int nunits = num_units[0];
    const int G = gridDim.x;
    const int mine = (int)blockIdx.x < nunits ? (nunits - 1 - (int)blockIdx.x) / G + 1 : 0;

    if (warp == kBtMmaWarp) tc::tmem_alloc(sb + SM::TMEM, 512);
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar(kBQdFull + i), 128);
            tc::mbar_init(bar(kBQdEmpty + i), 1);
            tc::mbar_init(bar(kBDqFull + i), 1);
            tc::mbar_init(bar(kBDqEmpty + i), 256);
        }
        for (int i = 0; i < 4; ++i) tc::mbar_init(bar(kBEReady + i), 128);
        tc::mbar_init(bar(kBKvFull), 1);
        tc::mbar_init(bar(kBKvEmpty), 1);
        tc::mbar_init(bar(kBSFull), 1);
        tc::mbar_init(bar(kBSEmpty), 128);
        tc::mbar_init(bar(kBDsFull), 128);
        tc::mbar_init(bar(kBDsEmpty), 1);
        tc::mbar_init(bar(kBAccFull), 1);
        tc::mbar_init(bar(kBAccEmpty), 256);
        tc::fence_mbar_init();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<uint32_t *>(s + SM::TMEM);
    bool ok = true;
    BtCursor cur{units, (int)blockIdx.x, G, mine};
    cur.load();

    if (warp >= kBtLoaderWarp0 && warp < kBtMmaWarp) {
        // ================= loaders: one pair row per thread for the metadata =================
        constexpr int CPR = D / 8, RPW = 32 / CPR, ITER = 32 / RPW;  // 16-byte chunks, rows per copy, copies
        const int lw = warp - kBtLoaderWarp0, lt = tid - 32 * kBtLoaderWarp0;
        const int rsub = lane / CPR, ch = lane % CPR;
        const int myr = 32 * lw + lane;
        // this thread's pair of the current tile: token row, weight, delta (fetched one tile ahead)
        auto fetch = [&](const BtCursor &t, int &row, float &wt, float &dl, int &sl) {
            const int p = t.i * kBtTile + myr;
            row = (!t.done() && p < t.u.count) ? pair_row[t.u.start + p] : -1;
            wt = row >= 0 ? pair_w[t.u.start + p] : 0.0f;
            dl = row >= 0 ? delta[row] : 0.0f;
            sl = (QSLC && row >= 0) ? pair_slot[t.u.start + p] : 0;
            if (QSLC && row >= 0) {  // the retrieval query's row is read by do_dl two tiles later: into L2 now
                const uint16_t *qr = Qs + (size_t)row * D;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(qr));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(qr + 64));
            }
        };
        int myrow, myslot;
        float myw, mydel;
        fetch(cur, myrow, myw, mydel, myslot);
        // dL_c += sum over a tile's pairs of ds q, computed here from the tile's Q rows just before the
        // stage is reloaded (the tile two back). Thread lt takes the 16-byte column chunk cc of pairs
        // 16 gq .. + 15; each loader warp keeps its own partial row in s_dl.
        BtCursor lag = cur;
        auto do_dl = [&]() {
            const int jl = lag.j, slot = jl & 3, stl = jl & 1;
            // qd_full (all loaders' copies of that tile) and e_ready (its ds) have completed long ago
            // and cannot run a phase ahead: the stage's next fill and that slot's next tile come after
            ok = ok && tc::mbar_wait(bar(kBQdFull + stl), (uint32_t)(jl >> 1) & 1u) &&
                 tc::mbar_wait(bar(kBEReady + slot), (uint32_t)(jl >> 2) & 1u);
            if (!ok) return;
            // CPR column chunks x (128 / CPR) groups of CPR pairs
            const int cc = lt % CPR, gq = lt / CPR;
            const unsigned char *qt = s + SM::STG + stl * SM::QD + (cc >> 3) * SM::HALF;
            float a8[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 4
            for (int i = 0; i < CPR; ++i) {
                const int p = CPR * gq + i;
                uint4 qv;
                if constexpr (QSLC) {  // the retrieval query's row (the stage's metadata is still this tile's)
                    const int rp = s_row[stl * 128 + p];
                    qv = rp >= 0 ? __ldg(reinterpret_cast<const uint4 *>(Qs + (size_t)rp * D + 8 * cc))
                                 : make_uint4(0u, 0u, 0u, 0u);
                } else {
                    qv = *reinterpret_cast<const uint4 *>(qt + tc::sw128(p, cc & 7));
                }
                const float dsp = e_ds[slot * 128 + p];
                a8[0] = fmaf(dsp, bf16_lo(qv.x), a8[0]); a8[1] = fmaf(dsp, bf16_hi(qv.x), a8[1]);
                a8[2] = fmaf(dsp, bf16_lo(qv.y), a8[2]); a8[3] = fmaf(dsp, bf16_hi(qv.y), a8[3]);
                a8[4] = fmaf(dsp, bf16_lo(qv.z), a8[4]); a8[5] = fmaf(dsp, bf16_hi(qv.z), a8[5]);
                a8[6] = fmaf(dsp, bf16_lo(qv.w), a8[6]); a8[7] = fmaf(dsp, bf16_hi(qv.w), a8[7]);
            }
#pragma unroll
            for (int o = CPR; o < 32; o <<= 1)  // the lanes of this warp with the same cc
#pragma unroll
                for (int k = 0; k < 8; ++k) a8[k] += __shfl_xor_sync(0xffffffffu, a8[k], o);
            float4 *own = reinterpret_cast<float4 *>(s_dl + lw * D + 8 * cc);  // only this lane writes these
            if (lane < CPR) {
                const float4 x0 = own[0], x1 = own[1];
                own[0] = make_float4(x0.x + a8[0], x0.y + a8[1], x0.z + a8[2], x0.w + a8[3]);
                own[1] = make_float4(x1.x + a8[4], x1.y + a8[5], x1.z + a8[6], x1.w + a8[7]);
            }
            if (lag.last_tile()) {  // the unit's dL: thread lt = column d
                const int bhl = lag.u.chunk / N / Gh, cl = lag.u.chunk % N;  // key head
                asm volatile("bar.sync 2, 128;" ::: "memory");  // every loader warp's partials are in s_dl
                if (lt < D)
                    atomicAdd(dL + ((size_t)bhl * N + cl) * D + lt,
                              scale * ((s_dl[lt] + s_dl[D + lt]) + (s_dl[2 * D + lt] + s_dl[3 * D + lt])));
                asm volatile("bar.sync 2, 128;" ::: "memory");  // all reads done before the owners reset
                if (lane < CPR) own[0] = own[1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
            lag.next();
        };
        for (; !cur.done() && ok; cur.next()) {
            const int j = cur.j, st = j & 1;
            const int bh = cur.u.chunk / N / Gh, c = cur.u.chunk % N;  // key head
            if (j >= 2) do_dl();  // the stage about to be reloaded holds tile j - 2
            ok = ok && tc::mbar_wait(bar(kBQdEmpty + st), ((uint32_t)(j >> 1) & 1u) ^ 1u);
            if (!ok) break;
            s_row[st * 128 + myr] = myrow;
            s_w[st * 128 + myr] = myw;
            s_del[st * 128 + myr] = mydel;
            if constexpr (QSLC) s_slot[st * 128 + myr] = myslot;
            const uint32_t sq = sb + SM::STG + st * SM::QD;
#pragma unroll
            for (int k = 0; k < ITER; ++k) {  // padding rows (token -1) are zero-filled
                const int r = 32 * lw + RPW * k + rsub;
                const int src = __shfl_sync(0xffffffffu, myrow, RPW * k + rsub);
                const uint32_t off = (ch >> 3) * SM::HALF + tc::sw128(r, ch & 7);
                cp_async16_u32(sq + off, src >= 0 ? (const void *)(Q + (size_t)src * D + ch * 8) : (const void *)Q,
                               src >= 0 ? 16 : 0);
                cp_async16_u32(sq + 2 * SM::HALF + off,
                               src >= 0 ? (const void *)(dout + (size_t)src * D + ch * 8) : (const void *)dout,
                               src >= 0 ? 16 : 0);
            }
            cp_async_commit();
            if (cur.first_tile() && lt == 0) {
                // the unit's K and V, once the previous unit's last MMA is done with them (the Q / dO
                // copies of this tile are already in flight); the next unit's tiles are prefetched to L2
                ok = tc::mbar_wait(bar(kBKvEmpty), ((uint32_t)cur.k & 1u) ^ 1u);
                if (ok) {
                    tc::mbar_arrive_expect_tx(bar(kBKvFull), 2 * KHALVES * SM::KH);
                    const int y = bh * T + c * kChunk;
#pragma unroll
                    for (int h = 0; h < KHALVES; ++h) {
                        tc::tma_load_2d(sb + SM::KO + h * SM::KH, &tmK, h * 64, y, bar(kBKvFull));
                        tc::tma_load_2d(sb + SM::VO + h * SM::KH, &tmV, h * 64, y, bar(kBKvFull));
                    }
                    if (cur.k + 1 < mine) {
                        const PairTile nu = units[blockIdx.x + (size_t)(cur.k + 1) * G];
                        const int yn = (nu.chunk / N / Gh) * T + (nu.chunk % N) * kChunk;
#pragma unroll
                        for (int h = 0; h < KHALVES; ++h) {
                            tc::tma_prefetch_2d(&tmK, h * 64, yn);
                            tc::tma_prefetch_2d(&tmV, h * 64, yn);
                        }
                    }
                }
            }
            {  // the next tile's metadata while the copies run
                BtCursor nx = cur;
                nx.next();
                fetch(nx, myrow, myw, mydel, myslot);
            }
            // publish this tile as soon as its copies have landed: the next stage frees only after the
            // previous tile's gradient MMAs, so waiting for it first would serialise the tiles
            cp_async_wait<0>();
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(bar(kBQdFull + st));
        }
        while (ok && !lag.done()) do_dl();  // the last tiles
        cp_async_wait<0>();
    } else if (warp == kBtMmaWarp) {
        // ================= MMA issuer =================
        if (mine > 0) {  // the whole warp runs the issue loop; one elected lane issues (tc::*_w)
            constexpr uint32_t id_s = tc::idesc_bf16(128, 64, 0, 0);   // S, dP': A, B K-major
            constexpr uint32_t id_q = tc::idesc_bf16(128, D, 0, 1);    // dQ: A K-major, B (K) MN-major
            constexpr uint32_t id_t = tc::idesc_bf16(128, 64, 1, 1);   // dK^T, dV^T: A, B MN-major (M = D, or
                                                                       // 128 with zero rows past D = 64)
            BtCursor cs = cur, cg = cur;  // S / dP' and gradient cursors
            uint32_t idle = 0;
            while (!cg.done()) {
                bool progress = false;
                if (cg.j < cs.j && tc::mbar_test(bar(kBDsFull), (uint32_t)cg.j & 1u) &&
                    tc::mbar_test(bar(kBDqEmpty + (cg.j & 1)), ((uint32_t)(cg.j >> 1) & 1u) ^ 1u) &&
                    (!cg.first_tile() || tc::mbar_test(bar(kBAccEmpty), ((uint32_t)cg.k & 1u) ^ 1u))) {
                    tc::fence_after();
                    const int st = cg.j & 1;
                    const uint32_t sq = sb + SM::STG + st * SM::QD, sdo = sq + 2 * SM::HALF;
#pragma unroll 1
                    for (int ks = 0; ks < kChunk / 16; ++ks)  // dQ = dS K: K = 64 keys
                        tc::mma_bf16_ss_w(tmem + SM::DQ_COL + st * 128, tc::desc_kmajor(sb + SM::DS + ks * 32),
                                        tc::desc_mnmajor(sb + SM::KO + ks * 2048, SM::KH), id_q, ks > 0 ? 1u : 0u);
                    const uint32_t acc0 = cg.first_tile() ? 0u : 1u;
#pragma unroll 1
                    for (int ks = 0; ks < kBtTile / 16; ++ks) {  // K = the tile's 128 pairs
                        tc::mma_bf16_ss_w(tmem + SM::DV_COL, tc::desc_mnmajor(sdo + ks * 2048, SM::HALF),
                                        tc::desc_mnmajor(sb + SM::WP + ks * 2048, 8192), id_t, ks > 0 ? 1u : acc0);
                        tc::mma_bf16_ss_w(tmem + SM::DK_COL, tc::desc_mnmajor(sq + ks * 2048, SM::HALF),
                                        tc::desc_mnmajor(sb + SM::DS + ks * 2048, 8192), id_t, ks > 0 ? 1u : acc0);
                    }
                    tc::commit_w(bar(kBDqFull + st));
                    tc::commit_w(bar(kBDsEmpty));
                    tc::commit_w(bar(kBQdEmpty + st));
                    if (cg.last_tile()) {
                        tc::commit_w(bar(kBAccFull));
                        tc::commit_w(bar(kBKvEmpty));
                    }
                    cg.next();
                    progress = true;
                }
                if (!cs.done() && cs.j < cg.j + 2 &&
                    tc::mbar_test(bar(kBQdFull + (cs.j & 1)), (uint32_t)(cs.j >> 1) & 1u) &&
                    tc::mbar_test(bar(kBSEmpty), ((uint32_t)cs.j & 1u) ^ 1u) &&
                    (!cs.first_tile() || tc::mbar_test(bar(kBKvFull), (uint32_t)cs.k & 1u))) {
                    tc::fence_after();
                    const int b = cs.j & 1;
                    const uint32_t sq = sb + SM::STG + b * SM::QD, sdo = sq + 2 * SM::HALF;
#pragma unroll 1
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t koff = (uint32_t)((ks >> 2) * SM::HALF + (ks & 3) * 32);
                        const uint32_t kk = (uint32_t)((ks >> 2) * SM::KH + (ks & 3) * 32);
                        tc::mma_bf16_ss_w(tmem + SM::S_COL, tc::desc_kmajor(sq + koff),
                                        tc::desc_kmajor(sb + SM::KO + kk), id_s, ks > 0 ? 1u : 0u);
                        tc::mma_bf16_ss_w(tmem + SM::DP_COL, tc::desc_kmajor(sdo + koff),
                                        tc::desc_kmajor(sb + SM::VO + kk), id_s, ks > 0 ? 1u : 0u);
                    }
                    tc::commit_w(bar(kBSFull));
                    cs.next();
                    progress = true;
                }
                if (progress) {
                    idle = 0;
                } else if (++idle > (1u << 26)) {
                    ok = false;
                    break;
                }
            }
        }
        __syncwarp();
    }
    else if (warp < kBtEpiWarp0) {
        // ================= compute: one pair row per thread (= TMEM lane) =================
        const int r = tid;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const float sl2 = scale * 1.4426950408889634f;
        for (; !cur.done() && ok; cur.next()) {
            const int j = cur.j, b = j & 1;
            const uint32_t ph = (uint32_t)(j >> 1) & 1u;
            // qd_full publishes the loaders' rows / weights / deltas of this stage; it cannot run a phase
            // ahead of this wait (stage b is reloaded only after this tile's gradient MMAs, which need
            // this warpgroup's ds_full)
            ok = tc::mbar_wait(bar(kBQdFull + b), ph) && tc::mbar_wait(bar(kBSFull), (uint32_t)j & 1u);
            if (!ok) break;
            tc::fence_after();
            const int row = s_row[b * 128 + r];
            const float w = s_w[b * 128 + r], del = s_del[b * 128 + r];
            if (cur.first_tile()) {
                // the unit's landmark row (fp32) for the ds L_c term of dQ, slot k % 4: the dQ epilogue
                // of unit k - 4 is done with that slot, since this tile's S needed unit k - 1's last
                // MMA, which needed the epilogue of a tile after unit k - 4's last
                const int bhu = cur.u.chunk / N / Gh, cu = cur.u.chunk % N;  // key head
                if (r < D) s_L[(cur.k & 3) * 128 + r] = __uint_as_float((uint32_t)L[((size_t)bhu * N + cu) * D + r] << 16);
            }
            const uint32_t tS = tmem + lane_off + SM::S_COL;
            const uint32_t tDP = tmem + lane_off + SM::DP_COL;
            {  // P = softmax over the chunk's 64 keys (fp32), written back over S
                float v0[32], v1[32];
                tc::tmem_ld32x2(tS, v0, tS + 32, v1);
                float m8[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    m8[k] = fmaxf(fmaxf(fmaxf(v0[k], v0[k + 8]), fmaxf(v0[k + 16], v0[k + 24])),
                                  fmaxf(fmaxf(v1[k], v1[k + 8]), fmaxf(v1[k + 16], v1[k + 24])));
                const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                const float mxs = mx * sl2;
                float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    v0[i] = ex2_approx(fmaf(v0[i], sl2, -mxs));
                    v1[i] = ex2_approx(fmaf(v1[i], sl2, -mxs));
                    l4[i & 3] += v0[i] + v1[i];
                }
                const float inv = 1.0f / ((l4[0] + l4[1]) + (l4[2] + l4[3]));
#pragma unroll
                for (int i = 0; i < 32; ++i) v0[i] *= inv;
                tc::tmem_st32f(tS, v0);
#pragma unroll
                for (int i = 0; i < 32; ++i) v1[i] *= inv;
                tc::tmem_st32f(tS + 32, v1);
            }
            float g4[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // g = sum over keys of P dP'
#pragma unroll 1
            for (int h = 0; h < 4; ++h) {
                float pv[16], dv[16];
                tc::tmem_ld16x2(tS + 16 * h, pv, tDP + 16 * h, dv);
#pragma unroll
                for (int i = 0; i < 16; ++i) g4[i & 3] = fmaf(pv[i], dv[i], g4[i & 3]);
            }
            const float g = (g4[0] + g4[1]) + (g4[2] + g4[3]);
            const float ds = row >= 0 ? w * (g - del) : 0.0f;
            if (QSLC && row >= 0) ds_pair[(size_t)row * Kslots + s_slot[b * 128 + r]] = ds;
            // w P and dS into shared memory once the previous tile's dQ / dK / dV MMAs have read them
            ok = tc::mbar_wait(bar(kBDsEmpty), ((uint32_t)j & 1u) ^ 1u);
            if (!ok) break;
#pragma unroll 1
            for (int h = 0; h < 4; ++h) {
                float pv[16], dv[16];
                tc::tmem_ld16x2(tS + 16 * h, pv, tDP + 16 * h, dv);
#pragma unroll
                for (int q = 0; q < 2; ++q) {  // 16-byte chunk 2h + q = keys 16h + 8q .. + 7
                    uint32_t a[4], d4[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float p0 = w * pv[8 * q + 2 * e], p1 = w * pv[8 * q + 2 * e + 1];
                        a[e] = pack_bf16x2(p0, p1);
                        d4[e] = pack_bf16x2(p0 * (dv[8 * q + 2 * e] - g), p1 * (dv[8 * q + 2 * e + 1] - g));
                    }
                    const uint32_t off = tc::sw128(r, 2 * h + q);
                    *reinterpret_cast<uint4 *>(s + SM::WP + off) = make_uint4(a[0], a[1], a[2], a[3]);
                    *reinterpret_cast<uint4 *>(s + SM::DS + off) = make_uint4(d4[0], d4[1], d4[2], d4[3]);
                }
            }
            tc::fence_before();
            tc::mbar_arrive(bar(kBSEmpty));  // P / dP' are consumed: S(j + 1) may overwrite them
            const int slot = j & 3;
            e_row[slot * 128 + r] = row;
            e_ds[slot * 128 + r] = ds;
            tc::fence_proxy_async_smem();  // w P / dS stores -> tensor core reads
            tc::mbar_arrive(bar(kBDsFull));
            tc::mbar_arrive(bar(kBEReady + slot));
        }
    } else {
        // ================= dQ epilogue: warpgroup e takes columns [D/2 e, D/2 e + D/2) =================
        const int e = (warp - kBtEpiWarp0) >> 2;
        const int r = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        unsigned char *wstage = s + SM::OUT + (warp - kBtEpiWarp0) * 32 * SM::OUT_ROW;
        unsigned char *stage = wstage + lane * SM::OUT_ROW;
        for (; !cur.done() && ok; cur.next()) {
            const int j = cur.j, b = j & 1;
            // e_ready (slot j % 4) cannot run a phase ahead: the compute warps write tile j + 4's rows
            // only after dQ(j + 3) was issued, which needs this warpgroup's dq_empty for tile j + 1
            const int slot = j & 3;
            ok = tc::mbar_wait(bar(kBEReady + slot), (uint32_t)(j >> 2) & 1u) &&
                 tc::mbar_wait(bar(kBDqFull + b), (uint32_t)(j >> 1) & 1u);
            if (!ok) break;
            tc::fence_after();
            const int row = e_row[slot * 128 + r];
            const float ds = QSLC ? 0.0f : e_ds[slot * 128 + r];  // the ds L_c term belongs to dQ only without Qs
            const float *Lr = s_L + (cur.k & 3) * 128;  // published with e_ready
#pragma unroll 1
            for (int cb = 0; cb < D / 2 / (int)SM::SLAB; ++cb) {
                const int col0 = D / 2 * e + cb * (int)SM::SLAB;
                float o[16];
                tc::tmem_ld16(tmem + lane_off + SM::DQ_COL + b * 128 + col0, o);
                __syncwarp();  // the previous slab has been read back
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<float4 *>(stage + q * 16) =
                        make_float4(scale * fmaf(ds, Lr[col0 + 4 * q], o[4 * q]),
                                    scale * fmaf(ds, Lr[col0 + 4 * q + 1], o[4 * q + 1]),
                                    scale * fmaf(ds, Lr[col0 + 4 * q + 2], o[4 * q + 2]),
                                    scale * fmaf(ds, Lr[col0 + 4 * q + 3], o[4 * q + 3]));
                __syncwarp();
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // each reduction: 8 rows x 64 contiguous bytes
                    const int rr = 8 * q + (lane >> 2), c4 = (lane & 3) * 4;
                    const int dst = __shfl_sync(0xffffffffu, row, rr);
                    const float4 val = *reinterpret_cast<const float4 *>(wstage + rr * SM::OUT_ROW + c4 * 4);
                    if (dst >= 0) red_add_v4(dQ + (size_t)dst * D + col0 + c4, val.x, val.y, val.z, val.w);
                }
            }
            tc::fence_before();
            tc::mbar_arrive(bar(kBDqEmpty + b));
            if (cur.last_tile()) {
                // the unit's dV (warpgroup 0) or dK (warpgroup 1): thread = column d = TMEM lane of
                // dV^T / dK^T; each warp-wide reduction covers one key row's 32 consecutive columns
                ok = tc::mbar_wait(bar(kBAccFull), (uint32_t)cur.k & 1u);
                if (!ok) break;
                tc::fence_after();
                const int bh = cur.u.chunk / N / Gh, c = cur.u.chunk % N;  // key head
                const size_t krow0 = (size_t)bh * T + (size_t)c * kChunk;
                float *dst = e == 0 ? dV : dK;
                const float f = e == 0 ? 1.0f : scale;
                const uint32_t tacc = tmem + lane_off + (e == 0 ? SM::DV_COL : SM::DK_COL);
                if ((warp & 3) * 32 < D) {  // lanes past D hold the zero rows of a head-dim-64 product
#pragma unroll 1
                    for (int h = 0; h < 2; ++h) {
                        float v[32];
                        tc::tmem_ld32(tacc + 32 * h, v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) atomicAdd(dst + (krow0 + 32 * h + i) * D + r, f * v[i]);
                    }
                }
                tc::fence_before();
                tc::mbar_arrive(bar(kBAccEmpty));
            }
        }
    }
    if (!ok) atomicOr(err, 1);
    tc::fence_before();
    __syncthreads();
    if (warp == kBtMmaWarp) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

cudaError_t launch_backward_tc(const BackwardArgs &a, cudaStream_t s) {
    if (a.D != 64 && a.D != 128) return cudaErrorInvalidValue;
    const size_t smem = BtSmem::DYN;
    auto kern = a.D == 128 ? (a.Qs ? chunk_bwd_tc_kernel<128, true> : chunk_bwd_tc_kernel<128, false>)
                           : (a.Qs ? chunk_bwd_tc_kernel<64, true> : chunk_bwd_tc_kernel<64, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const uint64_t rows = (uint64_t)a.B * a.Hkv * a.T;  // units address K, V by key head
    CUtensorMap tk, tv;
    if (!make_tmap_bf16(&tk, a.K, rows, a.D, kChunk) || !make_tmap_bf16(&tv, a.V, rows, a.D, kChunk))
        return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = sms < a.max_tiles ? sms : a.max_tiles;
    HSA_PROF("chunk_bwd", s);
    kern<<<grid, kBtThreads, smem, s>>>(a.Q, a.L, a.dout, a.delta, a.T, a.N, a.scale, a.tiles, a.num_tiles,
                                        a.pair_row, a.pair_w, a.dQ, a.dK, a.dV, a.dL, a.err, a.Qs, a.pair_slot,
                                        a.ds_pair, a.topk, a.H / a.Hkv, tk, tv);
    return cudaGetLastError();
}

}  // namespace hsa
