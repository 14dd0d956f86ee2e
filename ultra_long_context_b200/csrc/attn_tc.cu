// attn_tc.cu -- Step 3 + Step 4 blend of the HSA forward on the 5th-generation tensor cores.
//
// Explainer page of "Every Token Counts", "How It Works (Technically)": every selected chunk is
// attended separately (Step 3) and the chunk outputs are blended by the retrieval softmax (Step 4).
// Work is chunk-major: a tile is up to 128 (token, weight) pairs that selected the same chunk c of
// one (batch, head); for a tile
//   S = Q_tile K_c^T   (128 x 64, fp32 in TMEM)      P = softmax over the 64 keys (bf16, in TMEM)
//   O = P V_c          (128 x D, fp32 in TMEM)       o_acc[token] += (w / rowsum) * O[row]
//
// Persistent, warp-specialised kernel, one CTA per SM, tiles assigned round-robin. Tile j of a CTA
// uses Q/K slot j % 2 (free again once S(j) is computed), V slot j % 3 (free once O(j) is computed)
// and TMEM buffers / warpgroups b = j % 2:
//   warps 16-19 loaders: the tile's Q rows gathered with cp.async (a warp-wide copy covers whole
//               256-byte rows) into the 128-byte-swizzled layout tcgen05 reads, up to two tiles of
//               copies in flight per thread; K_c and V_c as 64-row TMA tiles. Each loader thread's
//               arrival on the tile's barrier is tied to its copies (cp.async.mbarrier.arrive), so a
//               tile is published the moment its rows land; tile descriptors are fetched two tiles
//               ahead and token ids one tile ahead, so the loop never waits on a dependent load;
//   warp 20     MMA issuer: allocates TMEM; the warp runs the issue loop and one elected lane issues
//               S(j) = Q K^T and O(j) = P V as soon as each is ready (neither order is forced); O takes P straight from TMEM (A operand in
//               TMEM); completion via tcgen05.commit. S buffer b is free again as soon as O(j) has
//               read P, so the next softmax of a warpgroup overlaps the epilogue of the previous tile;
//   warps 0-7   two softmax warpgroups (b = 0, 1), one thread per pair row: S row from TMEM, exact
//               fp32 softmax, P (bf16) written back over its S columns; then the epilogue of the
//               first half of the O columns;
//   warps 8-15  two epilogue warpgroups (b = 0, 1): the second half of the O columns.
// The combine into the tokens' fp32 accumulator rows is bound by the rate of global reductions,
// which needs many warps issuing them: here 16 warps do, each red.global.add.v4.f32 covering
// 4 rows x 128 contiguous bytes (the O row, scaled by w / rowsum, goes 32 columns at a time through
// the warp's padded smem tile).
// Hand-offs (mbarriers, every wait bounded): qk_full / qk_empty, v_full / v_empty, s_full, p_full,
// o_full, s_empty (P consumed), o_empty (O buffer read by both epilogue halves), e_ready (token rows
// and scale factors of a tile handed from the softmax to the epilogue warpgroup).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "launch.h"
#include "profile.h"
#include "tc.cuh"

namespace hsa {

constexpr int kTcTile = 128;   // pairs per tile = MMA M
constexpr int kTcGroups = 2;   // TMEM buffers = softmax warpgroups = epilogue warpgroups
constexpr int kTcQkSlots = 2;  // Q + K operand slots
constexpr int kTcVSlots = 3;   // V operand slots (also index the per-tile token rows and weights)
constexpr int kTcEpiWarp0 = 4 * kTcGroups;                 // warps 8-15
constexpr int kTcLoaderWarps = 4;
constexpr int kTcLoaderWarp0 = kTcEpiWarp0 + 4 * kTcGroups;  // warps 16-19
constexpr int kTcMmaWarp = kTcLoaderWarp0 + kTcLoaderWarps;  // warp 20
constexpr int kTcThreads = 32 * (kTcMmaWarp + 1);

template <int D>
struct TcAttnSmem {
    static constexpr int KH = D / 64;                          // 128-byte column blocks of D
    static constexpr uint32_t QB = KH * 16384, KB = KH * 8192; // Q block [128][D], K or V block [64][D]
    static constexpr uint32_t QK = QB + KB;                    // one Q + K slot
    static constexpr uint32_t OPS = 0;                         // Q+K slots, then V slots
    static constexpr uint32_t VS = OPS + kTcQkSlots * QK;
    static constexpr uint32_t SLAB = 32;                       // epilogue columns per pass
    static constexpr int NSLAB = D / SLAB;
    // slabs [0, SPLIT) go to the softmax warpgroup, the rest to the epilogue warpgroup: the softmax
    // warpgroup's chain (softmax, wait for O, its slabs) is the longer one, so it takes fewer
    static constexpr int SPLIT = NSLAB >= 4 ? NSLAB / 4 : 1;
    static constexpr uint32_t OUT_ROW = SLAB * 4 + 16;         // fp32 staging row + pad (conflict-free)
    static constexpr uint32_t OUT = VS + kTcVSlots * KB;       // per epilogue warp: [32 rows][OUT_ROW]
    static constexpr uint32_t ROW = OUT + 16 * 32 * OUT_ROW;   // int[V slots][128]: token rows
    static constexpr uint32_t W = ROW + kTcVSlots * 512;       // float[V slots][128]: fusion weights
    static constexpr uint32_t EROW = W + kTcVSlots * 512;      // int[groups][2][128]: rows for the epilogue
    static constexpr uint32_t EF = EROW + kTcGroups * 2 * 512; // float[groups][2][128]: w / rowsum
    static constexpr uint32_t BAR = EF + kTcGroups * 2 * 512;  // mbarriers
    static constexpr int NBAR = 2 * kTcQkSlots + 2 * kTcVSlots + 7 * kTcGroups;
    static constexpr uint32_t TMEM = BAR + NBAR * 8;
    static constexpr uint32_t BYTES = TMEM + 16;
    static constexpr size_t DYN = BYTES + 1024;                // slack for the 1 KB alignment
    static constexpr uint32_t S_COL = 0;                       // S / P buffers: columns [0, 128)
    static constexpr uint32_t O_COL = 128;                     // O buffers: columns [128, 128 + 2D)
    static constexpr uint32_t TMEM_COLS = D == 128 ? 512 : 256;
    static_assert(DYN <= 227 * 1024, "shared memory budget");
};

// mbarrier slots
enum { kQkFull = 0, kQkEmpty = kTcQkSlots, kVFull = 2 * kTcQkSlots, kVEmpty = kVFull + kTcVSlots,
       kSFull = kVEmpty + kTcVSlots, kPFull = kSFull + kTcGroups,
       kOFull = kPFull + kTcGroups, kSEmpty = kOFull + kTcGroups, kOEmpty = kSEmpty + kTcGroups,
       kEReady = kOEmpty + kTcGroups /* [group][2 slots] */ };

// Arrive on an mbarrier once every cp.async this thread has issued so far has completed (the arrival
// counts against the barrier's expected count: no increment first).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t mbar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(mbar) : "memory");
}

// Slabs [cb0, cb1) of 32 O columns of one tile, scaled by f and added into the tokens' fp32 rows:
// TMEM (thread = row) -> this warp's padded smem tile -> read back so that each warp-wide reduction
// covers 4 rows x 128 contiguous bytes.
template <int D>
__device__ __forceinline__ void epilogue_slabs(uint32_t tO, int cb0, int cb1, int row, float f, unsigned char *wstage,
                                               int lane, float *__restrict__ o_acc) {
    using SM = TcAttnSmem<D>;
    unsigned char *stage = wstage + lane * SM::OUT_ROW;
#pragma unroll 1
    for (int cb = cb0; cb < cb1; ++cb) {
        float o[32];
        tc::tmem_ld32(tO + cb * SM::SLAB, o);
        __syncwarp();  // the previous slab has been read back
#pragma unroll
        for (int q = 0; q < 8; ++q)
            *reinterpret_cast<float4 *>(stage + q * 16) =
                make_float4(o[4 * q] * f, o[4 * q + 1] * f, o[4 * q + 2] * f, o[4 * q + 3] * f);
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int rr = 4 * q + (lane >> 3), c4 = (lane & 7) * 4;
            const int dst = __shfl_sync(0xffffffffu, row, rr);
            const float4 val = *reinterpret_cast<const float4 *>(wstage + rr * SM::OUT_ROW + c4 * 4);
            if (dst >= 0) red_add_v4(o_acc + (size_t)dst * D + cb * SM::SLAB + c4, val.x, val.y, val.z, val.w);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) chunk_attn_tc_kernel(
    const uint16_t *__restrict__ Q, int T, int N, int Gh, float scale, const PairTile *__restrict__ tiles,
    const int32_t *__restrict__ num_tiles, const int32_t *__restrict__ pair_row, const float *__restrict__ pair_w,
    float *__restrict__ o_acc, int32_t *__restrict__ err, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV) {
    // launched as a programmatic dependent of the dispatch: its tile list first. No early release of the
    // finalize: its blocks would sit beside this persistent kernel's for its whole run.
    pdl_wait();
    using SM = TcAttnSmem<D>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;  // 1 KB aligned (swizzle atoms)
    unsigned char *s = smem_raw + (sb - raw);
    int *s_row = reinterpret_cast<int *>(s + SM::ROW);
    float *s_w = reinterpret_cast<float *>(s + SM::W);
    int *e_row = reinterpret_cast<int *>(s + SM::EROW);
    float *e_f = reinterpret_cast<float *>(s + SM::EF);
    auto bar = [&](int i) { return sb + SM::BAR + 8u * (uint32_t)i; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntiles = num_tiles[0];
    const int G = gridDim.x;
    const int mine = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / G + 1 : 0;

    if (warp == kTcMmaWarp) tc::tmem_alloc(sb + SM::TMEM, SM::TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < kTcQkSlots; ++i) {
            tc::mbar_init(bar(kQkFull + i), 32 * kTcLoaderWarps);  // loader arrivals after their Q copies (+ K bytes)
            tc::mbar_init(bar(kQkEmpty + i), 1);
        }
        for (int i = 0; i < kTcVSlots; ++i) {
            tc::mbar_init(bar(kVFull + i), 32 * kTcLoaderWarps);   // loader arrivals after the rows / weights (+ V bytes)
            tc::mbar_init(bar(kVEmpty + i), 1);
        }
        for (int i = 0; i < kTcGroups; ++i) {
            tc::mbar_init(bar(kSFull + i), 1);
            tc::mbar_init(bar(kPFull + i), kTcTile);
            tc::mbar_init(bar(kOFull + i), 1);
            tc::mbar_init(bar(kSEmpty + i), 1);
            tc::mbar_init(bar(kOEmpty + i), 2 * kTcTile);
            tc::mbar_init(bar(kEReady + 2 * i), kTcTile);
            tc::mbar_init(bar(kEReady + 2 * i + 1), kTcTile);
        }
        tc::fence_mbar_init();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<uint32_t *>(s + SM::TMEM);
    bool ok = true;

    if (warp >= kTcLoaderWarp0 && warp < kTcMmaWarp) {
        // ================= loaders =================
        constexpr int CPR = D / 8;        // 16-byte chunks per row
        constexpr int RPW = 32 / CPR;     // rows per warp-wide load: 2 (D = 128) or 4 (D = 64)
        constexpr int ITER = 32 / RPW;    // loads per thread per tile
        const int lw = warp - kTcLoaderWarp0, lt = tid - 32 * kTcLoaderWarp0;
        const int rsub = lane / CPR, ch = lane % CPR;
        const int myr = 32 * lw + lane;  // the tile row whose token id this thread fetches
        // descriptors run two tiles ahead and token ids one tile ahead, so no load the loop waits on
        // is issued less than a tile before it is needed
        PairTile t = mine > 0 ? tiles[blockIdx.x] : PairTile{0, 0, 0, 0};
        PairTile t_next = mine > 1 ? tiles[blockIdx.x + G] : PairTile{0, 0, 0, 0};
        int myrow = (mine > 0 && myr < t.count) ? pair_row[t.start + myr] : -1;
        float myw = (mine > 0 && myr < t.count) ? pair_w[t.start + myr] : 0.0f;
        for (int j = 0; j < mine && ok; ++j) {
            const int sq = j % kTcQkSlots, sv = j % kTcVSlots;
            ok = tc::mbar_wait(bar(kQkEmpty + sq), ((uint32_t)(j / kTcQkSlots) & 1u) ^ 1u) &&
                 tc::mbar_wait(bar(kVEmpty + sv), ((uint32_t)(j / kTcVSlots) & 1u) ^ 1u);
            if (!ok) break;
            const uint32_t sqa = sb + SM::OPS + sq * SM::QK;
            if (lt == 0) {
                const int kvh = t.chunk / N / Gh, c = t.chunk % N;  // Gh query heads per key head
                tc::mbar_expect_tx(bar(kQkFull + sq), SM::KB);  // this thread arrives below, after its copies
                tc::mbar_expect_tx(bar(kVFull + sv), SM::KB);
                const int y = kvh * T + c * kChunk;
#pragma unroll
                for (int h = 0; h < SM::KH; ++h) {
                    tc::tma_load_2d(sqa + SM::QB + h * 8192, &tmK, h * 64, y, bar(kQkFull + sq));
                    tc::tma_load_2d(sb + SM::VS + sv * SM::KB + h * 8192, &tmV, h * 64, y, bar(kVFull + sv));
                }
            }
            s_row[sv * kTcTile + myr] = myrow;
            s_w[sv * kTcTile + myr] = myw;
            tc::mbar_arrive(bar(kVFull + sv));
#pragma unroll
            for (int k = 0; k < ITER; ++k) {  // padding rows (token -1) are zero-filled
                const int r = 32 * lw + RPW * k + rsub;
                const int src = __shfl_sync(0xffffffffu, myrow, RPW * k + rsub);
                cp_async16_u32(sqa + (ch >> 3) * 16384 + tc::sw128(r, ch & 7),
                               src >= 0 ? (const void *)(Q + (size_t)src * D + ch * 8) : (const void *)Q,
                               src >= 0 ? 16 : 0);
            }
            cp_async_commit();
            // this thread's arrival on qk_full fires by itself once its copies so far (this tile's among
            // them) have landed, so a tile is published when its rows are in shared memory, whatever
            // the loader waits for next; the MMA thread fences the proxies after its wait
            cp_async_mbar_arrive_noinc(bar(kQkFull + sq));
            // the next tile's token ids (its descriptor is already here) and the descriptor after it,
            // fetched while the copies run
            if (j + 1 < mine) {
                t = t_next;
                const bool valid = myr < t.count;
                myrow = valid ? pair_row[t.start + myr] : -1;
                myw = valid ? pair_w[t.start + myr] : 0.0f;
                if (j + 2 < mine) t_next = tiles[blockIdx.x + (size_t)(j + 2) * G];
            }
        }
        cp_async_wait<0>();  // nothing in flight when the CTA exits
    } else if (warp == kTcMmaWarp) {
        // ================= MMA issuer: the whole warp runs the loop, one elected lane issues =================
        if (mine > 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16(kTcTile, kChunk, 0, 0);
            constexpr uint32_t idesc_o = tc::idesc_bf16(kTcTile, D, 0, 1);
            auto issue_s = [&](int jj) {  // S(jj) = Q(jj) K_c(jj)^T into TMEM buffer jj % 2
                const int b = jj & 1;
                const uint32_t sq = sb + SM::OPS + (jj % kTcQkSlots) * SM::QK;
                const uint32_t sk = sq + SM::QB;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t koff = (uint32_t)((ks & 3) * 32);  // K step inside a 128-byte row
                    tc::mma_bf16_ss_w(tmem + SM::S_COL + b * kChunk, tc::desc_kmajor(sq + (ks >> 2) * 16384 + koff),
                                    tc::desc_kmajor(sk + (ks >> 2) * 8192 + koff), idesc_s, ks > 0 ? 1u : 0u);
                }
                tc::commit_w(bar(kSFull + b));
                tc::commit_w(bar(kQkEmpty + jj % kTcQkSlots));  // Q and K are free once S is computed
            };
            auto issue_o = [&](int jj) {  // O(jj) = P(jj) V_c(jj), P read from TMEM
                const int b = jj & 1;
                const uint32_t sv = sb + SM::VS + (jj % kTcVSlots) * SM::KB;
#pragma unroll
                for (int ks = 0; ks < kChunk / 16; ++ks)
                    tc::mma_bf16_ts_w(tmem + SM::O_COL + b * D, tmem + SM::S_COL + b * kChunk + ks * 8,
                                    tc::desc_mnmajor(sv + ks * 2048, 8192), idesc_o, ks > 0 ? 1u : 0u);
                tc::commit_w(bar(kOFull + b));
                tc::commit_w(bar(kSEmpty + b));                // P has been read: S buffer b is free
                tc::commit_w(bar(kVEmpty + jj % kTcVSlots));   // and V slot jj % 3
            };
            // Issue whichever is ready first: O(next_o) once its P is in TMEM and the epilogue of tile
            // next_o - 2 has read O buffer b, or S(next_s) once its operands have landed and O(next_s - 2)
            // has consumed P. The probe loop is bounded: a long stretch without progress is an error.
            int next_s = 0, next_o = 0;
            uint32_t idle = 0;
            while (next_o < mine) {
                bool progress = false;
                if (next_o < next_s && tc::mbar_test(bar(kPFull + (next_o & 1)), (uint32_t)(next_o >> 1) & 1u) &&
                    tc::mbar_test(bar(kOEmpty + (next_o & 1)), ((uint32_t)(next_o >> 1) & 1u) ^ 1u) &&
                    tc::mbar_test(bar(kVFull + next_o % kTcVSlots), (uint32_t)(next_o / kTcVSlots) & 1u)) {
                    tc::fence_after();
                    issue_o(next_o++);
                    progress = true;
                }
                if (next_s < mine && next_s < next_o + kTcGroups &&
                    tc::mbar_test(bar(kQkFull + next_s % kTcQkSlots), (uint32_t)(next_s / kTcQkSlots) & 1u) &&
                    tc::mbar_test(bar(kSEmpty + (next_s & 1)), ((uint32_t)(next_s >> 1) & 1u) ^ 1u)) {
                    tc::fence_after();
                    tc::fence_proxy_async_smem();  // the Q rows came by cp.async (generic proxy)
                    issue_s(next_s++);
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
    } else {
        // ================= softmax (warps 0-7) and epilogue (warps 0-15) =================
        const bool softmax = warp < kTcEpiWarp0;
        const int g = (warp >> 2) & 1;                        // TMEM buffer / tile parity
        const int r = (warp & 3) * 32 + lane;                 // pair row = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const float sl2 = scale * 1.4426950408889634f;
        unsigned char *wstage = s + SM::OUT + warp * 32 * SM::OUT_ROW;  // this warp's 32 staging rows
        const uint32_t tS = tmem + lane_off + SM::S_COL + g * kChunk;
        const uint32_t tO = tmem + lane_off + SM::O_COL + g * D;
        for (int j = g; j < mine && ok; j += kTcGroups) {
            const int sv = j % kTcVSlots;
            const uint32_t ph = (uint32_t)(j >> 1) & 1u;
            const int slot = (j >> 1) & 1;  // e_row / e_f double buffer of this group
            int row;
            float f;
            if (softmax) {
                // v_full also publishes the loaders' token rows and weights of this tile; it cannot run a
                // phase ahead of this wait (tile j + 3 needs V slot j % 3, freed only by O(j))
                ok = tc::mbar_wait(bar(kVFull + sv), (uint32_t)(j / kTcVSlots) & 1u) &&
                     tc::mbar_wait(bar(kSFull + g), ph);
                if (!ok) break;
                tc::fence_after();
                row = s_row[sv * kTcTile + r];
                const float w = s_w[sv * kTcTile + r];
                float s0[32], s1[32];
                tc::tmem_ld32(tS, s0);
                tc::tmem_ld32(tS + 32, s1);
                float m8[8];  // row max as a tree (no 64-deep dependent chain)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    m8[k] = fmaxf(fmaxf(s0[k], s0[k + 8]), fmaxf(s0[k + 16], s0[k + 24]));
                    m8[k] = fmaxf(m8[k], fmaxf(fmaxf(s1[k], s1[k + 8]), fmaxf(s1[k + 16], s1[k + 24])));
                }
                const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                const float mxs = mx * sl2;
                float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                uint32_t pk[32];  // P row as bf16 pairs: the A operand of O = P V, written over S
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    // exponent <= 0: exp2 of (s - max) * scale * log2(e) by the MUFU instruction
                    const float a0 = ex2_approx(fmaf(s0[2 * i], sl2, -mxs)), a1 = ex2_approx(fmaf(s0[2 * i + 1], sl2, -mxs));
                    const float b0 = ex2_approx(fmaf(s1[2 * i], sl2, -mxs)), b1 = ex2_approx(fmaf(s1[2 * i + 1], sl2, -mxs));
                    l4[i & 3] += (a0 + a1) + (b0 + b1);
                    pk[i] = pack_bf16x2(a0, a1);
                    pk[16 + i] = pack_bf16x2(b0, b1);
                }
                const float l = (l4[0] + l4[1]) + (l4[2] + l4[3]);
                tc::tmem_st32(tS, pk);
                f = row >= 0 ? w / l : 0.0f;
                tc::fence_before();
                tc::mbar_arrive(bar(kPFull + g));
                e_row[(g * 2 + slot) * kTcTile + r] = row;  // for the other half of the epilogue
                e_f[(g * 2 + slot) * kTcTile + r] = f;
                tc::mbar_arrive(bar(kEReady + g * 2 + slot));
                ok = tc::mbar_wait(bar(kOFull + g), ph);
            } else {
                // e_ready (one per group and slot, a phase per 4 tiles) orders the softmax threads'
                // e_row / e_f stores before these loads; it cannot run a phase ahead of this wait, as
                // tile j + 4 needs this warpgroup's o_empty arrival for tile j first
                ok = tc::mbar_wait(bar(kEReady + g * 2 + slot), (uint32_t)(j >> 2) & 1u) &&
                     tc::mbar_wait(bar(kOFull + g), ph);
                row = e_row[(g * 2 + slot) * kTcTile + r];
                f = e_f[(g * 2 + slot) * kTcTile + r];
            }
            if (!ok) break;
            tc::fence_after();
            epilogue_slabs<D>(tO, softmax ? 0 : SM::SPLIT, softmax ? SM::SPLIT : SM::NSLAB, row, f, wstage, lane,
                              o_acc);
            tc::fence_before();
            tc::mbar_arrive(bar(kOEmpty + g));
        }
    }
    if (!ok) atomicOr(err, 1);
    tc::fence_before();
    __syncthreads();
    if (warp == kTcMmaWarp) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, SM::TMEM_COLS);
    }
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2D bf16 tensor [rows, D] (row stride D * 2 bytes), boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool make_tmap_bf16(CUtensorMap *m, const void *base, uint64_t rows, int D, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_attn_tc_d(const ForwardArgs &a, cudaStream_t s) {
    const size_t smem = TcAttnSmem<D>::DYN;
    cudaError_t e = cudaFuncSetAttribute(chunk_attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const uint64_t rows = (uint64_t)a.B * a.Hkv * a.T;  // tiles address K, V by key head
    CUtensorMap tk, tv;
    if (!make_tmap_bf16(&tk, a.K, rows, D, kChunk) || !make_tmap_bf16(&tv, a.V, rows, D, kChunk)) return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = sms < a.max_tiles ? sms : a.max_tiles;
    HSA_PROF("chunk_attn", s);
    e = launch_pdl(chunk_attn_tc_kernel<D>, dim3(grid), dim3(kTcThreads), smem, s, a.Q, a.T, a.N, a.H / a.Hkv,
                   a.scale, (const PairTile *)a.tiles, (const int32_t *)a.num_tiles, (const int32_t *)a.pair_row,
                   (const float *)a.pair_w, a.o_acc, a.err, tk, tv);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_attn_tc(const ForwardArgs &a, cudaStream_t s) {
    return a.D == 128 ? launch_attn_tc_d<128>(a, s) : launch_attn_tc_d<64>(a, s);
}

}  // namespace hsa
