// attn_tc.cu -- Step 3 + Step 4 blend of the HSA forward on the 5th-generation tensor cores.
//
// Explainer page of "Every Token Counts", "How It Works (Technically)": every selected chunk is
// attended separately (Step 3) and the chunk outputs are blended by the retrieval softmax (Step 4).
// Work is chunk-major: one CTA takes a tile of up to 128 (token, weight) pairs that selected the
// same chunk c of one (batch, head).
//
//   smem      Q rows of the tile (gathered), K_c and V_c (64 x D), P (128 x 64) -- all bf16 in the
//             canonical 128-byte-swizzled layouts the tensor core reads; filled with cp.async.
//   TMEM      S = Q K_c^T (128 x 64 fp32) and O = P V_c (128 x D fp32), accumulated by tcgen05.mma
//             issued from one thread, completion signalled through an mbarrier.
//   softmax   one thread per pair row reads its S row from TMEM (tcgen05.ld), exact softmax over the
//             chunk's 64 keys in fp32, P rounded to bf16 into shared memory.
//   epilogue  O row * (w / rowsum) staged as fp32 in shared memory, then added into the token's
//             fp32 accumulator row with one bulk asynchronous reduction (cp.reduce.async.bulk .add.f32,
//             D*4 contiguous bytes) per pair.
#include "launch.h"
#include "profile.h"
#include "tc.cuh"

namespace hsa {

constexpr int kTcTile = 128;  // pairs per tile = MMA M
constexpr int kTcThreads = 128;

template <int D>
struct TcAttnSmem {
    static constexpr int KH = D / 64;                    // 64-element (128-byte) column blocks of D
    static constexpr uint32_t Q = 0;                     // KH x [128 rows][128 B]
    static constexpr uint32_t K = Q + KH * 16384;        // KH x [64 rows][128 B]
    static constexpr uint32_t V = K + KH * 8192;         // KH x [64 rows][128 B]
    static constexpr uint32_t P = V + KH * 8192;         // [128 rows][128 B]
    static constexpr uint32_t OPS = P + 16384;
    static constexpr uint32_t STAGE = D * 4 + 16;        // fp32 staging row stride (padded)
    static_assert(kTcTile * STAGE <= OPS, "staging must fit over the operand buffers");
    static constexpr uint32_t ROW = OPS;                 // int[128]
    static constexpr uint32_t W = ROW + 512;             // float[128]
    static constexpr uint32_t MBAR = W + 512;            // u64
    static constexpr uint32_t TMEM = MBAR + 8;           // u32
    static constexpr uint32_t BYTES = TMEM + 8;
    static constexpr size_t DYN = BYTES + 1024;          // + slack for 1 KB alignment
    static constexpr uint32_t TMEM_COLS = D == 128 ? 256 : 128;  // S: 64 columns, O: D columns
};

template <int D>
__global__ void __launch_bounds__(kTcThreads) chunk_attn_tc_kernel(
    const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K, const uint16_t *__restrict__ V, int T, int N,
    float scale, const PairTile *__restrict__ tiles, const int32_t *__restrict__ num_tiles,
    const int32_t *__restrict__ pair_row, const float *__restrict__ pair_w, float *__restrict__ o_acc,
    int32_t *__restrict__ err) {
    using SM = TcAttnSmem<D>;
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;  // 1 KB aligned base (swizzle atoms)
    unsigned char *s = smem_raw + (sb - raw);
    int *s_row = reinterpret_cast<int *>(s + SM::ROW);
    float *s_w = reinterpret_cast<float *>(s + SM::W);
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(s + SM::TMEM);
    const uint32_t mbar = sb + SM::MBAR;

    if ((int)blockIdx.x >= num_tiles[0]) return;
    const PairTile pt = tiles[blockIdx.x];
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = pt.chunk / N, c = pt.chunk % N;
    const uint16_t *Kc = K + ((size_t)bh * T + (size_t)c * kChunk) * D;
    const uint16_t *Vc = V + ((size_t)bh * T + (size_t)c * kChunk) * D;

    if (warp == 0) tc::tmem_alloc(sb + SM::TMEM, SM::TMEM_COLS);
    if (tid == 0) {
        tc::mbar_init(mbar, 1);
        tc::fence_mbar_init();
    }
    {
        const bool ok = tid < pt.count;
        s_row[tid] = ok ? pair_row[pt.start + tid] : -1;
        s_w[tid] = ok ? pair_w[pt.start + tid] : 0.0f;
    }
    __syncthreads();

    // ---- operands into swizzled shared memory (16-byte cp.async; consecutive lanes cover a row) ----
    for (int i = tid; i < kTcTile * CPR; i += kTcThreads) {
        const int r = i / CPR, ch = i % CPR;
        const int row = s_row[r];
        cp_async16(s + SM::Q + (ch >> 3) * 16384 + tc::sw128(r, ch & 7),
                   row >= 0 ? (const void *)(Q + (size_t)row * D + ch * 8) : (const void *)Q, row >= 0 ? 16 : 0);
    }
    for (int i = tid; i < kChunk * CPR; i += kTcThreads) {
        const int r = i / CPR, ch = i % CPR;
        cp_async16(s + SM::K + (ch >> 3) * 8192 + tc::sw128(r, ch & 7), Kc + (size_t)r * D + ch * 8, 16);
        cp_async16(s + SM::V + (ch >> 3) * 8192 + tc::sw128(r, ch & 7), Vc + (size_t)r * D + ch * 8, 16);
    }
    cp_async_commit();
    cp_async_wait<0>();
    tc::fence_proxy_async_smem();
    __syncthreads();
    tc::fence_after();

    const uint32_t tmem = *s_tmem;
    const uint32_t tS = tmem, tO = tmem + 64;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lanes
    bool failed = false;
    uint32_t pending_parity = 0;

    // ---- S = Q K_c^T (M = 128 pairs, N = 64 keys, K = D) ----
    if (tid == 0) {
        constexpr uint32_t idesc = tc::idesc_bf16(kTcTile, kChunk, 0, 0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t koff = (uint32_t)((ks & 3) * 32);  // K step inside a 128-byte row
            const uint64_t a = tc::desc_kmajor(sb + SM::Q + (ks >> 2) * 16384 + koff);
            const uint64_t b = tc::desc_kmajor(sb + SM::K + (ks >> 2) * 8192 + koff);
            tc::mma_bf16_ss(tS, a, b, idesc, ks > 0 ? 1u : 0u);
        }
        tc::commit(mbar);
    }
    failed = __syncthreads_or(!tc::mbar_wait(mbar, 0));
    if (!failed) {
        tc::fence_after();
        const int row = s_row[tid];
        // ---- exact softmax over the chunk's 64 keys (fp32), P -> bf16 in shared memory ----
        float s0[32], s1[32];
        tc::tmem_ld32(tS + lane_off, s0);
        tc::tmem_ld32(tS + lane_off + 32, s1);
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fmaxf(s0[i], s1[i]));
        const float sl2 = scale * 1.4426950408889634f;
        float l = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            s0[i] = exp2f((s0[i] - mx) * sl2);
            s1[i] = exp2f((s1[i] - mx) * sl2);
            l += s0[i] + s1[i];
        }
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
            const float *p = cc < 4 ? s0 + cc * 8 : s1 + (cc - 4) * 8;
            uint4 v;
            v.x = pack_bf16x2(p[0], p[1]);
            v.y = pack_bf16x2(p[2], p[3]);
            v.z = pack_bf16x2(p[4], p[5]);
            v.w = pack_bf16x2(p[6], p[7]);
            *reinterpret_cast<uint4 *>(s + SM::P + tc::sw128(tid, cc)) = v;
        }
        tc::fence_proxy_async_smem();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        // ---- O = P V_c (M = 128 pairs, N = D, K = 64 keys); V is the MN-major B operand ----
        if (tid == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16(kTcTile, D, 0, 1);
#pragma unroll
            for (int ks = 0; ks < kChunk / 16; ++ks) {
                const uint64_t a = tc::desc_kmajor(sb + SM::P + ks * 32);
                const uint64_t b = tc::desc_mnmajor(sb + SM::V + ks * 2048, 8192);
                tc::mma_bf16_ss(tO, a, b, idesc, ks > 0 ? 1u : 0u);
            }
            tc::commit(mbar);
        }
        pending_parity = 1;
        failed = __syncthreads_or(!tc::mbar_wait(mbar, 1));
        if (!failed) {
            tc::fence_after();
            // ---- epilogue: O row * (w / l) -> fp32 staging row -> bulk reduction into o_acc ----
            const float f = row >= 0 ? s_w[tid] / l : 0.0f;
            unsigned char *stage = s + tid * SM::STAGE;  // overlays the (consumed) operand buffers
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                float o[32];
                tc::tmem_ld32(tO + lane_off + cb * 32, o);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<float4 *>(stage + (cb * 32 + q * 4) * 4) =
                        make_float4(o[4 * q] * f, o[4 * q + 1] * f, o[4 * q + 2] * f, o[4 * q + 3] * f);
            }
            tc::fence_proxy_async_smem();
            if (row >= 0) tc::bulk_reduce_add_f32(o_acc + (size_t)row * D, sb + tid * SM::STAGE, D * 4);
            tc::bulk_commit();
            tc::bulk_wait_all();
        }
    }
    if (failed) {
        if (tid == 0) atomicOr(err, 1);
        tc::mbar_wait(mbar, pending_parity);  // bounded: let an MMA still in flight finish
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, SM::TMEM_COLS);
}

template <int D>
static cudaError_t launch_attn_tc_d(const ForwardArgs &a, cudaStream_t s) {
    const size_t smem = TcAttnSmem<D>::DYN;
    cudaError_t e = cudaFuncSetAttribute(chunk_attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    HSA_PROF("chunk_attn", s);
    chunk_attn_tc_kernel<D><<<a.max_tiles, kTcThreads, smem, s>>>(a.Q, a.K, a.V, a.T, a.N, a.scale, a.tiles,
                                                                   a.num_tiles, a.pair_row, a.pair_w, a.o_acc,
                                                                   a.err);
    return cudaGetLastError();
}

cudaError_t launch_attn_tc(const ForwardArgs &a, cudaStream_t s) {
    return a.D == 128 ? launch_attn_tc_d<128>(a, s) : launch_attn_tc_d<64>(a, s);
}

}  // namespace hsa
