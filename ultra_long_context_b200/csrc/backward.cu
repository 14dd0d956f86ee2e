// backward.cu -- gradients of the HSA forward for the selection the forward made.
//
// Explainer page of "Every Token Counts", "How It Works (Technically)", Step 4: because the fusion
// weight w = softmax(s over the selected chunks) multiplies the output, the loss gradient reaches
// the retrieval scores and through them the landmarks; the discrete top-K choice itself is held
// fixed. Per (token t, selected chunk c) pair with weight w and chunk output O_c = P V_c,
// P = softmax(scale * q K_c^T):
//   g    = dO . O_c                      (= rowsum(P * dP'), dP' = dO V_c^T)
//   ds   = w (g - delta_t),  delta_t = dO . O_t                       (fusion-softmax Jacobian)
//   dS   = w P * (dP' - g)                                             (in-chunk softmax Jacobian)
//   dQ_t += scale dS K_c + scale ds L_c;     dK_c += scale dS^T q;     dV_c += w P^T dO
//   dL_c += scale ds q
// The pairs are processed chunk-major with the same dispatch as the forward (tiles of <= 64 pairs
// of one chunk): the chunk's K, V and the tile's gathered Q, dO rows sit in shared memory, the five
// contractions run on the tensor cores, and every gradient is accumulated with fp32 vector
// reductions (a chunk may span several tiles, a token several chunks). This file holds the delta
// kernel, the head-dim-64 chunk kernel (mma.sync; head dim 128 runs bwd_tc.cu), the query-gradient
// finish for a separate retrieval query or query-key normalisation, and the launch sequence.
#include "common.cuh"
#include "launch.h"
#include "profile.h"

namespace hsa {

// delta_t = dO_t . O_t (bf16 inputs, fp32). D/8 lanes per token row (one 16-byte vector each), and
// kDeltaGroups groups of rows per warp whose loads are all in flight before the first product: the
// kernel streams out and dout once and is bound by HBM.
constexpr int kDeltaGroups = 4;

template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const uint16_t *__restrict__ out, const uint16_t *__restrict__ dout,
                                                    size_t rows, float *__restrict__ delta) {
    constexpr int LPR = D / 8, RPW = 32 / LPR;  // lanes per row, rows per warp-wide load
    const int lane = threadIdx.x & 31, sub = lane % LPR, rw = lane / LPR;
    const size_t warp_g = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const size_t row0 = warp_g * (RPW * kDeltaGroups) + rw;
    uint4 o[kDeltaGroups], g[kDeltaGroups];
#pragma unroll
    for (int u = 0; u < kDeltaGroups; ++u) {
        const size_t r = row0 + (size_t)u * RPW;
        o[u] = r < rows ? *reinterpret_cast<const uint4 *>(out + r * D + sub * 8) : make_uint4(0u, 0u, 0u, 0u);
        g[u] = r < rows ? *reinterpret_cast<const uint4 *>(dout + r * D + sub * 8) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kDeltaGroups; ++u) {
        float acc = 0.0f;
        acc = fmaf(bf16_lo(o[u].x), bf16_lo(g[u].x), acc); acc = fmaf(bf16_hi(o[u].x), bf16_hi(g[u].x), acc);
        acc = fmaf(bf16_lo(o[u].y), bf16_lo(g[u].y), acc); acc = fmaf(bf16_hi(o[u].y), bf16_hi(g[u].y), acc);
        acc = fmaf(bf16_lo(o[u].z), bf16_lo(g[u].z), acc); acc = fmaf(bf16_hi(o[u].z), bf16_hi(g[u].z), acc);
        acc = fmaf(bf16_lo(o[u].w), bf16_lo(g[u].w), acc); acc = fmaf(bf16_hi(o[u].w), bf16_hi(g[u].w), acc);
#pragma unroll
        for (int x = LPR / 2; x > 0; x >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, x);
        const size_t r = row0 + (size_t)u * RPW;
        if (sub == 0 && r < rows) delta[r] = acc;
    }
}

constexpr int kBwdThreads = 128;  // 4 warps x 16 pairs

template <int D>
struct BwdSmem {
    static constexpr int SD = D + 8, SP = kChunk + 8;
    static constexpr size_t mat = (size_t)kChunk * SD * 2;  // one [64][SD] bf16 tile
    static constexpr size_t pm = (size_t)kPairTile * SP * 2;
    static constexpr size_t total = 4 * mat + 2 * pm;
};

// acc[m-tile rows 16][n] += A(16 x 64, from a [64][SP] or [64][SD] bf16 tile read transposed) * B
// Helper for the two "transposed" contractions dV_c = (wP)^T dO and dK_c = dS^T Q, where the
// reduction runs over the tile's 64 pairs: A[m = key][k = pair] = X[pair][key] (ldmatrix.trans),
// B[k = pair][n = d] = Y[pair][d] (ldmatrix.trans).
template <int D>
__device__ __forceinline__ void contract_over_pairs(float (&acc)[D / 8][4], const uint16_t *X, int sx,
                                                    const uint16_t *Y, int sy, int m0, int lane) {
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[nt][r] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < kPairTile / 16; ++kk) {
        uint32_t a[4];
        ldmatrix_x4_trans(a[0], a[1], a[2], a[3],
                          X + (kk * 16 + (lane & 7) + (lane >> 4) * 8) * sx + m0 + ((lane >> 3) & 1) * 8);
#pragma unroll
        for (int np = 0; np < D / 16; ++np) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(b0, b1, b2, b3,
                              Y + (kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * sy + np * 16 + (lane >> 4) * 8);
            mma_bf16_16816(acc[2 * np], a, b0, b1);
            mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
        }
    }
}

// S-shaped contraction: out(16 pairs x 64 keys) = A(16 x D rows of a [64][SD] tile) * B^T where
// B is a [64 keys][SD] tile (non-transposed ldmatrix, as for Q K^T).
template <int D>
__device__ __forceinline__ void contract_rows_keys(float (&s)[8][4], const uint16_t *A, const uint16_t *Bm, int row0,
                                                   int lane) {
    constexpr int SD = D + 8;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) s[nt][r] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4];
        ldmatrix_x4(a[0], a[1], a[2], a[3], A + (row0 + (lane & 15)) * SD + ks * 16 + (lane >> 4) * 8);
#pragma unroll
        for (int np = 0; np < 4; ++np) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4(b0, b1, b2, b3,
                        Bm + (np * 16 + (lane & 7) + (lane >> 4) * 8) * SD + ks * 16 + ((lane >> 3) & 1) * 8);
            mma_bf16_16816(s[2 * np], a, b0, b1);
            mma_bf16_16816(s[2 * np + 1], a, b2, b3);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads) chunk_bwd_kernel(
    const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K, const uint16_t *__restrict__ V,
    const uint16_t *__restrict__ L, const uint16_t *__restrict__ dout, const float *__restrict__ delta, int T, int N,
    float scale, const PairTile *__restrict__ tiles, const int32_t *__restrict__ num_tiles,
    const int32_t *__restrict__ pair_row, const float *__restrict__ pair_w, float *__restrict__ dQ,
    float *__restrict__ dK, float *__restrict__ dV, float *__restrict__ dL, const uint16_t *__restrict__ Qs,
    const int32_t *__restrict__ pair_slot, float *__restrict__ ds_pair, int Kslots, int Gh) {
    // Qs != NULL: separate retrieval queries. dL takes ds times the retrieval query, dQ leaves out the
    // ds L_c term, and ds goes to ds_pair[token row, slot] for the retrieval query's gradient.
    using SM = BwdSmem<D>;
    constexpr int SD = SM::SD, SP = SM::SP, VPR = D / 8;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint16_t *sK = reinterpret_cast<uint16_t *>(smem_raw);
    uint16_t *sV = sK + kChunk * SD;
    uint16_t *sQ = sV + kChunk * SD;
    uint16_t *sG = sQ + kChunk * SD;        // gathered dO rows
    uint16_t *sP = sG + kChunk * SD;        // w P     [pair][key]
    uint16_t *sdS = sP + kPairTile * SP;    // dS      [pair][key]
    __shared__ int s_row[kPairTile], s_slot[kPairTile];
    __shared__ float s_w[kPairTile], s_ds[kPairTile], s_L[D];

    if ((int)blockIdx.x >= num_tiles[0]) return;
    const PairTile pt = tiles[blockIdx.x];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bh = pt.chunk / N / Gh, c = pt.chunk % N;  // key head (Gh query heads per key head)
    const size_t krow0 = (size_t)bh * T + (size_t)c * kChunk;
    if (tid < kPairTile) {
        const bool ok = tid < pt.count;
        s_row[tid] = ok ? pair_row[pt.start + tid] : -1;
        s_w[tid] = ok ? pair_w[pt.start + tid] : 0.0f;
        s_slot[tid] = ok && Qs ? pair_slot[pt.start + tid] : 0;
    }
    for (int d = tid; d < D; d += kBwdThreads) s_L[d] = __uint_as_float((uint32_t)L[((size_t)bh * N + c) * D + d] << 16);
    __syncthreads();
    for (int i = tid; i < kChunk * VPR; i += kBwdThreads) {
        const int r = i / VPR, v = i % VPR;
        cp_async16(sK + r * SD + v * 8, K + (krow0 + r) * D + v * 8, 16);
        cp_async16(sV + r * SD + v * 8, V + (krow0 + r) * D + v * 8, 16);
        const int row = s_row[r];
        cp_async16(sQ + r * SD + v * 8, row >= 0 ? (const void *)(Q + (size_t)row * D + v * 8) : (const void *)Q,
                   row >= 0 ? 16 : 0);
        cp_async16(sG + r * SD + v * 8, row >= 0 ? (const void *)(dout + (size_t)row * D + v * 8) : (const void *)dout,
                   row >= 0 ? 16 : 0);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();

    const int r0 = warp * 16;
    const int p0 = r0 + (lane >> 2), p1 = p0 + 8;
    // P = softmax(scale * q K_c^T), normalised, rows p0 / p1
    float P[8][4];
    contract_rows_keys<D>(P, sQ, sK, r0, lane);
    {
        const float sl2 = scale * 1.4426950408889634f;
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            mx0 = fmaxf(mx0, fmaxf(P[nt][0], P[nt][1]));
            mx1 = fmaxf(mx1, fmaxf(P[nt][2], P[nt][3]));
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        float z0 = 0.0f, z1 = 0.0f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            P[nt][0] = exp2f((P[nt][0] - mx0) * sl2);
            P[nt][1] = exp2f((P[nt][1] - mx0) * sl2);
            P[nt][2] = exp2f((P[nt][2] - mx1) * sl2);
            P[nt][3] = exp2f((P[nt][3] - mx1) * sl2);
            z0 += P[nt][0] + P[nt][1];
            z1 += P[nt][2] + P[nt][3];
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            z0 += __shfl_xor_sync(0xffffffffu, z0, o);
            z1 += __shfl_xor_sync(0xffffffffu, z1, o);
        }
        const float i0 = 1.0f / z0, i1 = 1.0f / z1;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            P[nt][0] *= i0; P[nt][1] *= i0; P[nt][2] *= i1; P[nt][3] *= i1;
        }
    }
    // dP' = dO V_c^T ; g = rowsum(P * dP')
    float dP[8][4];
    contract_rows_keys<D>(dP, sG, sV, r0, lane);
    float g0 = 0.0f, g1 = 0.0f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        g0 += P[nt][0] * dP[nt][0] + P[nt][1] * dP[nt][1];
        g1 += P[nt][2] * dP[nt][2] + P[nt][3] * dP[nt][3];
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
        g0 += __shfl_xor_sync(0xffffffffu, g0, o);
        g1 += __shfl_xor_sync(0xffffffffu, g1, o);
    }
    const int row0 = s_row[p0], row1 = s_row[p1];
    const float w0 = s_w[p0], w1 = s_w[p1];
    const float ds0 = row0 >= 0 ? w0 * (g0 - delta[row0]) : 0.0f;
    const float ds1 = row1 >= 0 ? w1 * (g1 - delta[row1]) : 0.0f;
    if ((lane & 3) == 0) {
        s_ds[p0] = ds0;
        s_ds[p1] = ds1;
        if (Qs) {
            if (row0 >= 0) ds_pair[(size_t)row0 * Kslots + s_slot[p0]] = ds0;
            if (row1 >= 0) ds_pair[(size_t)row1 * Kslots + s_slot[p1]] = ds1;
        }
    }
    const float lsel = Qs ? 0.0f : 1.0f;  // the ds L_c term belongs to dQ only when Q retrieves
    // dS = w P (dP' - g) and w P, both to shared memory as bf16 [pair][key]
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int col = nt * 8 + (lane & 3) * 2;
        *reinterpret_cast<uint32_t *>(sP + p0 * SP + col) = pack_bf16x2(w0 * P[nt][0], w0 * P[nt][1]);
        *reinterpret_cast<uint32_t *>(sP + p1 * SP + col) = pack_bf16x2(w1 * P[nt][2], w1 * P[nt][3]);
        dP[nt][0] = w0 * P[nt][0] * (dP[nt][0] - g0);
        dP[nt][1] = w0 * P[nt][1] * (dP[nt][1] - g0);
        dP[nt][2] = w1 * P[nt][2] * (dP[nt][2] - g1);
        dP[nt][3] = w1 * P[nt][3] * (dP[nt][3] - g1);
        *reinterpret_cast<uint32_t *>(sdS + p0 * SP + col) = pack_bf16x2(dP[nt][0], dP[nt][1]);
        *reinterpret_cast<uint32_t *>(sdS + p1 * SP + col) = pack_bf16x2(dP[nt][2], dP[nt][3]);
    }
    // dQ_t += scale (dS K_c + ds L_c)   (dS from registers as the A operand)
    {
        float acc[D / 8][4];
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[nt][r] = 0.0f;
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
            uint32_t a[4];
            a[0] = pack_bf16x2(dP[2 * kk][0], dP[2 * kk][1]);
            a[1] = pack_bf16x2(dP[2 * kk][2], dP[2 * kk][3]);
            a[2] = pack_bf16x2(dP[2 * kk + 1][0], dP[2 * kk + 1][1]);
            a[3] = pack_bf16x2(dP[2 * kk + 1][2], dP[2 * kk + 1][3]);
#pragma unroll
            for (int np = 0; np < D / 16; ++np) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(b0, b1, b2, b3,
                                  sK + (kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * SD + np * 16 + (lane >> 4) * 8);
                mma_bf16_16816(acc[2 * np], a, b0, b1);
                mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
            }
        }
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            const int col = nt * 8 + (lane & 3) * 2;
            if (row0 >= 0)
                red_add_v2(dQ + (size_t)row0 * D + col, scale * (acc[nt][0] + lsel * ds0 * s_L[col]),
                           scale * (acc[nt][1] + lsel * ds0 * s_L[col + 1]));
            if (row1 >= 0)
                red_add_v2(dQ + (size_t)row1 * D + col, scale * (acc[nt][2] + lsel * ds1 * s_L[col]),
                           scale * (acc[nt][3] + lsel * ds1 * s_L[col + 1]));
        }
    }
    __syncthreads();  // sP, sdS, s_ds complete
    // dV_c += (wP)^T dO ; dK_c += scale dS^T Q   (warp w owns keys 16w .. 16w+15)
    {
        float acc[D / 8][4];
        const int key0 = r0 + (lane >> 2), key1 = key0 + 8;
        contract_over_pairs<D>(acc, sP, SP, sG, SD, r0, lane);
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            const int col = nt * 8 + (lane & 3) * 2;
            red_add_v2(dV + (krow0 + key0) * D + col, acc[nt][0], acc[nt][1]);
            red_add_v2(dV + (krow0 + key1) * D + col, acc[nt][2], acc[nt][3]);
        }
        contract_over_pairs<D>(acc, sdS, SP, sQ, SD, r0, lane);
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            const int col = nt * 8 + (lane & 3) * 2;
            red_add_v2(dK + (krow0 + key0) * D + col, scale * acc[nt][0], scale * acc[nt][1]);
            red_add_v2(dK + (krow0 + key1) * D + col, scale * acc[nt][2], scale * acc[nt][3]);
        }
    }
    // dL_c += scale * sum_pairs ds q (q: the retrieval query)
    for (int d = tid; d < D; d += kBwdThreads) {
        float acc = 0.0f;
        for (int p = 0; p < pt.count; ++p) {
            const uint16_t qv = Qs ? Qs[(size_t)s_row[p] * D + d] : sQ[p * SD + d];
            acc = fmaf(s_ds[p], __uint_as_float((uint32_t)qv << 16), acc);
        }
        atomicAdd(dL + ((size_t)bh * N + c) * D + d, scale * acc);
    }
}

// The query gradients once the chunk kernel ran with a retrieval query of its own (a separate Qs, or
// the raw Q under query-key normalisation), when dQ holds only the attention part. One warp per token
// row, D / 32 columns per lane; the selected landmark rows are few and stay in L2.
//   ret[t] = scale * sum_j ds[t, j] L[c_j]           (the retrieval query's gradient)
//   QKN: dQ[t] <- dQ[t] taken back through q / max(|q|, eps) at the raw query Qraw[t]
//   dQs != NULL: dQs[t] = ret[t];  else dQ[t] += ret[t] (one query did both)
template <int D, bool QKN>
__global__ void __launch_bounds__(256) dq_finish_kernel(const int32_t *__restrict__ sel_idx,
                                                        const float *__restrict__ ds_pair,
                                                        const uint16_t *__restrict__ L, int T, int N, int K, int G,
                                                        float scale, size_t rows, const uint16_t *__restrict__ Qraw,
                                                        float *__restrict__ dQ, float *__restrict__ dQs) {
    constexpr int PER = D / 32;
    const size_t row = (size_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const size_t kvh = row / T / G;  // the landmark head of this token's query head
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.0f;
    // slots in groups of 32: lane j holds slot j0 + j's chunk and ds; the landmark loads of the slots are
    // independent, so several are in flight at once
    for (int j0 = 0; j0 < K; j0 += 32) {
        const int kj = min(32, K - j0);
        const int c_l = lane < kj ? sel_idx[row * K + j0 + lane] : -1;
        const float ds_l = lane < kj ? ds_pair[row * K + j0 + lane] : 0.0f;
#pragma unroll 8
        for (int j = 0; j < kj; ++j) {
            const int c = __shfl_sync(0xffffffffu, c_l, j);
            const float ds = __shfl_sync(0xffffffffu, ds_l, j);
            if (c < 0 || c >= N) continue;  // empty slot (the dispatch skips the same ids); warp-uniform
            const uint16_t *lr = L + (kvh * N + c) * D + lane * PER;
            if constexpr (PER == 4) {
                const uint2 v = *reinterpret_cast<const uint2 *>(lr);
                acc[0] = fmaf(ds, bf16_lo(v.x), acc[0]);
                acc[1] = fmaf(ds, bf16_hi(v.x), acc[1]);
                acc[2] = fmaf(ds, bf16_lo(v.y), acc[2]);
                acc[3] = fmaf(ds, bf16_hi(v.y), acc[3]);
            } else {
                const uint32_t v = *reinterpret_cast<const uint32_t *>(lr);
                acc[0] = fmaf(ds, bf16_lo(v), acc[0]);
                acc[1] = fmaf(ds, bf16_hi(v), acc[1]);
            }
        }
    }
    float *dq = dQ + row * D + lane * PER;
    float g[PER];
    if constexpr (QKN) {
        float x[PER];
        const uint16_t *xr = Qraw + row * D + lane * PER;
        if constexpr (PER == 4) {
            const uint2 xv = *reinterpret_cast<const uint2 *>(xr);
            const float4 gv = *reinterpret_cast<const float4 *>(dq);
            x[0] = bf16_lo(xv.x); x[1] = bf16_hi(xv.x); x[2] = bf16_lo(xv.y); x[3] = bf16_hi(xv.y);
            g[0] = gv.x; g[1] = gv.y; g[2] = gv.z; g[3] = gv.w;
        } else {
            const uint32_t xv = *reinterpret_cast<const uint32_t *>(xr);
            const float2 gv = *reinterpret_cast<const float2 *>(dq);
            x[0] = bf16_lo(xv); x[1] = bf16_hi(xv);
            g[0] = gv.x; g[1] = gv.y;
        }
        float n2 = 0.0f, xg = 0.0f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            n2 = fmaf(x[i], x[i], n2);
            xg = fmaf(x[i], g[i], xg);
        }
        n2 = warp_sum(n2);
        xg = warp_sum(xg);
        if (n2 > kQkNormEps * kQkNormEps) {  // (g - y (y . g)) / |x|, y = x / |x|
            const float rn = rsqrtf(n2), c = xg * rn * rn;
#pragma unroll
            for (int i = 0; i < PER; ++i) g[i] = (g[i] - x[i] * c) * rn;
        } else {
#pragma unroll
            for (int i = 0; i < PER; ++i) g[i] *= 1.0f / kQkNormEps;
        }
        if (!dQs) {
#pragma unroll
            for (int i = 0; i < PER; ++i) g[i] = fmaf(scale, acc[i], g[i]);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) dq[i] = g[i];
    }
    if (dQs) {
        float *dst = dQs + row * D + lane * PER;
#pragma unroll
        for (int i = 0; i < PER; ++i) dst[i] = scale * acc[i];
    } else if constexpr (!QKN) {
#pragma unroll
        for (int i = 0; i < PER; ++i) dq[i] += scale * acc[i];
    }
}

cudaError_t launch_backward(const BackwardArgs &a0, cudaStream_t s) {
    BackwardArgs a = a0;
    if (a.Hkv <= 0) a.Hkv = a.H;
    if (a.H % a.Hkv != 0) return cudaErrorInvalidValue;
    const int G = a.H / a.Hkv;  // query heads per key head
    const size_t kv_rows = (size_t)a.B * a.Hkv * a.T, chunks = (size_t)a.B * a.H * a.N;
    if (a0.qk_norm) {  // the kernels run on the normalised Q and K; the raw Q retrieves unless Qs does
        cudaError_t e = launch_l2norm_rows(a0.Q, a0.Qn, (size_t)a.B * a.H * a.T, a0.K, a0.Kn, kv_rows, a.D, s);
        if (e != cudaSuccess) return e;
        a.Q = a0.Qn;
        a.K = a0.Kn;
        if (!a.Qs) a.Qs = a0.Q;
    }
    const int BH = a.B * a.H;
    const size_t rows = (size_t)BH * a.T;
    cudaError_t e;
    {
        HSA_PROF("memset", s);
        e = cudaMemsetAsync(a.dQ, 0, rows * a.D * sizeof(float), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.dK, 0, kv_rows * a.D * sizeof(float), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.dV, 0, kv_rows * a.D * sizeof(float), s);
        if (e == cudaSuccess && a.N > 0)
            e = cudaMemsetAsync(a.dL, 0, (size_t)a.B * a.Hkv * a.N * a.D * sizeof(float), s);
        if (e == cudaSuccess) e = zero_dispatch_state(a.err, a.chunk_count, a.chunk_cursor, a.N > 0 ? chunks : 0, s);
        // with chunks, dq_finish_kernel writes every row of dQs
        if (e == cudaSuccess && a.dQs && a.N == 0) e = cudaMemsetAsync(a.dQs, 0, rows * a.D * sizeof(float), s);
    }
    if (e != cudaSuccess || a.N == 0) return e;
    const size_t rows_per_block = 8 * (32 / (a.D / 8)) * kDeltaGroups;  // 8 warps
    const unsigned dblocks = (unsigned)((rows + rows_per_block - 1) / rows_per_block);
    {
        HSA_PROF("bwd_delta", s);
        if (a.D == 128) delta_kernel<128><<<dblocks, 256, 0, s>>>(a.out, a.dout, rows, a.delta);
        else delta_kernel<64><<<dblocks, 256, 0, s>>>(a.out, a.dout, rows, a.delta);
    }
    // head dim 128: tcgen05 kernel over work units of up to kBwdUnitPairs pairs of one chunk;
    // head dim 64: the mma.sync kernel over tiles of kPairTile pairs
    const bool tc = a.D == 128;
    e = launch_dispatch(a.sel_idx, a.sel_w, a.B, a.H, a.T, a.N, a.topk, a.chunk_count, a.chunk_off, a.tile_off,
                        a.chunk_cursor, a.pair_row, a.pair_w, a.pair_slot, a.tiles, a.num_tiles, a.max_tiles,
                        tc ? kBwdUnitPairs : kPairTile, false, s);
    if (e != cudaSuccess) return e;
    if (tc) {
        e = launch_backward_tc(a, s);
    } else {
        const size_t smem = BwdSmem<64>::total;
        e = cudaFuncSetAttribute(chunk_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        HSA_PROF("chunk_bwd", s);
        chunk_bwd_kernel<64><<<a.max_tiles, kBwdThreads, smem, s>>>(a.Q, a.K, a.V, a.L, a.dout, a.delta, a.T, a.N,
                                                                     a.scale, a.tiles, a.num_tiles, a.pair_row,
                                                                     a.pair_w, a.dQ, a.dK, a.dV, a.dL, a.Qs,
                                                                     a.pair_slot, a.ds_pair, a.topk, G);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess || !a.Qs) return e;
    {  // the retrieval query's gradient (and the attention part back through the normalisation)
        HSA_PROF("bwd_dq_finish", s);
        const unsigned blocks = (unsigned)((rows + 7) / 8);
        auto kern = a.D == 128 ? (a0.qk_norm ? dq_finish_kernel<128, true> : dq_finish_kernel<128, false>)
                               : (a0.qk_norm ? dq_finish_kernel<64, true> : dq_finish_kernel<64, false>);
        kern<<<blocks, 256, 0, s>>>(a.sel_idx, a.ds_pair, a.L, a.T, a.N, a.topk, G, a.scale, rows, a0.Q, a.dQ, a.dQs);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess || !a0.qk_norm) return e;
    return launch_l2norm_grad_rows(a0.K, a.dK, kv_rows, a.D, s);
}

}  // namespace hsa
