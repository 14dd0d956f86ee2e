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
// The pairs are processed chunk-major with the same dispatch as the forward (work units of up to
// kBwdUnitPairs pairs of one chunk), by the tcgen05 kernel of bwd_tc.cu. This file holds the delta
// kernel, the query-gradient finish for a separate retrieval query or query-key normalisation, and
// the launch sequence.
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
    // the tcgen05 kernel over work units of up to kBwdUnitPairs pairs of one chunk
    e = launch_dispatch(a.sel_idx, a.sel_w, a.B, a.H, a.T, a.N, a.topk, a.chunk_count, a.chunk_off, a.tile_off,
                        a.chunk_cursor, a.pair_row, a.pair_w, a.pair_slot, a.tiles, a.num_tiles, a.max_tiles,
                        kBwdUnitPairs, false, s);
    if (e != cudaSuccess) return e;
    e = launch_backward_tc(a, s);
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
