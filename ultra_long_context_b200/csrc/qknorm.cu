// qknorm.cu -- query-key normalisation for the in-chunk attention.
//
// Explainer page of "Every Token Counts", "How It Works (Technically)", Step 3: the logits inside a
// selected chunk are norm(q_attn) . norm(K_c)^T / sqrt(d_h), with norm the L2 normalisation (the
// per-token procedure of "The algorithm, simplified" calls l2norm on the attention query and on the
// keys). Reading: norm(x) = x / max(|x|_2, eps) with eps = 1e-6, per row of D elements.
//
//   l2norm_rows_kernel       y = norm(x), bf16 rows in and out (the prefill forward and backward run
//                            their tensor-core kernels on these copies). HBM-bound streaming: each
//                            row is read once and written once, 16 bytes per lane, several rows in
//                            flight per thread.
//   l2norm_grad_rows_kernel  dx = J(x)^T dy in place, J the Jacobian of norm at x:
//                            (dy - y (y . dy)) / |x| when |x| > eps, dy / eps otherwise.
#include "common.cuh"
#include "launch.h"
#include "profile.h"

namespace hsa {

constexpr int kNormThreads = 256;
constexpr int kNormUnroll = 4;  // rows in flight per thread

template <int D>
__global__ void __launch_bounds__(kNormThreads) l2norm_rows_kernel(const uint16_t *__restrict__ X0,
                                                                   uint16_t *__restrict__ Y0, size_t R0,
                                                                   const uint16_t *__restrict__ X1,
                                                                   uint16_t *__restrict__ Y1, size_t R1) {
    constexpr int LPR = D / 8;        // lanes per row, 8 elements (16 bytes) each
    constexpr int RPW = 32 / LPR;     // rows per warp step
    const int lane = threadIdx.x & 31, sub = lane % LPR;
    const size_t total = R0 + R1;
    const size_t steps = (total + RPW - 1) / RPW;
    const size_t nwarps = (size_t)gridDim.x * (kNormThreads / 32);
    const size_t w0 = (size_t)blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5);
    for (size_t g0 = w0; g0 < steps; g0 += nwarps * kNormUnroll) {
        uint4 v[kNormUnroll];
        size_t row[kNormUnroll];
#pragma unroll
        for (int u = 0; u < kNormUnroll; ++u) {  // issue every load first
            const size_t g = g0 + (size_t)u * nwarps;
            row[u] = g * RPW + lane / LPR;
            v[u] = (g < steps && row[u] < total)
                       ? ld_stream16((row[u] < R0 ? X0 + row[u] * D : X1 + (row[u] - R0) * D) + sub * 8)
                       : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kNormUnroll; ++u) {
            const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
            float x[8], n2 = 0.0f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                x[2 * k] = bf16_lo(w[k]);
                x[2 * k + 1] = bf16_hi(w[k]);
                n2 = fmaf(x[2 * k], x[2 * k], n2);
                n2 = fmaf(x[2 * k + 1], x[2 * k + 1], n2);
            }
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) n2 += __shfl_xor_sync(0xffffffffu, n2, o);
            // 1 / max(|x|, eps) = rsqrt(max(|x|^2, eps^2))
            const float rn = rsqrtf(fmaxf(n2, kQkNormEps * kQkNormEps));
            const size_t g = g0 + (size_t)u * nwarps;
            if (g < steps && row[u] < total) {
                uint16_t *dst = row[u] < R0 ? Y0 + row[u] * D : Y1 + (row[u] - R0) * D;
                *reinterpret_cast<uint4 *>(dst + sub * 8) =
                    make_uint4(pack_bf16x2(x[0] * rn, x[1] * rn), pack_bf16x2(x[2] * rn, x[3] * rn),
                               pack_bf16x2(x[4] * rn, x[5] * rn), pack_bf16x2(x[6] * rn, x[7] * rn));
            }
        }
    }
}

// One warp per row; lane holds D/32 consecutive elements.
template <int D>
__global__ void __launch_bounds__(kNormThreads) l2norm_grad_rows_kernel(const uint16_t *__restrict__ X,
                                                                        float *__restrict__ dX, size_t rows) {
    constexpr int PER = D / 32;
    const int lane = threadIdx.x & 31;
    const size_t nwarps = (size_t)gridDim.x * (kNormThreads / 32);
    for (size_t r = (size_t)blockIdx.x * (kNormThreads / 32) + (threadIdx.x >> 5); r < rows; r += nwarps) {
        float x[PER], g[PER];
        const uint16_t *xr = X + r * D + lane * PER;
        float *gr = dX + r * D + lane * PER;
        if constexpr (PER == 4) {
            const uint2 xv = *reinterpret_cast<const uint2 *>(xr);
            const float4 gv = *reinterpret_cast<const float4 *>(gr);
            x[0] = bf16_lo(xv.x); x[1] = bf16_hi(xv.x); x[2] = bf16_lo(xv.y); x[3] = bf16_hi(xv.y);
            g[0] = gv.x; g[1] = gv.y; g[2] = gv.z; g[3] = gv.w;
        } else {
            const uint32_t xv = *reinterpret_cast<const uint32_t *>(xr);
            const float2 gv = *reinterpret_cast<const float2 *>(gr);
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
        if (n2 > kQkNormEps * kQkNormEps) {
            const float rn = rsqrtf(n2);          // 1 / |x|
            const float c = xg * rn * rn;         // (y . dy) / |x| with y = x / |x|
#pragma unroll
            for (int i = 0; i < PER; ++i) g[i] = (g[i] - x[i] * c) * rn;
        } else {
#pragma unroll
            for (int i = 0; i < PER; ++i) g[i] *= 1.0f / kQkNormEps;
        }
        if constexpr (PER == 4) {
            *reinterpret_cast<float4 *>(gr) = make_float4(g[0], g[1], g[2], g[3]);
        } else {
            *reinterpret_cast<float2 *>(gr) = make_float2(g[0], g[1]);
        }
    }
}

static unsigned norm_grid(size_t work_warps) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t per_block = kNormThreads / 32;
    size_t blocks = (work_warps + per_block - 1) / per_block;
    const size_t cap = (size_t)sms * 8;  // 8 resident blocks of 256 threads per SM
    return (unsigned)(blocks < 1 ? 1 : (blocks < cap ? blocks : cap));
}

cudaError_t launch_l2norm_rows(const uint16_t *X0, uint16_t *Y0, size_t R0, const uint16_t *X1, uint16_t *Y1,
                               size_t R1, int D, cudaStream_t s) {
    if (R0 + R1 == 0) return cudaSuccess;
    const int rpw = 32 / (D / 8);
    const unsigned grid = norm_grid((R0 + R1 + rpw - 1) / rpw / kNormUnroll);
    HSA_PROF("qk_norm", s);
    if (D == 128) l2norm_rows_kernel<128><<<grid, kNormThreads, 0, s>>>(X0, Y0, R0, X1, Y1, R1);
    else if (D == 64) l2norm_rows_kernel<64><<<grid, kNormThreads, 0, s>>>(X0, Y0, R0, X1, Y1, R1);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_l2norm_grad_rows(const uint16_t *X, float *dX, size_t rows, int D, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const unsigned grid = norm_grid(rows);
    HSA_PROF("qk_norm_grad", s);
    if (D == 128) l2norm_grad_rows_kernel<128><<<grid, kNormThreads, 0, s>>>(X, dX, rows);
    else if (D == 64) l2norm_grad_rows_kernel<64><<<grid, kNormThreads, 0, s>>>(X, dX, rows);
    else return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace hsa
