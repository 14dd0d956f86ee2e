// score_tc.cu -- Step 2 (retrieval scores + top-K) and the Step 4 fusion weights of the HSA forward,
// on the 5th-generation tensor cores.
//
// Explainer page of "Every Token Counts", "How It Works (Technically)", Step 2: each token t scores
// every chunk that has ended at or before it, s[t,c] = scale * Q[t].L[c], and keeps the top-K; the
// per-token procedure ("The algorithm, simplified") sorts the scores in descending order, stably,
// so equal scores keep the lower chunk first. Step 4: w = softmax of the kept scores.
//
// One CTA per (128-token tile, batch*head), 4 warps, thread = token row = TMEM lane:
//   * Q tile (128 x D) and landmark blocks (64 x D) arrive by TMA in the 128-byte-swizzled layout;
//     one thread issues S_blk = Q L_blk^T (M = 128, N = 64, fp32) into one of two TMEM buffers while
//     the warps read the other (tcgen05.ld), so the tensor core runs ahead of the selection.
//   * Each 32-score slab read from TMEM is first compacted into a per-thread column of shared memory
//     (only the scores that can matter), and only those are processed, so a warp's cost follows
//     the candidates of its rows rather than every score.
//   * Pass 1 keeps, per row, the K largest score VALUES in a sorted register list. A score that
//     beats the current K-th value is inserted with new[i] = max(old[i], min(old[i-1], x)), which
//     touches every slot independently (no dependent chain). The K-th value tau results.
//   * Pass 2 recomputes the same blocks (bit-identical: same operands, same instruction sequence)
//     and emits every chunk with s > tau, plus the lowest-index chunks with s == tau until K are
//     kept -- exactly the stable-sort rule. A chunk's output slot is the number of kept values above
//     it, ties taking the next free slot in chunk order (a bitmask of used slots).
//   * Fusion weights w = softmax over the kept values (fp32, max-subtracted).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "launch.h"
#include "profile.h"
#include "tc.cuh"

namespace hsa {

constexpr int kStRows = 128;      // tokens per CTA (MMA M)
constexpr int kStCols = 64;       // landmarks per block (MMA N)
constexpr int kStThreads = 128;

template <int D>
struct StSmem {
    static constexpr int KH = D / 64;
    static constexpr uint32_t QB = KH * 16384;      // [128 rows][D] bf16, swizzled halves
    static constexpr uint32_t LB = KH * 8192;       // [64 rows][D] per landmark buffer
    static constexpr uint32_t Qo = 0, L0 = QB, L1 = QB + LB;
    static constexpr uint32_t CV = L1 + LB;         // candidate values [32][128 threads] fp32
    static constexpr uint32_t CC = CV + 32 * 128 * 4;  // candidate chunk ids [32][128] (pass 2)
    static constexpr uint32_t BAR = CC + 32 * 128 * 4;  // bar_q, bar_l[2], bar_s[2]
    static constexpr uint32_t TMEM = BAR + 5 * 8;
    static constexpr uint32_t BYTES = TMEM + 8;
    static constexpr size_t DYN = BYTES + 1024;
};

template <int D, int K>
__global__ void __launch_bounds__(kStThreads) score_topk_tc_kernel(int T, int N, float scale, int kout,
                                                                   int32_t *__restrict__ sel_idx,
                                                                   float *__restrict__ sel_w, int32_t *__restrict__ err,
                                                                   const __grid_constant__ CUtensorMap tmQ,
                                                                   const __grid_constant__ CUtensorMap tmL) {
    using SM = StSmem<D>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    unsigned char *s = smem_raw + (sb - raw);
    const uint32_t bar_q = sb + SM::BAR;
    auto bar_l = [&](int i) { return sb + SM::BAR + 8u * (1 + i); };
    auto bar_s = [&](int i) { return sb + SM::BAR + 8u * (3 + i); };

    const int tid = threadIdx.x, warp = tid >> 5;
    const int ntile = (T + kStRows - 1) / kStRows;
    const int tile = ntile - 1 - blockIdx.x;  // longest rows first
    const int bh = blockIdx.y;
    const int t0 = tile * kStRows;
    const int t_last = min(T - 1, t0 + kStRows - 1);
    const int n_max = min(N, (t_last + 1) / kChunk);
    const int nblk = (n_max + kStCols - 1) / kStCols;
    const int my_t = t0 + tid;
    const int my_n = my_t < T ? min(N, (my_t + 1) / kChunk) : 0;
    const size_t row = (size_t)bh * T + my_t;

    if (nblk == 0) {  // no token of this tile has a complete chunk
        if (my_t < T)
            for (int i = 0; i < kout; ++i) {
                sel_idx[row * kout + i] = -1;
                sel_w[row * kout + i] = 0.0f;
            }
        return;
    }

    if (warp == 0) tc::tmem_alloc(sb + SM::TMEM, 2 * kStCols);
    if (tid == 0) {
        for (int i = 0; i < 5; ++i) tc::mbar_init(sb + SM::BAR + 8u * i, 1);
        tc::fence_mbar_init();
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *reinterpret_cast<uint32_t *>(s + SM::TMEM);
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int G = 2 * nblk;  // blocks visited: pass 1, then pass 2
    bool ok = true;

    auto load_l = [&](int g) {  // landmark block (g % nblk) into buffer g % 2
        const int b = g % nblk;
        const uint32_t dst = sb + (g & 1 ? SM::L1 : SM::L0);
        tc::mbar_arrive_expect_tx(bar_l(g & 1), SM::LB);
#pragma unroll
        for (int h = 0; h < SM::KH; ++h) tc::tma_load_2d(dst + h * 8192, &tmL, h * 64, bh * N + b * kStCols, bar_l(g & 1));
    };
    auto issue_mma = [&](int g) -> bool {
        if (!tc::mbar_wait(bar_l(g & 1), (uint32_t)(g >> 1) & 1u)) return false;
        tc::fence_after();
        constexpr uint32_t idesc = tc::idesc_bf16(kStRows, kStCols, 0, 0);
        const uint32_t lb = sb + (g & 1 ? SM::L1 : SM::L0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t kin = (uint32_t)((ks & 3) * 32);  // K step inside a 128-byte row
            tc::mma_bf16_ss(tmem + (g & 1) * kStCols, tc::desc_kmajor(sb + SM::Qo + (ks >> 2) * 16384 + kin),
                            tc::desc_kmajor(lb + (ks >> 2) * 8192 + kin), idesc, ks > 0 ? 1u : 0u);
        }
        tc::commit(bar_s(g & 1));
        return true;
    };

    if (tid == 0) {
        tc::mbar_arrive_expect_tx(bar_q, SM::QB);
#pragma unroll
        for (int h = 0; h < SM::KH; ++h) tc::tma_load_2d(sb + SM::Qo + h * 16384, &tmQ, h * 64, bh * T + t0, bar_q);
        load_l(0);
        if (G > 1) load_l(1);
        ok = tc::mbar_wait(bar_q, 0) && issue_mma(0);
    }

    float ls[K];  // pass 1: the K largest score values of this row, descending
#pragma unroll
    for (int i = 0; i < K; ++i) ls[i] = -INFINITY;
    float tau = -INFINITY, top = 0.0f, z = 0.0f;
    int need_eq = 0;
    uint64_t used = 0;  // pass 2: output slots taken
    const int k_keep = min(kout, my_n);

    for (int g = 0; g < G; ++g) {
        if (tid == 0 && ok && g + 1 < G) ok = issue_mma(g + 1);
        const bool fail = __syncthreads_or(!(ok && tc::mbar_wait(bar_s(g & 1), (uint32_t)(g >> 1) & 1u)));
        if (fail) {
            ok = false;
            break;
        }
        tc::fence_after();
        if (tid == 0 && g + 2 < G) load_l(g + 2);  // MMA(g) is done with that landmark buffer
        if (g == nblk) {
            // end of pass 1: tau = the k_keep-th largest value; ties at tau are taken lowest chunk first
            tau = k_keep > 0 ? -INFINITY : INFINITY;
            int gt = 0;
#pragma unroll
            for (int i = 0; i < K; ++i)
                if (i < k_keep) tau = ls[i];
#pragma unroll
            for (int i = 0; i < K; ++i) gt += (i < k_keep && ls[i] > tau) ? 1 : 0;
            need_eq = k_keep - gt;
            top = ls[0];
#pragma unroll
            for (int i = 0; i < K; ++i) z += i < k_keep ? expf(ls[i] - top) : 0.0f;
        }
        const int b = g % nblk;
        const int ncol = min(kStCols, my_n - b * kStCols);
        const uint32_t tS = tmem + lane_off + (g & 1) * kStCols;
        float *cv = reinterpret_cast<float *>(s + SM::CV) + tid;  // this thread's column of slots
        int *cc = reinterpret_cast<int *>(s + SM::CC) + tid;
#pragma unroll 1
        for (int q = 0; q < kStCols / 32; ++q) {
            float v[32];
            tc::tmem_ld32(tS + q * 32, v);
            // compact this slab's candidates (cheap predicated stores), then handle only those, so a
            // warp never pays an insertion for lanes that have nothing to insert
            int n = 0;
            if (g < nblk) {
                const float thr = ls[K - 1];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float x = v[i] * scale;
                    if (q * 32 + i < ncol && x > thr) cv[128 * n++] = x;
                }
                for (int k = 0; k < n; ++k) {
                    const float x = cv[128 * k];
                    if (x > ls[K - 1]) {
#pragma unroll
                        for (int j = K - 1; j > 0; --j) ls[j] = fmaxf(ls[j], fminf(ls[j - 1], x));
                        ls[0] = fmaxf(ls[0], x);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float x = v[i] * scale;
                    if (q * 32 + i < ncol && x >= tau) {
                        cv[128 * n] = x;
                        cc[128 * n] = b * kStCols + q * 32 + i;
                        ++n;
                    }
                }
                for (int k = 0; k < n; ++k) {
                    const float x = cv[128 * k];
                    bool take = x > tau;
                    if (!take && need_eq > 0) {  // x == tau: lowest chunks first (they arrive in order)
                        take = true;
                        --need_eq;
                    }
                    if (take) {
                        int lo = 0;
#pragma unroll
                        for (int j = 0; j < K; ++j) lo += (j < k_keep && ls[j] > x) ? 1 : 0;
                        const uint64_t freeb = ~used & (~0ull << lo);
                        const int slot = __ffsll((long long)freeb) - 1;
                        used |= 1ull << slot;
                        sel_idx[row * kout + slot] = cc[128 * k];
                        sel_w[row * kout + slot] = expf(x - top) / z;
                    }
                }
            }
        }
        tc::fence_before();
        __syncthreads();  // TMEM buffer g % 2 is rewritten by MMA(g + 2)
    }
    if (ok && my_t < T)
        for (int i = k_keep; i < kout; ++i) {
            sel_idx[row * kout + i] = -1;
            sel_w[row * kout + i] = 0.0f;
        }
    if (!ok && tid == 0) atomicOr(err, 1);
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, 2 * kStCols);
    }
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
static PFN_cuTensorMapEncodeTiled_v12000 st_encode_fn() {
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

static bool st_tmap(CUtensorMap *m, const void *base, uint64_t rows, int D, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = st_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int K>
static cudaError_t launch_st(const ForwardArgs &a, const CUtensorMap &tq, const CUtensorMap &tl, cudaStream_t s) {
    const size_t smem = StSmem<D>::DYN;
    cudaError_t e = cudaFuncSetAttribute(score_topk_tc_kernel<D, K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.T + kStRows - 1) / kStRows, a.B * a.H);
    HSA_PROF("score_topk", s);
    score_topk_tc_kernel<D, K><<<grid, kStThreads, smem, s>>>(a.T, a.N, a.scale, a.topk, a.sel_idx, a.sel_w, a.err,
                                                              tq, tl);
    return cudaGetLastError();
}

template <int D>
static cudaError_t launch_st_d(const ForwardArgs &a, cudaStream_t s) {
    CUtensorMap tq, tl;
    if (!st_tmap(&tq, a.Q, (uint64_t)a.B * a.H * a.T, D, kStRows)) return cudaErrorInvalidValue;
    // with no complete chunk the landmark tensor may be empty: point the map at Q (never read)
    if (!st_tmap(&tl, a.N > 0 ? (const void *)a.L : (const void *)a.Q,
                 a.N > 0 ? (uint64_t)a.B * a.H * a.N : (uint64_t)a.B * a.H * a.T, D, kStCols))
        return cudaErrorInvalidValue;
    if (a.topk <= 8) return launch_st<D, 8>(a, tq, tl, s);
    if (a.topk <= 16) return launch_st<D, 16>(a, tq, tl, s);
    return launch_st<D, 32>(a, tq, tl, s);
}

cudaError_t launch_score_tc(const ForwardArgs &a, cudaStream_t s) {
    return a.D == 128 ? launch_st_d<128>(a, s) : launch_st_d<64>(a, s);
}

}  // namespace hsa
