// varlen.cu -- variable-length batches in the packed, token-major layout.
//
// The packed layout is the one model code holds between layers: the tokens of all sequences one after
// another, [total, heads, row], sequence b at token rows cu[b] .. cu[b+1] - 1 (cu_seqlens), and its
// floor(len_b / 64) complete chunks' landmarks likewise at landmark rows cuN[b] .. (cuN the prefix
// sums of the chunk counts). The HSA kernels take a head-major batch [B, heads, T, row]; these kernels
// move rows between the two. Both sides are row-contiguous, so every copy is a coalesced streaming
// pass (HBM-bound). The batch rows past a sequence's end are filled only where a kernel reads them (the
// selection that a backward gets: chunk -1, weight 0); the forward never reads them.
#include "common.cuh"
#include "launch.h"
#include "profile.h"

namespace hsa {

constexpr int kVarlenThreads = 256;

// cuN[b] = sum over b' < b of floor((cu[b'+1] - cu[b']) / 64), for b = 0 .. B. One block.
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(const int32_t *__restrict__ cu, int B,
                                                             int32_t *__restrict__ cuN) {
    __shared__ int s_part[1024];
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int per = (B + nthr - 1) / nthr;
    const int lo = min(B, tid * per), hi = min(B, lo + per);
    int sum = 0;
    for (int b = lo; b < hi; ++b) sum += (cu[b + 1] - cu[b]) / kChunk;
    s_part[tid] = sum;
    __syncthreads();
    for (int o = 1; o < nthr; o <<= 1) {  // inclusive scan of the per-thread sums
        const int x = tid >= o ? s_part[tid - o] : 0;
        __syncthreads();
        s_part[tid] += x;
        __syncthreads();
    }
    int off = s_part[tid] - sum;
    for (int b = lo; b < hi; ++b) {
        cuN[b] = off;
        off += (cu[b + 1] - cu[b]) / kChunk;
    }
    if (tid == nthr - 1) cuN[B] = s_part[tid];
}

// Rows of V copy units (U = 16 or 4 bytes) between the packed side (row (cu[b] + t) * Hs + h) and
// the batch side (row (b * Hs + h) * Tp + t). pack: batch <- packed, and with fill_pad the rows
// t >= len_b get `fill` (otherwise they are left as they are: no kernel reads them); unpack: packed <-
// batch for t < len_b. 2^lpr_log2 lanes share a row.
template <typename Unit>
__global__ void __launch_bounds__(kVarlenThreads) varlen_rows_kernel(const Unit *__restrict__ src,
                                                                     Unit *__restrict__ dst,
                                                                     const int32_t *__restrict__ cu, int B, int Hs,
                                                                     int Tp, int V, int lpr_log2, bool pack,
                                                                     bool fill_pad, uint32_t fill) {
    const int lpr = 1 << lpr_log2, sub = threadIdx.x & (lpr - 1);
    const size_t rows = (size_t)B * Hs * Tp;
    const size_t nsub = ((size_t)gridDim.x * kVarlenThreads) >> lpr_log2;
    Unit f;
    if constexpr (sizeof(Unit) == 16) f = make_uint4(fill, fill, fill, fill);
    else f = fill;
    for (size_t row = ((size_t)blockIdx.x * kVarlenThreads + threadIdx.x) >> lpr_log2; row < rows; row += nsub) {
        const int t = (int)(row % Tp);
        const size_t bh = row / Tp;
        const int h = (int)(bh % Hs), b = (int)(bh / Hs);
        const int base = cu[b], len = cu[b + 1] - base;
        if (t >= len && !(pack && fill_pad)) continue;
        const size_t packed = ((size_t)(base + t) * Hs + h) * V, batch = row * V;
        for (int v = sub; v < V; v += lpr) {
            if (pack) dst[batch + v] = t < len ? src[packed + v] : f;
            else if (t < len) dst[packed + v] = src[batch + v];
        }
    }
}

cudaError_t launch_chunk_offsets(const int32_t *cu, int B, int32_t *cuN, cudaStream_t s) {
    HSA_PROF("varlen_offsets", s);
    chunk_offsets_kernel<<<1, 1024, 0, s>>>(cu, B, cuN);
    return cudaGetLastError();
}

cudaError_t launch_varlen_rows(const void *src, void *dst, const int32_t *cu, int B, int Hs, int Tp, int row_bytes,
                               bool pack, bool fill_pad, uint32_t fill, cudaStream_t s) {
    if ((size_t)B * Hs * Tp == 0 || row_bytes <= 0) return cudaSuccess;
    if (row_bytes % 4 != 0) return cudaErrorInvalidValue;
    const bool wide = row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(src) % 16 == 0 &&
                      reinterpret_cast<uintptr_t>(dst) % 16 == 0;
    const int V = wide ? row_bytes / 16 : row_bytes / 4;
    int lpr_log2 = 0;
    while ((1 << lpr_log2) < V && lpr_log2 < 5) ++lpr_log2;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t rows = (size_t)B * Hs * Tp;
    const size_t want = (rows << lpr_log2) / kVarlenThreads + 1;
    const unsigned grid = (unsigned)(want < (size_t)sms * 8 ? want : (size_t)sms * 8);
    HSA_PROF(pack ? "varlen_pack" : "varlen_unpack", s);
    if (wide)
        varlen_rows_kernel<uint4><<<grid, kVarlenThreads, 0, s>>>(static_cast<const uint4 *>(src),
                                                                  static_cast<uint4 *>(dst), cu, B, Hs, Tp, V,
                                                                  lpr_log2, pack, fill_pad, fill);
    else
        varlen_rows_kernel<uint32_t><<<grid, kVarlenThreads, 0, s>>>(static_cast<const uint32_t *>(src),
                                                                     static_cast<uint32_t *>(dst), cu, B, Hs, Tp, V,
                                                                     lpr_log2, pack, fill_pad, fill);
    return cudaGetLastError();
}

}  // namespace hsa
