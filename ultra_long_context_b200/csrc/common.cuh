// common.cuh -- device helpers shared by the HSA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hsa {

constexpr int kChunk = 64;  // chunk length S (explainer, "How It Works", Step 1)

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// fp32 -> bf16 pair, round to nearest even (cvt.rn.bf16x2.f32).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&r);
}

// Order-preserving map fp32 -> u32 (larger float -> larger integer). -0 is folded onto +0 so
// that equal scores compare equal.
__device__ __forceinline__ uint32_t float_to_ordered(float s) {
    uint32_t u = __float_as_uint(s == 0.0f ? 0.0f : s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ordered_to_float(uint32_t o) {
    return __uint_as_float((o & 0x80000000u) ? (o ^ 0x80000000u) : ~o);
}

// Unique 64-bit selection key: higher score first, then LOWER chunk index first. Comparing keys
// as unsigned integers therefore realises "score descending, ties to the lower chunk index".
// Key 0 never encodes a finite score and marks an empty slot.
__device__ __forceinline__ uint64_t make_key(float s, uint32_t idx) {
    return ((uint64_t)float_to_ordered(s) << 32) | (uint64_t)(0xffffffffu - idx);
}
__device__ __forceinline__ float key_score(uint64_t k) { return ordered_to_float((uint32_t)(k >> 32)); }
__device__ __forceinline__ int key_index(uint64_t k) { return (int)(0xffffffffu - (uint32_t)k); }

// Programmatic dependent launch. A kernel that may be launched as a programmatic dependent calls
// pdl_wait() before anything else: it returns once the previous kernel in the stream has completed and
// its memory is visible (a no-op under an ordinary launch). pdl_launch_dependents() lets the next
// kernel's blocks be scheduled once every block of this grid has issued it, so they are resident and
// waiting when this grid ends; the launch latency is hidden, the ordering is that of the stream.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// 2^x by the hardware's approximate base-2 exponential (PTX ex2.approx.ftz.f32; relative error
// about 2^-22, subnormal results flushed to zero) -- ample for probabilities stored as bf16.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- cp.async (Ampere-style async copies into shared memory) ----
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// 16-byte copy; src_bytes = 0 writes zeros (used for rows past the end).
__device__ __forceinline__ void cp_async16(void *dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async16_u32(uint32_t dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// ---- legacy warp MMA (mma.sync m16n8k16, bf16 in, fp32 accumulate) ----
__device__ __forceinline__ void ldmatrix_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3, const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                                  const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// fp32 vector reductions into global memory (sm_90+).
__device__ __forceinline__ void red_add_v2(float *p, float a, float b) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};\n" ::"l"(p), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};\n" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Streaming 16-byte global load that is not kept in L1 (data read once).
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Dot product of 8 bf16 values (one 16-byte vector) with 8 fp32 values.
__device__ __forceinline__ float dot8(const uint4 v, const float (&q)[8]) {
    float a = bf16_lo(v.x) * q[0];
    a = fmaf(bf16_hi(v.x), q[1], a);
    a = fmaf(bf16_lo(v.y), q[2], a);
    a = fmaf(bf16_hi(v.y), q[3], a);
    a = fmaf(bf16_lo(v.z), q[4], a);
    a = fmaf(bf16_hi(v.z), q[5], a);
    a = fmaf(bf16_lo(v.w), q[6], a);
    a = fmaf(bf16_hi(v.w), q[7], a);
    return a;
}

/*
 * Exact block-wide top-K of n 64-bit keys held in shared memory (MSB-first radix select, 8 bits
 * per pass, stopping as soon as the boundary bin is taken whole). Keys are unique except for
 * repeated zeros (empty slots), which compare equal and are interchangeable. Writes the min(n, K)
 * largest keys, in no particular order, to out[] (shared) and returns that count. hist must hold
 * 256 u32 and misc 4 ints, both in shared memory. Must be called by every thread of the block;
 * blockDim.x must be a multiple of 32.
 */
__device__ inline int block_topk_u64(const uint64_t *keys, int n, int K, uint64_t *out, uint32_t *hist, int *misc) {
    const int tid = threadIdx.x, lane = tid & 31, nthr = blockDim.x;
    if (n <= K) {
        for (int i = tid; i < n; i += nthr) out[i] = keys[i];
        __syncthreads();
        return n;
    }
    uint64_t prefix = 0;
    int krem = K;
    int keep_shift = 0;
    for (int pass = 0; pass < 8; ++pass) {
        const int shift = 56 - 8 * pass;
        for (int i = tid; i < 256; i += nthr) hist[i] = 0;
        __syncthreads();
        const int n_round = (n + 31) & ~31;
        for (int i = tid; i < n_round; i += nthr) {
            int digit = 256;
            if (i < n) {
                const uint64_t k = keys[i];
                const bool match = pass == 0 || ((k >> (shift + 8)) == (prefix >> (shift + 8)));
                if (match) digit = (int)((k >> shift) & 0xffu);
            }
            const unsigned peers = __match_any_sync(0xffffffffu, digit);
            if (digit < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
        }
        __syncthreads();
        if (tid < 32) {
            // lane l owns bins 255-8l .. 248-8l (descending); find the bin holding the krem-th key
            uint32_t local = 0;
            for (int j = 0; j < 8; ++j) local += hist[255 - 8 * lane - j];
            uint32_t incl = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t excl = incl - local;
            if (excl < (uint32_t)krem && (uint32_t)krem <= incl) {
                uint32_t above = excl;
                for (int j = 0; j < 8; ++j) {
                    const int bin = 255 - 8 * lane - j;
                    const uint32_t c = hist[bin];
                    if (above + c >= (uint32_t)krem) {
                        misc[0] = bin;
                        misc[1] = (int)above;
                        misc[2] = (int)c;
                        break;
                    }
                    above += c;
                }
            }
        }
        __syncthreads();
        const int bin = misc[0], above = misc[1], cnt = misc[2];
        prefix |= (uint64_t)bin << shift;
        krem -= above;
        keep_shift = shift;
        __syncthreads();  // misc is rewritten by the next pass
        if (cnt == krem) break;
    }
    // Keys whose top (64 - keep_shift) bits exceed the prefix's are all selected first; keys equal
    // to it fill the remaining slots (with unique keys exactly krem of them; duplicated keys, such
    // as repeated empty-slot zeros, are identical, so which copies are taken does not matter).
    if (tid == 0) misc[3] = 0;
    __syncthreads();
    const uint64_t bound = prefix >> keep_shift;
    for (int i = tid; i < n; i += nthr) {
        const uint64_t k = keys[i];
        if ((k >> keep_shift) > bound) out[atomicAdd(&misc[3], 1)] = k;
    }
    __syncthreads();
    for (int i = tid; i < n; i += nthr) {
        const uint64_t k = keys[i];
        if ((k >> keep_shift) == bound) {
            const int pos = atomicAdd(&misc[3], 1);
            if (pos < K) out[pos] = k;
        }
    }
    __syncthreads();
    return K;
}

// Sort up to 64 keys descending in shared memory by rank counting. Equal keys (repeated empty-slot
// zeros) are ranked by position, so every output slot 0..n-1 is written exactly once.
__device__ inline void block_sort_desc_small(const uint64_t *in, int n, uint64_t *out) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const uint64_t k = in[i];
        int r = 0;
        for (int j = 0; j < n; ++j) r += (in[j] > k) || (in[j] == k && j < i);
        out[r] = k;
    }
    __syncthreads();
}

}  // namespace hsa
