// decode_noalloc.cu -- hsa_decode_noalloc: HSA decode for callers that cannot allocate device
// memory.
//
// hsa_decode needs a caller-provided workspace for its scratch data (per-range candidates, ticket
// counters, per-chunk partial outputs). Some callers cannot obtain one at the moment they run a
// decode step: an inference engine that has handed all of HBM to its KV-cache pool and allows no
// allocation while serving, a plain C caller with no caching allocator for whom a cudaMalloc /
// cudaFree pair per step would synchronise the whole device, or a host thread that must not take
// the driver's allocation locks on a latency-critical path. For them this entry point keeps the
// scratch in one fixed array of device memory that belongs to the library, so the call allocates
// nothing; the caller passes only inputs and outputs. It launches the same kernels as hsa_decode.
#include <cmath>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/hsa.h"
#include "common.cuh"
#include "launch.h"

namespace {

// Fixed scratch for hsa_decode_noalloc. Every GPU that loads the library holds these bytes until the
// process exits. In host code the name is only a host-side stand-in for the device array, never a
// device address: the device address is looked up with cudaGetSymbolAddress below.
constexpr size_t kNoAllocScratchBytes = HSA_DECODE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

hsa_status fail(hsa_status st, const std::string &msg) {
    hsa::set_last_error(msg.c_str());
    return st;
}

size_t round_up(size_t x) { return (x + 255) / 256 * 256; }

// Layout inside the fixed array: error flag, ticket counters, candidates, selection (when the caller
// passes none), per-chunk partial outputs -- the scratch the decode kernels need. The number of scan
// ranges comes from the same plan that hsa_decode's workspace and launches use (one query row per key
// head here), so the two cannot disagree.
struct NoAllocLayout {
    size_t err, cand, counters, sel_idx, sel_w, partial, total;
};

NoAllocLayout layout(const hsa::DecodePlan &plan, int B, int H, int D, int topk) {
    const int64_t nsplit = plan.nsplit;
    const size_t BH = (size_t)B * H;
    NoAllocLayout l{};
    size_t off = 0;
    l.err = off;      off += round_up(sizeof(int32_t));
    l.counters = off; off += round_up(2 * BH * sizeof(unsigned));  // after the flag: one memset clears both
    l.cand = off;     off += round_up(BH * nsplit * topk * sizeof(uint64_t));
    l.sel_idx = off;  off += round_up(BH * topk * sizeof(int32_t));
    l.sel_w = off;    off += round_up(BH * topk * sizeof(float));
    l.partial = off;  off += round_up(BH * topk * D * sizeof(float));
    l.total = off;
    return l;
}

// Device address of the fixed array on the current device, looked up once per device with that
// device current. The first call on a device therefore does this set-up.
hsa_status scratch_address(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(HSA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(HSA_ERR_UNSUPPORTED, "device ordinal beyond 63");
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || !p)
            return fail(HSA_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return HSA_OK;
}

}  // namespace

extern "C" {

hsa_status hsa_decode_noalloc(const hsa_bf16 *q, const hsa_bf16 *Kc, const hsa_bf16 *Vc, const hsa_bf16 *Lc,
                              const int64_t *cache_len, int64_t Tmax, int B, int H, int D, int chunk, int topk,
                              float scale, hsa_bf16 *out, int32_t *sel_idx, float *sel_w, void *stream) {
    hsa::set_last_error("");
    // the argument checks of hsa_decode
    if (B < 1 || H < 1 || topk < 1 || D < 1 || chunk < 1 || Tmax < 0)
        return fail(HSA_ERR_INVALID_ARG, "B, H, topk, D, chunk must be >= 1 and Tmax >= 0");
    if (D != 64 && D != 128) return fail(HSA_ERR_UNSUPPORTED, "head dim must be 64 or 128");
    if (chunk != hsa::kChunk) return fail(HSA_ERR_UNSUPPORTED, "chunk must be 64");
    if (topk > 64) return fail(HSA_ERR_UNSUPPORTED, "topk must be <= 64");
    if (!q || !Kc || !Vc || !Lc || !cache_len || !out)
        return fail(HSA_ERR_INVALID_ARG, "q, Kc, Vc, Lc, cache_len and out must not be NULL");
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!al16(q) || !al16(Kc) || !al16(Vc) || !al16(Lc) || !al16(out) || (sel_idx && !al16(sel_idx)) ||
        (sel_w && !al16(sel_w)) || (reinterpret_cast<uintptr_t>(cache_len) & 7u))
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned (cache_len 8-byte)");
    const int64_t Nmax = Tmax / hsa::kChunk;
    if (Nmax >= 2147483647LL) return fail(HSA_ERR_UNSUPPORTED, "Tmax / 64 must stay below 2^31");
    const hsa::DecodePlan plan = hsa::decode_plan(Nmax, topk, B, H, H, 1);
    if (hsa::decode_plan_smem(plan, topk) > 227 * 1024)
        return fail(HSA_ERR_UNSUPPORTED, "Tmax too large for this topk (scan merge exceeds shared memory)");
    const NoAllocLayout l = layout(plan, B, H, D, topk);
    if (l.total > kNoAllocScratchBytes) {
        char buf[256];
        snprintf(buf, sizeof(buf),
                 "hsa_decode_noalloc: this call needs %zu bytes of scratch but the built-in array holds %zu; "
                 "use hsa_decode with a caller-provided workspace",
                 l.total, kNoAllocScratchBytes);
        return fail(HSA_ERR_UNSUPPORTED, buf);
    }
    void *base = nullptr;
    hsa_status st = scratch_address(&base);
    if (st != HSA_OK) return st;
    char *b = static_cast<char *>(base);
    hsa::DecodeArgs a{};
    a.qs = q; a.q = q; a.Kc = Kc; a.Vc = Vc; a.Lc = Lc; a.cache_len = cache_len;
    a.Tmax = Tmax; a.Nmax = Nmax;
    a.B = B; a.H = H; a.Hkv = H; a.D = D; a.K = topk;
    a.scale = scale > 0.0f ? scale : 1.0f / sqrtf((float)D);
    a.out = out;
    a.sel_idx = sel_idx ? sel_idx : reinterpret_cast<int32_t *>(b + l.sel_idx);
    a.sel_w = sel_w ? sel_w : reinterpret_cast<float *>(b + l.sel_w);
    a.cand = reinterpret_cast<uint64_t *>(b + l.cand);
    a.counters = reinterpret_cast<unsigned *>(b + l.counters);  // zeroed (with the flag) by launch_decode
    a.partial = reinterpret_cast<float *>(b + l.partial);
    a.err = reinterpret_cast<int32_t *>(b + l.err);
    const cudaError_t e = hsa::launch_decode(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(HSA_ERR_CUDA, std::string("hsa_decode_noalloc: ") + cudaGetErrorString(e));
    return HSA_OK;
}

}  // extern "C"
