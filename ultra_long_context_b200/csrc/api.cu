// api.cu -- the C ABI declared in include/hsa.h: host-side validation, workspace carving and
// launches on the caller's stream. Nothing here allocates device memory or computes any part of the
// operator (hsa_workspace_status alone synchronises, by its definition); every step of HSA runs in the
// kernels of decode.cu / prefill.cu / score_wide.cu / score_tc.cu / attn_tc.cu / backward.cu / bwd_tc.cu / qknorm.cu /
// varlen.cu.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/hsa.h"
#include "common.cuh"
#include "launch.h"

namespace {

thread_local std::string g_last_error;

hsa_status fail(hsa_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

hsa_status cuda_status(cudaError_t e, const char *where) {
    if (e == cudaSuccess) return HSA_OK;
    return fail(HSA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Sequential carve-out of a caller-provided workspace.
struct Carver {
    char *base;
    size_t used = 0;
    template <typename T>
    T *take(size_t count) {
        T *p = base ? reinterpret_cast<T *>(base + used) : nullptr;
        used += round_up(count * sizeof(T));
        return p;
    }
};

hsa_status check_common(int B, int H, int D, int chunk, int topk, int topk_max) {
    if (B < 1 || H < 1) return fail(HSA_ERR_INVALID_ARG, "B and H must be >= 1 (got B=%d H=%d)", B, H);
    if (topk < 1) return fail(HSA_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", topk);
    if (D < 1) return fail(HSA_ERR_INVALID_ARG, "D must be >= 1 (got %d)", D);
    if (chunk < 1) return fail(HSA_ERR_INVALID_ARG, "chunk must be >= 1 (got %d)", chunk);
    if (D != 64 && D != 128) return fail(HSA_ERR_UNSUPPORTED, "head dim D=%d not supported (64 or 128)", D);
    if (chunk != hsa::kChunk) return fail(HSA_ERR_UNSUPPORTED, "chunk=%d not supported (64 only)", chunk);
    if (topk > topk_max) return fail(HSA_ERR_UNSUPPORTED, "topk=%d not supported (max %d)", topk, topk_max);
    return HSA_OK;
}

hsa_status check_ws(void *ws, size_t bytes, size_t need) {
    if (need == 0) return HSA_OK;
    if (!ws) return fail(HSA_ERR_WORKSPACE, "workspace is NULL but %zu bytes are needed", need);
    if (reinterpret_cast<uintptr_t>(ws) % kAlign) return fail(HSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    if (bytes < need) return fail(HSA_ERR_WORKSPACE, "workspace too small: %zu < %zu bytes", bytes, need);
    return HSA_OK;
}

// ---- forward / backward workspace layout ----
struct FwdLayout {
    float *o_acc;
    int32_t *sel_idx;
    float *sel_w;
    int32_t *chunk_count, *chunk_off, *tile_off, *chunk_cursor, *pair_row;
    float *pair_w;
    hsa::PairTile *tiles;
    int32_t *num_tiles, *err;
    float *delta;
    int32_t *pair_slot;
    float *ds_pair;  // [B*H*T, topk] ds per (token, slot): separate retrieval query or query-key norm
    uint16_t *Qn, *Kn;  // [B*H*T, D] bf16 normalised copies: query-key norm only
    size_t bytes;
    int max_tiles;
};

// qslc: the backward keeps ds per pair (a separate retrieval query, or the raw query retrieving while
// the normalised one attends); qk_norm: room for the normalised copies of Q and K.
FwdLayout fwd_layout(void *ws, int B, int H, int T, int D, int topk, bool backward, bool qslc = false,
                     bool qk_norm = false) {
    FwdLayout l{};
    Carver c{static_cast<char *>(ws)};
    l.err = c.take<int32_t>(1);  // first: hsa_workspace_status reads it at offset 0
    const size_t rows = (size_t)B * H * T, chunks = (size_t)B * H * (T / 64), pairs = rows * topk;
    l.max_tiles = (int)hsa::forward_max_tiles(B, H, T, topk);
    // right after the error flag: the three are zeroed by one memset
    l.chunk_count = c.take<int32_t>(chunks);
    l.chunk_cursor = c.take<int32_t>(chunks);
    l.o_acc = backward ? nullptr : c.take<float>(rows * D);
    l.sel_idx = backward ? nullptr : c.take<int32_t>(pairs);
    l.sel_w = backward ? nullptr : c.take<float>(pairs);
    l.chunk_off = c.take<int32_t>(chunks + 1);
    l.tile_off = c.take<int32_t>(chunks + 1);
    l.pair_row = c.take<int32_t>(pairs);
    l.pair_w = c.take<float>(pairs);
    l.tiles = c.take<hsa::PairTile>((size_t)l.max_tiles);
    l.num_tiles = c.take<int32_t>(1);
    l.delta = backward ? c.take<float>(rows) : nullptr;
    l.pair_slot = backward ? c.take<int32_t>(pairs) : nullptr;
    l.ds_pair = backward && (qslc || qk_norm) ? c.take<float>(pairs) : nullptr;
    l.Qn = qk_norm ? c.take<uint16_t>(rows * D) : nullptr;
    l.Kn = qk_norm ? c.take<uint16_t>(rows * D) : nullptr;
    l.bytes = c.used;
    return l;
}

struct DecLayout {
    int32_t *err;
    uint64_t *cand;
    unsigned *counters;
    int32_t *sel_idx;
    float *sel_w, *partial;
    size_t bytes;
};

DecLayout dec_layout(void *ws, int B, int H, int Hkv, int Tq, int64_t Tmax, int D, int topk) {
    DecLayout l{};
    Carver c{static_cast<char *>(ws)};
    const hsa::DecodePlan pl = hsa::decode_plan(Tmax / 64, topk, B, H, Hkv, Tq);
    const int64_t nsplit = pl.nsplit;
    const size_t BH = (size_t)B * H * Tq;  // query rows
    l.err = c.take<int32_t>(1);  // first: hsa_workspace_status reads it at offset 0
    l.counters = c.take<unsigned>(2 * BH);  // right after the flag: launch_decode zeroes both with one memset
    l.cand = c.take<uint64_t>(BH * nsplit * topk);
    l.sel_idx = c.take<int32_t>(BH * topk);
    l.sel_w = c.take<float>(BH * topk);
    l.partial = c.take<float>(BH * topk * D);
    l.bytes = c.used;
    return l;
}

float resolve_scale(float scale, int D) { return scale > 0.0f ? scale : 1.0f / sqrtf((float)D); }

// Checks of the *_ex arguments shared by the three calls.
hsa_status check_ex(int H, int Hkv, unsigned flags) {
    if (flags & ~HSA_QK_NORM) return fail(HSA_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags & ~HSA_QK_NORM);
    if (Hkv < 1 || H % Hkv != 0)
        return fail(HSA_ERR_INVALID_ARG, "H (%d) must be a positive multiple of Hkv (%d)", H, Hkv);
    return HSA_OK;
}

}  // namespace

namespace hsa {
// Lets other translation units of the library report through hsa_last_error().
void set_last_error(const char *msg) { g_last_error = msg ? msg : ""; }
}  // namespace hsa

extern "C" {

const char *hsa_last_error(void) { return g_last_error.c_str(); }

hsa_status hsa_workspace_status(const void *workspace, void *stream) {
    g_last_error.clear();
    if (!workspace) return fail(HSA_ERR_INVALID_ARG, "workspace must not be NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    int32_t flag = 0;
    if (e == cudaSuccess) e = cudaMemcpy(&flag, workspace, sizeof(flag), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e, "hsa_workspace_status");
    if (flag != 0)
        return fail(HSA_ERR_TIMEOUT, "a bounded device-side wait ran out in the last call on this workspace (flag %d)",
                    (int)flag);
    return HSA_OK;
}

size_t hsa_forward_workspace_size(int B, int H, int T, int D, int chunk, int topk) {
    (void)chunk;
    if (B < 1 || H < 1 || T < 1 || D < 1 || topk < 1) return 0;
    return fwd_layout(nullptr, B, H, T, D, topk, false).bytes;
}

size_t hsa_forward_ex_workspace_size(int B, int H, int Hkv, int T, int D, int chunk, int topk, unsigned flags) {
    (void)chunk;
    if (B < 1 || H < 1 || Hkv < 1 || T < 1 || D < 1 || topk < 1) return 0;
    return fwd_layout(nullptr, B, H, T, D, topk, false, false, (flags & HSA_QK_NORM) != 0).bytes;
}

// Qs retrieves (Step 2 scores, Step 4 weights), Q attends (Step 3); the single-query call passes Q twice.
static hsa_status forward_impl(const char *name, const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K,
                               const hsa_bf16 *V, const hsa_bf16 *L, int B, int H, int Hkv, int T, int D, int chunk,
                               int topk,
                               float scale, bool qk_norm, hsa_bf16 *out, int32_t *sel_idx, float *sel_w,
                               void *workspace, size_t workspace_bytes, void *stream,
                               const int32_t *cu_seqlens = nullptr) {
    g_last_error.clear();
    hsa_status st = check_common(B, H, D, chunk, topk, 64);
    if (st != HSA_OK) return st;
    if (T < 1) return fail(HSA_ERR_INVALID_ARG, "T must be >= 1 (got %d)", T);
    if ((double)B * H * T * topk >= 2147483647.0 || (double)B * H * T * D >= 9.0e15)
        return fail(HSA_ERR_UNSUPPORTED, "B*H*T*topk must stay below 2^31");
    if (!Qs || !Q || !K || !V || !out) return fail(HSA_ERR_INVALID_ARG, "Q, Qs, K, V and out must not be NULL");
    if (T >= 64 && !L) return fail(HSA_ERR_INVALID_ARG, "L must not be NULL when T >= 64");
    if (!aligned16(Qs) || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || (L && !aligned16(L)))
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if ((sel_idx && !aligned16(sel_idx)) || (sel_w && !aligned16(sel_w)))
        return fail(HSA_ERR_INVALID_ARG, "sel_idx / sel_w must be 16-byte aligned");
    FwdLayout need = fwd_layout(nullptr, B, H, T, D, topk, false, false, qk_norm);
    if ((st = check_ws(workspace, workspace_bytes, need.bytes)) != HSA_OK) return st;
    FwdLayout l = fwd_layout(workspace, B, H, T, D, topk, false, false, qk_norm);
    hsa::ForwardArgs a{};
    a.qk_norm = qk_norm; a.Qn = l.Qn; a.Kn = l.Kn;
    a.cu_seqlens = cu_seqlens;
    a.Qs = Qs; a.Q = Q; a.K = K; a.V = V; a.L = L;
    a.B = B; a.H = H; a.Hkv = Hkv; a.T = T; a.D = D; a.N = T / 64; a.topk = topk;
    a.scale = resolve_scale(scale, D);
    a.out = out;
    a.sel_idx = sel_idx ? sel_idx : l.sel_idx;
    a.sel_w = sel_w ? sel_w : l.sel_w;
    a.o_acc = l.o_acc;
    a.chunk_count = l.chunk_count; a.chunk_off = l.chunk_off; a.tile_off = l.tile_off;
    a.chunk_cursor = l.chunk_cursor;
    a.pair_row = l.pair_row; a.pair_w = l.pair_w; a.tiles = l.tiles; a.num_tiles = l.num_tiles;
    a.err = l.err;
    a.max_tiles = l.max_tiles;
    return cuda_status(hsa::launch_forward(a, static_cast<cudaStream_t>(stream)), name);
}

hsa_status hsa_forward(const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V, const hsa_bf16 *L, int B, int H,
                       int T, int D, int chunk, int topk, float scale, hsa_bf16 *out, int32_t *sel_idx,
                       float *sel_w, void *workspace, size_t workspace_bytes, void *stream) {
    return forward_impl("hsa_forward", Q, Q, K, V, L, B, H, H, T, D, chunk, topk, scale, false, out, sel_idx, sel_w,
                        workspace, workspace_bytes, stream);
}

hsa_status hsa_forward_ex(const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V,
                          const hsa_bf16 *L, int B, int H, int Hkv, int T, int D, int chunk, int topk, float scale,
                          unsigned flags, hsa_bf16 *out, int32_t *sel_idx, float *sel_w, void *workspace,
                          size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    hsa_status st = check_ex(H, Hkv, flags);
    if (st != HSA_OK) return st;
    return forward_impl("hsa_forward_ex", Qs ? Qs : Q, Q, K, V, L, B, H, Hkv, T, D, chunk, topk, scale,
                        (flags & HSA_QK_NORM) != 0, out, sel_idx, sel_w, workspace, workspace_bytes, stream);
}

size_t hsa_decode_workspace_size(int B, int H, int64_t Tmax, int D, int chunk, int topk) {
    (void)chunk;
    if (B < 1 || H < 1 || Tmax < 0 || D < 1 || topk < 1) return 0;
    return dec_layout(nullptr, B, H, H, 1, Tmax, D, topk).bytes;
}

size_t hsa_decode_ex_workspace_size(int B, int H, int Hkv, int Tq, int64_t Tmax, int D, int chunk, int topk,
                                    unsigned flags) {
    (void)chunk;
    (void)flags;
    if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || Tq < 1 || Tmax < 0 || D < 1 || topk < 1) return 0;
    return dec_layout(nullptr, B, H, Hkv, Tq, Tmax, D, topk).bytes;
}

static hsa_status decode_impl(const char *name, const hsa_bf16 *qs, const hsa_bf16 *q, const hsa_bf16 *Kc,
                              const hsa_bf16 *Vc, const hsa_bf16 *Lc, const int64_t *cache_len, int64_t Tmax, int B,
                              int H, int Hkv, int Tq, int D, int chunk, int topk, float scale, bool qk_norm,
                              hsa_bf16 *out,
                              int32_t *sel_idx, float *sel_w, void *workspace, size_t workspace_bytes,
                              void *stream) {
    g_last_error.clear();
    hsa_status st = check_common(B, H, D, chunk, topk, 64);
    if (st != HSA_OK) return st;
    if (Tmax < 0) return fail(HSA_ERR_INVALID_ARG, "Tmax must be >= 0");
    if (Tmax / 64 >= 2147483647LL) return fail(HSA_ERR_UNSUPPORTED, "Tmax / 64 must stay below 2^31");
    if (!qs || !q || !Kc || !Vc || !Lc || !cache_len || !out)
        return fail(HSA_ERR_INVALID_ARG, "q, qs, Kc, Vc, Lc, cache_len and out must not be NULL");
    if (!aligned16(qs) || !aligned16(q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(Lc) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(cache_len) & 7u))
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned (cache_len 8-byte)");
    if ((sel_idx && !aligned16(sel_idx)) || (sel_w && !aligned16(sel_w)))
        return fail(HSA_ERR_INVALID_ARG, "sel_idx / sel_w must be 16-byte aligned");
    if (Tq < 1 || Tq > 64) return fail(HSA_ERR_INVALID_ARG, "Tq must be in [1, 64] (got %d)", Tq);
    if ((double)B * H * Tq >= 2147483647.0) return fail(HSA_ERR_UNSUPPORTED, "B*H*Tq must stay below 2^31");
    const hsa::DecodePlan plan = hsa::decode_plan(Tmax / 64, topk, B, H, Hkv, Tq);
    if (Tq > 1 && !plan.grouped)
        return fail(HSA_ERR_UNSUPPORTED, "several query tokens per step need topk <= 32 (got %d) and a cache whose "
                    "landmark ranges fit the grouped scan", topk);
    if (hsa::decode_plan_smem(plan, topk) > 227 * 1024)
        return fail(HSA_ERR_UNSUPPORTED, "Tmax=%lld too large for topk=%d (scan merge exceeds shared memory)",
                    (long long)Tmax, topk);
    DecLayout need = dec_layout(nullptr, B, H, Hkv, Tq, Tmax, D, topk);
    if ((st = check_ws(workspace, workspace_bytes, need.bytes)) != HSA_OK) return st;
    DecLayout l = dec_layout(workspace, B, H, Hkv, Tq, Tmax, D, topk);
    hsa::DecodeArgs a{};
    a.qs = qs; a.q = q; a.Kc = Kc; a.Vc = Vc; a.Lc = Lc; a.cache_len = cache_len;
    a.Tmax = Tmax; a.Nmax = Tmax / 64;
    a.B = B; a.H = H; a.Hkv = Hkv; a.Tq = Tq; a.D = D; a.K = topk;
    a.scale = resolve_scale(scale, D);
    a.out = out;
    a.sel_idx = sel_idx ? sel_idx : l.sel_idx;
    a.sel_w = sel_w ? sel_w : l.sel_w;
    a.cand = l.cand; a.counters = l.counters; a.partial = l.partial;
    a.qk_norm = qk_norm;
    a.err = l.err;  // cleared by launch_decode with the counters, so a status query reports this call
    return cuda_status(hsa::launch_decode(a, static_cast<cudaStream_t>(stream)), name);
}

hsa_status hsa_decode(const hsa_bf16 *q, const hsa_bf16 *Kc, const hsa_bf16 *Vc, const hsa_bf16 *Lc,
                      const int64_t *cache_len, int64_t Tmax, int B, int H, int D, int chunk, int topk,
                      float scale, hsa_bf16 *out, int32_t *sel_idx, float *sel_w, void *workspace,
                      size_t workspace_bytes, void *stream) {
    return decode_impl("hsa_decode", q, q, Kc, Vc, Lc, cache_len, Tmax, B, H, H, 1, D, chunk, topk, scale, false, out,
                       sel_idx, sel_w, workspace, workspace_bytes, stream);
}

hsa_status hsa_decode_ex(const hsa_bf16 *qs, const hsa_bf16 *q, const hsa_bf16 *Kc, const hsa_bf16 *Vc,
                         const hsa_bf16 *Lc, const int64_t *cache_len, int64_t Tmax, int B, int H, int Hkv, int Tq,
                         int D, int chunk, int topk, float scale, unsigned flags, hsa_bf16 *out, int32_t *sel_idx,
                         float *sel_w, void *workspace, size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    hsa_status st = check_ex(H, Hkv, flags);
    if (st != HSA_OK) return st;
    return decode_impl("hsa_decode_ex", qs ? qs : q, q, Kc, Vc, Lc, cache_len, Tmax, B, H, Hkv, Tq, D, chunk, topk,
                       scale, (flags & HSA_QK_NORM) != 0, out, sel_idx, sel_w, workspace, workspace_bytes, stream);
}

size_t hsa_backward_workspace_size(int B, int H, int T, int D, int chunk, int topk) {
    (void)chunk;
    if (B < 1 || H < 1 || T < 1 || D < 1 || topk < 1) return 0;
    return fwd_layout(nullptr, B, H, T, D, topk, true).bytes;
}

size_t hsa_backward_ex_workspace_size(int B, int H, int Hkv, int T, int D, int chunk, int topk, unsigned flags) {
    (void)chunk;
    if (B < 1 || H < 1 || Hkv < 1 || T < 1 || D < 1 || topk < 1) return 0;
    return fwd_layout(nullptr, B, H, T, D, topk, true, true, (flags & HSA_QK_NORM) != 0).bytes;
}

// Qs / dQs are NULL for the single-query call (Q retrieves too and dQ takes both parts).
static hsa_status backward_impl(const char *name, const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K,
                                const hsa_bf16 *V, const hsa_bf16 *L, const hsa_bf16 *out, const hsa_bf16 *dout,
                                const int32_t *sel_idx, const float *sel_w, int B, int H, int Hkv, int T, int D,
                                int chunk, int topk, float scale, float *dQ, float *dK, float *dV, float *dL, float *dQs,
                                bool qslc, bool qk_norm, void *workspace, size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    hsa_status st = check_common(B, H, D, chunk, topk, 64);
    if (st != HSA_OK) return st;
    if (T < 1) return fail(HSA_ERR_INVALID_ARG, "T must be >= 1 (got %d)", T);
    if ((double)B * H * T * topk >= 2147483647.0)
        return fail(HSA_ERR_UNSUPPORTED, "B*H*T*topk must stay below 2^31");
    if (!Q || !K || !V || !out || !dout || !sel_idx || !sel_w || !dQ || !dK || !dV)
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must not be NULL");
    if (T >= 64 && (!L || !dL)) return fail(HSA_ERR_INVALID_ARG, "L and dL must not be NULL when T >= 64");
    if (qslc && (!Qs || !dQs)) return fail(HSA_ERR_INVALID_ARG, "Qs and dQs must not be NULL");
    if (qslc && (!aligned16(Qs) || !aligned16(dQs)))
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out) || !aligned16(dout) ||
        !aligned16(sel_idx) || !aligned16(sel_w) || !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) ||
        (L && !aligned16(L)) || (dL && !aligned16(dL)))
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    FwdLayout need = fwd_layout(nullptr, B, H, T, D, topk, true, qslc, qk_norm);
    if ((st = check_ws(workspace, workspace_bytes, need.bytes)) != HSA_OK) return st;
    FwdLayout l = fwd_layout(workspace, B, H, T, D, topk, true, qslc, qk_norm);
    hsa::BackwardArgs a{};
    a.qk_norm = qk_norm; a.Qn = l.Qn; a.Kn = l.Kn;
    a.Qs = qslc ? Qs : nullptr; a.dQs = qslc ? dQs : nullptr; a.ds_pair = l.ds_pair;
    a.Q = Q; a.K = K; a.V = V; a.L = L; a.out = out; a.dout = dout;
    a.sel_idx = sel_idx; a.sel_w = sel_w;
    a.B = B; a.H = H; a.Hkv = Hkv; a.T = T; a.D = D; a.N = T / 64; a.topk = topk;
    a.scale = resolve_scale(scale, D);
    a.dQ = dQ; a.dK = dK; a.dV = dV; a.dL = dL;
    a.delta = l.delta;
    a.chunk_count = l.chunk_count; a.chunk_off = l.chunk_off; a.tile_off = l.tile_off;
    a.chunk_cursor = l.chunk_cursor;
    a.pair_row = l.pair_row; a.pair_w = l.pair_w; a.pair_slot = l.pair_slot;
    a.tiles = l.tiles; a.num_tiles = l.num_tiles; a.max_tiles = l.max_tiles; a.err = l.err;
    return cuda_status(hsa::launch_backward(a, static_cast<cudaStream_t>(stream)), name);
}

hsa_status hsa_backward(const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V, const hsa_bf16 *L,
                        const hsa_bf16 *out, const hsa_bf16 *dout, const int32_t *sel_idx, const float *sel_w,
                        int B, int H, int T, int D, int chunk, int topk, float scale, float *dQ, float *dK,
                        float *dV, float *dL, void *workspace, size_t workspace_bytes, void *stream) {
    return backward_impl("hsa_backward", nullptr, Q, K, V, L, out, dout, sel_idx, sel_w, B, H, H, T, D, chunk, topk,
                         scale, dQ, dK, dV, dL, nullptr, false, false, workspace, workspace_bytes, stream);
}

hsa_status hsa_backward_ex(const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V,
                           const hsa_bf16 *L, const hsa_bf16 *out, const hsa_bf16 *dout, const int32_t *sel_idx,
                           const float *sel_w, int B, int H, int Hkv, int T, int D, int chunk, int topk, float scale,
                           unsigned flags, float *dQ, float *dK, float *dV, float *dL, float *dQs, void *workspace,
                           size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    hsa_status st = check_ex(H, Hkv, flags);
    if (st != HSA_OK) return st;
    if ((Qs == nullptr) != (dQs == nullptr))
        return fail(HSA_ERR_INVALID_ARG, "dQs must be given exactly when Qs is (got Qs %s, dQs %s)",
                    Qs ? "set" : "NULL", dQs ? "set" : "NULL");
    return backward_impl("hsa_backward_ex", Qs, Q, K, V, L, out, dout, sel_idx, sel_w, B, H, Hkv, T, D, chunk, topk,
                         scale, dQ, dK, dV, dL, dQs, Qs != nullptr, (flags & HSA_QK_NORM) != 0, workspace,
                         workspace_bytes, stream);
}

}  // extern "C"

// ---- variable-length batches: packed token-major tensors <-> a padded head-major batch ----

struct VarlenLayout {
    size_t inner;  // the padded call's own workspace, first, so that its status flag sits at offset 0
    int32_t *cuN;
    uint16_t *Q, *Qs, *K, *V, *L, *out, *dout;
    int32_t *sel_idx;
    float *sel_w;
    float *dQ, *dK, *dV, *dL, *dQs;
    size_t bytes;
};

static VarlenLayout varlen_layout(void *ws, int B, int H, int Hkv, int Tp, int D, int topk, bool qk_norm,
                                  bool backward) {
    VarlenLayout l{};
    l.inner = round_up(backward ? fwd_layout(nullptr, B, H, Tp, D, topk, true, true, qk_norm).bytes
                                : fwd_layout(nullptr, B, H, Tp, D, topk, false, false, qk_norm).bytes);
    Carver c{ws ? static_cast<char *>(ws) + l.inner : nullptr};
    const size_t rq = (size_t)B * H * Tp, rk = (size_t)B * Hkv * Tp, rl = (size_t)B * Hkv * (Tp / 64);
    l.cuN = c.take<int32_t>((size_t)B + 1);
    l.Q = c.take<uint16_t>(rq * D);
    l.Qs = c.take<uint16_t>(rq * D);  // room for a separate retrieval query (used only when one is given)
    l.K = c.take<uint16_t>(rk * D);
    l.V = c.take<uint16_t>(rk * D);
    l.L = c.take<uint16_t>(rl * D);
    l.out = c.take<uint16_t>(rq * D);
    l.sel_idx = c.take<int32_t>(rq * topk);
    l.sel_w = c.take<float>(rq * topk);
    if (backward) {
        l.dout = c.take<uint16_t>(rq * D);
        l.dQ = c.take<float>(rq * D);
        l.dK = c.take<float>(rk * D);
        l.dV = c.take<float>(rk * D);
        l.dL = c.take<float>(rl * D);
        l.dQs = c.take<float>(rq * D);
    }
    l.bytes = l.inner + c.used;
    return l;
}

// Shared checks of the two varlen calls; fills the padded length Tp.
static hsa_status varlen_check(const int32_t *cu_seqlens, int B, int max_seqlen, int H, int Hkv, int D, int chunk,
                               int topk, unsigned flags) {
    hsa_status st = check_ex(H, Hkv, flags);
    if (st != HSA_OK) return st;
    if ((st = check_common(B, H, D, chunk, topk, 64)) != HSA_OK) return st;
    if (max_seqlen < 1) return fail(HSA_ERR_INVALID_ARG, "max_seqlen must be >= 1 (got %d)", max_seqlen);
    if (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
        return fail(HSA_ERR_INVALID_ARG, "cu_seqlens must be a 4-byte aligned device array of B + 1 entries");
    if ((double)B * H * max_seqlen * topk >= 2147483647.0)
        return fail(HSA_ERR_UNSUPPORTED, "B*H*max_seqlen*topk must stay below 2^31");
    return HSA_OK;
}

extern "C" {

size_t hsa_forward_varlen_workspace_size(int B, int H, int Hkv, int max_seqlen, int D, int chunk, int topk,
                                         unsigned flags) {
    (void)chunk;
    if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || max_seqlen < 1 || D < 1 || topk < 1) return 0;
    return varlen_layout(nullptr, B, H, Hkv, max_seqlen, D, topk, (flags & HSA_QK_NORM) != 0, false).bytes;
}

hsa_status hsa_forward_varlen(const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V,
                              const hsa_bf16 *L, const int32_t *cu_seqlens, int B, int max_seqlen, int H, int Hkv,
                              int D, int chunk, int topk, float scale, unsigned flags, hsa_bf16 *out,
                              int32_t *sel_idx, float *sel_w, void *workspace, size_t workspace_bytes,
                              void *stream) {
    g_last_error.clear();
    hsa_status st = varlen_check(cu_seqlens, B, max_seqlen, H, Hkv, D, chunk, topk, flags);
    if (st != HSA_OK) return st;
    if (!Q || !K || !V || !L || !out || !sel_idx || !sel_w)
        return fail(HSA_ERR_INVALID_ARG, "Q, K, V, L, out, sel_idx and sel_w must not be NULL");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(L) || !aligned16(out) || (Qs && !aligned16(Qs)) ||
        (reinterpret_cast<uintptr_t>(sel_idx) & 3u) || (reinterpret_cast<uintptr_t>(sel_w) & 3u))
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned (sel_idx, sel_w 4-byte)");
    const bool qk = (flags & HSA_QK_NORM) != 0;
    const int Tp = max_seqlen;
    if ((st = check_ws(workspace, workspace_bytes, varlen_layout(nullptr, B, H, Hkv, Tp, D, topk, qk, false).bytes)) !=
        HSA_OK)
        return st;
    const VarlenLayout l = varlen_layout(workspace, B, H, Hkv, Tp, D, topk, qk, false);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = hsa::launch_chunk_offsets(cu_seqlens, B, l.cuN, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(Q, l.Q, cu_seqlens, B, H, Tp, D * 2, true, false, 0u, s);
    if (e == cudaSuccess && Qs) e = hsa::launch_varlen_rows(Qs, l.Qs, cu_seqlens, B, H, Tp, D * 2, true, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(K, l.K, cu_seqlens, B, Hkv, Tp, D * 2, true, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(V, l.V, cu_seqlens, B, Hkv, Tp, D * 2, true, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(L, l.L, l.cuN, B, Hkv, Tp / 64, D * 2, true, false, 0u, s);
    if (e != cudaSuccess) return cuda_status(e, "hsa_forward_varlen");
    st = forward_impl("hsa_forward_varlen", Qs ? l.Qs : l.Q, l.Q, l.K, l.V, l.L, B, H, Hkv, Tp, D, chunk, topk, scale,
                      qk, l.out, l.sel_idx, l.sel_w, workspace, l.inner, stream, cu_seqlens);
    if (st != HSA_OK) return st;
    e = hsa::launch_varlen_rows(l.out, out, cu_seqlens, B, H, Tp, D * 2, false, false, 0u, s);
    if (e == cudaSuccess)
        e = hsa::launch_varlen_rows(l.sel_idx, sel_idx, cu_seqlens, B, H, Tp, topk * 4, false, false, 0u, s);
    if (e == cudaSuccess)
        e = hsa::launch_varlen_rows(l.sel_w, sel_w, cu_seqlens, B, H, Tp, topk * 4, false, false, 0u, s);
    return cuda_status(e, "hsa_forward_varlen");
}

size_t hsa_backward_varlen_workspace_size(int B, int H, int Hkv, int max_seqlen, int D, int chunk, int topk,
                                          unsigned flags) {
    (void)chunk;
    if (B < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || max_seqlen < 1 || D < 1 || topk < 1) return 0;
    return varlen_layout(nullptr, B, H, Hkv, max_seqlen, D, topk, (flags & HSA_QK_NORM) != 0, true).bytes;
}

hsa_status hsa_backward_varlen(const hsa_bf16 *Qs, const hsa_bf16 *Q, const hsa_bf16 *K, const hsa_bf16 *V,
                               const hsa_bf16 *L, const hsa_bf16 *out, const hsa_bf16 *dout, const int32_t *sel_idx,
                               const float *sel_w, const int32_t *cu_seqlens, int B, int max_seqlen, int H, int Hkv,
                               int D, int chunk, int topk, float scale, unsigned flags, float *dQ, float *dK, float *dV,
                               float *dL, float *dQs, void *workspace, size_t workspace_bytes, void *stream) {
    g_last_error.clear();
    hsa_status st = varlen_check(cu_seqlens, B, max_seqlen, H, Hkv, D, chunk, topk, flags);
    if (st != HSA_OK) return st;
    if (!Q || !K || !V || !L || !out || !dout || !sel_idx || !sel_w || !dQ || !dK || !dV || !dL)
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must not be NULL (dQs: exactly when Qs is given)");
    if ((Qs == nullptr) != (dQs == nullptr))
        return fail(HSA_ERR_INVALID_ARG, "dQs must be given exactly when Qs is");
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(L) || !aligned16(out) || !aligned16(dout) ||
        !aligned16(dQ) || !aligned16(dK) || !aligned16(dV) || !aligned16(dL) || (Qs && !aligned16(Qs)) ||
        (dQs && !aligned16(dQs)) || (reinterpret_cast<uintptr_t>(sel_idx) & 3u) ||
        (reinterpret_cast<uintptr_t>(sel_w) & 3u))
        return fail(HSA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned (sel_idx, sel_w 4-byte)");
    const bool qk = (flags & HSA_QK_NORM) != 0;
    const int Tp = max_seqlen;
    if ((st = check_ws(workspace, workspace_bytes, varlen_layout(nullptr, B, H, Hkv, Tp, D, topk, qk, true).bytes)) !=
        HSA_OK)
        return st;
    const VarlenLayout l = varlen_layout(workspace, B, H, Hkv, Tp, D, topk, qk, true);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int row = D * 2;
    cudaError_t e = hsa::launch_chunk_offsets(cu_seqlens, B, l.cuN, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(Q, l.Q, cu_seqlens, B, H, Tp, row, true, false, 0u, s);
    if (e == cudaSuccess && Qs) e = hsa::launch_varlen_rows(Qs, l.Qs, cu_seqlens, B, H, Tp, row, true, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(K, l.K, cu_seqlens, B, Hkv, Tp, row, true, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(V, l.V, cu_seqlens, B, Hkv, Tp, row, true, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(L, l.L, l.cuN, B, Hkv, Tp / 64, row, true, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(out, l.out, cu_seqlens, B, H, Tp, row, true, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(dout, l.dout, cu_seqlens, B, H, Tp, row, true, false, 0u, s);
    // padded rows select nothing: chunk -1, weight 0
    if (e == cudaSuccess)
        e = hsa::launch_varlen_rows(sel_idx, l.sel_idx, cu_seqlens, B, H, Tp, topk * 4, true, true, 0xffffffffu, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(sel_w, l.sel_w, cu_seqlens, B, H, Tp, topk * 4, true, true, 0u, s);
    if (e != cudaSuccess) return cuda_status(e, "hsa_backward_varlen");
    st = backward_impl("hsa_backward_varlen", Qs ? l.Qs : nullptr, l.Q, l.K, l.V, l.L, l.out, l.dout, l.sel_idx,
                       l.sel_w, B, H, Hkv, Tp, D, chunk, topk, scale, l.dQ, l.dK, l.dV, l.dL, Qs ? l.dQs : nullptr,
                       Qs != nullptr, qk, workspace, l.inner, stream);
    if (st != HSA_OK) return st;
    const int frow = D * 4;
    e = hsa::launch_varlen_rows(l.dQ, dQ, cu_seqlens, B, H, Tp, frow, false, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(l.dK, dK, cu_seqlens, B, Hkv, Tp, frow, false, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(l.dV, dV, cu_seqlens, B, Hkv, Tp, frow, false, false, 0u, s);
    if (e == cudaSuccess) e = hsa::launch_varlen_rows(l.dL, dL, l.cuN, B, Hkv, Tp / 64, frow, false, false, 0u, s);
    if (e == cudaSuccess && Qs) e = hsa::launch_varlen_rows(l.dQs, dQs, cu_seqlens, B, H, Tp, frow, false, false, 0u, s);
    return cuda_status(e, "hsa_backward_varlen");
}

}  // extern "C"
