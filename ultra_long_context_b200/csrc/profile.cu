// profile.cu -- optional per-launch timing with CUDA events on the launching stream.
//
// When enabled (hsa_profile_enable(1)), every kernel launch and memset issued by the library is
// bracketed by two events recorded on the caller's stream; hsa_profile_summary() waits for them and
// reports, per launch site, the number of launches and their summed device time. Disabled (the
// default), a scope costs one relaxed atomic load and records nothing.
#include <atomic>
#include <cstdio>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/hsa.h"
#include "profile.h"

namespace hsa {
namespace {

struct Record {
    const char *name;
    cudaEvent_t begin, end;
};

std::atomic<bool> g_enabled{false};
std::mutex g_mu;
std::vector<Record> g_records;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

}  // namespace

ProfScope::ProfScope(const char *name, cudaStream_t s) : idx_(-1), s_(s) {
    if (!g_enabled.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_mu);
    Record r{name, take_event(), take_event()};
    if (!r.begin || !r.end) return;
    cudaEventRecord(r.begin, s);
    g_records.push_back(r);
    idx_ = (int)g_records.size() - 1;
}

ProfScope::~ProfScope() {
    if (idx_ < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    if (idx_ < (int)g_records.size()) cudaEventRecord(g_records[idx_].end, s_);
}

}  // namespace hsa

extern "C" {

int hsa_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(hsa::g_mu);
    for (auto &r : hsa::g_records) {
        hsa::g_pool.push_back(r.begin);
        hsa::g_pool.push_back(r.end);
    }
    hsa::g_records.clear();
    hsa::g_enabled.store(on != 0);
    return 0;
}

int hsa_profile_summary(char *buf, size_t cap) {
    std::lock_guard<std::mutex> lk(hsa::g_mu);
    std::vector<std::string> names;
    std::vector<double> ms;
    std::vector<int> count;
    for (auto &r : hsa::g_records) {
        if (cudaEventSynchronize(r.end) != cudaSuccess) return -1;
        float t = 0.0f;
        if (cudaEventElapsedTime(&t, r.begin, r.end) != cudaSuccess) return -1;
        size_t i = 0;
        while (i < names.size() && names[i] != r.name) ++i;
        if (i == names.size()) {
            names.push_back(r.name);
            ms.push_back(0.0);
            count.push_back(0);
        }
        ms[i] += t;
        count[i] += 1;
    }
    std::string out;
    char line[256];
    for (size_t i = 0; i < names.size(); ++i) {
        snprintf(line, sizeof(line), "%s,%d,%.6f\n", names[i].c_str(), count[i], ms[i]);
        out += line;
    }
    if (buf && cap > 0) {
        const size_t n = out.size() < cap - 1 ? out.size() : cap - 1;
        memcpy(buf, out.data(), n);
        buf[n] = '\0';
    }
    return (int)out.size();
}

}  // extern "C"
