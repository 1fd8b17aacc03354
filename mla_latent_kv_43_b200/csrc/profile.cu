// Per-kernel timing with CUDA events recorded on the launching stream.
#include <cuda_runtime.h>
#include <string.h>

#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "mla.h"
#include "profile.h"

namespace mla {
namespace {

struct Rec {
    std::string name;
    cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
std::vector<cudaEvent_t> g_free;
std::vector<Rec> g_done;
thread_local Rec g_open;
thread_local bool g_has_open = false;

cudaEvent_t take_event() {
    if (!g_free.empty()) {
        cudaEvent_t e = g_free.back();
        g_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

}  // namespace

void prof_begin(cudaStream_t stream, const char* name) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_on) return;
    g_open.name = name;
    g_open.a = take_event();
    g_open.b = take_event();
    cudaEventRecord(g_open.a, stream);
    g_has_open = true;
}

void prof_end(cudaStream_t stream) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_on || !g_has_open) return;
    cudaEventRecord(g_open.b, stream);
    g_done.push_back(g_open);
    g_has_open = false;
}

}  // namespace mla

extern "C" {

int mla_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(mla::g_mu);
    mla::g_on = on != 0;
    if (!mla::g_on) {
        for (auto& r : mla::g_done) {
            cudaEventSynchronize(r.b);
            mla::g_free.push_back(r.a);
            mla::g_free.push_back(r.b);
        }
        mla::g_done.clear();
        for (cudaEvent_t e : mla::g_free) cudaEventDestroy(e);
        mla::g_free.clear();
    }
    return MLA_OK;
}

int mla_profile_read(char* names, size_t names_len, int32_t* counts, float* total_ms,
                     int32_t max_kernels) {
    if (!names || !counts || !total_ms || max_kernels <= 0) return -MLA_ERR_ARG;
    std::lock_guard<std::mutex> lk(mla::g_mu);
    std::map<std::string, std::pair<int, double>> agg;
    int rc = 0;
    for (auto& r : mla::g_done) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
            rc = -MLA_ERR_CUDA;
        auto& v = agg[r.name];
        v.first += 1;
        v.second += ms;
        mla::g_free.push_back(r.a);
        mla::g_free.push_back(r.b);
    }
    mla::g_done.clear();
    if (rc) return rc;
    int n = 0;
    size_t pos = 0;
    for (auto& kv : agg) {
        if (n >= max_kernels || pos + kv.first.size() + 1 > names_len) break;
        memcpy(names + pos, kv.first.c_str(), kv.first.size() + 1);
        pos += kv.first.size() + 1;
        counts[n] = kv.second.first;
        total_ms[n] = (float)kv.second.second;
        ++n;
    }
    return n;
}

}  // extern "C"
