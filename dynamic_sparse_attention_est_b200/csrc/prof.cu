// prof.cu -- optional launch timing: a CUDA event pair around each of the
// library's kernel launches (or short launch sequences), on the launching
// stream, aggregated by name when read back.  Off by default; when on, each
// scope costs two event records.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace minf {

namespace {

std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mu;

struct ProfRec {
    const char *name;
    int dev;  // device the events belong to
    cudaEvent_t a, b;
};
std::vector<ProfRec> g_recs;
std::vector<std::pair<int, cudaEvent_t>> g_pool;  // (device, event) ready for reuse

// An event of device `dev` (the current device); the caller holds g_prof_mu.
cudaEvent_t take_event(int dev) {
    for (size_t i = 0; i < g_pool.size(); ++i) {
        if (g_pool[i].first == dev) {
            const cudaEvent_t e = g_pool[i].second;
            g_pool[i] = g_pool.back();
            g_pool.pop_back();
            return e;
        }
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return e;
}

}  // namespace

ProfScope::ProfScope(const char *name, cudaStream_t st) : st_(st), end_(nullptr) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return;
    }
    std::lock_guard<std::mutex> lk(g_prof_mu);
    const cudaEvent_t a = take_event(dev), b = take_event(dev);
    if (!a || !b || cudaEventRecord(a, st) != cudaSuccess) {
        cudaGetLastError();
        if (a) g_pool.emplace_back(dev, a);
        if (b) g_pool.emplace_back(dev, b);
        return;
    }
    g_recs.push_back({name, dev, a, b});
    end_ = b;
}

ProfScope::~ProfScope() {
    if (end_ && cudaEventRecord(end_, st_) != cudaSuccess) cudaGetLastError();
}

}  // namespace minf

using namespace minf;

extern "C" void minf_profile_enable(int on) { g_prof_on.store(on != 0); }

extern "C" int minf_profile_read(char *buf, size_t len) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    std::map<std::string, std::pair<long, double>> agg;  // name -> (launches, total ms)
    for (const ProfRec &r : g_recs) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
            auto &e = agg[r.name];
            e.first += 1;
            e.second += ms;
        } else {
            cudaGetLastError();
        }
    }
    if (buf) {  // a read, not a size query: the records go back to the pool
        for (const ProfRec &r : g_recs) {
            g_pool.emplace_back(r.dev, r.a);
            g_pool.emplace_back(r.dev, r.b);
        }
        g_recs.clear();
    }
    std::string out;
    char line[256];
    for (const auto &kv : agg) {
        snprintf(line, sizeof(line), "%s\t%ld\t%.6f\n", kv.first.c_str(), kv.second.first, kv.second.second);
        out += line;
    }
    if (buf && len > 0) {
        const size_t nc = std::min(len - 1, out.size());
        memcpy(buf, out.data(), nc);
        buf[nc] = '\0';
    }
    return (int)out.size();
}
