// twiddle.cu -- host-built twiddle tables in one static device array.
#include <cmath>
#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "fft_core.cuh"
#include "status.h"
#include "twiddle.h"

namespace hy {

namespace {

constexpr int kCapacity = 1 << 18;   // float2 entries (2 MiB)
__device__ float2 g_tw[kCapacity];

enum Kind { KIND_STAGES = 0, KIND_SPLIT = 1, KIND_POW2 = 2 };
using Key = std::tuple<int, int, int>;

// exp(-2πi e / N) with e reduced mod N exactly, in double, rounded to float
float2 w_forward(int64_t e, int64_t N) {
    int64_t r = e % N;
    if (r < 0) r += N;
    const double ang = 2.0 * 3.14159265358979323846264338327950288 * (double)r / (double)N;
    return make_float2((float)std::cos(ang), (float)(-std::sin(ang)));
}

struct Registry {
    std::vector<float2> host;
    std::map<Key, int64_t> offset;

    void add(const Key &key, const std::vector<float2> &v) {
        // 16-byte align each table
        while (host.size() % 2) host.push_back(make_float2(0.f, 0.f));
        offset[key] = (int64_t)host.size();
        host.insert(host.end(), v.begin(), v.end());
    }
    void add_stages(int log_m, int log_p) {
        Key key{KIND_STAGES, log_m, log_p};
        if (offset.count(key)) return;
        std::vector<float2> v;
        const int ns = plan_stages(log_m, log_p);
        for (int s = 1; s < ns; ++s) {
            const int R = 1 << plan_log_radix(log_m, log_p, s);
            const int p = 1 << plan_log_p(log_m, log_p, s);
            const int cols = plan_tw_cols(log_m, log_p, s);   // min(p, T): see fft_core.cuh
            for (int r = 1; r < R; ++r)
                for (int k = 0; k < cols; ++k) v.push_back(w_forward((int64_t)k * r, (int64_t)p * R));
        }
        if (v.empty()) v.push_back(make_float2(1.f, 0.f));
        add(key, v);
    }
    void add_split(int log_m) {
        Key key{KIND_SPLIT, log_m, 0};
        if (offset.count(key)) return;
        const int64_t M = int64_t(1) << log_m;
        std::vector<float2> v;
        for (int64_t k = 0; k <= M / 2; ++k) v.push_back(w_forward(k, 2 * M));
        add(key, v);
    }
    void add_pow2(int log_n, int lo) {
        Key key{KIND_POW2, log_n, lo};
        if (offset.count(key)) return;
        const int64_t N = int64_t(1) << log_n, nlo = int64_t(1) << lo;
        std::vector<float2> v;
        for (int64_t j = 0; j < nlo; ++j) v.push_back(w_forward(j, N));
        for (int64_t j = 0; j < N / nlo; ++j) v.push_back(w_forward(j * nlo, N));
        add(key, v);
    }
};

Registry &registry() {
    static Registry reg = [] {
        Registry r;
        // block FFTs of the resident path and the multi-pass sub-transforms
        for (int log_m = 2; log_m <= 14; ++log_m)
            for (int log_p = 2; log_p <= 5 && log_p <= log_m; ++log_p) r.add_stages(log_m, log_p);
        for (int log_m = 1; log_m <= 14; ++log_m) r.add_split(log_m);
        // multi-pass inter-pass twiddles, N = 2^15 .. 2^22 complex points
        for (int log_n = 15; log_n <= 22; ++log_n) r.add_pow2(log_n, log_n / 2);
        return r;
    }();
    return reg;
}

std::mutex g_mu;
float2 *g_dev_base[64] = {nullptr};

}  // namespace

hy_status tw_ensure_device() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error("cudaGetDevice", e);
    if (dev < 0 || dev >= 64) return set_error(HY_ERR_UNSUPPORTED, "device index %d >= 64", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_dev_base[dev]) return HY_OK;
    Registry &reg = registry();
    if ((int64_t)reg.host.size() > kCapacity)
        return set_error(HY_ERR_UNSUPPORTED, "twiddle tables (%zu) exceed capacity", reg.host.size());
    void *base = nullptr;
    e = cudaGetSymbolAddress(&base, g_tw);
    if (e != cudaSuccess) return set_cuda_error("cudaGetSymbolAddress(twiddles)", e);
    e = cudaMemcpy(base, reg.host.data(), reg.host.size() * sizeof(float2), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return set_cuda_error("cudaMemcpy(twiddles)", e);
    g_dev_base[dev] = (float2 *)base;
    return HY_OK;
}

static const float2 *lookup(int kind, int a, int b) {
    int dev = 0;
    cudaGetDevice(&dev);
    const Registry &reg = registry();
    auto it = reg.offset.find(Key{kind, a, b});
    if (it == reg.offset.end() || dev < 0 || dev >= 64 || !g_dev_base[dev]) return nullptr;
    return g_dev_base[dev] + it->second;
}

const float2 *tw_stages(int log_m, int log_p) { return lookup(KIND_STAGES, log_m, log_p); }
const float2 *tw_split(int log_m) { return lookup(KIND_SPLIT, log_m, 0); }
const float2 *tw_pow2(int log_n, int lo_bits) { return lookup(KIND_POW2, log_n, lo_bits); }

}  // namespace hy
