// Opt-in per-kernel timing with CUDA events recorded on the launching stream (see msa.h).
#include <mutex>
#include <string.h>

#include "msa.h"
#include "msa_internal.h"

namespace msa {

namespace {
constexpr int kMaxRec = 4096;
struct Rec {
    const char* name;
    cudaEvent_t a, b;
};
std::mutex g_mu;
bool g_on = false;
Rec g_rec[kMaxRec];
int g_n = 0;
cudaEvent_t g_pool[2 * kMaxRec];
int g_pool_n = 0;
bool g_pool_ok = false;

bool ensure_pool() {
    if (g_pool_ok) return true;
    for (; g_pool_n < 2 * kMaxRec; ++g_pool_n)
        if (cudaEventCreate(&g_pool[g_pool_n]) != cudaSuccess) return false;
    g_pool_ok = true;
    return true;
}
}  // namespace

int prof_begin(const char* name, cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_on || g_n >= kMaxRec || !ensure_pool()) return -1;
    const int x = g_n++;
    g_rec[x].name = name;
    g_rec[x].a = g_pool[2 * x];
    g_rec[x].b = g_pool[2 * x + 1];
    cudaEventRecord(g_rec[x].a, st);
    return x;
}

void prof_end(int x, cudaStream_t st) {
    if (x < 0) return;
    std::lock_guard<std::mutex> lk(g_mu);
    cudaEventRecord(g_rec[x].b, st);
}

}  // namespace msa

extern "C" {

void msa_profile_enable(int on) {
    std::lock_guard<std::mutex> lk(msa::g_mu);
    msa::g_on = on != 0;
}

int msa_profile_read(const char** names, double* total_ms, int* launches, int cap) {
    std::lock_guard<std::mutex> lk(msa::g_mu);
    int nout = 0;
    for (int x = 0; x < msa::g_n; ++x) {
        if (cudaEventSynchronize(msa::g_rec[x].b) != cudaSuccess) { msa::g_n = 0; return -1; }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, msa::g_rec[x].a, msa::g_rec[x].b) != cudaSuccess) { msa::g_n = 0; return -1; }
        int k = 0;
        while (k < nout && strcmp(names[k], msa::g_rec[x].name) != 0) ++k;
        if (k == nout) {
            if (nout >= cap) continue;
            names[k] = msa::g_rec[x].name;
            total_ms[k] = 0.0;
            launches[k] = 0;
            ++nout;
        }
        total_ms[k] += ms;
        launches[k] += 1;
    }
    msa::g_n = 0;
    return nout;
}

}  // extern "C"
