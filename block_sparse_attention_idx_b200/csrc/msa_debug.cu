// Test hooks of the failure-detection path: a shorter limit for the bounded waits of later calls,
// and a launch whose wait can never be satisfied.
//
// Every wait in this library is bounded: when it runs out, the kernel sets MSA_DEV_TIMEOUT in the
// call's status word, drains the copies and MMAs it issued, frees its TMEM and returns, so the
// context stays usable. The probe below exercises that path on purpose without any fault: a
// consumer waits on an mbarrier whose producer skips its arrival, while a real bulk copy is in
// flight and TMEM is held. Nothing here traps, asserts or touches memory outside its buffers.
#include <algorithm>

#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

// Writes a call's wait limit into its (already cleared) status word.
__global__ void k_set_wait(DevStatus* st, unsigned long long ns) { st->wait_ns = ns; }

constexpr int kProbeBytes = 4096;
constexpr int kProbeCols = 32;

// Warp 0 owns 32 TMEM columns; warp 1 (producer) issues one bulk copy of kProbeBytes from `src`
// into shared memory on barrier `full` and never arrives on `ready`; warp 2 (consumer) waits on
// `ready`, which can only run out. Then the producer waits (bounded) for its copy to land, and
// warp 0 frees the TMEM after a CTA barrier.
__global__ void __launch_bounds__(96, 1) k_wait_probe(const uint8_t* __restrict__ src, DevStatus* st) {
    __shared__ alignas(128) uint8_t buf[kProbeBytes];
    __shared__ uint64_t full, ready;
    __shared__ uint32_t tmem_base;
    const int warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        mbar_init(&full, 1);
        mbar_init(&ready, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base, kProbeCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1 && lane == 0) {
        mbar_arrive_expect_tx(&full, kProbeBytes);
        bulk_load(buf, src, kProbeBytes, &full);
        // the arrival on `ready` is deliberately left out
        mbar_wait(&full, 0, st, 0xF02);  // drain: the copy lands before the CTA leaves
    } else if (warp == 2 && lane == 0) {
        mbar_wait(&ready, 0, st, 0xF01);  // runs out: raises MSA_DEV_TIMEOUT
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem_base, kProbeCols);
}

}  // namespace

cudaError_t run_set_wait(DevStatus* st, unsigned long long ns, cudaStream_t s) {
    k_set_wait<<<1, 1, 0, s>>>(st, ns);
    return cudaGetLastError();
}

size_t wait_probe_bytes() { return kProbeBytes; }

namespace {
// y[i] = 2^x[i] by the FMA-pipe exponential the MUFU-bound loops use (pairs; a lone last value is
// paired with 0).
__global__ void k_exp2_fma(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
    for (int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x); i < n; i += 2 * (int64_t)gridDim.x * blockDim.x) {
        const bool two = i + 1 < n;
        float lo, hi;
        f2_unpack(exp2_fma_x2(f2_packf(x[i], two ? x[i + 1] : 0.f)), lo, hi);
        y[i] = lo;
        if (two) y[i + 1] = hi;
    }
}
}  // namespace

cudaError_t run_exp2_fma(const float* x, float* y, int64_t n, int num_sms, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    const int64_t threads = (n + 1) / 2;
    const int grid = (int)std::min<int64_t>((threads + 255) / 256, (int64_t)num_sms * 8);
    k_exp2_fma<<<grid, 256, 0, s>>>(x, y, n);
    return cudaGetLastError();
}

cudaError_t run_wait_probe(const void* src, DevStatus* st, cudaStream_t s) {
    k_wait_probe<<<1, 96, 0, s>>>(static_cast<const uint8_t*>(src), st);
    return cudaGetLastError();
}

}  // namespace msa
