// Decode step without a caller-provided workspace, for callers that cannot allocate device memory.
//
// Some callers of the decode step have no way to obtain device memory at the point where they
// decode: a plugin running inside a host application that owns every device allocation, a
// serving loop whose memory budget is fixed at start-up, or a latency-bound path that must not
// call cudaMalloc (which can synchronise the device). This entry point uses a file-scope static
// device array as the decode scratch instead of a workspace argument. The array has a fixed size
// (MSA_DECODE_STATIC_SCRATCH_BYTES); every GPU that loads this library holds it until the process
// exits. The caller still passes all inputs and outputs.
//
// The array's name in host code is only a host-side stand-in, never a device address, so the host
// side asks the runtime for the real device address once per device (cudaGetSymbolAddress, with
// that device current) and hands that to the existing decode path. All calls on a device share
// the one array: the decode path clears what must start at zero (its status word) and overwrites
// the rest, but two calls that overlap on the GPU (different streams, no ordering) race on it.
#include <mutex>

#include "msa.h"
#include "msa_internal.h"

namespace {

__device__ __align__(256) unsigned char g_decode_scratch[MSA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device (looked up on first use).
msa_status scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) return MSA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MSA_OK;
}

}  // namespace

// Status word of the last call on the current device: the first bytes of the static array.
extern "C" msa_status msa_decode_noalloc_status(msa_stream_t stream) {
    void* scratch = nullptr;
    msa_status s = scratch_address(&scratch);
    if (s != MSA_OK) return s;
    return msa_get_device_status(scratch, stream);
}

extern "C" msa_status msa_sparse_attn_decode_noalloc(const msa_dims* dims, const int32_t* cache_len, const void* q,
                                                      const void* q_idx, const void* k_cache, const void* v_cache,
                                                      const void* k_idx_cache, float* out, int32_t* blocks_out,
                                                      msa_stream_t stream) {
    size_t need = 0;
    msa_status s = msa_workspace_size(MSA_OP_DECODE, dims, &need);
    if (s != MSA_OK) return s;
    if (need > (size_t)MSA_DECODE_STATIC_SCRATCH_BYTES) return MSA_ERR_WORKSPACE;
    void* scratch = nullptr;
    s = scratch_address(&scratch);
    if (s != MSA_OK) return s;
    return msa_sparse_attn_decode(dims, cache_len, q, q_idx, k_cache, v_cache, k_idx_cache, out, blocks_out, nullptr, scratch,
                                  (size_t)MSA_DECODE_STATIC_SCRATCH_BYTES, stream);
}
