// C ABI of libmsa (declared in include/msa.h): argument checks, workspace layout and dispatch.
// Nothing here allocates, frees or synchronises device memory; every call enqueues on `stream`.
#include <math.h>
#include <string.h>

#include <atomic>

#include "msa.h"
#include "msa_common.cuh"
#include "msa_internal.h"

using namespace msa;

namespace {

constexpr size_t kStatusBytes = 256;

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

// Sizes shared by every entry point.
msa_status check_common(const msa_dims* d) {
    if (!d) return MSA_ERR_INVALID_ARG;
    if (d->B < 1 || d->N < 1 || d->H_q < 1 || d->H_kv < 1 || d->topk < 1) return MSA_ERR_INVALID_ARG;
    if (d->H_q % d->H_kv != 0) return MSA_ERR_INVALID_ARG;
    if (!(d->scale >= 0.f) || !(d->scale_idx >= 0.f)) return MSA_ERR_INVALID_ARG;
    const int G = d->H_q / d->H_kv;
    if (128 % G != 0 || G > 32 || 128 % d->H_kv != 0 || d->H_kv > 8) return MSA_ERR_UNSUPPORTED;
    if (d->d != 64 && d->d != 128) return MSA_ERR_UNSUPPORTED;
    if (d->d_idx != 32 && d->d_idx != 64) return MSA_ERR_UNSUPPORTED;
    if (d->block_k != 32 && d->block_k != 64 && d->block_k != 128) return MSA_ERR_UNSUPPORTED;
    if (d->topk > 16) return MSA_ERR_UNSUPPORTED;
    if (d->N >= (1 << 24)) return MSA_ERR_UNSUPPORTED;
    const double entries = (double)d->B * d->N * d->H_kv * (d->topk + 1);
    if (entries >= 2147483647.0 / 2) return MSA_ERR_UNSUPPORTED;
    return MSA_OK;
}

float eff_scale(float s, int dim) { return s > 0.f ? s : 1.0f / sqrtf((float)dim); }

size_t csr_need(const msa_dims* d) { return csr_bytes(d->B, d->N, d->H_kv, d->block_k, d->topk, 0); }

size_t rows_kv(const msa_dims* d) { return (size_t)d->B * d->N * d->H_kv; }

size_t ws_index_lse(const msa_dims* d) {
    return kStatusBytes + csr_need(d) + al256(rows_kv(d) * (d->topk + 1) * sizeof(float2));
}
// The prefill attention indexes its (query, head, slot) partial rows with 31 bits.
bool attn_rows_fit(const msa_dims* d) {
    return (double)d->B * d->N * d->H_q * (d->topk + 1) < 2147483647.0;
}
size_t ws_attn(const msa_dims* d) {
    return kStatusBytes + attn_ws_bytes(d->B, d->N, d->H_q, d->H_kv, d->d, d->block_k, d->topk);
}
size_t ws_decode(const msa_dims* d) {
    return kStatusBytes + decode_ws_bytes(d->B, d->N, d->H_q, d->H_kv, d->d, d->block_k, d->topk);
}
size_t ws_lse_local(const msa_dims* d) {
    return ws_index_lse(d) + al256(rows_kv(d) * (d->topk + 1) * 4);
}

size_t ws_bwd(const msa_dims* d) {
    return kStatusBytes + csr_need(d) + al256((size_t)d->B * d->N * d->H_q * 4);
}
size_t ws_kl(const msa_dims* d) {
    const size_t nb = (size_t)(d->N + d->block_k - 1) / d->block_k;
    const size_t nl = (size_t)d->B * d->H_kv * nb;
    const size_t me = rows_kv(d) * (d->topk + 1);
    const size_t csr_idx_extra = al256((nl + 1) * 4) + al256(me * 16) + 256;
    return kStatusBytes + csr_need(d) + csr_idx_extra + al256(me * sizeof(float2)) + al256(rows_kv(d) * 4) +
           al256(me * d->d_idx * 4) + al256(me * 8) + al256(rows_kv(d) * 8);
}

// Dense warm-up KL: teacher LSE, LSE_idx, the dense lists (shared entries, items of 128/G queries for
// the KL and of kIdxQpc for LSE_idx), per-(row, block) (max, sum-exp) of the index logits, KL rows.
struct DenseLayout {
    long long entries, items_kl, items_idx;
    size_t nb;
};
DenseLayout dense_layout(const msa_dims* d) {
    DenseLayout L;
    const int G = d->H_q / d->H_kv;
    dense_list_sizes(d->B, d->N, d->H_kv, d->block_k, 128 / G, &L.entries, &L.items_kl);
    long long e2 = 0;
    dense_list_sizes(d->B, d->N, d->H_kv, d->block_k, kIdxQpc, &e2, &L.items_idx);
    L.nb = (size_t)(d->N + d->block_k - 1) / d->block_k;
    return L;
}
size_t ws_kl_dense(const msa_dims* d) {
    const DenseLayout L = dense_layout(d);
    const size_t nl = (size_t)d->B * d->H_kv * L.nb;
    return kStatusBytes + al256((size_t)d->B * d->N * d->H_q * 4) + al256(rows_kv(d) * 4) +
           al256((size_t)L.entries * 4) + al256((size_t)L.items_kl * 16) + al256((size_t)L.items_idx * 16) + 256 +
           256 + al256(rows_kv(d) * L.nb * sizeof(float2)) + al256(rows_kv(d) * 8) + al256((nl + 1) * 4);
}
// The dense lists index entries and items with 31 bits.
bool dense_fits(const msa_dims* d) {
    const DenseLayout L = dense_layout(d);
    return L.entries < 2147483647LL && L.items_kl < 2147483647LL && rows_kv(d) * L.nb < (1ull << 40);
}

msa_status ws_check(const void* ws, size_t have, size_t need) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MSA_ERR_WORKSPACE;
    if (have < need) return MSA_ERR_WORKSPACE;
    return MSA_OK;
}

msa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

// Wait limit that the test hook msa_debug_set_wait_ns put in place (0: the default, nothing to do).
std::atomic<unsigned long long> g_wait_ns{0};

// Clears a call's status word on its stream; with the test hook set, also writes the shorter limit
// of the call's bounded waits.
cudaError_t status_init(DevStatus* status, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(status, 0, kStatusBytes, st);
    const unsigned long long w = g_wait_ns.load(std::memory_order_relaxed);
    if (e == cudaSuccess && w != 0) e = run_set_wait(status, w, st);
    return e;
}

struct Carver {
    uint8_t* p;
    uint8_t* take(size_t bytes) {
        uint8_t* r = p;
        p += al256(bytes);
        return r;
    }
};

}  // namespace

extern "C" {

const char* msa_version(void) { return "msa-b200 0.1.0"; }

const char* msa_status_string(msa_status s) {
    switch (s) {
        case MSA_OK: return "MSA_OK";
        case MSA_ERR_INVALID_ARG: return "MSA_ERR_INVALID_ARG";
        case MSA_ERR_UNSUPPORTED: return "MSA_ERR_UNSUPPORTED";
        case MSA_ERR_WORKSPACE: return "MSA_ERR_WORKSPACE";
        case MSA_ERR_CUDA: return "MSA_ERR_CUDA";
        case MSA_ERR_TIMEOUT: return "MSA_ERR_TIMEOUT";
        case MSA_ERR_DEVICE_CHECK: return "MSA_ERR_DEVICE_CHECK";
    }
    return "MSA_ERR_UNKNOWN";
}

msa_status msa_workspace_size(int op, const msa_dims* d, size_t* bytes) {
    if (!bytes) return MSA_ERR_INVALID_ARG;
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    switch (op) {
        case MSA_OP_INDEX_TOPK: *bytes = kStatusBytes; return MSA_OK;
        case MSA_OP_INDEX_TOPK_LSE: *bytes = ws_index_lse(d); return MSA_OK;
        case MSA_OP_ATTN_FWD:
            if (!attn_rows_fit(d)) return MSA_ERR_UNSUPPORTED;
            *bytes = ws_attn(d);
            return MSA_OK;
        case MSA_OP_DECODE: *bytes = ws_decode(d); return MSA_OK;
        case MSA_OP_KL: *bytes = ws_kl(d); return MSA_OK;
        case MSA_OP_LSE_IDX_LOCAL: *bytes = ws_lse_local(d); return MSA_OK;
        case MSA_OP_ATTN_BWD:
            if (!bwd_supported(d->d, d->H_q / d->H_kv)) return MSA_ERR_UNSUPPORTED;
            *bytes = ws_bwd(d);
            return MSA_OK;
        case MSA_OP_KL_DENSE:
            if (!kl_supported(d->d, d->d_idx, d->H_q / d->H_kv) ||
                !dense_lse_supported(d->d, d->block_k, d->H_q / d->H_kv) || !dense_fits(d))
                return MSA_ERR_UNSUPPORTED;
            *bytes = ws_kl_dense(d);
            return MSA_OK;
    }
    return MSA_ERR_INVALID_ARG;
}

msa_status msa_index_topk(const msa_dims* d, const void* q_idx, const void* k_idx, int32_t* blocks, float* lse_idx,
                          void* ws, size_t ws_bytes, msa_stream_t stream_) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if (!q_idx || !k_idx || !blocks || !aligned16(q_idx) || !aligned16(k_idx) || !aligned16(blocks) ||
        (lse_idx && !aligned16(lse_idx)))
        return MSA_ERR_INVALID_ARG;
    s = ws_check(ws, ws_bytes, lse_idx ? ws_index_lse(d) : kStatusBytes);
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    IndexArgs a{d->B, d->N, d->H_kv, d->d_idx, d->block_k, d->topk, blocks, status, 0, d->N, nullptr, nullptr};
    e = run_index_topk(a, q_idx, k_idx, num_sms(), st);
    if (e != cudaSuccess || !lse_idx) return cuda_status(e);
    // LSE_idx over the selected token sets: per-(query, selected block) sum-exps, merged
    Carver cv{static_cast<uint8_t*>(ws) + kStatusBytes};
    KlArgs k{};
    k.B = d->B; k.N = d->N; k.H_q = d->H_q; k.H_kv = d->H_kv; k.d = d->d; k.d_idx = d->d_idx;
    k.block_k = d->block_k; k.topk = d->topk;
    k.scale = eff_scale(d->scale, d->d); k.scale_idx = eff_scale(d->scale_idx, d->d_idx);
    csr_carve(&k.csr_idx, cv.take(csr_need(d)), d->B, d->N, d->H_kv, d->block_k, d->topk, 0);
    k.ml_part = reinterpret_cast<float2*>(cv.take(rows_kv(d) * (d->topk + 1) * sizeof(float2)));
    k.kv_tok0 = 0;
    k.kv_ntok = d->N;
    k.lse_idx = lse_idx;
    k.blocks = blocks;
    k.status = status;
    e = run_csr_build(k.csr_idx, blocks, d->B, d->N, d->H_kv, d->block_k, d->topk, kIdxQpc, status, st);
    if (e == cudaSuccess) e = run_lse_idx(k, q_idx, k_idx, num_sms(), st);
    return cuda_status(e);
}

static msa_status attn_fwd(const msa_dims* d, const void* q, const void* k, const void* v, const int32_t* blocks,
                           void* out, bool out_bf16, float* lse, void* ws, size_t ws_bytes, msa_stream_t stream_) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if (!attn_rows_fit(d)) return MSA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !blocks || !out || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(blocks) ||
        !aligned16(out) || (lse && !aligned16(lse)))
        return MSA_ERR_INVALID_ARG;
    s = ws_check(ws, ws_bytes, ws_attn(d));
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    AttnArgs a{};
    a.B = d->B; a.N = d->N; a.H_q = d->H_q; a.H_kv = d->H_kv; a.d = d->d; a.block_k = d->block_k;
    a.topk = d->topk; a.scale = eff_scale(d->scale, d->d);
    attn_carve(&a, static_cast<uint8_t*>(ws) + kStatusBytes);
    a.blocks = blocks;
    a.out = out_bf16 ? nullptr : static_cast<float*>(out);
    a.out_bf16 = out_bf16 ? static_cast<__nv_bfloat16*>(out) : nullptr;
    a.lse = lse;
    a.status = status;
    e = run_attn(a, q, k, v, num_sms(), st);
    return cuda_status(e);
}

msa_status msa_sparse_attn_fwd(const msa_dims* d, const void* q, const void* k, const void* v, const int32_t* blocks,
                               float* out, float* lse, void* ws, size_t ws_bytes, msa_stream_t stream) {
    return attn_fwd(d, q, k, v, blocks, out, false, lse, ws, ws_bytes, stream);
}

msa_status msa_sparse_attn_fwd_bf16(const msa_dims* d, const void* q, const void* k, const void* v,
                                    const int32_t* blocks, void* out, float* lse, void* ws, size_t ws_bytes,
                                    msa_stream_t stream) {
    return attn_fwd(d, q, k, v, blocks, out, true, lse, ws, ws_bytes, stream);
}

// The decode step with a bf16 K_idx cache (k_idx_scale null) or an e4m3 one (codes + scales).
static msa_status decode_step(const msa_dims* d, const int32_t* cache_len, const void* q, const void* q_idx,
                              const void* k_cache, const void* v_cache, const void* k_idx, const float* k_idx_scale,
                              float* out, int32_t* blocks_out, float* margin_out, void* ws, size_t ws_bytes,
                              msa_stream_t stream_) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if ((d->N + d->block_k - 1) / d->block_k > 8192) return MSA_ERR_UNSUPPORTED;
    if (!cache_len || !q || !q_idx || !k_cache || !v_cache || !k_idx || !out || !aligned16(q) ||
        !aligned16(q_idx) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(k_idx) ||
        !aligned16(out) || (blocks_out && !aligned16(blocks_out)) || (margin_out && !aligned16(margin_out)) ||
        (k_idx_scale && !aligned16(k_idx_scale)))
        return MSA_ERR_INVALID_ARG;
    s = ws_check(ws, ws_bytes, ws_decode(d));
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    Carver cv{static_cast<uint8_t*>(ws) + kStatusBytes};
    const size_t nb = (size_t)(d->N + d->block_k - 1) / d->block_k;
    const size_t G = (size_t)d->H_q / d->H_kv, K1 = (size_t)d->topk + 1;
    DecodeArgs a{};
    a.B = d->B; a.L = d->N; a.H_q = d->H_q; a.H_kv = d->H_kv; a.d = d->d; a.d_idx = d->d_idx;
    a.block_k = d->block_k; a.topk = d->topk;
    a.scale = eff_scale(d->scale, d->d); a.scale_idx = eff_scale(d->scale_idx, d->d_idx);
    a.cache_len = cache_len;
    a.bmax = reinterpret_cast<float*>(cv.take((size_t)d->B * d->H_kv * nb * 4));
    a.sel = reinterpret_cast<int32_t*>(cv.take((size_t)d->B * d->H_kv * K1 * 4));
    a.o_part = reinterpret_cast<float*>(cv.take((size_t)d->B * d->H_kv * K1 * G * d->d * 4));
    a.lse_part = reinterpret_cast<float*>(cv.take((size_t)d->B * d->H_kv * K1 * G * 4));
    a.blocks_out = blocks_out;
    a.margin_out = margin_out;
    a.k_idx_scale = k_idx_scale;
    a.status = status;
    e = run_decode(a, q, q_idx, k_cache, v_cache, k_idx, out, num_sms(), st);
    return cuda_status(e);
}

msa_status msa_sparse_attn_decode(const msa_dims* d, const int32_t* cache_len, const void* q, const void* q_idx,
                                  const void* k_cache, const void* v_cache, const void* k_idx_cache, float* out,
                                  int32_t* blocks_out, float* margin_out, void* ws, size_t ws_bytes,
                                  msa_stream_t stream) {
    return decode_step(d, cache_len, q, q_idx, k_cache, v_cache, k_idx_cache, nullptr, out, blocks_out, margin_out,
                       ws, ws_bytes, stream);
}

msa_status msa_sparse_attn_decode_fp8idx(const msa_dims* d, const int32_t* cache_len, const void* q,
                                         const void* q_idx, const void* k_cache, const void* v_cache,
                                         const uint8_t* k_idx_codes, const float* k_idx_scale, float* out,
                                         int32_t* blocks_out, float* margin_out, void* ws, size_t ws_bytes,
                                         msa_stream_t stream) {
    if (!k_idx_scale) return MSA_ERR_INVALID_ARG;
    return decode_step(d, cache_len, q, q_idx, k_cache, v_cache, k_idx_codes, k_idx_scale, out, blocks_out,
                       margin_out, ws, ws_bytes, stream);
}

msa_status msa_quantize_e4m3_rows(const void* x, int64_t rows, int n, uint8_t* codes, float* scale,
                                  msa_stream_t stream) {
    if (rows < 0 || (rows > 0 && (!x || !codes || !scale || !aligned16(x) || !aligned16(codes) || !aligned16(scale))))
        return MSA_ERR_INVALID_ARG;
    if (n != 16 && n != 32 && n != 64 && n != 128 && n != 256) return MSA_ERR_UNSUPPORTED;
    if (rows > ((int64_t)1 << 40) / n) return MSA_ERR_UNSUPPORTED;
    return cuda_status(run_quantize_e4m3_rows(x, rows, n, codes, scale, num_sms(),
                                              reinterpret_cast<cudaStream_t>(stream)));
}

static bool sp_range_ok(const msa_dims* d, int tok0, int ntok) {
    return tok0 >= 0 && ntok > 0 && tok0 % d->block_k == 0 && (long long)tok0 + ntok <= d->N &&
           (ntok % d->block_k == 0 || tok0 + ntok == d->N);
}

// one or two ranges of whole blocks, the second after the first
static bool sp_held_ok(const msa_dims* d, const msa_key_ranges* h) {
    if (!h || h->n < 1 || h->n > 2 || !sp_range_ok(d, h->tok0[0], h->ntok[0])) return false;
    return h->n == 1 || (sp_range_ok(d, h->tok0[1], h->ntok[1]) && h->tok0[1] >= h->tok0[0] + h->ntok[0]);
}

msa_status msa_index_topk_local(const msa_dims* d, const void* q_idx, const void* k_idx_local,
                                const msa_key_ranges* held, float* cand_scores, int32_t* cand_ids, void* ws,
                                size_t ws_bytes, msa_stream_t stream_) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if (!q_idx || !k_idx_local || !cand_scores || !cand_ids || !aligned16(q_idx) || !aligned16(k_idx_local) ||
        !aligned16(cand_scores) || !aligned16(cand_ids) || !sp_held_ok(d, held))
        return MSA_ERR_INVALID_ARG;
    s = ws_check(ws, ws_bytes, kStatusBytes);
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    IndexArgs a{d->B, d->N, d->H_kv, d->d_idx, d->block_k, d->topk, nullptr, status, held->tok0[0], held->ntok[0],
                cand_scores, cand_ids, held->n == 2 ? held->tok0[1] : 0, held->n == 2 ? held->ntok[1] : 0};
    return cuda_status(run_index_topk(a, q_idx, k_idx_local, num_sms(), st));
}

msa_status msa_topk_merge(const msa_dims* d, int P, const float* cand_scores, const int32_t* cand_ids,
                          int32_t* blocks, msa_stream_t stream) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if (P < 1 || P > 8) return MSA_ERR_UNSUPPORTED;
    if (!cand_scores || !cand_ids || !blocks || !aligned16(cand_scores) || !aligned16(cand_ids) || !aligned16(blocks))
        return MSA_ERR_INVALID_ARG;
    return cuda_status(run_topk_merge(d->B, d->N, d->H_kv, d->block_k, d->topk, P, cand_scores, cand_ids, blocks,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

msa_status msa_lse_idx_local(const msa_dims* d, const void* q_idx, const void* k_idx_local, const msa_key_ranges* held,
                             const int32_t* blocks, float* ml, void* ws, size_t ws_bytes, msa_stream_t stream_) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if (!q_idx || !k_idx_local || !blocks || !ml || !aligned16(q_idx) || !aligned16(k_idx_local) ||
        !aligned16(blocks) || !aligned16(ml) || !sp_held_ok(d, held))
        return MSA_ERR_INVALID_ARG;
    s = ws_check(ws, ws_bytes, ws_lse_local(d));
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    Carver cv{static_cast<uint8_t*>(ws) + kStatusBytes};
    KlArgs k{};
    k.B = d->B; k.N = d->N; k.H_q = d->H_q; k.H_kv = d->H_kv; k.d = d->d; k.d_idx = d->d_idx;
    k.block_k = d->block_k; k.topk = d->topk;
    k.scale = eff_scale(d->scale, d->d); k.scale_idx = eff_scale(d->scale_idx, d->d_idx);
    csr_carve(&k.csr_idx, cv.take(csr_need(d)), d->B, d->N, d->H_kv, d->block_k, d->topk, 0);
    k.ml_part = reinterpret_cast<float2*>(cv.take(rows_kv(d) * (d->topk + 1) * sizeof(float2)));
    int32_t* mine = reinterpret_cast<int32_t*>(cv.take(rows_kv(d) * (d->topk + 1) * 4));  // the held selected blocks
    k.blocks = mine;
    k.status = status;
    k.kv_tok0 = held->tok0[0];
    k.kv_ntok = held->ntok[0];
    k.kv_tok0b = held->n == 2 ? held->tok0[1] : 0;
    k.kv_ntokb = held->n == 2 ? held->ntok[1] : 0;
    k.ml_out = reinterpret_cast<float2*>(ml);
    // first block of each range and the block past it (a range that ends at N may end inside a block)
    const int bk = d->block_k;
    const int blk0 = k.kv_tok0 / bk, blk1 = (k.kv_tok0 + k.kv_ntok + bk - 1) / bk;
    const int blk2 = k.kv_tok0b / bk, blk3 = (k.kv_tok0b + k.kv_ntokb + bk - 1) / bk;
    e = run_blocks_in_range((long long)rows_kv(d), d->topk + 1, blk0, blk1, blk2, blk3, blocks, mine, st);
    if (e == cudaSuccess)
        e = run_csr_build(k.csr_idx, mine, d->B, d->N, d->H_kv, d->block_k, d->topk, kIdxQpc, status, st);
    if (e == cudaSuccess) e = run_lse_idx(k, q_idx, k_idx_local, num_sms(), st);
    return cuda_status(e);
}

msa_status msa_lse_combine(const msa_dims* d, int P, const float* ml, float* lse_idx, msa_stream_t stream) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if (P < 1) return MSA_ERR_INVALID_ARG;
    if (!ml || !lse_idx || !aligned16(ml) || !aligned16(lse_idx)) return MSA_ERR_INVALID_ARG;
    return cuda_status(run_lse_combine(P, (long long)d->B * d->N * d->H_kv, reinterpret_cast<const float2*>(ml),
                                       lse_idx, reinterpret_cast<cudaStream_t>(stream)));
}

msa_status msa_sparse_attn_bwd(const msa_dims* d, const void* q, const void* k, const void* v, const int32_t* blocks,
                               const float* out, const float* lse, const void* dout, float* dq, float* dk, float* dv,
                               void* ws, size_t ws_bytes, msa_stream_t stream_) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if (!bwd_supported(d->d, d->H_q / d->H_kv)) return MSA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !blocks || !out || !lse || !dout || !dq || !dk || !dv || !aligned16(q) || !aligned16(k) ||
        !aligned16(v) || !aligned16(blocks) || !aligned16(out) || !aligned16(lse) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return MSA_ERR_INVALID_ARG;
    s = ws_check(ws, ws_bytes, ws_bwd(d));
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    Carver cv{static_cast<uint8_t*>(ws) + kStatusBytes};
    BwdArgs a{};
    a.B = d->B; a.N = d->N; a.H_q = d->H_q; a.H_kv = d->H_kv; a.d = d->d; a.block_k = d->block_k;
    a.topk = d->topk; a.scale = eff_scale(d->scale, d->d);
    csr_carve(&a.csr, cv.take(csr_need(d)), d->B, d->N, d->H_kv, d->block_k, d->topk, 0);
    a.delta = reinterpret_cast<float*>(cv.take((size_t)d->B * d->N * d->H_q * 4));
    a.lse = lse;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.status = status;
    const int G = d->H_q / d->H_kv;
    e = run_csr_build(a.csr, blocks, d->B, d->N, d->H_kv, d->block_k, d->topk, 128 / G, status, st);
    if (e == cudaSuccess) e = run_attn_bwd(a, q, k, v, dout, out, num_sms(), st);
    return cuda_status(e);
}

msa_status msa_kl_fwd_grad(const msa_dims* d, const void* q, const void* k, const void* q_idx, const void* k_idx,
                           const int32_t* blocks, const float* lse, const float* lse_idx, float grad_scale,
                           float* loss, float* dq_idx, float* dk_idx, void* ws, size_t ws_bytes,
                           msa_stream_t stream_) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    if (!kl_supported(d->d, d->d_idx, d->H_q / d->H_kv)) return MSA_ERR_UNSUPPORTED;
    if (!q || !k || !q_idx || !k_idx || !blocks || !lse || !loss || !dq_idx || !dk_idx || !aligned16(q) ||
        !aligned16(k) || !aligned16(q_idx) || !aligned16(k_idx) || !aligned16(blocks) || !aligned16(dq_idx) ||
        !aligned16(dk_idx))
        return MSA_ERR_INVALID_ARG;
    if (!isfinite(grad_scale)) return MSA_ERR_INVALID_ARG;
    s = ws_check(ws, ws_bytes, ws_kl(d));
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    Carver cv{static_cast<uint8_t*>(ws) + kStatusBytes};
    const size_t nb = (size_t)(d->N + d->block_k - 1) / d->block_k;
    const size_t nl = (size_t)d->B * d->H_kv * nb;
    const size_t me = rows_kv(d) * (d->topk + 1);
    KlArgs a{};
    a.B = d->B; a.N = d->N; a.H_q = d->H_q; a.H_kv = d->H_kv; a.d = d->d; a.d_idx = d->d_idx;
    a.block_k = d->block_k; a.topk = d->topk;
    a.scale = eff_scale(d->scale, d->d); a.scale_idx = eff_scale(d->scale_idx, d->d_idx);
    a.grad_scale = grad_scale;
    a.kv_tok0 = 0;
    a.kv_ntok = d->N;
    csr_carve(&a.csr, cv.take(csr_need(d)), d->B, d->N, d->H_kv, d->block_k, d->topk, 0);
    a.csr_idx = a.csr;  // same lists, its own chunking
    a.csr_idx.chunk_off = reinterpret_cast<int32_t*>(cv.take((nl + 1) * 4));
    a.csr_idx.items = reinterpret_cast<int4*>(cv.take(me * 16));
    a.csr_idx.n_items = reinterpret_cast<int32_t*>(cv.take(256));
    a.ml_part = reinterpret_cast<float2*>(cv.take(me * sizeof(float2)));
    float* lse_idx_ws = reinterpret_cast<float*>(cv.take(rows_kv(d) * 4));
    a.dq_part = reinterpret_cast<float*>(cv.take(me * d->d_idx * 4));
    a.kl_part = reinterpret_cast<double*>(cv.take(me * 8));
    a.kl_rows = reinterpret_cast<double*>(cv.take(rows_kv(d) * 8));
    a.lse = lse;
    a.dq_idx = dq_idx;
    a.dk_idx = dk_idx;
    a.loss = loss;
    a.blocks = blocks;
    a.status = status;
    const int G = d->H_q / d->H_kv;
    e = run_csr_build(a.csr, blocks, d->B, d->N, d->H_kv, d->block_k, d->topk, 128 / G, status, st);
    if (e == cudaSuccess && !lse_idx) {
        a.lse_idx = lse_idx_ws;
        e = run_csr_items(a.csr_idx, kIdxQpc, st);
        if (e == cudaSuccess) e = run_lse_idx(a, q_idx, k_idx, num_sms(), st);
    } else {
        a.lse_idx = const_cast<float*>(lse_idx);
    }
    if (e == cudaSuccess) e = run_kl(a, q, k, q_idx, k_idx, num_sms(), st);
    return cuda_status(e);
}

msa_status msa_kl_dense_fwd_grad(const msa_dims* d, const void* q, const void* k, const void* q_idx,
                                 const void* k_idx, float grad_scale, float* loss, float* dq_idx, float* dk_idx,
                                 float* lse_out, void* ws, size_t ws_bytes, msa_stream_t stream_) {
    msa_status s = check_common(d);
    if (s != MSA_OK) return s;
    const int G = d->H_q / d->H_kv;
    if (!kl_supported(d->d, d->d_idx, G) || !dense_lse_supported(d->d, d->block_k, G) || !dense_fits(d))
        return MSA_ERR_UNSUPPORTED;
    if (!q || !k || !q_idx || !k_idx || !loss || !dq_idx || !dk_idx || !aligned16(q) || !aligned16(k) ||
        !aligned16(q_idx) || !aligned16(k_idx) || !aligned16(dq_idx) || !aligned16(dk_idx) ||
        (lse_out && !aligned16(lse_out)))
        return MSA_ERR_INVALID_ARG;
    if (!isfinite(grad_scale)) return MSA_ERR_INVALID_ARG;
    s = ws_check(ws, ws_bytes, ws_kl_dense(d));
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    const DenseLayout L = dense_layout(d);
    const size_t nl = (size_t)d->B * d->H_kv * L.nb;
    Carver cv{static_cast<uint8_t*>(ws) + kStatusBytes};
    float* lse_ws = reinterpret_cast<float*>(cv.take((size_t)d->B * d->N * d->H_q * 4));
    float* lse_main = lse_out ? lse_out : lse_ws;
    float* lse_idx = reinterpret_cast<float*>(cv.take(rows_kv(d) * 4));
    KlArgs a{};
    a.B = d->B; a.N = d->N; a.H_q = d->H_q; a.H_kv = d->H_kv; a.d = d->d; a.d_idx = d->d_idx;
    a.block_k = d->block_k; a.topk = d->topk;
    a.scale = eff_scale(d->scale, d->d); a.scale_idx = eff_scale(d->scale_idx, d->d_idx);
    a.grad_scale = grad_scale;
    a.kv_tok0 = 0;
    a.kv_ntok = d->N;
    a.dense = 1;
    // lists: one window per sequence (nW = 1), list (b, r, c) = queries c*block_k .. N-1
    a.csr.nb = (int)L.nb;
    a.csr.nW = 1;
    a.csr.wq = d->N;
    a.csr.nlists = (int)nl;
    a.csr.entries = reinterpret_cast<int32_t*>(cv.take((size_t)L.entries * 4));
    a.csr.items = reinterpret_cast<int4*>(cv.take((size_t)L.items_kl * 16));
    a.csr_idx = a.csr;
    a.csr_idx.items = reinterpret_cast<int4*>(cv.take((size_t)L.items_idx * 16));
    a.csr.n_items = reinterpret_cast<int32_t*>(cv.take(256));
    a.csr_idx.n_items = reinterpret_cast<int32_t*>(cv.take(256));
    a.ml_part = reinterpret_cast<float2*>(cv.take(rows_kv(d) * L.nb * sizeof(float2)));
    a.kl_rows = reinterpret_cast<double*>(cv.take(rows_kv(d) * 8));
    a.lse = lse_main;
    a.lse_idx = lse_idx;
    a.dq_idx = dq_idx;
    a.dk_idx = dk_idx;
    a.loss = loss;
    a.blocks = nullptr;
    a.status = status;
    DenseLseArgs dl{d->B, d->N, d->H_q, d->H_kv, G, d->d, d->block_k, a.scale, lse_main, status};
    e = run_dense_lse(dl, q, k, num_sms(), st);
    if (e == cudaSuccess) e = run_dense_lists(a.csr, d->B, d->N, d->H_kv, d->block_k, 128 / G, true, st);
    if (e == cudaSuccess) e = run_dense_lists(a.csr_idx, d->B, d->N, d->H_kv, d->block_k, kIdxQpc, false, st);
    if (e == cudaSuccess) e = run_lse_idx(a, q_idx, k_idx, num_sms(), st);
    if (e == cudaSuccess) e = run_kl(a, q, k, q_idx, k_idx, num_sms(), st);
    return cuda_status(e);
}

void msa_debug_set_wait_ns(unsigned long long ns) { g_wait_ns.store(ns, std::memory_order_relaxed); }

msa_status msa_debug_wait_probe(void* ws, size_t ws_bytes, msa_stream_t stream_) {
    msa_status s = ws_check(ws, ws_bytes, kStatusBytes + wait_probe_bytes());
    if (s != MSA_OK) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    DevStatus* status = static_cast<DevStatus*>(ws);
    cudaError_t e = status_init(status, st);
    if (e == cudaSuccess) e = run_wait_probe(static_cast<uint8_t*>(ws) + kStatusBytes, status, st);
    return cuda_status(e);
}

msa_status msa_debug_exp2_fma(const float* x, float* y, int64_t n, msa_stream_t stream_) {
    if (n < 0 || (n > 0 && (!x || !y))) return MSA_ERR_INVALID_ARG;
    return cuda_status(run_exp2_fma(x, y, n, num_sms(), reinterpret_cast<cudaStream_t>(stream_)));
}

msa_status msa_get_device_status(const void* ws, msa_stream_t stream_) {
    if (!ws) return MSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream_);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MSA_ERR_CUDA;
    DevStatus h;
    if (cudaMemcpy(&h, ws, sizeof(unsigned int) * 2, cudaMemcpyDeviceToHost) != cudaSuccess) return MSA_ERR_CUDA;
    if (h.flags & MSA_DEV_TIMEOUT) return MSA_ERR_TIMEOUT;
    if (h.flags & MSA_DEV_BAD_BLOCK) return MSA_ERR_DEVICE_CHECK;
    return MSA_OK;
}

}  // extern "C"
