// Inverse selection lists for the KV-outer kernels (MSA blog, KV-outer sparse attention: organise
// the work around the selected KV blocks and gather the queries that need each block).
//
// From blocks[b,i,r,:] we build, for every (b, r, block c), the list of (query i, slot s) pairs
// that selected c, then cut every list into work items of at most `qpc` queries. Items are
// ordered by (b, r, c), so consecutive items share their K/V block; every item costs about the
// same, which is what keeps hot blocks (block 0, needle blocks, local blocks) from becoming
// stragglers: a block chosen by 20 000 queries simply yields 20 000/qpc items.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t csr_bytes(int B, int N, int H_kv, int block_k, int topk) {
    const size_t nb = (size_t)(N + block_k - 1) / block_k;
    const size_t nl = (size_t)B * H_kv * nb;
    const size_t me = (size_t)B * N * H_kv * (topk + 1);
    return align256(nl * 4) * 2 + align256((nl + 1) * 4) * 2 + align256(me * 4) + align256(me * 8) + 256;
}

void csr_carve(Csr* c, void* base, int B, int N, int H_kv, int block_k, int topk) {
    uint8_t* p = static_cast<uint8_t*>(base);
    c->nb = (N + block_k - 1) / block_k;
    c->nlists = B * H_kv * c->nb;
    c->max_entries = B * N * H_kv * (topk + 1);
    auto take = [&](size_t bytes) {
        uint8_t* r = p;
        p += align256(bytes);
        return r;
    };
    c->counts = reinterpret_cast<int32_t*>(take((size_t)c->nlists * 4));
    c->cursor = reinterpret_cast<int32_t*>(take((size_t)c->nlists * 4));
    c->offsets = reinterpret_cast<int32_t*>(take(((size_t)c->nlists + 1) * 4));
    c->chunk_off = reinterpret_cast<int32_t*>(take(((size_t)c->nlists + 1) * 4));
    c->entries = reinterpret_cast<int32_t*>(take((size_t)c->max_entries * 4));
    c->items = reinterpret_cast<int2*>(take((size_t)c->max_entries * 8));
    c->n_items = reinterpret_cast<int32_t*>(take(256));
}

namespace {

// One thread per selection row: validate it (ids in [0, i/block_k], strictly ascending among the
// non-negative entries) and count its entries. Invalid entries are skipped and flagged.
__global__ void k_csr_count(const int32_t* __restrict__ blocks, int B, int N, int H_kv, int block_k, int K1, int nb,
                            int32_t* counts, DevStatus* st) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= (long long)B * N * H_kv) return;
    const int r = (int)(row % H_kv);
    const int i = (int)((row / H_kv) % N);
    const int b = (int)(row / ((long long)H_kv * N));
    const int bi = i / block_k;
    const int32_t* sel = blocks + row * K1;
    int prev = -1;
    for (int s = 0; s < K1; ++s) {
        const int c = sel[s];
        if (c < 0) continue;
        if (c > bi || c <= prev) {
            raise_flag(st, MSA_DEV_BAD_BLOCK, 0x401);
            continue;
        }
        prev = c;
        atomicAdd(&counts[((size_t)b * H_kv + r) * nb + c], 1);
    }
}

// Single CTA: exclusive scans of the list sizes (entry offsets) and of their chunk counts.
__global__ void k_csr_scan(const int32_t* __restrict__ counts, int nlists, int qpc, int32_t* offsets,
                           int32_t* chunk_off, int32_t* n_items) {
    __shared__ int s_e[1024], s_c[1024];
    __shared__ int carry_e, carry_c;
    if (threadIdx.x == 0) { carry_e = 0; carry_c = 0; }
    __syncthreads();
    for (int base = 0; base < nlists; base += 1024) {
        const int x = base + threadIdx.x;
        const int n = x < nlists ? counts[x] : 0;
        s_e[threadIdx.x] = n;
        s_c[threadIdx.x] = (n + qpc - 1) / qpc;
        __syncthreads();
        for (int off = 1; off < 1024; off <<= 1) {  // Hillis-Steele inclusive scan
            const int ve = threadIdx.x >= off ? s_e[threadIdx.x - off] : 0;
            const int vc = threadIdx.x >= off ? s_c[threadIdx.x - off] : 0;
            __syncthreads();
            s_e[threadIdx.x] += ve;
            s_c[threadIdx.x] += vc;
            __syncthreads();
        }
        if (x < nlists) {
            offsets[x] = carry_e + s_e[threadIdx.x] - n;
            chunk_off[x] = carry_c + s_c[threadIdx.x] - (n + qpc - 1) / qpc;
        }
        __syncthreads();
        if (threadIdx.x == 1023) { carry_e += s_e[1023]; carry_c += s_c[1023]; }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        offsets[nlists] = carry_e;
        chunk_off[nlists] = carry_c;
        *n_items = carry_c;
    }
}

// One thread per selection row: place each valid entry (i << 5 | slot) into its list.
__global__ void k_csr_fill(const int32_t* __restrict__ blocks, int B, int N, int H_kv, int block_k, int K1, int nb,
                           const int32_t* __restrict__ offsets, int32_t* cursor, int32_t* entries) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= (long long)B * N * H_kv) return;
    const int r = (int)(row % H_kv);
    const int i = (int)((row / H_kv) % N);
    const int b = (int)(row / ((long long)H_kv * N));
    const int bi = i / block_k;
    const int32_t* sel = blocks + row * K1;
    int prev = -1;
    for (int s = 0; s < K1; ++s) {
        const int c = sel[s];
        if (c < 0 || c > bi || c <= prev) continue;
        prev = c;
        const size_t L = ((size_t)b * H_kv + r) * nb + c;
        const int pos = offsets[L] + atomicAdd(&cursor[L], 1);
        entries[pos] = (i << 5) | s;
    }
}

// One warp per list: write its work items (list id, first entry of the chunk).
__global__ void k_csr_items(const int32_t* __restrict__ counts, const int32_t* __restrict__ chunk_off, int nlists,
                            int qpc, int2* items) {
    const int L = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (L >= nlists) return;
    const int n = counts[L];
    const int nch = (n + qpc - 1) / qpc;
    const int o = chunk_off[L];
    for (int ch = threadIdx.x & 31; ch < nch; ch += 32) items[o + ch] = make_int2(L, ch * qpc);
}

}  // namespace

cudaError_t run_csr_build(const Csr& c, const int32_t* blocks, int B, int N, int H_kv, int block_k, int topk, int qpc,
                          DevStatus* st, cudaStream_t stream) {
    const int K1 = topk + 1;
    const long long rows = (long long)B * N * H_kv;
    cudaError_t e = cudaMemsetAsync(c.counts, 0, (size_t)c.nlists * 4, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(c.cursor, 0, (size_t)c.nlists * 4, stream);
    if (e != cudaSuccess) return e;
    const int tpb = 256;
    const unsigned grid = (unsigned)((rows + tpb - 1) / tpb);
    ProfScope ps("csr_build", stream);
    k_csr_count<<<grid, tpb, 0, stream>>>(blocks, B, N, H_kv, block_k, K1, c.nb, c.counts, st);
    k_csr_scan<<<1, 1024, 0, stream>>>(c.counts, c.nlists, qpc, c.offsets, c.chunk_off, c.n_items);
    k_csr_fill<<<grid, tpb, 0, stream>>>(blocks, B, N, H_kv, block_k, K1, c.nb, c.offsets, c.cursor, c.entries);
    k_csr_items<<<(c.nlists + 7) / 8, 256, 0, stream>>>(c.counts, c.chunk_off, c.nlists, qpc, c.items);
    return cudaGetLastError();
}

cudaError_t run_csr_items(const Csr& c, int qpc, cudaStream_t stream) {
    k_csr_scan<<<1, 1024, 0, stream>>>(c.counts, c.nlists, qpc, c.offsets, c.chunk_off, c.n_items);
    k_csr_items<<<(c.nlists + 7) / 8, 256, 0, stream>>>(c.counts, c.chunk_off, c.nlists, qpc, c.items);
    return cudaGetLastError();
}

}  // namespace msa
