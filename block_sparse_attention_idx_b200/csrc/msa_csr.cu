// Inverse selection lists for the KV-outer kernels (MSA blog, KV-outer sparse attention: organise
// the work around the selected KV blocks and gather the queries that need each block).
//
// From blocks[b,i,r,:] we build, for every (b, query window w, r, block c), the list of
// (query i, slot s) pairs that selected c, then cut every list into work items of at most `qpc`
// queries. Items are ordered by (b, w, r, c): consecutive items share their K/V block, and the
// items of one window are contiguous, so the partial results of a window are produced (and
// consumed) close together in time. Every item costs about the same, which keeps hot blocks
// (block 0, needle blocks, local blocks) from becoming stragglers: a block chosen by 20 000 queries
// simply yields about 20 000/qpc items.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static void csr_dims(int B, int N, int H_kv, int block_k, int topk, int wq, int* nb, int* nW, int* w, int* nl,
                     int* me, int* nscan) {
    *nb = (N + block_k - 1) / block_k;
    *w = wq > 0 ? wq : N;
    *nW = (N + *w - 1) / *w;
    *nl = B * *nW * H_kv * *nb;
    *me = B * N * H_kv * (topk + 1);
    *nscan = (*nl + 1023) / 1024;
}

size_t csr_bytes(int B, int N, int H_kv, int block_k, int topk, int wq) {
    int nb, nW, w, nl, me, nscan;
    csr_dims(B, N, H_kv, block_k, topk, wq, &nb, &nW, &w, &nl, &me, &nscan);
    return align256((size_t)nl * 4) * 2 + align256(((size_t)nl + 1) * 4) * 2 + align256((size_t)me * 4) +
           align256((size_t)me * 16) + 256 + align256(((size_t)2 * nscan + 2) * 4) + align256((size_t)B * N * H_kv);
}

void csr_carve(Csr* c, void* base, int B, int N, int H_kv, int block_k, int topk, int wq) {
    uint8_t* p = static_cast<uint8_t*>(base);
    csr_dims(B, N, H_kv, block_k, topk, wq, &c->nb, &c->nW, &c->wq, &c->nlists, &c->max_entries, &c->nscan);
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
    c->items = reinterpret_cast<int4*>(take((size_t)c->max_entries * 16));
    c->n_items = reinterpret_cast<int32_t*>(take(256));
    c->bsum = reinterpret_cast<int32_t*>(take(((size_t)2 * c->nscan + 2) * 4));
    c->nsel = take((size_t)B * N * H_kv);
}

namespace {

__device__ __forceinline__ size_t list_of(int b, int i, int r, int c, int H_kv, int nb, int nW, int wq) {
    return (((size_t)b * nW + i / wq) * H_kv + r) * nb + c;
}

// One thread per selection row: validate it (ids in [0, i/block_k], strictly ascending among the
// non-negative entries), count its entries per list and record how many blocks the row holds.
// Invalid entries are skipped and flagged.
__global__ void k_csr_count(const int32_t* __restrict__ blocks, int B, int N, int H_kv, int block_k, int K1, int nb,
                            int nW, int wq, int32_t* counts, uint8_t* nsel, DevStatus* st) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= (long long)B * N * H_kv) return;
    const int r = (int)(row % H_kv);
    const int i = (int)((row / H_kv) % N);
    const int b = (int)(row / ((long long)H_kv * N));
    const int bi = i / block_k;
    const int32_t* sel = blocks + row * K1;
    int prev = -1, n = 0;
    for (int s = 0; s < K1; ++s) {
        const int c = sel[s];
        if (c < 0) continue;
        if (c > bi || c <= prev) {
            raise_flag(st, MSA_DEV_BAD_BLOCK, 0x401);
            continue;
        }
        prev = c;
        ++n;
        atomicAdd(&counts[list_of(b, i, r, c, H_kv, nb, nW, wq)], 1);
    }
    nsel[row] = (uint8_t)n;
}

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// Exclusive scan over a 1024-thread block; *total receives the block's sum. sh: 33 ints.
__device__ __forceinline__ int block_excl_scan(int v, int* sh, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int inc = warp_incl_scan(v);
    if (lane == 31) sh[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int wv = sh[lane];
        const int wi = warp_incl_scan(wv);
        sh[lane] = wi - wv;
        if (lane == 31) sh[32] = wi;
    }
    __syncthreads();
    const int r = inc - v + sh[warp];
    *total = sh[32];
    __syncthreads();
    return r;
}

// Pass 1: per 1024 lists, the sums of the entry counts and of the chunk counts.
__global__ void __launch_bounds__(1024) k_scan_reduce(const int32_t* __restrict__ counts, int nlists, int qpc,
                                                      int32_t* bsum, int nscan) {
    __shared__ int sh[33];
    const int x = blockIdx.x * 1024 + threadIdx.x;
    const int n = x < nlists ? counts[x] : 0;
    int te, tc;
    block_excl_scan(n, sh, &te);
    block_excl_scan((n + qpc - 1) / qpc, sh, &tc);
    if (threadIdx.x == 0) {
        bsum[blockIdx.x] = te;
        bsum[nscan + blockIdx.x] = tc;
    }
}

// Pass 2 (one block): exclusive scan of the block sums in place; totals at bsum[2*nscan ..].
__global__ void __launch_bounds__(1024) k_scan_top(int32_t* bsum, int nscan) {
    __shared__ int sh[33];
    int carry_e = 0, carry_c = 0;
    for (int base = 0; base < nscan; base += 1024) {
        const int x = base + threadIdx.x;
        const int e = x < nscan ? bsum[x] : 0;
        const int c = x < nscan ? bsum[nscan + x] : 0;
        int te, tc;
        const int se = block_excl_scan(e, sh, &te);
        const int sc = block_excl_scan(c, sh, &tc);
        if (x < nscan) {
            bsum[x] = carry_e + se;
            bsum[nscan + x] = carry_c + sc;
        }
        carry_e += te;
        carry_c += tc;
    }
    if (threadIdx.x == 0) {
        bsum[2 * nscan] = carry_e;
        bsum[2 * nscan + 1] = carry_c;
    }
}

// Pass 3: list offsets and chunk offsets.
__global__ void __launch_bounds__(1024) k_scan_down(const int32_t* __restrict__ counts, int nlists, int qpc,
                                                    const int32_t* __restrict__ bsum, int nscan, int32_t* offsets,
                                                    int32_t* chunk_off, int32_t* n_items) {
    __shared__ int sh[33];
    const int x = blockIdx.x * 1024 + threadIdx.x;
    const int n = x < nlists ? counts[x] : 0;
    int te, tc;
    const int se = block_excl_scan(n, sh, &te);
    const int sc = block_excl_scan((n + qpc - 1) / qpc, sh, &tc);
    if (x < nlists) {
        offsets[x] = bsum[blockIdx.x] + se;
        chunk_off[x] = bsum[nscan + blockIdx.x] + sc;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        offsets[nlists] = bsum[2 * nscan];
        chunk_off[nlists] = bsum[2 * nscan + 1];
        *n_items = bsum[2 * nscan + 1];
    }
}

// One thread per selection row: place each valid entry (i << 5 | slot) into its list.
__global__ void k_csr_fill(const int32_t* __restrict__ blocks, int B, int N, int H_kv, int block_k, int K1, int nb,
                           int nW, int wq, const int32_t* __restrict__ offsets, int32_t* cursor, int32_t* entries) {
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
        const size_t L = list_of(b, i, r, c, H_kv, nb, nW, wq);
        const int pos = offsets[L] + atomicAdd(&cursor[L], 1);
        entries[pos] = (i << 5) | s;
    }
}

// One warp per list: write its work items (list id, index of the chunk's first entry, queries).
__global__ void k_csr_items(const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                            const int32_t* __restrict__ chunk_off, int nlists, int qpc, int4* items) {
    const int L = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (L >= nlists) return;
    const int n = counts[L];
    const int nch = (n + qpc - 1) / qpc;
    const int o = chunk_off[L], e0 = offsets[L];
    for (int ch = threadIdx.x & 31; ch < nch; ch += 32)
        items[o + ch] = make_int4(L, e0 + ch * qpc, min(qpc, n - ch * qpc), 0);
}

}  // namespace

cudaError_t run_csr_items(const Csr& c, int qpc, cudaStream_t stream) {
    k_scan_reduce<<<c.nscan, 1024, 0, stream>>>(c.counts, c.nlists, qpc, c.bsum, c.nscan);
    k_scan_top<<<1, 1024, 0, stream>>>(c.bsum, c.nscan);
    k_scan_down<<<c.nscan, 1024, 0, stream>>>(c.counts, c.nlists, qpc, c.bsum, c.nscan, c.offsets, c.chunk_off,
                                              c.n_items);
    k_csr_items<<<(c.nlists + 7) / 8, 256, 0, stream>>>(c.counts, c.offsets, c.chunk_off, c.nlists, qpc, c.items);
    return cudaGetLastError();
}

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
    k_csr_count<<<grid, tpb, 0, stream>>>(blocks, B, N, H_kv, block_k, K1, c.nb, c.nW, c.wq, c.counts, c.nsel, st);
    k_scan_reduce<<<c.nscan, 1024, 0, stream>>>(c.counts, c.nlists, qpc, c.bsum, c.nscan);
    k_scan_top<<<1, 1024, 0, stream>>>(c.bsum, c.nscan);
    k_scan_down<<<c.nscan, 1024, 0, stream>>>(c.counts, c.nlists, qpc, c.bsum, c.nscan, c.offsets, c.chunk_off,
                                              c.n_items);
    k_csr_fill<<<grid, tpb, 0, stream>>>(blocks, B, N, H_kv, block_k, K1, c.nb, c.nW, c.wq, c.offsets, c.cursor,
                                         c.entries);
    k_csr_items<<<(c.nlists + 7) / 8, 256, 0, stream>>>(c.counts, c.offsets, c.chunk_off, c.nlists, qpc, c.items);
    return cudaGetLastError();
}

}  // namespace msa
