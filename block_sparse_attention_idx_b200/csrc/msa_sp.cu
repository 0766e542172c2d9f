// Sequence-parallel indexer ("4.1.1 · 监督与联合训练", section 3): P ranks each hold a contiguous
// range of every sequence's key blocks. Each takes the Top-k of its own complete past blocks
// (k_index_topk in key-range mode); only the (score, block id) pairs are exchanged, and the merge
// below reproduces the single-device selection. LSE_idx over the selected tokens is rebuilt from
// each rank's local (maximum a_p, exp-sum z_p) by eq (16): a = max a_p, z = sum exp(a_p - a) z_p;
// a rank's pair comes from the single-device LSE_idx pass (k_lse_idx) run on the selection
// restricted to its blocks.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kMaxCand = 128;  // P * topk candidates per row (at most 8 ranks x 16)

// One warp per (b, i, r) row: Top-k of the P ranks' candidates by (score desc, block id asc), then
// the local block b_i, written ascending and -1 padded. The scores are raw block maxima computed
// the same way on every rank, so the order is the single-device order, ties included.
__global__ void __launch_bounds__(256) k_topk_merge(int B, int N, int H_kv, int block_k, int topk, int P,
                                                    const float* __restrict__ cs, const int32_t* __restrict__ ci,
                                                    int32_t* __restrict__ blocks) {
    const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long rows = (long long)B * N * H_kv;
    if (row >= rows) return;
    const int i = (int)((row / H_kv) % N);
    const int bi = i / block_k;
    const int nc = P * topk;  // candidate x = p * topk + slot
    float v[kMaxCand / 32];
    int id[kMaxCand / 32];
#pragma unroll
    for (int u = 0; u < kMaxCand / 32; ++u) {
        const int x = lane + 32 * u;
        const int p = x / topk, sl = x % topk;
        const size_t o = ((size_t)p * rows + row) * topk + sl;
        id[u] = x < nc ? ci[o] : -1;
        v[u] = id[u] >= 0 ? cs[o] : -INFINITY;
    }
    int mine = 0x7fffffff;  // lane p < topk: the p-th chosen id
    int take = 0;
    for (int p = 0; p < topk; ++p) {
        // this lane's best untaken candidate
        float bv = -INFINITY;
        int bid = 0x7fffffff, bu = -1;
#pragma unroll
        for (int u = 0; u < kMaxCand / 32; ++u)
            if (id[u] >= 0 && (v[u] > bv || (v[u] == bv && id[u] < bid))) {
                bv = v[u];
                bid = id[u];
                bu = u;
            }
        // warp-wide best, ties to the lower block id
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
            if (ov > bv || (ov == bv && oid < bid)) {
                bv = ov;
                bid = oid;
            }
        }
        if (bid == 0x7fffffff) break;  // no candidates left (warp-uniform)
        if (lane == p) mine = bid;
        // a block id appears on at most one rank: retire it wherever it sits
#pragma unroll
        for (int u = 0; u < kMaxCand / 32; ++u)
            if (id[u] == bid) id[u] = -1;
        (void)bu;
        ++take;
    }
    if (lane == take) mine = bi;
    const int n = take + 1;
    int rank = 0;
    for (int x = 0; x < n; ++x) rank += (__shfl_sync(0xffffffffu, mine, x) < mine);
    int32_t* out = blocks + row * (topk + 1);
    if (lane < n) out[rank] = mine;
    else if (lane < topk + 1) out[lane] = -1;
}

// The selection restricted to the blocks [blk0, blk1) a rank holds (others -1): the LSE_idx pass
// over it yields the rank's (a_p, z_p) per row.
__global__ void k_blocks_in_range(long long n, int blk0, int blk1, const int32_t* __restrict__ blocks,
                                  int32_t* __restrict__ out) {
    const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= n) return;
    const int c = blocks[x];
    out[x] = (c >= blk0 && c < blk1) ? c : -1;
}

// eq (16) over the P ranks' pairs [P][rows]: LSE = a + log z.
__global__ void k_lse_combine(int P, long long rows, const float2* __restrict__ ml, float* __restrict__ lse) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= rows) return;
    float a = -INFINITY;
    for (int p = 0; p < P; ++p) a = fmaxf(a, ml[(size_t)p * rows + row].x);
    float z = 0.f;
    for (int p = 0; p < P; ++p) {
        const float2 v = ml[(size_t)p * rows + row];
        if (v.x != -INFINITY) z += v.y * __expf(v.x - a);
    }
    lse[row] = a + logf(z);
}

}  // namespace

cudaError_t run_topk_merge(int B, int N, int H_kv, int block_k, int topk, int P, const float* cand_scores,
                           const int32_t* cand_ids, int32_t* blocks, cudaStream_t st) {
    const long long rows = (long long)B * N * H_kv;
    ProfScope ps("sp_topk_merge", st);
    k_topk_merge<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(B, N, H_kv, block_k, topk, P, cand_scores,
                                                                      cand_ids, blocks);
    return cudaGetLastError();
}

cudaError_t run_blocks_in_range(long long rows, int K1, int blk0, int blk1, const int32_t* blocks, int32_t* out,
                                cudaStream_t st) {
    const long long n = rows * K1;
    k_blocks_in_range<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(n, blk0, blk1, blocks, out);
    return cudaGetLastError();
}

cudaError_t run_lse_combine(int P, long long rows, const float2* ml, float* lse, cudaStream_t st) {
    ProfScope ps("sp_lse_combine", st);
    k_lse_combine<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(P, rows, ml, lse);
    return cudaGetLastError();
}

}  // namespace msa
