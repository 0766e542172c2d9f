// Sequence-parallel indexer ("4.1.1 · 监督与联合训练", section 3): P ranks each hold one or two
// ranges of every sequence's key blocks. Each takes the Top-k of its own complete past blocks
// (k_index_topk in key-range mode); only the (score, block id) pairs are exchanged, and the merge
// below reproduces the single-device selection. LSE_idx over the selected tokens is rebuilt from
// each rank's local (maximum a_p, exp-sum z_p) by eq (16): a = max a_p, z = sum exp(a_p - a) z_p;
// a rank's pair comes from the single-device LSE_idx pass (k_lse_idx) run on the selection
// restricted to its blocks.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kMaxRanks = 8;

// One thread per (b, i, r) row: each rank's candidate list is already ordered best first by
// (score desc, block id asc), so the Top-k of the union is a P-way merge of the list heads. The
// scores are raw block maxima computed the same way on every rank, so the order is the
// single-device order, ties included. Then the local block b_i; written ascending, -1 padded.
__global__ void __launch_bounds__(256) k_topk_merge(int B, int N, int H_kv, int block_k, int topk, int P,
                                                    const float* __restrict__ cs, const int32_t* __restrict__ ci,
                                                    int32_t* __restrict__ blocks) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long rows = (long long)B * N * H_kv;
    if (row >= rows) return;
    const int i = (int)((row / H_kv) % N);
    int head[kMaxRanks];
    for (int p = 0; p < P; ++p) head[p] = 0;
    int sel[17];
    int n = 0;
    for (; n < topk; ++n) {
        int best = -1, bid = 0x7fffffff;
        float bv = -INFINITY;
        for (int p = 0; p < P; ++p) {
            if (head[p] >= topk) continue;
            const size_t o = ((size_t)p * rows + row) * topk + head[p];
            const int id = ci[o];
            if (id < 0) continue;
            const float v = cs[o];
            if (best < 0 || v > bv || (v == bv && id < bid)) {
                best = p;
                bv = v;
                bid = id;
            }
        }
        if (best < 0) break;
        ++head[best];
        sel[n] = bid;
    }
    sel[n] = i / block_k;  // the local block (larger than every past block)
    // ascending: insertion sort of at most 17 ids
    for (int x = 1; x <= n; ++x) {
        const int v = sel[x];
        int y = x - 1;
        while (y >= 0 && sel[y] > v) {
            sel[y + 1] = sel[y];
            --y;
        }
        sel[y + 1] = v;
    }
    int32_t* out = blocks + row * (topk + 1);
    for (int x = 0; x <= topk; ++x) out[x] = x <= n ? sel[x] : -1;
}

// The selection restricted to the blocks [blk0, blk1) a rank holds (others -1): the LSE_idx pass
// over it yields the rank's (a_p, z_p) per row.
__global__ void k_blocks_in_range(long long n, int blk0, int blk1, int blk2, int blk3,
                                  const int32_t* __restrict__ blocks, int32_t* __restrict__ out) {
    const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= n) return;
    const int c = blocks[x];
    out[x] = ((c >= blk0 && c < blk1) || (c >= blk2 && c < blk3)) ? c : -1;
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
    k_topk_merge<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(B, N, H_kv, block_k, topk, P, cand_scores, cand_ids,
                                                                 blocks);
    return cudaGetLastError();
}

cudaError_t run_blocks_in_range(long long rows, int K1, int blk0, int blk1, int blk2, int blk3, const int32_t* blocks,
                                int32_t* out, cudaStream_t st) {
    const long long n = rows * K1;
    k_blocks_in_range<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(n, blk0, blk1, blk2, blk3, blocks, out);
    return cudaGetLastError();
}

cudaError_t run_lse_combine(int P, long long rows, const float2* ml, float* lse, cudaStream_t st) {
    ProfScope ps("sp_lse_combine", st);
    k_lse_combine<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(P, rows, ml, lse);
    return cudaGetLastError();
}

}  // namespace msa
