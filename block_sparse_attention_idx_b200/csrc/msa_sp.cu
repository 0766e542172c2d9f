// Sequence-parallel indexer ("4.1.1 · 监督与联合训练", section 3): P ranks each hold a contiguous
// range of every sequence's key blocks. Each takes the Top-k of its own complete past blocks
// (k_index_topk in key-range mode); only the (score, block id) pairs are exchanged, and the merge
// below reproduces the single-device selection. LSE_idx over the selected tokens is rebuilt from
// each rank's local (maximum a_p, exp-sum z_p) by eq (16): a = max a_p, z = sum exp(a_p - a) z_p.
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

// One warp per (b, i, r) row: (a_p, z_p) of the index scores (scale_idx included) over the causal
// tokens of the row's selected blocks that this rank holds. Lanes take tokens; each keeps a running
// (max, exp-sum) and the warp merges them. (-inf, 0) when the rank holds none of them.
template <int DI>
__global__ void __launch_bounds__(256) k_lse_idx_local(int B, int N, int H_kv, int block_k, int topk, float scale_idx,
                                                       const __nv_bfloat16* __restrict__ q_idx,
                                                       const __nv_bfloat16* __restrict__ k_idx, int tok0, int ntok,
                                                       const int32_t* __restrict__ blocks, float2* __restrict__ ml) {
    const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= (long long)B * N * H_kv) return;
    const int i = (int)((row / H_kv) % N);
    const int b = (int)(row / ((long long)H_kv * N));
    const int bi = i / block_k;
    const int K1 = topk + 1;
    float q[DI];
    {
        const __nv_bfloat162* qr = reinterpret_cast<const __nv_bfloat162*>(q_idx + row * DI);
#pragma unroll
        for (int c = 0; c < DI / 2; ++c) {
            const float2 f = __bfloat1622float2(qr[c]);
            q[2 * c] = f.x;
            q[2 * c + 1] = f.y;
        }
    }
    float m = -INFINITY, z = 0.f;
    int prev = -1;
    for (int s = 0; s < K1; ++s) {
        const int c = blocks[row * K1 + s];
        if (c < 0 || c > bi || c <= prev) continue;  // the selection rule of the inverse lists
        prev = c;
        const int j0 = c * block_k, j1 = min(j0 + block_k, i + 1);
        if (j0 < tok0 || j0 >= tok0 + ntok) continue;  // a block this rank does not hold
        for (int j = j0 + lane; j < j1; j += 32) {
            const uint4* kr = reinterpret_cast<const uint4*>(k_idx + ((size_t)b * ntok + (j - tok0)) * DI);
            float acc = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < DI / 8; ++c8) {
                const uint4 u = kr[c8];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc = fmaf(q[8 * c8 + 2 * e], __uint_as_float(w[e] << 16), acc);
                    acc = fmaf(q[8 * c8 + 2 * e + 1], __uint_as_float(w[e] & 0xffff0000u), acc);
                }
            }
            const float sc = acc * scale_idx;
            if (sc > m) {
                z = z * __expf(m - sc) + 1.f;
                m = sc;
            } else {
                z += __expf(sc - m);
            }
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        const float om = __shfl_xor_sync(0xffffffffu, m, o), oz = __shfl_xor_sync(0xffffffffu, z, o);
        const float nm = fmaxf(m, om);
        z = (m == -INFINITY ? 0.f : z * __expf(m - nm)) + (om == -INFINITY ? 0.f : oz * __expf(om - nm));
        m = nm;
    }
    if (lane == 0) ml[row] = make_float2(m, z);
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

cudaError_t run_lse_idx_local(int B, int N, int H_kv, int d_idx, int block_k, int topk, float scale_idx,
                              const void* q_idx, const void* k_idx_local, int tok0, int ntok, const int32_t* blocks,
                              float2* ml, cudaStream_t st) {
    const long long rows = (long long)B * N * H_kv;
    const unsigned grid = (unsigned)((rows * 32 + 255) / 256);
    const auto* q = static_cast<const __nv_bfloat16*>(q_idx);
    const auto* k = static_cast<const __nv_bfloat16*>(k_idx_local);
    ProfScope ps("sp_lse_local", st);
    if (d_idx == 64)
        k_lse_idx_local<64><<<grid, 256, 0, st>>>(B, N, H_kv, block_k, topk, scale_idx, q, k, tok0, ntok, blocks, ml);
    else
        k_lse_idx_local<32><<<grid, 256, 0, st>>>(B, N, H_kv, block_k, topk, scale_idx, q, k, tok0, ntok, blocks, ml);
    return cudaGetLastError();
}

cudaError_t run_lse_combine(int P, long long rows, const float2* ml, float* lse, cudaStream_t st) {
    ProfScope ps("sp_lse_combine", st);
    k_lse_combine<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(P, rows, ml, lse);
    return cudaGetLastError();
}

}  // namespace msa
