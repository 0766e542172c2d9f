// Index branch of MSA: scoring, causal block max-pool and softmax-free Top-k in one kernel
// ("MSA Indexer 与 DSA Lightning Indexer 的差别", sections 2.1-2.2; MSA blog, softmax-free Top-K).
//
// One CTA owns 128 consecutive (query, group) rows of one sequence: rows are the flattened
// Q_idx [N*H_kv, d_idx] slab, so a row tile is a single TMA box. The CTA walks the key tiles of
// 128 tokens that hold the complete past blocks of its rows; for each tile one elected thread issues
// tcgen05.mma (M=128 rows, N=128 tokens, K=d_idx) into one of two TMEM accumulators while four
// epilogue warps read the other accumulator (one TMEM lane = one row per thread), take the max of
// every block of block_k columns and insert it into the row's sorted Top-16 list in registers.
// Scores never leave the SM. The scale is positive, so the ranking uses raw dot products.
//
// Selection rule: Top-k over the complete past blocks {0 .. b_i-1} by (max desc, block id asc),
// plus the local block b_i; written ascending and padded with -1.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kRows = 128;      // rows per CTA (one TMEM lane each)
constexpr int kCols = 128;      // key tokens per tile
constexpr int kStages = 4;      // K_idx ring depth
constexpr int kKMax = 16;       // largest supported topk
constexpr int kThreads = 192;   // warps 0-3 epilogue, 4 TMA, 5 MMA

template <int DIDX>
struct IndexSmem {
    static constexpr int kTileBytes = kRows * DIDX * 2;
    alignas(1024) uint8_t q[kTileBytes];
    alignas(1024) uint8_t k[kStages][kCols * DIDX * 2];
    uint64_t q_full;
    uint64_t k_full[kStages];
    uint64_t k_empty[kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// MINB CTAs per SM: 2 caps the registers at 168 (a few spill to the stack and the loop runs ~20 %
// more instructions) so that two CTAs share an SM and hide each other's waits; 1 leaves them
// uncapped for grids that would not fill two slots per SM anyway.
template <int DIDX, int MINB>
__global__ void __launch_bounds__(kThreads, MINB)
    k_index_topk(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, IndexArgs a) {
    extern __shared__ uint8_t smem_raw[];
    IndexSmem<DIDX>& s = *reinterpret_cast<IndexSmem<DIDX>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    constexpr uint32_t kPitch = DIDX * 2;                 // bytes per row (64 or 128)
    constexpr uint32_t kLayout = DIDX == 64 ? 2u : 4u;    // SWIZZLE_128B / SWIZZLE_64B
    constexpr uint32_t kSBO = 8 * kPitch;
    constexpr uint32_t kIdesc = umma_idesc_bf16(kRows, kCols, false, false);

    const int tiles_per_seq = gridDim.x;
    const int tile = tiles_per_seq - 1 - (int)blockIdx.x;  // longest tiles first
    const int b = blockIdx.y;
    const int rows_per_seq = a.N * a.H_kv;
    const int R0 = tile * kRows;
    const int i_hi = min(a.N - 1, (R0 + kRows - 1) / a.H_kv);
    const int bmax = i_hi / a.block_k;                      // largest local block among the rows
    const int ntok = bmax * a.block_k;                      // tokens of complete past blocks
    // tiles of the held key ranges that hold complete past blocks: those of [tok0, tok0 + ntok),
    // then those of the second range [tok0b, tok0b + ntokb), whose tokens follow in k_idx
    const int span_a = min(ntok, a.tok0 + a.ntok) - a.tok0;
    const int nkt_a = span_a > 0 ? (span_a + kCols - 1) / kCols : 0;
    const int span_b = a.ntokb > 0 ? min(ntok, a.tok0b + a.ntokb) - a.tok0b : 0;
    const int nkt = nkt_a + (span_b > 0 ? (span_b + kCols - 1) / kCols : 0);
    const int blk_end_a = (a.tok0 + a.ntok) / a.block_k;    // first block past each held range
    const int blk_end_b = (a.tok0b + a.ntokb) / a.block_k;

    const int warp = warp_id(), lane = lane_id();
    if (threadIdx.x == 0) {
        mbar_init(&s.q_full, 1);
        for (int st = 0; st < kStages; ++st) {
            mbar_init(&s.k_full[st], 1);
            mbar_init(&s.k_empty[st], 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s.acc_full[x], 1);
            mbar_init(&s.acc_empty[x], kRows);
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&s.tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 4) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0 && nkt > 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            mbar_arrive_expect_tx(&s.q_full, IndexSmem<DIDX>::kTileBytes);
            tma_load_2d(s.q, &tm_q, &s.q_full, 0, b * rows_per_seq + R0);
            int kt = 0;
            for (; kt < nkt; ++kt) {
                const int st = kt % kStages;
                const uint32_t ph = (kt / kStages) & 1;
                if (!mbar_wait(&s.k_empty[st], ph ^ 1, a.status, 0x101)) { s.abort = 1; break; }
                mbar_arrive_expect_tx(&s.k_full[st], kCols * DIDX * 2);
                const int row0 = kt < nkt_a ? kt * kCols : a.ntok + (kt - nkt_a) * kCols;  // token row in k_idx
                tma_load_3d(s.k[st], &tm_k, &s.k_full[st], 0, row0, b);
            }
            // make sure no copy of ours is still landing when the CTA leaves
            for (int x = max(0, kt - kStages); x < kt; ++x)
                mbar_wait(&s.k_full[x % kStages], (x / kStages) & 1, a.status, 0x102);
            mbar_wait(&s.q_full, 0, a.status, 0x103);
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0 && nkt > 0) {
            bool ok = mbar_wait(&s.q_full, 0, a.status, 0x201);
            const uint32_t q_base = smem_u32(s.q);
            for (int kt = 0; ok && kt < nkt; ++kt) {
                const int st = kt % kStages;
                const int acc = kt & 1;
                if (!mbar_wait(&s.k_full[st], (kt / kStages) & 1, a.status, 0x202)) { ok = false; break; }
                if (!mbar_wait(&s.acc_empty[acc], ((kt >> 1) & 1) ^ 1, a.status, 0x203)) { ok = false; break; }
                tc_fence_after();
                const uint32_t k_base = smem_u32(s.k[st]);
#pragma unroll
                for (int ks = 0; ks < DIDX / 16; ++ks) {
                    const uint64_t da = umma_sdesc(q_base + ks * 32, 16, kSBO, kLayout);
                    const uint64_t db = umma_sdesc(k_base + ks * 32, 16, kSBO, kLayout);
                    umma_bf16(tmem + acc * kCols, da, db, kIdesc, ks > 0);
                }
                umma_commit(&s.k_empty[st]);
                umma_commit(&s.acc_full[acc]);
            }
            if (!ok) s.abort = 1;
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, a.status, 0x204);
        }
    } else {
        // ---------------------------------------------------------------- epilogue warps 0-3
        const int m = threadIdx.x;  // TMEM lane == row within the tile
        const int R = R0 + m;
        const bool valid = R < rows_per_seq;
        const int i = valid ? R / a.H_kv : 0;
        const int r = valid ? R % a.H_kv : 0;
        const int bi = i / a.block_k;
        float topv[kKMax];
        int topi[kKMax];
#pragma unroll
        for (int p = 0; p < kKMax; ++p) { topv[p] = -INFINITY; topi[p] = -1; }
        bool ok = true;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        for (int kt = 0; kt < nkt; ++kt) {
            const int acc = kt & 1;
            const bool got = mbar_wait(&s.acc_full[acc], (kt >> 1) & 1, a.status, 0x301);
            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
            tc_fence_after();
            // the tile's 128 scores of this row: four loads in flight, one wait, then the maxima of
            // its 32-column chunks (three-input max)
            float cmax[4];
            {
                uint32_t v[4][32];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(lane_addr + acc * kCols + q4 * 32, v[q4]);
                tmem_ld_wait();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    reg_fence(v[q4]);
                    const float* f = reinterpret_cast<const float*>(v[q4]);
                    float m0 = max3f(f[0], f[1], f[2]), m1 = max3f(f[3], f[4], f[5]);
#pragma unroll
                    for (int c = 6; c < 30; c += 4) {  // columns 6 .. 29
                        m0 = max3f(m0, f[c], f[c + 1]);
                        m1 = max3f(m1, f[c + 2], f[c + 3]);
                    }
                    cmax[q4] = max3f(m0, m1, fmaxf(f[30], f[31]));
                }
            }
            tc_fence_before();
            mbar_arrive(&s.acc_empty[acc]);
            // one candidate per complete past block inside this tile (a tile of the first range that
            // runs past its end holds blocks at or past blk_end_a, which the test below drops)
            const int chunks_per_block = a.block_k / 32;
            const int tile_tok = kt < nkt_a ? a.tok0 + kt * kCols : a.tok0b + (kt - nkt_a) * kCols;
            const int blk_end = kt < nkt_a ? blk_end_a : blk_end_b;
            for (int c0 = 0; c0 < 4; c0 += chunks_per_block) {
                const int cb = (tile_tok + c0 * 32) / a.block_k;
                float v = cmax[c0];
                for (int x = 1; x < chunks_per_block; ++x) v = fmaxf(v, cmax[c0 + x]);
                if (cb < bi && cb < blk_end && v > topv[kKMax - 1]) {
                    // stable insertion: equal maxima keep the earlier (lower) block id first
#pragma unroll
                    for (int p = kKMax - 1; p > 0; --p) {
                        const bool sh = topv[p - 1] < v;
                        const bool put = !sh && topv[p] < v;
                        topv[p] = sh ? topv[p - 1] : (put ? v : topv[p]);
                        topi[p] = sh ? topi[p - 1] : (put ? cb : topi[p]);
                    }
                    if (topv[0] < v) { topv[0] = v; topi[0] = cb; }
                }
            }
        }
        if (!ok) s.abort = 1;
        if (valid && ok && a.cand_ids) {
            // the row's Top-k of the held range, best first, unmerged
            const size_t o = ((size_t)b * rows_per_seq + R) * a.topk;
#pragma unroll
            for (int p = 0; p < kKMax; ++p)
                if (p < a.topk) {
                    a.cand_scores[o + p] = topi[p] >= 0 ? topv[p] : -INFINITY;
                    a.cand_ids[o + p] = topi[p];
                }
        } else if (valid && ok) {
            // first topk entries plus the local block, ascending, -1 padded
            int sel[kKMax + 1];
#pragma unroll
            for (int p = 0; p < kKMax; ++p) sel[p] = (p < a.topk && topi[p] >= 0) ? topi[p] : 0x7fffffff;
            sel[kKMax] = bi;
#pragma unroll
            for (int pass = 0; pass < kKMax + 1; ++pass) {
#pragma unroll
                for (int p = (pass & 1); p + 1 < kKMax + 1; p += 2) {
                    const int lo = min(sel[p], sel[p + 1]), hi = max(sel[p], sel[p + 1]);
                    sel[p] = lo;
                    sel[p + 1] = hi;
                }
            }
            int32_t* out = a.blocks + ((size_t)b * rows_per_seq + R) * (a.topk + 1);
#pragma unroll
            for (int p = 0; p < kKMax + 1; ++p)
                if (p <= a.topk) out[p] = sel[p] == 0x7fffffff ? -1 : sel[p];
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 256);
}

}  // namespace

template <int DIDX, int MINB>
static cudaError_t launch_index(const IndexArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, int tiles,
                                cudaStream_t st) {
    // at least 80 KB so that no more than two CTAs (2 x 256 TMEM columns) share an SM
    const size_t smem = std::max<size_t>(sizeof(IndexSmem<DIDX>) + 1024, 80 * 1024);
    cudaError_t e =
        cudaFuncSetAttribute(k_index_topk<DIDX, MINB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("index_topk", st);
    k_index_topk<DIDX, MINB><<<dim3(tiles, a.B), kThreads, smem, st>>>(tq, tk, a);
    return cudaGetLastError();
}

template <int DIDX>
static cudaError_t launch_index(const IndexArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, int num_sms,
                                cudaStream_t st) {
    const int tiles = (a.N * a.H_kv + kRows - 1) / kRows;
    // two CTAs per SM once the grid fills two slots on every SM (measured: N=32768 0.55 -> 0.40 ms;
    // at N=8192, 256 CTAs, one per SM is 8 % faster)
    if ((long long)tiles * a.B >= 2LL * num_sms) return launch_index<DIDX, 2>(a, tq, tk, tiles, st);
    return launch_index<DIDX, 1>(a, tq, tk, tiles, st);
}

cudaError_t run_index_topk(const IndexArgs& a, const void* q_idx, const void* k_idx, int num_sms, cudaStream_t st) {
    CUtensorMap tq, tk;
    const uint64_t rows = (uint64_t)a.B * a.N * a.H_kv;
    const int sw = a.d_idx == 64 ? 128 : 64;
    if (!make_tmap_2d(&tq, q_idx, a.d_idx, rows, (uint64_t)a.d_idx * 2, a.d_idx, kRows, sw)) return cudaErrorInvalidValue;
    const uint64_t held = (uint64_t)a.ntok + a.ntokb;
    if (!make_tmap_3d(&tk, k_idx, a.d_idx, held, a.B, (uint64_t)a.d_idx * 2, held * a.d_idx * 2,
                      a.d_idx, kCols, 1, sw))
        return cudaErrorInvalidValue;
    return a.d_idx == 64 ? launch_index<64>(a, tq, tk, num_sms, st) : launch_index<32>(a, tq, tk, num_sms, st);
}

}  // namespace msa
