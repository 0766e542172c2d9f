// Backward of the main-branch sparse attention with the selection held fixed ("2.4 · 训练原生稀疏",
// section 2.2, eq (11): on the fixed set, selected attention is ordinary attention, and positions
// outside the set get no gradient; the backward must stay on the sparse edges, section 3.2).
// For each (query i, head h) with token set J, upstream gradient g = dO and output o:
//   P_j  = exp(scale q.k_j - LSE)           (recomputed from the forward's LSE)
//   dS_j = P_j (g.v_j - g.o)                (the gradient of the logit, eq (11))
//   dV_j += P_j g,  dK_j += scale dS_j q,  dQ += scale sum_j dS_j k_j
//
// KV-outer over the inverse lists of the forward: one item = one selected block c of group r plus
// up to 128/G queries that chose it (their G heads are the 128 rows). Per item, in TMEM:
//   S^T  = K_c . Q^T          tcgen05.mma M=128 tokens, N=128 rows, K=d       cols [0,128)
//   dP^T = V_c . dO^T         tcgen05.mma                                      cols [128,256)
//   thread = token: P^T, dS^T = P^T (dP^T - delta) as bf16 back into TMEM over S^T / dP^T, and dS^T
//   as bf16 into shared memory
//   dV_c += P^T . dO          tcgen05.mma A = P^T from TMEM, B = dO (MN-major)  cols [256,256+d)
//   dK_c += dS^T . Q          tcgen05.mma A = dS^T from TMEM, B = Q (MN-major)  cols [384,384+d)
//   dQ    = dS . K_c          tcgen05.mma A = dS (MN-major smem), B = K_c, in 64-column halves
//                             placed in the free upper halves of the S^T and dP^T columns
// dQ rows are added to the fp32 output with vector reductions after every item; dK_c and dV_c stay
// in TMEM across the consecutive items of one block and are added to the outputs when the block
// changes (a block's items can be split between two CTAs, hence reductions rather than stores).
// P and dS enter the tensor cores as bf16, as in the forward's P.
//
// Warp roles (320 threads): warps 0-7 epilogue (warp w: TMEM lane quarter w % 4, i.e. 32 tokens,
// or 32 item rows for dQ; column half w / 4), warp 8 loads (item metadata, the Q and dO rows by one
// 5-D TMA box per query, K and V tiles), warp 9 issues the MMAs and owns TMEM.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kRows = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kEpiWarps = 8;  // two per TMEM lane quarter: item rows (S^T columns) split in halves
constexpr int kEpi = kEpiWarps * 32;
constexpr int kProdWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 10 * 32;

__device__ __forceinline__ void red_add_v4(float* p, float x, float y, float z, float w) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(x), "f"(y), "f"(z), "f"(w)
                 : "memory");
}

template <int QPC>
struct BwdMeta {
    int L, count, flush, pad;  // list id (b, r, c), item queries, 1 when the next item is another block or none
    int qi[QPC];               // query index of each item query
    float lse2[kRows];         // LSE * log2(e) per item row (query-major, head-minor)
    float delta[kRows];        // dO . O per item row
};

template <int D, int QPC>
struct BwdSmem {
    alignas(1024) uint8_t q[2][kRows * D * 2];     // Q rows: 8-row x 64-column 128B-swizzled atoms [row/8][D/64]
    alignas(1024) uint8_t dout[2][kRows * D * 2];  // dO rows, same layout
    alignas(1024) uint8_t k[kRows * D * 2];     // K tile: D/64 sub-tiles of [128 token rows x 128 B], rows >= BK zero
    alignas(1024) uint8_t v[kRows * D * 2];     // V tile, same
    alignas(1024) uint8_t ds[kRows * kRows * 2];  // dS^T: 2 sub-tiles of [128 token rows x 64 item rows]
    BwdMeta<QPC> meta;
    uint64_t meta_full, meta_empty, q_full[2], q_empty[2], kv_full, kv_empty, s_full, p_full, d_full, t_free, drain;
    uint32_t tmem_base;
    int abort;
};

template <int D, int BK, int G>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_bwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, BwdArgs a) {
    constexpr int QPC = kRows / G;
    using Sm = BwdSmem<D, QPC>;
    static_assert(G % 8 == 0 && G <= 32, "one 5-D box of G/8 head groups per query");
    extern __shared__ uint8_t smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kIdescS = umma_idesc_bf16(kRows, kRows, false, false);  // S^T, dP^T
    constexpr uint32_t kIdescKV = umma_idesc_bf16(kRows, D, false, true);      // dV, dK (A from TMEM)
    constexpr uint32_t kIdescQ = umma_idesc_bf16(kRows, 64, true, true);       // dQ halves
    constexpr uint32_t kColS = 0, kColP = 128, kColDV = 256, kColDK = 384;

    const Csr& cs = a.csr;
    const int T = *cs.n_items;
    const int per = (T + gridDim.x - 1) / gridDim.x;
    const int t0 = blockIdx.x * per, t1 = min(T, t0 + per);
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        mbar_init(&s.meta_full, 32);
        mbar_init(&s.meta_empty, kEpi + 1);  // the epilogue threads and the MMA issuer
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s.q_full[x], 1);
            mbar_init(&s.q_empty[x], 1);
        }
        mbar_init(&s.kv_full, 1);
        mbar_init(&s.kv_empty, 1);
        mbar_init(&s.s_full, 1);
        mbar_init(&s.p_full, kEpi);
        mbar_init(&s.d_full, 1);
        mbar_init(&s.t_free, kEpi);
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    // every tile row an MMA may read must hold finite values: Q / dO rows past an item's count and
    // K / V rows past block_k are multiplied by zeros, and start as zeros
    {
        uint4* z = reinterpret_cast<uint4*>(s.q);
        for (int x = threadIdx.x; x < 6 * kRows * D * 2 / 16; x += kThreads) z[x] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async();
    if (warp == kMmaWarp) {
        tmem_alloc(&s.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------------------ loads
        // Item n: its Q and dO rows into buffer n % 2 once the MMA has released it (item n-2), then
        // its metadata (plain loads into registers, stored once the epilogue is done with item n-1,
        // then one arrival per lane: no load is in flight at these release arrives), then K / V of a
        // new block once the MMA has released the previous block. Loads thus run one item ahead.
        bool ok = true;
        int kv_loads = 0, prevL = -1, issued = 0;
        int4 rec = t0 < t1 ? cs.items[t0] : make_int4(-1, 0, 0, 0);
        for (int t = t0, n = 0; t < t1; ++t, ++n) {
            const int L = rec.x, count = rec.z;
            const int c = L % cs.nb, r = (L / cs.nb) % a.H_kv, b = L / (cs.nb * a.H_kv);
            const int4 nrec = t + 1 < t1 ? cs.items[t + 1] : make_int4(-1, 0, 0, 0);
            const int e = lane < count ? cs.entries[rec.y + lane] : 0;
            const int qi = e >> 5;
            float l2[4], dl[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int row = lane + 32 * x;
                const int m = row / G, h = row % G;
                const int qm = __shfl_sync(0xffffffffu, qi, m < QPC ? m : 0);
                const size_t o = ((size_t)b * a.N + qm) * a.H_q + (size_t)r * G + h;
                l2[x] = m < count ? a.lse[o] * kLog2e : 0.f;
                dl[x] = m < count ? a.delta[o] : 0.f;
            }
            const int qb = n & 1;
            int okl = 1;
            // Q and dO rows of the item queries
            if (lane == 0) okl = mbar_wait(&s.q_empty[qb], ((n >> 1) & 1) ^ 1, a.status, 0xa02);
            if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
            if (lane == 0) mbar_arrive_expect_tx_relaxed(&s.q_full[qb], (uint32_t)(2 * count * G * D * 2));
            __syncwarp();
            if (lane < count) {
                tma_load_5d(s.q[qb] + lane * G * D * 2, &tm_q, &s.q_full[qb], 0, 0, 0, r * G / 8, b * a.N + qi);
                tma_load_5d(s.dout[qb] + lane * G * D * 2, &tm_do, &s.q_full[qb], 0, 0, 0, r * G / 8, b * a.N + qi);
            }
            if (lane == 0) okl = mbar_wait(&s.meta_empty, (n & 1) ^ 1, a.status, 0xa01);
            if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
            BwdMeta<QPC>& mt = s.meta;
            if (lane == 0) {
                mt.L = L;
                mt.count = count;
                mt.flush = nrec.x != L;
            }
            if (lane < QPC) mt.qi[lane] = lane < count ? qi : 0;
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                mt.lse2[lane + 32 * x] = l2[x];
                mt.delta[lane + 32 * x] = dl[x];
            }
            mbar_arrive(&s.meta_full);
            // K and V of a new block
            if (L != prevL) {
                if (lane == 0) {
                    if (kv_loads > 0) okl = mbar_wait(&s.kv_empty, (kv_loads - 1) & 1, a.status, 0xa03);
                    if (okl) {
                        mbar_arrive_expect_tx_relaxed(&s.kv_full, 2 * (D / 64) * BK * 128);
#pragma unroll
                        for (int sub = 0; sub < D / 64; ++sub) {
                            tma_load_4d(s.k + sub * kRows * 128, &tm_k, &s.kv_full, sub * 64, r, c * BK, b);
                            tma_load_4d(s.v + sub * kRows * 128, &tm_v, &s.kv_full, sub * 64, r, c * BK, b);
                        }
                    }
                }
                if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
                ++kv_loads;
                prevL = L;
            }
            ++issued;
            rec = nrec;
        }
        if (!ok) s.abort = 1;
        // nothing may still be landing in shared memory when the CTA exits
        if (lane == 0) {
            for (int x = 0; x < 2 && x < issued; ++x) {
                const int nl = issued - 1 - x;  // last use of buffer nl & 1
                mbar_wait(&s.q_full[nl & 1], (nl >> 1) & 1, a.status, 0xa04);
            }
            if (kv_loads > 0) mbar_wait(&s.kv_full, (kv_loads - 1) & 1, a.status, 0xa05);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            int kv_group = -1, prevL = -1;
            const uint32_t ka = smem_u32(s.k), va = smem_u32(s.v), dsa = smem_u32(s.ds);
            for (int t = t0, n = 0; t < t1; ++t, ++n) {
                const int qb = n & 1;
                const uint32_t qa = smem_u32(s.q[qb]), da = smem_u32(s.dout[qb]);
                if (!mbar_wait(&s.meta_full, n & 1, a.status, 0xa11)) { ok = false; break; }
                const int L = s.meta.L;
                mbar_arrive(&s.meta_empty);
                bool first = false;
                if (L != prevL) {
                    if (kv_group >= 0) umma_commit(&s.kv_empty);  // the previous block's tiles are no longer read
                    ++kv_group;
                    prevL = L;
                    first = true;
                    if (!mbar_wait(&s.kv_full, kv_group & 1, a.status, 0xa12)) { ok = false; break; }
                }
                if (!mbar_wait(&s.q_full[qb], (n >> 1) & 1, a.status, 0xa13)) { ok = false; break; }
                if (n > 0 && !mbar_wait(&s.t_free, (n - 1) & 1, a.status, 0xa14)) { ok = false; break; }
                tc_fence_after();
                // S^T = K . Q^T and dP^T = V . dO^T (both operands K-major)
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t sub = (ks * 16) / 64, off = (ks & 3) * 32;
                    const uint64_t dk_ = umma_sdesc(ka + sub * (kRows * 128) + off, 16, 1024, 2);
                    const uint64_t dq_ = umma_sdesc(qa + sub * 1024 + off, 16, (D / 64) * 1024, 2);
                    umma_bf16(tmem + kColS, dk_, dq_, kIdescS, ks > 0);
                }
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t sub = (ks * 16) / 64, off = (ks & 3) * 32;
                    const uint64_t dv_ = umma_sdesc(va + sub * (kRows * 128) + off, 16, 1024, 2);
                    const uint64_t do_ = umma_sdesc(da + sub * 1024 + off, 16, (D / 64) * 1024, 2);
                    umma_bf16(tmem + kColP, dv_, do_, kIdescS, ks > 0);
                }
                umma_commit(&s.s_full);
                if (!mbar_wait(&s.p_full, n & 1, a.status, 0xa15)) { ok = false; break; }
                tc_fence_after();
                // dV += P^T . dO, dK += dS^T . Q: A from TMEM (bf16 pairs, 8 columns per 16 rows),
                // B = the row tiles read MN-major (16 rows = two 8-row atom groups per k-step)
#pragma unroll
                for (int ks = 0; ks < kRows / 16; ++ks) {
                    const uint64_t bdo = umma_sdesc(da + 2 * ks * (D / 64) * 1024, 1024, (D / 64) * 1024, 2);
                    umma_bf16_tmem_a(tmem + kColDV, tmem + kColS + 8 * ks, bdo, kIdescKV, (first && ks == 0) ? 0u : 1u);
                }
#pragma unroll
                for (int ks = 0; ks < kRows / 16; ++ks) {
                    const uint64_t bq = umma_sdesc(qa + 2 * ks * (D / 64) * 1024, 1024, (D / 64) * 1024, 2);
                    umma_bf16_tmem_a(tmem + kColDK, tmem + kColP + 8 * ks, bq, kIdescKV, (first && ks == 0) ? 0u : 1u);
                }
                // dQ = dS . K in 64-column halves: A = dS^T tile read MN-major, B = K sub-tile MN-major
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks) {
                        const uint64_t ads = umma_sdesc(dsa + ks * 16 * 128, kRows * 128, 1024, 2);
                        const uint64_t bk_ = umma_sdesc(ka + h * (kRows * 128) + ks * 16 * 128, kRows * 128, 1024, 2);
                        umma_bf16(tmem + (h == 0 ? 64u : 192u), ads, bk_, kIdescQ, ks > 0);
                    }
                }
                umma_commit(&s.d_full);
                umma_commit(&s.q_empty[qb]);
            }
            if (!ok) s.abort = 1;
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, a.status, 0xa16);
        }
    } else {
        // ------------------------------------------------------------------------ epilogue
        const int wq = warp & 3, hf = warp >> 2;
        const int tt = wq * 32 + lane;  // token lane for S^T / dP^T / dV / dK, item row for dQ
        const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
        const float sl2 = a.scale * kLog2e;
        for (int t = t0, n = 0; t < t1; ++t, ++n) {
            if (!__all_sync(0xffffffffu, mbar_wait(&s.meta_full, n & 1, a.status, 0xa21))) {
                s.abort = 1;
                break;
            }
            const BwdMeta<QPC>& mt = s.meta;
            const int L = mt.L, count = mt.count, flush = mt.flush;
            const int c = L % cs.nb, r = (L / cs.nb) % a.H_kv, b = L / (cs.nb * a.H_kv);
            const int tok = c * BK + tt;
            const int nrows = count * G;
            if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full, n & 1, a.status, 0xa22))) {
                s.abort = 1;
                break;
            }
            tc_fence_after();
            // Each warp forms P and dS of its two 32-row chunks in registers first: P / dS are stored
            // packed over columns that the other warp half of the lane quarter may not have read yet
            // (chunk cc goes to columns 16cc..16cc+15), so the stores wait for a barrier of the
            // epilogue warps.
            uint32_t pk[2][16], dk[2][16];
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cc = 2 * hf + k2;
                uint32_t sv[32], pv[32];
                tmem_ld32(lane_addr + kColS + 32 * cc, sv);
                tmem_ld32(lane_addr + kColP + 32 * cc, pv);
                // rows 32cc..32cc+31 hold 32 / G queries (or part of one): is each query's block token
                // causal for this thread?
                bool cz[(32 + G - 1) / G];
#pragma unroll
                for (int u = 0; u < (32 + G - 1) / G; ++u) {
                    const int row0 = 32 * cc + u * G;
                    cz[u] = row0 < nrows && tt < BK && tok <= mt.qi[row0 / G];
                }
                tmem_ld_wait();
                reg_fence(sv);
                reg_fence(pv);
#pragma unroll
                for (int e = 0; e < 32; e += 4) {
                    const float4 l4 = *reinterpret_cast<const float4*>(&mt.lse2[32 * cc + e]);
                    const float4 d4 = *reinterpret_cast<const float4*>(&mt.delta[32 * cc + e]);
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
                    float p4[4], g4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const bool valid = cz[(e + u) / G];
                        const float p = fast_exp2(fmaf(__uint_as_float(sv[e + u]), sl2, -lv[u]));
                        p4[u] = valid ? p : 0.f;
                        g4[u] = valid ? p * (__uint_as_float(pv[e + u]) - dv[u]) : 0.f;
                    }
                    pk[k2][e / 2] = pack_bf16x2(p4[0], p4[1]);
                    pk[k2][e / 2 + 1] = pack_bf16x2(p4[2], p4[3]);
                    dk[k2][e / 2] = pack_bf16x2(g4[0], g4[1]);
                    dk[k2][e / 2 + 1] = pack_bf16x2(g4[2], g4[3]);
                }
            }
            bar_sync_named(1, kEpi);  // every epilogue warp has read its S^T / dP^T columns
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int cc = 2 * hf + k2;
                tmem_st16(lane_addr + kColS + 16 * cc, pk[k2]);
                tmem_st16(lane_addr + kColP + 16 * cc, dk[k2]);
                // dS^T row of this token: item rows 32cc..32cc+31, four 16-byte chunks of 8 rows
                uint8_t* dsrow = s.ds + (cc >> 1) * (kRows * 128);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t ch = 4 * (cc & 1) + j;
                    *reinterpret_cast<uint4*>(dsrow + swz(tt, ch * 16, 128)) =
                        make_uint4(dk[k2][4 * j], dk[k2][4 * j + 1], dk[k2][4 * j + 2], dk[k2][4 * j + 3]);
                }
            }
            tmem_st_wait();
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&s.p_full);
            if (!__all_sync(0xffffffffu, mbar_wait(&s.d_full, n & 1, a.status, 0xa23))) {
                s.abort = 1;
                break;
            }
            tc_fence_after();
            // The reductions leave TMEM a lane (row) per thread. Each 32 x 32 chunk goes through a
            // per-warp 4 KB buffer in the dS^T tile (free here: the dQ MMA that read it is complete,
            // and the next item's dS^T is written only after this item releases TMEM), so that one
            // warp instruction adds 8 consecutive float4s to each of 4 rows instead of one float4 to
            // each of 32 rows. Float4 columns are XOR-swizzled by row against bank conflicts.
            float4* xb = reinterpret_cast<float4*>(s.ds) + warp * 32 * 8;  // [32 rows][8 float4]
            auto red_chunk = [&](const uint32_t (&x)[32], float* row, float mul) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    xb[lane * 8 + (e ^ (lane & 7))] =
                        make_float4(__uint_as_float(x[4 * e]) * mul, __uint_as_float(x[4 * e + 1]) * mul,
                                    __uint_as_float(x[4 * e + 2]) * mul, __uint_as_float(x[4 * e + 3]) * mul);
                __syncwarp();
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int rr = 4 * j + (lane >> 3), c4 = lane & 7;
                    float* p = reinterpret_cast<float*>(
                        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(row), rr));
                    const float4 v4 = xb[rr * 8 + (c4 ^ (rr & 7))];
                    if (p) red_add_v4(p + 4 * c4, v4.x, v4.y, v4.z, v4.w);
                }
                __syncwarp();
            };
            // dQ row tt of the item (TMEM lane = item row); warp half hf takes dQ columns 64hf..
            if (hf < D / 64) {
                const bool rv = tt < nrows;
                const int m = rv ? tt / G : 0, h = tt % G;
                float* dst = rv ? a.dq + (((size_t)b * a.N + mt.qi[m]) * a.H_q + (size_t)r * G + h) * D : nullptr;
#pragma unroll
                for (int q2 = 0; q2 < 2; ++q2) {
                    uint32_t x[32];
                    tmem_ld32(lane_addr + (hf == 0 ? 64u : 192u) + 32 * q2, x);
                    tmem_ld_wait();
                    reg_fence(x);
                    red_chunk(x, dst ? dst + 64 * hf + 32 * q2 : nullptr, a.scale);
                }
            }
            // the block's dV and dK when its last item of this CTA is done (TMEM lane = token)
            if (flush) {
                const bool tv = tt < BK && tok < a.N;
                float* dvp = tv ? a.dv + (((size_t)b * a.N + tok) * a.H_kv + r) * D : nullptr;
                float* dkp = tv ? a.dk + (((size_t)b * a.N + tok) * a.H_kv + r) * D : nullptr;
#pragma unroll
                for (int q2 = hf * (D / 64); q2 < (hf + 1) * (D / 64); ++q2) {
                    uint32_t xv[32], xk[32];
                    tmem_ld32(lane_addr + kColDV + 32 * q2, xv);
                    tmem_ld32(lane_addr + kColDK + 32 * q2, xk);
                    tmem_ld_wait();
                    reg_fence(xv);
                    reg_fence(xk);
                    red_chunk(xv, dvp ? dvp + 32 * q2 : nullptr, 1.f);
                    red_chunk(xk, dkp ? dkp + 32 * q2 : nullptr, a.scale);
                }
            }
            tc_fence_before();
            mbar_arrive(&s.t_free);
            mbar_arrive(&s.meta_empty);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// delta[b,i,h] = dO . O (one warp per row)
template <int D>
__global__ void __launch_bounds__(256) k_bwd_delta(const __nv_bfloat16* __restrict__ dout, const float* __restrict__ out,
                                                   float* __restrict__ delta, long long rows) {
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= rows) return;
    constexpr int kPer = D / 32;
    float acc = 0.f;
    const __nv_bfloat16* g = dout + w * D + lane * kPer;
    const float* o = out + w * D + lane * kPer;
#pragma unroll
    for (int x = 0; x < kPer; ++x) acc = fmaf(__bfloat162float(g[x]), o[x], acc);
#pragma unroll
    for (int s = 16; s; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) delta[w] = acc;
}

template <int D, int BK, int G>
cudaError_t launch_bwd(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                       const CUtensorMap& tv, int num_sms, cudaStream_t st) {
    const size_t smem = sizeof(BwdSmem<D, kRows / G>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_attn_bwd<D, BK, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("attn_bwd", st);
    k_attn_bwd<D, BK, G><<<num_sms, kThreads, smem, st>>>(tq, tdo, tk, tv, a);
    return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_bwd_bk(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                          const CUtensorMap& tv, int num_sms, cudaStream_t st) {
    switch (a.block_k) {
        case 128: return launch_bwd<D, 128, G>(a, tq, tdo, tk, tv, num_sms, st);
        case 64: return launch_bwd<D, 64, G>(a, tq, tdo, tk, tv, num_sms, st);
        case 32: return launch_bwd<D, 32, G>(a, tq, tdo, tk, tv, num_sms, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool bwd_supported(int d, int G) { return (d == 64 || d == 128) && (G == 8 || G == 16 || G == 32); }

cudaError_t run_attn_bwd(const BwdArgs& a, const void* q, const void* k, const void* v, const void* dout,
                         const float* out, int num_sms, cudaStream_t st) {
    const int G = a.H_q / a.H_kv;
    const size_t nq = (size_t)a.B * a.N * a.H_q * a.d, nkv = (size_t)a.B * a.N * a.H_kv * a.d;
    cudaError_t e = cudaMemsetAsync(a.dq, 0, nq * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dk, 0, nkv * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dv, 0, nkv * 4, st);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.B * a.N * a.H_q;
    {
        ProfScope ps("bwd_delta", st);
        const unsigned grid = (unsigned)((rows * 32 + 255) / 256);
        if (a.d == 128)
            k_bwd_delta<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(dout), out, a.delta, rows);
        else
            k_bwd_delta<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(dout), out, a.delta, rows);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap tq, tdo, tk, tv;
    const uint64_t dims[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2, (uint64_t)a.N * a.H_kv * a.d * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)a.block_k, 1};
    if (!make_tmap_4d(&tk, k, dims, strides, box, 128) || !make_tmap_4d(&tv, v, dims, strides, box, 128) ||
        !make_tmap_qrows(&tq, q, a.B, a.N, a.H_q, a.d, G) || !make_tmap_qrows(&tdo, dout, a.B, a.N, a.H_q, a.d, G))
        return cudaErrorInvalidValue;
    if (a.d == 128) {
        if (G == 16) return launch_bwd_bk<128, 16>(a, tq, tdo, tk, tv, num_sms, st);
        if (G == 8) return launch_bwd_bk<128, 8>(a, tq, tdo, tk, tv, num_sms, st);
        if (G == 32) return launch_bwd_bk<128, 32>(a, tq, tdo, tk, tv, num_sms, st);
    } else {
        if (G == 16) return launch_bwd_bk<64, 16>(a, tq, tdo, tk, tv, num_sms, st);
        if (G == 8) return launch_bwd_bk<64, 8>(a, tq, tdo, tk, tv, num_sms, st);
        if (G == 32) return launch_bwd_bk<64, 32>(a, tq, tdo, tk, tv, num_sms, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace msa
