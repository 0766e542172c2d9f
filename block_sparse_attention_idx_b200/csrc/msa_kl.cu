// KL alignment of the index branch to the main branch ("MSA 中的 KL 对齐与局部知识蒸馏",
// sections 2, 3 and 6): teacher P = group average of per-head softmaxes on the selected token
// set J (probability space), student P_idx = index softmax on J, loss KL(stopgrad(P) || P_idx)
// and the logit gradient P_idx - P reduced to dQ_idx and dK_idx.
//
// As on the page, probabilities are rebuilt from logits and the two log-sum-exps, so no separate
// KL-forward softmax pass exists: the main forward supplies LSE_main, and LSE_idx comes from a
// light KV-outer pass over the selected blocks (k_lse_idx) that reduces per-block sum-exps over the
// selected blocks.
//
// k_kl_kv_outer walks the same inverse lists as the attention: one item = one selected block c
// of group r plus up to 128/G queries. One tcgen05.mma computes S^T = K_c . Q_rows^T (M = 128
// tokens, N = 128 (query, head) rows, K = d) into TMEM, so one epilogue thread owns one token and
// holds the G head logits of every query of the item: the teacher's head average needs no
// cross-thread traffic. The index logits, the gradient terms and the dK_idx accumulation of that
// token run on the same thread; dQ_idx and the loss are reduced across tokens in shared memory
// into per-(query, slot) partials, which a final kernel sums in a fixed order.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kRows = 128;
constexpr float kLog2e = 1.4426950408889634f;

// ============================================================================ LSE_idx pass
// Item = one selected block c of group r and up to kIdxQpc queries; each CTA takes a contiguous
// range of items, so the block's K_idx rows stay in shared memory across the items of one list.
// The index logits of the item (128 tokens x 32 queries) come from bf16 mma.sync, warp w holding
// tokens 32w..32w+31; each warp reduces its tokens to a (max, sum-exp) pair per query and the four
// pairs are merged in a fixed order into the (query, slot) partial.
template <int DI>
__global__ void __launch_bounds__(128) k_lse_idx(KlArgs a, const __nv_bfloat16* __restrict__ q_idx,
                                                  const __nv_bfloat16* __restrict__ k_idx) {
    constexpr int QP = kIdxQpc;
    constexpr int KBP = DI + 8;  // bf16 row pitch: ldmatrix rows on distinct banks
    static_assert(QP == 32, "four query n-tiles per item");
    __shared__ alignas(16) __nv_bfloat16 kb[kRows * KBP];
    __shared__ alignas(16) __nv_bfloat16 qb[QP * KBP];
    __shared__ float red_m[4][QP], red_s[4][QP];
    __shared__ int s_i[QP], s_slot[QP];
    const Csr& cs = a.csr_idx;
    const int T = *cs.n_items;
    const int per = (T + gridDim.x - 1) / gridDim.x;
    const int t0 = blockIdx.x * per, t1 = min(T, t0 + per);
    const int tt = threadIdx.x, warp = tt >> 5, lane = tt & 31;
    const int g8 = lane >> 2, t4 = lane & 3;
    // partial slots per row: the selection's k+1, or every block of the sequence in dense mode
    // (the slot of a dense entry is its block)
    const int K1 = a.dense ? cs.nb : a.topk + 1;
    const uint32_t kb_u32 = smem_u32(kb), qb_u32 = smem_u32(qb);
    int curL = -1;
    for (int t = t0; t < t1; ++t) {
        const int4 it = cs.items[t];
        const int L = it.x, count = it.z;
        const int c = L % cs.nb, r = (L / cs.nb) % a.H_kv, b = L / (cs.nb * a.H_kv);
        __syncthreads();  // the previous item is done with kb / qb / s_i / red
        if (L != curL) {
            const int tok = c * a.block_k + tt;
            // the token's row in the held K_idx: first range, then the second one
            int lt = -1;
            if (tok >= a.kv_tok0 && tok < a.kv_tok0 + a.kv_ntok) lt = tok - a.kv_tok0;
            else if (tok >= a.kv_tok0b && tok < a.kv_tok0b + a.kv_ntokb) lt = a.kv_ntok + (tok - a.kv_tok0b);
            const bool tvalid = tt < a.block_k && tok < a.N && lt >= 0;
            const size_t held = (size_t)a.kv_ntok + a.kv_ntokb;
#pragma unroll
            for (int x = 0; x < DI / 8; ++x) {
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (tvalid) v = *reinterpret_cast<const uint4*>(k_idx + ((size_t)b * held + lt) * DI + x * 8);
                *reinterpret_cast<uint4*>(&kb[tt * KBP + x * 8]) = v;
            }
            curL = L;
        }
        if (tt < QP) {
            const int e = tt < count ? cs.entries[it.y + tt] : 0;
            s_i[tt] = tt < count ? (e >> 5) : -1;
            s_slot[tt] = a.dense ? c : (e & 31);
        }
        for (int x = tt; x < QP * (DI / 8); x += 128) {
            const int m = x / (DI / 8), part = x % (DI / 8);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (m < count) {
                const int qi = cs.entries[it.y + m] >> 5;
                v = *reinterpret_cast<const uint4*>(q_idx + (((size_t)b * a.N + qi) * a.H_kv + r) * DI + part * 8);
            }
            *reinterpret_cast<uint4*>(&qb[m * KBP + part * 8]) = v;
        }
        __syncthreads();
        float acc[2][4][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int x = 0; x < 4; ++x) acc[mt][nt][x] = 0.f;
#pragma unroll
        for (int ks = 0; ks < DI / 16; ++ks) {
            uint32_t af[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const uint32_t ad = kb_u32 + ((warp * 32 + mt * 16 + (lane & 15)) * KBP + ks * 16 + (lane >> 4) * 8) * 2;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(af[mt][0]), "=r"(af[mt][1]), "=r"(af[mt][2]), "=r"(af[mt][3])
                             : "r"(ad));
            }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t bf[4];
                const uint32_t ad =
                    qb_u32 + ((np * 16 + (lane & 7) + ((lane >> 4) << 3)) * KBP + ks * 16 + ((lane >> 3) & 1) * 8) * 2;
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(bf[0]), "=r"(bf[1]), "=r"(bf[2]), "=r"(bf[3])
                             : "r"(ad));
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    mma_16816_bf16(acc[mt][2 * np], af[mt], bf[0], bf[1]);
                    mma_16816_bf16(acc[mt][2 * np + 1], af[mt], bf[2], bf[3]);
                }
            }
        }
        // per query: the warp's (max, sum-exp) over its 32 tokens
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int cx = 0; cx < 2; ++cx) {
                const int m = nt * 8 + 2 * t4 + cx;
                const int qi = s_i[m];
                float v[4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int hx = 0; hx < 2; ++hx) {
                        const int row = warp * 32 + mt * 16 + g8 + 8 * hx;
                        const int tok = c * a.block_k + row;
                        const bool ok = m < count && row < a.block_k && tok < a.N && tok <= qi;
                        v[mt * 2 + hx] = ok ? acc[mt][nt][2 * hx + cx] * a.scale_idx : -INFINITY;
                    }
                float mx = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                float z = 0.f;
                if (mx != -INFINITY) {
#pragma unroll
                    for (int u = 0; u < 4; ++u) z += v[u] == -INFINITY ? 0.f : __expf(v[u] - mx);
                }
#pragma unroll
                for (int o = 4; o < 32; o <<= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
                if (g8 == 0) {
                    red_m[warp][m] = mx;
                    red_s[warp][m] = z;
                }
            }
        __syncthreads();
        if (tt < count) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w][tt]);
            float Z = 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (red_m[w][tt] != -INFINITY) Z += red_s[w][tt] * __expf(red_m[w][tt] - M);
            a.ml_part[(((size_t)b * a.N + s_i[tt]) * a.H_kv + r) * K1 + s_slot[tt]] = make_float2(M, Z);
        }
    }
}

// One thread per (b, i, r): LSE_idx = merge of the per-slot (max, sum-exp) pairs.
__global__ void k_lse_idx_merge(KlArgs a) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= (long long)a.B * a.N * a.H_kv) return;
    const int i = (int)((row / a.H_kv) % a.N);
    if (a.dense) {
        // every causal block 0 .. i / block_k, slot = block
        const int nb = a.csr_idx.nb, nc = i / a.block_k + 1;
        const float2* mp = a.ml_part + row * nb;
        float mx = -INFINITY;
        for (int c = 0; c < nc; ++c) mx = fmaxf(mx, mp[c].x);
        float z = 0.f;
        for (int c = 0; c < nc; ++c) z += mp[c].y * __expf(mp[c].x - mx);
        a.lse_idx[row] = mx + logf(z);
        return;
    }
    const int K1 = a.topk + 1;
    const int32_t* sel = a.blocks + row * K1;
    float mx = -INFINITY;
    int prev = -1;
    for (int s = 0; s < K1; ++s) {
        const int c = sel[s];
        if (c < 0 || c > i / a.block_k || c <= prev) continue;
        prev = c;
        mx = fmaxf(mx, a.ml_part[row * K1 + s].x);
    }
    float z = 0.f;
    prev = -1;
    for (int s = 0; s < K1; ++s) {
        const int c = sel[s];
        if (c < 0 || c > i / a.block_k || c <= prev) continue;
        prev = c;
        const float2 ml = a.ml_part[row * K1 + s];
        z += ml.y * __expf(ml.x - mx);
    }
    if (a.ml_out) a.ml_out[row] = make_float2(mx, z);
    else a.lse_idx[row] = mx + logf(z);
}

// ============================================================================ KL kernel
// tf32 operand (round to nearest) of a float; bf16 values are exact in tf32.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ uint32_t bf16_as_tf32(__nv_bfloat16 x) {
    return (uint32_t)(*reinterpret_cast<const uint16_t*>(&x)) << 16;
}
// D += A(16x8, tf32, row) * B(8x8, tf32, col), fp32 accumulate.
__device__ __forceinline__ void mma_1688_tf32(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four (or two) 8x8 b16 matrices from shared memory, not transposed.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// 4-, 8- or 16-byte asynchronous copy global -> shared.
template <int BYTES>
__device__ __forceinline__ void cp_async_ca(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(src), "n"(BYTES) : "memory");
}
// One arrival on `bar` once every cp.async this thread issued so far has landed (counted in the
// barrier's expected arrivals).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// D += A(16x8, bf16, row) * B(8x8, bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_1688_bf16(float (&c)[4], const uint32_t (&a)[2], uint32_t b) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%0,%1,%2,%3};"
                 : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                 : "r"(a[0]), "r"(a[1]), "r"(b));
}
// x ~= hi + lo with both parts tf32: products with a tf32-exact operand keep ~fp32 accuracy.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = to_tf32(x);
    lo = to_tf32(x - __uint_as_float(hi));
}

// Epilogue teams: with G >= 8 (8 or 16 queries per item) two teams of four warps take alternate
// items, so that one team's mma and reduction work overlaps the other's exponentials.
template <int G>
__host__ __device__ constexpr int kl_teams() { return G >= 8 ? 2 : 1; }
// Producer warps: with G >= 8 one warp issues the Q and K tiles and another the item metadata, so
// that the two sets of copies are issued side by side.
template <int G>
__host__ __device__ constexpr int kl_prods() { return G >= 8 ? 2 : 1; }
template <int G>
__host__ __device__ constexpr int kl_threads() { return (4 * kl_teams<G>() + kl_prods<G>() + 1) * 32; }
// Item metadata stages (Q_idx rows, LSE values, query ids): the Q tile itself has two stages that
// the MMA releases, the metadata more, released by the epilogue, so loads run ahead of it.
template <int G>
__host__ __device__ constexpr int kl_meta_stages() { return G >= 8 ? 4 : 2; }

// Row pitches keep the mma fragment loads of a warp on distinct banks (or at most two-way) and the
// per-token row writes conflict-free.
template <int D, int DI, int QPC, int TEAMS, int NMETA, int PRODS>
struct KlSmem {
    static constexpr int KBP = DI + 8;   // K_idx / Q_idx bf16 rows
    static constexpr int GSP = QPC + 1;  // gradient rows [token][query]
    static constexpr int SIP = QPC + 1;  // index log-probability / KL rows [token][query]
    alignas(1024) uint8_t q[2][kRows * D * 2];
    alignas(1024) uint8_t k[kRows * D * 2];             // 128 token rows (rows >= block_k unused)
    alignas(16) __nv_bfloat16 kb[TEAMS][kRows * KBP];   // K_idx rows of each team's block (zero past the end)
    alignas(16) __nv_bfloat16 qb[NMETA][QPC * KBP];     // Q_idx rows of the item queries
    alignas(16) float lse[NMETA][kRows];                // LSE_main of the item rows (query-major, head-minor)
    // g * scale_idx per (token, query): fp32 for the tf32 gradient products (items of more than 16
    // queries), or split as bf16 hi + lo in [token][query] and [query][token] order for the bf16 ones
    static constexpr bool kBf = QPC <= 16;
    static constexpr int GBP = kRows + 8;
    float gs[TEAMS][kBf ? 1 : kRows * GSP];
    alignas(16) __nv_bfloat16 ga[TEAMS][2][kBf ? kRows * QPC : 8];
    alignas(16) __nv_bfloat16 gb[TEAMS][2][kBf ? QPC * GBP : 8];
    float sidx[TEAMS][kRows * SIP];                     // log P_idx per (token, query), then the KL terms
    float lidx[NMETA][QPC];                             // LSE_idx of the item queries
    int ent[NMETA][QPC];                                // query entries (i << 5 | slot) of the item
    int4 rec[NMETA];                                    // item record (L, first entry, count, -)
    int4 crec[PRODS][2][32];                            // per producer warp: item records of the current /
    int cent[PRODS][2][32][QPC];                        // next chunk of 32 items and their query entries
    uint64_t q_full[2], q_empty[2], meta_full[NMETA], meta_empty[NMETA];
    uint64_t kv_full, kv_empty, s_full[4], s_free[4], drain;
    uint32_t tmem_base;
    int abort;
};

template <int D, int DI, int G>
__global__ void __launch_bounds__(kl_threads<G>(), 1)
    k_kl_kv_outer(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ q_idx,
                  const __nv_bfloat16* __restrict__ k_idx, KlArgs a) {
    constexpr int QPC = kRows / G;
    constexpr int TEAMS = kl_teams<G>();
    constexpr int NMETA = kl_meta_stages<G>();
    constexpr int PRODS = kl_prods<G>();
    constexpr int kProdWarp = 4 * TEAMS, kMmaWarp = 4 * TEAMS + PRODS;
    using Sm = KlSmem<D, DI, QPC, TEAMS, NMETA, PRODS>;
    constexpr int KBP = Sm::KBP, GSP = Sm::GSP, SIP = Sm::SIP;
    extern __shared__ uint8_t smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kIdesc = umma_idesc_bf16(kRows, kRows, false, false);
    static_assert(QPC % 8 == 0 && QPC <= 64, "KL items hold 8 to 64 queries");
    static_assert(DI % 16 == 0, "index head dim must be a multiple of 16");
    static_assert(G % 2 == 0, "heads are processed in pairs");
    // S^T buffers in TMEM, 128 columns each: one per epilogue team with two teams.
    constexpr int kSBuf = 2;

    const int K1 = a.topk + 1;
    const int BK = a.block_k;
    const float coef = a.grad_scale / ((float)a.B * (float)a.N * (float)a.H_kv);
    const Csr& cs = a.csr;
    const int T = *cs.n_items;
    const int per = (T + gridDim.x - 1) / gridDim.x;
    const int t0 = blockIdx.x * per, t1 = min(T, t0 + per);
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s.q_full[x], 1);
            mbar_init(&s.q_empty[x], 1);
        }
        for (int x = 0; x < kSBuf; ++x) {
            mbar_init(&s.s_full[x], 1);
            mbar_init(&s.s_free[x], kRows);
        }
        for (int x = 0; x < NMETA; ++x) {
            mbar_init(&s.meta_full[x], 32);
            mbar_init(&s.meta_empty[x], kRows);
        }
        mbar_init(&s.kv_full, 1);
        mbar_init(&s.kv_empty, 1);
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp < 4) {
        // Q_idx rows past an item's count are read by the gradient mma (times a zero gradient), so
        // they must hold finite values: start from zeros.
        uint32_t* z = reinterpret_cast<uint32_t*>(s.qb);
        for (int x = threadIdx.x; x < NMETA * QPC * KBP / 2; x += kRows) z[x] = 0u;
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&s.tmem_base, 128 * kSBuf);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp >= kProdWarp && warp < kProdWarp + PRODS) {
        // ---------------------------------------------------------------- loads + item records
        // Item records and query entries come in chunks of 32 items, one per lane: the next chunk's
        // records are loaded at item 0 of a chunk, their entries at item 8, and both are stored to
        // the warp's shared ring at item 16, so no global load latency sits on the per-item path.
        // Everything an item's consumers read arrives by cp.async (metadata, counted by one arrival
        // per lane once its copies land) or by TMA (Q and K tiles, relaxed arrives): no release arrive
        // here, which would wait for this warp's copies still in flight.
        const int pw = warp - kProdWarp;
        const bool do_meta = PRODS == 1 || pw == 1, do_q = PRODS == 1 || pw == 0;
        constexpr int CH = 32;
        int4 (*crec)[32] = s.crec[pw];
        int (*cent)[32][QPC] = s.cent[pw];
        int kv_loads = 0, prevL = -1, issued = 0;
        bool ok = true;
        int4 r_next = make_int4(-1, 0, 0, 0);
        int e_next[QPC];
        {
            const int4 rr = t0 + lane < t1 ? cs.items[t0 + lane] : make_int4(-1, 0, 0, 0);
            crec[0][lane] = rr;
#pragma unroll
            for (int x = 0; x < QPC; ++x) cent[0][lane][x] = x < rr.z ? cs.entries[rr.y + x] : 0;
            __syncwarp();
        }
        for (int t = t0, n = 0; t < t1; ++t, ++n) {
            const int j = n % CH, cb = (n / CH) & 1;
            const int4 itm = crec[cb][j];
            const int L = itm.x, count = itm.z;
            const int c = L % cs.nb, r = (L / cs.nb) % a.H_kv, b = L / (cs.nb * a.H_kv);
            const int* qe = cent[cb][j];
            const int ms = n % NMETA, buf = n & 1;
            int okl = 1;
            if (do_meta) {
                if (lane == 0) okl = mbar_wait(&s.meta_empty[ms], ((n / NMETA) & 1) ^ 1, a.status, 0x801);
                if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
                // item record, query entries, LSE_idx of each query, LSE_main of its G heads, its Q_idx row
                if (lane == 0) cp_async_ca<16>(smem_u32(&s.rec[ms]), cs.items + t);
                for (int m = lane; m < count; m += 32) {
                    cp_async_ca<4>(smem_u32(&s.ent[ms][m]), cs.entries + itm.y + m);
                    cp_async_ca<4>(smem_u32(&s.lidx[ms][m]),
                                   a.lse_idx + ((size_t)b * a.N + (qe[m] >> 5)) * a.H_kv + r);
                }
                constexpr int LB = G * 4 >= 16 ? 16 : G * 4;  // bytes per copy of one query's LSE_main
                constexpr int LPQ = G * 4 / LB;
                for (int x = lane; x < count * LPQ; x += 32) {
                    const int m = x / LPQ, part = x % LPQ;
                    const float* src =
                        a.lse + ((size_t)b * a.N + (qe[m] >> 5)) * a.H_q + (size_t)r * G + part * (LB / 4);
                    cp_async_ca<LB>(smem_u32(&s.lse[ms][m * G + part * (LB / 4)]), src);
                }
                constexpr int QIC = DI / 8;  // 16-byte chunks per Q_idx row
                for (int x = lane; x < count * QIC; x += 32) {
                    const int m = x / QIC, part = x % QIC;
                    const __nv_bfloat16* src =
                        q_idx + (((size_t)b * a.N + (qe[m] >> 5)) * a.H_kv + r) * DI + part * 8;
                    cp_async_ca<16>(smem_u32(&s.qb[ms][m * KBP + part * 8]), src);
                }
                cp_async_arrive_noinc(&s.meta_full[ms]);
            }
            if (do_q) {
                // Q: the G head rows of each query, in the 128B-swizzled K-major tile the MMA reads
                if (lane == 0) okl = mbar_wait(&s.q_empty[buf], ((n >> 1) & 1) ^ 1, a.status, 0x805);
                if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
                if constexpr (G % 8 == 0) {
                    if (lane == 0) mbar_arrive_expect_tx_relaxed(&s.q_full[buf], (uint32_t)(count * G * D * 2));
                    __syncwarp();
                    for (int m = lane; m < count; m += 32)
                        tma_load_5d(s.q[buf] + m * G * D * 2, &tm_q, &s.q_full[buf], 0, 0, 0, r * G / 8,
                                    b * a.N + (qe[m] >> 5));
                } else {
                    const uint32_t qs = smem_u32(s.q[buf]);
                    constexpr int kChunksPerRow = D * 2 / 16;
                    for (int x = lane; x < count * G * kChunksPerRow; x += 32) {
                        const int row = x / kChunksPerRow, ch = x % kChunksPerRow;
                        const int m = row / G, h = row % G;
                        const __nv_bfloat16* src =
                            q + ((((size_t)b * a.N + (qe[m] >> 5)) * a.H_q + (size_t)r * G + h) * D + ch * 8);
                        cp_async_16(qs + qtile_off<D>(row, ch * 16), src);
                    }
                    cp_async_wait_all();
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&s.q_full[buf]);
                }
                // K tile of a new (block, group); the MMA releases the previous one when it reaches
                // the first item of this one
                if (L != prevL) {
                    if (lane == 0) {
                        if (kv_loads > 0) okl = mbar_wait(&s.kv_empty, (kv_loads - 1) & 1, a.status, 0x802);
                        if (okl) {
                            mbar_arrive_expect_tx_relaxed(&s.kv_full, (D / 64) * BK * 128);
#pragma unroll
                            for (int sub = 0; sub < D / 64; ++sub)
                                tma_load_4d(s.k + sub * kRows * 128, &tm_k, &s.kv_full, sub * 64, r, c * BK, b);
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, okl, 0)) { ok = false; break; }
                    ++kv_loads;
                    prevL = L;
                }
            }
            ++issued;
            // next chunk of item records and entries
            if (j == 0) r_next = t + CH + lane < t1 ? cs.items[t + CH + lane] : make_int4(-1, 0, 0, 0);
            if (j == 8) {
#pragma unroll
                for (int x = 0; x < QPC; ++x) e_next[x] = x < r_next.z ? cs.entries[r_next.y + x] : 0;
            }
            if (j == 16) {
                crec[cb ^ 1][lane] = r_next;
#pragma unroll
                for (int x = 0; x < QPC; ++x) cent[cb ^ 1][lane][x] = e_next[x];
                __syncwarp();
            }
        }
        if (!ok) s.abort = 1;
        // nothing may still be landing in shared memory when the CTA exits
        cp_async_wait_all();
        if (lane == 0) {
            if (do_q) {
                for (int x = 0; x < 2 && x < issued; ++x) {
                    const int nl = issued - 1 - x;  // last use of buffer nl & 1
                    mbar_wait(&s.q_full[nl & 1], (nl >> 1) & 1, a.status, 0x803);
                }
                if (kv_loads > 0) mbar_wait(&s.kv_full, (kv_loads - 1) & 1, a.status, 0x804);
            }
            if (do_meta) {
                for (int x = 0; x < NMETA && x < issued; ++x) {
                    const int nl = issued - 1 - x;  // last use of metadata stage nl % NMETA
                    mbar_wait(&s.meta_full[nl % NMETA], (nl / NMETA) & 1, a.status, 0x806);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------------- MMA issuer: S^T = K Q^T
        if (lane == 0) {
            bool ok = true;
            int kv_group = -1, prevL = -1;
            for (int t = t0, n = 0; t < t1; ++t, ++n) {
                const int buf = n & 1, sb = n % kSBuf, ms = n % NMETA;
                if (!mbar_wait(&s.meta_full[ms], (n / NMETA) & 1, a.status, 0x905)) { ok = false; break; }
                const int L = s.rec[ms].x;
                if (!mbar_wait(&s.q_full[buf], (n >> 1) & 1, a.status, 0x901)) { ok = false; break; }
                if (L != prevL) {
                    if (kv_group >= 0) umma_commit(&s.kv_empty);  // previous K tile no longer read
                    ++kv_group;
                    prevL = L;
                    if (!mbar_wait(&s.kv_full, kv_group & 1, a.status, 0x902)) { ok = false; break; }
                }
                if (!mbar_wait(&s.s_free[sb], ((n / kSBuf) & 1) ^ 1, a.status, 0x903)) { ok = false; break; }
                tc_fence_after();
                const uint32_t qa = smem_u32(s.q[buf]), ka = smem_u32(s.k);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t sub = (ks * 16) / 64, off = (ks & 3) * 32;
                    const uint64_t da = umma_sdesc(ka + sub * (kRows * 128) + off, 16, 1024, 2);
                    const uint64_t db = umma_sdesc(qa + sub * 1024 + off, 16, (D / 64) * 1024, 2);
                    umma_bf16(tmem + sb * kRows, da, db, kIdesc, ks > 0);
                }
                umma_commit(&s.s_full[sb]);
                umma_commit(&s.q_empty[buf]);
            }
            if (!ok) s.abort = 1;
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, a.status, 0x904);
        }
    } else {
        // ---------------------------------------------------------------- epilogue: thread = token
        // Team `team` takes the CTA's items team, team + TEAMS, ...; its warp wq owns tokens
        // 32wq..32wq+31 of the block (TMEM lane quarter wq). Control flow stays uniform across the
        // team's 128 threads (named barrier per team): a failed wait sets the CTA abort flag and
        // every thread then skips the work but not the barriers.
        const int team = warp / 4, wq = warp % 4;
        const int tt = wq * 32 + lane;
        const int g8 = lane >> 2, t4 = lane & 3;
        const uint32_t lane_addr = tmem + ((uint32_t)(wq * 32) << 16);
        const uint64_t sl2x2 = f2_packf(a.scale * kLog2e, a.scale * kLog2e);
        __nv_bfloat16* kbt = s.kb[team];
        float* gst = s.gs[team];
        float* sit = s.sidx[team];
        const uint32_t kb_u32 = smem_u32(kbt);
        constexpr int NDT = DI / 8;  // dK n-tiles
        float dk[2][NDT][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < NDT; ++nt)
#pragma unroll
                for (int x = 0; x < 4; ++x) dk[mt][nt][x] = 0.f;
        int myL = -1, prev_b = 0, prev_c = 0;
        auto team_bar = [&]() { asm volatile("bar.sync %0, 128;" ::"r"(1 + team) : "memory"); };

        auto flush_dk = [&]() {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int hx = 0; hx < 2; ++hx) {
                    const int row = wq * 32 + mt * 16 + g8 + hx * 8;
                    const int tok = prev_c * BK + row;
                    if (row < BK && tok < a.N) {
                        float* dst = a.dk_idx + ((size_t)prev_b * a.N + tok) * DI + 2 * t4;
#pragma unroll
                        for (int nt = 0; nt < NDT; ++nt)
                            atomicAdd(reinterpret_cast<float2*>(dst + nt * 8),
                                      make_float2(dk[mt][nt][2 * hx], dk[mt][nt][2 * hx + 1]));
                    }
                }
        };

        for (int t = t0 + team, n = team; t < t1; t += TEAMS, n += TEAMS) {
            const int buf = n % NMETA, sb = n % kSBuf;
            team_bar();  // (A) the team's previous item is done with gs / sidx / kb
            bool ok = s.abort == 0;
            if (ok) ok = mbar_wait(&s.meta_full[buf], (n / NMETA) & 1, a.status, 0xa01);
            ok = __all_sync(0xffffffffu, ok);
            const int4 rec = s.rec[buf];
            const int L = rec.x, count = rec.z;
            const int c = L % cs.nb, r = (L / cs.nb) % a.H_kv, b = L / (cs.nb * a.H_kv);
            const int tok = c * BK + tt;
            const bool tvalid = tt < BK && tok < a.N;
            if (ok && L != myL) {
                // new K block for this team: flush dK_idx, load this token's K_idx row (zeros past the end)
                if (myL >= 0) flush_dk();
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NDT; ++nt)
#pragma unroll
                        for (int x = 0; x < 4; ++x) dk[mt][nt][x] = 0.f;
#pragma unroll
                for (int x = 0; x < DI / 8; ++x) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (tvalid) v = *reinterpret_cast<const uint4*>(k_idx + ((size_t)b * a.N + tok) * DI + x * 8);
                    *reinterpret_cast<uint4*>(&kbt[tt * KBP + x * 8]) = v;
                }
                myL = L;
                prev_b = b;
                prev_c = c;
                __syncwarp();
            }
            if (ok) {
                // index log-probabilities log P_idx = S_idx scale_idx - LSE_idx for the warp's 32 tokens
                const uint32_t qb_u32 = smem_u32(s.qb[buf]);
                float acc[2][QPC / 8][4];
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int nt = 0; nt < QPC / 8; ++nt)
#pragma unroll
                        for (int x = 0; x < 4; ++x) acc[mt][nt][x] = 0.f;
#pragma unroll
                for (int ks = 0; ks < DI / 16; ++ks) {
                    uint32_t af[2][4];
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
                        ldsm_x4(kb_u32 + ((wq * 32 + mt * 16 + (lane & 15)) * KBP + ks * 16 + (lane >> 4) * 8) * 2,
                                af[mt]);
#pragma unroll
                    for (int nt = 0; nt < QPC / 8; ++nt) {
                        uint32_t b0, b1;
                        ldsm_x2(qb_u32 + ((nt * 8 + (lane & 7)) * KBP + ks * 16 + ((lane >> 3) & 1) * 8) * 2, b0, b1);
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) mma_16816_bf16(acc[mt][nt], af[mt], b0, b1);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < QPC / 8; ++nt) {
                    const int m0 = nt * 8 + 2 * t4;
                    const float l0 = s.lidx[buf][m0], l1 = s.lidx[buf][m0 + 1];
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                        for (int hx = 0; hx < 2; ++hx) {
                            const int row = wq * 32 + mt * 16 + g8 + hx * 8;
                            sit[row * SIP + m0] = fmaf(acc[mt][nt][2 * hx], a.scale_idx, -l0);
                            sit[row * SIP + m0 + 1] = fmaf(acc[mt][nt][2 * hx + 1], a.scale_idx, -l1);
                        }
                }
                __syncwarp();
            }
            if (ok) {
                // LSE_main of the item's rows, pre-scaled once: exp(S scale - LSE) = 2^(S sl2 + lse')
                s.lse[buf][tt] *= -kLog2e;
            }
            team_bar();  // the scaled LSE_main values of the whole item are in place
            if (ok) ok = mbar_wait(&s.s_full[sb], (n / kSBuf) & 1, a.status, 0xa02);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) s.abort = 1;
            if (ok) {
                // teacher P = mean over the G heads of exp(S scale - LSE_main); gradient and KL terms
                tc_fence_after();
                constexpr int QC = 32 / G > 0 ? 32 / G : 1;  // queries per 32-column TMEM chunk
                constexpr int CW = QC * G;                    // columns per chunk
                constexpr int NCH = QPC / QC;
                static_assert(G % 4 == 0 || G == 2, "LSE_main rows are read four or two at a time");
                // the next chunk's TMEM load is in flight while the current one is processed
                uint32_t sv[2][CW];
                alignas(16) __nv_bfloat16 gha[Sm::kBf ? QPC : 8], gla[Sm::kBf ? QPC : 8];
                tmem_ld<CW>(lane_addr + sb * kRows, sv[0]);
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) {
                    tmem_ld_wait();
                    reg_fence(sv[ch & 1]);
                    if (ch + 1 < NCH) {
                        tmem_ld<CW>(lane_addr + sb * kRows + (ch + 1) * CW, sv[(ch + 1) & 1]);
                    } else {
                        tc_fence_before();
                        mbar_arrive(&s.s_free[sb]);
                    }
                    const uint32_t* cv = sv[ch & 1];
#pragma unroll
                    for (int qq = 0; qq < QC; ++qq) {
                        const int m = ch * QC + qq;
                        uint64_t pacc = f2_packf(0.f, 0.f);
                        if constexpr (G % 4 == 0) {
                            const float4* l4 = reinterpret_cast<const float4*>(&s.lse[buf][m * G]);
#pragma unroll
                            for (int hq = 0; hq < G / 4; ++hq) {
                                const float4 lv = l4[hq];
                                const uint64_t x0 =
                                    f2_fma(f2_pack(cv[qq * G + 4 * hq], cv[qq * G + 4 * hq + 1]), sl2x2, f2_packf(lv.x, lv.y));
                                const uint64_t x1 = f2_fma(f2_pack(cv[qq * G + 4 * hq + 2], cv[qq * G + 4 * hq + 3]), sl2x2,
                                                           f2_packf(lv.z, lv.w));
                                float e0, e1, e2, e3;
                                f2_unpack(x0, e0, e1);
                                f2_unpack(x1, e2, e3);
                                pacc = f2_add(pacc, f2_packf(fast_exp2(e0), fast_exp2(e1)));
                                pacc = f2_add(pacc, f2_packf(fast_exp2(e2), fast_exp2(e3)));
                            }
                        } else {
                            const float2 lv = *reinterpret_cast<const float2*>(&s.lse[buf][m * G]);
                            const uint64_t x0 = f2_fma(f2_pack(cv[qq * G], cv[qq * G + 1]), sl2x2, f2_packf(lv.x, lv.y));
                            float e0, e1;
                            f2_unpack(x0, e0, e1);
                            pacc = f2_packf(fast_exp2(e0), fast_exp2(e1));
                        }
                        float p0, p1;
                        f2_unpack(pacc, p0, p1);
                        const float P = (p0 + p1) * (1.f / (float)G);
                        const bool valid = m < count && tvalid && tok <= (s.ent[buf][m] >> 5);
                        const float lp = sit[tt * SIP + m];
                        const float gval = coef * (__expf(lp) - P) * a.scale_idx;
                        const float klv = P > 0.f ? P * (__logf(P) - lp) : 0.f;
                        const float gv = valid ? gval : 0.f;
                        if constexpr (Sm::kBf) {
                            const __nv_bfloat16 hi = __float2bfloat16_rn(gv);
                            const __nv_bfloat16 lo = __float2bfloat16_rn(gv - __bfloat162float(hi));
                            gha[m] = hi;
                            gla[m] = lo;
                            s.gb[team][0][m * Sm::GBP + tt] = hi;
                            s.gb[team][1][m * Sm::GBP + tt] = lo;
                        } else {
                            gst[tt * GSP + m] = gv;
                        }
                        sit[tt * SIP + m] = valid ? klv : 0.f;
                    }
                }
                if constexpr (Sm::kBf) {
#pragma unroll
                    for (int x = 0; x < QPC; x += 8) {
                        *reinterpret_cast<uint4*>(&s.ga[team][0][tt * QPC + x]) = *reinterpret_cast<const uint4*>(&gha[x]);
                        *reinterpret_cast<uint4*>(&s.ga[team][1][tt * QPC + x]) = *reinterpret_cast<const uint4*>(&gla[x]);
                    }
                }
                __syncwarp();
                // dK_idx[token] += sum_q g(token, q) scale_idx Q_idx[q]: bf16 mma, gradient split in hi + lo
                if constexpr (Sm::kBf) {
                    const uint32_t ga_hi = smem_u32(s.ga[team][0]), ga_lo = smem_u32(s.ga[team][1]);
                    const uint32_t qbu = smem_u32(s.qb[buf]);
#pragma unroll
                    for (int kq = 0; kq < QPC / 8; ++kq) {
                        uint32_t ah[2][2], al[2][2];
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            const uint32_t off = ((wq * 32 + mt * 16 + (lane & 15)) * QPC + kq * 8) * 2;
                            ldsm_x2(ga_hi + off, ah[mt][0], ah[mt][1]);
                            ldsm_x2(ga_lo + off, al[mt][0], al[mt][1]);
                        }
#pragma unroll
                        for (int j = 0; j < NDT / 4; ++j) {
                            uint32_t bq[4];
                            ldsm_x4_trans(qbu + ((kq * 8 + (lane & 7)) * KBP + (j * 4 + (lane >> 3)) * 8) * 2, bq[0], bq[1],
                                          bq[2], bq[3]);
#pragma unroll
                            for (int u = 0; u < 4; ++u)
#pragma unroll
                                for (int mt = 0; mt < 2; ++mt) {
                                    mma_1688_bf16(dk[mt][j * 4 + u], ah[mt], bq[u]);
                                    mma_1688_bf16(dk[mt][j * 4 + u], al[mt], bq[u]);
                                }
                        }
                    }
                } else
#pragma unroll
                for (int kq = 0; kq < QPC / 8; ++kq) {
                    uint32_t ah[2][4], al[2][4];
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        const int row = wq * 32 + mt * 16 + g8;
                        split_tf32(gst[row * GSP + kq * 8 + t4], ah[mt][0], al[mt][0]);
                        split_tf32(gst[(row + 8) * GSP + kq * 8 + t4], ah[mt][1], al[mt][1]);
                        split_tf32(gst[row * GSP + kq * 8 + t4 + 4], ah[mt][2], al[mt][2]);
                        split_tf32(gst[(row + 8) * GSP + kq * 8 + t4 + 4], ah[mt][3], al[mt][3]);
                    }
#pragma unroll
                    for (int nt = 0; nt < NDT; ++nt) {
                        const uint32_t b0 = bf16_as_tf32(s.qb[buf][(kq * 8 + t4) * KBP + nt * 8 + g8]);
                        const uint32_t b1 = bf16_as_tf32(s.qb[buf][(kq * 8 + t4 + 4) * KBP + nt * 8 + g8]);
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            mma_1688_tf32(dk[mt][nt], ah[mt][0], ah[mt][1], ah[mt][2], ah[mt][3], b0, b1);
                            mma_1688_tf32(dk[mt][nt], al[mt][0], al[mt][1], al[mt][2], al[mt][3], b0, b1);
                        }
                    }
                }
            }
            team_bar();  // (B) gradients and KL terms of all 128 tokens are in shared memory
            if (ok) {
                // dQ_idx^T[d][q] = sum_token K_idx[token][d] g(token, q) scale_idx: (d, q) tiles over
                // the team's warps, four independent accumulator chains summed at the end
                constexpr int MT = DI / 16, NT = QPC / 8;
                if constexpr (Sm::kBf) {
                    // K_idx^T fragments by transposed ldmatrix of the token-major tile, the gradient's
                    // (query, token) hi and lo rows by ldmatrix; hi and lo in separate accumulators
                    const uint32_t kbu = smem_u32(kbt);
                    for (int x = wq; x < MT * NT; x += 4) {
                        const int mt = x % MT, nt = x / MT;
                        float ch[4] = {0.f, 0.f, 0.f, 0.f}, cl[4] = {0.f, 0.f, 0.f, 0.f};
                        const uint32_t gsrc = smem_u32(s.gb[team][lane >> 4]);
#pragma unroll
                        for (int ks = 0; ks < kRows / 16; ++ks) {
                            uint32_t af[4], bg[4];
                            ldsm_x4_trans(kbu + ((ks * 16 + (lane & 7) + ((lane >> 4) << 3)) * KBP + mt * 16 +
                                                 ((lane >> 3) & 1) * 8) * 2,
                                          af[0], af[1], af[2], af[3]);
                            ldsm_x4(gsrc + ((nt * 8 + (lane & 7)) * Sm::GBP + ks * 16 + ((lane >> 3) & 1) * 8) * 2, bg);
                            mma_16816_bf16(ch, af, bg[0], bg[1]);
                            mma_16816_bf16(cl, af, bg[2], bg[3]);
                        }
                        const int d0 = mt * 16 + g8;
#pragma unroll
                        for (int cx = 0; cx < 2; ++cx) {
                            const int m = nt * 8 + 2 * t4 + cx;
                            if (m < count) {
                                const int qe = s.ent[buf][m];
                                const size_t row = ((size_t)b * a.N + (qe >> 5)) * a.H_kv + r;
                                if (a.dense) {
                                    atomicAdd(a.dq_idx + row * DI + d0, ch[cx] + cl[cx]);
                                    atomicAdd(a.dq_idx + row * DI + d0 + 8, ch[2 + cx] + cl[2 + cx]);
                                } else {
                                    const size_t pr = row * K1 + (qe & 31);
                                    a.dq_part[pr * DI + d0] = ch[cx] + cl[cx];
                                    a.dq_part[pr * DI + d0 + 8] = ch[2 + cx] + cl[2 + cx];
                                }
                            }
                        }
                    }
                } else
                for (int x = wq; x < MT * NT; x += 4) {
                    const int mt = x % MT, nt = x / MT;
                    float cq[4][4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int v = 0; v < 4; ++v) cq[u][v] = 0.f;
#pragma unroll
                    for (int ks = 0; ks < kRows / 8; ++ks) {
                        const __nv_bfloat16* k0 = &kbt[(ks * 8 + t4) * KBP + mt * 16 + g8];
                        const __nv_bfloat16* k1 = k0 + 4 * KBP;
                        uint32_t bh0, bl0, bh1, bl1;
                        split_tf32(gst[(ks * 8 + t4) * GSP + nt * 8 + g8], bh0, bl0);
                        split_tf32(gst[(ks * 8 + t4 + 4) * GSP + nt * 8 + g8], bh1, bl1);
                        const uint32_t a0 = bf16_as_tf32(k0[0]), a1 = bf16_as_tf32(k0[8]);
                        const uint32_t a2 = bf16_as_tf32(k1[0]), a3 = bf16_as_tf32(k1[8]);
                        mma_1688_tf32(cq[(ks & 1) * 2], a0, a1, a2, a3, bh0, bh1);
                        mma_1688_tf32(cq[(ks & 1) * 2 + 1], a0, a1, a2, a3, bl0, bl1);
                    }
                    const int d0 = mt * 16 + g8;
#pragma unroll
                    for (int cx = 0; cx < 2; ++cx) {
                        const int m = nt * 8 + 2 * t4 + cx;
                        if (m < count) {
                            const int qe = s.ent[buf][m];
                            const size_t row = ((size_t)b * a.N + (qe >> 5)) * a.H_kv + r;
                            const float v0 = (cq[0][cx] + cq[1][cx]) + (cq[2][cx] + cq[3][cx]);
                            const float v1 = (cq[0][2 + cx] + cq[1][2 + cx]) + (cq[2][2 + cx] + cq[3][2 + cx]);
                            if (a.dense) {
                                atomicAdd(a.dq_idx + row * DI + d0, v0);
                                atomicAdd(a.dq_idx + row * DI + d0 + 8, v1);
                            } else {
                                const size_t pr = row * K1 + (qe & 31);
                                a.dq_part[pr * DI + d0] = v0;
                                a.dq_part[pr * DI + d0 + 8] = v1;
                            }
                        }
                    }
                }
                // KL of each (query, slot): sum of its token terms, fixed order
                constexpr int TPQ = kRows / QPC;  // threads per query
                const int m = tt / TPQ, part = tt % TPQ;
                float kl = 0.f;
#pragma unroll 8
                for (int j = 0; j < QPC; ++j) kl += sit[(part + TPQ * j) * SIP + m];
#pragma unroll
                for (int o = TPQ / 2; o; o >>= 1) kl += __shfl_xor_sync(0xffffffffu, kl, o);
                if (part == 0 && m < count) {
                    const int qe = s.ent[buf][m];
                    const size_t row = ((size_t)b * a.N + (qe >> 5)) * a.H_kv + r;
                    if (a.dense) atomicAdd(a.kl_rows + row, (double)kl);
                    else a.kl_part[row * K1 + (qe & 31)] = (double)kl;
                }
                mbar_arrive(&s.meta_empty[buf]);
            }
        }
        team_bar();
        if (myL >= 0 && s.abort == 0) flush_dk();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 128 * kSBuf);
}

// One warp per (b, i, r): dQ_idx = sum of the slot partials, KL row = sum of the slot partials, both
// in ascending slot order (each slot's dQ_idx row read as one coalesced 4 * d_idx byte segment).
template <int DI>
__global__ void k_kl_rows(KlArgs a) {
    const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= (long long)a.B * a.N * a.H_kv) return;
    const int K1 = a.topk + 1;
    const int i = (int)((row / a.H_kv) % a.N);
    const int32_t* sel = a.blocks + row * K1;
    // slots holding a distinct causal block (the same rule as the list build)
    uint32_t mask = 0;
    if (lane == 0) {
        int prev = -1;
        for (int s = 0; s < K1; ++s) {
            const int c = sel[s];
            if (c < 0 || c > i / a.block_k || c <= prev) continue;
            prev = c;
            mask |= 1u << s;
        }
    }
    mask = __shfl_sync(0xffffffffu, mask, 0);
    constexpr int VPL = DI / 32;  // dQ_idx values per lane
    float acc[VPL];
#pragma unroll
    for (int x = 0; x < VPL; ++x) acc[x] = 0.f;
    for (uint32_t m = mask; m; m &= m - 1) {
        const int s = __ffs(m) - 1;
        const float* dp = a.dq_part + (row * K1 + s) * DI + lane * VPL;
        if constexpr (VPL == 2) {
            const float2 v = *reinterpret_cast<const float2*>(dp);
            acc[0] += v.x;
            acc[1] += v.y;
        } else {
            acc[0] += dp[0];
        }
    }
    if constexpr (VPL == 2)
        *reinterpret_cast<float2*>(a.dq_idx + row * DI + lane * 2) = make_float2(acc[0], acc[1]);
    else
        a.dq_idx[row * DI + lane] = acc[0];
    const double kv = (lane < K1 && ((mask >> lane) & 1u)) ? a.kl_part[row * K1 + lane] : 0.0;
    double kl = 0.0;
    for (int s = 0; s < K1; ++s) kl += __shfl_sync(0xffffffffu, kv, s);
    if (lane == 0) a.kl_rows[row] = kl;
}

// Single CTA: loss = sum of the KL rows / (B N H_kv), in a fixed order (float64).
__global__ void k_kl_loss(KlArgs a) {
    __shared__ double part[1024];
    const long long n = (long long)a.B * a.N * a.H_kv;
    double acc = 0.0;
    for (long long x = threadIdx.x; x < n; x += 1024) acc += a.kl_rows[x];
    part[threadIdx.x] = acc;
    __syncthreads();
    for (int o = 512; o; o >>= 1) {
        if (threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *a.loss = (float)(part[0] / ((double)a.B * a.N * a.H_kv));
}

template <int D, int DI, int G>
cudaError_t launch_kl(const KlArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const void* q,
                      const void* q_idx, const void* k_idx, int num_sms, cudaStream_t st) {
    const size_t smem = std::max<size_t>(sizeof(KlSmem<D, DI, kRows / G, kl_teams<G>(), kl_meta_stages<G>(), kl_prods<G>()>) + 1024, 116 * 1024);  // one CTA per SM
    cudaError_t e = cudaFuncSetAttribute(k_kl_kv_outer<D, DI, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("kl_kv_outer", st);
    k_kl_kv_outer<D, DI, G><<<num_sms, kl_threads<G>(), smem, st>>>(tq, tk, static_cast<const __nv_bfloat16*>(q),
                                                              static_cast<const __nv_bfloat16*>(q_idx),
                                                              static_cast<const __nv_bfloat16*>(k_idx), a);
    return cudaGetLastError();
}

}  // namespace

bool kl_supported(int d, int d_idx, int G) {
    return ((d == 128 && d_idx == 64) || (d == 64 && d_idx == 32)) && (G == 2 || G == 16);
}

cudaError_t run_lse_idx(const KlArgs& a, const void* q_idx, const void* k_idx, int num_sms, cudaStream_t st) {
    const auto* qi = static_cast<const __nv_bfloat16*>(q_idx);
    const auto* ki = static_cast<const __nv_bfloat16*>(k_idx);
    ProfScope ps("lse_idx", st);
    if (a.d_idx == 64)
        k_lse_idx<64><<<num_sms * 6, 128, 0, st>>>(a, qi, ki);
    else
        k_lse_idx<32><<<num_sms * 6, 128, 0, st>>>(a, qi, ki);
    const long long rows = (long long)a.B * a.N * a.H_kv;
    k_lse_idx_merge<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t run_kl(const KlArgs& a, const void* q, const void* k, const void* q_idx, const void* k_idx, int num_sms,
                   cudaStream_t st) {
    const int G = a.H_q / a.H_kv;
    CUtensorMap tq, tk;
    const uint64_t dims[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2, (uint64_t)a.N * a.H_kv * a.d * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)a.block_k, 1};
    if (!make_tmap_4d(&tk, k, dims, strides, box, 128)) return cudaErrorInvalidValue;
    if (G % 8 == 0) {
        if (!make_tmap_qrows(&tq, q, a.B, a.N, a.H_q, a.d, G)) return cudaErrorInvalidValue;
    } else {
        tq = tk;  // not read: the query rows are copied without TMA
    }
    cudaError_t e = cudaMemsetAsync(a.dk_idx, 0, (size_t)a.B * a.N * a.d_idx * 4, st);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.B * a.N * a.H_kv;
    if (a.dense) {
        // dQ_idx and the KL rows are accumulated by the kernel
        e = cudaMemsetAsync(a.dq_idx, 0, (size_t)rows * a.d_idx * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(a.kl_rows, 0, (size_t)rows * 8, st);
        if (e != cudaSuccess) return e;
    }
    if (a.d == 128 && G == 16) e = launch_kl<128, 64, 16>(a, tq, tk, q, q_idx, k_idx, num_sms, st);
    else if (a.d == 128 && G == 2) e = launch_kl<128, 64, 2>(a, tq, tk, q, q_idx, k_idx, num_sms, st);
    else if (a.d == 64 && G == 16) e = launch_kl<64, 32, 16>(a, tq, tk, q, q_idx, k_idx, num_sms, st);
    else if (a.d == 64 && G == 2) e = launch_kl<64, 32, 2>(a, tq, tk, q, q_idx, k_idx, num_sms, st);
    else return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    ProfScope ps("kl_finalize", st);
    const unsigned grid_rows = (unsigned)((rows * 32 + 255) / 256);
    if (a.dense) {
        // the rows are complete; only the loss remains
    } else if (a.d_idx == 64) {
        k_kl_rows<64><<<grid_rows, 256, 0, st>>>(a);
    } else {
        k_kl_rows<32><<<grid_rows, 256, 0, st>>>(a);
    }
    k_kl_loss<<<1, 1024, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace msa
