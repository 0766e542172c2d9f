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

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void load_bf16_row(const __nv_bfloat16* src, float* dst, int n) {
#pragma unroll
    for (int c = 0; c < n; c += 8) {
        const uint4 u = *reinterpret_cast<const uint4*>(src + c);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float2 f = __bfloat1622float2(h[x]);
            dst[c + 2 * x] = f.x;
            dst[c + 2 * x + 1] = f.y;
        }
    }
}

// ============================================================================ LSE_idx pass
// Item = one selected block c of group r and up to kIdxQpc queries. Thread t owns token c*BK+t.
// Writes (max, sum-exp) of the scaled index logits of every (query, slot) over its causal tokens.
template <int DI>
__global__ void __launch_bounds__(128) k_lse_idx(KlArgs a, const __nv_bfloat16* __restrict__ q_idx,
                                                  const __nv_bfloat16* __restrict__ k_idx) {
    __shared__ float s_q[kIdxQpc][DI];
    __shared__ float s_s[kIdxQpc][129];
    __shared__ int s_i[kIdxQpc], s_slot[kIdxQpc];
    const Csr& cs = a.csr_idx;
    const int T = *cs.n_items;
    const int t = threadIdx.x;
    float kr[DI];
    int prevL = -1;
    for (int item = blockIdx.x; item < T; item += gridDim.x) {
        const int4 it = cs.items[item];
        const int L = it.x, count = it.z;
        const int c = L % cs.nb, r = (L / cs.nb) % a.H_kv, b = L / (cs.nb * a.H_kv);
        const int tok = c * a.block_k + t;
        const bool tvalid = t < a.block_k && tok < a.N;
        __syncthreads();  // previous item done with s_q / s_s / s_i
        if (L != prevL) {
            if (tvalid) load_bf16_row(k_idx + ((size_t)b * a.N + tok) * DI, kr, DI);
            prevL = L;
        }
        if (t < count) {
            const int e = cs.entries[it.y + t];
            s_i[t] = e >> 5;
            s_slot[t] = e & 31;
        }
        __syncthreads();
        for (int x = t; x < count * DI; x += 128) {
            const int m = x / DI, dd = x % DI;
            s_q[m][dd] = __bfloat162float(q_idx[(((size_t)b * a.N + s_i[m]) * a.H_kv + r) * DI + dd]);
        }
        __syncthreads();
        for (int m = 0; m < count; ++m) {
            float acc = 0.f;
#pragma unroll
            for (int dd = 0; dd < DI; ++dd) acc = fmaf(s_q[m][dd], kr[dd], acc);
            s_s[m][t] = (tvalid && tok <= s_i[m]) ? acc * a.scale_idx : -INFINITY;
        }
        __syncthreads();
        // one warp per query: max and sum-exp over the 128 token lanes
        const int w = t >> 5, ln = t & 31;
        for (int m = w; m < count; m += 4) {
            float mx = -INFINITY;
            for (int x = ln; x < 128; x += 32) mx = fmaxf(mx, s_s[m][x]);
#pragma unroll
            for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float z = 0.f;
            for (int x = ln; x < 128; x += 32) z += s_s[m][x] == -INFINITY ? 0.f : __expf(s_s[m][x] - mx);
#pragma unroll
            for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
            if (ln == 0)
                a.ml_part[(((size_t)b * a.N + s_i[m]) * a.H_kv + r) * (a.topk + 1) + s_slot[m]] = make_float2(mx, z);
        }
    }
}

// One thread per (b, i, r): LSE_idx = merge of the per-slot (max, sum-exp) pairs.
__global__ void k_lse_idx_merge(KlArgs a) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= (long long)a.B * a.N * a.H_kv) return;
    const int K1 = a.topk + 1;
    const int i = (int)((row / a.H_kv) % a.N);
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
    a.lse_idx[row] = mx + logf(z);
}

// ============================================================================ KL kernel
constexpr int kQpcMax = 64;  // queries per item when G >= 2

template <int D, int DI>
struct KlSmem {
    alignas(1024) uint8_t q[2][kRows * D * 2];
    alignas(1024) uint8_t k[kRows * D * 2];  // 128 token rows (rows >= block_k unused)
    float kf[kRows][DI + 1];                 // K_idx rows of the current block (float, padded)
    float gs[kRows][kQpcMax + 1];            // [token][query] scaled gradient g * scale_idx
    float klw[4][kQpcMax];                   // per-warp KL sums
    float lse[2][kRows];                     // LSE_main of the item rows
    float qf[2][kQpcMax][DI];                // Q_idx of the item queries (float)
    float lidx[2][kQpcMax];                  // LSE_idx of the item queries
    int qi[2][kQpcMax], qslot[2][kQpcMax];
    uint64_t q_full[2], q_empty[2], kv_full, kv_empty, s_full, s_free, drain;
    uint32_t tmem_base;
    int abort;
};

template <int D, int DI, int G>
__global__ void __launch_bounds__(kThreads, 1)
    k_kl_kv_outer(const __grid_constant__ CUtensorMap tm_k, const __nv_bfloat16* __restrict__ q,
                  const __nv_bfloat16* __restrict__ q_idx, const __nv_bfloat16* __restrict__ k_idx, KlArgs a) {
    using Sm = KlSmem<D, DI>;
    extern __shared__ uint8_t smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kIdesc = umma_idesc_bf16(kRows, kRows, false, false);
    constexpr int QPC = kRows / G;
    static_assert(QPC <= kQpcMax, "KL items hold at most 64 queries");

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
            mbar_init(&s.q_empty[x], 1 + kRows);
        }
        mbar_init(&s.kv_full, 1);
        mbar_init(&s.kv_empty, 1);
        mbar_init(&s.s_full, 1);
        mbar_init(&s.s_free, kRows);
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&s.tmem_base, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 4) {
        // ---------------------------------------------------------------- loads + item metadata
        int kv_loads = 0, prevL = -1;
        int ok = 1;
        for (int t = t0, n = 0; t < t1 && ok; ++t, ++n) {
            const int4 itm = cs.items[t];
            const int L = itm.x, count = itm.z;
            const int c = L % cs.nb, r = (L / cs.nb) % a.H_kv, b = L / (cs.nb * a.H_kv);
            const int buf = n & 1;
            if (lane == 0) ok = mbar_wait(&s.q_empty[buf], ((n >> 1) & 1) ^ 1, a.status, 0x801);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const int* ent = cs.entries + itm.y;
            for (int m = lane; m < QPC; m += 32) {
                const int e = m < count ? ent[m] : 0;
                s.qi[buf][m] = m < count ? (e >> 5) : -1;
                s.qslot[buf][m] = e & 31;
                s.lidx[buf][m] = m < count ? a.lse_idx[((size_t)b * a.N + (e >> 5)) * a.H_kv + r] : 0.f;
            }
            __syncwarp();
            for (int x = lane; x < count * G; x += 32) {
                const int m = x / G, h = x % G;
                s.lse[buf][x] = a.lse[((size_t)b * a.N + s.qi[buf][m]) * a.H_q + (size_t)r * G + h];
            }
            for (int x = lane; x < count * DI; x += 32) {
                const int m = x / DI, dd = x % DI;
                s.qf[buf][m][dd] = __bfloat162float(q_idx[(((size_t)b * a.N + s.qi[buf][m]) * a.H_kv + r) * DI + dd]);
            }
            const uint32_t qs = smem_u32(s.q[buf]);
            constexpr int kChunksPerRow = D * 2 / 16;
            const int nchunks = count * G * kChunksPerRow;
            for (int x = lane; x < nchunks; x += 32) {
                const int row = x / kChunksPerRow, ch = x % kChunksPerRow;
                const int m = row / G, h = row % G;
                const __nv_bfloat16* src =
                    q + ((((size_t)b * a.N + s.qi[buf][m]) * a.H_q + (size_t)r * G + h) * D + ch * 8);
                cp_async_16(qs + ((ch * 16) / 128) * (kRows * 128) + swz(row, (ch * 16) % 128, 128), src);
            }
            cp_async_wait_all();
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.q_full[buf]);
            if (L != prevL) {
                if (lane == 0) {
                    if (kv_loads > 0) ok = mbar_wait(&s.kv_empty, (kv_loads - 1) & 1, a.status, 0x802);
                    if (ok) {
                        mbar_arrive_expect_tx(&s.kv_full, (D / 64) * BK * 128);
#pragma unroll
                        for (int sub = 0; sub < D / 64; ++sub)
                            tma_load_4d(s.k + sub * kRows * 128, &tm_k, &s.kv_full, sub * 64, r, c * BK, b);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                ++kv_loads;
                prevL = L;
            }
        }
        if (!ok) s.abort = 1;
        if (lane == 0 && kv_loads > 0) mbar_wait(&s.kv_full, (kv_loads - 1) & 1, a.status, 0x803);
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            bool ok = true;
            int kv_group = -1, prevL = -1;
            for (int t = t0, n = 0; t < t1; ++t, ++n) {
                const int L = cs.items[t].x;
                const int buf = n & 1;
                if (!mbar_wait(&s.q_full[buf], (n >> 1) & 1, a.status, 0x901)) { ok = false; break; }
                if (L != prevL) {
                    ++kv_group;
                    prevL = L;
                    if (!mbar_wait(&s.kv_full, kv_group & 1, a.status, 0x902)) { ok = false; break; }
                }
                if (!mbar_wait(&s.s_free, (n & 1) ^ 1, a.status, 0x903)) { ok = false; break; }
                tc_fence_after();
                const uint32_t qb = smem_u32(s.q[buf]), kb = smem_u32(s.k);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t sub = (ks * 16) / 64, off = (ks & 3) * 32;
                    const uint64_t da = umma_sdesc(kb + sub * (kRows * 128) + off, 16, 1024, 2);
                    const uint64_t db = umma_sdesc(qb + sub * (kRows * 128) + off, 16, 1024, 2);
                    umma_bf16(tmem, da, db, kIdesc, ks > 0);
                }
                umma_commit(&s.s_full);
                umma_commit(&s.q_empty[buf]);
                const bool last_of_group = (t + 1 >= t1) || (cs.items[t + 1].x != L);
                if (last_of_group) umma_commit(&s.kv_empty);
            }
            if (!ok) s.abort = 1;
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, a.status, 0x904);
        }
    } else {
        // ---------------------------------------------------------------- epilogue: thread = token
        // Control flow stays uniform across the 128 threads (named barriers below): a failed wait
        // sets the CTA abort flag, and every thread then skips the work but not the barriers.
        const int tt = threadIdx.x;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        const float sl2 = a.scale * kLog2e;
        float dk[DI];
#pragma unroll
        for (int x = 0; x < DI; ++x) dk[x] = 0.f;
        int prevL = -1, prev_b = 0, prev_tok = 0;
        bool prev_valid = false;
        for (int t = t0, n = 0; t < t1; ++t, ++n) {
            const int4 itm = cs.items[t];
            const int L = itm.x, count = itm.z;
            const int c = L % cs.nb, r = (L / cs.nb) % a.H_kv, b = L / (cs.nb * a.H_kv);
            const int buf = n & 1;
            const int tok = c * BK + tt;
            const bool tvalid = tt < BK && tok < a.N;
            epi_bar();
            const bool alive = s.abort == 0;
            if (L != prevL) {
                if (prev_valid && alive) {
                    float* dst = a.dk_idx + ((size_t)prev_b * a.N + prev_tok) * DI;
#pragma unroll
                    for (int x = 0; x < DI; ++x) atomicAdd(dst + x, dk[x]);
                }
#pragma unroll
                for (int x = 0; x < DI; ++x) dk[x] = 0.f;
                {
                    float kr[DI];
#pragma unroll
                    for (int x = 0; x < DI; ++x) kr[x] = 0.f;
                    if (tvalid) load_bf16_row(k_idx + ((size_t)b * a.N + tok) * DI, kr, DI);
#pragma unroll
                    for (int x = 0; x < DI; ++x) s.kf[tt][x] = kr[x];
                }
                prevL = L;
                prev_b = b;
                prev_tok = tok;
                prev_valid = tvalid;
            }
            bool ok = alive;
            if (ok) ok = mbar_wait(&s.q_full[buf], (n >> 1) & 1, a.status, 0xa01);
            if (ok) ok = mbar_wait(&s.s_full, n & 1, a.status, 0xa02);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) s.abort = 1;
            float sv[kRows];
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < kRows; c0 += 32) {
                    uint32_t r32[32];
                    tmem_ld32(lane_addr + c0, r32);
                    tmem_ld_wait();
#pragma unroll
                    for (int x = 0; x < 32; ++x) sv[c0 + x] = __uint_as_float(r32[x]);
                }
                tc_fence_before();
                mbar_arrive(&s.s_free);
            }
#pragma unroll
            for (int m = 0; m < QPC; ++m) {
                float gval = 0.f, klv = 0.f;
                if (ok && m < count && tvalid && tok <= s.qi[buf][m]) {
                    float P = 0.f;
#pragma unroll
                    for (int h = 0; h < G; ++h)
                        P += fast_exp2(fmaf(sv[m * G + h], sl2, -s.lse[buf][m * G + h] * kLog2e));
                    P *= 1.f / (float)G;
                    float si = 0.f;
#pragma unroll
                    for (int x = 0; x < DI; ++x) si = fmaf(s.qf[buf][m][x], s.kf[tt][x], si);
                    const float lp_idx = si * a.scale_idx - s.lidx[buf][m];
                    const float g = coef * (__expf(lp_idx) - P);
                    klv = P > 0.f ? P * (__logf(P) - lp_idx) : 0.f;
                    gval = g * a.scale_idx;
#pragma unroll
                    for (int x = 0; x < DI; ++x) dk[x] = fmaf(gval, s.qf[buf][m][x], dk[x]);
                }
                s.gs[tt][m] = gval;
#pragma unroll
                for (int o = 16; o; o >>= 1) klv += __shfl_xor_sync(0xffffffffu, klv, o);
                if (lane == 0) s.klw[warp][m] = klv;
            }
            epi_bar();
            // per-(query, slot) reductions over the 128 tokens, fixed order
            if (ok) {
                for (int x = tt; x < count * (DI / 4); x += kRows) {
                    const int m = x / (DI / 4), dg = (x % (DI / 4)) * 4;
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int u = 0; u < kRows; ++u) {
                        const float g = s.gs[u][m];
                        acc.x = fmaf(g, s.kf[u][dg], acc.x);
                        acc.y = fmaf(g, s.kf[u][dg + 1], acc.y);
                        acc.z = fmaf(g, s.kf[u][dg + 2], acc.z);
                        acc.w = fmaf(g, s.kf[u][dg + 3], acc.w);
                    }
                    const size_t pr = (((size_t)b * a.N + s.qi[buf][m]) * a.H_kv + r) * K1 + s.qslot[buf][m];
                    *reinterpret_cast<float4*>(a.dq_part + pr * DI + dg) = acc;
                }
                if (tt < count) {
                    const double kl = ((double)s.klw[0][tt] + (double)s.klw[1][tt]) +
                                      ((double)s.klw[2][tt] + (double)s.klw[3][tt]);
                    const size_t pr = (((size_t)b * a.N + s.qi[buf][tt]) * a.H_kv + r) * K1 + s.qslot[buf][tt];
                    a.kl_part[pr] = kl;
                }
                mbar_arrive(&s.q_empty[buf]);
            }
        }
        epi_bar();
        if (prev_valid && s.abort == 0) {
            float* dst = a.dk_idx + ((size_t)prev_b * a.N + prev_tok) * DI;
#pragma unroll
            for (int x = 0; x < DI; ++x) atomicAdd(dst + x, dk[x]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 128);
}

// One thread per (b, i, r): dQ_idx = sum of the slot partials; KL row = sum of the slot partials.
template <int DI>
__global__ void k_kl_rows(KlArgs a) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= (long long)a.B * a.N * a.H_kv) return;
    const int K1 = a.topk + 1;
    const int i = (int)((row / a.H_kv) % a.N);
    const int32_t* sel = a.blocks + row * K1;
    float acc[DI];
#pragma unroll
    for (int x = 0; x < DI; ++x) acc[x] = 0.f;
    double kl = 0.0;
    int prev = -1;
    for (int s = 0; s < K1; ++s) {
        const int c = sel[s];
        if (c < 0 || c > i / a.block_k || c <= prev) continue;
        prev = c;
        const float* dp = a.dq_part + (row * K1 + s) * DI;
#pragma unroll
        for (int x = 0; x < DI; ++x) acc[x] += dp[x];
        kl += a.kl_part[row * K1 + s];
    }
#pragma unroll
    for (int x = 0; x < DI; ++x) a.dq_idx[row * DI + x] = acc[x];
    a.kl_rows[row] = kl;
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
cudaError_t launch_kl(const KlArgs& a, const CUtensorMap& tk, const void* q, const void* q_idx, const void* k_idx,
                      int num_sms, cudaStream_t st) {
    const size_t smem = std::max<size_t>(sizeof(KlSmem<D, DI>) + 1024, 116 * 1024);  // one CTA per SM
    cudaError_t e = cudaFuncSetAttribute(k_kl_kv_outer<D, DI, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("kl_kv_outer", st);
    k_kl_kv_outer<D, DI, G><<<num_sms, kThreads, smem, st>>>(tk, static_cast<const __nv_bfloat16*>(q),
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
        k_lse_idx<64><<<num_sms * 8, 128, 0, st>>>(a, qi, ki);
    else
        k_lse_idx<32><<<num_sms * 8, 128, 0, st>>>(a, qi, ki);
    const long long rows = (long long)a.B * a.N * a.H_kv;
    k_lse_idx_merge<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t run_kl(const KlArgs& a, const void* q, const void* k, const void* q_idx, const void* k_idx, int num_sms,
                   cudaStream_t st) {
    CUtensorMap tk;
    const uint64_t dims[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2, (uint64_t)a.N * a.H_kv * a.d * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)a.block_k, 1};
    if (!make_tmap_4d(&tk, k, dims, strides, box, 128)) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(a.dk_idx, 0, (size_t)a.B * a.N * a.d_idx * 4, st);
    if (e != cudaSuccess) return e;
    const int G = a.H_q / a.H_kv;
    if (a.d == 128 && G == 16) e = launch_kl<128, 64, 16>(a, tk, q, q_idx, k_idx, num_sms, st);
    else if (a.d == 128 && G == 2) e = launch_kl<128, 64, 2>(a, tk, q, q_idx, k_idx, num_sms, st);
    else if (a.d == 64 && G == 16) e = launch_kl<64, 32, 16>(a, tk, q, q_idx, k_idx, num_sms, st);
    else if (a.d == 64 && G == 2) e = launch_kl<64, 32, 2>(a, tk, q, q_idx, k_idx, num_sms, st);
    else return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    const long long rows = (long long)a.B * a.N * a.H_kv;
    ProfScope ps("kl_finalize", st);
    if (a.d_idx == 64)
        k_kl_rows<64><<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(a);
    else
        k_kl_rows<32><<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(a);
    k_kl_loss<<<1, 1024, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace msa
