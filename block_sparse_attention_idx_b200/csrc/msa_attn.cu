// Main branch of MSA: exact softmax attention over the selected blocks, KV-outer
// (MSA blog, KV-outer sparse attention and hot blocks; "2.4 · 训练原生稀疏", eq (2) and the
// online-softmax partition merge eq (18)).
//
// A work item is one selected KV block c of group r of sequence b plus up to 128/G queries that
// selected it: their G query heads form the 128 rows of the tile. Per item:
//   S = Q_rows . K_c^T         tcgen05.mma, M=128 rows, N=block_k tokens, K=d      -> TMEM
//   P = exp(S*scale - max)     epilogue warps, one row per thread (TMEM lane), causal mask j <= i
//   O = P . V_c                tcgen05.mma, M=128, N=d, K=block_k (V read MN-major) -> TMEM
// and the normalised partial (o = O/l, lse = max*scale + log l) of every row goes to the workspace
// slot of that (query, head, selection slot). A second kernel merges the <= topk+1 partials of
// every (query, head) with the log-sum-exp merge. Each CTA takes a contiguous range of items, so
// consecutive items reuse the K/V block already in shared memory.
//
// Warp roles (192 threads): warps 0-3 softmax/epilogue (thread = TMEM lane = tile row), warp 4
// loads (cp.async gather of the Q rows, TMA for K/V), warp 5 issues the MMAs and owns TMEM.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;

template <int D, int BK>
struct AttnSmem {
    static constexpr int kQBytes = kRows * D * 2;      // D/64 sub-tiles of [128 rows x 128 B]
    static constexpr int kKVBytes = BK * D * 2;        // D/64 sub-tiles of [BK rows x 128 B]
    static constexpr int kPPitch = BK >= 64 ? 128 : BK * 2;
    static constexpr int kPBytes = kRows * BK * 2;     // max(1, BK/64) sub-tiles of [128 x kPPitch]
    alignas(1024) uint8_t q[2][kQBytes];
    alignas(1024) uint8_t k[kKVBytes];
    alignas(1024) uint8_t v[kKVBytes];
    alignas(1024) uint8_t p[kPBytes];
    uint64_t q_full[2], q_empty[2];
    uint64_t kv_full, kv_empty;
    uint64_t s_full, s_free, p_full, p_free, o_full, o_free;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

struct ItemInfo {
    int L, start, count, b, r, c;
};

__device__ __forceinline__ ItemInfo decode_item(const AttnArgs& a, int t, int qpc) {
    const int2 it = a.csr.items[t];
    ItemInfo x;
    x.L = it.x;
    x.start = it.y;
    x.count = min(qpc, a.csr.counts[it.x] - it.y);
    x.c = it.x % a.csr.nb;
    x.r = (it.x / a.csr.nb) % a.H_kv;
    x.b = it.x / (a.csr.nb * a.H_kv);
    return x;
}

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_kv_outer(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __nv_bfloat16* __restrict__ q, AttnArgs a) {
    using Sm = AttnSmem<D, BK>;
    extern __shared__ uint8_t smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    constexpr uint32_t kIdescS = umma_idesc_bf16(kRows, BK, false, false);
    constexpr uint32_t kIdescO = umma_idesc_bf16(kRows, D, false, true);
    constexpr uint32_t kPLayout = Sm::kPPitch == 128 ? 2u : (Sm::kPPitch == 64 ? 4u : 6u);
    constexpr int kTmemS = 0, kTmemO = 128;

    const int G = a.H_q / a.H_kv;
    const int qpc = kRows / G;
    const int K1 = a.topk + 1;
    const int T = *a.csr.n_items;
    const int per = (T + gridDim.x - 1) / gridDim.x;
    const int t0 = blockIdx.x * per;
    const int t1 = min(T, t0 + per);
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s.q_full[x], 1);
            mbar_init(&s.q_empty[x], 1);
        }
        mbar_init(&s.kv_full, 1);
        mbar_init(&s.kv_empty, 1);
        mbar_init(&s.s_full, 1);
        mbar_init(&s.s_free, kRows);
        mbar_init(&s.p_full, kRows);
        mbar_init(&s.p_free, 1);
        mbar_init(&s.o_full, 1);
        mbar_init(&s.o_free, kRows);
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
        // ------------------------------------------------------------------ loads
        int kv_loads = 0, prevL = -1;
        bool ok = true;
        for (int t = t0, n = 0; t < t1 && ok; ++t, ++n) {
            const ItemInfo it = decode_item(a, t, qpc);
            const int buf = n & 1;
            int got = 1;
            if (lane == 0) got = mbar_wait(&s.q_empty[buf], ((n >> 1) & 1) ^ 1, a.status, 0x501);
            if (!__shfl_sync(0xffffffffu, got, 0)) { ok = false; break; }
            // gather the G head rows of each query of the item (rows of absent queries are left as is)
            const uint32_t qs = smem_u32(s.q[buf]);
            constexpr int kChunksPerRow = D * 2 / 16;
            const int nchunks = it.count * G * kChunksPerRow;
            const int* ent = a.csr.entries + a.csr.offsets[it.L] + it.start;
            for (int x = lane; x < nchunks; x += 32) {
                const int row = x / kChunksPerRow;      // tile row = m*G + h
                const int ch = x % kChunksPerRow;       // 16-byte chunk along d
                const int m = row / G, h = row % G;
                const int i = ent[m] >> 5;
                const __nv_bfloat16* src =
                    q + ((((size_t)it.b * a.N + i) * a.H_q + (size_t)it.r * G + h) * D + ch * 8);
                const uint32_t sub = (ch * 16) / 128, bir = (ch * 16) % 128;
                cp_async_16(qs + sub * (kRows * 128) + swz(row, bir, 128), src);
            }
            cp_async_wait_all();
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.q_full[buf]);
            // K/V of the item's block, when it changes
            if (it.L != prevL) {
                if (lane == 0) {
                    if (kv_loads > 0 && !mbar_wait(&s.kv_empty, (kv_loads - 1) & 1, a.status, 0x502)) ok = false;
                    if (ok) {
                        mbar_arrive_expect_tx(&s.kv_full, 2 * Sm::kKVBytes);
#pragma unroll
                        for (int sub = 0; sub < D / 64; ++sub) {
                            tma_load_4d(s.k + sub * BK * 128, &tm_k, &s.kv_full, sub * 64, it.r, it.c * BK, it.b);
                            tma_load_4d(s.v + sub * BK * 128, &tm_v, &s.kv_full, sub * 64, it.r, it.c * BK, it.b);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                ++kv_loads;
                prevL = it.L;
            }
        }
        if (!ok) s.abort = 1;
        if (lane == 0 && kv_loads > 0) mbar_wait(&s.kv_full, (kv_loads - 1) & 1, a.status, 0x503);
    } else if (warp == 5) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            int kv_group = -1, prevL = -1;
            for (int t = t0, n = 0; t < t1; ++t, ++n) {
                const int L = a.csr.items[t].x;
                const int buf = n & 1;
                if (!mbar_wait(&s.q_full[buf], (n >> 1) & 1, a.status, 0x601)) { ok = false; break; }
                if (L != prevL) {
                    ++kv_group;
                    prevL = L;
                    if (!mbar_wait(&s.kv_full, kv_group & 1, a.status, 0x602)) { ok = false; break; }
                }
                if (!mbar_wait(&s.s_free, (n & 1) ^ 1, a.status, 0x603)) { ok = false; break; }
                tc_fence_after();
                const uint32_t qb = smem_u32(s.q[buf]), kb = smem_u32(s.k), vb = smem_u32(s.v), pb = smem_u32(s.p);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks & 3) * 32;
                    const uint64_t da = umma_sdesc(qb + ((ks * 16) / 64) * (kRows * 128) + off, 16, 1024, 2);
                    const uint64_t db = umma_sdesc(kb + ((ks * 16) / 64) * (BK * 128) + off, 16, 1024, 2);
                    umma_bf16(tmem + kTmemS, da, db, kIdescS, ks > 0);
                }
                umma_commit(&s.s_full);
                umma_commit(&s.q_empty[buf]);
                if (!mbar_wait(&s.p_full, n & 1, a.status, 0x604)) { ok = false; break; }
                if (!mbar_wait(&s.o_free, (n & 1) ^ 1, a.status, 0x605)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < BK / 16; ++ks) {
                    const int tok = ks * 16;
                    uint64_t da;
                    if (Sm::kPPitch == 128)
                        da = umma_sdesc(pb + (tok / 64) * (kRows * 128) + (tok % 64) * 2, 16, 1024, kPLayout);
                    else
                        da = umma_sdesc(pb + tok * 2, 16, 8 * Sm::kPPitch, kPLayout);
                    const uint64_t db = umma_sdesc(vb + tok * 128, BK * 128, 1024, 2);
                    umma_bf16(tmem + kTmemO, da, db, kIdescO, ks > 0);
                }
                umma_commit(&s.o_full);
                umma_commit(&s.p_free);
                const bool last_of_group = (t + 1 >= t1) || (a.csr.items[t + 1].x != L);
                if (last_of_group) umma_commit(&s.kv_empty);
            }
            if (!ok) s.abort = 1;
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, a.status, 0x606);
        }
    } else {
        // ------------------------------------------------------------------ softmax / epilogue
        const int row = threadIdx.x;  // == TMEM lane
        const int m = row / G, h = row % G;
        const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
        const float sl2 = a.scale * 1.4426950408889634f;  // scale * log2(e)
        bool ok = true;
        for (int t = t0, n = 0; t < t1; ++t, ++n) {
            const ItemInfo it = decode_item(a, t, qpc);
            const bool valid = m < it.count;
            int i = 0, slot = 0;
            if (valid) {
                const int e = a.csr.entries[a.csr.offsets[it.L] + it.start + m];
                i = e >> 5;
                slot = e & 31;
            }
            const int lim = valid ? i - it.c * BK : -1;  // columns j <= lim are causal for this row
            if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full, n & 1, a.status, 0x701))) { ok = false; break; }
            tc_fence_after();
            float sv[BK];
#pragma unroll
            for (int c0 = 0; c0 < BK; c0 += 32) {
                uint32_t r32[32];
                tmem_ld32(lane_addr + kTmemS + c0, r32);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 32; ++c) sv[c0 + c] = __uint_as_float(r32[c]);
            }
            tc_fence_before();
            mbar_arrive(&s.s_free);
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < BK; ++c) mx = (c <= lim) ? fmaxf(mx, sv[c]) : mx;
            const float moff = valid ? mx * sl2 : 0.f;
            // l: exact sum for the LSE; lr: sum of the bf16-rounded weights the PV MMA actually
            // uses, so that o = (P_bf16 . V) / lr stays a convex combination of the V rows.
            float l = 0.f, lr = 0.f;
#pragma unroll
            for (int c = 0; c < BK; ++c) {
                const float p = (c <= lim) ? fast_exp2(fmaf(sv[c], sl2, -moff)) : 0.f;
                const float pr = __bfloat162float(__float2bfloat16_rn(p));
                sv[c] = pr;
                l += p;
                lr += pr;
            }
            // P (bf16) into the swizzled K-major tile read by the PV MMA
            if (!__all_sync(0xffffffffu, mbar_wait(&s.p_free, (n & 1) ^ 1, a.status, 0x702))) { ok = false; break; }
#pragma unroll
            for (int c0 = 0; c0 < BK; c0 += 8) {
                uint4 pk;
                pk.x = pack_bf16x2(sv[c0 + 0], sv[c0 + 1]);
                pk.y = pack_bf16x2(sv[c0 + 2], sv[c0 + 3]);
                pk.z = pack_bf16x2(sv[c0 + 4], sv[c0 + 5]);
                pk.w = pack_bf16x2(sv[c0 + 6], sv[c0 + 7]);
                uint32_t addr;
                if (Sm::kPPitch == 128)
                    addr = (c0 / 64) * (kRows * 128) + swz(row, (c0 % 64) * 2, 128);
                else
                    addr = swz(row, c0 * 2, Sm::kPPitch);
                *reinterpret_cast<uint4*>(s.p + addr) = pk;
            }
            fence_proxy_async();
            tc_fence_before();
            mbar_arrive(&s.p_full);
            if (!__all_sync(0xffffffffu, mbar_wait(&s.o_full, n & 1, a.status, 0x703))) { ok = false; break; }
            tc_fence_after();
            float ov[D];
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t r32[32];
                tmem_ld32(lane_addr + kTmemO + c0, r32);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 32; ++c) ov[c0 + c] = __uint_as_float(r32[c]);
            }
            tc_fence_before();
            mbar_arrive(&s.o_free);
            if (valid) {
                const float inv = 1.f / lr;
                const size_t prow = (((size_t)it.b * a.N + i) * a.H_q + (size_t)it.r * G + h) * K1 + slot;
                float4* dst = reinterpret_cast<float4*>(a.o_part + prow * D);
#pragma unroll
                for (int c = 0; c < D; c += 4)
                    dst[c / 4] = make_float4(ov[c] * inv, ov[c + 1] * inv, ov[c + 2] * inv, ov[c + 3] * inv);
                a.lse_part[prow] = mx * a.scale + logf(l);
            }
        }
        if (!ok) s.abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 256);
}

// One warp per (b, i, h): log-sum-exp merge of the per-slot partials, bf16 output.
template <int D>
__global__ void k_attn_merge(AttnArgs a, const int32_t* __restrict__ blocks, __nv_bfloat16* __restrict__ out,
                             float* __restrict__ lse_out) {
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long total = (long long)a.B * a.N * a.H_q;
    if (w >= total) return;
    const int G = a.H_q / a.H_kv;
    const int K1 = a.topk + 1;
    const int h = (int)(w % a.H_q);
    const long long bi = w / a.H_q;  // b * N + i
    const int i = (int)(bi % a.N);
    const int32_t* sel = blocks + (bi * a.H_kv + h / G) * K1;
    const float* lp = a.lse_part + w * K1;
    float mx = -INFINITY;
    int prev = -1;
    for (int sidx = 0; sidx < K1; ++sidx) {
        const int c = sel[sidx];
        if (c < 0 || c > i / a.block_k || c <= prev) continue;
        prev = c;
        mx = fmaxf(mx, lp[sidx]);
    }
    constexpr int kPer = D / 32;
    float acc[kPer];
#pragma unroll
    for (int x = 0; x < kPer; ++x) acc[x] = 0.f;
    float z = 0.f;
    prev = -1;
    for (int sidx = 0; sidx < K1; ++sidx) {
        const int c = sel[sidx];
        if (c < 0 || c > i / a.block_k || c <= prev) continue;
        prev = c;
        const float wgt = __expf(lp[sidx] - mx);
        z += wgt;
        const float* op = a.o_part + (w * K1 + sidx) * D + lane * kPer;
#pragma unroll
        for (int x = 0; x < kPer; ++x) acc[x] = fmaf(wgt, op[x], acc[x]);
    }
    const float inv = z > 0.f ? 1.f / z : 0.f;
    __nv_bfloat16* o = out + w * D + lane * kPer;
#pragma unroll
    for (int x = 0; x < kPer; ++x) o[x] = __float2bfloat16_rn(acc[x] * inv);
    if (lse_out && lane == 0) lse_out[w] = z > 0.f ? mx + logf(z) : -INFINITY;
}

template <int D, int BK>
cudaError_t launch_attn(const AttnArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, const void* q, int grid,
                        cudaStream_t st) {
    // at least 116 KB: one CTA per SM, so the 256 TMEM columns of each CTA are always available
    const size_t smem = std::max<size_t>(sizeof(AttnSmem<D, BK>) + 1024, 116 * 1024);
    cudaError_t e =
        cudaFuncSetAttribute(k_attn_kv_outer<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("attn_kv_outer", st);
    k_attn_kv_outer<D, BK><<<grid, kThreads, smem, st>>>(tk, tv, static_cast<const __nv_bfloat16*>(q), a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t run_attn_kv_outer(const AttnArgs& a, const void* q, const void* k, const void* v, int num_sms,
                              cudaStream_t st) {
    CUtensorMap tk, tv;
    const uint64_t dims[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2, (uint64_t)a.N * a.H_kv * a.d * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)a.block_k, 1};
    if (!make_tmap_4d(&tk, k, dims, strides, box, 128) || !make_tmap_4d(&tv, v, dims, strides, box, 128))
        return cudaErrorInvalidValue;
    const int grid = num_sms;
    if (a.d == 128) {
        if (a.block_k == 128) return launch_attn<128, 128>(a, tk, tv, q, grid, st);
        if (a.block_k == 64) return launch_attn<128, 64>(a, tk, tv, q, grid, st);
        return launch_attn<128, 32>(a, tk, tv, q, grid, st);
    }
    if (a.block_k == 128) return launch_attn<64, 128>(a, tk, tv, q, grid, st);
    if (a.block_k == 64) return launch_attn<64, 64>(a, tk, tv, q, grid, st);
    return launch_attn<64, 32>(a, tk, tv, q, grid, st);
}

cudaError_t run_attn_merge(const AttnArgs& a, const int32_t* blocks, void* out, float* lse, cudaStream_t st) {
    const long long warps = (long long)a.B * a.N * a.H_q;
    const int tpb = 256;
    const unsigned grid = (unsigned)((warps * 32 + tpb - 1) / tpb);
    ProfScope ps("attn_merge", st);
    if (a.d == 128)
        k_attn_merge<128><<<grid, tpb, 0, st>>>(a, blocks, static_cast<__nv_bfloat16*>(out), lse);
    else
        k_attn_merge<64><<<grid, tpb, 0, st>>>(a, blocks, static_cast<__nv_bfloat16*>(out), lse);
    return cudaGetLastError();
}

}  // namespace msa
