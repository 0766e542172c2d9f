// Decode step of MSA for one new token per sequence (MSA blog: decode reads only the selected
// KV; "2.4 · 训练原生稀疏", section 3.2: decode must compute the same selection and attention as the
// parallel causal path).
//
// The newest token sits at position len-1 of the caches. Its index scores against every cached
// token are needed for the causal block max-pool, so the step streams the whole K_idx cache once:
// that scan is about 88% of the bytes of a step and is HBM-bound by design. Then:
//   k_dec_scan     split-L over (chunk of tokens, sequence): 4 group scores per token, block max
//   k_dec_topk     per (sequence, group): Top-k over the complete past blocks + local block
//   k_dec_attn     split-KV over (sequence, group, selected slot): one block of K/V for the G heads
//   k_dec_combine  per (sequence, head): log-sum-exp merge of the slot partials
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kScanThreads = 256;
constexpr int kHkvMax = 8;

// One warp per complete past block of one sequence: the block's index scores for every group and
// their maximum. A token's d_idx row is split over DI/8 lanes (one 16-byte load each), so one warp
// load instruction covers whole 128-byte lines; eight rounds of loads are in flight before the
// first use. Partial dot products are summed over the token's lanes by shuffles.
template <int DI, int HKV>
__global__ void __launch_bounds__(kScanThreads, 2) k_dec_scan(DecodeArgs a, const __nv_bfloat16* __restrict__ q_idx,
                                                           const __nv_bfloat16* __restrict__ k_idx) {
    constexpr int LPT = DI / 8;    // lanes per token
    constexpr int TPR = 32 / LPT;  // tokens per warp round
    constexpr int U = HKV >= 8 ? 4 : 8;  // rounds in flight (fewer when q takes more registers)
    const int b = blockIdx.y;
    const int len = a.cache_len[b];
    const int nfull = (len - 1) / a.block_k;  // complete past blocks (the local block is not scored)
    const int nb = (a.L + a.block_k - 1) / a.block_k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int part = lane % LPT, tsub = lane / LPT;
    float qv[HKV][8];
#pragma unroll
    for (int r = 0; r < HKV; ++r) {
        const __nv_bfloat162* q2 =
            reinterpret_cast<const __nv_bfloat162*>(q_idx + ((size_t)b * HKV + r) * DI + part * 8);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float2 f = __bfloat1622float2(q2[x]);
            qv[r][2 * x] = f.x;
            qv[r][2 * x + 1] = f.y;
        }
    }
    for (int blk = blockIdx.x * (kScanThreads / 32) + warp; blk < nfull; blk += gridDim.x * (kScanThreads / 32)) {
        const __nv_bfloat16* base = k_idx + ((size_t)b * a.L + (size_t)blk * a.block_k) * DI + part * 8;
        float mx[HKV];
#pragma unroll
        for (int r = 0; r < HKV; ++r) mx[r] = -INFINITY;
        for (int t0 = 0; t0 < a.block_k; t0 += TPR * U) {
            uint4 u0[U];
#pragma unroll
            for (int j = 0; j < U; ++j) {
                const int tok = t0 + j * TPR + tsub;
                u0[j] = tok < a.block_k ? __ldcs(reinterpret_cast<const uint4*>(base + (size_t)tok * DI))
                                        : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < U; ++j) {
                float kv[8];
                const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&u0[j]);
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float2 f0 = __bfloat1622float2(h0[x]);
                    kv[2 * x] = f0.x;
                    kv[2 * x + 1] = f0.y;
                }
                const bool valid = t0 + j * TPR + tsub < a.block_k;
#pragma unroll
                for (int r = 0; r < HKV; ++r) {
                    float p = 0.f;
#pragma unroll
                    for (int x = 0; x < 8; ++x) p = fmaf(qv[r][x], kv[x], p);
#pragma unroll
                    for (int o = 1; o < LPT; o <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
                    if (valid) mx[r] = fmaxf(mx[r], p);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < HKV; ++r) {
#pragma unroll
            for (int o = LPT; o < 32; o <<= 1) mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], o));
        }
        if (lane < HKV) {
            float v = mx[0];
#pragma unroll
            for (int r = 1; r < HKV; ++r) v = lane == r ? mx[r] : v;
            a.bmax[((size_t)b * HKV + lane) * nb + blk] = v;
        }
    }
}

// One CTA per (sequence, group): Top-k of the block maxima of the complete past blocks by
// (max desc, id asc), plus the local block; written ascending, -1 padded.
__global__ void __launch_bounds__(256) k_dec_topk(DecodeArgs a) {
    __shared__ unsigned char taken[8192];
    __shared__ float s_v[8];
    __shared__ int s_i[8];
    __shared__ int chosen[17];
    const int b = blockIdx.x / a.H_kv, r = blockIdx.x % a.H_kv;
    const int len = a.cache_len[b];
    const int bi = (len - 1) / a.block_k;
    const int nb = (a.L + a.block_k - 1) / a.block_k;
    const float* vals = a.bmax + ((size_t)b * a.H_kv + r) * nb;
    const int K1 = a.topk + 1;
    for (int c = threadIdx.x; c < bi; c += blockDim.x) taken[c] = 0;
    __syncthreads();
    const int take = min(a.topk, bi);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int round = 0; round < take; ++round) {
        float bv = -INFINITY;
        int bidx = 0x7fffffff;
        for (int c = threadIdx.x; c < bi; c += blockDim.x) {
            if (taken[c]) continue;
            const float v = vals[c];
            if (v > bv || (v == bv && c < bidx)) { bv = v; bidx = c; }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
            if (ov > bv || (ov == bv && oi < bidx)) { bv = ov; bidx = oi; }
        }
        if (lane == 0) { s_v[warp] = bv; s_i[warp] = bidx; }
        __syncthreads();
        if (threadIdx.x == 0) {
            float v = s_v[0];
            int id = s_i[0];
            for (int w = 1; w < (int)(blockDim.x / 32); ++w)
                if (s_v[w] > v || (s_v[w] == v && s_i[w] < id)) { v = s_v[w]; id = s_i[w]; }
            if (id == 0x7fffffff) id = 0;  // every candidate was -inf; pick the lowest untaken id
            chosen[round] = id;
            taken[id] = 1;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        int n = take;
        chosen[n++] = bi;
        for (int x = 1; x < n; ++x) {  // insertion sort, ascending
            const int v = chosen[x];
            int y = x - 1;
            while (y >= 0 && chosen[y] > v) { chosen[y + 1] = chosen[y]; --y; }
            chosen[y + 1] = v;
        }
        int32_t* out = a.sel + ((size_t)b * a.H_kv + r) * K1;
        for (int x = 0; x < K1; ++x) out[x] = x < n ? chosen[x] : -1;
        if (a.blocks_out) {
            int32_t* bo = a.blocks_out + ((size_t)b * a.H_kv + r) * K1;
            for (int x = 0; x < K1; ++x) bo[x] = x < n ? chosen[x] : -1;
        }
    }
}

// One CTA (4 warps) per (sequence, group, selected slot): attention of the group's G heads over one
// block. K and V of the block are staged in shared memory as bf16 (rows padded by 16 bytes so the
// fragment loads are conflict-free) with cp.async, all in flight at once. The G heads are the M=16
// rows of warp-level mma.sync.m16n8k16 tiles (G=32 takes two row tiles, fewer heads are padded
// with zero rows); each warp owns 16-token units of the block. S = Q.K^T stays in registers, the
// row max and sum are combined across the warps in shared memory, P is reused from the S
// accumulators as the A operand of P.V (V fragments via ldmatrix.trans), and the warps' O tiles
// are summed in shared memory. Writes the slot's normalised fp32 partial and its LSE.
template <int D, int BK>
__global__ void __launch_bounds__(128) k_dec_attn(DecodeArgs a, const __nv_bfloat16* __restrict__ q,
                                                  const __nv_bfloat16* __restrict__ kc,
                                                  const __nv_bfloat16* __restrict__ vc) {
    constexpr int KP = D + 8;          // padded row (bf16)
    constexpr int NU = BK / 16;        // 16-token units
    constexpr int UPW = (NU + 3) / 4;  // units per warp
    extern __shared__ __align__(16) uint8_t dec_smem[];
    __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(dec_smem);  // [BK][KP]
    __nv_bfloat16* sV = sK + BK * KP;                                 // [BK][KP]
    float* sO = reinterpret_cast<float*>(sV + BK * KP);               // [16][D]
    float* sRed = sO + 16 * D;                                        // [4][16] per-warp max, then exact sums
    float* sRedR = sRed + 64;                                         // [4][16] per-warp rounded sums
    float* sRow = sRedR + 64;                                         // [3][16]: max (log2), exact sum, rounded sum
    const int G = a.H_q / a.H_kv;
    const int K1 = a.topk + 1;
    const int bs = blockIdx.x;  // b * H_kv + r
    const int slot = blockIdx.y;
    const int b = bs / a.H_kv, r = bs % a.H_kv;
    const int c = a.sel[(size_t)bs * K1 + slot];
    float* lse_out = a.lse_part + ((size_t)bs * K1 + slot) * G;
    if (c < 0) {
        for (int h = threadIdx.x; h < G; h += blockDim.x) lse_out[h] = -INFINITY;
        return;
    }
    const int len = a.cache_len[b];
    for (int x = threadIdx.x; x < BK * D / 8; x += blockDim.x) {
        const int t = x / (D / 8), c8 = x % (D / 8);
        const bool ok = (size_t)c * BK + t < (size_t)a.L;
        const size_t go = (((size_t)b * a.L + (ok ? (size_t)c * BK + t : 0)) * a.H_kv + r) * D + c8 * 8;
        cp_async_16_zfill(smem_u32(sK + t * KP + c8 * 8), kc + go, ok);
        cp_async_16_zfill(smem_u32(sV + t * KP + c8 * 8), vc + go, ok);
    }
    cp_async_wait_all();
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    const float sl2 = a.scale * 1.4426950408889634f;
    float* o_out = a.o_part + ((size_t)bs * K1 + slot) * G * D;
    for (int mt = 0; mt * 16 < G; ++mt) {
        for (int x = threadIdx.x; x < 16 * D; x += blockDim.x) sO[x] = 0.f;
        // Q fragments: rows h0 = 16mt + g and h1 = h0 + 8 (zero beyond G)
        const int h0 = mt * 16 + g, h1 = h0 + 8;
        const int h0c = min(h0, G - 1), h1c = min(h1, G - 1);  // padded rows read nothing
        const uint32_t* q0 = reinterpret_cast<const uint32_t*>(q + ((size_t)b * a.H_q + (size_t)r * G + h0c) * D);
        const uint32_t* q1 = reinterpret_cast<const uint32_t*>(q + ((size_t)b * a.H_q + (size_t)r * G + h1c) * D);
        uint32_t qa[D / 16][4];
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = h0 < G ? q0[8 * ks + t4] : 0u;
            qa[ks][1] = h1 < G ? q1[8 * ks + t4] : 0u;
            qa[ks][2] = h0 < G ? q0[8 * ks + 4 + t4] : 0u;
            qa[ks][3] = h1 < G ? q1[8 * ks + 4 + t4] : 0u;
        }
        // S (log2 units) of the warp's units; tokens past the query are -inf
        float sc[UPW][2][4];
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < UPW; ++j) {
            const int u = warp + 4 * j;
#pragma unroll
            for (int tl = 0; tl < 2; ++tl) {
                sc[j][tl][0] = sc[j][tl][1] = sc[j][tl][2] = sc[j][tl][3] = 0.f;
                if (u < NU) {
                    const int n0 = 16 * u + 8 * tl;
                    const uint32_t* krow = reinterpret_cast<const uint32_t*>(sK + (n0 + g) * KP);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) mma_16816_bf16(sc[j][tl], qa[ks], krow[8 * ks + t4], krow[8 * ks + 4 + t4]);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = c * BK + 16 * u + 8 * tl + 2 * t4 + (e & 1);
                    sc[j][tl][e] = (u < NU && tok <= len - 1) ? sc[j][tl][e] * sl2 : -INFINITY;
                }
                mx0 = fmaxf(mx0, fmaxf(sc[j][tl][0], sc[j][tl][1]));
                mx1 = fmaxf(mx1, fmaxf(sc[j][tl][2], sc[j][tl][3]));
            }
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        if (t4 == 0) {
            sRed[warp * 16 + g] = mx0;
            sRed[warp * 16 + g + 8] = mx1;
        }
        __syncthreads();
        const float m0 = fmaxf(fmaxf(sRed[g], sRed[16 + g]), fmaxf(sRed[32 + g], sRed[48 + g]));
        const float m1 = fmaxf(fmaxf(sRed[8 + g], sRed[24 + g]), fmaxf(sRed[40 + g], sRed[56 + g]));
        __syncthreads();
        // P; l: exact sums (for the LSE); lr: sums of the bf16-rounded P the MMA multiplies (for the
        // normalisation, as in the prefill attention)
        float l0 = 0.f, l1 = 0.f, lr0 = 0.f, lr1 = 0.f;
        uint32_t pk[UPW][4];
#pragma unroll
        for (int j = 0; j < UPW; ++j) {
#pragma unroll
            for (int tl = 0; tl < 2; ++tl) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float m = e < 2 ? m0 : m1;
                    const float p = sc[j][tl][e] == -INFINITY ? 0.f : exp2f(sc[j][tl][e] - m);
                    sc[j][tl][e] = p;
                    if (e < 2) l0 += p; else l1 += p;
                }
                pk[j][2 * tl] = pack_bf16x2(sc[j][tl][0], sc[j][tl][1]);
                pk[j][2 * tl + 1] = pack_bf16x2(sc[j][tl][2], sc[j][tl][3]);
                lr0 += __uint_as_float(pk[j][2 * tl] << 16) + __uint_as_float(pk[j][2 * tl] & 0xffff0000u);
                lr1 += __uint_as_float(pk[j][2 * tl + 1] << 16) + __uint_as_float(pk[j][2 * tl + 1] & 0xffff0000u);
            }
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, o);
            l1 += __shfl_xor_sync(0xffffffffu, l1, o);
            lr0 += __shfl_xor_sync(0xffffffffu, lr0, o);
            lr1 += __shfl_xor_sync(0xffffffffu, lr1, o);
        }
        if (t4 == 0) {
            sRed[warp * 16 + g] = l0;
            sRed[warp * 16 + g + 8] = l1;
            sRedR[warp * 16 + g] = lr0;
            sRedR[warp * 16 + g + 8] = lr1;
        }
        // O = P.V over the warp's units
        float ov[D / 8][4];
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) ov[nd][0] = ov[nd][1] = ov[nd][2] = ov[nd][3] = 0.f;
#pragma unroll
        for (int j = 0; j < UPW; ++j) {
            const int u = warp + 4 * j;
            if (u >= NU) continue;
            // A fragment of P: rows g / g+8, tokens 2t4.. of the unit's first and second 8-token tile
            const uint32_t pa[4] = {pk[j][0], pk[j][1], pk[j][2], pk[j][3]};
            // lane L addresses row (16u + 8*((L/8)%2) + L%8) of V at column 8*(nd + L/16)
            const int vrow = 16 * u + 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
            for (int nd = 0; nd < D / 8; nd += 2) {
                uint32_t b00, b01, b10, b11;
                ldsm_x4_trans(smem_u32(sV + vrow * KP + 8 * (nd + (lane >> 4))), b00, b01, b10, b11);
                mma_16816_bf16(ov[nd], pa, b00, b01);
                mma_16816_bf16(ov[nd + 1], pa, b10, b11);
            }
        }
        __syncthreads();
        if (t4 == 0 && warp == 0) {
            sRow[g] = m0;
            sRow[g + 8] = m1;
            sRow[16 + g] = sRed[g] + sRed[16 + g] + sRed[32 + g] + sRed[48 + g];
            sRow[16 + g + 8] = sRed[8 + g] + sRed[24 + g] + sRed[40 + g] + sRed[56 + g];
            sRow[32 + g] = sRedR[g] + sRedR[16 + g] + sRedR[32 + g] + sRedR[48 + g];
            sRow[32 + g + 8] = sRedR[8 + g] + sRedR[24 + g] + sRedR[40 + g] + sRedR[56 + g];
        }
#pragma unroll
        for (int nd = 0; nd < D / 8; ++nd) {
            atomicAdd(&sO[g * D + nd * 8 + 2 * t4], ov[nd][0]);
            atomicAdd(&sO[g * D + nd * 8 + 2 * t4 + 1], ov[nd][1]);
            atomicAdd(&sO[(g + 8) * D + nd * 8 + 2 * t4], ov[nd][2]);
            atomicAdd(&sO[(g + 8) * D + nd * 8 + 2 * t4 + 1], ov[nd][3]);
        }
        __syncthreads();
        for (int x = threadIdx.x; x < 16 * D; x += blockDim.x) {
            const int hh = x / D, h = mt * 16 + hh;
            if (h < G) o_out[(size_t)h * D + x % D] = sO[x] / sRow[32 + hh];
        }
        if (threadIdx.x < 16 && mt * 16 + threadIdx.x < G)
            lse_out[mt * 16 + threadIdx.x] = sRow[threadIdx.x] * 0.6931471805599453f + logf(sRow[16 + threadIdx.x]);
        __syncthreads();
    }
}

// One warp per (sequence, head): merge the slot partials.
template <int D>
__global__ void k_dec_combine(DecodeArgs a, float* __restrict__ out) {
    const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= a.B * a.H_q) return;
    const int G = a.H_q / a.H_kv;
    const int K1 = a.topk + 1;
    const int b = w / a.H_q, h = w % a.H_q, r = h / G, hg = h % G;
    const size_t bs = (size_t)b * a.H_kv + r;
    float mx = -INFINITY;
    for (int s = 0; s < K1; ++s) mx = fmaxf(mx, a.lse_part[(bs * K1 + s) * G + hg]);
    constexpr int kPer = D / 32;
    float acc[kPer];
#pragma unroll
    for (int x = 0; x < kPer; ++x) acc[x] = 0.f;
    float z = 0.f;
    for (int s = 0; s < K1; ++s) {
        const float l = a.lse_part[(bs * K1 + s) * G + hg];
        if (l == -INFINITY) continue;
        const float wg = __expf(l - mx);
        z += wg;
        const float* op = a.o_part + ((bs * K1 + s) * G + hg) * D + lane * kPer;
#pragma unroll
        for (int x = 0; x < kPer; ++x) acc[x] = fmaf(wg, op[x], acc[x]);
    }
    const float inv = 1.f / z;
    float* o = out + ((size_t)b * a.H_q + h) * D + lane * kPer;
#pragma unroll
    for (int x = 0; x < kPer; ++x) o[x] = acc[x] * inv;
}

}  // namespace

size_t decode_ws_bytes(int B, int L, int H_q, int H_kv, int d, int block_k, int topk) {
    const size_t nb = (size_t)(L + block_k - 1) / block_k;
    const size_t G = (size_t)H_q / H_kv, K1 = (size_t)topk + 1;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    return al((size_t)B * H_kv * nb * 4) + al((size_t)B * H_kv * K1 * 4) + al((size_t)B * H_kv * K1 * G * d * 4) +
           al((size_t)B * H_kv * K1 * G * 4);
}

cudaError_t run_decode(const DecodeArgs& a, const void* q, const void* q_idx, const void* k_cache,
                       const void* v_cache, const void* k_idx_cache, void* out, cudaStream_t st) {
    const auto* qi = static_cast<const __nv_bfloat16*>(q_idx);
    const auto* ki = static_cast<const __nv_bfloat16*>(k_idx_cache);
    const int nb = (a.L + a.block_k - 1) / a.block_k;
    const dim3 sgrid((nb + kScanThreads / 32 - 1) / (kScanThreads / 32), a.B);
    {
        ProfScope ps("dec_scan", st);
        const bool d64 = a.d_idx == 64;
        switch (a.H_kv) {
            case 1: d64 ? k_dec_scan<64, 1><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki)
                        : k_dec_scan<32, 1><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki); break;
            case 2: d64 ? k_dec_scan<64, 2><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki)
                        : k_dec_scan<32, 2><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki); break;
            case 4: d64 ? k_dec_scan<64, 4><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki)
                        : k_dec_scan<32, 4><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki); break;
            default: d64 ? k_dec_scan<64, 8><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki)
                         : k_dec_scan<32, 8><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki); break;
        }
    }
    {
        ProfScope ps("dec_topk", st);
        k_dec_topk<<<a.B * a.H_kv, 256, 0, st>>>(a);
    }
    ProfScope ps("dec_attn_combine", st);
    const dim3 agrid(a.B * a.H_kv, a.topk + 1);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k_cache);
    const auto* vb = static_cast<const __nv_bfloat16*>(v_cache);
    const size_t smem = (size_t)2 * a.block_k * (a.d + 8) * 2 + (size_t)16 * a.d * 4 + (64 + 64 + 48) * 4;
    auto launch = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<agrid, 128, smem, st>>>(a, qb, kb, vb);
        return cudaGetLastError();
    };
    cudaError_t e;
    if (a.d == 128) {
        e = a.block_k == 128 ? launch(k_dec_attn<128, 128>) : a.block_k == 64 ? launch(k_dec_attn<128, 64>)
                                                                               : launch(k_dec_attn<128, 32>);
        if (e != cudaSuccess) return e;
        k_dec_combine<128><<<(a.B * a.H_q * 32 + 255) / 256, 256, 0, st>>>(a, static_cast<float*>(out));
    } else {
        e = a.block_k == 128 ? launch(k_dec_attn<64, 128>) : a.block_k == 64 ? launch(k_dec_attn<64, 64>)
                                                                              : launch(k_dec_attn<64, 32>);
        if (e != cudaSuccess) return e;
        k_dec_combine<64><<<(a.B * a.H_q * 32 + 255) / 256, 256, 0, st>>>(a, static_cast<float*>(out));
    }
    return cudaGetLastError();
}

}  // namespace msa
