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
constexpr int kScanTokens = 2048;  // tokens per scan CTA
constexpr int kHkvMax = 8;

template <int DI>
__global__ void __launch_bounds__(kScanThreads) k_dec_scan(DecodeArgs a, const __nv_bfloat16* __restrict__ q_idx,
                                                           const __nv_bfloat16* __restrict__ k_idx) {
    __shared__ float s_q[kHkvMax][DI];
    __shared__ float s_wmax[kScanThreads / 32][kHkvMax];
    const int b = blockIdx.y;
    const int len = a.cache_len[b];
    const int nscored = ((len - 1) / a.block_k) * a.block_k;  // tokens of the complete past blocks
    const int t_begin = blockIdx.x * kScanTokens;
    if (t_begin >= nscored) return;
    const int nb = (a.L + a.block_k - 1) / a.block_k;
    for (int x = threadIdx.x; x < a.H_kv * DI; x += kScanThreads)
        s_q[x / DI][x % DI] = __bfloat162float(q_idx[(size_t)b * a.H_kv * DI + x]);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_end = min(nscored, t_begin + kScanTokens);
    for (int base = t_begin; base < t_end; base += kScanThreads) {
        const int tok = base + threadIdx.x;
        float sc[kHkvMax];
#pragma unroll
        for (int r = 0; r < kHkvMax; ++r) sc[r] = -INFINITY;
        if (tok < t_end) {
            const uint4* src = reinterpret_cast<const uint4*>(k_idx + ((size_t)b * a.L + tok) * DI);
            float acc[kHkvMax];
#pragma unroll
            for (int r = 0; r < kHkvMax; ++r) acc[r] = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < DI / 8; ++c8) {
                const uint4 u = __ldg(src + c8);
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
                float kv[8];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float2 f = __bfloat1622float2(h2[x]);
                    kv[2 * x] = f.x;
                    kv[2 * x + 1] = f.y;
                }
#pragma unroll
                for (int r = 0; r < kHkvMax; ++r) {
                    if (r < a.H_kv) {
#pragma unroll
                        for (int x = 0; x < 8; ++x) acc[r] = fmaf(s_q[r][c8 * 8 + x], kv[x], acc[r]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < kHkvMax; ++r) sc[r] = acc[r];
        }
        // block max: warps first, then the warps of one block
#pragma unroll
        for (int r = 0; r < kHkvMax; ++r) {
            float v = sc[r];
#pragma unroll
            for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) s_wmax[warp][r] = v;
        }
        __syncthreads();
        const int wpb = a.block_k / 32;  // warps per block
        const int nblk = kScanThreads / a.block_k;
        if (threadIdx.x < nblk * a.H_kv) {
            const int blk = threadIdx.x / a.H_kv, r = threadIdx.x % a.H_kv;
            const int c = (base / a.block_k) + blk;
            if (c * a.block_k < t_end) {
                float v = -INFINITY;
                for (int w = 0; w < wpb; ++w) v = fmaxf(v, s_wmax[blk * wpb + w][r]);
                a.bmax[((size_t)b * a.H_kv + r) * nb + c] = v;
            }
        }
        __syncthreads();
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

// One CTA per (sequence, group, slot): attention of the G heads over one selected block.
template <int D>
__global__ void __launch_bounds__(128) k_dec_attn(DecodeArgs a, const __nv_bfloat16* __restrict__ q,
                                                  const __nv_bfloat16* __restrict__ kc,
                                                  const __nv_bfloat16* __restrict__ vc) {
    extern __shared__ float dsm[];
    const int G = a.H_q / a.H_kv;
    const int BK = a.block_k;
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
    float* s_q = dsm;                  // [G][D]
    float* s_k = s_q + G * D;          // [BK][D + 1]
    float* s_v = s_k + BK * (D + 1);   // [BK][D]
    float* s_p = s_v + BK * D;         // [G][BK]
    for (int x = threadIdx.x; x < G * D; x += blockDim.x)
        s_q[x] = __bfloat162float(q[((size_t)b * a.H_q + (size_t)r * G) * D + x]);
    for (int x = threadIdx.x; x < BK * D / 8; x += blockDim.x) {
        const int t = x / (D / 8), c8 = x % (D / 8);
        const size_t go = (((size_t)b * a.L + (size_t)c * BK + t) * a.H_kv + r) * D + c8 * 8;
        uint4 ku = make_uint4(0, 0, 0, 0), vu = make_uint4(0, 0, 0, 0);
        if ((size_t)c * BK + t < (size_t)a.L) {
            ku = *reinterpret_cast<const uint4*>(kc + go);
            vu = *reinterpret_cast<const uint4*>(vc + go);
        }
        const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&ku);
        const __nv_bfloat162* v2 = reinterpret_cast<const __nv_bfloat162*>(&vu);
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            const float2 kf = __bfloat1622float2(k2[y]);
            const float2 vf = __bfloat1622float2(v2[y]);
            s_k[t * (D + 1) + c8 * 8 + 2 * y] = kf.x;
            s_k[t * (D + 1) + c8 * 8 + 2 * y + 1] = kf.y;
            s_v[t * D + c8 * 8 + 2 * y] = vf.x;
            s_v[t * D + c8 * 8 + 2 * y + 1] = vf.y;
        }
    }
    __syncthreads();
    // scores: thread = token
    for (int t = threadIdx.x; t < BK; t += blockDim.x) {
        const bool ok = c * BK + t <= len - 1;
        for (int h = 0; h < G; ++h) {
            float acc = 0.f;
            for (int x = 0; x < D; ++x) acc = fmaf(s_q[h * D + x], s_k[t * (D + 1) + x], acc);
            s_p[h * BK + t] = ok ? acc * a.scale : -INFINITY;
        }
    }
    __syncthreads();
    // softmax per head: one warp per head
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int h = warp; h < G; h += blockDim.x / 32) {
        float mx = -INFINITY;
        for (int t = lane; t < BK; t += 32) mx = fmaxf(mx, s_p[h * BK + t]);
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float z = 0.f;
        for (int t = lane; t < BK; t += 32) {
            const float e = s_p[h * BK + t] == -INFINITY ? 0.f : __expf(s_p[h * BK + t] - mx);
            s_p[h * BK + t] = e;
            z += e;
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        const float inv = 1.f / z;
        for (int t = lane; t < BK; t += 32) s_p[h * BK + t] *= inv;
        if (lane == 0) lse_out[h] = mx + logf(z);
    }
    __syncthreads();
    // PV: thread = output dim
    float* o_out = a.o_part + ((size_t)bs * K1 + slot) * G * D;
    for (int dd = threadIdx.x; dd < D; dd += blockDim.x) {
        for (int h = 0; h < G; ++h) {
            float acc = 0.f;
            for (int t = 0; t < BK; ++t) acc = fmaf(s_p[h * BK + t], s_v[t * D + dd], acc);
            o_out[h * D + dd] = acc;
        }
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
    const dim3 sgrid((a.L + kScanTokens - 1) / kScanTokens, a.B);
    {
        ProfScope ps("dec_scan", st);
        if (a.d_idx == 64)
            k_dec_scan<64><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki);
        else
            k_dec_scan<32><<<sgrid, kScanThreads, 0, st>>>(a, qi, ki);
    }
    {
        ProfScope ps("dec_topk", st);
        k_dec_topk<<<a.B * a.H_kv, 256, 0, st>>>(a);
    }
    ProfScope ps("dec_attn_combine", st);
    const int G = a.H_q / a.H_kv;
    const size_t smem = ((size_t)G * a.d + (size_t)a.block_k * (a.d + 1) + (size_t)a.block_k * a.d +
                         (size_t)G * a.block_k) * 4;
    const dim3 agrid(a.B * a.H_kv, a.topk + 1);
    const auto* qb = static_cast<const __nv_bfloat16*>(q);
    const auto* kb = static_cast<const __nv_bfloat16*>(k_cache);
    const auto* vb = static_cast<const __nv_bfloat16*>(v_cache);
    cudaError_t e;
    if (a.d == 128) {
        e = cudaFuncSetAttribute(k_dec_attn<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k_dec_attn<128><<<agrid, 128, smem, st>>>(a, qb, kb, vb);
        k_dec_combine<128><<<(a.B * a.H_q * 32 + 255) / 256, 256, 0, st>>>(a, static_cast<float*>(out));
    } else {
        e = cudaFuncSetAttribute(k_dec_attn<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        k_dec_attn<64><<<agrid, 128, smem, st>>>(a, qb, kb, vb);
        k_dec_combine<64><<<(a.B * a.H_q * 32 + 255) / 256, 256, 0, st>>>(a, static_cast<float*>(out));
    }
    return cudaGetLastError();
}

}  // namespace msa
