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
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <type_traits>

#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

// Launch after the previous kernel of the stream with programmatic serialisation (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}


// Index scan: every complete past block of every sequence, its index scores for all groups and
// their maximum. Persistent CTAs (one per SM): warp 4 streams the blocks' K_idx tiles into an
// 8-stage shared-memory ring by TMA (128- or 64-byte swizzled rows); warps 0-3 take the ring's
// tiles in turn and compute S^T = K_idx_tile . Q_idx^T with warp-level mma.sync (16 tokens x 8
// group columns x 16 dims per instruction, A fragments by ldmatrix from the swizzled tile, the
// groups' Q_idx as B fragments held in registers); each block's maxima come straight from the
// accumulators. The kernel is HBM-bound: it reads every K_idx byte once.
// The scan's work list: the complete past blocks of all sequences in (sequence, block) order, T
// items in all. CTA c takes the contiguous range [c*T/grid, (c+1)*T/grid): a CTA streams one
// contiguous stretch of the cache and meets at most a few sequences, so it reloads a sequence's
// length and its Q_idx rarely. A cursor walks the range.
struct ScanCursor {
    int b, blk, nbv;  // current item: block blk of sequence b, which has nbv complete past blocks
};
// cache_len[b] clamped to [1, L]: every kernel reads the length through this, so a value outside
// the caches' capacity can never index past them (the Top-k kernel reports it).
__device__ __forceinline__ int dec_len(const DecodeArgs& a, int b) { return min(max(a.cache_len[b], 1), a.L); }
__device__ __forceinline__ int complete_blocks(const DecodeArgs& a, int b, int BK) {
    return (dec_len(a, b) - 1) / BK;
}
// Called by all lanes of a warp: sets c to the CTA's first item, returns its number of items.
__device__ int scan_range(const DecodeArgs& a, int BK, ScanCursor& c) {
    const int lane = threadIdx.x & 31;
    long long T = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
        int v = b0 + lane < a.B ? complete_blocks(a, b0 + lane, BK) : 0;
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        T += v;
    }
    const long long lo = T * blockIdx.x / gridDim.x, hi = T * (blockIdx.x + 1) / gridDim.x;
    long long cum = 0;  // items before sequence b0
    for (int b0 = 0; b0 < a.B && lo < hi; b0 += 32) {
        const int v = b0 + lane < a.B ? complete_blocks(a, b0 + lane, BK) : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, cum + incl > lo);
        if (hit) {
            const int l = __ffs(hit) - 1;
            c.b = b0 + l;
            c.nbv = __shfl_sync(0xffffffffu, v, l);
            c.blk = (int)(lo - (cum + __shfl_sync(0xffffffffu, incl, l) - c.nbv));
            return (int)(hi - lo);
        }
        cum += __shfl_sync(0xffffffffu, incl, 31);
    }
    c.b = a.B;
    c.blk = c.nbv = 0;
    return 0;
}
// Moves c forward by k items (sequences without complete past blocks are skipped).
__device__ __forceinline__ void scan_advance(const DecodeArgs& a, int BK, ScanCursor& c, int k) {
    c.blk += k;
    while (c.b < a.B && c.blk >= c.nbv) {
        c.blk -= c.nbv;
        if (++c.b < a.B) c.nbv = complete_blocks(a, c.b, BK);
    }
}

constexpr int kScanStages = 8;
constexpr int kScanWarps = 4;

template <int DI, int BK>
struct ScanSmem {
    alignas(1024) __nv_bfloat16 tile[kScanStages][BK * DI];
    uint64_t full[kScanStages], empty[kScanStages];
};

template <int DI, int BK>
__global__ void __launch_bounds__((kScanWarps + 1) * 32, 1)
    k_dec_scan(const __grid_constant__ CUtensorMap tm_kidx, DecodeArgs a, const __nv_bfloat16* __restrict__ q_idx) {
    using Sm = ScanSmem<DI, BK>;
    extern __shared__ uint8_t scan_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(scan_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = (a.L + BK - 1) / BK;
    if (threadIdx.x == 0) {
        for (int x = 0; x < kScanStages; ++x) {
            mbar_init(&s.full[x], 1);
            mbar_init(&s.empty[x], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();
    ScanCursor cur;
    const int count = scan_range(a, BK, cur);
    if (warp == kScanWarps) {
        if (lane == 0) {
            int n = 0;
            for (; n < count; ++n, scan_advance(a, BK, cur, 1)) {
                const int st = n % kScanStages;
                if (n >= kScanStages && !mbar_wait(&s.empty[st], ((n / kScanStages) - 1) & 1, a.status, 0x901)) break;
                mbar_arrive_expect_tx(&s.full[st], (uint32_t)(BK * DI * 2));
                tma_load_3d(s.tile[st], &tm_kidx, &s.full[st], 0, cur.blk * BK, cur.b);
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int m = max(0, n - kScanStages); m < n; ++m)
                mbar_wait(&s.full[m % kScanStages], (m / kScanStages) & 1, a.status, 0x902);
        }
        pdl_trigger();
        return;
    }
    // consumers: B fragments of Q_idx^T (k = dim, n = group; groups beyond H_kv are zero)
    const int g = lane >> 2, t4 = lane & 3;
    int cur_b = -1;
    uint32_t qb[DI / 16][2];
    scan_advance(a, BK, cur, warp);
    for (int n = warp; n < count; n += kScanWarps, scan_advance(a, BK, cur, kScanWarps)) {
        const int b = cur.b, blk = cur.blk;
        if (b != cur_b) {
            cur_b = b;
            const uint32_t* qrow = reinterpret_cast<const uint32_t*>(q_idx + ((size_t)b * a.H_kv + min(g, a.H_kv - 1)) * DI);
#pragma unroll
            for (int ks = 0; ks < DI / 16; ++ks) {
                qb[ks][0] = g < a.H_kv ? qrow[8 * ks + t4] : 0u;
                qb[ks][1] = g < a.H_kv ? qrow[8 * ks + 4 + t4] : 0u;
            }
        }
        const int st = n % kScanStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&s.full[st], (n / kScanStages) & 1, a.status, 0x903))) break;
        const uint32_t base = smem_u32(s.tile[st]);
        float m0 = -INFINITY, m1 = -INFINITY;  // groups 2*t4, 2*t4+1
#pragma unroll
        for (int mt = 0; mt < BK / 16; ++mt) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const int row = mt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
            for (int ks = 0; ks < DI / 16; ++ks) {
                uint32_t a4[4];
                const uint32_t addr = base + swz(row, (2 * ks + (lane >> 4)) * 16, DI * 2);
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(a4[0]), "=r"(a4[1]), "=r"(a4[2]), "=r"(a4[3])
                             : "r"(addr));
                mma_16816_bf16(acc, a4, qb[ks][0], qb[ks][1]);
            }
            m0 = fmaxf(m0, fmaxf(acc[0], acc[2]));
            m1 = fmaxf(m1, fmaxf(acc[1], acc[3]));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[st]);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        }
        if (lane < 4) {
            if (2 * t4 < a.H_kv) a.bmax[((size_t)b * a.H_kv + 2 * t4) * nb + blk] = m0;
            if (2 * t4 + 1 < a.H_kv) a.bmax[((size_t)b * a.H_kv + 2 * t4 + 1) * nb + blk] = m1;
        }
    }
    pdl_trigger();
}

// ------------------------------------------------------------------------------ FP8 index keys
// e4m3 helpers. Conversions go through cuda_fp8.h: float -> e4m3 rounds to nearest even and, with
// __NV_SATFINITE, clamps to +-448; e4m3 -> f16 is exact (every e4m3 value is an f16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}
__device__ __forceinline__ uint32_t e4m3_code(float x, float scale) {
    return (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(x, scale), __NV_SATFINITE, __NV_E4M3);
}
// Row scale max|x| / 448 (1 for an all-zero row), correctly rounded in fp32.
__device__ __forceinline__ float e4m3_row_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f; }

__device__ __forceinline__ void mma_16816_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Row-wise e4m3 quantisation (the serving copy of the index keys: keys kept in bf16 for training
// are quantised to FP8 for inference). Each row gets the scale max|x| / 448 and codes
// e4m3(x / scale). Threads own 8 consecutive elements; the NL = n / 8 threads of a row are
// consecutive lanes of one warp and combine their maxima by shuffles. HBM-bound.
template <int NL>
__global__ void __launch_bounds__(256) k_quant_e4m3_rows(const __nv_bfloat16* __restrict__ x, int64_t rows,
                                                         uint8_t* __restrict__ codes, float* __restrict__ scale) {
    const int64_t per_pass = (int64_t)gridDim.x * blockDim.x;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < rows * NL; t += per_pass) {
        const int64_t row = t / NL;
        const uint4 raw = *reinterpret_cast<const uint4*>(x + t * 8);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h[e]);
            v[2 * e] = f.x;
            v[2 * e + 1] = f.y;
        }
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
        // the NL lanes of a row are aligned within the warp (NL divides 32 and every pass moves by
        // whole rows), so they are active together; the last pass may leave other rows' lanes idle
        const int lane = threadIdx.x & 31;
        const uint32_t row_mask = (NL == 32 ? 0xffffffffu : ((1u << NL) - 1u)) << (lane & ~(NL - 1));
#pragma unroll
        for (int o = 1; o < NL; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(row_mask, amax, o));
        const float sc = e4m3_row_scale(amax);
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e >> 2] |= e4m3_code(v[e], sc) << (8 * (e & 3));
        *reinterpret_cast<uint2*>(codes + t * 8) = make_uint2(w[0], w[1]);
        if (t % NL == 0) scale[row] = sc;
    }
}

// FP8 index scan: the pass of k_dec_scan over every complete past block, reading K_idx as e4m3
// codes (DI bytes per token, half the bf16 bytes) plus one fp32 scale per token. Q_idx is rounded
// to e4m3 here with the row scale of k_quant_e4m3_rows, per (sequence, group). The score of token
// j for group r is scale_q[r] * scale_k[j] * (q8[r] . k8[j]).
// Each 16-byte chunk of a token's codes (16 dims) is one k=16 step of f16 mma.sync: e4m3 values
// are exact in f16, so every product is exact and only the fp32 accumulation rounds, as in the
// bf16 scan. ldmatrix gives each lane 4 consecutive dims (4*t4 .. 4*t4+3) of a chunk for its
// rows; they are widened into the A fragment's k slots (2*t4, 2*t4+1) and (8+2*t4, 9+2*t4), and
// Q's B fragment places the same dims in the same slots (a dot product only needs A and B to agree
// on which dim each k slot holds). The producer (one thread) streams the code tiles by TMA; each
// consumer warp loads the token scales of its next block itself (plain coalesced loads, one block
// ahead) and parks them in its own shared-memory row while it computes.
// Eight consumer warps and a 16-stage ring (128 KB of code tiles for 128-token blocks of 64 dims):
// at this tile size a CTA must keep more tiles in flight than the bf16 scan to reach the same HBM
// rate, and its per-tile compute (widening plus 32 MMAs) needs more warps to keep up.
constexpr int kScan8Warps = 8;
constexpr int kScan8Stages = 12;  // stages of two consecutive blocks each

template <int DI, int BK>
struct ScanSmem8 {
    alignas(1024) uint8_t tile[kScan8Stages][2 * BK * DI];  // [stage][block 2k, block 2k+1]
    float scale[kScan8Warps][BK];
    uint64_t full[kScan8Stages], empty[kScan8Stages];
};

template <int DI, int BK>
__global__ void __launch_bounds__((kScan8Warps + 1) * 32, 1)
    k_dec_scan_e4m3(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_codes2,
                    DecodeArgs a, const __nv_bfloat16* __restrict__ q_idx) {
    static_assert(DI % 32 == 0 && BK % 32 == 0, "chunk pairs and 32-row scale loads");
    // The CTA's blocks go in pairs: pair k (blocks 2k, 2k+1) uses stage k % stages, one 2*BK-token
    // TMA box when both are consecutive blocks of one sequence (the common case: half the copies of
    // one box per block), else one box per block. Block n goes to warp n % warps, so the two blocks
    // of a stage's next use belong to the same two warps and no warp can wait on a stage's full
    // barrier a phase early.
    static_assert((2 * kScan8Stages) % kScan8Warps == 0, "a stage's uses must cycle through the same warps");
    using Sm = ScanSmem8<DI, BK>;
    extern __shared__ uint8_t scan8_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(scan8_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nb = (a.L + BK - 1) / BK;
    if (threadIdx.x == 0) {
        for (int x = 0; x < kScan8Stages; ++x) {
            mbar_init(&s.full[x], 1);
            mbar_init(&s.empty[x], 2);  // the warps of the stage's two blocks (a last lone block: one, never reused)
        }
        fence_mbar_init();
    }
    __syncthreads();
    ScanCursor cur;
    const int count = scan_range(a, BK, cur);
    if (warp == kScan8Warps) {
        if (lane == 0) {
            int k = 0;
            for (int n = 0; n < count; n += 2, ++k) {
                const int st = k % kScan8Stages;
                if (k >= kScan8Stages && !mbar_wait(&s.empty[st], ((k / kScan8Stages) - 1) & 1, a.status, 0x911))
                    break;
                ScanCursor nxt = cur;
                scan_advance(a, BK, nxt, 1);  // block n + 1
                const bool two = n + 1 < count;
                mbar_arrive_expect_tx(&s.full[st], (uint32_t)((two ? 2 : 1) * BK * DI));
                if (two && nxt.b == cur.b && nxt.blk == cur.blk + 1) {
                    tma_load_3d(s.tile[st], &tm_codes2, &s.full[st], 0, cur.blk * BK, cur.b);
                } else {
                    tma_load_3d(s.tile[st], &tm_codes, &s.full[st], 0, cur.blk * BK, cur.b);
                    if (two) tma_load_3d(s.tile[st] + BK * DI, &tm_codes, &s.full[st], 0, nxt.blk * BK, nxt.b);
                }
                cur = nxt;
                scan_advance(a, BK, cur, 1);  // block n + 2
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int m = max(0, k - kScan8Stages); m < k; ++m)
                mbar_wait(&s.full[m % kScan8Stages], (m / kScan8Stages) & 1, a.status, 0x912);
        }
        pdl_trigger();
        return;
    }
    const int g = lane >> 2, t4 = lane & 3;
    int cur_b = -1;
    uint32_t qb[DI / 16][2];
    float sq0 = 0.f, sq1 = 0.f;  // Q scales of groups 2*t4 and 2*t4+1
    float scn[BK / 32];          // token scales of this warp's next block, rows lane + 32*x
    auto load_scales = [&](const ScanCursor& c) {
        const float* src = a.k_idx_scale + (size_t)c.b * a.L + (size_t)c.blk * BK;
#pragma unroll
        for (int x = 0; x < BK / 32; ++x) scn[x] = __ldg(src + lane + 32 * x);
    };
    scan_advance(a, BK, cur, warp);
    if (warp < count) load_scales(cur);
    for (int n = warp; n < count; n += kScan8Warps) {
        const int b = cur.b, blk = cur.blk;
        // park this block's scales, then start loading the next block's
#pragma unroll
        for (int x = 0; x < BK / 32; ++x) s.scale[warp][lane + 32 * x] = scn[x];
        __syncwarp();
        scan_advance(a, BK, cur, kScan8Warps);
        if (n + kScan8Warps < count) load_scales(cur);
        if (b != cur_b) {
            // Q_idx row of group g (zero for g >= H_kv): this lane's dims 16c + 4*t4 + {0..3}
            cur_b = b;
            const bool gv = g < a.H_kv;
            const __nv_bfloat16* qrow = q_idx + ((size_t)b * a.H_kv + min(g, a.H_kv - 1)) * DI;
            float qv[DI / 16][4];
            float amax = 0.f;
#pragma unroll
            for (int c = 0; c < DI / 16; ++c) {
                const uint2 raw = *reinterpret_cast<const uint2*>(qrow + 16 * c + 4 * t4);
                const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
                const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
                qv[c][0] = lo.x;
                qv[c][1] = lo.y;
                qv[c][2] = hi.x;
                qv[c][3] = hi.y;
#pragma unroll
                for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(qv[c][e]));
            }
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
            const float sq = e4m3_row_scale(amax);
#pragma unroll
            for (int c = 0; c < DI / 16; ++c) {
                const uint32_t c01 = e4m3_code(qv[c][0], sq) | (e4m3_code(qv[c][1], sq) << 8);
                const uint32_t c23 = e4m3_code(qv[c][2], sq) | (e4m3_code(qv[c][3], sq) << 8);
                qb[c][0] = gv ? e4m3x2_to_f16x2(c01) : 0u;
                qb[c][1] = gv ? e4m3x2_to_f16x2(c23) : 0u;
            }
            sq0 = __shfl_sync(0xffffffffu, sq, 8 * t4);      // lane of (group 2*t4, t4 = 0)
            sq1 = __shfl_sync(0xffffffffu, sq, 8 * t4 + 4);  // lane of (group 2*t4+1, t4 = 0)
        }
        const int pair = n >> 1, st = pair % kScan8Stages;
        if (!__all_sync(0xffffffffu, mbar_wait(&s.full[st], (pair / kScan8Stages) & 1, a.status, 0x913))) break;
        const uint32_t base = smem_u32(s.tile[st]) + (uint32_t)((n & 1) * BK * DI);  // this block's half
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int mt = 0; mt < BK / 16; ++mt) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            const int row = mt * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
            for (int cc = 0; cc < DI / 32; ++cc) {
                uint32_t r[4];
                const uint32_t addr = base + swz(row, (2 * cc + (lane >> 4)) * 16, DI);
                asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                             : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                             : "r"(addr));
                // r[0] / r[1]: rows g / g+8 of chunk 2*cc; r[2] / r[3]: the same rows of chunk 2*cc+1
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t a4[4] = {e4m3x2_to_f16x2(r[2 * h]), e4m3x2_to_f16x2(r[2 * h + 1]),
                                            e4m3x2_to_f16x2(r[2 * h] >> 16), e4m3x2_to_f16x2(r[2 * h + 1] >> 16)};
                    mma_16816_f16(acc, a4, qb[2 * cc + h][0], qb[2 * cc + h][1]);
                }
            }
            const float sk0 = s.scale[warp][mt * 16 + g], sk1 = s.scale[warp][mt * 16 + g + 8];
            m0 = fmaxf(m0, fmaxf(acc[0] * sk0, acc[2] * sk1));
            m1 = fmaxf(m1, fmaxf(acc[1] * sk0, acc[3] * sk1));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[st]);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        }
        if (lane < 4) {
            if (2 * t4 < a.H_kv) a.bmax[((size_t)b * a.H_kv + 2 * t4) * nb + blk] = m0 * sq0;
            if (2 * t4 + 1 < a.H_kv) a.bmax[((size_t)b * a.H_kv + 2 * t4 + 1) * nb + blk] = m1 * sq1;
        }
    }
    pdl_trigger();
}

// One CTA per (sequence, group): Top-k of the block maxima of the complete past blocks by
// (max desc, id asc), plus the local block; written ascending, -1 padded. Radix select: candidate c
// gets the 64-bit key (order-preserving bits of its max) << 32 | (0xffffffff - c), unique and
// larger for the block that ranks first. Byte by byte from the first byte where the smallest and
// largest keys differ (the bytes above it are common to all), a histogram finds the bin that holds
// the k-th largest key; once that boundary bin holds at most 256 keys, the keys of higher bins are
// taken and the boundary keys are ranked against each other directly.
__global__ void __launch_bounds__(256) k_dec_topk(DecodeArgs a) {
    constexpr int kMaxK = 16;
    constexpr int kList = 256;
    extern __shared__ unsigned long long s_key[];  // [blocks per sequence] (at most 8192)
    __shared__ int hist[256];
    __shared__ unsigned long long s_list[kList];
    __shared__ unsigned long long s_prefix;
    __shared__ int s_want, s_bin, s_cnt, s_nlist, s_p0;
    __shared__ unsigned long long s_kmin[8], s_kmax[8];
    __shared__ int chosen[kMaxK];
    pdl_wait();  // the block maxima come from the scan
    const int b = blockIdx.x / a.H_kv, r = blockIdx.x % a.H_kv;
    const int len = dec_len(a, b);
    if (threadIdx.x == 0 && r == 0 && len != a.cache_len[b]) raise_flag(a.status, MSA_DEV_BAD_BLOCK, 0x931);
    const int bi = (len - 1) / a.block_k;  // local block; candidates are 0 .. bi-1
    const int nb = (a.L + a.block_k - 1) / a.block_k;
    const float* vals = a.bmax + ((size_t)b * a.H_kv + r) * nb;
    const int K1 = a.topk + 1;
    const int take = min(a.topk, bi);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    unsigned long long kmin = ~0ull, kmax = 0ull;
    for (int c = tid; c < bi; c += blockDim.x) {
        const uint32_t u = __float_as_uint(vals[c]);
        const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
        const unsigned long long k = ((unsigned long long)ord << 32) | (0xffffffffu - (uint32_t)c);
        s_key[c] = k;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        kmin = min(kmin, (unsigned long long)__shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, (unsigned long long)__shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
        s_kmin[warp] = kmin;
        s_kmax[warp] = kmax;
    }
    __syncthreads();
    if (tid == 0) {
        for (int w = 1; w < 8; ++w) {
            kmin = min(kmin, s_kmin[w]);
            kmax = max(kmax, s_kmax[w]);
        }
        int p0 = 7;
        while (p0 > 0 && ((kmin ^ kmax) >> (8 * p0)) == 0) --p0;
        s_p0 = p0;
        s_prefix = p0 == 7 ? 0ull : (kmax >> (8 * (p0 + 1)));
        s_want = take;
        s_cnt = 0;
        s_nlist = 0;
    }
    __syncthreads();
    int p = s_p0;
    for (; take > 0; --p) {
        hist[tid] = 0;
        __syncthreads();
        const unsigned long long prefix = s_prefix;
        const int shift = 8 * p;
        for (int c = tid; c < bi; c += blockDim.x) {
            const unsigned long long k = s_key[c];
            if (p == 7 || (k >> (shift + 8)) == prefix) atomicAdd(&hist[(int)((k >> shift) & 255u)], 1);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l owns digits 255-8l .. 248-8l, visited from the top
            int cnt[8], sum = 0;
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                cnt[x] = hist[255 - 8 * lane - x];
                sum += cnt[x];
            }
            int above = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, above, o);
                if (lane >= o) above += t;
            }
            above -= sum;
            const int want = s_want;
            int run = above;
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                if (run < want && want <= run + cnt[x]) {
                    s_prefix = (prefix << 8) | (unsigned long long)(255 - 8 * lane - x);
                    s_want = want - run;
                    s_bin = cnt[x];
                }
                run += cnt[x];
            }
        }
        __syncthreads();
        if (s_bin <= kList || p == 0) break;
    }
    if (take > 0) {
        // keys above the boundary bin are taken; the boundary bin's keys are listed and ranked
        const unsigned long long P = s_prefix;
        const int shift = 8 * p;
        for (int c = tid; c < bi; c += blockDim.x) {
            const unsigned long long top = s_key[c] >> shift;
            if (top > P) chosen[atomicAdd(&s_cnt, 1)] = c;
            else if (top == P) s_list[atomicAdd(&s_nlist, 1)] = s_key[c];
        }
        __syncthreads();
        const int nlist = s_nlist, want = s_want;
        if (tid < nlist) {
            const unsigned long long mk = s_list[tid];
            int rank = 0;
            for (int j = 0; j < nlist; ++j) rank += s_list[j] > mk;
            if (rank < want) chosen[atomicAdd(&s_cnt, 1)] = (int)(0xffffffffu - (uint32_t)(mk & 0xffffffffu));
        }
    }
    __syncthreads();
    if (a.margin_out) {
        // cutoff margin r_(k) - r_(k+1) of the ranking (+inf when every candidate is taken): the
        // k-th key is the smallest chosen key, the (k+1)-th the largest key below it
        __shared__ unsigned long long s_kth, s_next[8];
        float* mo = a.margin_out + (size_t)b * a.H_kv + r;
        if (bi > a.topk) {
            if (tid == 0) {
                unsigned long long m = ~0ull;
                for (int x = 0; x < take; ++x) m = min(m, s_key[chosen[x]]);
                s_kth = m;
            }
            __syncthreads();
            const unsigned long long kth = s_kth;
            unsigned long long nx = 0ull;
            for (int c = tid; c < bi; c += blockDim.x) {
                const unsigned long long k = s_key[c];
                if (k < kth) nx = max(nx, k);
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) nx = max(nx, (unsigned long long)__shfl_xor_sync(0xffffffffu, nx, o));
            if (lane == 0) s_next[warp] = nx;
            __syncthreads();
            if (tid == 0) {
                for (int w = 1; w < 8; ++w) nx = max(nx, s_next[w]);
                const int id_k = (int)(0xffffffffu - (uint32_t)(kth & 0xffffffffu));
                const int id_k1 = (int)(0xffffffffu - (uint32_t)(nx & 0xffffffffu));
                *mo = (vals[id_k] - vals[id_k1]) * a.scale_idx;
            }
        } else if (tid == 0) {
            *mo = INFINITY;
        }
    }
    pdl_trigger();
    if (warp != 0) return;
    // the chosen ids plus the local block, ascending: each lane places its id by its rank
    const int n = take + 1;
    const int mine = lane < take ? chosen[lane] : (lane == take ? bi : 0x7fffffff);
    int rank = 0;
    for (int x = 0; x < n; ++x) rank += (__shfl_sync(0xffffffffu, mine, x) < mine);
    int32_t* out = a.sel + ((size_t)b * a.H_kv + r) * K1;
    int32_t* bo = a.blocks_out ? a.blocks_out + ((size_t)b * a.H_kv + r) * K1 : nullptr;
    if (lane < n) {
        out[rank] = mine;
        if (bo) bo[rank] = mine;
    } else if (lane < K1) {
        out[lane] = -1;
        if (bo) bo[lane] = -1;
    }
}

// Decode attention, persistent: one CTA per SM takes the (sequence, group, slot) items c, c + grid,
// ... of the selection. Warp 8 streams each item's K and V block and the group's Q rows by TMA
// (64-column boxes, 128B-swizzled) through a 3-stage ring; warps 0-7 compute the items: S = Q.K^T
// for the G heads (mma.sync with Q by ldmatrix, 16-token units spread over the warps), the softmax
// statistics (combined across warps in shared memory), P as bf16 in shared memory, then P.V split
// by output columns. With NG = 2 the eight warps form two groups of four that take alternate
// items, so two items' dependent mma.sync chains are in flight at once (groups have their own P
// tile, reduction rows and named barrier); NG = 1 keeps all eight on every item for G = 32, whose
// two 16-row Q tiles per stage leave no room for a second P tile. The slot's partial is normalised by the sum of the bf16-rounded P that the MMA
// multiplies, as in the prefill attention, with its LSE from the exact sum; k_dec_combine merges
// the slots.
constexpr int kAttnStages = 3;
constexpr int kAttnWarps = 8;

template <int D, int BK, int NG, int MT>
struct AttnSmem {
    alignas(1024) __nv_bfloat16 kv[kAttnStages][2][BK * D];  // [stage][K, V][D/64 halves of BK x 64]
    __nv_bfloat16 qt[kAttnStages][MT][16 * D];               // [stage][row tile][D/64 halves of 16 x 64]
    __nv_bfloat16 p[NG][16][BK + 8];                         // [group] P rows (heads) of one 16-row tile
    float red[NG][3][kAttnWarps / NG][16];                   // [group] per-warp maxima, exact sums, rounded sums
    uint64_t full[kAttnStages], empty[kAttnStages];
};

// byte offset of (row, column col) in a tile of D/64 swizzled halves of `rows` x 64 bf16
template <int ROWS>
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
    return (uint32_t)(col >> 6) * (ROWS * 128) + swz(row, (col & 63) * 2, 128);
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

template <int D, int BK, int NG, int MT>
__global__ void __launch_bounds__((kAttnWarps + 1) * 32, 1)
    k_dec_attn_tma(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, DecodeArgs a) {
    using Sm = AttnSmem<D, BK, NG, MT>;
    constexpr int GW = kAttnWarps / NG;          // warps per group
    constexpr int NU = BK / 16;                  // 16-token units
    constexpr int UPW = (NU + GW - 1) / GW;      // units per warp
    constexpr int DW = D / GW;                   // output columns per warp (8, 16 or 32)
    constexpr uint32_t kTileBytes = BK * D * 2;
    extern __shared__ uint8_t attn_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(attn_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t4 = lane & 3;
    const int G = a.H_q / a.H_kv;
    const int n_mt = (G + 15) / 16;
    const int K1 = a.topk + 1;
    const int n_items = a.B * a.H_kv * K1;
    if (threadIdx.x == 0) {
        for (int x = 0; x < kAttnStages; ++x) {
            mbar_init(&s.full[x], 1);
            mbar_init(&s.empty[x], GW);  // each warp of the consuming group releases the stage after its reads
        }
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();  // the selection comes from the Top-k
    if (warp == kAttnWarps) {
        if (lane == 0) {
            int n = 0;
            for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
                const int c = a.sel[it];  // items are numbered like the selection [B, H_kv, K1]
                if (c < 0) continue;
                const int st = n % kAttnStages;
                if (n >= kAttnStages && !mbar_wait(&s.empty[st], ((n / kAttnStages) - 1) & 1, a.status, 0x921)) break;
                mbar_arrive_expect_tx(&s.full[st], 2 * kTileBytes + (uint32_t)n_mt * 16 * D * 2);
                const int bs = it / K1, b = bs / a.H_kv, r = bs % a.H_kv;
#pragma unroll
                for (int h = 0; h < D / 64; ++h) {
                    tma_load_4d(&s.kv[st][0][h * BK * 64], &tm_k, &s.full[st], 64 * h, r, c * BK, b);
                    tma_load_4d(&s.kv[st][1][h * BK * 64], &tm_v, &s.full[st], 64 * h, r, c * BK, b);
                    for (int mt = 0; mt < n_mt; ++mt)
                        tma_load_2d(&s.qt[st][mt][h * 16 * 64], &tm_q, &s.full[st], 64 * h,
                                    b * a.H_q + r * G + 16 * mt);
                }
                ++n;
            }
            for (int m = max(0, n - kAttnStages); m < n; ++m)
                mbar_wait(&s.full[m % kAttnStages], (m / kAttnStages) & 1, a.status, 0x922);
        }
        pdl_trigger();
        return;
    }
    const float sl2 = a.scale * 1.4426950408889634f;
    const int grp = warp / GW, lw = warp % GW;  // this warp's group and its rank in the group
    const uint32_t bar = 1 + grp;               // the group's named barrier
    int n_all = 0;                              // selected items seen so far (both groups)
    // the next item's block and its sequence's length are loaded while this item runs
    int c_next = blockIdx.x < n_items ? a.sel[blockIdx.x] : -1;
    int len_next = blockIdx.x < n_items ? dec_len(a, (blockIdx.x / K1) / a.H_kv) : 1;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
        const int c = c_next, len = len_next;
        if (it + (int)gridDim.x < n_items) {
            c_next = a.sel[it + gridDim.x];
            len_next = dec_len(a, ((it + (int)gridDim.x) / K1) / a.H_kv);
        }
        float* lse_out = a.lse_part + (size_t)it * G;
        if (c < 0) {
            if (grp == 0)
                for (int h = lw * 32 + lane; h < G; h += GW * 32) lse_out[h] = -INFINITY;
            continue;
        }
        const int n = n_all++;  // the item's place in the stage ring
        if (n % NG != grp) continue;
        const int st = n % kAttnStages;
        const uint32_t kbase = smem_u32(&s.kv[st][0][0]), vbase = smem_u32(&s.kv[st][1][0]);
        float* o_out = a.o_part + (size_t)it * G * D;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&s.full[st], (n / kAttnStages) & 1, a.status, 0x923));
        // every warp learns whether any warp timed out
        if (bar_red_or(bar, GW * 32, !ok)) break;
        for (int mt = 0; mt < n_mt; ++mt) {
            const int h0 = mt * 16 + g, h1 = h0 + 8;
            const uint32_t qbase = smem_u32(&s.qt[st][mt][0]);
            // S (log2 units) of the warp's units; tokens past the query are -inf
            float sc[UPW][2][4];
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int j = 0; j < UPW; ++j) {
                const int u = lw + GW * j;
#pragma unroll
                for (int tl = 0; tl < 2; ++tl) sc[j][tl][0] = sc[j][tl][1] = sc[j][tl][2] = sc[j][tl][3] = 0.f;
                if (u < NU) {
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        uint32_t qa[4];
                        asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                                     : "=r"(qa[0]), "=r"(qa[1]), "=r"(qa[2]), "=r"(qa[3])
                                     : "r"(qbase + tile_off<16>((lane & 7) + 8 * ((lane >> 3) & 1),
                                                                16 * ks + 8 * (lane >> 4))));
#pragma unroll
                        for (int tl = 0; tl < 2; ++tl) {
                            const int t = 16 * u + 8 * tl + g;
                            uint32_t b0, b1;
                            asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b0) : "r"(kbase + tile_off<BK>(t, 16 * ks + 2 * t4)));
                            asm volatile("ld.shared.b32 %0, [%1];" : "=r"(b1) : "r"(kbase + tile_off<BK>(t, 16 * ks + 8 + 2 * t4)));
                            mma_16816_bf16(sc[j][tl], qa, b0, b1);
                        }
                    }
                }
#pragma unroll
                for (int tl = 0; tl < 2; ++tl) {
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
                s.red[grp][0][lw][g] = mx0;
                s.red[grp][0][lw][g + 8] = mx1;
            }
            bar_sync_named(bar, GW * 32);
            float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
            for (int w = 0; w < GW; ++w) {
                m0 = fmaxf(m0, s.red[grp][0][w][g]);
                m1 = fmaxf(m1, s.red[grp][0][w][g + 8]);
            }
            // P (bf16 into shared memory); l: exact sums, lr: sums of the rounded P
            float l0 = 0.f, l1 = 0.f, lr0 = 0.f, lr1 = 0.f;
#pragma unroll
            for (int j = 0; j < UPW; ++j) {
                const int u = lw + GW * j;
                if (u >= NU) continue;
#pragma unroll
                for (int tl = 0; tl < 2; ++tl) {
                    float p[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        p[e] = sc[j][tl][e] == -INFINITY ? 0.f : exp2f(sc[j][tl][e] - (e < 2 ? m0 : m1));
                        if (e < 2) l0 += p[e]; else l1 += p[e];
                    }
                    const uint32_t w0 = pack_bf16x2(p[0], p[1]), w1 = pack_bf16x2(p[2], p[3]);
                    lr0 += __uint_as_float(w0 << 16) + __uint_as_float(w0 & 0xffff0000u);
                    lr1 += __uint_as_float(w1 << 16) + __uint_as_float(w1 & 0xffff0000u);
                    const int col = 16 * u + 8 * tl + 2 * t4;
                    *reinterpret_cast<uint32_t*>(&s.p[grp][g][col]) = w0;
                    *reinterpret_cast<uint32_t*>(&s.p[grp][g + 8][col]) = w1;
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
                s.red[grp][1][lw][g] = l0;
                s.red[grp][1][lw][g + 8] = l1;
                s.red[grp][2][lw][g] = lr0;
                s.red[grp][2][lw][g + 8] = lr1;
            }
            bar_sync_named(bar, GW * 32);
            // O[:, this warp's DW columns] = P.V over all tokens, even and odd units in two
            // accumulator sets (two independent MMA chains)
            float ov[DW / 8][4], ow[DW / 8][4];
#pragma unroll
            for (int nd = 0; nd < DW / 8; ++nd)
                ov[nd][0] = ov[nd][1] = ov[nd][2] = ov[nd][3] = ow[nd][0] = ow[nd][1] = ow[nd][2] = ow[nd][3] = 0.f;
#pragma unroll
            for (int u = 0; u < NU; ++u) {
                float (&acc)[DW / 8][4] = (u & 1) ? ow : ov;
                uint32_t pa[4];
                {
                    const int prow = ((lane >> 3) & 1) * 8 + (lane & 7), pcol = 16 * u + 8 * (lane >> 4);
                    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                                 : "=r"(pa[0]), "=r"(pa[1]), "=r"(pa[2]), "=r"(pa[3])
                                 : "r"(smem_u32(&s.p[grp][prow][pcol])));
                }
                const int vrow = 16 * u + 8 * ((lane >> 3) & 1) + (lane & 7);
                if constexpr (DW >= 16) {
#pragma unroll
                    for (int np = 0; np < DW / 16; ++np) {
                        uint32_t b00, b01, b10, b11;
                        ldsm_x4_trans(vbase + tile_off<BK>(vrow, lw * DW + 16 * np + 8 * (lane >> 4)), b00, b01, b10, b11);
                        mma_16816_bf16(acc[2 * np], pa, b00, b01);
                        mma_16816_bf16(acc[2 * np + 1], pa, b10, b11);
                    }
                } else {
                    uint32_t b00, b01;
                    ldsm_x2_trans(vbase + tile_off<BK>(vrow, lw * DW), b00, b01);
                    mma_16816_bf16(acc[0], pa, b00, b01);
                }
            }
            // this warp's last read of the stage is done: release it after the last row tile
            if (mt == n_mt - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive_relaxed(&s.empty[st]);
            }
#pragma unroll
            for (int nd = 0; nd < DW / 8; ++nd)
#pragma unroll
                for (int e = 0; e < 4; ++e) ov[nd][e] += ow[nd][e];
            float L0 = 0.f, L1 = 0.f, Lr0 = 0.f, Lr1 = 0.f;
#pragma unroll
            for (int w = 0; w < GW; ++w) {
                L0 += s.red[grp][1][w][g];
                L1 += s.red[grp][1][w][g + 8];
                Lr0 += s.red[grp][2][w][g];
                Lr1 += s.red[grp][2][w][g + 8];
            }
            const float i0 = 1.f / Lr0, i1 = 1.f / Lr1;
#pragma unroll
            for (int nd = 0; nd < DW / 8; ++nd) {
                const int col = lw * DW + 8 * nd + 2 * t4;
                if (h0 < G) *reinterpret_cast<float2*>(o_out + (size_t)h0 * D + col) = make_float2(ov[nd][0] * i0, ov[nd][1] * i0);
                if (h1 < G) *reinterpret_cast<float2*>(o_out + (size_t)h1 * D + col) = make_float2(ov[nd][2] * i1, ov[nd][3] * i1);
            }
            if (lw == 0 && t4 == 0) {
                if (h0 < G) lse_out[h0] = m0 * 0.6931471805599453f + logf(L0);
                if (h1 < G) lse_out[h1] = m1 * 0.6931471805599453f + logf(L1);
            }
            // the group's P tile and reduction rows are rewritten only after the next row tile's (or
            // the group's next item's) first barrier, which every warp of the group reaches after its
            // reads here
        }
    }
    pdl_trigger();
}

// One warp per (sequence, head): merge the slot partials ("2.4" page eq (18)). Lane s holds slot s's
// LSE (at most 32 slots); the max and the weights come from warp shuffles, and every slot's partial
// load is issued before the first is used.
template <int D>
__global__ void k_dec_combine(DecodeArgs a, float* __restrict__ out) {
    constexpr int kMaxK1 = 17;
    const int w = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= a.B * a.H_q) return;
    const int G = a.H_q / a.H_kv;
    const int K1 = a.topk + 1;
    const int b = w / a.H_q, h = w % a.H_q, r = h / G, hg = h % G;
    const size_t bs = (size_t)b * a.H_kv + r;
    pdl_wait();  // the partials come from the attention
    const float my_l = lane < K1 ? a.lse_part[(bs * K1 + lane) * G + hg] : -INFINITY;
    float mx = my_l;
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float my_w = my_l == -INFINITY ? 0.f : __expf(my_l - mx);
    float z = my_w;
#pragma unroll
    for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    constexpr int kPer = D / 32;
    float ov[kMaxK1][kPer];
#pragma unroll
    for (int s = 0; s < kMaxK1; ++s) {
        const float* op = a.o_part + ((bs * K1 + s) * G + hg) * D + lane * kPer;
        const bool live = s < K1 && __shfl_sync(0xffffffffu, my_w, s) > 0.f;
#pragma unroll
        for (int x = 0; x < kPer; ++x) ov[s][x] = live ? op[x] : 0.f;
    }
    float acc[kPer];
#pragma unroll
    for (int x = 0; x < kPer; ++x) acc[x] = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxK1; ++s) {
        const float ws = __shfl_sync(0xffffffffu, my_w, s);
#pragma unroll
        for (int x = 0; x < kPer; ++x) acc[x] = fmaf(ws, ov[s][x], acc[x]);
    }
    const float inv = 1.f / z;
    float* o = out + ((size_t)b * a.H_q + h) * D + lane * kPer;
#pragma unroll
    for (int x = 0; x < kPer; ++x) o[x] = acc[x] * inv;
}

}  // namespace

cudaError_t run_quantize_e4m3_rows(const void* x, int64_t rows, int n, uint8_t* codes, float* scale, int num_sms,
                                   cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    ProfScope ps("quant_e4m3_rows", st);
    const auto* xb = static_cast<const __nv_bfloat16*>(x);
    const int64_t threads = rows * (n / 8);
    const int grid = (int)std::min<int64_t>((threads + 255) / 256, (int64_t)num_sms * 8);
    switch (n) {
        case 16: k_quant_e4m3_rows<2><<<grid, 256, 0, st>>>(xb, rows, codes, scale); break;
        case 32: k_quant_e4m3_rows<4><<<grid, 256, 0, st>>>(xb, rows, codes, scale); break;
        case 64: k_quant_e4m3_rows<8><<<grid, 256, 0, st>>>(xb, rows, codes, scale); break;
        case 128: k_quant_e4m3_rows<16><<<grid, 256, 0, st>>>(xb, rows, codes, scale); break;
        case 256: k_quant_e4m3_rows<32><<<grid, 256, 0, st>>>(xb, rows, codes, scale); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

size_t decode_ws_bytes(int B, int L, int H_q, int H_kv, int d, int block_k, int topk) {
    const size_t nb = (size_t)(L + block_k - 1) / block_k;
    const size_t G = (size_t)H_q / H_kv, K1 = (size_t)topk + 1;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    return al((size_t)B * H_kv * nb * 4) + al((size_t)B * H_kv * K1 * 4) + al((size_t)B * H_kv * K1 * G * d * 4) +
           al((size_t)B * H_kv * K1 * G * 4);
}

cudaError_t run_decode(const DecodeArgs& a, const void* q, const void* q_idx, const void* k_cache,
                       const void* v_cache, const void* k_idx_cache, void* out, int num_sms, cudaStream_t st) {
    const auto* qi = static_cast<const __nv_bfloat16*>(q_idx);
    if (a.k_idx_scale) {
        ProfScope ps("dec_scan_e4m3", st);
        CUtensorMap tm, tm2;  // boxes of one block and of two consecutive blocks
        if (!make_tmap_3d_u8(&tm, k_idx_cache, (uint64_t)a.d_idx, (uint64_t)a.L, (uint64_t)a.B, (uint64_t)a.d_idx,
                             (uint64_t)a.L * a.d_idx, (uint32_t)a.d_idx, (uint32_t)a.block_k, a.d_idx) ||
            !make_tmap_3d_u8(&tm2, k_idx_cache, (uint64_t)a.d_idx, (uint64_t)a.L, (uint64_t)a.B, (uint64_t)a.d_idx,
                             (uint64_t)a.L * a.d_idx, (uint32_t)a.d_idx, (uint32_t)(2 * a.block_k), a.d_idx))
            return cudaErrorInvalidValue;
        auto launch = [&](auto kern, size_t bytes) -> cudaError_t {
            const size_t smem = bytes + 1024;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            kern<<<num_sms, (kScan8Warps + 1) * 32, smem, st>>>(tm, tm2, a, qi);
            return cudaGetLastError();
        };
        cudaError_t e;
        if (a.d_idx == 64)
            e = a.block_k == 128 ? launch(k_dec_scan_e4m3<64, 128>, sizeof(ScanSmem8<64, 128>))
                : a.block_k == 64 ? launch(k_dec_scan_e4m3<64, 64>, sizeof(ScanSmem8<64, 64>))
                                  : launch(k_dec_scan_e4m3<64, 32>, sizeof(ScanSmem8<64, 32>));
        else
            e = a.block_k == 128 ? launch(k_dec_scan_e4m3<32, 128>, sizeof(ScanSmem8<32, 128>))
                : a.block_k == 64 ? launch(k_dec_scan_e4m3<32, 64>, sizeof(ScanSmem8<32, 64>))
                                  : launch(k_dec_scan_e4m3<32, 32>, sizeof(ScanSmem8<32, 32>));
        if (e != cudaSuccess) return e;
    } else {
        ProfScope ps("dec_scan", st);
        CUtensorMap tm;
        if (!make_tmap_3d(&tm, k_idx_cache, (uint64_t)a.d_idx, (uint64_t)a.L, (uint64_t)a.B, (uint64_t)a.d_idx * 2,
                          (uint64_t)a.L * a.d_idx * 2, (uint32_t)a.d_idx, (uint32_t)a.block_k, 1, a.d_idx * 2))
            return cudaErrorInvalidValue;
        auto launch = [&](auto kern, size_t bytes) -> cudaError_t {
            const size_t smem = bytes + 1024;
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            kern<<<num_sms, (kScanWarps + 1) * 32, smem, st>>>(tm, a, qi);
            return cudaGetLastError();
        };
        cudaError_t e;
        if (a.d_idx == 64)
            e = a.block_k == 128 ? launch(k_dec_scan<64, 128>, sizeof(ScanSmem<64, 128>))
                : a.block_k == 64 ? launch(k_dec_scan<64, 64>, sizeof(ScanSmem<64, 64>))
                                  : launch(k_dec_scan<64, 32>, sizeof(ScanSmem<64, 32>));
        else
            e = a.block_k == 128 ? launch(k_dec_scan<32, 128>, sizeof(ScanSmem<32, 128>))
                : a.block_k == 64 ? launch(k_dec_scan<32, 64>, sizeof(ScanSmem<32, 64>))
                                  : launch(k_dec_scan<32, 32>, sizeof(ScanSmem<32, 32>));
        if (e != cudaSuccess) return e;
    }
    {
        ProfScope ps("dec_topk", st);
        const size_t ksmem = (size_t)((a.L + a.block_k - 1) / a.block_k) * sizeof(unsigned long long);
        cudaError_t e = cudaFuncSetAttribute(k_dec_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ksmem);
        if (e != cudaSuccess) return e;
        e = launch_pdl(k_dec_topk, dim3(a.B * a.H_kv), dim3(256), ksmem, st, a);
        if (e != cudaSuccess) return e;
    }
    ProfScope ps("dec_attn_combine", st);
    CUtensorMap tk, tv, tq;
    const uint64_t dims[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.L, (uint64_t)a.B};
    const uint64_t strides[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2, (uint64_t)a.L * a.H_kv * a.d * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)a.block_k, 1};
    if (!make_tmap_4d(&tk, k_cache, dims, strides, box, 128) || !make_tmap_4d(&tv, v_cache, dims, strides, box, 128) ||
        !make_tmap_2d(&tq, q, (uint64_t)a.d, (uint64_t)a.B * a.H_q, (uint64_t)a.d * 2, 64, 16, 128))
        return cudaErrorInvalidValue;
    auto launch = [&](auto kern, size_t bytes) -> cudaError_t {
        const size_t smem = bytes + 1024;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, dim3(num_sms), dim3((kAttnWarps + 1) * 32), smem, st, tk, tv, tq, a);
    };
    // two consumer groups when one 16-row Q tile holds the group's heads, else one (G = 32)
    auto launch_nm = [&](auto d_c, auto bk_c) -> cudaError_t {
        constexpr int D = decltype(d_c)::value, BK = decltype(bk_c)::value;
        if (a.H_q / a.H_kv <= 16) return launch(k_dec_attn_tma<D, BK, 2, 1>, sizeof(AttnSmem<D, BK, 2, 1>));
        return launch(k_dec_attn_tma<D, BK, 1, 2>, sizeof(AttnSmem<D, BK, 1, 2>));
    };
    using I64 = std::integral_constant<int, 64>;
    using I128 = std::integral_constant<int, 128>;
    using I32 = std::integral_constant<int, 32>;
    cudaError_t e;
    if (a.d == 128)
        e = a.block_k == 128 ? launch_nm(I128{}, I128{}) : a.block_k == 64 ? launch_nm(I128{}, I64{}) : launch_nm(I128{}, I32{});
    else
        e = a.block_k == 128 ? launch_nm(I64{}, I128{}) : a.block_k == 64 ? launch_nm(I64{}, I64{}) : launch_nm(I64{}, I32{});
    if (e != cudaSuccess) return e;
    const dim3 cgrid((a.B * a.H_q * 32 + 255) / 256);
    e = a.d == 128 ? launch_pdl(k_dec_combine<128>, cgrid, dim3(256), 0, st, a, static_cast<float*>(out))
                   : launch_pdl(k_dec_combine<64>, cgrid, dim3(256), 0, st, a, static_cast<float*>(out));
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace msa
