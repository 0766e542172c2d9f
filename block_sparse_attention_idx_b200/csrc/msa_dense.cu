// Dense warm-up of the KL alignment ("MSA 中的 KL 对齐与局部知识蒸馏", section 5: before sparse
// training the index branch is aligned to a teacher over the whole causal context; "2.4 · 训练原生
// 稀疏", section 3.2). With k covering every block the selected set J of query i is all of j <= i,
// so the teacher LSE is that of dense causal attention and the KL kernels run on dense lists.
//
// k_dense_lse: the teacher's per-head log-sum-exp over all causal keys, query-outer. A tile is
// 128 rows = 128/G queries x their G heads of one group (the queries of a tile lie in one key block,
// so only the tile's last block needs the causal mask). Warp 8 loads the tile's Q rows once and
// streams the K blocks 0 .. last through a 3-stage ring by TMA; warp 9 issues S = Q K_c^T (tcgen05,
// M = 128 rows, N = block_k, K = d) into one of two TMEM buffers; two teams of four warps take
// alternate blocks, one thread per row, each keeping a running (max, sum of exp) of its blocks; the
// two teams' pairs meet in shared memory at the end of the tile.
//
// k_dense_lists: the inverse lists of the dense selection (list (b, r, c) = queries c*block_k .. N-1
// in order, cut into items of qpc queries), in the layout the sparse KL and LSE_idx kernels read;
// entries carry the query in the upper bits (i << 5), the block itself is the slot.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kRows = 128;
constexpr int kTeams = 2;
constexpr int kProdWarp = 4 * kTeams, kMmaWarp = 4 * kTeams + 1;
constexpr int kThreads = (4 * kTeams + 2) * 32;
constexpr int kKStages = 3;

__device__ __forceinline__ bool wait_lane(uint64_t* bar, uint32_t parity, DevStatus* st, unsigned where) {
    int ok = 1;
    if (lane_id() == 0) ok = mbar_wait(bar, parity, st, where);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <int D, int BK>
struct DenseSmem {
    static constexpr int kQBytes = kRows * D * 2;
    static constexpr int kKBytes = BK * D * 2;
    alignas(1024) uint8_t q[2][kQBytes];
    alignas(1024) uint8_t k[kKStages][kKBytes];
    float red_m[2][kRows], red_l[2][kRows];  // team 1's running pair, per tile parity
    uint64_t q_full[2], q_empty[2], k_full[kKStages], k_empty[kKStages];
    // red_bar[p]: team 1's pair of a tile of parity p is in; red_ack[p]: team 0 has read it
    uint64_t s_full[kTeams], s_free[kTeams], red_bar[2], red_ack[2], drain;
    uint32_t tmem_base;
    int abort;
};

// Tiles in decreasing length (queries late in the sequence have the most blocks): tile u of the
// CTA's sequence is global tile blockIdx.x + u * gridDim.x.
struct DenseTile {
    int b, r, q0, nq, nblk;
};
__device__ __forceinline__ DenseTile dense_tile(const DenseLseArgs& a, int t) {
    const int QPT = kRows / a.G;
    const int nQT = (a.N + QPT - 1) / QPT;
    const int bh = t % (a.B * a.H_kv);
    const int qt = nQT - 1 - t / (a.B * a.H_kv);
    DenseTile d;
    d.b = bh / a.H_kv;
    d.r = bh % a.H_kv;
    d.q0 = qt * QPT;
    d.nq = min(QPT, a.N - d.q0);
    d.nblk = (d.q0 + d.nq - 1) / a.block_k + 1;
    return d;
}

// Column pairs of every 8 whose exponentials the teacher-LSE loop computes on the FMA pipe.
constexpr int kPolyOf8 = 2;

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1)
    k_dense_lse(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __nv_bfloat16* __restrict__ q, DenseLseArgs a) {
    using Sm = DenseSmem<D, BK>;
    extern __shared__ uint8_t smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kIdesc = umma_idesc_bf16(kRows, BK, false, false);
    const int G = a.G;
    const int QPT = kRows / G;
    const int nQT = (a.N + QPT - 1) / QPT;
    const int T = a.B * a.H_kv * nQT;
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s.q_full[x], 1);
            mbar_init(&s.q_empty[x], 1);
            mbar_init(&s.red_bar[x], 4);
            mbar_init(&s.red_ack[x], 4);
        }
        for (int x = 0; x < kKStages; ++x) {
            mbar_init(&s.k_full[x], 1);
            mbar_init(&s.k_empty[x], 1);
        }
        for (int x = 0; x < kTeams; ++x) {
            mbar_init(&s.s_full[x], 1);
            mbar_init(&s.s_free[x], 4);
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&s.tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ Q tile, K ring
        int kc = 0, n = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < T && ok; t += gridDim.x, ++n) {
            const DenseTile d = dense_tile(a, t);
            const int qb = n & 1;
            if (!wait_lane(&s.q_empty[qb], ((n >> 1) & 1) ^ 1, a.status, 0xb01)) { ok = false; break; }
            if (G % 8 == 0) {
                if (lane == 0) mbar_arrive_expect_tx_relaxed(&s.q_full[qb], (uint32_t)(d.nq * G * D * 2));
                __syncwarp();
                for (int m = lane; m < d.nq; m += 32)
                    tma_load_5d(s.q[qb] + m * G * D * 2, &tm_q, &s.q_full[qb], 0, 0, 0, d.r * G / 8,
                                d.b * a.N + d.q0 + m);
            } else {
                const uint32_t qsm = smem_u32(s.q[qb]);
                constexpr int kChunksPerRow = D * 2 / 16;
                for (int x = lane; x < d.nq * G * kChunksPerRow; x += 32) {
                    const int row = x / kChunksPerRow, ch = x % kChunksPerRow;
                    const int m = row / G, h = row % G;
                    const __nv_bfloat16* src =
                        q + ((((size_t)d.b * a.N + d.q0 + m) * a.H_q + (size_t)d.r * G + h) * D + ch * 8);
                    cp_async_16(qsm + qtile_off<D>(row, ch * 16), src);
                }
                cp_async_wait_all();
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.q_full[qb]);
            }
            for (int c = 0; c < d.nblk; ++c, ++kc) {
                const int st = kc % kKStages;
                if (!wait_lane(&s.k_empty[st], ((kc / kKStages) & 1) ^ 1, a.status, 0xb02)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx_relaxed(&s.k_full[st], (uint32_t)Sm::kKBytes);
#pragma unroll
                    for (int sub = 0; sub < D / 64; ++sub)
                        tma_load_4d(s.k[st] + sub * BK * 128, &tm_k, &s.k_full[st], sub * 64, d.r, c * BK, d.b);
                }
                __syncwarp();
            }
        }
        if (!ok) s.abort = 1;
        if (lane == 0) {  // no copy of ours may still be landing when the CTA leaves
            for (int x = max(0, kc - kKStages); x < kc; ++x)
                mbar_wait(&s.k_full[x % kKStages], (x / kKStages) & 1, a.status, 0xb03);
            for (int x = max(0, n - 2); x < n; ++x) mbar_wait(&s.q_full[x & 1], (x >> 1) & 1, a.status, 0xb04);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ S = Q K_c^T
        if (lane == 0) {
            int kc = 0, n = 0, sc = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < T && ok; t += gridDim.x, ++n) {
                const DenseTile d = dense_tile(a, t);
                const int qb = n & 1;
                if (!mbar_wait(&s.q_full[qb], (n >> 1) & 1, a.status, 0xb11)) { ok = false; break; }
                for (int c = 0; c < d.nblk; ++c, ++kc, ++sc) {
                    const int st = kc % kKStages, sb = sc % kTeams;
                    if (!mbar_wait(&s.k_full[st], (kc / kKStages) & 1, a.status, 0xb12) ||
                        !mbar_wait(&s.s_free[sb], ((sc / kTeams) & 1) ^ 1, a.status, 0xb13)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t qa = smem_u32(s.q[qb]), ka = smem_u32(s.k[st]);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t sub = (ks * 16) / 64, off = (ks & 3) * 32;
                        const uint64_t da = umma_sdesc(qa + sub * 1024 + off, 16, (D / 64) * 1024, 2);
                        const uint64_t db = umma_sdesc(ka + sub * (BK * 128) + off, 16, 1024, 2);
                        umma_bf16(tmem + sb * 128, da, db, kIdesc, ks > 0);
                    }
                    umma_commit(&s.s_full[sb]);
                    umma_commit(&s.k_empty[st]);
                }
                if (ok) umma_commit(&s.q_empty[qb]);
            }
            if (!ok) s.abort = 1;
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, a.status, 0xb14);
        }
    } else {
        // ------------------------------------------------------------ running (max, sum of exp)
        // Team tm handles the tile's blocks c with (sc % 2) == tm, where sc counts the CTA's S
        // products; thread = row (query m = row / G, head h = row % G).
        const int tm = warp >> 2, qtr = warp & 3;
        const int row = qtr * 32 + lane;
        const uint32_t tS = tmem + ((uint32_t)(qtr * 32) << 16) + tm * 128;
        const float sl2 = a.scale * 1.4426950408889634f;
        int sc = 0, n = 0, mine = 0;  // mine: S products of this team so far
        bool ok = true;
        for (int t = blockIdx.x; t < T && ok; t += gridDim.x, ++n) {
            const DenseTile d = dense_tile(a, t);
            const int m = row / G, h = row % G;
            const bool valid = m < d.nq;
            const int i = d.q0 + (valid ? m : 0);
            float mx = -INFINITY, l = 0.f;
            for (int c = 0; c < d.nblk; ++c, ++sc) {
                if (sc % kTeams != tm) continue;
                if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full[tm], mine & 1, a.status, 0xb21))) {
                    ok = false;
                    break;
                }
                ++mine;
                tc_fence_after();
                uint32_t sv[BK];
#pragma unroll
                for (int c0 = 0; c0 < BK; c0 += 32) tmem_ld32p(tS + c0, sv + c0);
                tmem_ld_wait();
                reg_fence(sv);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.s_free[tm]);
                const int lim = valid ? i - c * BK : -1;  // columns x <= lim are causal
                if (__any_sync(0xffffffffu, lim < BK - 1)) {
#pragma unroll
                    for (int x = 0; x < BK; ++x) sv[x] = x <= lim ? sv[x] : 0xff800000u;
                }
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int x = 0; x < BK; x += 2)
                    m4[(x >> 1) & 3] = max3f(m4[(x >> 1) & 3], __uint_as_float(sv[x]), __uint_as_float(sv[x + 1]));
                const float bm = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                // a row without a causal column here (a later query block of the tile) adds nothing:
                // its masked scores give exp2(-inf) = 0 around a finite reference
                const float mn = fmaxf(mx, bm);
                const float mref = mn == -INFINITY ? 0.f : mn;
                const uint64_t sl2x2 = f2_packf(sl2, sl2), moffx2 = f2_packf(-mref * sl2, -mref * sl2);
                uint64_t acc[2] = {f2_packf(0.f, 0.f), f2_packf(0.f, 0.f)};
                // the MUFU pipe bounds this loop: kPolyOf8 of every 8 column pairs take their
                // exponentials on the FMA pipe instead
#pragma unroll
                for (int y = 0; y < BK; y += 2) {
                    const uint64_t xx = f2_fma(f2_pack(sv[y], sv[y + 1]), sl2x2, moffx2);
                    uint64_t ex;
                    if (((y >> 1) & 7) < kPolyOf8) {
                        ex = exp2_fma_x2(xx);
                    } else {
                        float x0, x1;
                        f2_unpack(xx, x0, x1);
                        ex = f2_packf(fast_exp2(x0), fast_exp2(x1));
                    }
                    acc[(y >> 1) & 1] = f2_add(acc[(y >> 1) & 1], ex);
                }
                float a0, a1, a2, a3;
                f2_unpack(acc[0], a0, a1);
                f2_unpack(acc[1], a2, a3);
                l = (mx == -INFINITY ? 0.f : l * fast_exp2((mx - mref) * sl2)) + ((a0 + a1) + (a2 + a3));
                mx = mn;
            }
            if (!ok) break;
            // team 1 hands its pair to team 0, which merges and stores the row's LSE
            const int pb = n & 1;
            if (tm == 1) {
                // the pair of the tile two before, in the same slot, has been read by team 0
                if (n >= 2 && !__all_sync(0xffffffffu, mbar_wait(&s.red_ack[pb], ((n >> 1) & 1) ^ 1, a.status, 0xb23))) {
                    ok = false;
                    break;
                }
                s.red_m[pb][row] = mx;
                s.red_l[pb][row] = l;
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.red_bar[pb]);
            } else {
                if (!__all_sync(0xffffffffu, mbar_wait(&s.red_bar[pb], (n >> 1) & 1, a.status, 0xb22))) {
                    ok = false;
                    break;
                }
                const float m1 = s.red_m[pb][row], l1 = s.red_l[pb][row];
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.red_ack[pb]);
                const float M = fmaxf(mx, m1);
                float L = 0.f;
                if (mx != -INFINITY) L += l * fast_exp2((mx - M) * sl2);
                if (m1 != -INFINITY) L += l1 * fast_exp2((m1 - M) * sl2);
                if (valid) a.lse[((size_t)d.b * a.N + i) * a.H_q + (size_t)d.r * G + h] = M * a.scale + logf(L);
            }
        }
        if (!ok) s.abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 256);
}

template <int D, int BK>
cudaError_t launch_dense_lse(const DenseLseArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const void* q,
                             int num_sms, cudaStream_t st) {
    const size_t smem = sizeof(DenseSmem<D, BK>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_dense_lse<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("dense_lse", st);
    k_dense_lse<D, BK><<<num_sms, kThreads, smem, st>>>(tq, tk, static_cast<const __nv_bfloat16*>(q), a);
    return cudaGetLastError();
}

// One CTA per list (b, r, c): its items (chunks of qpc consecutive queries) and its entries, written
// by the CTA's threads in order. Entry and item offsets of list c within its (b, r) are sums over the
// lists before it.
__global__ void __launch_bounds__(256) k_dense_lists(int N, int block_k, int qpc, int nb, long long ents_per_bh,
                                                     long long items_per_bh, int4* items, int32_t* entries,
                                                     int write_entries) {
    const long long L = blockIdx.x;
    const int c = (int)(L % nb);
    const long long bh = L / nb;
    long long e0 = bh * ents_per_bh, i0 = bh * items_per_bh;
    for (int cc = 0; cc < c; ++cc) {
        const int cnt = N - cc * block_k;
        e0 += cnt;
        i0 += (cnt + qpc - 1) / qpc;
    }
    const int cnt = N - c * block_k;
    for (int k = threadIdx.x; k * qpc < cnt; k += blockDim.x)
        items[i0 + k] = make_int4((int)L, (int)(e0 + (long long)k * qpc), min(qpc, cnt - k * qpc), 0);
    if (write_entries)
        for (int x = threadIdx.x; x < cnt; x += blockDim.x) entries[e0 + x] = (c * block_k + x) << 5;
}

__global__ void k_set_count(int32_t* dst, int32_t v) { *dst = v; }

}  // namespace

void dense_list_sizes(int B, int N, int H_kv, int block_k, int qpc, long long* entries, long long* items) {
    const int nb = (N + block_k - 1) / block_k;
    long long e = 0, it = 0;
    for (int c = 0; c < nb; ++c) {
        const int cnt = N - c * block_k;
        e += cnt;
        it += (cnt + qpc - 1) / qpc;
    }
    *entries = e * B * H_kv;
    *items = it * B * H_kv;
}

cudaError_t run_dense_lists(const Csr& cs, int B, int N, int H_kv, int block_k, int qpc, bool write_entries,
                            cudaStream_t st) {
    long long e = 0, it = 0;
    dense_list_sizes(1, N, 1, block_k, qpc, &e, &it);
    const long long lists = (long long)B * H_kv * cs.nb;
    k_dense_lists<<<(unsigned)lists, 256, 0, st>>>(N, block_k, qpc, cs.nb, e, it, cs.items, cs.entries,
                                                   write_entries ? 1 : 0);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    k_set_count<<<1, 1, 0, st>>>(cs.n_items, (int32_t)(it * B * H_kv));
    return cudaGetLastError();
}

bool dense_lse_supported(int d, int block_k, int G) {
    return (d == 64 || d == 128) && (block_k == 32 || block_k == 64 || block_k == 128) && G >= 2 && 128 % G == 0;
}

cudaError_t run_dense_lse(const DenseLseArgs& a, const void* q, const void* k, int num_sms, cudaStream_t st) {
    CUtensorMap tq, tk;
    const uint64_t dkv[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t skv[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2, (uint64_t)a.N * a.H_kv * a.d * 2};
    const uint32_t bkv[4] = {64, 1, (uint32_t)a.block_k, 1};
    if (!make_tmap_4d(&tk, k, dkv, skv, bkv, 128)) return cudaErrorInvalidValue;
    if (a.G % 8 == 0) {
        if (!make_tmap_qrows(&tq, q, a.B, a.N, a.H_q, a.d, a.G)) return cudaErrorInvalidValue;
    } else {
        tq = tk;  // not read: the query rows are copied without TMA
    }
    if (a.d == 128) {
        if (a.block_k == 128) return launch_dense_lse<128, 128>(a, tq, tk, q, num_sms, st);
        if (a.block_k == 64) return launch_dense_lse<128, 64>(a, tq, tk, q, num_sms, st);
        return launch_dense_lse<128, 32>(a, tq, tk, q, num_sms, st);
    }
    if (a.block_k == 128) return launch_dense_lse<64, 128>(a, tq, tk, q, num_sms, st);
    if (a.block_k == 64) return launch_dense_lse<64, 64>(a, tq, tk, q, num_sms, st);
    return launch_dense_lse<64, 32>(a, tq, tk, q, num_sms, st);
}

}  // namespace msa
