// Main branch of MSA: exact softmax attention over the selected blocks, KV-outer
// (MSA blog, KV-outer sparse attention and hot blocks; "2.4 · 训练原生稀疏", eq (2) and the
// online-softmax partition merge eq (18)).
//
// A work item is one selected KV block c of group r plus up to 128/G queries of one 128-query
// window that selected it; their G query heads form the 128 rows of the tile. Per item:
//   S = Q_rows . K_c^T        tcgen05.mma, M=128 rows, N=block_k tokens, K=d        -> TMEM
//   P = exp(S*scale - max)    epilogue warpgroup, one row per thread; causal mask j <= i;
//                             P (bf16) is written back into TMEM over the S columns already read
//   O = P . V_c               tcgen05.mma with A = P from TMEM, B = V_c (MN-major)  -> TMEM
// The normalised partial (o = O / sum P, lse) of every row goes to its (query, head, slot) place
// in the workspace (fp16 o, fp32 lse). Each (query, group) row counts its finished items; the item
// that finishes last hands the row to the merge warps, which combine the row's <= topk+1 partials
// with the log-sum-exp rule, write the bf16 output and the LSE, and discard the partial lines from
// L2. Items are handed out in (window, group, block) order by an atomic counter, four at a time, so
// the partials of a window are produced and merged while they are still in L2 and consecutive items
// of a CTA often share their K/V block.
//
// Warp roles (480 threads): warps 0-3 and 4-7 are two epilogue warpgroups taking alternate items
// (each owns one S/P and one O accumulator in TMEM), warp 8 hands out items (prefetching the next
// item's record and query list), stages their metadata and loads Q (TMA gather of each query's G head
// rows) and K, warp 9 loads V, warp 10 issues the MMAs and owns TMEM, warps 11-14 merge finished rows.
// Q, K and V are double-buffered; the MMA issuer polls and issues whichever of the next S or the
// next PV is ready.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kThreads = 480;
constexpr int kRows = 128;
constexpr int kMeta = 4;        // depth of the item metadata ring
constexpr int kGrab = 4;        // items taken per scheduler fetch
constexpr int kMergeWarps = 4;  // warps 11..14
constexpr int kMQ = 256;        // merge task ring
constexpr int kEpiWarps = 8;

struct ItemMeta {
    int t;  // item index; -1: no more items
    int b, r, c, count, kv_new;
    int qi[kRows];
    int8_t qs[kRows];  // query index and selection slot of each item query
};

struct MergeTask {
    int b, i, r;
    volatile int full;  // generation (k / kMQ + 1) of the task stored here
    volatile int done;  // generation of the last task consumed from here
};

template <int D, int BK>
struct AttnSmem {
    static constexpr int kQBytes = kRows * D * 2;   // D/64 sub-tiles of [128 rows x 128 B]
    static constexpr int kKVBytes = BK * D * 2;     // D/64 sub-tiles of [BK rows x 128 B]
    alignas(1024) uint8_t q[2][kQBytes];
    alignas(1024) uint8_t k[2][kKVBytes];
    alignas(1024) uint8_t v[2][kKVBytes];
    ItemMeta meta[kMeta];
    MergeTask mq[kMQ];
    int mq_tail;
    int epi_done;
    uint64_t meta_full[kMeta], meta_empty[kMeta];
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[2], k_release[2], v_full[2], v_release[2];  // release[b]: one completion per use of buffer b
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool wait_lane0(uint64_t* bar, uint32_t parity, DevStatus* st, unsigned where) {
    int ok = 1;
    if (lane_id() == 0) ok = mbar_wait(bar, parity, st, where);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ void discard_l2(const void* p) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_kv_outer(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ q, AttnArgs a) {
    using Sm = AttnSmem<D, BK>;
    extern __shared__ uint8_t smem_raw[];
    Sm& s = *reinterpret_cast<Sm*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    constexpr uint32_t kIdescS = umma_idesc_bf16(kRows, BK, false, false);
    constexpr uint32_t kIdescO = umma_idesc_bf16(kRows, D, false, true);

    const int G = a.H_q / a.H_kv;
    const int K1 = a.topk + 1;
    const int T = *a.csr.n_items;
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int x = 0; x < kMeta; ++x) {
            mbar_init(&s.meta_full[x], 1);
            mbar_init(&s.meta_empty[x], 2 + kRows);  // V loader, MMA issuer, one epilogue warpgroup
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s.q_full[x], 1);
            mbar_init(&s.q_empty[x], 1);
            mbar_init(&s.k_full[x], 1);
            mbar_init(&s.v_full[x], 1);
            mbar_init(&s.s_full[x], 1);
            mbar_init(&s.p_full[x], kRows);
            mbar_init(&s.o_full[x], 1);
            mbar_init(&s.o_free[x], kRows);
            mbar_init(&s.k_release[x], 1);
            mbar_init(&s.v_release[x], 1);
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        s.mq_tail = 0;
        s.epi_done = 0;
        fence_mbar_init();
    }
    for (int x = threadIdx.x; x < kMQ; x += blockDim.x) {
        s.mq[x].full = 0;
        s.mq[x].done = 0;
    }
    if (warp == 10) {
        tmem_alloc(&s.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == 8) {
        // ------------------------------------------------------------ items, metadata, Q and K
        // The record and query list of the next item are loaded one item ahead, so their global
        // latency overlaps the waits of the current item.
        int prevL = -1, kgroup = -1;
        bool ok = true;
        int batch = 0;
        if (lane == 0) batch = atomicAdd(a.sched, kGrab);
        batch = __shfl_sync(0xffffffffu, batch, 0);
        int t_nx = batch;
        int4 rec_nx = t_nx < T ? a.csr.items[t_nx] : make_int4(-1, 0, 0, 0);
        int e_nx[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = lane + 32 * j;
            e_nx[j] = (t_nx < T && m < rec_nx.z) ? a.csr.entries[rec_nx.y + m] : 0;
        }
        for (int n = 0;; ++n) {
            const int t = t_nx;
            const int4 rec = rec_nx;
            int e[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) e[j] = e_nx[j];
            // prefetch item n+1
            if ((n + 1) % kGrab == 0) {
                int b2 = 0;
                if (lane == 0) b2 = atomicAdd(a.sched, kGrab);
                batch = __shfl_sync(0xffffffffu, b2, 0);
                t_nx = batch;
            } else {
                t_nx = batch + (n + 1) % kGrab;
            }
            if (t_nx < T) {
                rec_nx = a.csr.items[t_nx];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int m = lane + 32 * j;
                    e_nx[j] = m < rec_nx.z ? a.csr.entries[rec_nx.y + m] : 0;
                }
            }
            const int slot = n % kMeta;
            if (!wait_lane0(&s.meta_empty[slot], ((n / kMeta) & 1) ^ 1, a.status, 0x501)) { ok = false; break; }
            ItemMeta& mt = s.meta[slot];
            if (t >= T || s.abort) {
                // two end markers: one for each epilogue warpgroup
                if (lane == 0) { mt.t = -1; mbar_arrive(&s.meta_full[slot]); }
                const int slot2 = (n + 1) % kMeta;
                if (!wait_lane0(&s.meta_empty[slot2], (((n + 1) / kMeta) & 1) ^ 1, a.status, 0x502)) { ok = false; break; }
                if (lane == 0) { s.meta[slot2].t = -1; mbar_arrive(&s.meta_full[slot2]); }
                break;
            }
            const int L = rec.x, count = rec.z;
            const int c = L % a.csr.nb;
            const int r = (L / a.csr.nb) % a.H_kv;
            const int b = L / (a.csr.nb * a.H_kv * a.csr.nW);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int m = lane + 32 * j;
                if (m < count) {
                    mt.qi[m] = e[j] >> 5;
                    mt.qs[m] = (int8_t)(e[j] & 31);
                }
            }
            if (lane == 0) {
                mt.t = t; mt.b = b; mt.r = r; mt.c = c; mt.count = count; mt.kv_new = (L != prevL);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.meta_full[slot]);
            // Q: the G head rows of each query of the item
            const int buf = n & 1;
            if (!wait_lane0(&s.q_empty[buf], ((n >> 1) & 1) ^ 1, a.status, 0x503)) { ok = false; break; }
            if (G >= 8) {
                if (lane == 0) mbar_arrive_expect_tx(&s.q_full[buf], (uint32_t)(count * G * D * 2));
                __syncwarp();
                for (int m = lane; m < count; m += 32) {
#pragma unroll
                    for (int sub = 0; sub < D / 64; ++sub)
                        tma_load_4d(s.q[buf] + sub * (kRows * 128) + m * G * 128, &tm_q, &s.q_full[buf], sub * 64,
                                    r * G, mt.qi[m], b);
                }
            } else {
                const uint32_t qsm = smem_u32(s.q[buf]);
                constexpr int kChunksPerRow = D * 2 / 16;
                for (int x = lane; x < count * G * kChunksPerRow; x += 32) {
                    const int row = x / kChunksPerRow, ch = x % kChunksPerRow;
                    const int m = row / G, h = row % G;
                    const __nv_bfloat16* src =
                        q + ((((size_t)b * a.N + mt.qi[m]) * a.H_q + (size_t)r * G + h) * D + ch * 8);
                    cp_async_16(qsm + ((ch * 16) / 128) * (kRows * 128) + swz(row, (ch * 16) % 128, 128), src);
                }
                cp_async_wait_all();
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.q_full[buf]);
            }
            // K of block group g goes to buffer g % 2 once the S MMAs of group g-2 (the buffer's
            // previous use, release number (g-2)/2 of that buffer) are done
            if (L != prevL) {
                ++kgroup;
                if (kgroup >= 2 &&
                    !wait_lane0(&s.k_release[kgroup & 1], ((kgroup - 2) >> 1) & 1, a.status, 0x504)) { ok = false; break; }
                if (lane == 0) {
                    const int kb = kgroup & 1;
                    mbar_arrive_expect_tx(&s.k_full[kb], (uint32_t)Sm::kKVBytes);
#pragma unroll
                    for (int sub = 0; sub < D / 64; ++sub)
                        tma_load_4d(s.k[kb] + sub * BK * 128, &tm_k, &s.k_full[kb], sub * 64, r, c * BK, b);
                }
                prevL = L;
            }
        }
        if (!ok) s.abort = 1;
        if (lane == 0) {  // no copy of ours may still be landing when the CTA leaves
            for (int g = max(0, kgroup - 1); g <= kgroup; ++g) mbar_wait(&s.k_full[g & 1], (g >> 1) & 1, a.status, 0x505);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ V loader
        int vgroup = -1;
        bool ok = true;
        for (int n = 0;; ++n) {
            const int slot = n % kMeta;
            if (!wait_lane0(&s.meta_full[slot], (n / kMeta) & 1, a.status, 0x511)) { ok = false; break; }
            const ItemMeta& mt = s.meta[slot];
            const int t = mt.t, b = mt.b, r = mt.r, c = mt.c, kv_new = mt.kv_new;
            __syncwarp();
            if (lane == 0 && t >= 0) mbar_arrive(&s.meta_empty[slot]);
            if (t < 0) break;
            if (kv_new) {
                // V of block group g goes to buffer g % 2 once the PV MMAs of group g-2 are done
                ++vgroup;
                if (vgroup >= 2 &&
                    !wait_lane0(&s.v_release[vgroup & 1], ((vgroup - 2) >> 1) & 1, a.status, 0x512)) { ok = false; break; }
                if (lane == 0) {
                    const int vb = vgroup & 1;
                    mbar_arrive_expect_tx(&s.v_full[vb], (uint32_t)Sm::kKVBytes);
#pragma unroll
                    for (int sub = 0; sub < D / 64; ++sub)
                        tma_load_4d(s.v[vb] + sub * BK * 128, &tm_v, &s.v_full[vb], sub * 64, r, c * BK, b);
                }
            }
        }
        if (!ok) s.abort = 1;
        if (lane == 0) {
            for (int g = max(0, vgroup - 1); g <= vgroup; ++g) mbar_wait(&s.v_full[g & 1], (g >> 1) & 1, a.status, 0x513);
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ MMA issuer
        // S(ns) needs its metadata, Q, its K buffer, and PV(ns-2) issued (P(ns-2) lives in the TMEM
        // columns S(ns) overwrites; MMAs of one thread execute in issue order). PV(np) needs P(np),
        // its V buffer and the O accumulator freed by the epilogue. Both are polled; whichever is
        // ready goes first.
        if (lane == 0) {
            bool ok = true;
            int ns = 0, np = 0, n_end = -1;
            bool meta_read = false;
            int cur_kvn = 0, cur_grp = -1;
            int groups = -1;          // block groups seen so far (metadata order)
            int pend_pv = -1;         // PV issued whose item's successor group was not yet known
            int grp_ring[kMeta] = {0, 0, 0, 0};
            uint64_t t_idle = globaltimer();
            while (true) {
                bool progressed = false;
                if (n_end < 0) {
                    if (!meta_read && mbar_test(&s.meta_full[ns % kMeta], (ns / kMeta) & 1)) {
                        const int t = s.meta[ns % kMeta].t;
                        cur_kvn = s.meta[ns % kMeta].kv_new;
                        if (t < 0) {
                            n_end = ns;
                        } else {
                            mbar_arrive(&s.meta_empty[ns % kMeta]);
                            meta_read = true;
                            if (cur_kvn) {
                                ++groups;
                                if (ns > 0) {
                                    // item ns-1 closed block group groups-1: every S of it has been
                                    // issued, so its K buffer is free once they complete
                                    umma_commit(&s.k_release[(groups - 1) & 1]);
                                }
                            }
                            cur_grp = groups;
                            // a PV waiting to learn whether it closed its group
                            if (pend_pv >= 0 && pend_pv == ns - 1) {
                                if (cur_kvn) umma_commit(&s.v_release[grp_ring[pend_pv % kMeta] & 1]);
                                pend_pv = -1;
                            }
                        }
                        progressed = true;
                    }
                    if (meta_read && np >= ns - 1 && mbar_test(&s.q_full[ns & 1], (ns >> 1) & 1) &&
                        mbar_test(&s.k_full[cur_grp & 1], (cur_grp >> 1) & 1)) {
                        tc_fence_after();
                        const uint32_t qb = smem_u32(s.q[ns & 1]), kb = smem_u32(s.k[cur_grp & 1]);
                        const uint32_t tS = tmem + (ns & 1) * 256;
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t sub = (ks * 16) / 64, off = (ks & 3) * 32;
                            const uint64_t da = umma_sdesc(qb + sub * (kRows * 128) + off, 16, 1024, 2);
                            const uint64_t db = umma_sdesc(kb + sub * (BK * 128) + off, 16, 1024, 2);
                            umma_bf16(tS, da, db, kIdescS, ks > 0);
                        }
                        umma_commit(&s.s_full[ns & 1]);
                        umma_commit(&s.q_empty[ns & 1]);
                        grp_ring[ns % kMeta] = cur_grp;
                        ++ns;
                        meta_read = false;
                        progressed = true;
                    }
                }
                if (np < ns && mbar_test(&s.p_full[np & 1], (np >> 1) & 1) &&
                    mbar_test(&s.o_free[np & 1], ((np >> 1) & 1) ^ 1)) {
                    const int g = grp_ring[np % kMeta];
                    if (mbar_test(&s.v_full[g & 1], (g >> 1) & 1)) {
                        tc_fence_after();
                        const uint32_t vb = smem_u32(s.v[g & 1]);
                        const uint32_t tP = tmem + (np & 1) * 256;        // P (bf16 pairs) over S
                        const uint32_t tO = tmem + (np & 1) * 256 + 128;
#pragma unroll
                        for (int ks = 0; ks < BK / 16; ++ks) {
                            const uint64_t db = umma_sdesc(vb + ks * 16 * 128, BK * 128, 1024, 2);
                            umma_bf16_tmem_a(tO, tP + ks * 8, db, kIdescO, ks > 0);
                        }
                        umma_commit(&s.o_full[np & 1]);
                        // if item np closed its block group, its V buffer is free once this PV is done
                        if (np + 1 < ns) {
                            if (grp_ring[(np + 1) % kMeta] != g) umma_commit(&s.v_release[g & 1]);
                        } else if (np + 1 == ns && meta_read) {
                            if (cur_grp != g) umma_commit(&s.v_release[g & 1]);
                        } else {
                            pend_pv = np;
                        }
                        ++np;
                        progressed = true;
                    }
                }
                if (n_end >= 0 && np == n_end) break;
                if (progressed) {
                    t_idle = globaltimer();
                } else {
                    __nanosleep(20);
                }
                if (!progressed && globaltimer() - t_idle > MSA_WAIT_NS) {
                    raise_flag(a.status, MSA_DEV_TIMEOUT, 0x601);
                    ok = false;
                    break;
                }
            }
            if (!ok) s.abort = 1;
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, a.status, 0x608);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax / epilogue
        const int wg = warp >> 2;                  // epilogue warpgroup: items n = wg, wg+2, ...
        const int row = threadIdx.x - wg * 128;    // TMEM lane
        const int m = row / G, h = row % G;
        const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const uint32_t tS = lane_addr + wg * 256, tO = lane_addr + wg * 256 + 128;
        const float sl2 = a.scale * 1.4426950408889634f;
        // Row counting runs two items behind the stores it publishes: the increment for item n is
        // issued during item n+1 (its release then finds item n's partial stores long performed) and
        // its returned count is looked at during item n+2.
        bool inc = false, chk = false;
        int inc_nsel = 0, inc_b = 0, inc_i = 0, inc_r = 0;
        int chk_old = 0, chk_nsel = 0, chk_b = 0, chk_i = 0, chk_r = 0;
        auto push_task = [&](int tb, int ti, int tr, unsigned where) {
            const int k = atomicAdd(&s.mq_tail, 1);
            MergeTask& task = s.mq[k % kMQ];
            const int gen = k / kMQ;
            const uint64_t t0 = globaltimer();
            while (task.done != gen) {  // the slot's previous task must have been taken
                if (globaltimer() - t0 > MSA_WAIT_NS) {
                    raise_flag(a.status, MSA_DEV_TIMEOUT, where);
                    break;
                }
                __nanosleep(64);
            }
            task.b = tb;
            task.i = ti;
            task.r = tr;
            __threadfence_block();
            task.full = gen + 1;
        };
        for (int n = wg;; n += 2) {
            const int slot = n % kMeta;
            if (!__all_sync(0xffffffffu, mbar_wait(&s.meta_full[slot], (n / kMeta) & 1, a.status, 0x701))) {
                s.abort = 1;
                break;
            }
            const ItemMeta& mt = s.meta[slot];
            const int t = mt.t;
            if (t < 0) break;
            const int b = mt.b, r = mt.r, c = mt.c;
            const bool valid = m < mt.count;
            const int i = valid ? mt.qi[m] : 0;
            const int qslot = valid ? (int)mt.qs[m] : 0;
            mbar_arrive(&s.meta_empty[slot]);
            const int lim = valid ? i - c * BK : -1;  // columns j <= lim are causal for this row
            const int my_nsel = (valid && h == 0) ? (int)a.csr.nsel[((size_t)b * a.N + i) * a.H_kv + r] : 0;
            const int kk = n >> 1;                     // this warpgroup's item count
            if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full[wg], kk & 1, a.status, 0x702))) {
                s.abort = 1;
                break;
            }
            tc_fence_after();
            // pass 1: row max over the causal columns (two TMEM loads per wait)
            const bool full = __all_sync(0xffffffffu, lim >= BK - 1);  // whole item causal-complete
            float mx = -INFINITY;
#pragma unroll 1
            for (int c0 = 0; c0 < BK; c0 += 64) {
                uint32_t ra[32], rb2[32];
                tmem_ld32(tS + c0, ra);
                if (BK > 32) tmem_ld32(tS + c0 + 32, rb2);
                tmem_ld_wait();
                if (full) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) mx = fmaxf(mx, __uint_as_float(ra[x]));
                    if (BK > 32) {
#pragma unroll
                        for (int x = 0; x < 32; ++x) mx = fmaxf(mx, __uint_as_float(rb2[x]));
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < 32; ++x) mx = (c0 + x <= lim) ? fmaxf(mx, __uint_as_float(ra[x])) : mx;
                    if (BK > 32) {
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            mx = (c0 + 32 + x <= lim) ? fmaxf(mx, __uint_as_float(rb2[x])) : mx;
                    }
                }
            }
            const float moff = valid ? mx * sl2 : 0.f;
            // pass 2: P = exp(S - max) rounded to bf16, packed two per TMEM column over the S
            // columns already read. l: exact sum for the LSE; lr: sum of the rounded weights the
            // MMA uses, so that o = (P_bf16 . V) / lr stays a convex combination of the V rows.
            float l = 0.f, lr = 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < BK; c0 += 32) {
                uint32_t r32[32];
                tmem_ld32(tS + c0, r32);
                tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int y = 0; y < 32; y += 2) {
                    float p0 = fast_exp2(fmaf(__uint_as_float(r32[y]), sl2, -moff));
                    float p1 = fast_exp2(fmaf(__uint_as_float(r32[y + 1]), sl2, -moff));
                    if (!full) {
                        p0 = (c0 + y <= lim) ? p0 : 0.f;
                        p1 = (c0 + y + 1 <= lim) ? p1 : 0.f;
                    }
                    const __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
                    const uint32_t u = *reinterpret_cast<const uint32_t*>(&pb2);
                    l += p0 + p1;
                    lr += __uint_as_float(u << 16) + __uint_as_float(u & 0xffff0000u);
                    pk[y / 2] = u;
                }
                tmem_st16(tS + c0 / 2, pk);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&s.p_full[wg]);
            // rows whose count came back complete go to the merge warps; then count the previous item
            if (chk) {
                if (chk_old + 1 == chk_nsel) push_task(chk_b, chk_i, chk_r, 0x706);
                chk = false;
            }
            if (inc) {
                chk_old = atom_add_acq_rel_gpu(&a.counter[((size_t)inc_b * a.N + inc_i) * a.H_kv + inc_r], 1);
                chk_nsel = inc_nsel;
                chk_b = inc_b;
                chk_i = inc_i;
                chk_r = inc_r;
                chk = true;
                inc = false;
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&s.o_full[wg], kk & 1, a.status, 0x704))) {
                s.abort = 1;
                break;
            }
            tc_fence_after();
            const int hq = r * G + h;
            const size_t prow = (((size_t)b * a.N + i) * a.H_q + hq) * K1 + qslot;
            const float inv = valid ? 1.f / lr : 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 64) {
                uint32_t ra[32], rb2[32];
                tmem_ld32(tO + c0, ra);
                tmem_ld32(tO + c0 + 32, rb2);
                tmem_ld_wait();
                if (valid) {
                    uint32_t hv[32];
#pragma unroll
                    for (int x = 0; x < 32; x += 2) {
                        const __half2 h0 = __floats2half2_rn(__uint_as_float(ra[x]) * inv, __uint_as_float(ra[x + 1]) * inv);
                        const __half2 h1 =
                            __floats2half2_rn(__uint_as_float(rb2[x]) * inv, __uint_as_float(rb2[x + 1]) * inv);
                        hv[x / 2] = *reinterpret_cast<const uint32_t*>(&h0);
                        hv[16 + x / 2] = *reinterpret_cast<const uint32_t*>(&h1);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(a.o_part + prow * D + c0);
#pragma unroll
                    for (int x = 0; x < 8; ++x) dst[x] = make_uint4(hv[4 * x], hv[4 * x + 1], hv[4 * x + 2], hv[4 * x + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&s.o_free[wg]);
            if (valid) a.lse_part[prow] = mx * a.scale + logf(l);
            // ---- this item counts for its (query, group) rows. The warp barrier orders the G lanes'
            // partial stores before their leader's later acquire-release increment.
            __syncwarp();
            if (valid && h == 0) {
                inc_nsel = my_nsel;
                inc_b = b;
                inc_i = i;
                inc_r = r;
                inc = true;
            }
        }
        // flush the rows still being counted
        if (chk && chk_old + 1 == chk_nsel) push_task(chk_b, chk_i, chk_r, 0x707);
        if (inc) {
            const int old = atom_add_acq_rel_gpu(&a.counter[((size_t)inc_b * a.N + inc_i) * a.H_kv + inc_r], 1);
            if (old + 1 == inc_nsel) push_task(inc_b, inc_i, inc_r, 0x707);
        }
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            atomicAdd(&s.epi_done, 1);
        }
    } else if (warp >= 11 && warp < 11 + kMergeWarps) {
        // ------------------------------------------------------------ merge warps
        // Task k (a finished (query, group) row) belongs to merge warp k % kMergeWarps. Lanes take
        // units of 8 output values of one head; each unit loads the LSEs and the fp16 partials of all
        // the row's slots at once, then combines them with the log-sum-exp rule.
        const int mw = warp - 11;
        const int units = G * (D / 8);
        for (int k = mw;; k += kMergeWarps) {
            MergeTask& task = s.mq[k % kMQ];
            const int gen = k / kMQ;
            int have = 0;
            if (lane == 0) {
                const uint64_t t0 = globaltimer();
                while (true) {
                    if (task.full == gen + 1) { have = 1; break; }
                    if (*(volatile int*)&s.epi_done == kEpiWarps && k >= *(volatile int*)&s.mq_tail) break;
                    if (globaltimer() - t0 > MSA_WAIT_NS) {
                        raise_flag(a.status, MSA_DEV_TIMEOUT, 0x801);
                        break;
                    }
                    __nanosleep(128);
                }
            }
            have = __shfl_sync(0xffffffffu, have, 0);
            if (!have) break;
            __threadfence();
            const int b = task.b, i = task.i, r = task.r;
            __syncwarp();
            if (lane == 0) task.done = gen + 1;
            // valid slots of the row (same rule as the list builder)
            const int32_t* sel = a.blocks + (((size_t)b * a.N + i) * a.H_kv + r) * K1;
            // slot x is kept when its block is causal and above every kept block before it; the
            // largest kept block so far equals the largest in-range block so far (prefix max)
            const int cb = lane < K1 ? __ldg(sel + lane) : -1;
            const bool inr = cb >= 0 && cb <= i / BK;
            int pm = inr ? cb : -1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, pm, o);
                if (lane >= o) pm = max(pm, t);
            }
            int prev = __shfl_up_sync(0xffffffffu, pm, 1);
            if (lane == 0) prev = -1;
            const uint32_t vmask = __ballot_sync(0xffffffffu, inr && cb > prev);
            constexpr int kK1Max = 17;
            bool overflow = false;
            for (int u = lane; u < units; u += 32) {
                const int hh = u / (D / 8), d0 = (u % (D / 8)) * 8;
                const int hq = r * G + hh;
                const size_t rb = (((size_t)b * a.N + i) * a.H_q + hq) * K1;
                float lv[kK1Max];
                uint4 ov[kK1Max];
#pragma unroll
                for (int x = 0; x < kK1Max; ++x) {
                    if (vmask & (1u << x)) {
                        lv[x] = __ldcg(a.lse_part + rb + x);
                        ov[x] = __ldcg(reinterpret_cast<const uint4*>(a.o_part + (rb + x) * D + d0));
                    } else {
                        lv[x] = -INFINITY;
                        ov[x] = make_uint4(0, 0, 0, 0);
                    }
                }
                float lmax = -INFINITY;
#pragma unroll
                for (int x = 0; x < kK1Max; ++x) lmax = fmaxf(lmax, lv[x]);
                float z = 0.f, acc[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
                for (int x = 0; x < kK1Max; ++x) {
                    const float w = lv[x] == -INFINITY ? 0.f : __expf(lv[x] - lmax);
                    z += w;
                    const __half2* h2 = reinterpret_cast<const __half2*>(&ov[x]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __half22float2(h2[e]);
                        acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
                        acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
                    }
                }
                const float zi = 1.f / z;
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    overflow |= !isfinite(acc[2 * e]) || !isfinite(acc[2 * e + 1]);
                    pk[e] = pack_bf16x2(acc[2 * e] * zi, acc[2 * e + 1] * zi);
                }
                *reinterpret_cast<uint4*>(a.out + (((size_t)b * a.N + i) * a.H_q + hq) * D + d0) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
                if (a.lse && d0 == 0) a.lse[((size_t)b * a.N + i) * a.H_q + hq] = lmax + logf(z);
            }
            // fp16 partials overflow when entries of V exceed the fp16 range: report it
            if (overflow) raise_flag(a.status, MSA_DEV_BAD_BLOCK, 0x802);
            __syncwarp();
            // the partials of this row are consumed: drop their lines from L2 without write-back
            const int lines = D * 2 / 128;
            for (int x = lane; x < G * kK1Max * lines; x += 32) {
                const int hh = x / (kK1Max * lines), sl = (x / lines) % kK1Max, ln = x % lines;
                if (!(vmask & (1u << sl))) continue;
                const size_t rb = (((size_t)b * a.N + i) * a.H_q + r * G + hh) * K1 + sl;
                discard_l2(reinterpret_cast<const uint8_t*>(a.o_part + rb * D) + 128 * ln);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 10) tmem_dealloc(tmem, 512);
}

template <int D, int BK>
cudaError_t launch_attn(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const void* q, int grid, cudaStream_t st) {
    const size_t smem = std::max<size_t>(sizeof(AttnSmem<D, BK>) + 1024, 116 * 1024);  // one CTA per SM
    cudaError_t e =
        cudaFuncSetAttribute(k_attn_kv_outer<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    ProfScope ps("attn_kv_outer", st);
    k_attn_kv_outer<D, BK><<<grid, kThreads, smem, st>>>(tq, tk, tv, static_cast<const __nv_bfloat16*>(q), a);
    return cudaGetLastError();
}

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t attn_ws_bytes(int B, int N, int H_q, int H_kv, int d, int block_k, int topk) {
    const size_t pr = (size_t)B * N * H_q * (topk + 1);
    return csr_bytes(B, N, H_kv, block_k, topk, kAttnWindow) + al256(pr * d * sizeof(__half)) +
           al256(pr * sizeof(float)) + al256((size_t)B * N * H_kv * 4) + 256;
}

void attn_carve(AttnArgs* a, void* base) {
    uint8_t* p = static_cast<uint8_t*>(base);
    csr_carve(&a->csr, p, a->B, a->N, a->H_kv, a->block_k, a->topk, kAttnWindow);
    p += csr_bytes(a->B, a->N, a->H_kv, a->block_k, a->topk, kAttnWindow);
    const size_t pr = (size_t)a->B * a->N * a->H_q * (a->topk + 1);
    a->o_part = reinterpret_cast<__half*>(p);
    p += al256(pr * a->d * sizeof(__half));
    a->lse_part = reinterpret_cast<float*>(p);
    p += al256(pr * sizeof(float));
    a->counter = reinterpret_cast<int32_t*>(p);
    p += al256((size_t)a->B * a->N * a->H_kv * 4);
    a->sched = reinterpret_cast<int32_t*>(p);
}

cudaError_t run_attn(const AttnArgs& a, const void* q, const void* k, const void* v, int num_sms, cudaStream_t st) {
    const int G = a.H_q / a.H_kv;
    cudaError_t e = run_csr_build(a.csr, a.blocks, a.B, a.N, a.H_kv, a.block_k, a.topk, kRows / G, a.status, st);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(a.counter, 0, (size_t)a.B * a.N * a.H_kv * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.sched, 0, 4, st);
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tk, tv;
    const uint64_t dq[4] = {(uint64_t)a.d, (uint64_t)a.H_q, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t sq[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_q * a.d * 2, (uint64_t)a.N * a.H_q * a.d * 2};
    const uint32_t bq[4] = {64, (uint32_t)std::min(G, 256), 1, 1};
    const uint64_t dkv[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t skv[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2, (uint64_t)a.N * a.H_kv * a.d * 2};
    const uint32_t bkv[4] = {64, 1, (uint32_t)a.block_k, 1};
    if (!make_tmap_4d(&tq, q, dq, sq, bq, 128) || !make_tmap_4d(&tk, k, dkv, skv, bkv, 128) ||
        !make_tmap_4d(&tv, v, dkv, skv, bkv, 128))
        return cudaErrorInvalidValue;
    const int grid = num_sms;
    if (a.d == 128) {
        if (a.block_k == 128) return launch_attn<128, 128>(a, tq, tk, tv, q, grid, st);
        if (a.block_k == 64) return launch_attn<128, 64>(a, tq, tk, tv, q, grid, st);
        return launch_attn<128, 32>(a, tq, tk, tv, q, grid, st);
    }
    if (a.block_k == 128) return launch_attn<64, 128>(a, tq, tk, tv, q, grid, st);
    if (a.block_k == 64) return launch_attn<64, 64>(a, tq, tk, tv, q, grid, st);
    return launch_attn<64, 32>(a, tq, tk, tv, q, grid, st);
}

}  // namespace msa
