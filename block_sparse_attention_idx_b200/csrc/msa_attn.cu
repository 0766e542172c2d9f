// Main branch of MSA: exact softmax attention over the selected blocks, KV-outer
// (MSA blog, KV-outer sparse attention and hot blocks; "2.4 · 训练原生稀疏", eq (2) and the
// online-softmax partition merge eq (18)).
//
// A work item is one selected KV block c of group r plus up to 128/G queries of one query window
// that selected it; their G query heads form the 128 rows of the tile. Per item:
//   S = Q_rows . K_c^T        tcgen05.mma, M=128 rows, N=block_k tokens, K=d        -> TMEM
//   P = exp(S*scale - max)    16 epilogue warps, a quarter of the columns each; causal mask j <= i;
//                             P (bf16) is written back into TMEM over the S columns already read
//   O = P . V_c               tcgen05.mma with A = P from TMEM, B = V_c (MN-major)  -> TMEM
// The normalised partial (o = O / sum P, lse) of every row goes to its (query, head, slot) place
// in the workspace (fp16 o, fp32 lse). A second kernel combines each (query, group) row's <= topk+1
// partials with the log-sum-exp rule and writes the bf16 output and the LSE. Items are handed out
// in (window, group, block) order by an atomic counter, up to 16 at a time, so consecutive items of
// a CTA often share their K/V block; a wide window fills items with more queries.
//
// Warp roles (640 threads): warps 0-15 run the softmax and the epilogue of every item (warp w: TMEM
// lane quarter w % 4, column quarter w / 4), warp 16 hands out items and stages their metadata,
// warps 17 and 18 each gather half of an item's Q rows (TMA, each query's G head rows) and load K
// and V respectively, warp 19 issues the MMAs and owns TMEM. Q, K, V and the two accumulators (S/P
// and O) are double-buffered; the MMA issuer polls and issues whichever of the next S or the next
// PV is ready.
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {

namespace {

constexpr int kRows = 128;
constexpr int kMeta = 4;        // depth of the item metadata ring
constexpr int kEpiWarps = 16;   // warps 0..15: softmax / epilogue, two teams of 8
constexpr int kTeamWarps = 8;
constexpr int kSchedWarp = 16;  // hands out items, stages their metadata
constexpr int kQKWarp = 17;     // first half of each item's Q rows, K
constexpr int kQVWarp = 18;     // second half of each item's Q rows, V
constexpr int kMmaWarp = 19;    // MMA issue, TMEM owner
constexpr int kThreads = 20 * 32;
constexpr int kStage = 512;     // query entries staged per scheduler fetch

struct ItemMeta {
    int t;  // item index; -1: no more items
    int b, r, c, count, kv_new;
    int qi[kRows];
    int8_t qs[kRows];  // query index and selection slot of each item query
};

template <int D, int BK>
struct AttnSmem {
    static constexpr int kQBytes = kRows * D * 2;   // D/64 sub-tiles of [128 rows x 128 B]
    static constexpr int kKVBytes = BK * D * 2;     // D/64 sub-tiles of [BK rows x 128 B]
    alignas(1024) uint8_t q[2][kQBytes];
    alignas(1024) uint8_t k[2][kKVBytes];
    alignas(1024) uint8_t v[2][kKVBytes];
    ItemMeta meta[kMeta];
    int stage[kStage];  // query entries of the items of the current scheduler fetch
    // per-row partial max / sums of the two column halves: [team][team item parity][half][row]
    float red_max[2][2][2][kRows], red_l[2][2][2][kRows];
    uint64_t meta_full[kMeta], meta_empty[kMeta];
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[2], k_release[2], v_full[2], v_release[2];  // release[b]: one completion per use of buffer b
    uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
    // a team's row maxima of its item are in (max_bar[team]); its row sums are in
    // (sum_bar[team][team item parity]: read one item later, after the warp's own next arrival)
    uint64_t max_bar[2], sum_bar[2][2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ bool wait_lane0(uint64_t* bar, uint32_t parity, DevStatus* st, unsigned where) {
    int ok = 1;
    if (lane_id() == 0) ok = mbar_wait(bar, parity, st, where);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
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
    constexpr int kSC = BK / 2;  // S columns per epilogue warp

    const int G = a.H_q / a.H_kv;
    const int K1 = a.topk + 1;
    const int T = *a.csr.n_items;
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int x = 0; x < kMeta; ++x) {
            mbar_init(&s.meta_full[x], 1);
            mbar_init(&s.meta_empty[x], 3 + kTeamWarps);  // both Q loaders, the MMA issuer, the item's team
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(&s.q_full[x], 2);  // one arrival per Q loader
            mbar_init(&s.q_empty[x], 1);
            mbar_init(&s.k_full[x], 1);
            mbar_init(&s.v_full[x], 1);
            mbar_init(&s.s_full[x], 1);
            mbar_init(&s.p_full[x], kTeamWarps);
            mbar_init(&s.o_full[x], 1);
            mbar_init(&s.o_free[x], kTeamWarps);
            mbar_init(&s.max_bar[x], kTeamWarps);
            mbar_init(&s.sum_bar[x][0], kTeamWarps);
            mbar_init(&s.sum_bar[x][1], kTeamWarps);
            mbar_init(&s.k_release[x], 1);
            mbar_init(&s.v_release[x], 1);
        }
        mbar_init(&s.drain, 1);
        s.abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&s.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s.tmem_base;

    if (warp == kSchedWarp) {
        // ------------------------------------------------------------ item scheduler
        // Takes CH consecutive items per atomic fetch (their records, one per lane, and their query
        // entries, one contiguous range of the list arrays), then stages the items' metadata one by
        // one. No global load is in flight when a metadata slot is released to its consumers.
        const int QPC = max(1, kRows / G);
        const int CH = min(16, kStage / QPC);
        int n = 0, prevL = -1;
        bool ok = true;
        while (ok) {
            int base = 0;
            if (lane == 0) base = s.abort ? T : atomicAdd(a.sched, CH);
            base = __shfl_sync(0xffffffffu, base, 0);
            if (base >= T) {
                // two end markers: one for each epilogue team
                for (int x = 0; x < 2 && ok; ++x, ++n) {
                    const int slot = n % kMeta;
                    if (!wait_lane0(&s.meta_empty[slot], ((n / kMeta) & 1) ^ 1, a.status, 0x501)) { ok = false; break; }
                    if (lane == 0) { s.meta[slot].t = -1; mbar_arrive(&s.meta_full[slot]); }
                }
                break;
            }
            const int cnt = min(CH, T - base);
            const int4 rec = lane < cnt ? a.csr.items[base + lane] : make_int4(-1, 0, 0, 0);
            // the entries of consecutive items are contiguous in the list arrays
            const int y0 = __shfl_sync(0xffffffffu, rec.y, 0);
            const int y1 = __shfl_sync(0xffffffffu, rec.y + rec.z, cnt - 1);
            for (int x = lane; x < y1 - y0; x += 32) s.stage[x] = a.csr.entries[y0 + x];
            __syncwarp();
            for (int j = 0; j < cnt; ++j, ++n) {
                const int L = __shfl_sync(0xffffffffu, rec.x, j);
                const int off = __shfl_sync(0xffffffffu, rec.y, j) - y0;
                const int count = __shfl_sync(0xffffffffu, rec.z, j);
                const int slot = n % kMeta;
                if (!wait_lane0(&s.meta_empty[slot], ((n / kMeta) & 1) ^ 1, a.status, 0x502)) { ok = false; break; }
                ItemMeta& mt = s.meta[slot];
                for (int m = lane; m < count; m += 32) {
                    const int e = s.stage[off + m];
                    mt.qi[m] = e >> 5;
                    mt.qs[m] = (int8_t)(e & 31);
                }
                if (lane == 0) {
                    mt.t = base + j;
                    mt.c = L % a.csr.nb;
                    mt.r = (L / a.csr.nb) % a.H_kv;
                    mt.b = L / (a.csr.nb * a.H_kv * a.csr.nW);
                    mt.count = count;
                    mt.kv_new = (L != prevL);
                }
                prevL = L;
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.meta_full[slot]);
            }
            __syncwarp();  // the staged entries are read before the next fetch overwrites them
        }
        if (!ok) s.abort = 1;
    } else if (warp == kQKWarp || warp == kQVWarp) {
        // ------------------------------------------------------------ Q (half each), K / V
        // Both warps gather Q rows (the TMA issue rate of one warp is the limit otherwise): the
        // first loads the first half of the item's queries and the K blocks, the second the other
        // half and the V blocks. All their barriers carry TMA data only: relaxed arrives.
        const bool is_k = warp == kQKWarp;
        // a query's rows are read again by the items of its other selected blocks: keep them in L2
        const uint64_t q_policy = l2_policy_evict_last();
        int group = -1, n_issued = 0;
        bool ok = true;
        for (int n = 0;; ++n) {
            const int slot = n % kMeta;
            if (!wait_lane0(&s.meta_full[slot], (n / kMeta) & 1, a.status, 0x511)) { ok = false; break; }
            const ItemMeta& mt = s.meta[slot];
            const int t = mt.t;
            if (t < 0) break;
            const int b = mt.b, r = mt.r, c = mt.c, count = mt.count, kv_new = mt.kv_new;
            const int half = (count + 1) >> 1;
            const int m0 = is_k ? 0 : half, m1 = is_k ? half : count;
            const int buf = n & 1;
            if (!wait_lane0(&s.q_empty[buf], ((n >> 1) & 1) ^ 1, a.status, 0x512)) { ok = false; break; }
            if (G % 8 == 0) {
                if (lane == 0) mbar_arrive_expect_tx_relaxed(&s.q_full[buf], (uint32_t)((m1 - m0) * G * D * 2));
                __syncwarp();
                for (int m = m0 + lane; m < m1; m += 32)
                    tma_load_5d_hint(s.q[buf] + m * G * D * 2, &tm_q, &s.q_full[buf], 0, 0, 0, r * G / 8,
                                     b * a.N + mt.qi[m], q_policy);
            } else if (is_k) {
                // few heads per group: one warp copies every row, then makes them visible to the MMA
                const uint32_t qsm = smem_u32(s.q[buf]);
                constexpr int kChunksPerRow = D * 2 / 16;
                for (int x = lane; x < count * G * kChunksPerRow; x += 32) {
                    const int row = x / kChunksPerRow, ch = x % kChunksPerRow;
                    const int m = row / G, h = row % G;
                    const __nv_bfloat16* src =
                        q + ((((size_t)b * a.N + mt.qi[m]) * a.H_q + (size_t)r * G + h) * D + ch * 8);
                    cp_async_16(qsm + qtile_off<D>(row, ch * 16), src);
                }
                cp_async_wait_all();
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.q_full[buf]);
            } else {
                if (lane == 0) mbar_arrive_relaxed(&s.q_full[buf]);
            }
            ++n_issued;
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.meta_empty[slot]);
            // K (or V) of block group g goes to buffer g % 2 once the MMAs of group g-2 that read it
            // (the buffer's previous use, release number (g-2)/2) are done
            if (kv_new) {
                ++group;
                uint64_t* rel = is_k ? s.k_release : s.v_release;
                if (group >= 2 &&
                    !wait_lane0(&rel[group & 1], ((group - 2) >> 1) & 1, a.status, 0x513)) { ok = false; break; }
                if (lane == 0) {
                    const int kb = group & 1;
                    uint64_t* full = is_k ? &s.k_full[kb] : &s.v_full[kb];
                    uint8_t* dst = is_k ? s.k[kb] : s.v[kb];
                    const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
                    mbar_arrive_expect_tx_relaxed(full, (uint32_t)Sm::kKVBytes);
#pragma unroll
                    for (int sub = 0; sub < D / 64; ++sub)
                        tma_load_4d(dst + sub * BK * 128, tm, full, sub * 64, r, c * BK, b);
                }
            }
        }
        if (!ok) s.abort = 1;
        if (lane == 0) {  // no copy of ours may still be landing when the CTA leaves
            uint64_t* full = is_k ? s.k_full : s.v_full;
            for (int g = max(0, group - 1); g <= group; ++g) mbar_wait(&full[g & 1], (g >> 1) & 1, a.status, 0x514);
            for (int x = 0; x < 2 && x < n_issued; ++x) {
                const int nl = n_issued - 1 - x;
                mbar_wait(&s.q_full[nl & 1], (nl >> 1) & 1, a.status, 0x515);
            }
        }
    } else if (warp == kMmaWarp) {
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
            const uint64_t lim = wait_limit(a.status);
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
                            const uint64_t da = umma_sdesc(qb + sub * 1024 + off, 16, (D / 64) * 1024, 2);
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
                            // P of S columns [16ks, 16ks+16) sits packed in the columns of the
                            // epilogue warp that owns them (warp half e = 16ks / (BK/2))
                            umma_bf16_tmem_a(tO, tP + (ks * 16 / kSC) * kSC + (ks * 16 % kSC) / 2, db, kIdescO, ks > 0);
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
                if (!progressed && globaltimer() - t_idle > lim) {
                    raise_flag(a.status, MSA_DEV_TIMEOUT, 0x601);
                    ok = false;
                    break;
                }
            }
            if (!ok) s.abort = 1;
            umma_commit(&s.drain);
            mbar_wait(&s.drain, 0, a.status, 0x608);
        }
    } else if (warp < kEpiWarps) {
        // ------------------------------------------------------------ softmax / epilogue
        // Two teams of 8 warps take alternate items (team t: items n with n % 2 == t, always in TMEM
        // buffer t), so one team's exponentials overlap the other team's O read-out and waits.
        // Within a team, warp w reads TMEM lane quarter w % 4 (tile rows 32(w%4) .. +31) and column
        // half e of S (BK/2 tokens) and of O (D/2 values). Each team item starts by reading out the
        // O of the team's previous item, which frees the team's single O accumulator for the PV
        // product of the item that follows. The row max and row sums of the two halves
        // meet in shared memory, published by the team's max_bar / sum_bar mbarriers. S is read
        // twice (for the max, then for the exponentials), and each warp writes its P packed over its
        // own S columns. Every wait is bounded; a warp whose wait fails leaves, and the others run
        // into their own bounded waits.
        constexpr int SC = BK / 2, OC = D / 2;
        constexpr int CH = SC < 32 ? SC : 32;  // columns per TMEM load
        const int t = warp >> 3, qtr = warp & 3, e = (warp >> 2) & 1;
        const int row = qtr * 32 + lane;
        const int m = row / G, h = row % G;
        const uint32_t lane_addr = tmem + ((uint32_t)(qtr * 32) << 16);
        const uint32_t tS = lane_addr + t * 256 + e * SC, tO = lane_addr + t * 256 + 128 + e * OC;
        const float sl2 = a.scale * 1.4426950408889634f;
        // the team's item whose O is read out next: the row's partial index ((b, i, r, slot), head)
        // or -1 and its max (partial indices fit 31 bits, checked by the host)
        bool have_prev = false;
        int pv_prow = -1;
        float pv_mx = 0.f;
        // O of the team's item number kp: normalise by the row's weight sum l, store the fp16
        // partial and its LSE, free the accumulator
        // the partials are written once here and read once by the merge: they must not push the
        // query rows out of L2
        const uint64_t part_policy = l2_policy_evict_first();
        auto store_prev = [&](int kp) -> bool {
            const int pb = kp & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&s.o_full[t], pb, a.status, 0x704))) return false;
            if (!__all_sync(0xffffffffu, mbar_wait(&s.sum_bar[t][pb], (kp >> 1) & 1, a.status, 0x705))) return false;
            tc_fence_after();
            float inv = 0.f;
            if (pv_prow >= 0) inv = 1.f / (s.red_l[t][pb][0][row] + s.red_l[t][pb][1][row]);
            const uint64_t invx2 = f2_packf(inv, inv);
            // chunk x of 8 values goes to [(b, i, r, slot)][x][head]: the G heads of a query are
            // adjacent, so a warp's store covers whole 128-byte lines
            uint4* dst = reinterpret_cast<uint4*>(a.o_part) + (pv_prow >= 0 ? (size_t)(pv_prow - h) * (D / 8) + h : 0);
#pragma unroll
            for (int c0 = 0; c0 < OC; c0 += 32) {
                uint32_t ov[32];
                tmem_ld32(tO + c0, ov);
                tmem_ld_wait();
                if (pv_prow >= 0) {
                    uint32_t hv[16];
#pragma unroll
                    for (int x = 0; x < 32; x += 2) {
                        float o0, o1;
                        f2_unpack(f2_mul(f2_pack(ov[x], ov[x + 1]), invx2), o0, o1);
                        const __half2 hh2 = __floats2half2_rn(o0, o1);
                        hv[x / 2] = *reinterpret_cast<const uint32_t*>(&hh2);
                    }
#pragma unroll
                    for (int x = 0; x < 4; ++x)
                        st_global_v4_hint(&dst[(size_t)((e * OC + c0) / 8 + x) * G],
                                          make_uint4(hv[4 * x], hv[4 * x + 1], hv[4 * x + 2], hv[4 * x + 3]),
                                          part_policy);
                }
            }
            if (e == 0 && pv_prow >= 0)
                a.lse_part[pv_prow] = pv_mx * a.scale + logf(s.red_l[t][pb][0][row] + s.red_l[t][pb][1][row]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.o_free[t]);
            return true;
        };
        bool fail = false;
        int k = 0;
        for (;; ++k) {
            const int n = 2 * k + t, kb = k & 1;
            // the O buffer of the team is single: free it (item k-1) before this item's softmax, so
            // that the PV product of item k can start as soon as its P is in
            if (have_prev) {
                if (!store_prev(k - 1)) {
                    fail = true;
                    break;
                }
                have_prev = false;
            }
            const int slot = n % kMeta;
            if (!__all_sync(0xffffffffu, mbar_wait(&s.meta_full[slot], (n / kMeta) & 1, a.status, 0x701))) {
                fail = true;
                break;
            }
            const ItemMeta& mt = s.meta[slot];
            if (mt.t < 0) break;  // end of the item stream
            const int b = mt.b, r = mt.r, c = mt.c;
            const bool valid = m < mt.count;
            const int i = valid ? mt.qi[m] : 0;
            const int qslot = valid ? (int)mt.qs[m] : 0;
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.meta_empty[slot]);
            const int lim = valid ? i - c * BK - e * SC : -1;  // this warp's columns x <= lim are causal
            const bool full = __all_sync(0xffffffffu, lim >= SC - 1);
            if (!__all_sync(0xffffffffu, mbar_wait(&s.s_full[t], kb, a.status, 0x702))) {
                fail = true;
                break;
            }
            tc_fence_after();
            // pass 1: max over this warp's causal columns
            {
                float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c0 = 0; c0 < SC; c0 += CH) {
                    uint32_t sv[CH];
                    tmem_ld<CH>(tS + c0, sv);
                    tmem_ld_wait();
                    if (full) {
#pragma unroll
                        for (int x = 0; x < CH; x += 2)
                            m4[(x >> 1) & 3] = max3f(m4[(x >> 1) & 3], __uint_as_float(sv[x]), __uint_as_float(sv[x + 1]));
                    } else {
#pragma unroll
                        for (int x = 0; x < CH; ++x)
                            m4[x & 3] = c0 + x <= lim ? fmaxf(m4[x & 3], __uint_as_float(sv[x])) : m4[x & 3];
                    }
                }
                s.red_max[t][kb][e][row] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.max_bar[t]);
            if (!__all_sync(0xffffffffu, mbar_wait(&s.max_bar[t], kb, a.status, 0x703))) {
                fail = true;
                break;
            }
            // pass 2: P = exp(S - max) rounded to bf16, packed two per TMEM column over the warp's
            // own S columns already read. l, the fp32 sum of the weights before rounding, gives the LSE
            // and normalises O (the bf16 rounding of the weights changes their sum by ~1e-4 relative,
            // well inside the attention tolerance; a second, rounded sum cost four more instructions
            // per pair of columns and 2-4 % of the kernel's time).
            const float mx = fmaxf(s.red_max[t][kb][0][row], s.red_max[t][kb][1][row]);
            const float moff = valid ? mx * sl2 : 0.f;
            const uint64_t sl2x2 = f2_packf(sl2, sl2), moffx2 = f2_packf(-moff, -moff);
            uint64_t lx2 = f2_packf(0.f, 0.f);
#pragma unroll
            for (int c0 = 0; c0 < SC; c0 += CH) {
                uint32_t sv[CH];
                tmem_ld<CH>(tS + c0, sv);
                tmem_ld_wait();
                uint32_t pk[CH / 2];
#pragma unroll
                for (int y = 0; y < CH; y += 2) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(sv[y], sv[y + 1]), sl2x2, moffx2), x0, x1);
                    float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                    if (!full) {
                        p0 = c0 + y <= lim ? p0 : 0.f;
                        p1 = c0 + y + 1 <= lim ? p1 : 0.f;
                    }
                    const __nv_bfloat162 pb2 = __floats2bfloat162_rn(p0, p1);
                    const uint32_t u = *reinterpret_cast<const uint32_t*>(&pb2);
                    lx2 = f2_add(lx2, f2_packf(p0, p1));
                    pk[y / 2] = u;
                }
                tmem_st<CH / 2>(tS + c0 / 2, pk);
            }
            tmem_st_wait();
            tc_fence_before();
            {
                float l0, l1;
                f2_unpack(lx2, l0, l1);
                s.red_l[t][kb][e][row] = l0 + l1;
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&s.sum_bar[t][kb]);
                mbar_arrive(&s.p_full[t]);
            }
            have_prev = true;
            pv_prow = valid ? (((b * a.N + i) * a.H_kv + r) * K1 + qslot) * G + h : -1;
            pv_mx = mx;
        }
        if (fail) {
            s.abort = 1;
        } else if (have_prev) {
            store_prev(k - 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// Combines each (query, group) row's partials: out = sum_s exp(lse_s - LSE) o_s with
// LSE = log sum_s exp(lse_s) (the partition merge), over the row's valid slots. One warp per row;
// lanes take units of 8 output values of one head (head fastest, matching the partial layout
// [(b, i, r, slot)][d/8][head][8]) and keep every slot's load in flight at once.
template <int D, int BK>
__global__ void __launch_bounds__(256) k_attn_merge(AttnArgs a) {
    const int G = a.H_q / a.H_kv;
    const int K1 = a.topk + 1;
    const int lane = lane_id();
    const int rows = a.B * a.N * a.H_kv;
    const int units = G * (D / 8);
    constexpr int kK1Max = 17;
    bool overflow = false;
    for (int row = blockIdx.x * 8 + warp_id(); row < rows; row += gridDim.x * 8) {
        const int r = row % a.H_kv, i = (row / a.H_kv) % a.N, b = row / a.H_kv / a.N;
        // slot x is kept when its block is causal and above every kept block before it; the
        // largest kept block so far equals the largest in-range block so far (prefix max)
        const int32_t* sel = a.blocks + (size_t)row * K1;
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
        for (int u = lane; u < units; u += 32) {
            const int hh = u % G, ch = u / G, d0 = ch * 8;
            const int hq = r * G + hh;
            const size_t rb = (size_t)row * K1;  // first slot of the row
            float lv[kK1Max];
            uint4 ov[kK1Max];
#pragma unroll
            for (int x = 0; x < kK1Max; ++x) {
                if (vmask & (1u << x)) {
                    lv[x] = __ldcs(a.lse_part + (rb + x) * G + hh);
                    ov[x] = __ldcs(reinterpret_cast<const uint4*>(a.o_part) + ((rb + x) * (D / 8) + ch) * G + hh);
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
            for (int y = 0; y < 8; ++y) acc[y] = 0.f;
#pragma unroll
            for (int x = 0; x < kK1Max; ++x) {
                const float w = lv[x] == -INFINITY ? 0.f : __expf(lv[x] - lmax);
                z += w;
                const __half2* h2 = reinterpret_cast<const __half2*>(&ov[x]);
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const float2 f = __half22float2(h2[y]);
                    acc[2 * y] = fmaf(w, f.x, acc[2 * y]);
                    acc[2 * y + 1] = fmaf(w, f.y, acc[2 * y + 1]);
                }
            }
            const float zi = 1.f / z;
#pragma unroll
            for (int y = 0; y < 8; ++y) {
                overflow |= !isfinite(acc[y]);
                acc[y] *= zi;
            }
            const size_t oo = (((size_t)b * a.N + i) * a.H_q + hq) * D + d0;
            if (a.out_bf16) {
                uint4 pk;
                uint32_t* pw = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
                for (int y = 0; y < 4; ++y) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * y], acc[2 * y + 1]);
                    pw[y] = *reinterpret_cast<const uint32_t*>(&h);
                }
                *reinterpret_cast<uint4*>(a.out_bf16 + oo) = pk;
            } else {
                float4* o4 = reinterpret_cast<float4*>(a.out + oo);
                o4[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                o4[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
            }
            if (a.lse && d0 == 0) a.lse[((size_t)b * a.N + i) * a.H_q + hq] = lmax + logf(z);
        }
    }
    // fp16 partials overflow when entries of V exceed the fp16 range: report it
    if (overflow) raise_flag(a.status, MSA_DEV_BAD_BLOCK, 0x802);
}

template <int D, int BK>
cudaError_t launch_attn(const AttnArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const void* q, int num_sms, cudaStream_t st) {
    const size_t smem = std::max<size_t>(sizeof(AttnSmem<D, BK>) + 1024, 116 * 1024);  // one CTA per SM
    cudaError_t e =
        cudaFuncSetAttribute(k_attn_kv_outer<D, BK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    {
        ProfScope ps("attn_kv_outer", st);
        k_attn_kv_outer<D, BK><<<num_sms, kThreads, smem, st>>>(tq, tk, tv, static_cast<const __nv_bfloat16*>(q), a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    ProfScope pm("attn_merge", st);
    k_attn_merge<D, BK><<<num_sms * 8, 256, 0, st>>>(a);
    return cudaGetLastError();
}

size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t attn_ws_bytes(int B, int N, int H_q, int H_kv, int d, int block_k, int topk) {
    const size_t pr = (size_t)B * N * H_q * (topk + 1);
    return csr_bytes(B, N, H_kv, block_k, topk, kAttnWindow) + al256(pr * d * sizeof(__half)) +
           al256(pr * sizeof(float)) + 256;
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
    a->sched = reinterpret_cast<int32_t*>(p);
}

cudaError_t run_attn(const AttnArgs& a, const void* q, const void* k, const void* v, int num_sms, cudaStream_t st) {
    const int G = a.H_q / a.H_kv;
    cudaError_t e = run_csr_build(a.csr, a.blocks, a.B, a.N, a.H_kv, a.block_k, a.topk, kRows / G, a.status, st);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(a.sched, 0, 4, st);
    if (e != cudaSuccess) return e;
    CUtensorMap tq, tk, tv;
    const uint64_t dkv[4] = {(uint64_t)a.d, (uint64_t)a.H_kv, (uint64_t)a.N, (uint64_t)a.B};
    const uint64_t skv[3] = {(uint64_t)a.d * 2, (uint64_t)a.H_kv * a.d * 2, (uint64_t)a.N * a.H_kv * a.d * 2};
    const uint32_t bkv[4] = {64, 1, (uint32_t)a.block_k, 1};
    if (!make_tmap_4d(&tk, k, dkv, skv, bkv, 128) || !make_tmap_4d(&tv, v, dkv, skv, bkv, 128))
        return cudaErrorInvalidValue;
    if (G % 8 == 0) {
        if (!make_tmap_qrows(&tq, q, a.B, a.N, a.H_q, a.d, G)) return cudaErrorInvalidValue;
    } else {
        tq = tk;  // not read: the query rows are copied without TMA
    }
    if (a.d == 128) {
        if (a.block_k == 128) return launch_attn<128, 128>(a, tq, tk, tv, q, num_sms, st);
        if (a.block_k == 64) return launch_attn<128, 64>(a, tq, tk, tv, q, num_sms, st);
        return launch_attn<128, 32>(a, tq, tk, tv, q, num_sms, st);
    }
    if (a.block_k == 128) return launch_attn<64, 128>(a, tq, tk, tv, q, num_sms, st);
    if (a.block_k == 64) return launch_attn<64, 64>(a, tq, tk, tv, q, num_sms, st);
    return launch_attn<64, 32>(a, tq, tk, tv, q, num_sms, st);
}

}  // namespace msa
