// Internal declarations shared by the libmsa translation units (not part of the C ABI).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <algorithm>

namespace msa {

struct DevStatus;

// Opt-in kernel timing (msa_prof.cu): events around a launch on its stream; no-op when disabled.
int prof_begin(const char* name, cudaStream_t st);
void prof_end(int token, cudaStream_t st);
struct ProfScope {
    int tok;
    cudaStream_t st;
    ProfScope(const char* name, cudaStream_t s) : tok(prof_begin(name, s)), st(s) {}
    ~ProfScope() { prof_end(tok, st); }
};

// ---------------------------------------------------------------- tensor maps (msa_tmap.cu)
// bf16 tensor maps; `swizzle_bytes` is 128, 64, 32 or 0. Dimensions innermost first, strides in bytes.
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t stride1, uint32_t box0,
                  uint32_t box1, int swizzle_bytes);
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1,
                  uint64_t stride2, uint32_t box0, uint32_t box1, uint32_t box2, int swizzle_bytes);
bool make_tmap_4d(CUtensorMap* m, const void* base, const uint64_t dims[4], const uint64_t strides[3],
                  const uint32_t box[4], int swizzle_bytes);
// Query rows [B, N, H_q, d] as 5-D boxes of one query's G heads (G % 8 == 0, H_q % 8 == 0, d % 64 == 0)
// laid out in 8-row x 64-column 128B-swizzled atoms.
// Byte tensor [d2][d1][d0] (8-bit elements, e.g. e4m3), box {box0, box1, 1}.
bool make_tmap_3d_u8(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t stride1,
                     uint64_t stride2, uint32_t box0, uint32_t box1, int swizzle_bytes);
bool make_tmap_qrows(CUtensorMap* m, const void* q, int B, int N, int H_q, int d, int G);

// ---------------------------------------------------------------- index Top-k (msa_index.cu)
struct IndexArgs {
    int B, N, H_kv, d_idx, block_k, topk;
    int32_t* blocks;
    DevStatus* status;
    // key range held in k_idx: tokens [tok0, tok0 + ntok) of every sequence, then (ntokb > 0) a
    // second range [tok0b, tok0b + ntokb) after it; k_idx [B, ntok + ntokb, d_idx] stores the first
    // range's tokens, then the second's (0 and N, no second range, for the whole sequence). With
    // cand_ids set, the kernel writes each row's Top-k of the complete past blocks inside the held
    // ranges, unmerged (raw block maxima, -inf / -1 padded), instead of `blocks`.
    int tok0, ntok;
    float* cand_scores;   // [B, N, H_kv, topk]
    int32_t* cand_ids;    // [B, N, H_kv, topk]
    int tok0b, ntokb;
};
cudaError_t run_index_topk(const IndexArgs& a, const void* q_idx, const void* k_idx, int num_sms, cudaStream_t st);

// ---------------------------------------------------------------- sequence-parallel indexer (msa_sp.cu)
cudaError_t run_topk_merge(int B, int N, int H_kv, int block_k, int topk, int P, const float* cand_scores,
                           const int32_t* cand_ids, int32_t* blocks, cudaStream_t st);
// blocks kept where blk0 <= c < blk1 or blk2 <= c < blk3, else -1
cudaError_t run_blocks_in_range(long long rows, int K1, int blk0, int blk1, int blk2, int blk3, const int32_t* blocks,
                                int32_t* out, cudaStream_t st);
cudaError_t run_lse_combine(int P, long long rows, const float2* ml, float* lse, cudaStream_t st);

// ---------------------------------------------------------------- inverse selection lists (msa_csr.cu)
// For every (sequence b, query window w, group r, block c) the list of (query i, slot s) pairs
// whose selection row blocks[b,i,r,:] holds c at position s, cut into work items of at most `qpc`
// queries. A window is `wq` consecutive queries (wq = 0: one window per sequence). Items are
// ordered by (b, w, r, c).
struct Csr {
    int nlists;        // B * nW * H_kv * nb
    int nb;            // blocks per sequence
    int nW;            // windows per sequence
    int wq;            // queries per window (N when wq = 0)
    int max_entries;   // B * N * H_kv * (topk+1)
    int nscan;         // scan blocks: ceil(nlists / 1024)
    int32_t* counts;   // [nlists]
    int32_t* offsets;  // [nlists + 1]
    int32_t* cursor;   // [nlists]
    int32_t* chunk_off;// [nlists + 1]
    int32_t* entries;  // [max_entries]  (i << 5) | s
    int4* items;       // [max_entries]  (list, index of the chunk's first entry, queries, 0)
    int32_t* n_items;  // [1]
    int32_t* bsum;     // [2 * nscan + 2] scan block sums and totals
    uint8_t* nsel;     // [B * N * H_kv] number of valid blocks of each selection row
};
size_t csr_bytes(int B, int N, int H_kv, int block_k, int topk, int wq);
void csr_carve(Csr* c, void* base, int B, int N, int H_kv, int block_k, int topk, int wq);
cudaError_t run_csr_build(const Csr& c, const int32_t* blocks, int B, int N, int H_kv, int block_k, int topk,
                          int qpc, DevStatus* st, cudaStream_t stream);
cudaError_t run_csr_items(const Csr& c, int qpc, cudaStream_t stream);

// ---------------------------------------------------------------- sparse attention (msa_attn.cu)
constexpr int kAttnWindow = 1024;  // queries per window of the attention's inverse lists
struct AttnArgs {
    int B, N, H_q, H_kv, d, block_k, topk;
    float scale;
    Csr csr;             // windowed lists, items of 128/G queries
    __half* o_part;      // [B, N, H_kv, topk+1, d/8, G, 8]   normalised partial outputs
    float* lse_part;     // [B, N, H_kv, topk+1, G]
    int32_t* sched;      // [1]           next item to hand out
    const int32_t* blocks;
    float* out;          // [B, N, H_q, d]  fp32 (the fp32-accumulated result), or null when out_bf16 is set
    float* lse;          // [B, N, H_q] or null
    DevStatus* status;
    __nv_bfloat16* out_bf16;  // [B, N, H_q, d]  the same result rounded to bf16 (nearest even), or null
};
size_t attn_ws_bytes(int B, int N, int H_q, int H_kv, int d, int block_k, int topk);
void attn_carve(AttnArgs* a, void* base);
cudaError_t run_attn(const AttnArgs& a, const void* q, const void* k, const void* v, int num_sms, cudaStream_t st);

// ---------------------------------------------------------------- attention backward (msa_bwd.cu)
struct BwdArgs {
    int B, N, H_q, H_kv, d, block_k, topk;
    float scale;
    Csr csr;            // lists of the forward, items of 128/G queries
    const float* lse;   // [B, N, H_q] natural-log LSE of the forward
    float* delta;       // [B, N, H_q] dO . O (workspace)
    float* dq;          // [B, N, H_q, d]
    float* dk;          // [B, N, H_kv, d]
    float* dv;          // [B, N, H_kv, d]
    DevStatus* status;
};
bool bwd_supported(int d, int G);
cudaError_t run_attn_bwd(const BwdArgs& a, const void* q, const void* k, const void* v, const void* dout,
                         const float* out, int num_sms, cudaStream_t st);

// ---------------------------------------------------------------- KL alignment (msa_kl.cu)
struct KlArgs {
    int B, N, H_q, H_kv, d, d_idx, block_k, topk;
    float scale, scale_idx, grad_scale;
    Csr csr;            // chunks of 128/G queries
    Csr csr_idx;        // same lists, chunks of kIdxQpc queries for the LSE_idx pass
    const float* lse;   // [B, N, H_q]
    float* lse_idx;     // [B, N, H_kv]
    float2* ml_part;    // [B, N, H_kv, topk+1]  (max, sum-exp) of the index logits per slot
    float* dq_part;     // [B, N, H_kv, topk+1, d_idx]
    double* kl_part;    // [B, N, H_kv, topk+1]
    double* kl_rows;    // [B, N, H_kv]
    float* dq_idx;      // [B, N, H_kv, d_idx]
    float* dk_idx;      // [B, N, d_idx]
    float* loss;        // [1]
    const int32_t* blocks;
    DevStatus* status;
    // LSE_idx pass only: k_idx holds tokens [kv_tok0, kv_tok0 + kv_ntok), then those of a second
    // range [kv_tok0b, kv_tok0b + kv_ntokb) if kv_ntokb > 0 ([B, kv_ntok + kv_ntokb, d_idx]; 0 and N
    // for the whole sequence); with ml_out set, each row's (max, exp-sum) is written there instead
    // of lse_idx
    int kv_tok0, kv_ntok, kv_tok0b, kv_ntokb;
    float2* ml_out;     // [B, N, H_kv]
    // dense warm-up: every causal block is selected; the lists come from run_dense_lists, the
    // LSE_idx partial slot of an entry is its block (ml_part [B, N, H_kv, nb]), and dQ_idx / the
    // KL rows are accumulated with atomics instead of per-slot partials (blocks is not read)
    int dense;
};
constexpr int kIdxQpc = 32;
bool kl_supported(int d, int d_idx, int G);
cudaError_t run_lse_idx(const KlArgs& a, const void* q_idx, const void* k_idx, int num_sms, cudaStream_t st);
cudaError_t run_kl(const KlArgs& a, const void* q, const void* k, const void* q_idx, const void* k_idx, int num_sms,
                   cudaStream_t st);

// ---------------------------------------------------------------- decode (msa_decode.cu)
struct DecodeArgs {
    int B, L, H_q, H_kv, d, d_idx, block_k, topk;
    float scale, scale_idx;
    const int32_t* cache_len;
    float* bmax;       // [B, H_kv, nb]
    int32_t* sel;      // [B, H_kv, topk+1]
    float* o_part;     // [B, H_kv, topk+1, G, d]
    float* lse_part;   // [B, H_kv, topk+1, G]
    int32_t* blocks_out;
    float* margin_out;         // [B, H_kv] cutoff margins, or null
    const float* k_idx_scale;  // [B, L] per-token scales when the K_idx cache holds e4m3 codes, else null
    DevStatus* status;
};
size_t decode_ws_bytes(int B, int L, int H_q, int H_kv, int d, int block_k, int topk);
// Row-wise e4m3 quantisation of a bf16 [rows, n] array (n in {16, 32, 64, 128, 256}).
cudaError_t run_quantize_e4m3_rows(const void* x, int64_t rows, int n, uint8_t* codes, float* scale, int num_sms,
                                   cudaStream_t st);
// k_idx_cache is bf16 [B, L, d_idx], or e4m3 codes [B, L, d_idx] when a.k_idx_scale is set.
cudaError_t run_decode(const DecodeArgs& a, const void* q, const void* q_idx, const void* k_cache, const void* v_cache,
                       const void* k_idx_cache, void* out, int num_sms, cudaStream_t st);

// ---------------------------------------------------------------- dense warm-up (msa_dense.cu)
struct DenseLseArgs {
    int B, N, H_q, H_kv, G, d, block_k;
    float scale;
    float* lse;          // [B, N, H_q] natural-log LSE over all causal keys
    DevStatus* status;
};
bool dense_lse_supported(int d, int block_k, int G);
cudaError_t run_dense_lse(const DenseLseArgs& a, const void* q, const void* k, int num_sms, cudaStream_t st);
// Entry and item counts of the dense inverse lists (every query of block c and after, for every
// (b, r, c)), and their build into a Csr carved with room for them (nb, nW = 1 set by csr_carve).
void dense_list_sizes(int B, int N, int H_kv, int block_k, int qpc, long long* entries, long long* items);
cudaError_t run_dense_lists(const Csr& cs, int B, int N, int H_kv, int block_k, int qpc, bool write_entries,
                            cudaStream_t st);

// ---------------------------------------------------------------- test hooks (msa_debug.cu)
// Writes a wait limit (ns) into a cleared status word; the launch whose bounded wait can only run
// out (reads wait_probe_bytes() bytes at `src`).
cudaError_t run_set_wait(DevStatus* st, unsigned long long ns, cudaStream_t s);
size_t wait_probe_bytes();
cudaError_t run_wait_probe(const void* src, DevStatus* st, cudaStream_t s);
// y[i] = 2^x[i] through exp2_fma_x2 (the FMA-pipe exponential), for its accuracy test.
cudaError_t run_exp2_fma(const float* x, float* y, int64_t n, int num_sms, cudaStream_t s);

}  // namespace msa
