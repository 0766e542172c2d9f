/*
 * msa.h: C ABI of libmsa, the B200 (sm_100a) implementation of the MiniMax Sparse Attention (MSA)
 * layer hot path.
 *
 * The pages split a sparse layer into a candidate constructor and a main attention,
 *   S_t = R_theta(q_t, K_{:t}),   o_t = A_phi(q_t, K_{S_t}, V_{S_t})
 * ("2.4 · 训练原生稀疏", eq (3)). msa_index_topk is R_theta for MSA, msa_sparse_attn_fwd is A_phi,
 * msa_kl_fwd_grad is the KL alignment of the index branch to the main branch, and
 * msa_sparse_attn_bwd is A_phi's backward with the selection held fixed,
 * msa_sparse_attn_decode runs R_theta then A_phi for one new token per sequence, and
 * msa_sparse_attn_decode_fp8idx does the same from an e4m3 copy of the index keys.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor arguments are DEVICE pointers to dense, contiguous, row-major arrays, 16-byte
 *   aligned. "bf16" means IEEE bfloat16 stored as 2 bytes.
 * - The caller owns every buffer, the workspace and the stream. The library never allocates,
 *   frees or synchronises (except msa_get_device_status, which synchronises the given stream).
 *   Every call only enqueues work on `stream` and returns.
 * - Outputs are fully overwritten.
 * - The workspace `ws` must be at least msa_workspace_size(op, dims) bytes and 256-byte aligned.
 *   Its contents between calls are undefined, except the device status word, which holds the
 *   device-side error flags of the last call that used this workspace. Calls that share a
 *   workspace must be ordered on one stream.
 * - Host-side argument errors return a status before anything is enqueued. Device-side problems
 *   (a wait that ran past its time limit, an out-of-range block id in `blocks`) never trap: the
 *   kernel skips the offending work, sets a flag in the status word and returns; read it with
 *   msa_get_device_status.
 * - Deterministic: the same inputs give bit-identical `blocks`, attention outputs, LSEs and KL
 *   loss. dK_idx and the attention gradients are accumulated with float32 atomics and may differ
 *   in the last bits.
 *
 * Supported sizes (MSA_ERR_UNSUPPORTED otherwise): d in {64, 128}, d_idx in {32, 64},
 * block_k in {32, 64, 128}, 1 <= topk <= 16, H_q % H_kv == 0 with G = H_q/H_kv in {1,2,4,8,16,32},
 * H_kv in {1,2,4,8}, N >= 1, B >= 1, N < 2^24 and B*N*H_kv*(topk+1) < 2^30; msa_sparse_attn_fwd
 * also needs B*N*H_q*(topk+1) < 2^31. The attention keeps its per-slot partial outputs in fp16: entries of V must stay below 65504 in magnitude (larger
 * values are reported as MSA_ERR_DEVICE_CHECK). msa_kl_fwd_grad supports (d, d_idx) in
 * {(128, 64), (64, 32)} with G in {2, 16}.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle (cudaStream_t / CUstream); NULL is the legacy default stream. */
typedef struct CUstream_st *msa_stream_t;

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1,  /* null or misaligned pointer, inconsistent sizes */
    MSA_ERR_UNSUPPORTED = 2,  /* sizes outside the supported set above */
    MSA_ERR_WORKSPACE = 3,    /* ws too small or not 256-byte aligned */
    MSA_ERR_CUDA = 4,         /* a CUDA launch or driver call failed */
    MSA_ERR_TIMEOUT = 5,      /* device status: a bounded wait ran out */
    MSA_ERR_DEVICE_CHECK = 6  /* device status: invalid data found (e.g. a block id out of range) */
} msa_status;

/*
 * Problem sizes. B sequences of N tokens; H_q query heads and H_kv KV heads (G = H_q/H_kv query
 * heads per GQA group); head dim d; index dim d_idx; KV block size block_k (the pages' B_k);
 * topk = k, the number of past blocks each (query, group) selects.
 * scale = 0 means 1/sqrt(d); scale_idx = 0 means 1/sqrt(d_idx).
 */
typedef struct {
    int B, N, H_q, H_kv, d, d_idx, block_k, topk;
    float scale, scale_idx;
} msa_dims;

enum {
    MSA_OP_INDEX_TOPK = 0,
    MSA_OP_INDEX_TOPK_LSE = 1,
    MSA_OP_ATTN_FWD = 2,
    MSA_OP_DECODE = 3,
    MSA_OP_KL = 4,
    MSA_OP_ATTN_BWD = 5,
    MSA_OP_LSE_IDX_LOCAL = 6,
    MSA_OP_KL_DENSE = 7
};

/*
 * Workspace bytes `op` needs for `dims` (for MSA_OP_DECODE, dims->N is the cache capacity).
 * MSA_OP_DECODE also serves msa_sparse_attn_decode_fp8idx, MSA_OP_INDEX_TOPK also serves
 * msa_index_topk_local, MSA_OP_ATTN_BWD is msa_sparse_attn_bwd's (MSA_ERR_UNSUPPORTED for its
 * unsupported G), MSA_OP_LSE_IDX_LOCAL is msa_lse_idx_local's, MSA_OP_KL_DENSE is
 * msa_kl_dense_fwd_grad's (MSA_ERR_UNSUPPORTED for its unsupported sizes).
 */
MSA_API msa_status msa_workspace_size(int op, const msa_dims *dims, size_t *bytes);

/*
 * Index branch: block selection ("MSA Indexer 与 DSA Lightning Indexer 的差别", sections 2.1-2.2;
 * MSA blog, softmax-free Top-K).
 *   S^{idx,(r)}_{i,j} = Q^{idx,(r)}_i . K^{idx}_j * scale_idx        (one shared index-key head)
 *   M_{i,b}           = max_{j in block b, j <= i} S_{i,j}          (causal block max-pool)
 *   blocks[b,i,r,:]   = Top-k of {M_{i,c} : c < b_i} by (M desc, block id asc), plus the query's
 *                       local block b_i = i / block_k, sorted ascending, padded with -1.
 * A row therefore holds min(k, b_i) + 1 block ids. Scores are never materialised.
 *   q_idx   bf16  [B, N, H_kv, d_idx]
 *   k_idx   bf16  [B, N, d_idx]
 *   blocks  int32 [B, N, H_kv, topk+1]                              (output)
 *   lse_idx fp32  [B, N, H_kv] or NULL: log-sum-exp of S^idx over the selected causal token set J
 *           ("KL 对齐" page, section 6: the index pass supplies LSE_idx)  (output, op
 *           MSA_OP_INDEX_TOPK_LSE sizes the workspace when non-NULL)
 */
MSA_API msa_status msa_index_topk(const msa_dims *dims, const void *q_idx, const void *k_idx, int32_t *blocks,
                          float *lse_idx, void *ws, size_t ws_bytes, msa_stream_t stream);

/*
 * Main branch: exact causal softmax attention over the union of the selected blocks, each query
 * head using its group's list ("2.4 · 训练原生稀疏", eq (2); "MSA Indexer" page, section 2.3).
 *   o[b,i,h] = sum_{j in J} softmax_J(q[b,i,h] . k[b,j,r] * scale)_j v[b,j,r],  r = h / G,
 *   J = { j <= i : j / block_k in blocks[b,i,r,:] }.
 *   q      bf16  [B, N, H_q, d]
 *   k, v   bf16  [B, N, H_kv, d]
 *   blocks int32 [B, N, H_kv, topk+1]: ids in [0, i/block_k], -1 entries ignored; normally the
 *          output of msa_index_topk. The local block must be present for J to be non-empty.
 *   out    fp32  [B, N, H_q, d]: the fp32-accumulated result, not rounded to bf16 (output)
 *   lse    fp32  [B, N, H_q] or NULL: natural-log sum-exp of the scaled logits over J (output)
 */
MSA_API msa_status msa_sparse_attn_fwd(const msa_dims *dims, const void *q, const void *k, const void *v,
                               const int32_t *blocks, float *out, float *lse, void *ws, size_t ws_bytes,
                               msa_stream_t stream);
/*
 * The same computation with a bf16 output: out bf16 [B, N, H_q, d] holds the fp32 result above
 * rounded to the nearest bf16 (ties to even), element for element the value msa_sparse_attn_fwd
 * writes, rounded. Half the output bytes (for callers that copy O back to the host or keep it in
 * bf16); the rounding adds at most half a bf16 unit in the last place (2^-8 |o| or less) to the
 * fp32 result's error.
 * Same workspace (MSA_OP_ATTN_FWD), status and errors as msa_sparse_attn_fwd.
 */
MSA_API msa_status msa_sparse_attn_fwd_bf16(const msa_dims *dims, const void *q, const void *k, const void *v,
                                            const int32_t *blocks, void *out, float *lse, void *ws, size_t ws_bytes,
                                            msa_stream_t stream);

/*
 * Sequence-parallel index branch ("4.1.1 · 监督与联合训练", section 3, eq (16)): P ranks each hold
 * part of every sequence's keys; only (score, block id) candidates and per-row (max, exp-sum) pairs
 * are exchanged, and the result equals the single-device msa_index_topk.
 * A rank holds one or two ranges of tokens (msa_key_ranges, host memory, read during the call):
 * range x is tokens [tok0[x], tok0[x] + ntok[x]), tok0[x] a multiple of block_k, ntok[x] > 0 a
 * multiple of block_k unless the range ends at N, and the second range starts at or after the end
 * of the first. k_idx_local holds the first range's tokens, then the second's: bf16
 * [B, ntok[0] + ntok[1], d_idx]. Across the ranks the ranges tile [0, N) without overlap; any
 * assignment gives the same result. Under a causal mask the block at position c is in the past of
 * (N - c) queries, so contiguous ranges load the first rank most; two ranges per rank, chunk p and
 * chunk 2P-1-p of 2P equal chunks of blocks (zig-zag), give every rank about the same work.
 * A null or malformed msa_key_ranges gives MSA_ERR_INVALID_ARG.
 *
 * msa_index_topk_local: for every (b, i, r), the Top-k of the complete past blocks c < b_i that this
 *   rank holds, by (M desc, block id asc), best first. cand_scores fp32 [B, N, H_kv, topk] are the
 *   raw block maxima of Q^idx . K^idx (without scale_idx, so that every rank compares the same
 *   numbers as the single-device kernel), -inf padded; cand_ids int32, -1 padded. Workspace: the
 *   MSA_OP_INDEX_TOPK size.
 * msa_topk_merge: cand_scores / cand_ids [P, B, N, H_kv, topk] gathered in rank order -> blocks
 *   int32 [B, N, H_kv, topk+1]: Top-k of the union by (score desc, id asc) plus the local block,
 *   ascending, -1 padded (identical to msa_index_topk's output). 1 <= P <= 8.
 * msa_lse_idx_local: ml fp32 [B, N, H_kv, 2] = (a_p, z_p): the maximum of the index scores
 *   (scale_idx included) over the causal tokens of the row's selected blocks held here, and the
 *   sum of exp(score - a_p) over them; (-inf, 0) if this rank holds none. Workspace:
 *   msa_workspace_size(MSA_OP_LSE_IDX_LOCAL).
 * msa_lse_combine: eq (16) over ml [P, B, N, H_kv, 2] gathered in rank order: lse_idx fp32
 *   [B, N, H_kv] = a + log(z), a = max_p a_p, z = sum_p exp(a_p - a) z_p.
 */
typedef struct msa_key_ranges {
    int32_t n;        /* number of ranges: 1 or 2 */
    int32_t tok0[2];  /* first token of each range */
    int32_t ntok[2];  /* tokens in each range */
} msa_key_ranges;

MSA_API msa_status msa_index_topk_local(const msa_dims *dims, const void *q_idx, const void *k_idx_local,
                                        const msa_key_ranges *held, float *cand_scores, int32_t *cand_ids, void *ws,
                                        size_t ws_bytes, msa_stream_t stream);
MSA_API msa_status msa_topk_merge(const msa_dims *dims, int P, const float *cand_scores, const int32_t *cand_ids,
                                  int32_t *blocks, msa_stream_t stream);
MSA_API msa_status msa_lse_idx_local(const msa_dims *dims, const void *q_idx, const void *k_idx_local,
                                     const msa_key_ranges *held, const int32_t *blocks, float *ml, void *ws,
                                     size_t ws_bytes, msa_stream_t stream);
MSA_API msa_status msa_lse_combine(const msa_dims *dims, int P, const float *ml, float *lse_idx, msa_stream_t stream);

/*
 * Backward of msa_sparse_attn_fwd with the selection held fixed ("2.4 · 训练原生稀疏", section 2.2,
 * eq (11): on a fixed set the selected attention is ordinary attention, and positions outside the
 * set get no gradient). With J, o and LSE as in the forward and g = dout[b,i,h]:
 *   P_j = exp(q.k_j * scale - LSE),   dS_j = P_j * (g.v_j - g.o)        (j in J)
 *   dq[b,i,h]   = scale * sum_j dS_j k_j
 *   dk[b,j,r]   = scale * sum over (i, h in group r) with j in J of dS_j q[b,i,h]
 *   dv[b,j,r]   = sum over the same (i, h) of P_j g
 * The computation stays on the selected (query, block) pairs: no dense score matrix.
 *   q, k, v, blocks  as for msa_sparse_attn_fwd
 *   out    fp32 [B, N, H_q, d]   the forward's output (used for g.o)
 *   lse    fp32 [B, N, H_q]      the forward's LSE
 *   dout   bf16 [B, N, H_q, d]   upstream gradient
 *   dq fp32 [B, N, H_q, d]; dk, dv fp32 [B, N, H_kv, d]              (outputs)
 * P and dS enter the tensor cores as bf16 (as the forward's P does); the products accumulate in
 * fp32. dq, dk and dv are accumulated with fp32 reductions (atomics) and may differ in the last bits
 * between runs. Supports G = H_q / H_kv in {8, 16, 32} (MSA_ERR_UNSUPPORTED otherwise).
 */
MSA_API msa_status msa_sparse_attn_bwd(const msa_dims *dims, const void *q, const void *k, const void *v,
                                       const int32_t *blocks, const float *out, const float *lse, const void *dout,
                                       float *dq, float *dk, float *dv, void *ws, size_t ws_bytes,
                                       msa_stream_t stream);

/*
 * One decode step per sequence: index Top-k then sparse attention for the newest token, whose K, V
 * and K_idx are already in the caches at position cache_len[b]-1 (MSA blog, decode; the pages'
 * rule that decode and prefill compute the same R_theta and A_phi).
 *   dims->N    cache capacity L (rows of the caches)
 *   cache_len  int32 [B] device, 1 <= cache_len[b] <= N. A value outside [1, N] is clamped into it
 *              on the device and reported as MSA_ERR_DEVICE_CHECK by msa_get_device_status.
 *   q          bf16 [B, H_q, d];  q_idx bf16 [B, H_kv, d_idx]
 *   k_cache, v_cache bf16 [B, N, H_kv, d];  k_idx_cache bf16 [B, N, d_idx]
 *   out        fp32 [B, H_q, d]: the fp32-accumulated result        (output)
 *   blocks_out int32 [B, H_kv, topk+1] or NULL                       (output)
 *   margin_out fp32 [B, H_kv] or NULL: the cutoff margin r_(k) - r_(k+1) of each (sequence, group)
 *              ranking of block maxima (scaled by scale_idx), +inf when every complete past block
 *              is taken ("4.1.1 · 监督与联合训练", section 1.1, eq (9): a small margin marks
 *              the rows whose selection FP8 rounding or reduction order can flip)   (output)
 * Needs ceil(N / block_k) <= 8192 cache blocks (MSA_ERR_UNSUPPORTED otherwise).
 */
MSA_API msa_status msa_sparse_attn_decode(const msa_dims *dims, const int32_t *cache_len, const void *q, const void *q_idx,
                                  const void *k_cache, const void *v_cache, const void *k_idx_cache, float *out,
                                  int32_t *blocks_out, float *margin_out, void *ws, size_t ws_bytes,
                                  msa_stream_t stream);

/*
 * Row-wise e4m3 quantisation: the serving copy of the index keys. The selector keys are kept in
 * bf16 for training and quantised to FP8 for inference ("4.1.1 · 监督与联合训练", section 2;
 * "MSA Indexer 与 DSA Lightning Indexer 的差别", section 3.1: the indexer can run in FP8).
 * For each row r of x:
 *   scale[r]   = max_c |x[r,c]| / 448 in fp32 (1 for an all-zero row)
 *   codes[r,c] = e4m3(x[r,c] / scale[r]): the fp32 quotient rounded to the nearest e4m3 value
 *                (ties to even mantissa), saturated to +-448; e4m3 = 1 sign, 4 exponent (bias 7)
 *                and 3 mantissa bits, finite range +-448, no infinities
 *   x     bf16  [rows, n]
 *   codes uint8 [rows, n] (e4m3 bit patterns)                          (output)
 *   scale fp32  [rows]                                                 (output)
 * n in {16, 32, 64, 128, 256}; rows >= 0 (0 enqueues nothing). Used on a K_idx cache, rows = B*N
 * and n = d_idx give the layout msa_sparse_attn_decode_fp8idx reads.
 */
MSA_API msa_status msa_quantize_e4m3_rows(const void *x, int64_t rows, int n, uint8_t *codes, float *scale,
                                          msa_stream_t stream);

/*
 * msa_sparse_attn_decode with FP8 index scoring: the K_idx cache is held as e4m3 codes with one
 * fp32 scale per token (msa_quantize_e4m3_rows of the bf16 keys), half the bytes of the index
 * scan that dominates a decode step. Q_idx stays bf16 in memory; the step rounds each (sequence,
 * group) row to e4m3 with the same row-scale rule. The index score of token j for group r is
 *   S_j = scale_idx * sq_r * sk_j * sum_c q8_r[c] * k8_j[c]
 * with every product exact and the sum accumulated in fp32; pooling, Top-k, the local block and
 * the attention are those of msa_sparse_attn_decode. Rows whose bf16 margin is small may select
 * other blocks than the bf16 step: margin_out (the FP8 ranking's margin) reports them.
 *   k_idx_codes uint8 [B, N, d_idx];  k_idx_scale fp32 [B, N]
 * Other arguments, sizes and errors as msa_sparse_attn_decode; same workspace.
 */
MSA_API msa_status msa_sparse_attn_decode_fp8idx(const msa_dims *dims, const int32_t *cache_len, const void *q,
                                                 const void *q_idx, const void *k_cache, const void *v_cache,
                                                 const uint8_t *k_idx_codes, const float *k_idx_scale, float *out,
                                                 int32_t *blocks_out, float *margin_out, void *ws, size_t ws_bytes,
                                                 msa_stream_t stream);

/*
 * KL alignment of the index branch ("MSA 中的 KL 对齐与局部知识蒸馏", sections 2, 3 and 6).
 * On the selected causal token set J of each (query i, group r):
 *   teacher P_j     = (1/G) sum_{h in group r} exp(q_h . k_j * scale - lse[b,i,h])
 *   student P^idx_j = exp(S^idx_{i,j} - LSE_idx[b,i,r])
 *   loss            = sum_{b,i,r} KL(P || P^idx) / (B * N * H_kv)
 *   g_j             = grad_scale * (P^idx_j - P_j) / (B * N * H_kv)
 *   dq_idx[b,i,r]   = sum_j g_j * k_idx[b,j] * scale_idx
 *   dk_idx[b,j]     = sum_{i,r : j in J} g_j * q_idx[b,i,r] * scale_idx
 * The teacher is detached: no gradient reaches q or k.
 *   q bf16 [B,N,H_q,d]; k bf16 [B,N,H_kv,d]; q_idx bf16 [B,N,H_kv,d_idx]; k_idx bf16 [B,N,d_idx]
 *   blocks  int32 [B,N,H_kv,topk+1] (the selection the forward used)
 *   lse     fp32 [B,N,H_q]   the main forward's LSE (msa_sparse_attn_fwd)
 *   lse_idx fp32 [B,N,H_kv] or NULL (then computed here)
 *   loss fp32 [1]; dq_idx fp32 [B,N,H_kv,d_idx]; dk_idx fp32 [B,N,d_idx]   (outputs)
 */
MSA_API msa_status msa_kl_fwd_grad(const msa_dims *dims, const void *q, const void *k, const void *q_idx,
                           const void *k_idx, const int32_t *blocks, const float *lse, const float *lse_idx,
                           float grad_scale, float *loss, float *dq_idx, float *dk_idx, void *ws, size_t ws_bytes,
                           msa_stream_t stream);

/*
 * Dense warm-up of the KL alignment ("MSA 中的 KL 对齐与局部知识蒸馏", section 5: the index branch
 * is first aligned to a teacher over the whole causal context, before sparse training): the KL of
 * msa_kl_fwd_grad with every causal block selected, J = { j <= i }. The teacher's per-head LSE is
 * the dense causal attention LSE, computed here over all keys (or returned through lse_out); LSE_idx
 * likewise. With the same definitions as msa_kl_fwd_grad:
 *   loss            = sum_{b,i,r} KL(P || P^idx) / (B * N * H_kv)
 *   dq_idx, dk_idx  = grad_scale times the gradients of that loss
 *   q, k, q_idx, k_idx  as for msa_kl_fwd_grad (topk is not used)
 *   loss fp32 [1]; dq_idx fp32 [B,N,H_kv,d_idx]; dk_idx fp32 [B,N,d_idx]             (outputs)
 *   lse_out fp32 [B,N,H_q] or NULL: the teacher's LSE (natural log, scaled logits)  (output)
 * Sizes: those of msa_kl_fwd_grad, block_k in {32, 64, 128}, and B*H_kv*N*N/(2*block_k) < 2^31 list
 * entries (N = 262144 fits with H_kv = 4). The workspace (MSA_OP_KL_DENSE) holds the dense inverse
 * lists and one (max, sum-exp) pair per (row, block): about 1.5 GB at N = 65536, H_kv = 4. dQ_idx,
 * dK_idx and the per-row KL terms are accumulated with float atomics: the results may differ in the
 * last bits between runs.
 */
MSA_API msa_status msa_kl_dense_fwd_grad(const msa_dims *dims, const void *q, const void *k, const void *q_idx,
                                         const void *k_idx, float grad_scale, float *loss, float *dq_idx,
                                         float *dk_idx, float *lse_out, void *ws, size_t ws_bytes,
                                         msa_stream_t stream);

/*
 * Allocation-free decode step (no counterpart in the pages; a convenience of this library).
 * For callers that cannot allocate device memory where they decode (a plugin inside a host
 * application that owns every device allocation, a serving loop with a memory budget fixed at
 * start-up, a latency-bound path that must not call cudaMalloc, which can synchronise the device).
 * Same arguments, outputs and results as msa_sparse_attn_decode, minus the workspace and the
 * margin output: the scratch
 * is a static device array of MSA_DECODE_STATIC_SCRATCH_BYTES (16 MiB) that every GPU loading this
 * library holds until the process exits. It allocates and frees nothing.
 * - Returns MSA_ERR_WORKSPACE when `dims` need more scratch than that maximum
 *   (msa_workspace_size(MSA_OP_DECODE, dims) > MSA_DECODE_STATIC_SCRATCH_BYTES), e.g. the 16 x 262144
 *   decode step needs about 9.5 MiB, 32 sequences of 262144 tokens would not fit.
 * - The first call on a device looks up the array's device address with that device current
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 * - All calls on one device share the array and it keeps the last call's contents; calls that can
 *   overlap on the GPU (unordered streams) race on it and must be serialised by the caller.
 * - The device status word of these calls lives in the shared array: read it with
 *   msa_decode_noalloc_status, not msa_get_device_status.
 * - The array's device address is cached per device ordinal for the life of the process: the
 *   entry point assumes the device's primary context (the one the CUDA runtime uses) throughout,
 *   with no cudaDeviceReset in between.
 */
#define MSA_DECODE_STATIC_SCRATCH_BYTES (16u << 20)
MSA_API msa_status msa_sparse_attn_decode_noalloc(const msa_dims *dims, const int32_t *cache_len, const void *q,
                                                  const void *q_idx, const void *k_cache, const void *v_cache,
                                                  const void *k_idx_cache, float *out, int32_t *blocks_out,
                                                  msa_stream_t stream);
/*
 * Device status of the last msa_sparse_attn_decode_noalloc call on the current device: synchronises
 * `stream`, then reads the status word in the static array. MSA_OK, MSA_ERR_TIMEOUT or
 * MSA_ERR_DEVICE_CHECK (MSA_ERR_CUDA if the stream holds an error or the lookup fails). It
 * allocates nothing.
 */
MSA_API msa_status msa_decode_noalloc_status(msa_stream_t stream);

/*
 * Synchronises `stream`, then reads the device status word of the last call that used `ws`:
 * MSA_OK, MSA_ERR_TIMEOUT or MSA_ERR_DEVICE_CHECK (or MSA_ERR_CUDA if the stream holds an error).
 */
MSA_API msa_status msa_get_device_status(const void *ws, msa_stream_t stream);

/*
 * Test hooks of the failure-detection path (no counterpart in the pages). Every wait inside a
 * kernel of this library (an mbarrier, a copy or MMA completion, a work-queue poll) is bounded by
 * a time limit, 2 s by default. A wait that runs out sets MSA_ERR_TIMEOUT in the call's status
 * word; the kernel drains the copies and MMAs it issued, frees its TMEM and returns, leaving the
 * context usable.
 * msa_debug_set_wait_ns: the limit (ns) of every bounded wait of the calls made after it, in all
 *   threads of the process; 0 restores the default. For tests only: a short limit turns ordinary
 *   latency into timeouts.
 * msa_debug_wait_probe: one launch whose consumer waits on an mbarrier that its producer never
 *   arrives on, while the producer's bulk copy of 4096 bytes (read from ws + 256) is in flight and
 *   the CTA holds TMEM. The wait can only run out: msa_get_device_status(ws) then returns
 *   MSA_ERR_TIMEOUT. ws: at least 256 + 4096 bytes, 256-byte aligned (MSA_ERR_WORKSPACE otherwise).
 */
MSA_API void msa_debug_set_wait_ns(unsigned long long ns);
MSA_API msa_status msa_debug_wait_probe(void *ws, size_t ws_bytes, msa_stream_t stream);

/*
 * Test hook of the FMA-pipe exponential (no counterpart in the pages). The teacher-LSE loop of the
 * dense warm-up is bound by the MUFU pipe, so it computes part of its exponentials as 2^x = 2^j 2^f
 * (Cody-Waite reduction to f in [-1/2, 1/2], a degree-5 minimax polynomial for 2^f) on the FMA pipe.
 * msa_debug_exp2_fma: y[i] = that 2^x[i] for i < n (device pointers to n fp32 values, enqueued on
 *   `stream`). Relative error <= 3e-7 for -125 <= x <= 1/2; x below -125 (and -inf) gives 2^-125.
 *   MSA_ERR_INVALID_ARG for n < 0 or a null pointer with n > 0.
 */
MSA_API msa_status msa_debug_exp2_fma(const float *x, float *y, int64_t n, msa_stream_t stream);

/*
 * Kernel timing (off by default). While enabled, every entry point records a pair of CUDA events
 * on its stream around each kernel it launches. msa_profile_read synchronises on those events,
 * adds their durations per kernel name and clears the record: on return names[x] / total_ms[x] /
 * launches[x] hold up to `cap` kernels; the return value is the number of kernels written, or -1
 * on a CUDA error. At most 4096 launches are recorded between reads; later ones are not timed.
 */
MSA_API void msa_profile_enable(int on);
MSA_API int msa_profile_read(const char **names, double *total_ms, int *launches, int cap);

/* Static, human-readable name of a status code. */
MSA_API const char *msa_status_string(msa_status status);

/* Library version string ("msa-b200 <semver>"). */
MSA_API const char *msa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H */
