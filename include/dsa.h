/*
 * dsa.h - C ABI of the DeepSeek Sparse Attention (DSA) hot path on NVIDIA B200 (sm_100a).
 *
 * The path, as defined by the DeepSeek-V3.2 pages:
 *   1. lightning-indexer scores      ("DeepSeek-V3.2" analysis page, sec. 1.1, eq. (1))
 *   2. per-query top-k selection S_t (same page, sec. 1.1, eq. (2) and the S_t of eq. (4))
 *   3. attention in MLA's MQA mode over only the selected latent entries c_s
 *      (same page, sec. 1.1, eq. (2) and the MQA-mode paragraph; V3.2-Exp page, sec. 1)
 *   4. the sparse-stage indexer loss L^I = sum_t KL(p[t,S_t] || Softmax(I[t,S_t]))
 *      ("DSA Continued Pre-Training" page, Stage 2; analysis page eq. (4)), where p is the
 *      main attention summed over heads and L1-normalised ("DSA Continued Pre-Training",
 *      Stage 1).
 *
 * Shapes and positions.  B sequences; Lq queries and Lk keys per sequence.  Query i of a
 * sequence sits at absolute position t = i + (Lk - Lq) and sees keys s <= t (prefill:
 * Lq == Lk; decode: Lq == 1 and the query sees its whole context).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, dense, row-major,
 *     contiguous, 16-byte aligned.  The library never allocates, frees or synchronises
 *     (except dsa_last_device_status, which is documented as synchronising).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default).
 *   - Arguments are validated on the host before any launch; a failed check returns
 *     DSA_ERR_INVALID_ARG (bad pointer, size or alignment) or DSA_ERR_UNSUPPORTED (a shape
 *     outside the compiled kernels) and launches nothing.
 *   - A launch failure returns DSA_ERR_CUDA.  The device must be sm_100 (B200) or the call
 *     returns DSA_ERR_NO_SM100.
 *   - Every wait inside a kernel is bounded in time; on expiry the kernel records
 *     DSA_ERR_TIMEOUT in a device status word and exits.  dsa_last_device_status reads it.
 *   - `ws` / `ws_bytes` is caller-owned device scratch of at least dsa_workspace_bytes()
 *     for the same op and sizes (ws may be NULL when that size is 0).
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,
  DSA_ERR_UNSUPPORTED = 2,
  DSA_ERR_CUDA = 3,
  DSA_ERR_NO_SM100 = 4,
  DSA_ERR_TIMEOUT = 5
} dsa_status;

/* A cudaStream_t passed through the ABI without CUDA headers. */
typedef void* dsa_stream_t;

enum {
  DSA_OP_INDEXER = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_SPARSE_MLA_FWD = 2,
  DSA_OP_INDEXER_KL = 3,
  DSA_OP_DENSE_MLA_FWD = 4,
  DSA_OP_INDEXER_KL_DENSE = 5,
  DSA_OP_INDEXER_TOPK = 6,
  DSA_OP_MASKED_MHA = 7
};

/* Human-readable name of a status code (static string, never NULL). */
const char* dsa_status_str(dsa_status s);

/* ABI version of this library (major*100 + minor). */
int dsa_version(void);

/* Bytes of scratch the op needs for these sizes on the CURRENT device (0 if none).
 * op: DSA_OP_*.  Unused size arguments are ignored (pass 0).  Returns 0 for unknown ops. */
size_t dsa_workspace_bytes(int op, int B, int Lq, int Lk, int k, int H);

/*
 * Lightning indexer ("DeepSeek-V3.2" analysis page, sec. 1.1, eq. (1)):
 *   scores[b,i,s] = sum_{j<H_I} w[b,i,j] * max(0, sum_{d<d_I} q_I[b,i,j,d] * k_I[b,s,d])
 * for s <= t(i), and -infinity for s > t(i).
 *   q_fp8  [B, Lq, H_I, d_I]  FP8 E4M3 (OCP "fn"), one byte per element
 *   k_fp8  [B, Lk, d_I]       FP8 E4M3, the single shared key head
 *   w      [B, Lq, H_I]       fp32 per-head weights
 *   scores [B, Lq, Lk]        fp32 output
 * Products are exact in FP8 and accumulate in fp32 on the tensor cores; the ReLU, the
 * w-weighted head sum and the causal mask run in fp32 in the epilogue, so the
 * [Lq, Lk, H_I] intermediate is never written.  For integer-valued inputs whose
 * partial sums stay below 2^24 ulps the result is exact (bit-identical to fp64).
 * Supported: (H_I, d_I) with H_I in {4, 8, 16, 32, 64} and d_I in {32, 64, 128};
 * 1 <= Lq <= Lk.  ws: unused (pass NULL, 0).
 */
dsa_status dsa_indexer(const void* q_fp8, const void* k_fp8, const float* w, float* scores, int B,
                       int Lq, int Lk, int H_I, int d_I, void* ws, size_t ws_bytes,
                       dsa_stream_t stream);

/*
 * Top-k selection ("DeepSeek-V3.2" analysis page, sec. 1.1, eq. (2); S_t of eq. (4)):
 * for each query row, the n = min(k, t+1) positions s <= t with the largest scores.
 * Ties are broken toward the smaller position, so the set is unique.
 *   scores [B, Lq, Lk] fp32 (only s <= t is read)
 *   idx    [B, Lq, k]  int32 output: the n selected positions in ascending order,
 *                      then -1 in slots n..k-1
 * Scores must not be NaN.  Supported: 1 <= k <= 4096, Lk <= 262144.
 * ws: unused (pass NULL, 0).
 */
dsa_status dsa_topk(const float* scores, int32_t* idx, int B, int Lq, int Lk, int k, void* ws,
                    size_t ws_bytes, dsa_stream_t stream);

/*
 * Indexer and top-k in one call: dsa_indexer followed by dsa_topk, with identical results
 * (scores and idx as those two entry points define them).  For decode (Lq == 1, (H_I, d_I) in
 * {(64, 128), (32, 128)}) the two are fused: the indexer's epilogue also counts each row's
 * visible scores by the top-k's first radix digit, so the selection starts from that histogram
 * instead of counting the row itself (the "fused top-k" the "DeepSeek-V3.2" analysis page names
 * among the indexer's constant-factor savings, sec. 5.2 closing paragraph; decode step cost of
 * sec. 5.3, eq. (23)).
 *   ws: dsa_workspace_bytes(DSA_OP_INDEXER_TOPK, B, Lq, Lk, k, 0) bytes (the per-row histograms,
 *       B * Lq * 8 KiB for decode, 0 otherwise).  It must be zero-filled before its first use
 *       (e.g. one cudaMemset); every call whose kernels complete leaves it zero-filled again, so
 *       no clearing is needed between calls.  After a call that fails on the device (a status
 *       other than DSA_OK from dsa_last_device_status) clear it again.  Calls that share one ws
 *       must not overlap on the GPU.
 * Supported: the union of dsa_indexer's and dsa_topk's limits.
 */
dsa_status dsa_indexer_topk(const void* q_fp8, const void* k_fp8, const float* w, float* scores,
                            int32_t* idx, int B, int Lq, int Lk, int H_I, int d_I, int k, void* ws,
                            size_t ws_bytes, dsa_stream_t stream);

/*
 * Decode over a paged cache with per-row lengths ("DeepSeek-V3.2" analysis page, sec. 5.1: a
 * query's candidates may sit in a few contiguous cache pages or be spread over k pages, and a
 * per-row seq_lens keeps a batch of different context lengths from being padded to the longest).
 * The caches are pools of pages of page_size entries; sequence b's entry s sits in page
 * block_table[b * max_pages + s / page_size] at row s % page_size, max_pages =
 * ceil(max_len / page_size), and sequence b's query sees s < seq_lens[b] (t = seq_lens[b] - 1).
 * Same results as dsa_indexer_topk / dsa_sparse_mla_fwd on each sequence's contiguous cache.
 *   q_fp8 [B,1,H_I,d_I] e4m3, k_pages [num_pages,page_size,d_I] e4m3, w [B,1,H_I] fp32,
 *   block_table [B, max_pages] int32, seq_lens [B] int32 (device; values outside [0, max_len]
 *   are clamped and a page index outside [0, num_pages) reads as an empty entry, both recorded
 *   as DSA_ERR_INVALID_ARG in the device status word)
 *   scores [B,1,max_len] fp32 (-inf for s >= seq_lens[b]), idx [B,1,k] int32
 *   ws: dsa_workspace_bytes(DSA_OP_INDEXER_TOPK, B, 1, max_len, k, 0) bytes, zero-filled before
 *   its first use and left so by every call (as for dsa_indexer_topk)
 * Supported: page_size a multiple of 64, (H_I, d_I) in {(64, 128), (32, 128)}, k <= 4096,
 * max_len <= 262144.
 */
dsa_status dsa_indexer_topk_paged(const void* q_fp8, const void* k_pages, const float* w,
                                  const int32_t* block_table, const int32_t* seq_lens, float* scores,
                                  int32_t* idx, int B, int max_len, int num_pages, int page_size,
                                  int H_I, int d_I, int k, void* ws, size_t ws_bytes,
                                  dsa_stream_t stream);

/*
 * dsa_sparse_mla_fwd for decode over a paged latent cache (layout as dsa_indexer_topk_paged):
 *   q_bf16 [B,1,H,576] bf16, kv_pages [num_pages,page_size,576] bf16, idx [B,1,k] int32
 *   (positions within each sequence), out_bf16 [B,1,H,512], lse [B,1,H] (nullable)
 *   ws: dsa_workspace_bytes(DSA_OP_SPARSE_MLA_FWD, B, 1, max_len, k, H) bytes
 * Supported: page_size a multiple of 64, (d_qk, d_v) = (576, 512), H <= 128, k <= 65536.
 */
dsa_status dsa_sparse_mla_fwd_paged(const void* q_bf16, const void* kv_pages, const int32_t* idx,
                                    const int32_t* block_table, const int32_t* seq_lens, int B,
                                    int max_len, int num_pages, int page_size, int H, int d_qk,
                                    int d_v, int k, float scale, void* out_bf16, float* lse, void* ws,
                                    size_t ws_bytes, dsa_stream_t stream);

/*
 * Masked MHA for short prefill ("DeepSeek-V3.2-Exp" page, sec. 3, inference costs: for short
 * prefills DSA is simulated with MLA's MHA mode and a mask; "DeepSeek-V3.2" analysis page,
 * sec. 1.1, the MHA/MQA-mode paragraph and Fig. 7).  In MHA mode every head h has its own
 * decompressed keys and values; query t of head h attends only to the positions of its top-k
 * set S_t (idx, -1 = empty slot; a position is used only if it is also <= t):
 *   z_s = scale * <q[b,t,h,:], k[b,s,h,:]>,  P = softmax over s in S_t, s <= t
 *   out[b,t,h,:] = sum_s P_s v[b,s,h,:],  lse[b,t,h] = ln sum_s exp(z_s)
 * This equals DSA's MQA-mode attention over S_t once the decompression is absorbed.
 *   q_bf16, k_bf16 [B, L, H, 192] bf16 (128 + 64 rope dims), v_bf16 [B, L, H, 128] bf16,
 *   idx [B, L, k] int32, out_bf16 [B, L, H, 128] bf16, lse [B, L, H] fp32 (nullable)
 *   ws: dsa_workspace_bytes(DSA_OP_MASKED_MHA, B, L, L, k, H) bytes (the selection bitmap)
 * Causal prefill only (every query of the sequence, t = 0 .. L-1).  bf16 tensor-core products,
 * fp32 softmax and accumulation.  Supported: d_qk = 192, d_v = 128, L <= 65536.
 */
dsa_status dsa_masked_mha_fwd(const void* q_bf16, const void* k_bf16, const void* v_bf16,
                              const int32_t* idx, int B, int L, int H, int d_qk, int d_v, int k,
                              float scale, void* out_bf16, float* lse, void* ws, size_t ws_bytes,
                              dsa_stream_t stream);

/*
 * HISA, block -> token retrieval for decode ("DeepSeek-V3.2" analysis page, sec. 5.3: a coarse
 * stage over block representatives, then exact indexer scores inside the kept blocks; cost
 * model eq. (25), recall decomposition eq. (24)).  The cache of each sequence is cut into blocks
 * of `block` keys (Lk a multiple of block).  A block is represented by the mean of its keys and
 * scored with the indexer's formula on that mean key, sum_j w_j ReLU(q_I[b,j,:] . mean); the r
 * blocks with the largest scores are kept (ties -> smaller block); every key in them gets its
 * exact score (eq. (1)) and idx holds the min(k, r*block) best of those keys (ties -> smaller
 * position), ascending, -1 padded.  With r * block >= Lk this is exactly dsa_indexer_topk's set.
 *
 * dsa_hisa_block_sums: the cache summary, computed once when the cache is written:
 *   k_fp8 [B,Lk,d_I] e4m3 -> sums [B, ceil(Lk/block), d_I] fp32 (the sums of each block's keys).
 * dsa_hisa_topk: one decode step's selection:
 *   q_fp8 [B,1,H_I,d_I] e4m3, k_fp8 [B,Lk,d_I] e4m3, w [B,1,H_I] fp32, block_sums from above,
 *   idx [B,1,k] int32 (output), blocks [B,1,r] int32 (nullable output: the kept blocks, ascending,
 *   -1 padded when Lk / block < r),
 *   ws: dsa_hisa_workspace_bytes(B, Lk, block, r, k) bytes, zero-filled before its first use
 *   and left so by every call (its histograms are those of dsa_indexer_topk).
 * Supported: block a multiple of 64, d_I = 128, H_I in {64, 32}, k <= 4096, r <= 4096,
 * r * block <= 262144.
 */
size_t dsa_hisa_workspace_bytes(int B, int Lk, int block, int r, int k);
dsa_status dsa_hisa_block_sums(const void* k_fp8, int B, int Lk, int d_I, int block, float* sums,
                               dsa_stream_t stream);
dsa_status dsa_hisa_topk(const void* q_fp8, const void* k_fp8, const float* w, const float* block_sums,
                         int B, int Lk, int H_I, int d_I, int block, int r, int k, int32_t* idx,
                         int32_t* blocks, void* ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * Sparse attention in MLA's MQA mode over the selected latents ("DeepSeek-V3.2" analysis
 * page, sec. 1.1, eq. (2) and the MQA-mode paragraph; renormalised form eq. (19)).
 * Every query head shares the latent entry c_s = kv[b,s,:]; keys use all d_qk dims,
 * values are dims [0, d_v).  For each head h of query (b,i), over the valid slots
 * (idx >= 0) of idx[b,i,:]:
 *   z_h,j = scale * <q[b,i,h,:], kv[b,idx_j,:]>,   P_h,j = softmax_j(z_h,:)
 *   out[b,i,h,:] = sum_j P_h,j * kv[b,idx_j,0:d_v],  lse[b,i,h] = ln sum_j exp(z_h,j)
 * If p_sel is not NULL it also writes the head-summed, L1-normalised target
 * ("DSA Continued Pre-Training" page, Stage 1/2):
 *   p_sel[b,i,j] = sum_h P_h,j / sum_j' sum_h P_h,j'   (= sum_h P_h,j / H), 0 for empty slots.
 *   q_bf16  [B, Lq, H, d_qk] bf16     kv_bf16 [B, Lk, d_qk] bf16    idx [B, Lq, k] int32
 *   out_bf16 [B, Lq, H, d_v] bf16     lse [B, Lq, H] fp32 (nullable)
 *   p_sel   [B, Lq, k] fp32 (nullable)
 * Every valid idx must lie in [0, Lk); a row with no valid slot gets out = 0, lse = -infinity.
 * bf16 tensor-core products with fp32 accumulation and fp32 softmax; bf16 output (RNE).
 * Supported: H <= 128, (d_qk, d_v) in {(576, 512), (80, 64)}, 1 <= k <= 65536.
 * ws: dsa_workspace_bytes(DSA_OP_SPARSE_MLA_FWD, B, Lq, Lk, k, H) bytes (split-KV partials
 * when there are too few query rows to fill the GPU; 0 otherwise).
 */
dsa_status dsa_sparse_mla_fwd(const void* q_bf16, const void* kv_bf16, const int32_t* idx, int B,
                              int Lq, int Lk, int H, int d_qk, int d_v, int k, float scale,
                              void* out_bf16, float* lse, float* p_sel, void* ws, size_t ws_bytes,
                              dsa_stream_t stream);

/*
 * Sparse-stage indexer loss ("DSA Continued Pre-Training" page, Stage 2; "DeepSeek-V3.2"
 * analysis page, eq. (4)):
 *   L^I = sum_{b,i} sum_{j valid} p[b,i,j] * (ln p[b,i,j] - ln q[b,i,j]),
 *   q[b,i,:] = Softmax over the valid slots of scores[b,i,idx[b,i,:]],  0 * ln 0 = 0.
 *   scores [B, Lq, Lk] fp32, idx [B, Lq, k] int32, p_sel [B, Lq, k] fp32
 *   loss   device pointer to one fp32 (written)
 *   loss_per_query [B, Lq] fp32 (nullable): the per-row KL terms
 * fp32 per-row arithmetic; the sum over rows is taken in a fixed order (deterministic).
 * ws: dsa_workspace_bytes(DSA_OP_INDEXER_KL, B, Lq, 0, k, 0) bytes.
 */
dsa_status dsa_indexer_kl(const float* scores, const int32_t* idx, const float* p_sel, int B,
                          int Lq, int Lk, int k, float* loss, float* loss_per_query, void* ws,
                          size_t ws_bytes, dsa_stream_t stream);

/*
 * Dense warm-up, main attention and its target ("DSA Continued Pre-Training" page, Stage 1;
 * "DeepSeek-V3.2" analysis page, sec. 1.1, the dense warm-up paragraph and eq. (3)): causal MQA
 * over EVERY position s <= t(i), the attention the indexer is aligned with before top-k
 * selection is switched on.  Same arithmetic as dsa_sparse_mla_fwd with slot j read as position
 * j (k = Lk):
 *   out[b,i,h,:] = sum_{s<=t} P_h,s kv[b,s,0:d_v],  lse[b,i,h] = ln sum_{s<=t} exp(z_h,s)
 *   p_full[b,i,s] = sum_h P_h,s / H  for s <= t, 0 for s > t   (the target p[t,:] of eq. (3))
 *   q_bf16 [B,Lq,H,d_qk] bf16, kv_bf16 [B,Lk,d_qk] bf16, out_bf16 [B,Lq,H,d_v] bf16,
 *   lse [B,Lq,H] fp32 (nullable), p_full [B,Lq,Lk] fp32 (nullable)
 * Supported: H <= 128, (d_qk, d_v) in {(576, 512), (80, 64)}, Lk <= 65536.
 * ws: dsa_workspace_bytes(DSA_OP_DENSE_MLA_FWD, B, Lq, Lk, 0, H) bytes.
 */
dsa_status dsa_dense_mla_fwd(const void* q_bf16, const void* kv_bf16, int B, int Lq, int Lk, int H,
                             int d_qk, int d_v, float scale, void* out_bf16, float* lse, float* p_full,
                             void* ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * Dense warm-up indexer loss, eq. (3) ("DSA Continued Pre-Training" page, Stage 1):
 *   L^I = sum_{b,i} sum_{s<=t} p[b,i,s] (ln p[b,i,s] - ln q[b,i,s]),
 *   q[b,i,:] = Softmax(scores[b,i,0..t]),  0 * ln 0 = 0.
 *   scores [B,Lq,Lk] fp32 (dsa_indexer's output), p_full [B,Lq,Lk] fp32 (dsa_dense_mla_fwd's),
 *   loss: one fp32 (device), loss_per_query [B,Lq] fp32 (nullable)
 * fp32 per-row arithmetic, fixed-order fp64 sum over rows.
 * ws: dsa_workspace_bytes(DSA_OP_INDEXER_KL_DENSE, B, Lq, Lk, 0, 0) bytes (unused when
 * loss_per_query is given).
 */
dsa_status dsa_indexer_kl_dense(const float* scores, const float* p_full, int B, int Lq, int Lk,
                                float* loss, float* loss_per_query, void* ws, size_t ws_bytes,
                                dsa_stream_t stream);

/*
 * Gradient of the indexer loss with respect to the indexer's inputs.  The indexer is trained
 * from L^I alone, on a detached input ("DSA Continued Pre-Training" page, Stage 2; "DeepSeek-V3.2"
 * analysis page, eq. (4) and the detached-input paragraph), so this is the whole training signal
 * of q_I, w and k_I.  The selection is held fixed (top-k is piecewise constant); ReLU'(0) = 0:
 *   g_i       = Softmax_i(scores[b,i,idx_i]) * sum_i p_i - p_i          (dL/dI over the slots)
 *   dw[b,i,j] = sum_i g_i ReLU(a_ji),                a_ji = q_I[b,i,j,:] . k_I[b,idx_i,:]
 *   dq[b,i,j,:] = sum_i g_i w[b,i,j] [a_ji > 0] k_I[b,idx_i,:]
 *   dk[b,s,:] = sum over the queries i and slots with idx_i = s of g_i sum_j w[b,i,j] [a_ji > 0] q_I[b,i,j,:]
 * Dense warm-up (eq. (3)): idx = NULL and k = Lk; every s <= t is a slot and p_sel is the
 * [B, Lq, Lk] target of dsa_dense_mla_fwd.
 *   q_fp8 [B,Lq,H_I,d_I] e4m3, k_fp8 [B,Lk,d_I] e4m3, w [B,Lq,H_I] fp32, scores [B,Lq,Lk] fp32
 *   (dsa_indexer's output), idx [B,Lq,k] int32 (nullable), p_sel [B,Lq,k] fp32
 *   dq [B,Lq,H_I,d_I] fp32, dw [B,Lq,H_I] fp32, dk [B,Lk,d_I] fp32 (all written; dk is cleared on
 *   the stream, then accumulated with fp32 atomics, so its last bits depend on their order)
 * The recomputed q_I . k_I products run on the FP8 tensor cores; the gradient products on the
 * fp16 tensor cores with G split into two fp16 parts (inputs exact in fp16), fp32 accumulation.
 * Supported: H_I = 64, d_I = 128, k <= 65536.
 */
dsa_status dsa_indexer_bwd(const void* q_fp8, const void* k_fp8, const float* w, const float* scores,
                           const int32_t* idx, const float* p_sel, int B, int Lq, int Lk, int H_I,
                           int d_I, int k, float* dq, float* dw, float* dk, dsa_stream_t stream);

/*
 * The indexer loss of dsa_indexer_kl for callers that cannot hand the library any scratch
 * memory.  The pages have no counterpart to this entry point; it exists only for how memory
 * is provided.  Some callers cannot allocate device memory when they call in: a serving
 * runtime that reserves all of HBM up front and forbids further cudaMalloc, a plugin that
 * only receives pointers to its inputs and outputs, or a latency-critical thread that must
 * avoid the device-wide synchronisation cudaMalloc and cudaFree can cause.  This variant
 * takes the same arguments minus ws/ws_bytes and allocates nothing: when loss_per_query is
 * NULL, the per-row KL terms go to a fixed 4 MiB array inside the library (one per GPU that
 * loads it, held until the process exits).
 *   - At most 1048576 query rows (B * Lq); larger sizes return DSA_ERR_UNSUPPORTED without
 *     launching anything.
 *   - The first call on each device looks up that array's device address (with the device
 *     current); make that first call before any stream capture.
 *   - Every call shares the one array and leaves its rows in it; each call writes every row
 *     it reads, so nothing needs clearing, but calls whose kernels overlap on the GPU (on
 *     different streams, or from different host threads) race on it.  Serialise them.
 *   - No cudaMalloc, cudaFree or other allocating routine is called.  CUDA itself places the
 *     library's device code, this array included, in a device's memory when the library first
 *     launches a kernel or looks the array up on that device (already at load time under
 *     CUDA_MODULE_LOADING=EAGER).  A caller that will reserve all free device memory should
 *     therefore make one call of this entry point on each device before it does so.
 * Results are bit-identical to dsa_indexer_kl on the same inputs (same kernels, same
 * fixed-order sum).  Bad pointers, sizes or alignment (loss_per_query included) return
 * DSA_ERR_INVALID_ARG before anything is launched.
 */
dsa_status dsa_indexer_kl_noalloc(const float* scores, const int32_t* idx, const float* p_sel,
                                  int B, int Lq, int Lk, int k, float* loss,
                                  float* loss_per_query, dsa_stream_t stream);

/*
 * Failure detection ("DeepSeek-V3.2" analysis page, sec. 5.1: check inputs at entry and keep the
 * system observable).  Every wait inside a kernel of this library is bounded; by default a wait
 * gives up after 2 s, records DSA_ERR_TIMEOUT in the device status word and lets its kernel
 * return.  dsa_set_wait_limit_ns sets that bound, in nanoseconds, for kernels launched
 * afterwards on the CURRENT device (0 restores the default).  It is a synchronous copy: call it
 * while no kernel of this library runs on the device.
 */
dsa_status dsa_set_wait_limit_ns(uint64_t ns);

/*
 * Diagnostic: launches one warp on `stream` that waits on an mbarrier nothing arrives on.  The
 * wait expires after the current limit, DSA_ERR_TIMEOUT is recorded (read it with
 * dsa_last_device_status) and the kernel returns; the context stays usable.  Lets a test check
 * the failure-detection path without any fault.
 */
dsa_status dsa_selftest_wait(dsa_stream_t stream);

/*
 * Waits for `stream`, then returns and clears the device status word that kernels set
 * when a bounded wait expires (DSA_ERR_TIMEOUT) - DSA_OK if none did.  Synchronising;
 * meant for tests and diagnostics.  Returns DSA_ERR_CUDA if the stream itself failed.
 */
dsa_status dsa_last_device_status(dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
