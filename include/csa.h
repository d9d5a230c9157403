/*
 * csa.h — C ABI of libcsa.so: the forward hot path of a DeepSeek-V4-style
 * hybrid compressed attention layer (CSA: compressed sparse attention, HCA:
 * heavily compressed attention, SWA: sliding window, attention sink) on NVIDIA
 * B200 (sm_100a).
 *
 * Sources (secondary write-ups of the DeepSeek-V4 technical report):
 *   [CS] "DeepSeek V4 脱离 CUDA 全栈国产化：1.6T MoE 逐层拆解 + 昇腾迁移数据",
 *        §二 "CSA + HCA 混合注意力" (subsections "KV 压缩", "闪电索引器",
 *        "共享 KV MQA", "HCA（重压缩注意力）", "其他辅助设计").
 *   [LD] liduos.com "deepseek-v4-engineering-tradeoffs", "1M Context 的结构与取舍".
 *   [LQ] "Deepseek-V4 技术报告里最值得复现的三个改动", §3 (config block), §5.
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers owned by the caller; the library
 *     allocates no memory.  Scratch comes from a caller-supplied workspace whose
 *     size is queried first.
 *   - Tensors are dense row-major with the channel dimension innermost.  Every
 *     base pointer must be 16-byte aligned; row lengths in bytes must be
 *     multiples of 16.
 *   - dtype codes: CSA_F32 (float), CSA_BF16 (__nv_bfloat16), CSA_E4M3 (OCP FP8
 *     E4M3 "fn" byte).
 *   - Sequences: n_seq independent sequences; sequence b has T query tokens at
 *     absolute positions q_pos[b] + t (q_pos is a DEVICE int64 array [n_seq]).
 *     Per-sequence caches are strided by a row capacity `cap` (rows).
 *   - Compressed entry i of a sequence (compression ratio m) covers tokens
 *     [i*m, (i+1)*m) and is visible to the query at position p iff
 *     (i+1)*m - 1 <= p, i.e. n_vis(p) = min(cap, (p+1)/m).
 *   - All calls are asynchronous on `stream` and never abort.  Argument errors
 *     are reported before any launch; csa_last_error() describes the last
 *     failure.  Kernels that wait on on-chip barriers bound every wait and
 *     report expiry through the device error word (csa_check_device_error).
 *   - Results do not depend on batch position or launch geometry: no floating-
 *     point atomics are used (batch invariance, [CS] §八).
 */
#ifndef CSA_H_
#define CSA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CSA_OK = 0,
  CSA_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or flag */
  CSA_ERR_UNSUPPORTED = 2,   /* valid but unsupported shape/dtype combination */
  CSA_ERR_WORKSPACE = 3,     /* workspace missing or too small */
  CSA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  CSA_ERR_TIMEOUT = 5,       /* a bounded on-chip wait expired (device error word) */
  CSA_ERR_DEVICE = 6         /* a kernel recorded a bad gather index */
} csa_status_t;

typedef enum { CSA_F32 = 0, CSA_BF16 = 1, CSA_E4M3 = 2 } csa_dtype_t;

/* ABI version of this header (incremented on any signature change). */
int csa_abi_version(void);

/* Text of a status code, and a description of the most recent failure on the
 * calling thread (empty string if none).  Both pointers stay valid. */
const char* csa_status_string(csa_status_t s);
const char* csa_last_error(void);
/* Same text as csa_last_error(). */
const char* csa_get_last_error_string(void);

/* Synchronises `stream`, then reads and clears the device error words of the
 * current device.  Returns CSA_ERR_TIMEOUT or CSA_ERR_DEVICE if a kernel
 * recorded an expired wait or a bad gather index since the last check. */
csa_status_t csa_check_device_error(cudaStream_t stream);

/* Self-test of the failure path (no counterpart on the pages): launches one
 * thread that waits, through the same bounded on-chip wait the kernels use, on
 * a barrier phase that nothing completes, with a limit of limit_ns (1 us to
 * 100 ms) instead of the kernels' 2 s.  The wait expires, the expiry is
 * recorded in the device error word and the kernel returns, so the next
 * csa_check_device_error on the stream reports CSA_ERR_TIMEOUT and the context
 * stays usable.  No memory is touched besides the error word. */
csa_status_t csa_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_compress — softmax-gated KV compressor ([CS] "KV 压缩": an entry is the
 * per-channel Softmax(Z + B)-weighted sum of the content C over its block; CSA
 * blocks overlap the previous block, m = 4; HCA ([CS] "HCA") uses
 * non-overlapping m' = 128 blocks).  Tokens that do not fill a block form no
 * entry ([LQ] §5).
 *
 *   C, Z     [S, D] in_dtype (F32 or BF16): content and gate logits (stream a).
 *   Cb, Zb   previous-block stream [S, D] or NULL to reuse C, Z.
 *   B        [2m, D] fp32 if overlap (rows 0..m-1 weight the previous block,
 *            rows m..2m-1 the current block) else [m, D]; NULL = zero bias.
 *   overlap  1: entry i pools tokens [(i-1)m, (i+1)m) in ONE joint per-channel
 *            softmax (entry 0: its own block only); 0: tokens [i*m, (i+1)m).
 *   norm     1: RMSNorm over D (eps, unit gain) after pooling ([CS] "其他辅助设计").
 *   rope_dim RoPE on the last rope_dim dims (0 = off), entry i at position
 *            i*m, pairs (d, d + rope_dim/2), theta_j = rope_base^(-2j/rope_dim).
 *   out      [S/m, D] out_dtype (F32 or BF16).
 * Requires D % 8 == 0, 8 <= D <= 2048, 1 <= m <= 1024, S >= 0.
 * ------------------------------------------------------------------------- */
csa_status_t csa_compress(const void* C, const void* Z, const void* Cb, const void* Zb,
                          const float* B, int64_t S, int D, int m, int overlap,
                          csa_dtype_t in_dtype, int norm, int rope_dim, float rope_base,
                          float eps, void* out, csa_dtype_t out_dtype, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_rmsnorm_rope — QK normalisation and partial RoPE of raw rows ([CS]
 * "其他辅助设计": RMSNorm before core attention, RoPE on the last 64 dims).
 * Used for the queries (rows_per_pos = H heads share a position) and for the
 * raw window rows (rows_per_pos = 1).
 *   x   [rows, D] in_dtype; row r has position pos0 + r / rows_per_pos.
 *   out [rows, D] out_dtype.  norm, rope_dim, rope_base, eps as in csa_compress.
 * ------------------------------------------------------------------------- */
csa_status_t csa_rmsnorm_rope(const void* x, csa_dtype_t in_dtype, int64_t rows, int D,
                              int rows_per_pos, int64_t pos0, int norm, int rope_dim,
                              float rope_base, float eps, void* out, csa_dtype_t out_dtype,
                              cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_compress_append — decode-time cache writer ([CS] "KV 压缩": entries are
 * pooled block by block; "其他辅助设计": the non-RoPE dims are stored in FP8,
 * the 64 RoPE dims in BF16; [LD]: FP8 caches).  For every sequence b, the new
 * token at position p = q_pos[b] (rows c_tok[b], z_tok[b]) is stored in slot
 * p % 2m of the sequence's ring of the last 2m tokens; when it completes block
 * i = (p + 1) / m - 1, entry i is pooled from the ring exactly as csa_compress
 * pools it (per-channel softmax of Z + B over the current block and, with
 * overlap, the previous one), RMS-normalised (norm != 0), rotated at position
 * i * m, and written as cache row i:
 *     kv_nope[b, i, :D - rope_dim] = e4m3(entry / s),  s = max|entry[:D - rope_dim]| / 448
 *                                    (s = 1 for an all-zero row; round to nearest even, saturating)
 *     kv_rope[b, i, :]             = bf16(entry[D - rope_dim:])
 *     kv_scale[b, i]               = s
 * Tokens that complete no block only update the ring.
 *   c_tok, z_tok  [n_seq, D] in_dtype (F32 or BF16)    B [2m, D] (overlap) or [m, D] fp32
 *   q_pos         [n_seq] int64 (device): the new token's position
 *   ring_C/ring_Z [n_seq, 2m, D] in_dtype, caller-owned state: slot u % 2m holds
 *                 token u's rows; a stream that starts after a prefill copies the
 *                 last 2m prefill tokens' rows into their slots first
 *   kv_nope [n_seq, cap, D - rope_dim] e4m3, kv_rope [n_seq, cap, rope_dim] bf16,
 *   kv_scale [n_seq, cap] fp32: the cache layout the attention calls read; a
 *                 block whose index is >= cap writes nothing
 * Requires D a multiple of 8 in [64, 2048], 1 <= m <= 1024, rope_dim 0 or 64.
 * One CTA per sequence; asynchronous on `stream`.
 * ------------------------------------------------------------------------- */
csa_status_t csa_compress_append(const void* c_tok, const void* z_tok, csa_dtype_t in_dtype, const float* B,
                                 int n_seq, int D, int m, int overlap, const int64_t* q_pos, void* ring_C,
                                 void* ring_Z, uint8_t* kv_nope, void* kv_rope, float* kv_scale, int64_t cap,
                                 int norm, int rope_dim, float rope_base, float eps, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_cache_append — the whole decode-time cache write of a CSA layer in one
 * launch: the KV row as csa_compress_append (norm on) AND the lightning
 * indexer's key of the same block ([CS] "闪电索引器": the indexer scores the
 * compressed entries, so each entry has an index key; "KV 压缩": entries are
 * pooled block by block).  Reading taken where the pages are silent: the key
 * is pooled by the same per-channel softmax over its own stream (ci_tok,
 * zi_tok [n_seq, DI], bias B_I [2m or m, DI] fp32, ring_CI / ring_ZI
 * [n_seq, 2m, DI]) with no RMSNorm and no RoPE, and stored like a KV row with
 * rope_dim 0:  kI[b, i, :] = e4m3(key / s_I), kI_scale[b, i] = s_I =
 * max|key| / 448 (1 for an all-zero key) -- the layout csa_index_topk reads.
 * Other arguments, requirements and the ring contract are those of
 * csa_compress_append; DI a multiple of 16 in [16, 2048].  Grid: one CTA per
 * (sequence, stream).
 * ------------------------------------------------------------------------- */
csa_status_t csa_cache_append(const void* c_tok, const void* z_tok, csa_dtype_t in_dtype, const float* B, int n_seq,
                              int D, int m, int overlap, const int64_t* q_pos, void* ring_C, void* ring_Z,
                              uint8_t* kv_nope, void* kv_rope, float* kv_scale, int64_t cap, int rope_dim,
                              float rope_base, float eps, const void* ci_tok, const void* zi_tok, const float* B_I,
                              int DI, void* ring_CI, void* ring_ZI, uint8_t* kI, float* kI_scale,
                              cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_index_topk — lightning indexer + top-k ([CS] "闪电索引器": index heads,
 * ReLU of the similarity, weighted over heads; only the top-k entries are kept
 * for the query, [LD]).  For query token t of sequence b at p = q_pos[b] + t:
 *     I[s] = ks[s] * sum_h (w[h] * qs[h]) * ReLU(qI[h,:] . kI[s,:]),  s < n_vis(p)
 * computed with FP8 (e4m3) tensor-core products accumulated in fp32; the row
 * scales factor out of the ReLU because they are positive.  idx receives the
 * min(k, n_vis) entries with the largest I, equal scores going to the lower
 * entry index, in ascending order, padded with -1.
 *
 *   qI       [n_seq, T, HI, DI] e4m3     qI_scale [n_seq, T, HI] fp32 or NULL (1)
 *   w        [n_seq, T, HI] fp32 head weights
 *   kI       [n_seq, cap, DI] e4m3       kI_scale [n_seq, cap] fp32 or NULL (1)
 *   q_pos    [n_seq] int64 (device)
 *   idx      [n_seq, T, k] int32 out
 *   workspace / ws_bytes: at least csa_index_topk_workspace(n_seq, T, cap, k)
 *            bytes, 16-byte aligned, owned by the caller: the fp32 score matrix,
 *            for rows longer than 16384 entries the per-chunk candidates and a
 *            key histogram per row, and the work-item counter (the histograms
 *            and the counter are reset by the call with one stream-ordered memset).
 *            Contents are undefined afterwards; calls sharing one workspace must
 *            be ordered on one stream.  The selection kernels are launched as
 *            dependents of the scoring kernel (programmatic dependent launch):
 *            each waits for its predecessor's results before reading them.
 * Requires DI in {32, 64, 128}; HI in {1,2,4,...,64} (power of two <= 64 whose
 * product with the token block is a multiple of 16); 1 <= k <= 2048; cap >= 1.
 * Rows longer than 16384 entries are cut into chunks of 16384 whose candidates
 * are merged: ceil(cap / 16384) * k must not exceed 16384 (CSA_ERR_UNSUPPORTED
 * otherwise), which allows cap = 262144 entries (a 2^20-token context at
 * m = 4) at k = 1024 and cap = 131072 at k = 2048.
 * csa_index_topk_workspace returns 0 when n_seq * T * cap * 4 overflows size_t.
 * ------------------------------------------------------------------------- */
size_t csa_index_topk_workspace(int n_seq, int T, int64_t cap, int k);
csa_status_t csa_index_topk(const uint8_t* qI, const float* qI_scale, const float* w,
                            const uint8_t* kI, const float* kI_scale, const int64_t* q_pos,
                            int n_seq, int T, int HI, int DI, int64_t cap, int m, int k,
                            int32_t* idx, void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_index_topk_noalloc — csa_index_topk without a workspace argument.
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory, e.g. a plug-in inside an engine that has
 * already reserved the GPU's memory for its own pools, or a latency-critical
 * path that must not call cudaMalloc because it may synchronise the device.
 * Its scratch is one file-scope device array of 32 MiB in libcsa.so, which
 * every GPU that loads the library holds until the process exits.  Arguments
 * and results are those of csa_index_topk; a call whose scratch would exceed
 * 32 MiB (csa_index_topk_workspace(n_seq, T, cap, k), dominated by
 * n_seq * T * cap * 4 bytes of scores) returns CSA_ERR_UNSUPPORTED.
 * The first call in each CUDA context looks up the array's device address (a
 * CUDA runtime query, cached per context, so a context created after
 * cudaDeviceReset gets a fresh lookup); make that first call before any stream
 * capture.  Every call on a device shares the same array, which keeps the
 * previous call's contents: the call resets the work-item counter it uses
 * and, for rows longer than 16384 entries, its key histograms (one
 * stream-ordered memset inside the array before they are filled), and it
 * reads only score entries it has written itself, so earlier
 * contents never reach the result.  Calls that may overlap
 * on the GPU (different streams, or host threads racing) race on the array and
 * must be serialised by the caller.  No memory is allocated or freed.
 * ------------------------------------------------------------------------- */
csa_status_t csa_index_topk_noalloc(const uint8_t* qI, const float* qI_scale, const float* w,
                                    const uint8_t* kI, const float* kI_scale, const int64_t* q_pos,
                                    int n_seq, int T, int HI, int DI, int64_t cap, int m, int k,
                                    int32_t* idx, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_index_topk_fp4 — csa_index_topk with the QK path in FP4 ([CS] "闪电索引器":
 * the indexer's QK path runs in FP4; "其他辅助设计": the indexer is stored in
 * FP4).  Format (OCP MX FP4): E2M1 codes, two per byte with the even element in
 * the low nibble, and one E8M0 scale byte (2^(byte - 127)) per 32-element block.
 *   qI4 [n_seq, T, HI, 64] u8, qI4_scale [n_seq, T, HI, 4] u8,
 *   kI4 [n_seq, cap, 64] u8,   kI4_scale [n_seq, cap, 4] u8  (DI = 128).
 * Scores are those of csa_index_topk on the dequantised operands; on the GPU
 * the blocks are rescaled to each row's largest block scale in e4m3, exact while
 * a row's block scales span at most 2^8.  cap must be a multiple of 4.
 * Workspace: csa_index_topk_fp4_workspace(n_seq, T, HI, cap, k) bytes.
 * ------------------------------------------------------------------------- */
size_t csa_index_topk_fp4_workspace(int n_seq, int T, int HI, int64_t cap, int k);
csa_status_t csa_index_topk_fp4(const uint8_t* qI4, const uint8_t* qI4_scale, const float* w,
                                const uint8_t* kI4, const uint8_t* kI4_scale, const int64_t* q_pos, int n_seq,
                                int T, int HI, int64_t cap, int m, int k, int32_t* idx, void* workspace,
                                size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Attention over one shared K = V row set per query token ([CS] "共享 KV MQA":
 * the selected compressed entries act as both key and value; one KV head
 * shared by H query heads).  Logits are scale * q_h . row; softmax over the
 * row set.  Rows come from a KV store that is either
 *   kv_dtype BF16 / F32 : kv [n_seq, cap, D]
 *   kv_dtype E4M3       : kv [n_seq, cap, D - rope_dim] e4m3 codes (dequantised
 *                         as code * kv_scale[row]) + kv_rope [n_seq, cap, rope_dim]
 *                         bf16 ([CS] "其他辅助设计": RoPE dims BF16, rest FP8).
 * q [n_seq, T, H, D] (q_dtype BF16 or F32) is already normalised and rotated.
 * Outputs of the two partial calls: O_part [n_seq, T, H, D] fp32 normalised by
 * the branch's own softmax sum, lse_part [n_seq, T, H] fp32 natural-log
 * log-sum-exp of the branch logits (-inf and O = 0 when the set is empty).
 * Computation: when q, the entries and the window rows are all F32 (the
 * float32 workloads), fp32 arithmetic throughout on CUDA cores (fused
 * multiply-add dot products, expf); otherwise BF16 tensor-core products (an
 * F32 operand next to a BF16 one is rounded to BF16) with fp32 accumulation
 * and softmax.  Requires D in {128, 512}, H <= 64, rope_dim in {0, 64} (E4M3
 * needs 64).
 * ------------------------------------------------------------------------- */

/* csa_sparse_mqa — CSA main branch: rows kv[b, idx[b,t,j]] for idx >= 0.
 *   idx [n_seq, T, k] int32, ascending, -1 padded (as produced by csa_index_topk).
 *   An index >= cap is ignored and recorded as CSA_ERR_DEVICE. */
csa_status_t csa_sparse_mqa(const void* q, csa_dtype_t q_dtype, const void* kv,
                            csa_dtype_t kv_dtype, const void* kv_rope, const float* kv_scale,
                            int64_t cap, const int32_t* idx, int k, int n_seq, int T, int H,
                            int D, int rope_dim, float scale, float* O_part, float* lse_part,
                            cudaStream_t stream);

/* hca_dense_attn — HCA main branch ([CS] "HCA": no selection, dense attention
 * over all heavily compressed entries): rows kv[b, 0 : n_vis(q_pos[b]+t)] with
 * compression ratio m (entries complete at the query position). */
csa_status_t hca_dense_attn(const void* q, csa_dtype_t q_dtype, const void* kv,
                            csa_dtype_t kv_dtype, const void* kv_rope, const float* kv_scale,
                            int64_t cap, const int64_t* q_pos, int m, int n_seq, int T, int H,
                            int D, int rope_dim, float scale, float* O_part, float* lse_part,
                            cudaStream_t stream);

/* swa_sink_combine — sliding window + attention sink + merge ([LD]: a
 * 128-token uncompressed window joins the attention; the sink lets a head
 * abstain; [CS] "HCA": an uncompressed 128-window is kept next to the
 * compressed branch).  For each query token:
 *   window rows  window_mode 0 (prefill): kv_tok[b, u] for u in [max(0,p-W+1), p]
 *                window_mode 1 (decode) : kv_tok[b, 0 : min(W, p+1)], a cache
 *                of the newest tokens in position order, newest included.
 *   out = (e^{lse_part-M} O_part + sum_w e^{l_w-M} v_w) /
 *         (e^{lse_part-M} + sum_w e^{l_w-M} + e^{sink_h-M})      (one softmax)
 *   then, if inv_rope, the last rope_dim dims of out are rotated by -p ([LD]:
 *   inverse RoPE on the output side).  O_part / lse_part may be NULL (no
 *   compressed branch).  kv_tok has dtype kv_dtype (BF16 or F32), [n_seq, cap, D].
 *   out [n_seq, T, H, D] out_dtype (F32 or BF16).
 * ------------------------------------------------------------------------- */
csa_status_t swa_sink_combine(const void* q, csa_dtype_t q_dtype, const void* kv_tok,
                              csa_dtype_t kv_dtype, int64_t cap, const int64_t* q_pos, int W,
                              int window_mode, const float* sink, const float* O_part,
                              const float* lse_part, int n_seq, int T, int H, int D,
                              int rope_dim, float rope_base, int inv_rope, float scale,
                              void* out, csa_dtype_t out_dtype, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_fused_attention — the attention side of a CSA or HCA layer in one
 * kernel: the compressed-branch rows (CSA: kv[b, idx[b,t,:]] as in
 * csa_sparse_mqa; HCA, idx == NULL: kv[b, 0 : n_vis] with ratio m as in
 * hca_dense_attn), the raw window rows (as in swa_sink_combine, from kv_tok
 * with tok_cap rows per sequence) and the sink share ONE softmax ([CS]
 * "共享 KV MQA" and "HCA"; [LD] SWA channel and attention sink), followed by
 * the optional inverse RoPE of the output.  Same result as csa_sparse_mqa /
 * hca_dense_attn followed by swa_sink_combine, without the fp32 partials.
 *   kv_tok dtype must be BF16 (F32 when kv is F32).  out [n_seq, T, H, D].
 * ------------------------------------------------------------------------- */
csa_status_t csa_fused_attention(const void* q, csa_dtype_t q_dtype, const void* kv, csa_dtype_t kv_dtype,
                                 const void* kv_rope, const float* kv_scale, int64_t cap,
                                 const int32_t* idx, int k, int m, const void* kv_tok,
                                 csa_dtype_t tok_dtype, int64_t tok_cap, int W, int window_mode,
                                 const int64_t* q_pos, const float* sink, int n_seq, int T, int H,
                                 int D, int rope_dim, float rope_base, int inv_rope, float scale,
                                 void* out, csa_dtype_t out_dtype, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_fused_attention_splitkv — csa_fused_attention with each query token's
 * row set split into n_split consecutive ranges of 64-row half chunks processed
 * in parallel (more CTAs when there are few query tokens, e.g. decode), followed
 * by a merge of the n_split partial results and the sink in one softmax and the
 * optional inverse RoPE.  Same result as csa_fused_attention up to rounding.
 * Every token's rows are cut into ranges of one common length: the longest
 * possible row set (k gathered or cap dense entries, plus the window) divided
 * by n_split, so a short token takes fewer, fuller ranges and its remaining
 * ranges are empty (lse -inf, output not written, skipped by the merge).  When
 * the (token, range) items outnumber the SMs, CTAs claim them from a counter in
 * the workspace, so ranges of sequences of unequal context balance across the
 * GPU; otherwise each CTA takes one item and the counter is not used.
 *   n_split in [1, 32]; workspace of csa_fused_attention_workspace(n_seq, T, H, D,
 *   n_split) bytes, 16-byte aligned, owned by the caller (partials: fp32
 *   [n_seq*T*n_split, H, D] + lse, then the item counter, reset by the call with a
 *   stream-ordered memset when it is used); calls sharing one workspace must be
 *   ordered on one stream.
 * ------------------------------------------------------------------------- */
size_t csa_fused_attention_workspace(int n_seq, int T, int H, int D, int n_split);

/* Workspace for one layer step whose indexer call (csa_index_topk with
 * n_seq, T, cap, k) and attention call (csa_fused_attention_splitkv with
 * n_seq, T, H, D, n_split; n_split <= 1 needs none) share one buffer in
 * stream order: the larger of the two sizes.  Pure host arithmetic. */
size_t csa_workspace_size(int n_seq, int T, int64_t cap, int k, int H, int D, int n_split);
csa_status_t csa_fused_attention_splitkv(const void* q, csa_dtype_t q_dtype, const void* kv, csa_dtype_t kv_dtype,
                                         const void* kv_rope, const float* kv_scale, int64_t cap,
                                         const int32_t* idx, int k, int m, const void* kv_tok,
                                         csa_dtype_t tok_dtype, int64_t tok_cap, int W, int window_mode,
                                         const int64_t* q_pos, const float* sink, int n_seq, int T, int H,
                                         int D, int rope_dim, float rope_base, int inv_rope, float scale,
                                         int n_split, void* workspace, size_t ws_bytes, void* out,
                                         csa_dtype_t out_dtype, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * csa_grouped_out_proj — grouped output projection of a layer's attention
 * output ([LQ] §3 config block: output_proj_groups 8, intermediate_attn_dim
 * 1024, hidden_size 4096).  The H heads form G groups of H/G consecutive heads;
 *   mid[t, g*d_mid + r] = sum_j w_grp[g, r, j] * o[t, g*H/G + j/D, j%D]
 *                         (j < (H/G)*D: the group's heads concatenated in order)
 *   out[t, c]           = sum_i w_out[c, i] * mid[t, i]        (i < G*d_mid)
 * No bias.  Weights are laid out [out_features, in_features].
 *   o      [M, H, D] BF16 (e.g. the output of csa_fused_attention).
 *   w_grp  [G, d_mid, (H/G)*D] BF16.   w_out [d_model, G*d_mid] BF16.
 *   mid    [M, G*d_mid] BF16, caller-owned; holds the rounded intermediate on
 *          return (fp32 accumulation, one bf16 rounding).
 *   out    [M, d_model], out_dtype F32 or BF16 (fp32 accumulation).
 * Two launches on `stream` (group stage, output stage).  (H/G)*D must be a
 * multiple of 64, d_mid and d_model multiples of 256 (else
 * CSA_ERR_UNSUPPORTED); M = 0 is a no-op (pointers may then be NULL).
 * ------------------------------------------------------------------------- */
csa_status_t csa_grouped_out_proj(const void* o, const void* w_grp, const void* w_out, int M, int H, int D,
                                  int G, int d_mid, int d_model, void* mid, void* out, csa_dtype_t out_dtype,
                                  cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H_ */
