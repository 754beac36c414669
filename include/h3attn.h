/*
 * h3attn.h -- C ABI of the h3attn library: the attention hot path of a joint
 * video/audio diffusion transformer block (MiniMax-H3), written for one NVIDIA
 * B200 (sm_100a).
 *
 * The path: per-head Q/K RMSNorm + rotary position embedding (one prologue
 * kernel), then non-causal softmax(Q K^T * scale) V over a packed token
 * sequence (one attention kernel, dense or ragged).  Around it: attention
 * against a separate key block and the log-sum-exp merge of such partial
 * results (key-split schedules), block-sparse attention over given lists of key
 * tiles, the Q/K/V projection with the prologue fused into its epilogue, and a
 * self-test of the kernels' bounded waits.
 *
 * Sources of the operations (web pages about the H3 runtimes):
 *   - "H3 Runtime Current State", Owned Performance Kernels: a fused Q/K
 *     RMSNorm, RoPE and layout kernel is listed as missing; Implemented And
 *     Validated: "H3 packed denoising" (video and audio tokens in one
 *     sequence) and "Ragged Ulysses sequence parallelism" (ragged sequences).
 *   - "Buyer Questions: Current Evidence Status", block composition answer: in the profiled
 *     DiT block, attention is the largest share of time and norm/RoPE feeds it;
 *     strided-NHD Q/K/V (no copy of the QKV projection output) was a measured
 *     saving.
 *   - "Open-H3-Regenerate-2K", Forward table: the standard forward runs dense
 *     attention on one B200.
 *
 * Conventions shared by every call
 *   - Tensors are bfloat16, token-major "NHD": element (token n, head h, dim i)
 *     lives at base + n*tok_stride + h*head_stride + i (strides in elements, the
 *     last dimension contiguous).  Strided views of one fused QKV buffer are
 *     accepted as they are: no copy is made.
 *   - Every device pointer and every stride must be a multiple of 16 bytes
 *     (strides: multiples of 8 elements); otherwise H3ATTN_ERR_MISALIGNED.
 *   - The caller owns every buffer.  The library allocates and frees no device
 *     memory; it holds two small static device words for error reporting (the
 *     error word and the copy h3attn_device_status reads it through).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) of the current device and runs asynchronously: no call
 *     synchronises the device.  All argument checks happen on the host before
 *     anything is enqueued; a failed check enqueues nothing.
 *   - Device-side waits are bounded: a kernel that waits longer than about one
 *     second on an internal barrier stops, records the failure in the device
 *     error word and returns without writing its remaining outputs.
 *     h3attn_device_status() reads that word.
 *   - Calls with distinct output buffers may run concurrently.
 */
#ifndef H3ATTN_H
#define H3ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    H3ATTN_OK = 0,
    H3ATTN_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, bad section split, ... */
    H3ATTN_ERR_UNSUPPORTED = 2,    /* head_dim not in {64, 128}, sizes beyond the kernel limits */
    H3ATTN_ERR_MISALIGNED = 3,     /* pointer or stride not a multiple of 16 bytes */
    H3ATTN_ERR_CUDA = 4,           /* a CUDA runtime/driver call failed (see h3attn_last_error) */
    H3ATTN_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up on a bounded internal wait */
} h3attn_status;

/* Library version as 10000*major + 100*minor + patch. */
int h3attn_version(void);

/*
 * Build flags of the loaded library: H3ATTN_BUILD_DEBUG_BOUNDS is set in the
 * debug build (compiled with H3ATTN_DEBUG_BOUNDS), where every kernel checks
 * each global store's indices against its own launch's extents and, instead of
 * storing out of place, records the failure for h3attn_device_status (which
 * then returns H3ATTN_ERR_INVALID_ARG).  Release builds compile those checks
 * away.  The checks stand in for a memory checker where none can run.
 */
#define H3ATTN_BUILD_DEBUG_BOUNDS 1
int h3attn_build_flags(void);

/* Static text for a status code (never NULL). */
const char* h3attn_status_string(int status);

/* Human-readable detail of the last failure on the calling host thread, or "". */
const char* h3attn_last_error(void);

/*
 * Reads the device error word of the current device once the work already on
 * `stream` has finished, then synchronises `stream`: H3ATTN_OK;
 * H3ATTN_ERR_INVALID_ARG if a ragged launch's cu_seqlens or a block-sparse key
 * list broke its rules (h3attn_fwd_varlen, h3attn_fwd_block_sparse), or, in a
 * debug build, a bounds check fired;
 * H3ATTN_ERR_DEVICE_TIMEOUT if any kernel of this library gave up on a bounded
 * wait since the word was last cleared; H3ATTN_ERR_CUDA if the stream reports
 * an error.  The word is read and (clear != 0) zeroed by one atomic exchange
 * on the device, enqueued on `stream`: an error that work on another stream
 * records meanwhile is not lost but stays for the next call.
 */
int h3attn_device_status(void* stream, int clear);

/*
 * h3attn_selftest_wait_timeout -- failure-detection self-test of the bounded
 * waits every kernel uses.  Enqueues one small kernel that waits on a barrier
 * nothing will ever complete, with the same bounded wait as the production
 * kernels: after about one second the wait gives up, records a timeout in the
 * device error word and the kernel returns (no trap, no fault; the context
 * stays usable).  The next h3attn_device_status() on `stream` must return
 * H3ATTN_ERR_DEVICE_TIMEOUT.  Returns H3ATTN_ERR_CUDA if the launch fails.
 */
h3attn_status h3attn_selftest_wait_timeout(void* stream);

/*
 * h3attn_prologue -- per-head RMSNorm of Q and K followed by rotary position
 * embedding, rounded once to bfloat16.
 *
 * Source: "H3 Runtime Current State", Owned Performance Kernels (fused Q/K
 * RMSNorm and RoPE listed as missing); "Buyer Questions: Current Evidence
 * Status", block composition answer (norm/RoPE between the projection and
 * attention).  The pages give no formula: the textbook RMSNorm and the
 * interleaved-pair rotary form are used, with the 3D split of the task's
 * workloads.
 *
 * For every token n < n_tokens and head h < n_heads, on the row x of length
 * head_dim (Q and K alike, each with its own gamma):
 *   RMSNorm (skipped when that tensor's gamma is NULL):
 *       x_i <- x_i / sqrt(mean_j(x_j^2) + eps) * gamma_i
 *   RoPE (skipped when pos is NULL, or for tokens with kind[n] == 0):
 *       pair (x_{2i}, x_{2i+1}) rotated by angle a_i:
 *         y_{2i} = x_{2i} cos a_i - x_{2i+1} sin a_i,
 *         y_{2i+1} = x_{2i} sin a_i + x_{2i+1} cos a_i
 *       kind 1 (video, 3D): dims [0, sec_t) use pos[n][0] (t), [sec_t, sec_t+sec_h)
 *         use pos[n][1] (h), the rest use pos[n][2] (w); inside a section of
 *         width ds the i-th pair has a_i = p * theta^(-2i/ds).
 *       kind 2 (audio or ragged, 1D): a_i = pos[n][0] * theta^(-2i/head_dim).
 *   The result is rounded to the nearest bfloat16 once.
 *
 * q_in, k_in:   bf16 input rows, strides in_tok_stride / in_head_stride.
 * q_out, k_out: bf16 output rows, strides out_tok_stride / out_head_stride.
 *               In place is allowed (q_out == q_in with equal strides); other
 *               overlaps between inputs and outputs are not.
 * gamma_q, gamma_k: bf16 [head_dim] or NULL.     eps: added inside the sqrt.
 * pos:   device int32 [n_tokens][3] or NULL;  kind: device uint8 [n_tokens]
 *        (required when pos is given; values other than 0, 1, 2 act as 0).
 * sec_t + sec_h + sec_w must equal head_dim, each even (checked only when pos
 * is given).  head_dim: 64 or 128.  n_tokens == 0 is a no-op.
 * Arithmetic: sum of squares and scaling in fp32; angles and their sine and
 * cosine in fp64, each carried as a pair of floats (head + tail), and the
 * rotation in fp32 with error-free products, so every output is within one
 * bf16 ulp of the exactly rounded result.
 */
h3attn_status h3attn_prologue(const void* q_in, const void* k_in, void* q_out, void* k_out,
                              int64_t n_tokens, int32_t n_heads, int32_t head_dim,
                              int64_t in_tok_stride, int64_t in_head_stride,
                              int64_t out_tok_stride, int64_t out_head_stride,
                              const void* gamma_q, const void* gamma_k, double eps,
                              const int32_t* pos, const uint8_t* kind,
                              int32_t sec_t, int32_t sec_h, int32_t sec_w, double theta,
                              void* stream);

/*
 * h3attn_fwd -- dense non-causal attention over `batch` sequences of equal
 * length seqlen:  O = softmax(Q K^T * scale) V  per (sequence, head).
 *
 * Source: "Open-H3-Regenerate-2K", Forward table (the standard forward runs
 * dense attention on one B200); "Buyer Questions: Current Evidence Status",
 * block composition answer (attention is the largest share of the block).
 * Video and audio tokens of one clip form one sequence with no mask ("H3
 * Runtime Current State", Implemented And Validated: packed denoising).
 *
 * q, k, v, o: bf16 [batch][seqlen][n_heads][head_dim]; each has strides
 *   {batch, token, head} in elements (x_strides[0..2]), last dim contiguous.
 * softmax_scale <= 0 selects 1/sqrt(head_dim).
 * lse: NULL, or fp32 [batch][n_heads][seqlen] receiving the natural-log
 *   log-sum-exp of each row's scaled scores.
 * head_dim: 64 or 128; seqlen >= 1 (any value, no multiple of 128 needed);
 * n_heads >= 1; batch >= 1.  Rows of `o` outside the tensor are never written.
 * Arithmetic: bf16 tensor-core products with fp32 accumulation; softmax in
 * fp32 with exp2; P rounded to bf16 for the PV product; O rounded to bf16.
 */
h3attn_status h3attn_fwd(const void* q, const void* k, const void* v, void* o,
                         int32_t batch, int64_t seqlen, int32_t n_heads, int32_t head_dim,
                         const int64_t q_strides[3], const int64_t k_strides[3],
                         const int64_t v_strides[3], const int64_t o_strides[3],
                         float softmax_scale, float* lse, void* stream);

/*
 * h3attn_fwd_varlen -- the same attention over nseq ragged sequences packed
 * along the token dimension: sequence s owns tokens [cu_seqlens[s],
 * cu_seqlens[s+1]) and attends only to its own keys.
 *
 * Source: "H3 Runtime Current State", Implemented And Validated ("Ragged
 * Ulysses sequence parallelism": sequences of unequal length packed together).
 * The kernel takes the sequences longest first (cost grows with the square of
 * the length).
 *
 * q, k, v, o: bf16 [total_tokens][n_heads][head_dim], strides {token, head}.
 * cu_seqlens: DEVICE int32 [nseq + 1] with cu_seqlens[0] = 0, non-decreasing,
 *   no sequence longer than max_seqlen, cu_seqlens[nseq] = total_tokens; empty
 *   sequences are allowed and produce nothing.  It is device memory, so the
 *   host does not read it: the kernel checks these rules before it uses any
 *   bound, and a descriptor that breaks one makes the launch write nothing and
 *   the next h3attn_device_status() return H3ATTN_ERR_INVALID_ARG.
 * max_seqlen: host value >= every sequence length; it caps the launch's grid
 *   at nseq * ceil(max_seqlen / 256) query-tile pairs per head.
 * lse: NULL, or fp32 [n_heads][total_tokens].
 * nseq <= 65535.  Other rules as h3attn_fwd.
 */
h3attn_status h3attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                                const int32_t* cu_seqlens, int32_t nseq, int64_t total_tokens,
                                int32_t max_seqlen, int32_t n_heads, int32_t head_dim,
                                const int64_t q_strides[2], const int64_t k_strides[2],
                                const int64_t v_strides[2], const int64_t o_strides[2],
                                float softmax_scale, float* lse, void* stream);

/*
 * Partial attention and its combination: the pieces of a key-split schedule.
 *
 * Sequence-parallel execution of the block ("H3 Runtime Current State",
 * Implemented And Validated: ragged Ulysses sequence parallelism and
 * sequence-sharded block execution) can also split the KEYS of a sequence
 * across steps or ranks.  For the same query rows, each key block gives a
 * partial result (O_p, LSE_p): O_p the softmax-weighted mean of the block's
 * values, LSE_p the natural log of the block's total weight sum_j exp(s_j).
 * Combining all blocks by their LSE gives exactly the attention over all keys,
 * up to rounding.
 */

/*
 * h3attn_fwd_kv -- h3attn_fwd with the key/value length separate from the query
 * length: each of the seqlen_q query rows of a sequence attends to the
 * seqlen_kv key/value rows of the same batch entry.
 *
 * q, o: bf16 [batch][seqlen_q][n_heads][head_dim];  k, v: bf16
 *   [batch][seqlen_kv][n_heads][head_dim]; strides {batch, token, head}.
 * seqlen_q >= 1.  seqlen_kv >= 0: with no keys the result is the empty sum,
 *   O = 0 and LSE = -inf (k and v are not read and may be NULL).
 * lse: NULL, or fp32 [batch][n_heads][seqlen_q].  Other rules as h3attn_fwd,
 * which is this call with seqlen_kv = seqlen_q.
 */
h3attn_status h3attn_fwd_kv(const void* q, const void* k, const void* v, void* o, int32_t batch,
                            int64_t seqlen_q, int64_t seqlen_kv, int32_t n_heads, int32_t head_dim,
                            const int64_t q_strides[3], const int64_t k_strides[3],
                            const int64_t v_strides[3], const int64_t o_strides[3],
                            float softmax_scale, float* lse, void* stream);

/*
 * h3attn_fwd_block_sparse -- h3attn_fwd_kv in which each group of 256 query rows
 * attends only to listed blocks of 128 keys.
 *
 * The refine-stage timing table of "Open-H3-Regenerate-2K" gains its largest
 * step from a sparse attention backend ("+ Sol-Attn sparse attention"), and "H3
 * Runtime Current State" (Next Work) keeps such backends quality-gated; the pages
 * give no rule for choosing the blocks.  This call executes a given pattern: the
 * choice of blocks is the caller's.
 *
 * Query rows of a sequence form pairs of 128-row tiles, QP = ceil(seqlen_q / 256)
 * of them; keys form tiles of 128, KT = ceil(seqlen_kv / 128) of them.  List
 *   c = (b * n_heads + h) * QP + qp
 * is blk_idx[blk_off[c] .. blk_off[c + 1]): the key tiles that query rows
 * [256 qp, 256 qp + 256) of batch entry b, head h see.  Each row attends exactly
 * to the keys of its listed tiles (the last tile holds seqlen_kv - 128 (KT - 1)
 * keys); arithmetic and rounding are those of h3attn_fwd on that key set; an
 * empty list is the empty sum, O = 0 and LSE = -inf.
 *
 * blk_off: DEVICE int32 [batch * n_heads * QP + 1], non-decreasing, blk_off[0] = 0.
 * blk_idx: DEVICE int32, each list strictly ascending with entries in [0, KT).
 *   Both 4-byte aligned; neither is read on the host.  A list whose entries break
 *   these rules is detected by the kernel: the query rows it serves are not
 *   written, every other list is processed, and the next h3attn_device_status()
 *   returns H3ATTN_ERR_INVALID_ARG.  The offsets themselves are trusted: blk_off
 *   must have the stated length and its entries must lie in [0, entries of blk_idx].
 * Other arguments, layouts and rules as h3attn_fwd_kv.
 */
h3attn_status h3attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, int32_t batch,
                                      int64_t seqlen_q, int64_t seqlen_kv, int32_t n_heads, int32_t head_dim,
                                      const int64_t q_strides[3], const int64_t k_strides[3],
                                      const int64_t v_strides[3], const int64_t o_strides[3],
                                      const int32_t* blk_off, const int32_t* blk_idx, float softmax_scale,
                                      float* lse, void* stream);

/*
 * h3attn_merge -- combine two partial results of the same query rows over
 * disjoint key sets:
 *   L = log(exp(lse_a) + exp(lse_b))  (formed as M + log(sum exp(lse_p - M)),
 *                                      M = max(lse_a, lse_b)),
 *   O = exp(lse_a - L) * O_a + exp(lse_b - L) * O_b.
 * A part with lse = -inf is empty and has no weight (its O values must still be
 * finite, as h3attn_fwd_kv writes them); two empty parts give O = 0, L = -inf.
 *
 * o_a, o_b, o: bf16 [batch][seqlen][n_heads][head_dim], strides {batch, token,
 *   head}.  lse_a, lse_b, lse: fp32 [batch][n_heads][seqlen], contiguous.
 * In place is allowed: o == o_a (same strides) with lse == lse_a, or likewise
 *   with the b part; other overlaps are not.
 * Arithmetic: weights in fp32 (expf, logf), O = fma(w_a, O_a, w_b * O_b) in
 *   fp32, rounded once to bf16.
 * seqlen == 0 is a no-op.  Alignment rules as every call; head_dim 64 or 128.
 */
h3attn_status h3attn_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                           void* o, float* lse, int32_t batch, int64_t seqlen, int32_t n_heads,
                           int32_t head_dim, const int64_t oa_strides[3], const int64_t ob_strides[3],
                           const int64_t o_strides[3], void* stream);

/*
 * h3attn_qkv_fused -- the block's Q/K/V projection with the prologue fused into
 * it: Q', K', V straight from the token activations.
 *
 * "H3 Runtime Current State", Owned Performance Kernels, lists fused Q/K
 * RMSNorm, RoPE and layout work as missing; "Buyer Questions: Current Evidence
 * Status" (block composition) has the projection feed norm/RoPE, with its
 * strided NHD output read in place.  For token n and output feature
 *   f = sum_c x[n][c] * w[f][c] (+ bias[f]),   f in [0, 3*n_heads*head_dim):
 * features [0, H*d) are Q (head f / d), [H*d, 2*H*d) K, [2*H*d, 3*H*d) V.  Each
 * (token, head) row of Q and of K then goes through RMSNorm (gamma_q / gamma_k;
 * skipped where NULL) and RoPE (pos/kind/sections/theta exactly as
 * h3attn_prologue; skipped where pos is NULL); V is the projection.  Every
 * output is rounded once to bf16: the projection is not rounded before the norm.
 *
 * x:     bf16 [n_tokens][dim_in], token stride x_tok_stride (elements).
 * w:     bf16 [3*n_heads*head_dim][dim_in], contiguous (the layout of a linear
 *        layer's weight: one row per output feature).
 * bias:  bf16 [3*n_heads*head_dim] or NULL.
 * q_out, k_out, v_out: bf16 NHD outputs, strides {out_tok_strides[i],
 *        out_head_strides[i]} for i = 0 (Q), 1 (K), 2 (V) -- three views of one
 *        fused buffer work as they are.
 * gamma_q, gamma_k: bf16 [head_dim] or NULL.  eps: inside the square root.
 * pos, kind, sec_*, theta: as h3attn_prologue.
 * Requirements: head_dim 64 or 128; n_heads*head_dim a multiple of 256;
 *   dim_in a positive multiple of 64; n_tokens >= 0 (0 is a no-op).
 * Arithmetic: bf16 tensor-core products with fp32 accumulation; bias, sum of
 *   squares, 1/rms (rsqrtf) and the gamma scale in fp32; RoPE angles formed and
 *   reduced to [-pi, pi] in fp32 with error-free products (frequencies and 2 pi
 *   carried as float pairs), cos/sin and the rotation in fp32: about 1e-6
 *   absolute on cos/sin, far below the accumulation error of the projection.
 */
h3attn_status h3attn_qkv_fused(const void* x, const void* w, const void* bias, void* q_out, void* k_out,
                               void* v_out, int64_t n_tokens, int32_t dim_in, int32_t n_heads,
                               int32_t head_dim, int64_t x_tok_stride, const int64_t out_tok_strides[3],
                               const int64_t out_head_strides[3], const void* gamma_q, const void* gamma_k,
                               double eps, const int32_t* pos, const uint8_t* kind, int32_t sec_t,
                               int32_t sec_h, int32_t sec_w, double theta, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* H3ATTN_H */
