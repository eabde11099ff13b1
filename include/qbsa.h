/*
 * qbsa.h -- C ABI of the B200 (sm_100a) fused attention forward library (libqbsa.so).
 *
 * Sources, cited by page title and section:
 *   [NFA] npu_fusion_attention guide, "昇腾 NPU 融合注意力算子详解与迁移指南":
 *         §2 算子数学原理 (formula), §3 函数原型 (signature), §4.1-§4.3 (parameters),
 *         §5 输出说明 (outputs), §7 (constraints: GQA, head dim).
 *   [QBSA] EagleQBSA article, "昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,视频生成端到端加速1.6倍":
 *         section "EagleQBSA量化叠加稀疏方案设计" (Fig 2.1, quantisation scheme),
 *         section "MindIE SD调用方式" (operator call and its arguments).
 *
 * Conventions for every entry point:
 *   - The caller owns all memory.  Device pointers must be 16-byte aligned and stay
 *     valid until the work queued on `stream` has finished; the library never frees
 *     or retains them.  Only qbsa_quantize_v takes scratch memory of its own, from
 *     the stream-ordered allocator on `stream` (see there); no other entry point
 *     allocates device memory.
 *   - Work is queued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Argument checks run on the host before anything is queued: a
 *     non-OK status means nothing was launched.
 *   - QBSA_ERR_CUDA reports a launch or driver error.  A device-side wait that ran
 *     out of time (the kernels bound every wait) is reported by qbsa_check().
 *   - qbsa_last_error() returns a thread-local message for the last non-OK status.
 *   - Every kernel of the library issues plain (non-multicast) TMA loads only.
 */
#ifndef QBSA_H_
#define QBSA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QBSA_OK = 0,
  QBSA_ERR_INVALID = 1,      /* an argument is out of its documented domain */
  QBSA_ERR_UNSUPPORTED = 2,  /* a valid request this build does not implement */
  QBSA_ERR_CUDA = 3,         /* CUDA launch / driver error */
  QBSA_ERR_TIMEOUT = 4       /* a kernel's bounded wait expired (from qbsa_check) */
} qbsa_status;

typedef enum { QBSA_LAYOUT_BNSD = 0, QBSA_LAYOUT_BSND = 1, QBSA_LAYOUT_TND = 2 } qbsa_layout;

typedef enum {
  QBSA_MASK_NONE = 0, /* no explicit mask */
  QBSA_MASK_SS = 1,   /* [Sq, Skv], shared by all batches and heads */
  QBSA_MASK_B1SS = 2, /* [B, 1, Sq, Skv], shared by the heads of a batch */
  QBSA_MASK_BNSS = 3  /* [B, Nq, Sq, Skv] */
} qbsa_mask_shape;

/*
 * attn_fwd -- dense fused attention forward, [NFA] §2:
 *     attention_out = Softmax(Mask(Q·Kᵀ·scale + pse))·V      (keep_prob = 1: no dropout)
 * computed tile by tile with an online softmax; the score matrix is never stored.
 *
 * q, k, v        bf16 device tensors, contiguous in `input_layout` ([NFA] §4.1):
 *                  BNSD: q [B, Nq, Sq, D], k/v [B, Nkv, Skv, D]
 *                  BSND: q [B, Sq, Nq, D], k/v [B, Skv, Nkv, D]
 *                  TND : q [Sq, Nq, D],    k/v [Skv, Nkv, D]  (Sq, Skv = total tokens,
 *                        B = number of sequences)
 * Nq, Nkv        query / key-value heads; Nq % Nkv == 0 (GQA, [NFA] §7); query head
 *                h reads key/value head h / (Nq / Nkv).  head_num must equal Nq.
 * D              head dim of q, k and v (D_q = D_k = D_v); 64 or 128 in this build
 *                (other values of [NFA] §7's range return QBSA_ERR_UNSUPPORTED).
 * atten_mask     uint8 device tensor, 1 = masked, 0 = kept ([NFA] §4.2), shaped by
 *                mask_shape; used only with sparse_mode 0; NULL with QBSA_MASK_NONE.
 *                Not supported with TND.
 * pse            bf16 device tensor [B, Nq, Sq, Skv] (or [1, Nq, Sq, Skv] when
 *                pse_batch_bcast != 0), added after the scale; NULL for none.  BNSD /
 *                BSND only.
 * scale          the softmax scale ([NFA] §4.2), finite.
 * keep_prob      must be 1.0 (dropout is not implemented: QBSA_ERR_UNSUPPORTED).
 * sparse_mode    ([NFA] §4.3) 0: keep (i, j) with i - pre_tokens <= j <= i + next_tokens
 *                (0-based, top-left aligned), combined with atten_mask; 2: causal with
 *                the top-left vertex, j <= i; 3: causal with the bottom-right vertex,
 *                j <= i + (Skv - Sq), per sequence for TND.  Modes 2 and 3 ignore
 *                pre_tokens, next_tokens and atten_mask.  Other modes: UNSUPPORTED.
 * pre_tokens,
 * next_tokens    band of mode 0; 2147483647 (the [NFA] §3 default) means unbounded.
 * actual_seq_qlen,
 * actual_seq_kvlen  HOST arrays of B int64 cumulative end offsets without a leading
 *                0 ([NFA] §4.3: 累加长度); sequence b covers [cum[b-1], cum[b]).  The last
 *                entries must equal Sq and Skv.  TND only (NULL otherwise); B <= 128.
 * attention_out  bf16 device tensor, same layout and shape as q ([NFA] §5 item 1).
 * softmax_max,
 * softmax_sum    optional fp32 device tensors ([NFA] §5 items 2-3): per query row the
 *                max of the masked scores (natural-log domain) and Σ_j exp(S_ij - max).
 *                Layout [B, Nq, Sq] (BNSD/BSND) or [Nq, Sq] (TND).  A row with no kept
 *                key gets out = 0, max = -inf, sum = 0.  NULL skips the output.
 * stream         cudaStream_t.
 */
qbsa_status attn_fwd(const void* q, const void* k, const void* v, int B, int Nq, int Nkv, int Sq, int Skv, int D,
                     int head_num, qbsa_layout input_layout, const uint8_t* atten_mask, qbsa_mask_shape mask_shape,
                     const void* pse, int pse_batch_bcast, float scale, float keep_prob, int sparse_mode,
                     int64_t pre_tokens, int64_t next_tokens, const int64_t* actual_seq_qlen,
                     const int64_t* actual_seq_kvlen, void* attention_out, float* softmax_max, float* softmax_sum,
                     void* stream);

/*
 * bsa_fwd -- bf16 block-sparse attention: attn_fwd (BNSD, sparse_mode 0, no atten_mask,
 * no pse) computed only over the 128x128 blocks kept by block_mask.  This is the BF16
 * block-sparse baseline ("BSA") that [QBSA] "EagleQBSA单算子性能验证分析" compares the
 * quantized operator with, on the same block mask.
 *
 * q, k, v        bf16 BNSD device tensors as in attn_fwd.
 * block_mask     uint8 [B, Nq, ceil(Sq/128), ceil(Skv/128)], 1 = compute the block;
 *                ceil(Skv/128) <= 2048.  Keys of blocks not kept are masked; a row with
 *                no kept block gets out = 0, max = -inf, sum = 0.
 * Other arguments and outputs as in attn_fwd.
 */
qbsa_status bsa_fwd(const void* q, const void* k, const void* v, const uint8_t* block_mask, int B, int Nq, int Nkv,
                    int Sq, int Skv, int D, float scale, void* attention_out, float* softmax_max, float* softmax_sum,
                    void* stream);

/*
 * qbsa_fwd -- quantized block-sparse attention forward, [QBSA] "MindIE SD调用方式" and
 * "EagleQBSA量化叠加稀疏方案设计": INT8 Q·Kᵀ with per-128-token-block scales, online
 * softmax, P rounded to FP8 E4M3 (nearest even), FP8 P·V with per-channel V scales,
 * bf16 output, computed only for the 128x128 blocks the block mask keeps.
 *
 * q_i8           int8 [B, Nq, Sq, D] (BNSD)
 * k_i8           int8 [B, Nkv, Skv, D]
 * q_block_scale  fp32 [B, Nq, ceil(Sq/128)]      x ≈ q_i8 * scale of its 128-row block
 * k_block_scale  fp32 [B, Nkv, ceil(Skv/128)]
 * v_fp8          E4M3 bytes [B, Nkv, Skv, D]
 * v_channel_scale fp32 [B, Nkv, D]               v ≈ e4m3(v_fp8) * scale of its channel
 * block_mask     uint8 [B, Nq, ceil(Sq/128), ceil(Skv/128)], 1 = compute the block
 * D              128 (other values: QBSA_ERR_UNSUPPORTED); ceil(Skv/128) <= 2048.
 * scale          softmax scale (scale_value in [QBSA]'s call, 128^-0.5 there).
 * Score s = int_dot(q_i8, k_i8) * q_scale * k_scale * scale, z = s * log2(e).  Kept
 * key blocks are visited in ascending order, one 128-key block per step, and the
 * running max m = max z is updated at every block.  The weights are taken against a
 * power-of-two reference R (an integer, log2 units): R = ceil(m) at the first kept
 * block, and again whenever m exceeds R + 8, at which point the accumulated row sum
 * and output are multiplied by the exact power of two 2^(R_old - R_new).  Each weight
 * is held in FP16 and then rounded to E4M3: p8 = E4M3(FP16(2^(z - R))), both
 * round-to-nearest-even, E4M3 saturating ([QBSA] "昇腾亲和的量化叠加稀疏Attention算子优化":
 * the FP16 P matrix is converted to FP8).  2^(z - R) <= 2^8, below E4M3's 448.  The
 * row sum L is the sum of the rounded weights; out[:, c] = (Σ p8 v8)[c] / L * v_scale[c].
 * These codes equal those taken against the plain running max e^(s - m) up to one
 * E4M3 rounding on a shifted grid.  attention_out bf16 [B, Nq, Sq, D]; softmax_max /
 * softmax_sum optional fp32 [B, Nq, Sq]: the natural-log row max and L * 2^(R - m),
 * the rounded weights' sum against that max.  A row with no kept block gets out = 0,
 * max = -inf, sum = 0.
 */
qbsa_status qbsa_fwd(const int8_t* q_i8, const int8_t* k_i8, const float* q_block_scale, const float* k_block_scale,
                     const uint8_t* v_fp8, const float* v_channel_scale, const uint8_t* block_mask, int B, int Nq,
                     int Nkv, int Sq, int Skv, int D, float scale, void* attention_out, float* softmax_max,
                     float* softmax_sum, void* stream);

/*
 * qbsa_fwd_host -- qbsa_fwd on HOST buffers: the same operation, arguments, layouts and
 * outputs, but every data pointer (inputs, attention_out, the optional softmax_max /
 * softmax_sum) is host memory.  Page-locked memory lets the copies overlap the kernel;
 * pageable memory works, with the copies staged by the driver.
 * The work is split into about n_chunks independent (batch, kv-head range) chunks (n_chunks
 * >= 1; a chunk holds whole GQA groups).  Chunk c + 1's inputs are copied to the device on
 * one library-owned stream while chunk c runs on `stream` and chunk c - 1's outputs return
 * on another, ordered by events.  Device buffers come from a stream-ordered memory pool the
 * library keeps per device (its memory is kept for later calls, never freed before the
 * process exits).  The call returns after the results are in host memory; the host buffers
 * must not be touched by other threads during the call.  Errors as qbsa_fwd, plus
 * QBSA_ERR_INVALID for n_chunks < 1; a CUDA error during the copies returns QBSA_ERR_CUDA
 * (the outputs are then unspecified).
 */
qbsa_status qbsa_fwd_host(const int8_t* q_i8, const int8_t* k_i8, const float* q_block_scale,
                          const float* k_block_scale, const uint8_t* v_fp8, const float* v_channel_scale,
                          const uint8_t* block_mask, int B, int Nq, int Nkv, int Sq, int Skv, int D, float scale,
                          void* attention_out, float* softmax_max, float* softmax_sum, int n_chunks, void* stream);

/*
 * qbsa_quantize_qk -- per-128-token-block symmetric INT8 quantisation of Q or K
 * ([QBSA] "EagleQBSA量化叠加稀疏方案设计"): for each (b, h, block) a = max|x| (fp32),
 * s = a/127 (1 if a = 0), codes = rint_half_even(x/s) clamped to [-127, 127].
 * x bf16 [B, N, S, D] (BNSD); codes int8 [B, N, S, D]; scales fp32 [B, N, ceil(S/128)].
 * D in {64, 128, 256} (else QBSA_ERR_UNSUPPORTED); x and codes 16-byte aligned.
 */
qbsa_status qbsa_quantize_qk(const void* x_bf16, int B, int N, int S, int D, int8_t* codes, float* scales,
                             void* stream);

/*
 * qbsa_quantize_v -- per-channel FP8 E4M3 quantisation of V ([QBSA] same section):
 * for each (b, h, channel c) a = max over the sequence of |v[:, c]|, s_c = a/448 (1 if
 * a = 0), codes = e4m3_rne_satfinite(v / s_c).  v bf16 [B, N, S, D]; codes [B, N, S, D];
 * scales fp32 [B, N, D].  D in {64, 128, 256} (else QBSA_ERR_UNSUPPORTED); v, codes and
 * scales 16-byte aligned.
 * Two streaming passes: the column maxima of every (head, chunk), folded per head, then
 * the codes.  They need B*N*D * 4 bytes of scratch for the per-head maxima, which this call
 * takes, stream-ordered on `stream`, from a memory pool the library keeps per device
 * (created on first use; it keeps its memory between calls, so after the first call of a
 * size no allocation maps memory) and zeroes; an allocation failure returns QBSA_ERR_CUDA
 * before the kernels are queued.
 */
qbsa_status qbsa_quantize_v(const void* v_bf16, int B, int N, int S, int D, uint8_t* codes, float* scales,
                            void* stream);

/*
 * qbsa_quantize_v_noalloc -- qbsa_quantize_v for callers that cannot allocate device
 * memory during the call.  The source pages have no counterpart: this entry point exists
 * for callers such as code running inside a custom allocator or a memory-pool callback,
 * serving processes that reserve every byte of the device heap up front, and runtimes
 * that forbid cudaMalloc / cudaMallocAsync on their streams.  It produces the same codes
 * and scales as qbsa_quantize_v (same arguments, layouts and errors) and allocates
 * nothing: its scratch (the per-head column maxima: B*N*D 32-bit words) lives in a fixed
 * 256 KiB array in the library's device image, which every device that loads the library
 * holds until the process exits.
 *   - B*N*D above 65536 words (for D = 128: B*N above 512) returns QBSA_ERR_UNSUPPORTED
 *     before anything is queued.
 *   - The first call on a device looks up the array's device address for that device
 *     (cudaGetSymbolAddress) and keeps it; make that first call before any stream capture.
 *   - Every call zeroes the array with cudaMemsetAsync on `stream` and then reuses it, so
 *     calls whose work overlaps on the GPU (other streams, other host threads) race on the
 *     shared array: serialise them.
 */
qbsa_status qbsa_quantize_v_noalloc(const void* v_bf16, int B, int N, int S, int D, uint8_t* codes, float* scales,
                                    void* stream);

/*
 * attn_tile_schedule -- host-only export of the K-tile schedule attn_fwd's kernel uses
 * for one sequence under sparse_mode / pre_tokens / next_tokens ([NFA] §4.3): for each
 * 128-row query tile t < n_qtiles (= ceil(sq/128)), the K tiles [kt_begin[t],
 * kt_end[t]) are visited and those in [full_begin[t], full_end[t]) need no element
 * mask.  Output arrays are host memory of n_qtiles entries.  No GPU is used.
 */
qbsa_status attn_tile_schedule(int64_t sq, int64_t skv, int sparse_mode, int64_t pre_tokens, int64_t next_tokens,
                               int32_t* kt_begin, int32_t* kt_end, int32_t* full_begin, int32_t* full_end,
                               int64_t n_qtiles);

/*
 * qbsa_block_lists -- runs qbsa_fwd's in-kernel compaction of block-mask rows on the
 * GPU: for each of `rows` rows of n_kb bytes, lists[r, 0:count) = indices of non-zero
 * bytes in ascending order (-1 after), counts[r] = count.  Device pointers.  n_kb <= 2048.
 */
qbsa_status qbsa_block_lists(const uint8_t* block_mask, int64_t rows, int n_kb, int32_t* lists, int32_t* counts,
                             void* stream);

/*
 * qbsa_block_mean -- first step of block-mask estimation: the mean row of every 128-token
 * block.  The EagleQBSA article ([QBSA] 背景介绍) builds on block-sparse attention that
 * computes only the 128x128 blocks a block mask selects (block_sparse_mask, block_shape
 * [128, 128] in [QBSA] MindIE SD调用方式) but does not say how the mask is chosen; this
 * library's reading pools each block to its mean row, scores block pairs by the pooled dot
 * product and keeps the top blocks (qbsa_block_topk).
 *   x       bf16 [B, N, S, D] contiguous (BNSD), device, 16-byte aligned; D in {64, 128, 256}.
 *   x_mean  fp32 [B, N, ceil(S/128), D], device, caller-owned output: the mean over the
 *           block's rows that lie inside S (a tail block averages fewer rows), summed in fp32.
 * Asynchronous on `stream`.  QBSA_ERR_INVALID for null pointers, S < 1 or misalignment,
 * QBSA_ERR_UNSUPPORTED for other D.
 */
qbsa_status qbsa_block_mean(const void* x, int B, int N, int S, int D, float* x_mean, void* stream);

/*
 * qbsa_block_topk -- second step of block-mask estimation (reading stated at
 * qbsa_block_mean): score[b, h, i, j] = scale * <q_mean[b, h, i, :], k_mean[b, h / (Nq/Nkv), j, :]>
 * (fp32), and block_mask[b, h, i, j] = 1 for the n_keep largest scores of each (b, h, i)
 * row, equal scores going to the lower j; 0 elsewhere (1 = compute the block, the polarity
 * qbsa_fwd and bsa_fwd read).
 *   q_mean        fp32 [B, Nq, nqb, D], k_mean fp32 [B, Nkv, nkb, D] (qbsa_block_mean outputs), device.
 *   block_mask    uint8 [B, Nq, nqb, nkb], device, caller-owned output.
 *   block_scores  fp32 [B, Nq, nqb, nkb] or NULL: the scores, for inspection.
 * Requires Nq % Nkv == 0, 1 <= n_keep <= nkb <= 2048, D a multiple of 4 and <= 1024, k_mean
 * 16-byte aligned.  Asynchronous on `stream`.
 */
qbsa_status qbsa_block_topk(const float* q_mean, const float* k_mean, int B, int Nq, int Nkv, int nqb, int nkb, int D,
                            float scale, int n_keep, uint8_t* block_mask, float* block_scores, void* stream);

/*
 * qbsa_block_topk_keep -- qbsa_block_topk with the count given as a keep fraction: each
 * query block keeps n_keep = max(1, min(nkb, round(keep * nkb))) key blocks, the product
 * taken in double and rounded to nearest with ties to even (the count rule of the
 * keep-10% / keep-50% masks of [QBSA] "EagleQBSA单算子性能验证分析", sparsity 0.9 / 0.5).
 *   keep        in [0, 1]; other values return QBSA_ERR_INVALID before any launch.
 *   n_keep_out  host int, or NULL: receives the count used.
 * Other arguments, outputs and errors as in qbsa_block_topk.
 */
qbsa_status qbsa_block_topk_keep(const float* q_mean, const float* k_mean, int B, int Nq, int Nkv, int nqb, int nkb,
                                 int D, float scale, double keep, uint8_t* block_mask, float* block_scores,
                                 int* n_keep_out, void* stream);

/*
 * qbsa_wait_selftest -- test hook for failure detection (no counterpart on the source
 * pages): launches one thread that waits, through the same bounded mbarrier wait every
 * kernel of this library uses, on a phase that nothing ever completes.  After the wait
 * limit (2 s) the thread records a timeout in the device error word and the kernel ends
 * normally, so the next qbsa_check(stream) returns QBSA_ERR_TIMEOUT and the context stays
 * usable.  No fault, trap or endless loop is involved.
 */
qbsa_status qbsa_wait_selftest(void* stream);

/*
 * qbsa_check -- waits for `stream`, then reports and clears the device error word:
 * QBSA_ERR_TIMEOUT if a kernel's bounded wait expired since the last check,
 * QBSA_ERR_CUDA on an asynchronous CUDA error, QBSA_OK otherwise.
 */
qbsa_status qbsa_check(void* stream);

/* Thread-local description of the last non-OK status returned on this thread. */
const char* qbsa_last_error(void);

/* Library ABI version (major * 100 + minor): 103 (1.01 added qbsa_block_mean, qbsa_block_topk,
 * qbsa_wait_selftest; 1.02 qbsa_block_topk_keep and qbsa_quantize_v_noalloc; 1.03
 * qbsa_fwd_host). */
int qbsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QBSA_H_ */
