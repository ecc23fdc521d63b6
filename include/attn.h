/*
 * exact_tiled_attention_38_b200: exact scaled-dot-product attention for B200
 * (sm_100a), as a C ABI.
 *
 * What is computed (every entry point): for each batch b, query head h and
 * query row i,
 *     s_ij  = scale * sum_c q[b,h,i,c] * k[b,g,j,c],   g = h / (Hq / Hkv)
 *     s_ij  = -inf where key j is masked (causal: j > i + Nk - Nq)
 *     o[b,h,i,:] = sum_j softmax_j(s_i.) * v[b,g,j,:]
 *     lse[b,h,i] = ln sum_j exp(s_ij)
 * This is exact attention (not an approximation): the aikaboom page
 * "11.4d FlashAttention" lists the tiled method's result as the same
 * mathematical result as standard attention (comparison table), and the
 * zimaspace page "How Does Flash Attention Reduce Memory Traffic During Local
 * Inference?" says the tiled algorithm still produces exact attention. It is
 * computed tile by tile with a running (online) softmax, so the score matrix
 * never reaches device memory (aikaboom page, sections "Tiling" and "Online
 * Softmax"; zimaspace page, "Online Softmax Avoids Storing the Full Score
 * Matrix" and "Kernel Fusion Keeps More of the Attention Chain in One
 * Execution Path"). GQA grouping follows the sicorps page's last paragraph
 * (n < n_head key/value heads, each shared by a group of query heads; MQA is
 * Hkv = 1).
 *
 * Conventions shared by all entry points:
 *   - All pointers are DEVICE pointers owned by the caller. The library never
 *     frees or retains them. q, k, v, o, kcache, vcache must be 16-byte
 *     aligned; lse and seqlens 4-byte aligned. Tensors are contiguous.
 *   - Element type: attn_fwd / attn_decode take bfloat16 q, k, v and write
 *     bfloat16 o; the _f16 twins take and write IEEE fp16. lse is float32.
 *     Products accumulate in fp32; softmax statistics are fp32.
 *   - scale must be finite and > 0 (the usual value is 1/sqrt(d)).
 *   - lse may be NULL: the log-sum-exp is then not written.
 *   - Work is enqueued on `stream` (NULL = legacy default stream); calls return
 *     without synchronising. Errors detected on the host return a negative
 *     code before anything is enqueued.
 *   - A row with no visible key (causal with Nq > Nk, or an empty decode
 *     sequence) gets o = 0 and lse = -inf.
 *   - Head size d: d = 64 and d = 128 run on the tensor-core kernels
 *     (tcgen05 MMA, TMA-fed tiles). Any other d that is a multiple of 8 in
 *     [8, 256] runs on a generic CUDA-core kernel with the same results to
 *     rounding (16 query rows per block, 32-key tiles staged in shared
 *     memory, fp32 online softmax); it is correct but far from the tensor-core
 *     kernels' speed. Other d return ATTN_ERR_UNSUPPORTED.
 *   - Every wait inside a kernel is bounded (about 2 s). If one gives up, the
 *     kernel ends early, its outputs are undefined, and
 *     attn_get_device_status() reports ATTN_ERR_TIMEOUT. No kernel traps.
 */
#ifndef EXACT_TILED_ATTENTION_ATTN_H
#define EXACT_TILED_ATTENTION_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream; declared here so that callers need no
   CUDA header. */
typedef struct CUstream_st* attn_stream_t;

enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = -1,     /* null pointer, bad size, misaligned, Hq % Hkv != 0, bad scale */
  ATTN_ERR_UNSUPPORTED = -2, /* d not a multiple of 8 in [8, 256]; decode with d = 64 / 128 and
                                B > 65,535; or the device is not sm_100 */
  ATTN_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
  ATTN_ERR_TIMEOUT = -4,     /* a device-side wait gave up (see attn_get_device_status) */
  ATTN_ERR_SCRATCH = -5      /* attn_decode_noalloc: sizes exceed its fixed scratch */
};

/*
 * Prefill: many query tokens against keys/values of the same sequence
 * (aikaboom page, "The Core Problem" and "Tiling"; first page: prefill
 * processes n tokens, so the cost is quadratic).
 *   q   [B, Hq,  Nq, d]  bf16      k, v [B, Hkv, Nk, d] bf16
 *   o   [B, Hq,  Nq, d]  bf16      lse  [B, Hq, Nq] float32 (or NULL)
 *   causal != 0: bottom-right aligned mask, query i sees keys j <= i + Nk - Nq
 *                (equal to the usual lower-triangular mask when Nq == Nk).
 * Sizes: B >= 0, Nq >= 0, Nk >= 0 (B == 0 or Nq == 0: nothing to do;
 * Nk == 0: every row is empty), Hq >= 1, Hkv >= 1, Hq % Hkv == 0,
 * d a multiple of 8 in [8, 256], Nq <= 16,776,960, B * Hq < 2^31.
 * Allocates no device memory.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Nq, int Nk, int d, float scale, int causal, attn_stream_t stream);

/* attn_fwd with IEEE fp16 q, k, v and o. */
int attn_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                 int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                 attn_stream_t stream);

/*
 * Decode: one new query token per sequence over a ragged KV cache (first
 * page: generating a token re-reads the whole KV cache plus the new entry, a
 * cost linear in the cache length; zimaspace page, "Reduced IO Is Not the Same
 * as Eliminating KV Cache").
 *   q       [B, Hq, d]  bf16
 *   kcache, vcache: packed per sequence. Sequence b starts at token offset
 *           off_b = sum_{j<b} seqlens[j] and is laid out [Hkv][seqlens[b]][d],
 *           i.e. element (b, g, t, c) is at ((off_b * Hkv + g * L_b + t) * d + c).
 *           The new token's key/value must already be appended.
 *           kcache and vcache must be non-NULL even if every sequence is empty.
 *   seqlens [B] int32, DEVICE memory, read only on the device (negative
 *           values count as 0; 0 gives o = 0, lse = -inf).
 *   o       [B, Hq, d]  bf16       lse [B, Hq] float32 (or NULL)
 * Sizes: B >= 0 (0: nothing to do), Hq >= 1, Hkv >= 1, Hq % Hkv == 0,
 * d a multiple of 8 in [8, 256], B * Hq < 2^29; for d = 64 and 128 also
 * B <= 65,535 (larger B returns ATTN_ERR_UNSUPPORTED).
 * Device memory: the call takes one workspace block from cudaMallocFromPoolAsync
 * on `stream` and returns it with cudaFreeAsync on the same stream
 * (stream-ordered; no block outlives the call's work). Its size:
 *   - d = 128 with 2 to 32 query heads per KV head (G = Hq / Hkv), the
 *     persistent tensor-core pass: B * 8 + (B + 1) * 4 bytes of per-sequence
 *     offsets, 16 bytes per SM, and (B * Hkv + SMs - 1) * G * (d + 1) * 4 bytes
 *     of partial results, each part rounded up to 256 bytes;
 *   - other d = 64 and 128 cases, the CUDA-core split pass: nsplit * B * Hq *
 *     (d + 1) * 4 bytes of split partials (nsplit = attn_decode_num_splits),
 *     plus B * 8 bytes of token offsets when B > 1024;
 *   - other d: B * 8 bytes of token offsets when B > 1024, else nothing.
 * The pool is the library's own, one per device, created on first use; it
 * keeps up to 256 MiB of freed blocks cached, so callers that synchronise
 * between calls do not pay for re-mapping device memory each time. The
 * caller's pools are not touched.
 */
int attn_decode(const void* q, const void* kcache, const void* vcache, const int32_t* seqlens,
                void* o, float* lse, int B, int Hq, int Hkv, int d, float scale,
                attn_stream_t stream);

/* attn_decode with IEEE fp16 q, kcache, vcache and o. */
int attn_decode_f16(const void* q, const void* kcache, const void* vcache,
                    const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv, int d,
                    float scale, attn_stream_t stream);

/*
 * attn_decode that allocates nothing. The pages have no counterpart for this
 * entry point; it exists for callers that cannot allocate device memory where
 * they run decode: an engine that gives nearly all of HBM to its own KV-cache
 * pool at start-up, a latency-critical path where an allocator call may lock
 * or synchronise, or a runtime whose memory plan is fixed before serving.
 * Same arguments, layout and results as attn_decode (bf16), except:
 *   - The workspace is a fixed array of 2,097,152 floats (8 MiB) in this
 *     library's device memory, held by every GPU that loads the library
 *     until the process exits. It calls no cudaMalloc/cudaFree and no
 *     allocating library routine.
 *   - Persistent tensor-core pass (d = 128, 2 to 32 query heads per KV head):
 *     when its partial results (sizes as in attn_decode) do not fit, each SM
 *     takes whole (sequence, KV head) segments and writes o and lse itself;
 *     only the per-sequence offsets (under 1 MB for B <= 65,535) are kept in
 *     the array, so these calls are never refused. Results agree with
 *     attn_decode to rounding.
 *   - CUDA-core split pass (other d = 64 and 128 cases): one split needs
 *     B * Hq * (d + 1) floats besides the token offsets of a batch above 1024
 *     sequences. When the usual split count does not fit, fewer splits are
 *     used (results then agree with attn_decode to rounding); when not one
 *     split fits the call returns ATTN_ERR_SCRATCH and enqueues nothing.
 *   - Other d keep only the token offsets of a batch above 1024 sequences in
 *     the array (beyond a million sequences each block sums them itself).
 *   - The first call on a device looks up the array's device address (a
 *     runtime call); make that first call before any stream capture. The
 *     address is remembered with the id of the device's context; after
 *     cudaDeviceReset (a new context) the next call looks it up again, so
 *     make the first call after a reset before any capture too.
 *   - Every call on a device uses the same array, which keeps the previous
 *     call's contents (nothing in it needs to start at zero). Calls that can
 *     overlap on the GPU (different streams without ordering between them)
 *     race on it and give wrong results; order them on one stream or by events.
 */
int attn_decode_noalloc(const void* q, const void* kcache, const void* vcache,
                        const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                        int d, float scale, attn_stream_t stream);

/*
 * Sliding-window variants (the "windowing" scheme the zimaspace page names in
 * "Reduced IO Is Not the Same as Eliminating KV Cache", applied as a mask).
 * attn_fwd_window: causal prefill where query i keeps only keys j with
 *   i + (Nk - Nq) - window < j <= i + (Nk - Nq), i.e. its `window` most recent
 *   positions including its own (bottom-right alignment as in attn_fwd).
 *   Key tiles wholly outside every row's window are never loaded.
 * attn_decode_window: the new token of sequence b reads only the last
 *   min(window, L_b) cached tokens (cache layout as in attn_decode).
 * window must be >= 1 (a window at least as long as the keys gives the plain
 * causal / full result). Other arguments, layouts, ownership and errors are
 * those of attn_fwd / attn_decode; the _f16 twins take and write fp16.
 */
int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                    attn_stream_t stream);
int attn_fwd_window_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Nq, int Nk, int d, float scale, int window,
                        attn_stream_t stream);
int attn_decode_window(const void* q, const void* kcache, const void* vcache,
                       const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv, int d,
                       float scale, int window, attn_stream_t stream);
int attn_decode_window_f16(const void* q, const void* kcache, const void* vcache,
                           const int32_t* seqlens, void* o, float* lse, int B, int Hq, int Hkv,
                           int d, float scale, int window, attn_stream_t stream);

/*
 * Merge of partial results over disjoint key sets (context-parallel prefill:
 * each step computes a query block's attention over one key block with
 * attn_fwd, and the steps' results are folded together). The log-sum-exp
 * identity follows from the running softmax statistics (aikaboom page
 * "11.4d FlashAttention", "Online Softmax"): for one query row,
 *     LSE = ln(e^lse_acc + e^lse_part)
 *     O   = e^(lse_acc - LSE) * o_acc + e^(lse_part - LSE) * o_part.
 *   o_acc    [rows, d] float32, in/out: the running merged O (unrounded)
 *   lse_acc  [rows]    float32, in/out: the running LSE (natural log). A row
 *            whose lse_acc is -inf is empty and its o_acc is NOT read, so an
 *            accumulator starts as lse_acc = -inf with o_acc uninitialised.
 *   o_part   [rows, d] bf16 (attn_merge) or fp16 (attn_merge_f16), and
 *   lse_part [rows]    float32: one partial result, e.g. attn_fwd's o and lse
 *            over a key block (rows = B * Hq * Nq in attn_fwd's layout). A
 *            partial row with lse_part = -inf (no visible key) changes nothing.
 *   o_out    [rows, d] bf16 / fp16, or NULL: if not NULL, also receives the
 *            merged O rounded to nearest (the final merge of a sequence of
 *            merges writes the output this way); rows that stay empty get 0.
 * Sizes: rows >= 0 (0: nothing to do), d a multiple of 8 in [8, 256].
 * Pointers are device pointers owned by the caller; o_acc, o_part and o_out
 * 16-byte aligned, lse_acc and lse_part 4-byte aligned. o_out must not
 * overlap the other arrays. Allocates nothing.
 */
int attn_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
               void* o_out, long long rows, int d, attn_stream_t stream);
int attn_merge_f16(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                   void* o_out, long long rows, int d, attn_stream_t stream);

/*
 * Partial results kept in fp32, for a sequence of merges (context-parallel
 * prefill folds one query block's attention over every key block; rounding
 * each partial O to bf16 / fp16 before it is merged would add one rounding per
 * fold). The running-statistics merge is the aikaboom page's "Online Softmax"
 * applied to whole key blocks.
 * attn_fwd_partial / attn_fwd_partial_f16: attn_fwd / attn_fwd_f16 (bf16 /
 *   fp16 q, k, v; same layouts, masks, sizes and errors) except that o is
 *   float32 [B, Hq, Nq, d] holding O = sum_j softmax_j * v_j unrounded
 *   (16-byte aligned). No sliding window. Allocates nothing.
 * attn_merge_partial / attn_merge_partial_f16: attn_merge / attn_merge_f16
 *   with o_part float32 [rows, d] (such a partial O); o_out, if not NULL,
 *   receives the merged O rounded to bf16 / fp16.
 */
int attn_fwd_partial(const void* q, const void* k, const void* v, float* o, float* lse, int B,
                     int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                     attn_stream_t stream);
int attn_fwd_partial_f16(const void* q, const void* k, const void* v, float* o, float* lse, int B,
                         int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                         attn_stream_t stream);
int attn_merge_partial(float* o_acc, float* lse_acc, const float* o_part, const float* lse_part,
                       void* o_out, long long rows, int d, attn_stream_t stream);
int attn_merge_partial_f16(float* o_acc, float* lse_acc, const float* o_part,
                           const float* lse_part, void* o_out, long long rows, int d,
                           attn_stream_t stream);

/* Number of KV splits attn_decode uses for these sizes on the current device
   (>= 1; always 1 for d other than 64 and 128 and for the persistent pass of
   d = 128 with 2 to 32 query heads per KV head, which has no fixed split
   count), or a negative error code. */
int attn_decode_num_splits(int B, int Hq, int Hkv, int d);

/* The cudaError_t value (as an int) behind the calling thread's most recent
   ATTN_ERR_CUDA from this library, or 0 if there was none. */
int attn_last_cuda_error(void);

/* Human-readable text for a return code. Never NULL. */
const char* attn_strerror(int code);

/*
 * Synchronises `stream`, then reads and clears the library's device status
 * word on the current device. Returns ATTN_OK, ATTN_ERR_TIMEOUT (a device
 * wait gave up; *raw_code, if not NULL, receives the site code) or
 * ATTN_ERR_CUDA.
 */
int attn_get_device_status(attn_stream_t stream, unsigned int* raw_code);

/*
 * Test hook for the bounded waits (not part of the attention computation).
 * Enqueues the attn_fwd prefill kernel with the same arguments and checks,
 * but with its TMA producers issuing no copies, so the kernel's first waits
 * for data can never complete; every wait gives up after wait_us
 * microseconds (1..1000000). The kernel then ends early with no copy or
 * tensor-core operation in flight, o and lse are left undefined, and the next
 * attn_get_device_status() returns ATTN_ERR_TIMEOUT with raw code
 * 0x1000 | site (site: which wait gave up first). The CUDA context stays
 * usable. Returns the enqueue status like attn_fwd, or ATTN_ERR_INVALID for
 * wait_us out of range, or ATTN_ERR_UNSUPPORTED for d other than 64 and 128
 * (the generic kernel has no waits).
 */
int attn_fwd_stall_test(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                        unsigned int wait_us, attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_TILED_ATTENTION_ATTN_H */
