/*
 * varlen_attn.h — C ABI of the packed variable-length attention library for
 * NVIDIA B200 (sm_100a): the forward, its backward, a K/V-cache decode step
 * and the packed-layout helpers. Link: libvarlen_attn.so.
 *
 * The operation (pages cited by title and section):
 *   Many ragged sequences are concatenated into one token stream; explicit
 *   cumulative boundaries cu_seqlens say where each one starts, and each
 *   sequence attends only to itself ("[feat] pack the GenRec training forward
 *   through FlashAttention-2", summary and Test plan). Query heads share K/V
 *   heads in groups (GQA: "fix(flex): avoid decoding kernel selection for
 *   short GQA", Verification). An optional fp32 additive bias is either per
 *   key or a dense per-pair grid read per sequence through strides (GiGL pull
 *   request 858, Approach). For sequence i, query head h, local query row r
 *   and local key c, with G = n_heads / n_kv_heads and kvh = h / G:
 *
 *     s = softmax_scale * <Q[cu_q[i]+r, h, :], K[cu_k[i]+c, kvh, :]>
 *         + bias_per_key[cu_k[i]+c, h] + bias_pair[i*sb + h*sh + r*sq + c*sk]
 *     visible(r, c) = !causal || c <= r + (Lk_i - Lq_i)     (bottom-right)
 *     LSE[h, cu_q[i]+r] = ln sum_{visible c} exp(s)
 *     out[cu_q[i]+r, h, :] = sum_{visible c} exp(s - LSE) * V[cu_k[i]+c, kvh, :]
 *
 *   A row that sees no key (or only -inf scores) gets out = 0, LSE = -inf.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers on the current CUDA device,
 *     owned by the caller. The library never frees or keeps them.
 *   - Sizes and scalars are host values. `stream` is a cudaStream_t passed as
 *     void* (NULL = legacy default stream).
 *   - Calls are asynchronous on `stream`: nothing synchronises, and outputs
 *     are complete when the stream reaches the call.
 *   - The library owns one grow-only device workspace per (device, stream)
 *     for its work list; it is allocated on the first call that needs it (so
 *     make a first call before timing or capturing). Calls on one stream are
 *     ordered by the stream; calls on different streams use different
 *     workspaces.
 *   - Return value: VARLEN_ATTN_OK (0) or a positive varlen_attn_status.
 *     Argument errors are detected on the host before anything is launched.
 *     There is no fallback path: an unsupported case is an error.
 *   - The contents of cu_seqlens are validated on the device (cu[0] = 0,
 *     non-decreasing, cu[batch] <= total, each length <= its max_seqlen).
 *     Invalid boundaries launch no attention work, leave out/lse unwritten and
 *     raise VARLEN_ATTN_ERR_BAD_SEQLENS in the device error word, which
 *     varlen_attn_get_device_error() reports.
 */
#ifndef VARLEN_ATTN_H_
#define VARLEN_ATTN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum varlen_attn_status {
  VARLEN_ATTN_OK = 0,
  VARLEN_ATTN_ERR_NULL_POINTER = 1,     /* a required pointer is NULL */
  VARLEN_ATTN_ERR_BAD_SHAPE = 2,        /* batch/heads/totals/max lengths out of range,
                                           or a zero-sized dimension (zero-dimension guard,
                                           FDMA integration page, Key Implementation Points) */
  VARLEN_ATTN_ERR_GQA_MISMATCH = 3,     /* n_heads is not a multiple of n_kv_heads */
  VARLEN_ATTN_ERR_HEAD_DIM = 4,         /* head_dim not supported (bf16: 64 or 128;
                                           fp32: 64 or 128) */
  VARLEN_ATTN_ERR_MISALIGNED = 5,       /* q/k/v/out base not 16-byte aligned, or
                                           lse/bias base not 4-byte aligned */
  VARLEN_ATTN_ERR_BAD_BIAS = 6,         /* negative bias strides */
  VARLEN_ATTN_ERR_CUDA = 7,             /* a CUDA runtime/driver call failed */
  VARLEN_ATTN_ERR_DEVICE = 8,           /* current device is not sm_100 (B200 class) */
  VARLEN_ATTN_ERR_BAD_SEQLENS = 9,      /* device-detected: cu_seqlens content invalid */
  VARLEN_ATTN_ERR_DEVICE_TIMEOUT = 10,  /* device-detected: a bounded wait inside the
                                           kernel expired; outputs are unspecified */
  VARLEN_ATTN_ERR_TOO_LARGE = 11,       /* sizes overflow the library's 32-bit indexing */
  VARLEN_ATTN_ERR_SCRATCH_LIMIT = 12    /* varlen_attn_fwd_noalloc: the work list does not
                                           fit its fixed scratch */
} varlen_attn_status;

/*
 * Packed varlen attention forward, bf16 in / bf16 out, fp32 LSE.
 * Runs on tensor cores (tcgen05, accumulators in tensor memory).
 *
 *   q        [total_q, n_heads, head_dim] bf16, contiguous, 16-byte aligned.
 *   k, v     [total_k, n_kv_heads, head_dim] bf16, contiguous, 16-byte aligned
 *            (may be NULL when total_k is 0: no row then sees a key).
 *   cu_seqlens_q, cu_seqlens_k
 *            [batch + 1] int32 device arrays; sequence i owns query rows
 *            [cu_q[i], cu_q[i+1]) and key rows [cu_k[i], cu_k[i+1]).
 *            Zero-length sequences are allowed.
 *   batch    number of sequences B >= 1 (host value, so no device read is
 *            needed to size the launch).
 *   total_q, total_k
 *            row counts of q and k/v (host values; the leading dimension of
 *            the tensors). cu_q[B] <= total_q and cu_k[B] <= total_k.
 *   max_seqlen_q, max_seqlen_k
 *            upper bounds on the per-sequence lengths; they size the work list
 *            and are checked on the device. Results do not depend on them.
 *   n_heads, n_kv_heads
 *            query heads Hq and K/V heads Hkv; Hq % Hkv == 0.
 *   head_dim 64 or 128.
 *   softmax_scale  multiplies <q, k> before the biases are added.
 *   causal   0 or 1; 1 = bottom-right aligned mask c <= r + Lk - Lq.
 *   bias_per_key   NULL, or [total_k, n_heads] fp32 contiguous.
 *   bias_pair      NULL, or fp32 grid read at element offset
 *                  i*bias_stride_b + h*bias_stride_h + r*bias_stride_q + c*bias_stride_k
 *                  (strides in elements, >= 0; bias_stride_h = 0 shares one grid
 *                  across heads). Only in-sequence entries (r < Lq_i, c < Lk_i) are
 *                  read, so a grid sized [B, *, max_seqlen_q, max_seqlen_k] needs no
 *                  zero padding (GiGL pull request 858, Approach, strided view).
 *   out      [total_q, n_heads, head_dim] bf16 output, 16-byte aligned. Rows
 *            outside every sequence (beyond cu_q[B]) are not written.
 *   lse      NULL, or [n_heads, total_q] fp32 output: natural-log sum of exp of
 *            the scaled, biased scores (-inf for a row that sees no key).
 * Inputs are taken to be finite. A sequence's last key tile (128 rows) may
 * reach into the next sequence's rows, whose probabilities are exactly 0, so
 * an Inf or NaN in a neighbour's V would reach this sequence through 0 * Inf;
 * with finite inputs every sequence's results are independent of its
 * neighbours bit for bit.
 */
int varlen_attn_fwd(const void* q, const void* k, const void* v,
                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                    int batch, int total_q, int total_k,
                    int max_seqlen_q, int max_seqlen_k,
                    int n_heads, int n_kv_heads, int head_dim,
                    float softmax_scale, int causal,
                    const float* bias_per_key,
                    const float* bias_pair, int64_t bias_stride_b, int64_t bias_stride_h,
                    int64_t bias_stride_q, int64_t bias_stride_k,
                    void* out, float* lse, void* stream);

/* Flags of varlen_attn_fwd_ex. */
enum {
  /* The per-pair grid is per K/V head: query head h reads grid head h / G,
   * i.e. element i*bias_stride_b + (h / G)*bias_stride_h + r*bias_stride_q +
   * c*bias_stride_k. This is the attention_bias layout (batch, n_kv_heads,
   * q_len, k_len) of "Flash Dynamic Mask Attention (FDMA) Into
   * Transformers-Style Attention", Key Implementation Points, Attn Bias Path,
   * read without expanding it to the query heads. */
  VARLEN_ATTN_BIAS_PAIR_KV_HEADS = 1
};

/*
 * varlen_attn_fwd with option flags (a bitwise OR of the enum above; 0 gives
 * exactly varlen_attn_fwd). Unknown flag bits return VARLEN_ATTN_ERR_BAD_BIAS.
 * Same arguments, outputs, ownership and error rules as varlen_attn_fwd.
 */
int varlen_attn_fwd_ex(const void* q, const void* k, const void* v,
                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                       int batch, int total_q, int total_k,
                       int max_seqlen_q, int max_seqlen_k,
                       int n_heads, int n_kv_heads, int head_dim,
                       float softmax_scale, int causal,
                       const float* bias_per_key,
                       const float* bias_pair, int64_t bias_stride_b, int64_t bias_stride_h,
                       int64_t bias_stride_q, int64_t bias_stride_k, unsigned flags,
                       void* out, float* lse, void* stream);

/*
 * Same operation with fp32 q/k/v/out (fp32 arithmetic on the CUDA cores).
 * Same arguments and rules as varlen_attn_fwd, except that q, k, v and out
 * are fp32 arrays of the same shapes. Meant for parity checks at fp32
 * precision, where tensor-core TF32 rounding would be too coarse.
 */
int varlen_attn_fwd_f32(const float* q, const float* k, const float* v,
                        const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                        int batch, int total_q, int total_k,
                        int max_seqlen_q, int max_seqlen_k,
                        int n_heads, int n_kv_heads, int head_dim,
                        float softmax_scale, int causal,
                        const float* bias_per_key,
                        const float* bias_pair, int64_t bias_stride_b, int64_t bias_stride_h,
                        int64_t bias_stride_q, int64_t bias_stride_k,
                        float* out, float* lse, void* stream);

/*
 * varlen_attn_fwd without any device allocation by the library.
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot have a library allocate device memory on their behalf:
 * runtimes that reserve the whole device pool up front and fail any outside
 * cudaMalloc, request loops that must not stall (cudaMalloc/cudaFree can
 * synchronise the device and take unbounded time), and hosts that give a
 * plug-in a fixed memory budget.
 *
 * Same arguments, operation, outputs and rules as varlen_attn_fwd, except:
 *   - The work list lives in a fixed array compiled into the library
 *     (256 B + 2 x 16384 x 8 B, about 256 KiB) that every GPU loading the
 *     library holds until the process exits. It calls no cudaMalloc,
 *     cudaFree or other allocating routine; the caller still owns q/k/v,
 *     the biases, out and lse.
 *   - At most 16384 work-list pairs: batch * ceil(G * ceil(max_seqlen_q /
 *     128) / 2) with G = n_heads / n_kv_heads >= 2, batch *
 *     ceil(ceil(max_seqlen_q / 128) / 2) otherwise. Larger problems return
 *     VARLEN_ATTN_ERR_SCRATCH_LIMIT before anything is launched.
 *   - The first call on a device looks up that array's device address (with
 *     the device current) and caches it; make that first call before any
 *     stream capture.
 *   - Within a process, every call on a device shares that device's one
 *     array, and each call overwrites what the previous call left there.
 *     Calls that can run at the same time on one device (for example on two
 *     streams) race on it; the caller must order them.
 */
int varlen_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int batch, int total_q, int total_k,
                            int max_seqlen_q, int max_seqlen_k,
                            int n_heads, int n_kv_heads, int head_dim,
                            float softmax_scale, int causal,
                            const float* bias_per_key,
                            const float* bias_pair, int64_t bias_stride_b, int64_t bias_stride_h,
                            int64_t bias_stride_q, int64_t bias_stride_k,
                            void* out, float* lse, void* stream);

/*
 * Backward pass of varlen_attn_fwd (bf16). The gradients of a loss through
 * O = varlen_attn_fwd(...): the packed path's gradients that the TorchEasyRec
 * PR 663 page (GenRec, "Test plan") checks and the ASpec PR 25 page
 * ("Verification") bounds at 1% relative L2 for Q/K/V, including the bias
 * gradients that the GiGL PR 858 page ("Approach") lists as missing for a
 * per-sequence bias. With P the forward's probabilities and
 * delta = rowsum(dO * O):
 *
 *   dV = P^T dO,  dS = P * (dO V^T - delta),  dQ = scale dS K,  dK = scale dS^T Q,
 *   dbias_per_key[cu_k[i] + c, h] = sum_r dS[r, c],  dbias_pair[i, h, r, c] = dS[r, c].
 *
 * Inputs: everything varlen_attn_fwd took (same meaning, same flags), plus
 *   out  [total_q, n_heads, head_dim] bf16: the forward's output;
 *   lse  [n_heads, total_q] fp32: the forward's LSE (required);
 *   dout [total_q, n_heads, head_dim] bf16: the gradient of the loss w.r.t. out.
 * Outputs (caller-owned, written, not accumulated):
 *   dq [total_q, n_heads, head_dim], dk and dv [total_k, n_kv_heads, head_dim]
 *   bf16 (dk, dv summed over the n_heads / n_kv_heads query heads of a group;
 *   k, v, dk and dv may be NULL when total_k is 0);
 *   dbias_per_key [total_k, n_heads] fp32 or NULL (not computed);
 *   dbias_pair fp32 or NULL: entry (i, h, r, c) at i*dbias_stride_b +
 *   h*dbias_stride_h + r*dbias_stride_q + c for every query head h and every
 *   in-sequence (r, c); other entries are left as they are. A broadcast or
 *   per-K/V-head grid's gradient is the sum of these over the heads that read it.
 * Rows without a visible key get zero gradients. dq, dk, dv and dbias_pair
 * are bitwise reproducible (no atomics); dbias_per_key is the sum of four
 * partial sums added atomically into the zeroed buffer, so its last bits may
 * vary between runs. Launches: one validates cu_seqlens (a bad table raises
 * VARLEN_ATTN_ERR_BAD_SEQLENS on the device and writes no gradient), one
 * computes delta into the library workspace, one computes dK and dV per
 * (sequence, K/V head, 128-key block), one dQ per (sequence, query head,
 * 128-row block); with dbias_per_key a memset zeroes it first. Errors as for
 * varlen_attn_fwd; batch or n_heads above 65535: VARLEN_ATTN_ERR_TOO_LARGE.
 */
int varlen_attn_bwd(const void* q, const void* k, const void* v, const void* out,
                    const float* lse, const void* dout,
                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                    int batch, int total_q, int total_k,
                    int max_seqlen_q, int max_seqlen_k,
                    int n_heads, int n_kv_heads, int head_dim,
                    float softmax_scale, int causal,
                    const float* bias_per_key,
                    const float* bias_pair, int64_t bias_stride_b, int64_t bias_stride_h,
                    int64_t bias_stride_q, int64_t bias_stride_k, unsigned flags,
                    void* dq, void* dk, void* dv, float* dbias_per_key,
                    float* dbias_pair, int64_t dbias_stride_b, int64_t dbias_stride_h,
                    int64_t dbias_stride_q, void* stream);

/*
 * Decode attention over a per-sequence K/V cache (flash_attn_with_kvcache,
 * listed by the noether attention module page, module; the decoding-kernel
 * path that short GQA rows can reach, "fix(flex): avoid decoding kernel
 * selection for short GQA", Outcome; q_len = 1 decode steps, FDMA
 * integration page, Causality Handling). Same definition as varlen_attn_fwd
 * with the keys and values of sequence i taken from the cache:
 *
 *   k_cache, v_cache  [batch, cache_len, n_kv_heads, head_dim] bf16; sequence
 *            i's cached rows are i*cache_len .. i*cache_len + cache_seqlens[i]-1.
 *   k_new, v_new      NULL (both), or [total_q, n_kv_heads, head_dim] bf16
 *            packed like q: sequence i's new rows are first written into its
 *            cache rows cache_seqlens[i] .. cache_seqlens[i] + Lq_i - 1 (the
 *            cache is modified; cache_seqlens is not), and attended to.
 *   Lk_i = cache_seqlens[i] (+ Lq_i with new rows); causal is bottom-right as
 *   in varlen_attn_fwd (with Lq_i = 1 it changes nothing).
 *   q [total_q, n_heads, head_dim] bf16 with cu_seqlens_q [batch + 1];
 *   max_seqlen_q * (n_heads / n_kv_heads) <= 32 (decode-sized queries; longer
 *   ones belong to varlen_attn_fwd): else VARLEN_ATTN_ERR_BAD_SHAPE.
 *   out [total_q, n_heads, head_dim] bf16, lse [n_heads, total_q] fp32 or NULL.
 *   num_splits: 0 = automatic: the step runs on the tensor cores, the rows
 *            of all G query heads of a K/V group in one tile. When batch *
 *            n_kv_heads is at least the device's SM count, one work item per
 *            (sequence, K/V head). With fewer pairs, the cache's key positions
 *            are cut into fixed ranges (multiples of 128 keys, at least 512,
 *            sized from cache_len and the pair count for about eight work
 *            items per SM, at most 64 ranges), one work item per (range,
 *            pair); each range's output, normalised by its own sum, goes in
 *            fp32 to the library workspace, and a further launch merges the
 *            ranges by their LSE. num_splits > 0: the step runs on the CUDA
 *            cores (fp32) with the key positions cut into num_splits equal
 *            ranges (whole 32-key blocks), one CTA per (range, K/V head,
 *            sequence), merged the same way. Ranges past a sequence's length
 *            are empty and only mark their partial LSE as -inf. Results depend
 *            on the path and the ranges in the last bits (the order of the
 *            sums), so give a fixed num_splits where bitwise reproducibility
 *            across batch compositions matters.
 * HBM-bound (every cached key and value is read once); no bias. Errors as
 * for varlen_attn_fwd; a cache position beyond cache_len raises
 * VARLEN_ATTN_ERR_BAD_SEQLENS on the device.
 */
int varlen_attn_decode(const void* q, const int32_t* cu_seqlens_q, int batch, int total_q,
                       int max_seqlen_q, void* k_cache, void* v_cache, int cache_len,
                       const int32_t* cache_seqlens, const void* k_new, const void* v_new,
                       int n_heads, int n_kv_heads, int head_dim, float softmax_scale,
                       int causal, int num_splits, void* out, float* lse, void* stream);

/* ------------------------------------------------------------------------
 * Packed-layout helpers (device-side, asynchronous on `stream`).
 *
 * They turn a padded batch into the packed stream the forward reads and back
 * again, following the varlen unpad / pad pipeline of "Flash Dynamic Mask
 * Attention (FDMA) Into Transformers-Style Attention" (Key Implementation
 * Points, Variable Length Flow), and fold a per-pair bias row into a per-key
 * bias ("[GiGL] pull request 858", Approach: with query_is_first_token, row 0
 * of the per-pair bias is added to the per-key bias). Boundaries and indices
 * read from device memory are bounds-checked: a bad value raises
 * VARLEN_ATTN_ERR_BAD_SEQLENS in the device error word and the affected row is
 * skipped (never read or written out of range).
 * ------------------------------------------------------------------------ */

/*
 * Unpadding: mask [batch, seqlen] uint8 (nonzero = valid position), row-major.
 * Writes cu_seqlens [batch + 1] (sequence b = the valid positions of row b,
 * in increasing order), indices [cu_seqlens[batch]] (flat padded position
 * b * seqlen + s of every packed row; capacity batch * seqlen) and
 * max_seqlen [1] (the largest row count), all int32 device arrays. Three
 * kernel launches; nothing is read back to the host.
 */
int varlen_mask_to_seqlens(const uint8_t* mask, int batch, int seqlen, int32_t* cu_seqlens,
                           int32_t* indices, int32_t* max_seqlen, void* stream);

/*
 * Gather (unpad): dst[t] = src[indices[t]] for t < cu_seqlens[batch], rows of
 * row_bytes bytes (a multiple of 16; src and dst 16-byte aligned). src holds
 * src_rows rows, dst dst_rows rows, indices at least dst_rows entries.
 * cu_seqlens[batch] > dst_rows or an index outside [0, src_rows) is a device
 * error (VARLEN_ATTN_ERR_BAD_SEQLENS). Rows of dst past cu_seqlens[batch] are
 * not written.
 */
int varlen_gather_rows(const void* src, int64_t src_rows, int64_t row_bytes,
                       const int32_t* indices, const int32_t* cu_seqlens, int batch, void* dst,
                       int64_t dst_rows, void* stream);

/*
 * Scatter (pad): dst (dst_rows rows of row_bytes bytes) is zeroed, then
 * dst[indices[t]] = src[t] for t < cu_seqlens[batch]. src holds src_rows rows,
 * indices at least src_rows entries. cu_seqlens[batch] > src_rows or an index
 * outside [0, dst_rows) is a device error. Same alignment rules as the gather.
 */
int varlen_scatter_rows(const void* src, int64_t src_rows, int64_t row_bytes,
                        const int32_t* indices, const int32_t* cu_seqlens, int batch, void* dst,
                        int64_t dst_rows, void* stream);

/*
 * First-token fold: for every sequence i and key c < Lk_i (Lk_i from
 * cu_seqlens_k) and head h < n_heads,
 *   bias_out[cu_k[i] + c, h] = (bias_in ? bias_in[cu_k[i] + c, h] : 0)
 *       + bias_pair[i*bias_stride_b + (h / head_div)*bias_stride_h
 *                   + row*bias_stride_q + c*bias_stride_k]
 * with head_div = 1 for a grid over query heads, G for a grid over K/V heads.
 * bias_in and bias_out are [total_k, n_heads] fp32 (they may be the same
 * array); key rows past cu_seqlens_k[batch] are not written. A forward whose
 * sequences each query only row `row` then gives the same result with
 * bias_out as its per-key bias and no per-pair grid. The caller guarantees
 * that the grid covers the entries read.
 */
int varlen_fold_pair_bias_row(const float* bias_pair, int64_t bias_stride_b,
                              int64_t bias_stride_h, int64_t bias_stride_q, int64_t bias_stride_k,
                              int row, int head_div, const int32_t* cu_seqlens_k, int batch,
                              int total_k, int n_heads, const float* bias_in, float* bias_out,
                              void* stream);

/* Static description of a status code. Never NULL. */
const char* varlen_attn_strerror(int status);

/*
 * Synchronises `stream`, then returns and clears the device error word of the
 * current device (VARLEN_ATTN_OK if no kernel reported a problem). Returns
 * VARLEN_ATTN_ERR_CUDA if the synchronisation itself fails.
 */
int varlen_attn_get_device_error(void* stream);

/*
 * Measurement hook. When both events are non-NULL, later calls from this host
 * thread record `start_event` just before and `stop_event` just after the
 * attention kernel's launch, on the call's stream (cudaEvent_t passed as
 * void*). Pass NULL, NULL to stop. Does not change what is computed.
 */
int varlen_attn_set_profile_events(void* start_event, void* stop_event);

/*
 * Failure-detection control. Every wait of the tensor-core forward and
 * backward kernels on a pipeline barrier (shared-memory mbarrier) is bounded:
 * after `cycles` SM clock cycles without progress the kernel raises
 * VARLEN_ATTN_ERR_DEVICE_TIMEOUT in the device error word, every role of the
 * CTA leaves its loop, the copies already in flight are waited for (with a
 * fixed limit of 2^29 cycles), tensor memory is released and the kernel
 * returns; the outputs of that call are then undefined but the context stays
 * usable. 0 restores the default of 2^33 cycles (about 4 s at 2 GHz).
 * Applies to calls launched after it, from any host thread (process-wide).
 * A short limit is a test of the abort path, not a tuning knob: any wait
 * longer than the limit aborts the call. Negative values return
 * VARLEN_ATTN_ERR_BAD_SHAPE. (No counterpart on the pages: their kernels have
 * no failure detection.)
 */
int varlen_attn_set_wait_limit(long long cycles);

/*
 * Test hook of that abort path, off by default: while `on` is non-zero, the
 * MMA warp of every CTA of the tensor-core forward and backward kernels
 * launched afterwards first waits on a barrier phase that nothing completes,
 * so that wait runs out after the wait limit and aborts the call exactly as
 * a stalled pipeline would (VARLEN_ATTN_ERR_DEVICE_TIMEOUT, outputs
 * undefined). Process-wide; pass 0 to switch it off. Use it together with a
 * short varlen_attn_set_wait_limit, or each call waits the default ~4 s.
 */
int varlen_attn_set_test_stall(int on);

/* Number of kernels one varlen_attn_fwd / varlen_attn_fwd_f32 call launches. */
int varlen_attn_launches_per_call(int fp32_path);

/*
 * Detail of the last VARLEN_ATTN_ERR_CUDA raised on this host thread: the
 * failing step and CUDA's message. Empty string if none. Never NULL; the
 * buffer is owned by the library and overwritten by the next failure.
 */
const char* varlen_attn_last_error_detail(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int varlen_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* VARLEN_ATTN_H_ */
