/*
 * libattn -- exact IO-aware scaled-dot-product attention for B200 (sm_100a).
 *
 * Computes  O = softmax(scale * Q K^T + B) V  row by row, streaming K/V tiles
 * past a resident Q tile and carrying the online-softmax state (running max m,
 * normaliser l, unnormalised numerator a), rescaled by exp(m - m') whenever a
 * tile raises the maximum; the N_q x N_k score / probability matrix never
 * reaches device memory.  The backward keeps only the per-row log-sum-exp and
 * recomputes P tile by tile.
 *
 * Sources of the operation:
 *   - "Understanding FlashAttention Pt 1", 0.2 Notation: S = QK^T/sqrt(d) + B,
 *     P = softmax_row(S), O = PV, with B an optional additive mask or bias;
 *   - "Softmax does not need the matrix", section "Carry the Normalizer": the
 *     (m, l, a) state and its rescale-and-add merge of a new key block;
 *   - "Attention IO tiling" lesson card, The mechanism: tiles of Q/K/V staged
 *     on chip, the score block discarded, retained row statistics plus
 *     recomputation for the backward.
 *
 * Conventions shared by every entry point
 *   Pointers: caller-owned DEVICE memory unless stated otherwise; the library
 *     allocates nothing and keeps no state between calls except the device
 *     status word (see attn_device_status).  16-byte alignment is required for
 *     q, k, v, o, dq, dk, dv, dout.
 *   Layouts (row-major, innermost last):
 *     q, o, dout, dq : [batch, n_q, h_q, d]
 *     k, v, dk, dv   : [batch, n_k, h_kv, d]
 *     lse            : [batch, h_q, n_q]  fp32, natural log, -inf for a row that
 *                      sees no key
 *     bias           : fp32 [h_q, n_q, n_k] for batch element b at
 *                      bias + b * bias_batch_stride (stride 0 = broadcast)
 *   dtype: ATTN_BF16 (bf16 inputs/outputs, fp32 accumulation, sm_100a tensor
 *     cores; d in {64, 128}) or ATTN_F32 (fp32 everywhere, CUDA cores; d in
 *     {64, 128}).
 *   Heads: h_q must be a multiple of h_kv; query head h reads KV head
 *     h / (h_q / h_kv) (MHA when equal, MQA when h_kv == 1).
 *   Causal: key j is visible from query i iff j <= i + (n_k - n_q).
 *   Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *   Return: ATTN_OK or a negative ATTN_ERR_* code; on an error code nothing
 *     was launched.
 */
#ifndef ATTN_H
#define ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ATTN_BF16 0
#define ATTN_F32 1

#define ATTN_OK 0
#define ATTN_ERR_INVALID (-1)     /* null pointer, bad size, h_q % h_kv != 0, misaligned */
#define ATTN_ERR_UNSUPPORTED (-2) /* d not in {64,128}, a sequence over 2^28 rows, over 65535 heads or
                                     batch elements, no sm_100 device */
#define ATTN_ERR_WORKSPACE (-3)   /* workspace missing or smaller than attn_bwd_workspace_size */
#define ATTN_ERR_CUDA (-4)        /* a CUDA runtime/driver call failed */
#define ATTN_ERR_TIMEOUT (-5)     /* a kernel gave up a bounded wait (device status word) */

/*
 * Forward.  Writes o (same dtype as q) and lse.  bias may be NULL.
 * scale: multiplier of Q K^T (1/sqrt(d) for the standard definition).
 * A bf16 forward with a bias reads it fastest when its rows are 16-byte
 * aligned (bias 16-byte aligned, n_k and bias_batch_stride multiples of 4):
 * its blocks are then staged in shared memory by TMA.  Any other bias is read
 * directly, with the same results.
 */
int attn_fwd(const void* q, const void* k, const void* v, const float* bias,
             long long bias_batch_stride, void* o, float* lse, int batch, int h_q, int h_kv,
             int n_q, int n_k, int d, float scale, int causal, int dtype, void* stream);

/*
 * Forward with the additive bias given by per-head ALiBi slopes instead of a
 * dense tensor: B[h, i, j] = -slope_h * |j - (i + n_k - n_q)|, formed in
 * registers (the slope-based position bias the grouped-query workload uses,
 * "Understanding FlashAttention Pt 1", 0.2 Notation: B an additive bias).
 * alibi_slopes: DEVICE fp32 [h_q] (required).  Otherwise as attn_fwd.
 */
int attn_fwd_alibi(const void* q, const void* k, const void* v, const float* alibi_slopes, void* o,
                   float* lse, int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale,
                   int causal, int dtype, void* stream);

/*
 * Bytes of device workspace attn_bwd needs: an fp32 dQ accumulator
 * [batch, n_q, h_q, d] plus the fp32 row terms D_i = dO_i . O_i [batch, h_q, n_q]
 * (each region 256-byte aligned).  Linear in n, never n^2.
 */
size_t attn_bwd_workspace_size(int batch, int h_q, int n_q, int d);

/*
 * Backward of attn_fwd.  Inputs: q, k, v, bias (same as the forward), the
 * forward's o and lse, and the upstream gradient dout.  Outputs dq, dk, dv in
 * the dtype and layout of q, k, v; dk/dv sum the h_q / h_kv query heads of a
 * group.  workspace: caller-owned device buffer of at least
 * attn_bwd_workspace_size(...) bytes (contents need not be initialised).
 */
int attn_bwd(const void* q, const void* k, const void* v, const float* bias,
             long long bias_batch_stride, const void* o, const float* lse, const void* dout,
             void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int batch,
             int h_q, int h_kv, int n_q, int n_k, int d, float scale, int causal, int dtype,
             void* stream);

/* Backward of attn_fwd_alibi (same slopes); otherwise as attn_bwd. */
int attn_bwd_alibi(const void* q, const void* k, const void* v, const float* alibi_slopes,
                   const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                   void* workspace, size_t workspace_bytes, int batch, int h_q, int h_kv, int n_q,
                   int n_k, int d, float scale, int causal, int dtype, void* stream);

/*
 * Local (sliding-window) attention, optionally with ALiBi slopes.  With
 * a = i + n_k - n_q the key aligned with query row i, key j is visible iff
 *   a - window_left <= j <= a + window_right;
 * a negative size leaves that side unbounded, and causal != 0 caps the right
 * side at a (window_right is then ignored).  The kernels load only the key
 * tiles that meet this band and mask only the tiles on its edges
 * ("Understanding FlashAttention Pt 1", contents 3.5 and 4.2: tile skipping,
 * local attention).  Rows with no visible key get O = 0, LSE = -inf.
 * alibi_slopes: DEVICE fp32 [h_q] or NULL (as attn_fwd_alibi).
 * Sizes must be at most 2^28 rows per sequence.  Otherwise as attn_fwd.
 */
int attn_fwd_local(const void* q, const void* k, const void* v, const float* alibi_slopes, void* o,
                   float* lse, int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale,
                   int causal, int window_left, int window_right, int dtype, void* stream);

/* Backward of attn_fwd_local (same slopes and window); otherwise as attn_bwd. */
int attn_bwd_local(const void* q, const void* k, const void* v, const float* alibi_slopes,
                   const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                   void* workspace, size_t workspace_bytes, int batch, int h_q, int h_kv, int n_q,
                   int n_k, int d, float scale, int causal, int window_left, int window_right,
                   int dtype, void* stream);

/*
 * Forward with a value width of its own ("Understanding FlashAttention Pt 1",
 * 0.2 Notation: V and O have d_v columns, Q and K have d): v is
 * [batch, n_k, h_kv, d_v] and o is [batch, n_q, h_q, d_v], d and d_v each in
 * {64, 128}.  d_v == d is attn_fwd without a bias; d_v != d takes bf16 only
 * (ATTN_ERR_UNSUPPORTED for fp32).  Otherwise as attn_fwd.
 */
int attn_fwd_dv(const void* q, const void* k, const void* v, void* o, float* lse, int batch,
                int h_q, int h_kv, int n_q, int n_k, int d, int d_v, float scale, int causal,
                int dtype, void* stream);

/*
 * Backward of attn_fwd_dv: v, o, dout, dv have width d_v, q, k, dq, dk width
 * d.  workspace: attn_bwd_workspace_size(batch, h_q, n_q, d) bytes (the dQ
 * accumulator has width d).  d_v == d is attn_bwd without a bias; d_v != d
 * takes bf16 only.  Otherwise as attn_bwd.
 */
int attn_bwd_dv(const void* q, const void* k, const void* v, const void* o, const float* lse,
                const void* dout, void* dq, void* dk, void* dv, void* workspace,
                size_t workspace_bytes, int batch, int h_q, int h_kv, int n_q, int n_k, int d,
                int d_v, float scale, int causal, int dtype, void* stream);

/*
 * Backward of attn_fwd_varlen (packed sequences, same layouts and offsets):
 * o, lse and dout as attn_fwd_varlen produced / consumed them; dq like q,
 * dk / dv like k / v.  workspace: DEVICE, 256-byte aligned,
 * attn_bwd_workspace_size(1, h_q, total_q, d) bytes.  Causal masking applies
 * inside each sequence; no bias.  Otherwise as attn_bwd.
 */
int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dout, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                    const int* cu_seqlens_k, int num_seqs, int max_seqlen_q, int max_seqlen_k,
                    int total_q, int total_k, int h_q, int h_kv, int d, float scale, int causal,
                    void* workspace, size_t workspace_bytes, int dtype, void* stream);

/*
 * Split-KV forward: the keys are cut into num_splits contiguous ranges (whole
 * 128-key tiles); each (query tile, head, batch, split) is an independent CTA
 * that writes the exact attention of its rows over its own keys (O_t fp32,
 * LSE_t) to the workspace, and attn_merge_partials' kernel combines them into
 * o (bf16) and lse.  The result is the same function as attn_fwd; it gives a
 * launch enough CTAs when batch x heads x query tiles is small against the
 * 148 SMs (short query blocks over long key sequences).  num_splits <= 0
 * takes attn_splitkv_num_splits' choice; splits that would be empty are
 * dropped.  bf16 only (ATTN_ERR_UNSUPPORTED for fp32); dense inputs, no bias.
 * workspace: DEVICE, 256-byte aligned, attn_splitkv_workspace_size(batch, h_q,
 * n_q, d, num_splits) bytes (not needed when one split results).
 */
int attn_splitkv_num_splits(int batch, int h_q, int n_q, int n_k);
size_t attn_splitkv_workspace_size(int batch, int h_q, int n_q, int d, int num_splits);
int attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int batch,
                     int h_q, int h_kv, int n_q, int n_k, int d, float scale, int causal,
                     int num_splits, void* workspace, size_t workspace_bytes, int dtype,
                     void* stream);

/*
 * Merge exact partial results over disjoint key ranges (split-KV, or keys
 * sharded across devices and gathered): with m = max_t LSE_t and
 * w_t = exp(LSE_t - m), O = sum_t w_t O_t / sum_t w_t and
 * LSE = m + ln sum_t w_t; rows whose LSE_t are all -inf get O = 0, LSE = -inf
 * ("Softmax does not need the matrix", "Carry the Normalizer": the carried
 * running state resumes the softmax exactly).
 * o_parts: DEVICE fp32 [num_parts, batch, n_q, h_q, d] (each O_t normalised);
 * lse_parts: DEVICE fp32 [num_parts, batch, h_q, n_q]; o: DEVICE
 * [batch, n_q, h_q, d] of out_dtype (ATTN_BF16 or ATTN_F32); lse: DEVICE fp32
 * [batch, h_q, n_q].  d in {64, 128}.
 */
int attn_merge_partials(const float* o_parts, const float* lse_parts, int num_parts, void* o,
                        float* lse, int batch, int h_q, int n_q, int d, int out_dtype, void* stream);

/*
 * Partial forward over one block of keys: the exact attention of every query
 * row over the keys given here only, left unmerged for attn_merge_partials --
 * o_part: DEVICE fp32 [batch, n_q, h_q, d], O_t normalised over this block;
 * lse_part: DEVICE fp32 [batch, h_q, n_q], LSE_t over this block (-inf, with
 * O_t = 0, for a row that sees none of its keys).  Causal masking aligns the
 * block bottom-right (key j visible from row i iff j <= i + n_k - n_q), which
 * for n_q == n_k is the diagonal block of a sequence cut into equal chunks.
 * This is the per-shard step when the keys of a sequence are spread over
 * devices: each device attends to the key blocks it holds or receives and the
 * partials merge exactly ("Softmax does not need the matrix", "Carry the
 * Normalizer": the carried state resumes the softmax over the next block).
 * bf16 inputs only (ATTN_ERR_UNSUPPORTED for fp32); no bias.  Otherwise as
 * attn_fwd.
 */
int attn_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part,
                     int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale, int causal,
                     int dtype, void* stream);

/*
 * FP8 forward ("Understanding FlashAttention Pt 1", contents 5.6: FP8 buys
 * speed at a stated cost in precision).  Q and K are first quantised per
 * (batch, head) by attn_quantize_e4m3; S = Q8 K8^T then runs on the e4m3
 * tensor cores (fp32 accumulation) and is rescaled by q_scale * k_scale, while
 * P V stays in bf16.  The result is the exact attention of the dequantised
 * inputs Q8 * q_scale, K8 * k_scale and V, to the bf16 tolerances of attn_fwd.
 *
 * attn_quantize_e4m3: x bf16 [batch, n, heads, d] (d in {64, 128}) ->
 *   scales fp32 [batch, heads], scale = amax / 448 over that (batch, head)
 *   (fp32 division; 1 when the head is all zeros), and x8 e4m3 bytes of the
 *   same layout, x8 = e4m3(x / scale) with the quotient in fp32 (IEEE
 *   division), rounded to nearest even and saturated at +-448.  x8 and x
 *   16-byte aligned.
 * attn_fwd_fp8: q8 [batch, n_q, h_q, d], k8 [batch, n_k, h_kv, d] (e4m3 bytes),
 *   their scales [batch, h_q] / [batch, h_kv], v bf16 [batch, n_k, h_kv, d];
 *   o bf16 and lse as attn_fwd.  d = 128, scale > 0, no bias (otherwise
 *   ATTN_ERR_UNSUPPORTED).
 */
int attn_quantize_e4m3(const void* x, void* x8, float* scales, int batch, int n, int heads, int d,
                       void* stream);
int attn_fwd_fp8(const void* q8, const float* q_scales, const void* k8, const float* k_scales,
                 const void* v, void* o, float* lse, int batch, int h_q, int h_kv, int n_q, int n_k,
                 int d, float scale, int causal, void* stream);

/*
 * attn_bwd without a workspace argument, for callers that cannot allocate
 * device memory when they run the backward (code inside a framework that owns
 * all device memory, or latency-critical loops that cannot afford cudaMalloc's
 * implicit synchronisation).  The pages have no counterpart of this entry
 * point; it exists for those callers only.
 *
 * Arguments, layouts and results are attn_bwd's.  The scratch comes from a
 * fixed array inside the library (ATTN_NOALLOC_SCRATCH_BYTES per device, held
 * by every GPU that loads the library until the process exits); nothing is
 * allocated.  Returns ATTN_ERR_WORKSPACE when attn_bwd_workspace_size(batch,
 * h_q, n_q, d) exceeds ATTN_NOALLOC_SCRATCH_BYTES.  All calls on a device share
 * the array: calls that overlap on the GPU race.  The first call on a device
 * looks up the array's address with that device current and keeps it for the
 * life of the process; make it before any stream capture.  A device reset
 * (cudaDeviceReset) after that first call is not supported: the array may then
 * sit at another address.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int attn_bwd_noalloc(const void* q, const void* k, const void* v, const float* bias,
                     long long bias_batch_stride, const void* o, const float* lse,
                     const void* dout, void* dq, void* dk, void* dv, int batch, int h_q,
                     int h_kv, int n_q, int n_k, int d, float scale, int causal, int dtype,
                     void* stream);

/*
 * Packed variable-length forward.  q: [total_q, h_q, d], k/v: [total_k, h_kv, d],
 * o like q, lse: [h_q, total_q].  cu_seqlens_q / cu_seqlens_k: DEVICE int32
 * arrays of num_seqs + 1 non-decreasing prefix offsets starting at 0; sequence z
 * owns rows cu[z] .. cu[z+1]-1.  max_seqlen_q / max_seqlen_k bound the lengths
 * (they size the launch).  Causal masking applies inside each sequence.  No bias.
 * The offsets live in device memory and are not read on the host; the kernels
 * check them before any access: a sequence whose offsets are negative,
 * decrease, exceed total_q / total_k, or give a length above max_seqlen_q /
 * max_seqlen_k is neither read nor written, and ATTN_ERR_INVALID is raised in
 * the device status word (attn_device_status); the other sequences are
 * computed, and that sequence's outputs are left as they were.
 */
int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                    int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int h_q,
                    int h_kv, int d, float scale, int causal, int dtype, void* stream);

/*
 * Deliberately naive materialising forward, for measurement only (the
 * three-step "standard attention" the pages contrast with: write S to device
 * memory, read it back for the row softmax and write P, read P for P V).
 * s_scratch: fp32 [n_q, n_k], p_scratch: bf16 [n_q, n_k], both caller-owned
 * device buffers reused for every (batch, head).  bf16 only, no bias.
 */
size_t attn_naive_scratch_size(int n_q, int n_k);
int attn_fwd_naive(const void* q, const void* k, const void* v, void* o, float* lse,
                   void* scratch, size_t scratch_bytes, int batch, int h_q, int h_kv, int n_q,
                   int n_k, int d, float scale, int causal, void* stream);

/* Human-readable text for an ATTN_* code (static storage). */
const char* attn_strerror(int code);

/*
 * Synchronises `stream`, then returns and clears the device status word of the
 * current device: ATTN_OK; ATTN_ERR_TIMEOUT if a kernel launched since the
 * last call abandoned a bounded wait (its outputs are then undefined); or
 * ATTN_ERR_INVALID if a packed-sequence kernel met invalid offsets (that
 * sequence was skipped).
 */
int attn_device_status(void* stream);

/*
 * Self-test of the failure path: launches one warp that waits on a barrier
 * nothing arrives on and gives up after limit_cycles SM cycles (1000 ..
 * 2e9), exactly as every kernel's bounded waits do; the next
 * attn_device_status then returns ATTN_ERR_TIMEOUT and the context stays
 * usable.  No fault, no hang.
 */
int attn_selftest_wait_timeout(long long limit_cycles, void* stream);

/*
 * Self-test of the FMA-pipe exponential that the tensor-core kernels use for a
 * share of their exponentials instead of the MUFU unit: y[i] = 2^x[i] for
 * x[i] <= 0, by Cody-Waite range reduction (x = n + f, |f| <= 1/2) and a
 * degree-3 polynomial for 2^f of least maximum relative error (Remez fit),
 * relative error below 7.6e-5 -- well under the 2^-9 resolution of the bf16
 * probabilities it feeds.  Inputs below -125 (including -inf) give 2^-125 up
 * to that error; inputs above 0 are outside its domain.  x, y: DEVICE fp32
 * [n], caller-owned, n >= 0.  Asynchronous on `stream`.
 */
int attn_selftest_ex2(const float* x, float* y, long long n, void* stream);

/*
 * Kernel launches issued by this library on the calling host thread since the
 * last reset (reset = 1 clears after reading).  Lets callers count the GPU
 * work of a timed region.
 */
long long attn_launch_count(int reset);

/*
 * Measurement hook.  Until cleared, every launch of kernel `which`
 * (ATTN_KERNEL_FWD: the tensor-core forward kernel; ATTN_KERNEL_BWD: the
 * tensor-core backward main kernel) issued from the calling host thread is
 * bracketed by cudaEventRecord(start) / cudaEventRecord(stop) on the launch
 * stream.  start/stop are caller-owned cudaEvent_t handles; pass NULL for both
 * to clear.  Returns ATTN_ERR_INVALID for an unknown `which`.
 */
#define ATTN_KERNEL_FWD 0
#define ATTN_KERNEL_BWD 1
int attn_set_kernel_events(int which, void* start, void* stop);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H */
