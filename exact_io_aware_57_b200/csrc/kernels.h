// Host-side interface between the C-ABI layer (attn_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/attn.h"

namespace attn {

// Launch accounting (per host thread), read by attn_launch_count.
void count_launch(int n = 1);

// Events recorded around the main forward / backward kernel (measurement hook).
void record_kernel_event(int which, int stop, cudaStream_t st);

// Default bound on any single in-kernel wait, in SM clock cycles (~1 s).
constexpr long long kWaitLimitCycles = 2000000000LL;

// Device address of the library's status word on the current device.
int* device_status_ptr();
// Streaming multiprocessors of the current device (1 if the query fails).
int sm_count();

// ----------------------------------------------------------------- fp32 path
// Key visibility.  With a = i + Nk - Nq the key aligned with query row i, key j
// is visible iff a - win_l <= j <= a + win_r.  kWinNone marks an unbounded side;
// causal is the right side capped at 0.  Sequence lengths are limited to
// kMaxSeqLen so that a + kWinNone + 1 and a - kWinNone stay inside int.
constexpr int kWinNone = 1 << 30;
constexpr int kMaxSeqLen = 1 << 28;
inline int win_left(int window_left) {
  return (window_left < 0 || window_left >= kWinNone) ? kWinNone : window_left;
}
inline int win_right(int causal, int window_right) {
  if (causal) return 0;
  return (window_right < 0 || window_right >= kWinNone) ? kWinNone : window_right;
}

struct F32Params {
  const float *q, *k, *v, *bias, *alibi;
  float *o, *lse;
  const int *cu_q, *cu_k;   // packed sequences (device) or null
  long long q_bstride, k_bstride, bias_bstride, lse_bstride, lse_hstride;
  int Hq, Hkv, Nq, Nk, D, causal;
  int window_left = -1, window_right = -1;  // local attention sizes; negative: unbounded
  int win_l = kWinNone, win_r = kWinNone;  // folded from causal and the sizes by the launchers
  float scale;
  int max_nq = 0, max_nk = 0;  // packed: bounds on the sequence lengths (set by the launchers)
  int* status = nullptr;       // device status word (set by the launchers)
};

int launch_fwd_f32(const F32Params& p, int num_z, int max_nq, cudaStream_t st);
int launch_bwd_f32(const F32Params& p, const float* dout, const float* Drow, float* dq, float* dk, float* dv,
                   int num_z, int max_nq, int max_nk, cudaStream_t st);
template <typename T>
int launch_rowdot(const T* o, const T* dout, float* Drow, int B, int Hq, int Nq, int D, cudaStream_t st);

// ------------------------------------------------------- bf16 sm_100a path
// Geometry common to the tensor-core kernels.  Dense inputs use batch = B and
// per-batch lengths Nq/Nk; packed inputs use batch = 1, rows = totals, and
// per-sequence offsets from cu_q/cu_k.
struct TcGeom {
  const void *q, *k, *v;
  int B, Hq, Hkv, Nq, Nk, D;   // Nq/Nk: rows per batch element (totals when packed)
  const int *cu_q, *cu_k;      // null for dense
  int num_seqs, max_nq, max_nk;
  int causal;
  float scale;
  const float* bias;
  long long bias_bstride;
  const float* alibi;          // per-query-head ALiBi slopes (device) or null
  int window_left = -1, window_right = -1;  // local attention sizes; negative: unbounded
  int Dv = 0;                  // width of V and O when it differs from D (forward only), else 0
};

// Split-KV forward: keys cut into num_splits ranges of split_len (a multiple of
// 128); each writes O_t (fp32, normalised) and LSE_t for the merge.
struct SplitKV {
  int num_splits, split_len;
  float* o_part;    // [num_splits, B, Nq, Hq, D]
  float* lse_part;  // [num_splits, B, Hq, Nq]
};
// Parameters of the tensor-core forward kernels (built by launch_fwd_sm100).
struct FwdParams {
  __nv_bfloat16* o;
  float* lse;
  const float* bias;
  long long bias_bstride;
  int bias_vec4;       // dense bias rows 16-byte aligned: whole key tiles read as float4
  int batch_inner;     // grid (batch, row block, head): the batch elements sharing one bias run together
  const float* alibi;  // per-query-head slopes (BIAS == kBiasAlibi)
  const int* cu_q;
  const int* cu_k;
  int max_nq, max_nk;  // packed: bounds on the sequence lengths
  int Hq, Hkv, Nq, Nk;
  long long o_bstride, lse_bstride, lse_hstride;
  float scale_log2;
  int causal;
  int win_l, win_r;  // key j visible from row i iff i + diag - win_l <= j <= i + diag + win_r
  int num_splits, split_len;           // split-KV (1, unused: one split)
  float* o_part;                       // [num_splits, B, Nq, Hq, D] fp32, or null: O in bf16 to o
  float* lse_part;                     // [num_splits, B, Hq, Nq]
  long long part_o_stride, part_lse_stride;
  const float* q_scale;  // FP8 forward: per-(batch, head) e4m3 scales of Q [B, Hq] and K [B, Hkv]
  const float* k_scale;
  int* status;
  long long wait_limit;
  // Two-tile forward, dense grid (set by its launcher): grid_nblk row blocks of
  // 256 rows x grid_nu (batch, head) pairs.  Units from half_from on (in launch
  // order) are split into their two 128-row tiles, one CTA each, so that a last
  // wave that would leave SMs idle runs single tiles instead (a 1-D grid).
  int grid_nblk, grid_nu, half_from;
};

// Forward with two 128-row query tiles per CTA whose softmax warpgroups
// alternate on the tensor pipe (fwd_pp_sm100.cu).  fast: no bias and a
// positive scale (the row max may be taken on raw scores); partial: split-KV
// partials to p.o_part / p.lse_part.
int launch_fwd_pp(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const FwdParams& p, int bias_kind, bool fast, bool partial, cudaStream_t st);
// Forward with a dense bias: 64-key tiles and double-buffered scores
// (fwd_db_sm100.cu); K and V maps with 64-row boxes.  Dense batches, d = d_v.
int launch_fwd_db(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                  const FwdParams& p, cudaStream_t st);
// The same kernel with e4m3 Q/K tiles (maps over the quantised tensors).
int launch_fwd_pp_fp8(const TcGeom& g, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const FwdParams& p, cudaStream_t st);
// FwdParams of a forward launch (everything but the tensor maps).
int fwd_params(const TcGeom& g, __nv_bfloat16* o, float* lse, const SplitKV* split, FwdParams& p);

// Per-(batch, head) e4m3 quantisation of x [B, N, H, D] (bf16): scales[b, h] =
// amax / 448 (1 when amax = 0), x8 = e4m3(x / scale) (fp32 quotient, RNE, saturated).
int launch_quantize_e4m3(const __nv_bfloat16* x, uint8_t* x8, float* scales, int B, int N, int H, int D,
                         cudaStream_t st);
// FP8 forward: S = Q8 K8^T on e4m3 tensor cores, scaled by q_scale * k_scale;
// P V in bf16.  Dense inputs, D = DV = 128, no bias, positive scale.
int launch_fwd_fp8(const TcGeom& g, const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                   __nv_bfloat16* o, float* lse, cudaStream_t st);

int launch_fwd_sm100(const TcGeom& g, __nv_bfloat16* o, float* lse, cudaStream_t st, const SplitKV* split = nullptr);
// O = sum_t exp(LSE_t - LSE) O_t, LSE = log sum_t exp(LSE_t) over num_parts
// partials laid out as SplitKV's; o: bf16 (out_f32 = 0) or fp32 [B, Nq, Hq, D].
int launch_merge(const float* o_part, const float* lse_part, int num_parts, void* o, float* lse, int B, int Hq,
                 int Nq, int D, int out_f32, cudaStream_t st);
int launch_bwd_sm100(const TcGeom& g, const __nv_bfloat16* o, const float* lse, const __nv_bfloat16* dout,
                     __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, float* dq_acc, float* Drow,
                     cudaStream_t st);
int launch_fwd_naive(const TcGeom& g, __nv_bfloat16* o, float* lse, float* s_scratch, __nv_bfloat16* p_scratch,
                     cudaStream_t st);

// One warp that waits on a barrier nothing arrives on, giving up after
// limit_cycles (the shared bounded-wait failure path).
int launch_wait_selftest(long long limit_cycles, cudaStream_t st);
int launch_ex2_selftest(const float* x, float* y, long long n, cudaStream_t st);

// Tensor-map encoding (driver entry point resolved at run time).
int encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box);
int encode_tmap(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int rank, const uint64_t* dims,
                const uint64_t* strides_bytes, const uint32_t* box);

}  // namespace attn
