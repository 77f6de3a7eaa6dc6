// Merge of exact partial results over disjoint key ranges (split-KV, or keys
// sharded over devices): partial t holds the attention of each row over its
// own keys only, O_t (normalised, fp32) and LSE_t.  The combined row follows
// from the rescale-and-add merge of the running softmax state ("Softmax does
// not need the matrix", "Carry the Normalizer": the carried (m, l, a) state
// suffices to resume the softmax exactly), applied to whole partials:
//   m = max_t LSE_t,  w_t = exp(LSE_t - m),  O = sum_t w_t O_t / sum_t w_t,
//   LSE = m + ln sum_t w_t;  rows with every LSE_t = -inf give O = 0, LSE = -inf.
// HBM-bound: one warp per output row reads num_parts * D * 4 bytes.
#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

template <int D, bool OUT_F32>
__global__ void __launch_bounds__(256) merge_kernel(const float* __restrict__ o_part,
                                                    const float* __restrict__ lse_part, int T, long long o_stride,
                                                    long long lse_stride, void* __restrict__ o,
                                                    float* __restrict__ lse, int B, int Hq, int Nq) {
  constexpr int E = D / 32;  // floats per lane (2 or 4)
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);  // ((b * Nq + i) * Hq + h)
  const int lane = threadIdx.x & 31;
  if (row >= (long long)B * Nq * Hq) return;
  const int h = (int)(row % Hq);
  const long long bi = row / Hq;
  const int i = (int)(bi % Nq), b = (int)(bi / Nq);
  const long long li = ((long long)b * Hq + h) * Nq + i;
  float m = -INFINITY;
  for (int t = 0; t < T; ++t) m = fmaxf(m, __ldg(lse_part + t * lse_stride + li));
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float l = 0.f;
  if (m != -INFINITY) {
    for (int t = 0; t < T; ++t) {
      const float w = expf(__ldg(lse_part + t * lse_stride + li) - m);
      l += w;
      const float* src = o_part + t * o_stride + row * D + lane * E;
      if constexpr (E == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(src));
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]);
        acc[3] = fmaf(w, v.w, acc[3]);
      } else {
        const float2 v = __ldg(reinterpret_cast<const float2*>(src));
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
      }
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  if constexpr (OUT_F32) {
    float* dst = static_cast<float*>(o) + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) dst[e] = acc[e] * inv;
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(o) + row * D + lane * E;
    if constexpr (E == 4) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv));
    } else {
      *reinterpret_cast<uint32_t*>(dst) = pack_bf16(acc[0] * inv, acc[1] * inv);
    }
  }
  if (lane == 0) lse[li] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

int launch_merge(const float* o_part, const float* lse_part, int num_parts, void* o, float* lse, int B, int Hq,
                 int Nq, int D, int out_f32, cudaStream_t st) {
  const long long rows = (long long)B * Nq * Hq;
  const long long o_stride = rows * D, lse_stride = rows;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (D == 64) {
    if (out_f32)
      merge_kernel<64, true><<<blocks, 256, 0, st>>>(o_part, lse_part, num_parts, o_stride, lse_stride, o, lse, B, Hq, Nq);
    else
      merge_kernel<64, false><<<blocks, 256, 0, st>>>(o_part, lse_part, num_parts, o_stride, lse_stride, o, lse, B, Hq, Nq);
  } else {
    if (out_f32)
      merge_kernel<128, true><<<blocks, 256, 0, st>>>(o_part, lse_part, num_parts, o_stride, lse_stride, o, lse, B, Hq, Nq);
    else
      merge_kernel<128, false><<<blocks, 256, 0, st>>>(o_part, lse_part, num_parts, o_stride, lse_stride, o, lse, B, Hq, Nq);
  }
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
