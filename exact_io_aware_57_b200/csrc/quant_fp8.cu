// Per-head e4m3 quantisation of Q or K for the FP8 forward ("Understanding
// FlashAttention Pt 1", contents 5.6: FP8 attention trades precision for
// throughput, so the scale and rounding are stated exactly here).
//
// For every (batch b, head h) of x [B, N, H, d] (bf16):
//   amax = max |x[b, :, h, :]|,  scale = amax / 448 (fp32; 1 when amax = 0),
//   x8 = e4m3(x / scale)  -- the quotient in fp32 (IEEE division), rounded to
//        nearest-even e4m3 and saturated at +-448 --
// so that x8 * scale reproduces x to within e4m3's relative step 2^-4.
// Launches: zero the amax slots, per-block |x| maxima folded with atomicMax on
// the float bits (non-negative floats order like their bit patterns), the
// conversion, and amax -> scale in place.  All HBM-bound and small.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

constexpr int kRowsPerBlock = 256;

// One block per (row chunk, head, batch): 16 rows at a time, 16 threads per row
// reading d/16 bf16 each (d = 64 or 128: 8 bytes or 16 bytes per thread).
template <int D>
__global__ void __launch_bounds__(256) amax_kernel(const __nv_bfloat16* __restrict__ x, unsigned* __restrict__ amax,
                                                   int N, int H) {
  constexpr int E = D / 16;
  const int h = blockIdx.y, b = blockIdx.z;
  const int r0 = blockIdx.x * kRowsPerBlock;
  const int sub = threadIdx.x >> 4, part = threadIdx.x & 15;
  float mx = 0.f;
  for (int r = r0 + sub; r < min(N, r0 + kRowsPerBlock); r += 16) {
    const __nv_bfloat16* src = x + (((long long)b * N + r) * H + h) * D + part * E;
#pragma unroll
    for (int e = 0; e < E; ++e) mx = fmaxf(mx, fabsf(__bfloat162float(src[e])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = red[0];
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
    atomicMax(amax + b * H + h, __float_as_uint(m));
  }
}

ATTN_DEVINL float scale_of(unsigned amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a > 0.f ? __fdiv_rn(a, 448.f) : 1.f;
}

// 8 elements per thread; the row's (batch, head) fixes the scale.
__global__ void __launch_bounds__(256) quant_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ x8,
                                                    const unsigned* __restrict__ amax, long long n8, int N, int H,
                                                    int D) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const long long row = i * 8 / D;  // (b * N + n) * H + h
  const int h = (int)(row % H);
  const int b = (int)(row / ((long long)N * H));
  const float sc = scale_of(__ldg(amax + b * H + h));
  const uint4 raw = reinterpret_cast<const uint4*>(x)[i];
  const __nv_bfloat16* v = reinterpret_cast<const __nv_bfloat16*>(&raw);
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float qv = __fdiv_rn(__bfloat162float(v[e]), sc);
    const uint32_t code = __nv_cvt_float_to_fp8(qv, __NV_SATFINITE, __NV_E4M3);
    out[e >> 2] |= code << (8 * (e & 3));
  }
  reinterpret_cast<uint2*>(x8)[i] = make_uint2(out[0], out[1]);
}

__global__ void scales_kernel(float* __restrict__ s, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) s[i] = scale_of(__float_as_uint(s[i]));
}

}  // namespace

int launch_quantize_e4m3(const __nv_bfloat16* x, uint8_t* x8, float* scales, int B, int N, int H, int D,
                         cudaStream_t st) {
  unsigned* amax = reinterpret_cast<unsigned*>(scales);  // amax bits first, scales at the end
  if (cudaMemsetAsync(amax, 0, sizeof(float) * (size_t)B * H, st) != cudaSuccess) return ATTN_ERR_CUDA;
  dim3 g1((N + kRowsPerBlock - 1) / kRowsPerBlock, H, B);
  if (D == 64)
    amax_kernel<64><<<g1, 256, 0, st>>>(x, amax, N, H);
  else
    amax_kernel<128><<<g1, 256, 0, st>>>(x, amax, N, H);
  const long long n8 = (long long)B * N * H * D / 8;
  quant_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(x, x8, amax, n8, N, H, D);
  scales_kernel<<<(B * H + 255) / 256, 256, 0, st>>>(scales, B * H);
  count_launch(3);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
