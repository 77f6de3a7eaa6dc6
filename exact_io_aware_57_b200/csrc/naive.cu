// Deliberately naive, materialising attention forward -- a measurement
// comparator only.  It follows the three-step "standard attention" the pages
// set against the tiled method ("Understanding FlashAttention Pt 1", 0.1 and
// 1.2; "FlashAttention" (Triptych day 39), paragraph on the standard
// implementation): every score goes to device memory and comes back.
//   K1  S = scale * Q K^T (causal: -inf above the diagonal) -> fp32 [Nq, Nk]
//   K2  one CTA per row: read the S row once, P = softmax(S) -> bf16 [Nq, Nk],
//       LSE = m + ln l
//   K3  O = P V -> bf16
// Per (batch, head) the scratch S and P are rewritten, so the extra device
// traffic is 4 + 4 + 2 + 2 = 12 bytes per (query, key) pair.  CUDA-core
// arithmetic; only its bytes are of interest.
#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

constexpr int T = 64;  // output tile edge of K1 / rows per CTA of K3

// K1: 16x16 threads, each a 4x4 block of a 64x64 score tile.
template <int D>
__global__ void __launch_bounds__(256) naive_scores(const __nv_bfloat16* __restrict__ q,
                                                    const __nv_bfloat16* __restrict__ k, float* __restrict__ S,
                                                    int Nq, int Nk, int Hq, int Hkv, int b, int h, float scale,
                                                    int causal) {
  __shared__ __nv_bfloat16 qs[T][D + 8], ks[T][D + 8];
  const int hk = h / (Hq / Hkv);
  const int i0 = blockIdx.y * T, j0 = blockIdx.x * T;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  for (int e = threadIdx.x; e < T * D / 8; e += 256) {
    const int r = e / (D / 8), c8 = (e % (D / 8)) * 8;
    uint4 zq = make_uint4(0, 0, 0, 0), zk = zq;
    if (i0 + r < Nq) zq = *reinterpret_cast<const uint4*>(q + (((long long)b * Nq + i0 + r) * Hq + h) * D + c8);
    if (j0 + r < Nk) zk = *reinterpret_cast<const uint4*>(k + (((long long)b * Nk + j0 + r) * Hkv + hk) * D + c8);
    *reinterpret_cast<uint4*>(&qs[r][c8]) = zq;
    *reinterpret_cast<uint4*>(&ks[r][c8]) = zk;
  }
  __syncthreads();
  float acc[4][4] = {};
  for (int c = 0; c < D; ++c) {
    float a[4], bb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      a[u] = __bfloat162float(qs[ty * 4 + u][c]);
      bb[u] = __bfloat162float(ks[tx * 4 + u][c]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], bb[w], acc[u][w]);
  }
  const int diag = Nk - Nq;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    if (i >= Nq) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = j0 + tx * 4 + w;
      if (j >= Nk) continue;
      S[(long long)i * Nk + j] = (causal && j > i + diag) ? -INFINITY : acc[u][w] * scale;
    }
  }
}

// K2: one CTA per row; the row is read from device memory once into shared memory.
__global__ void __launch_bounds__(256) naive_softmax(const float* __restrict__ S, __nv_bfloat16* __restrict__ P,
                                                     float* __restrict__ lse, long long lse_off, int Nk) {
  extern __shared__ float row[];
  __shared__ float red[32];
  const int i = blockIdx.x;
  const float* src = S + (long long)i * Nk;
  float m = -INFINITY;
  for (int j = threadIdx.x; j < Nk; j += 256) {
    const float x = src[j];
    row[j] = x;
    m = fmaxf(m, x);
  }
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = -INFINITY;
  for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  const float mu = m == -INFINITY ? 0.f : m;
  float l = 0.f;
  for (int j = threadIdx.x; j < Nk; j += 256) l += expf(row[j] - mu);
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = l;
  __syncthreads();
  l = 0.f;
  for (int w = 0; w < 8; ++w) l += red[w];
  const float inv = l > 0.f ? 1.f / l : 0.f;
  __nv_bfloat16* dst = P + (long long)i * Nk;
  for (int j = threadIdx.x; j < Nk; j += 256) dst[j] = __float2bfloat16_rn(expf(row[j] - mu) * inv);
  if (threadIdx.x == 0) lse[lse_off + i] = l > 0.f ? mu + logf(l) : -INFINITY;
}

// K3: O rows [64 per CTA] = P V; 16x16 threads, each 4 rows x D/16 columns.
template <int D>
__global__ void __launch_bounds__(256) naive_pv(const __nv_bfloat16* __restrict__ P, const __nv_bfloat16* __restrict__ v,
                                                __nv_bfloat16* __restrict__ o, int Nq, int Nk, int Hq, int Hkv, int b,
                                                int h) {
  constexpr int CW = D / 16;
  __shared__ __nv_bfloat16 ps[T][T + 8], vs[T][D + 8];
  const int hk = h / (Hq / Hkv);
  const int i0 = blockIdx.x * T;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][CW] = {};
  for (int j0 = 0; j0 < Nk; j0 += T) {
    for (int e = threadIdx.x; e < T * T; e += 256) {
      const int r = e / T, c = e % T;
      ps[r][c] = (i0 + r < Nq && j0 + c < Nk) ? P[(long long)(i0 + r) * Nk + j0 + c] : __float2bfloat16_rn(0.f);
    }
    for (int e = threadIdx.x; e < T * D; e += 256) {
      const int r = e / D, c = e % D;
      vs[r][c] = (j0 + r < Nk) ? v[(((long long)b * Nk + j0 + r) * Hkv + hk) * D + c] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    for (int j = 0; j < T; ++j) {
      float pv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) pv[u] = __bfloat162float(ps[ty * 4 + u][j]);
#pragma unroll
      for (int w = 0; w < CW; ++w) {
        const float vv = __bfloat162float(vs[j][tx + 16 * w]);
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[u][w] = fmaf(pv[u], vv, acc[u][w]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    if (i >= Nq) continue;
#pragma unroll
    for (int w = 0; w < CW; ++w)
      o[(((long long)b * Nq + i) * Hq + h) * D + tx + 16 * w] = __float2bfloat16_rn(acc[u][w]);
  }
}

}  // namespace

int launch_fwd_naive(const TcGeom& g, __nv_bfloat16* o, float* lse, float* s_scratch, __nv_bfloat16* p_scratch,
                     cudaStream_t st) {
  const size_t row_smem = (size_t)g.Nk * sizeof(float);
  if (row_smem > 200 * 1024) return ATTN_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(naive_softmax, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)row_smem) != cudaSuccess)
    return ATTN_ERR_CUDA;
  const auto* q = static_cast<const __nv_bfloat16*>(g.q);
  const auto* k = static_cast<const __nv_bfloat16*>(g.k);
  const auto* v = static_cast<const __nv_bfloat16*>(g.v);
  const dim3 g1((g.Nk + T - 1) / T, (g.Nq + T - 1) / T);
  for (int b = 0; b < g.B; ++b) {
    for (int h = 0; h < g.Hq; ++h) {
      if (g.D == 64)
        naive_scores<64><<<g1, 256, 0, st>>>(q, k, s_scratch, g.Nq, g.Nk, g.Hq, g.Hkv, b, h, g.scale, g.causal);
      else
        naive_scores<128><<<g1, 256, 0, st>>>(q, k, s_scratch, g.Nq, g.Nk, g.Hq, g.Hkv, b, h, g.scale, g.causal);
      naive_softmax<<<g.Nq, 256, row_smem, st>>>(s_scratch, p_scratch, lse, ((long long)b * g.Hq + h) * g.Nq, g.Nk);
      if (g.D == 64)
        naive_pv<64><<<(g.Nq + T - 1) / T, 256, 0, st>>>(p_scratch, v, o, g.Nq, g.Nk, g.Hq, g.Hkv, b, h);
      else
        naive_pv<128><<<(g.Nq + T - 1) / T, 256, 0, st>>>(p_scratch, v, o, g.Nq, g.Nk, g.Hq, g.Hkv, b, h);
      count_launch(3);
      if (cudaGetLastError() != cudaSuccess) return ATTN_ERR_CUDA;
    }
  }
  return ATTN_OK;
}

}  // namespace attn
