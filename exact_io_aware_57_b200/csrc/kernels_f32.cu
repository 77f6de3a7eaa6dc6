// fp32 attention on CUDA cores (the fp32 workload: tensor-core tf32 cannot
// hold a 1e-4 max-abs error).  One warp per query row (forward, dQ) or per key
// row (dK/dV); lane c owns elements c, c+32, ... of the head dimension.  The
// forward carries the online-softmax state (m, l, a) exactly as in
// "Softmax does not need the matrix", "Carry the Normalizer", one key at a time;
// the backward recomputes P_ij = exp(s_ij - LSE_i) from the stored LSE.
#include "common.cuh"
#include "kernels.h"

namespace attn {

namespace {

ATTN_DEVINL float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Sequence geometry of one (batch or packed sequence) index z.
// ok is false for a packed sequence with invalid offsets (reported in the
// status word); the kernels then leave before touching any row.
struct Seq {
  int b, q0, nq, k0, nk;
  bool ok;
};

ATTN_DEVINL Seq seq_of(const F32Params& p, int z) {
  Seq s;
  s.ok = true;
  if (p.cu_q) {
    s.b = 0;
    s.ok = packed_seq(p.cu_q, z, p.Nq, p.max_nq, p.status, s.q0, s.nq) &&
           packed_seq(p.cu_k, z, p.Nk, p.max_nk, p.status, s.k0, s.nk);
    if (!s.ok) s.nq = s.nk = 0;
  } else {
    s.b = z;
    s.q0 = 0;
    s.nq = p.Nq;
    s.k0 = 0;
    s.nk = p.Nk;
  }
  return s;
}

// Keys lo .. end-1 are visible from row i: with a = i + nk - nq (bottom-right
// alignment), a - win_l <= j <= a + win_r (causal: win_r = 0).
struct KeyRange {
  int lo, end;
};
ATTN_DEVINL KeyRange visible(const F32Params& p, const Seq& s, int i) {
  const int a = i + (s.nk - s.nq);
  KeyRange r;
  r.lo = max(0, a - p.win_l);
  r.end = min(s.nk, a + p.win_r + 1);
  if (r.end < r.lo) r.end = r.lo;
  return r;
}

template <int D>
__global__ void __launch_bounds__(128) fwd_f32_kernel(F32Params p) {
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const Seq s = seq_of(p, blockIdx.z);
  const int i = blockIdx.x * 4 + warp;
  if (i >= s.nq) return;
  const int hk = h / (p.Hq / p.Hkv);
  const float* qrow = p.q + s.b * p.q_bstride + ((long long)(s.q0 + i) * p.Hq + h) * D;
  float qv[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = qrow[lane + 32 * e];
    acc[e] = 0.f;
  }
  const float* brow = p.bias ? p.bias + s.b * p.bias_bstride + ((long long)h * s.nq + i) * s.nk : nullptr;
  const float slope = p.alibi ? p.alibi[h] : 0.f;
  const KeyRange kr = visible(p, s, i);
  float m = -INFINITY, l = 0.f;
  for (int j = kr.lo; j < kr.end; ++j) {
    const long long kv = s.b * p.k_bstride + ((long long)(s.k0 + j) * p.Hkv + hk) * D;
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) dot = fmaf(qv[e], p.k[kv + lane + 32 * e], dot);
    float sc = warp_sum(dot) * p.scale;
    if (brow) sc += brow[j];
    if (p.alibi) sc -= slope * fabsf(static_cast<float>(j - i - (s.nk - s.nq)));
    const float mn = fmaxf(m, sc);
    if (mn == -INFINITY) continue;
    const float alpha = expf(m - mn);
    const float pj = expf(sc - mn);
    l = l * alpha + pj;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(acc[e], alpha, pj * p.v[kv + lane + 32 * e]);
    m = mn;
  }
  float* orow = p.o + s.b * p.q_bstride + ((long long)(s.q0 + i) * p.Hq + h) * D;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) orow[lane + 32 * e] = acc[e] * inv;
  if (lane == 0)
    p.lse[s.b * p.lse_bstride + (long long)h * p.lse_hstride + s.q0 + i] = l > 0.f ? m + logf(l) : -INFINITY;
}

// D_i = dO_i . O_i  (fp32) for every row, any element type.
template <typename T, int D>
__global__ void __launch_bounds__(128) rowdot_kernel(const T* __restrict__ o, const T* __restrict__ dout,
                                                     float* __restrict__ Dout, int B, int Hq, int Nq) {
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 4 + warp;  // over B * Nq * Hq in memory order
  if (row >= (long long)B * Nq * Hq) return;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e)
    acc = fmaf(static_cast<float>(o[row * D + lane + 32 * e]), static_cast<float>(dout[row * D + lane + 32 * e]),
               acc);
  acc = warp_sum(acc);
  if (lane == 0) {
    const int h = (int)(row % Hq);
    const long long bn = row / Hq;
    const int n = (int)(bn % Nq), b = (int)(bn / Nq);
    Dout[((long long)b * Hq + h) * Nq + n] = acc;
  }
}

template <int D>
__global__ void __launch_bounds__(128) bwd_dq_f32_kernel(F32Params p, const float* __restrict__ dout,
                                                         const float* __restrict__ Drow, float* __restrict__ dq) {
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const Seq s = seq_of(p, blockIdx.z);
  const int i = blockIdx.x * 4 + warp;
  if (i >= s.nq) return;
  const int hk = h / (p.Hq / p.Hkv);
  const long long qo = s.b * p.q_bstride + ((long long)(s.q0 + i) * p.Hq + h) * D;
  const long long li = s.b * p.lse_bstride + (long long)h * p.lse_hstride + s.q0 + i;
  const float lse = p.lse[li], Di = Drow[li];
  float qv[E], dov[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = p.q[qo + lane + 32 * e];
    dov[e] = dout[qo + lane + 32 * e];
    acc[e] = 0.f;
  }
  const float* brow = p.bias ? p.bias + s.b * p.bias_bstride + ((long long)h * s.nq + i) * s.nk : nullptr;
  const float slope = p.alibi ? p.alibi[h] : 0.f;
  KeyRange kr = visible(p, s, i);
  if (lse == -INFINITY) kr.end = kr.lo;
  for (int j = kr.lo; j < kr.end; ++j) {
    const long long kv = s.b * p.k_bstride + ((long long)(s.k0 + j) * p.Hkv + hk) * D;
    float dot = 0.f, dpv = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      dot = fmaf(qv[e], p.k[kv + lane + 32 * e], dot);
      dpv = fmaf(dov[e], p.v[kv + lane + 32 * e], dpv);
    }
    float sc = warp_sum(dot) * p.scale;
    if (brow) sc += brow[j];
    if (p.alibi) sc -= slope * fabsf(static_cast<float>(j - i - (s.nk - s.nq)));
    const float pij = expf(sc - lse);
    const float ds = pij * (warp_sum(dpv) - Di);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(ds, p.k[kv + lane + 32 * e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < E; ++e) dq[qo + lane + 32 * e] = acc[e] * p.scale;
}

template <int D>
__global__ void __launch_bounds__(128) bwd_dkdv_f32_kernel(F32Params p, const float* __restrict__ dout,
                                                           const float* __restrict__ Drow, float* __restrict__ dk,
                                                           float* __restrict__ dv) {
  constexpr int E = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hk = blockIdx.y;
  const Seq s = seq_of(p, blockIdx.z);
  const int j = blockIdx.x * 4 + warp;
  if (j >= s.nk) return;
  const int G = p.Hq / p.Hkv;
  const long long kv = s.b * p.k_bstride + ((long long)(s.k0 + j) * p.Hkv + hk) * D;
  float kvv[E], vv[E], dka[E], dva[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    kvv[e] = p.k[kv + lane + 32 * e];
    vv[e] = p.v[kv + lane + 32 * e];
    dka[e] = 0.f;
    dva[e] = 0.f;
  }
  // row i sees key j iff j - diag - win_r <= i <= j - diag + win_l
  const int diag = s.nk - s.nq;
  const int i0 = max(0, j - diag - p.win_r);
  const int i_end = min(s.nq, j - diag + p.win_l + 1);
  for (int g = 0; g < G; ++g) {
    const int h = hk * G + g;
    const float* bcol = p.bias ? p.bias + s.b * p.bias_bstride + (long long)h * s.nq * s.nk + j : nullptr;
    const float slope = p.alibi ? p.alibi[h] : 0.f;
    for (int i = i0; i < i_end; ++i) {
      const long long li = s.b * p.lse_bstride + (long long)h * p.lse_hstride + s.q0 + i;
      const float lse = p.lse[li];
      if (lse == -INFINITY) continue;
      const long long qo = s.b * p.q_bstride + ((long long)(s.q0 + i) * p.Hq + h) * D;
      float dot = 0.f, dpv = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        dot = fmaf(p.q[qo + lane + 32 * e], kvv[e], dot);
        dpv = fmaf(dout[qo + lane + 32 * e], vv[e], dpv);
      }
      float sc = warp_sum(dot) * p.scale;
      if (bcol) sc += bcol[(long long)i * s.nk];
      if (p.alibi) sc -= slope * fabsf(static_cast<float>(j - i - (s.nk - s.nq)));
      const float pij = expf(sc - lse);
      const float ds = pij * (warp_sum(dpv) - Drow[li]);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        dva[e] = fmaf(pij, dout[qo + lane + 32 * e], dva[e]);
        dka[e] = fmaf(ds, p.q[qo + lane + 32 * e], dka[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    dk[kv + lane + 32 * e] = dka[e] * p.scale;
    dv[kv + lane + 32 * e] = dva[e];
  }
}

}  // namespace

namespace {
F32Params folded(const F32Params& in) {
  F32Params p = in;
  p.win_l = win_left(in.window_left);
  p.win_r = win_right(in.causal, in.window_right);
  p.status = device_status_ptr();
  return p;
}
}  // namespace

int launch_fwd_f32(const F32Params& in, int num_z, int max_nq, cudaStream_t st) {
  const F32Params p = folded(in);
  if (!p.status) return ATTN_ERR_CUDA;
  dim3 grid((max_nq + 3) / 4, p.Hq, num_z);
  if (p.D == 64)
    fwd_f32_kernel<64><<<grid, 128, 0, st>>>(p);
  else
    fwd_f32_kernel<128><<<grid, 128, 0, st>>>(p);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

template <typename T>
int launch_rowdot(const T* o, const T* dout, float* Drow, int B, int Hq, int Nq, int D, cudaStream_t st) {
  const long long rows = (long long)B * Nq * Hq;
  const unsigned blocks = (unsigned)((rows + 3) / 4);
  if (D == 64)
    rowdot_kernel<T, 64><<<blocks, 128, 0, st>>>(o, dout, Drow, B, Hq, Nq);
  else
    rowdot_kernel<T, 128><<<blocks, 128, 0, st>>>(o, dout, Drow, B, Hq, Nq);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}
template int launch_rowdot<float>(const float*, const float*, float*, int, int, int, int, cudaStream_t);
template int launch_rowdot<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*, float*, int, int, int,
                                          int, cudaStream_t);

int launch_bwd_f32(const F32Params& in, const float* dout, const float* Drow, float* dq, float* dk, float* dv,
                   int num_z, int max_nq, int max_nk, cudaStream_t st) {
  const F32Params p = folded(in);
  if (!p.status) return ATTN_ERR_CUDA;
  dim3 gq((max_nq + 3) / 4, p.Hq, num_z), gk((max_nk + 3) / 4, p.Hkv, num_z);
  if (p.D == 64) {
    bwd_dq_f32_kernel<64><<<gq, 128, 0, st>>>(p, dout, Drow, dq);
    bwd_dkdv_f32_kernel<64><<<gk, 128, 0, st>>>(p, dout, Drow, dk, dv);
  } else {
    bwd_dq_f32_kernel<128><<<gq, 128, 0, st>>>(p, dout, Drow, dq);
    bwd_dkdv_f32_kernel<128><<<gk, 128, 0, st>>>(p, dout, Drow, dk, dv);
  }
  count_launch(2);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
