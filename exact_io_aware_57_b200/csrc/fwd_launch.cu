// Host side of the tensor-core forward: tensor maps over Q, K, V (4-D views
// (d, head, row, batch) with 128-byte swizzled 128-row boxes), the kernel
// parameters, and dispatch to the two-tile forward kernel (fwd_pp_sm100.cu)
// for every variant: bias kind, head widths, packed sequences, key splits and
// e4m3 Q/K.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace attn {

// Kernel parameters of a forward launch (everything but the tensor maps).
int fwd_params(const TcGeom& g, __nv_bfloat16* o, float* lse, const SplitKV* split, FwdParams& p) {
  const int dv = g.Dv ? g.Dv : g.D;
  p.o = o;
  p.lse = lse;
  p.bias = g.bias;
  p.bias_bstride = g.bias_bstride;
  p.bias_vec4 = g.bias && (reinterpret_cast<uintptr_t>(g.bias) % 16 == 0) && g.Nk % 4 == 0 && g.bias_bstride % 4 == 0;
  // a bias shared by the batch elements: run them side by side so that they
  // read each bias tile from L2 instead of each from memory
  p.batch_inner = g.bias && g.bias_bstride == 0 && !g.cu_q && g.B > 1 && !split;
  p.alibi = g.alibi;
  p.cu_q = g.cu_q;
  p.cu_k = g.cu_k;
  p.max_nq = g.max_nq;
  p.max_nk = g.max_nk;
  p.Hq = g.Hq;
  p.Hkv = g.Hkv;
  p.Nq = g.Nq;
  p.Nk = g.Nk;
  p.o_bstride = g.cu_q ? 0 : (long long)g.Nq * g.Hq * dv;
  p.lse_bstride = g.cu_q ? 0 : (long long)g.Hq * g.Nq;
  p.lse_hstride = g.Nq;  // packed: Nq is the total row count
  p.scale_log2 = g.scale * kLog2e;
  p.causal = g.causal;
  p.win_l = win_left(g.window_left);
  p.win_r = win_right(g.causal, g.window_right);
  p.num_splits = 1;
  p.split_len = g.Nk;
  if (split) {  // dense inputs only
    p.num_splits = split->num_splits;
    p.split_len = split->split_len;
    p.o_part = split->o_part;
    p.lse_part = split->lse_part;
    p.part_o_stride = (long long)g.B * g.Nq * g.Hq * g.D;
    p.part_lse_stride = (long long)g.B * g.Hq * g.Nq;
  }
  p.status = device_status_ptr();
  p.wait_limit = kWaitLimitCycles;
  return p.status ? ATTN_OK : ATTN_ERR_CUDA;
}

int launch_fwd_sm100(const TcGeom& g, __nv_bfloat16* o, float* lse, cudaStream_t st, const SplitKV* split) {
  // 4-D views (d, head, row, batch); packed inputs are one batch of `total` rows.
  const int B = g.cu_q ? 1 : g.B;
  const int dv = g.Dv ? g.Dv : g.D;  // width of V and O
  CUtensorMap mq, mk, mv;
  const uint32_t box[4] = {64, 1, 128, 1};
  {
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hq, (uint64_t)g.Nq, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)g.D * 2, (uint64_t)g.Hq * g.D * 2, (uint64_t)g.Nq * g.Hq * g.D * 2};
    if (encode_tmap_bf16(&mq, g.q, 4, dims, str, box) != ATTN_OK) return ATTN_ERR_CUDA;
  }
  {
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)g.D * 2, (uint64_t)g.Hkv * g.D * 2, (uint64_t)g.Nk * g.Hkv * g.D * 2};
    if (encode_tmap_bf16(&mk, g.k, 4, dims, str, box) != ATTN_OK) return ATTN_ERR_CUDA;
    const uint64_t dv_dims[4] = {(uint64_t)dv, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)B};
    const uint64_t dv_str[3] = {(uint64_t)dv * 2, (uint64_t)g.Hkv * dv * 2, (uint64_t)g.Nk * g.Hkv * dv * 2};
    if (encode_tmap_bf16(&mv, g.v, 4, dv_dims, dv_str, box) != ATTN_OK) return ATTN_ERR_CUDA;
  }
  FwdParams p{};
  if (fwd_params(g, o, lse, split, p) != ATTN_OK) return ATTN_ERR_CUDA;
  // FAST: no bias and a positive scale, so the row max can be taken on raw scores
  const bool fast = !g.bias && !g.alibi && g.scale > 0.f;
  if (dv != g.D && (split || g.bias || g.alibi)) return ATTN_ERR_UNSUPPORTED;
  const int bias_kind = g.bias ? kBiasDense : g.alibi ? kBiasAlibi : kBiasNone;
  if (bias_kind == kBiasDense && !split && !g.cu_q) {
    // dense bias: the 64-key kernel (K and V maps with 64-row boxes)
    const uint32_t box64[4] = {64, 1, 64, 1};
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)B};
    const uint64_t str[3] = {(uint64_t)g.D * 2, (uint64_t)g.Hkv * g.D * 2, (uint64_t)g.Nk * g.Hkv * g.D * 2};
    if (encode_tmap_bf16(&mk, g.k, 4, dims, str, box64) != ATTN_OK) return ATTN_ERR_CUDA;
    const uint64_t dv_dims[4] = {(uint64_t)dv, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)B};
    const uint64_t dv_str[3] = {(uint64_t)dv * 2, (uint64_t)g.Hkv * dv * 2, (uint64_t)g.Nk * g.Hkv * dv * 2};
    if (encode_tmap_bf16(&mv, g.v, 4, dv_dims, dv_str, box64) != ATTN_OK) return ATTN_ERR_CUDA;
    return launch_fwd_db(g, mq, mk, mv, p, st);
  }
  return launch_fwd_pp(g, mq, mk, mv, p, bias_kind, fast, split != nullptr, st);
}

}  // namespace attn

namespace attn {

int launch_fwd_fp8(const TcGeom& g, const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                   __nv_bfloat16* o, float* lse, cudaStream_t st) {
  // e4m3 Q/K: rows of D bytes, one 128-byte box per tile; V bf16 as usual
  CUtensorMap mq, mk, mv;
  const uint32_t box8[4] = {128, 1, 128, 1}, box[4] = {64, 1, 128, 1};
  {
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hq, (uint64_t)g.Nq, (uint64_t)g.B};
    const uint64_t str[3] = {(uint64_t)g.D, (uint64_t)g.Hq * g.D, (uint64_t)g.Nq * g.Hq * g.D};
    if (encode_tmap(&mq, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, dims, str, box8) != ATTN_OK) return ATTN_ERR_CUDA;
  }
  {
    const uint64_t dims[4] = {(uint64_t)g.D, (uint64_t)g.Hkv, (uint64_t)g.Nk, (uint64_t)g.B};
    const uint64_t str8[3] = {(uint64_t)g.D, (uint64_t)g.Hkv * g.D, (uint64_t)g.Nk * g.Hkv * g.D};
    if (encode_tmap(&mk, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, dims, str8, box8) != ATTN_OK) return ATTN_ERR_CUDA;
    const uint64_t str[3] = {(uint64_t)g.D * 2, (uint64_t)g.Hkv * g.D * 2, (uint64_t)g.Nk * g.Hkv * g.D * 2};
    if (encode_tmap_bf16(&mv, g.v, 4, dims, str, box) != ATTN_OK) return ATTN_ERR_CUDA;
  }
  FwdParams p{};
  if (fwd_params(g, o, lse, nullptr, p) != ATTN_OK) return ATTN_ERR_CUDA;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  return launch_fwd_pp_fp8(g, mq, mk, mv, p, st);
}

}  // namespace attn
