// C-ABI entry points of libattn (declared in include/attn.h): argument
// validation, dispatch by dtype / head dim / bias, workspace carving, and the
// device status word.  Nothing here computes attention; every step of the
// path runs in the kernels.
#include <algorithm>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace attn {

namespace {
thread_local long long g_launches = 0;
thread_local cudaEvent_t g_kernel_events[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
}  // namespace

void count_launch(int n) { g_launches += n; }

void record_kernel_event(int which, int stop, cudaStream_t st) {
  cudaEvent_t ev = g_kernel_events[which][stop];
  if (ev) cudaEventRecord(ev, st);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0)
    return 1;
  return n;
}

int* device_status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(ptr);
  }
  return g_status_ptr[dev];
}

int encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_tmap(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, dims, strides_bytes, box);
}

int encode_tmap(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int rank, const uint64_t* dims,
                const uint64_t* strides_bytes, const uint32_t* box) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return ATTN_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
  }
  cuuint64_t d[5];
  cuuint64_t s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) s[i] = strides_bytes[i];
  }
  const CUresult r = g_encode(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), d, s,
                              b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn

using namespace attn;

namespace {

int check_common(int batch, int h_q, int h_kv, int n_q, int n_k, int d, int dtype) {
  if (batch <= 0 || h_q <= 0 || h_kv <= 0 || n_q <= 0 || n_k <= 0) return ATTN_ERR_INVALID;
  if (h_q % h_kv != 0) return ATTN_ERR_INVALID;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (dtype != ATTN_BF16 && dtype != ATTN_F32) return ATTN_ERR_UNSUPPORTED;
  // the kernels index rows with 32-bit coordinates (TMA) and 64-bit offsets
  if ((long long)batch * n_q > (1ll << 31) - 1 || (long long)batch * n_k > (1ll << 31) - 1) return ATTN_ERR_INVALID;
  if (n_q > kMaxSeqLen || n_k > kMaxSeqLen) return ATTN_ERR_UNSUPPORTED;
  // grid y runs over heads and z over batch elements (times key splits): 65535 at most
  if (h_q > 65535 || batch > 65535) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

int fwd_impl(const void* q, const void* k, const void* v, const float* bias, long long bias_batch_stride,
             const float* alibi, void* o, float* lse, int batch, int h_q, int h_kv, int n_q, int n_k, int d,
             float scale, int causal, int window_left, int window_right, int dtype, void* stream) {
  int rc = check_common(batch, h_q, h_kv, n_q, n_k, d, dtype);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID;
  if (bias_batch_stride < 0) return ATTN_ERR_INVALID;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == ATTN_F32) {
    F32Params p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.bias = bias;
    p.alibi = alibi;
    p.o = static_cast<float*>(o);
    p.lse = lse;
    p.q_bstride = (long long)n_q * h_q * d;
    p.k_bstride = (long long)n_k * h_kv * d;
    p.bias_bstride = bias_batch_stride;
    p.lse_bstride = (long long)h_q * n_q;
    p.lse_hstride = n_q;
    p.Hq = h_q;
    p.Hkv = h_kv;
    p.Nq = n_q;
    p.Nk = n_k;
    p.D = d;
    p.causal = causal != 0;
    p.window_left = window_left;
    p.window_right = window_right;
    p.scale = scale;
    return launch_fwd_f32(p, batch, n_q, st);
  }
  TcGeom g{};
  g.q = q;
  g.k = k;
  g.v = v;
  g.B = batch;
  g.Hq = h_q;
  g.Hkv = h_kv;
  g.Nq = n_q;
  g.Nk = n_k;
  g.D = d;
  g.causal = causal != 0;
  g.window_left = window_left;
  g.window_right = window_right;
  g.scale = scale;
  g.bias = bias;
  g.bias_bstride = bias_batch_stride;
  g.alibi = alibi;
  return launch_fwd_sm100(g, static_cast<__nv_bfloat16*>(o), lse, st);
}

}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, const float* bias, long long bias_batch_stride, void* o,
             float* lse, int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale, int causal, int dtype,
             void* stream) {
  return fwd_impl(q, k, v, bias, bias_batch_stride, nullptr, o, lse, batch, h_q, h_kv, n_q, n_k, d, scale, causal,
                  -1, -1, dtype, stream);
}

int attn_fwd_alibi(const void* q, const void* k, const void* v, const float* alibi_slopes, void* o, float* lse,
                   int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale, int causal, int dtype,
                   void* stream) {
  if (!alibi_slopes) return ATTN_ERR_INVALID;
  return fwd_impl(q, k, v, nullptr, 0, alibi_slopes, o, lse, batch, h_q, h_kv, n_q, n_k, d, scale, causal, -1, -1,
                  dtype, stream);
}

int attn_fwd_local(const void* q, const void* k, const void* v, const float* alibi_slopes, void* o, float* lse,
                   int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale, int causal, int window_left,
                   int window_right, int dtype, void* stream) {
  return fwd_impl(q, k, v, nullptr, 0, alibi_slopes, o, lse, batch, h_q, h_kv, n_q, n_k, d, scale, causal,
                  window_left, window_right, dtype, stream);
}

size_t attn_bwd_workspace_size(int batch, int h_q, int n_q, int d) {
  if (batch <= 0 || h_q <= 0 || n_q <= 0 || d <= 0) return 0;
  return align256((size_t)batch * n_q * h_q * d * sizeof(float)) + align256((size_t)batch * h_q * n_q * sizeof(float));
}

}  // extern "C"

namespace {

int bwd_impl(const void* q, const void* k, const void* v, const float* bias, long long bias_batch_stride,
             const float* alibi, const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
             void* workspace, size_t workspace_bytes, int batch, int h_q, int h_kv, int n_q, int n_k, int d,
             float scale, int causal, int window_left, int window_right, int dtype, void* stream,
             const int* cu_q = nullptr, const int* cu_k = nullptr, int num_seqs = 0, int max_nq = 0,
             int max_nk = 0, int d_v = 0) {
  // packed sequences: batch 1 of n_q / n_k total rows, cu_q / cu_k prefix offsets
  int rc = check_common(batch, h_q, h_kv, n_q, n_k, d, dtype);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv))
    return ATTN_ERR_INVALID;
  if (bias_batch_stride < 0) return ATTN_ERR_INVALID;
  const size_t need = attn_bwd_workspace_size(batch, h_q, n_q, d);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return ATTN_ERR_WORKSPACE;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* dq_acc = static_cast<float*>(workspace);
  float* Drow = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                         align256((size_t)batch * n_q * h_q * d * sizeof(float)));
  if (dtype == ATTN_F32) {
    rc = launch_rowdot<float>(static_cast<const float*>(o), static_cast<const float*>(dout), Drow, batch, h_q, n_q, d,
                              st);
    if (rc) return rc;
    F32Params p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.bias = bias;
    p.alibi = alibi;
    p.lse = const_cast<float*>(lse);
    p.q_bstride = (long long)n_q * h_q * d;
    p.k_bstride = (long long)n_k * h_kv * d;
    p.bias_bstride = bias_batch_stride;
    p.lse_bstride = (long long)h_q * n_q;
    p.lse_hstride = n_q;
    p.cu_q = cu_q;
    p.cu_k = cu_k;
    p.max_nq = max_nq;
    p.max_nk = max_nk;
    p.Hq = h_q;
    p.Hkv = h_kv;
    p.Nq = n_q;
    p.Nk = n_k;
    p.D = d;
    p.causal = causal != 0;
    p.window_left = window_left;
    p.window_right = window_right;
    p.scale = scale;
    return launch_bwd_f32(p, static_cast<const float*>(dout), Drow, static_cast<float*>(dq), static_cast<float*>(dk),
                          static_cast<float*>(dv), cu_q ? num_seqs : batch, cu_q ? max_nq : n_q,
                          cu_q ? max_nk : n_k, st);
  }
  TcGeom g{};
  g.q = q;
  g.k = k;
  g.v = v;
  g.B = batch;
  g.Hq = h_q;
  g.Hkv = h_kv;
  g.Nq = n_q;
  g.Nk = n_k;
  g.D = d;
  g.causal = causal != 0;
  g.window_left = window_left;
  g.window_right = window_right;
  g.scale = scale;
  g.bias = bias;
  g.bias_bstride = bias_batch_stride;
  g.alibi = alibi;
  g.cu_q = cu_q;
  g.cu_k = cu_k;
  g.num_seqs = num_seqs;
  g.max_nq = max_nq;
  g.max_nk = max_nk;
  g.Dv = d_v;
  return launch_bwd_sm100(g, static_cast<const __nv_bfloat16*>(o), lse, static_cast<const __nv_bfloat16*>(dout),
                          static_cast<__nv_bfloat16*>(dq), static_cast<__nv_bfloat16*>(dk),
                          static_cast<__nv_bfloat16*>(dv), dq_acc, Drow, st);
}

}  // namespace

extern "C" {

int attn_bwd(const void* q, const void* k, const void* v, const float* bias, long long bias_batch_stride,
             const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
             size_t workspace_bytes, int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale, int causal,
             int dtype, void* stream) {
  return bwd_impl(q, k, v, bias, bias_batch_stride, nullptr, o, lse, dout, dq, dk, dv, workspace, workspace_bytes,
                  batch, h_q, h_kv, n_q, n_k, d, scale, causal, -1, -1, dtype, stream);
}

int attn_bwd_alibi(const void* q, const void* k, const void* v, const float* alibi_slopes, const void* o,
                   const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale,
                   int causal, int dtype, void* stream) {
  if (!alibi_slopes) return ATTN_ERR_INVALID;
  return bwd_impl(q, k, v, nullptr, 0, alibi_slopes, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, batch,
                  h_q, h_kv, n_q, n_k, d, scale, causal, -1, -1, dtype, stream);
}

int attn_bwd_local(const void* q, const void* k, const void* v, const float* alibi_slopes, const void* o,
                   const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                   size_t workspace_bytes, int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale,
                   int causal, int window_left, int window_right, int dtype, void* stream) {
  return bwd_impl(q, k, v, nullptr, 0, alibi_slopes, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, batch,
                  h_q, h_kv, n_q, n_k, d, scale, causal, window_left, window_right, dtype, stream);
}

int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                    void* dq, void* dk, void* dv, const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                    int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int h_q, int h_kv, int d,
                    float scale, int causal, void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  if (num_seqs <= 0 || max_seqlen_q <= 0 || max_seqlen_k <= 0 || !cu_seqlens_q || !cu_seqlens_k)
    return ATTN_ERR_INVALID;
  if (num_seqs > 65535) return ATTN_ERR_UNSUPPORTED;  // grid z runs over sequences
  if (max_seqlen_q > total_q || max_seqlen_k > total_k) return ATTN_ERR_INVALID;
  return bwd_impl(q, k, v, nullptr, 0, nullptr, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, 1, h_q, h_kv,
                  total_q, total_k, d, scale, causal, -1, -1, dtype, stream, cu_seqlens_q, cu_seqlens_k, num_seqs,
                  max_seqlen_q, max_seqlen_k);
}

int attn_bwd_dv(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int batch, int h_q, int h_kv,
                int n_q, int n_k, int d, int d_v, float scale, int causal, int dtype, void* stream) {
  if (d_v != 64 && d_v != 128) return ATTN_ERR_UNSUPPORTED;
  if (d_v != d && dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  return bwd_impl(q, k, v, nullptr, 0, nullptr, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, batch, h_q,
                  h_kv, n_q, n_k, d, scale, causal, -1, -1, dtype, stream, nullptr, nullptr, 0, 0, 0,
                  d_v == d ? 0 : d_v);
}

int attn_fwd_dv(const void* q, const void* k, const void* v, void* o, float* lse, int batch, int h_q, int h_kv,
                int n_q, int n_k, int d, int d_v, float scale, int causal, int dtype, void* stream) {
  int rc = check_common(batch, h_q, h_kv, n_q, n_k, d, dtype);
  if (rc) return rc;
  if (d_v != 64 && d_v != 128) return ATTN_ERR_UNSUPPORTED;
  if (d_v == d)
    return fwd_impl(q, k, v, nullptr, 0, nullptr, o, lse, batch, h_q, h_kv, n_q, n_k, d, scale, causal, -1, -1,
                    dtype, stream);
  if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  TcGeom g{};
  g.q = q;
  g.k = k;
  g.v = v;
  g.B = batch;
  g.Hq = h_q;
  g.Hkv = h_kv;
  g.Nq = n_q;
  g.Nk = n_k;
  g.D = d;
  g.Dv = d_v;
  g.causal = causal != 0;
  g.scale = scale;
  return launch_fwd_sm100(g, static_cast<__nv_bfloat16*>(o), lse, static_cast<cudaStream_t>(stream));
}

int attn_splitkv_num_splits(int batch, int h_q, int n_q, int n_k) {
  if (batch <= 0 || h_q <= 0 || n_q <= 0 || n_k <= 0) return 1;
  const long long ctas = (long long)((n_q + 255) / 256) * h_q * batch;  // 256 query rows per CTA
  const int kv_tiles = (n_k + 127) / 128;
  // One CTA per SM at a time (the forward holds all of TMEM): pick the split
  // count whose last wave is fullest, preferring fewer splits (each adds a
  // merge pass and a pipeline start); splits keep at least four key tiles.
  const int t_max = (int)std::max(1, std::min(64, kv_tiles / 4));
  auto fill = [&](long long t) {
    const long long n = ctas * t;
    return (double)n / (double)(((n + 147) / 148) * 148);
  };
  int best = 1;
  for (int t = 2; t <= t_max; ++t)
    if (fill(t) > fill(best) + 0.05) best = t;
  return best;
}

size_t attn_splitkv_workspace_size(int batch, int h_q, int n_q, int d, int num_splits) {
  if (batch <= 0 || h_q <= 0 || n_q <= 0 || d <= 0 || num_splits <= 0) return 0;
  const size_t rows = (size_t)batch * n_q * h_q;
  return align256(rows * d * num_splits * sizeof(float)) + align256(rows * num_splits * sizeof(float));
}

int attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int batch, int h_q, int h_kv,
                     int n_q, int n_k, int d, float scale, int causal, int num_splits, void* workspace,
                     size_t workspace_bytes, int dtype, void* stream) {
  int rc = check_common(batch, h_q, h_kv, n_q, n_k, d, dtype);
  if (rc) return rc;
  if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID;
  if (num_splits <= 0) num_splits = attn_splitkv_num_splits(batch, h_q, n_q, n_k);
  const int kv_tiles = (n_k + 127) / 128;
  const int tiles_per_split = (kv_tiles + std::min(num_splits, kv_tiles) - 1) / std::min(num_splits, kv_tiles);
  const int splits = (kv_tiles + tiles_per_split - 1) / tiles_per_split;  // none of them empty
  if ((long long)batch * splits > 65535) return ATTN_ERR_UNSUPPORTED;     // grid z
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  TcGeom g{};
  g.q = q;
  g.k = k;
  g.v = v;
  g.B = batch;
  g.Hq = h_q;
  g.Hkv = h_kv;
  g.Nq = n_q;
  g.Nk = n_k;
  g.D = d;
  g.causal = causal != 0;
  g.scale = scale;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (splits == 1) return launch_fwd_sm100(g, static_cast<__nv_bfloat16*>(o), lse, st);
  const size_t need = attn_splitkv_workspace_size(batch, h_q, n_q, d, splits);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ATTN_ERR_WORKSPACE;
  const size_t rows = (size_t)batch * n_q * h_q;
  SplitKV sp;
  sp.num_splits = splits;
  sp.split_len = tiles_per_split * 128;
  sp.o_part = static_cast<float*>(workspace);
  sp.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(rows * d * splits * sizeof(float)));
  rc = launch_fwd_sm100(g, static_cast<__nv_bfloat16*>(o), lse, st, &sp);
  if (rc) return rc;
  return launch_merge(sp.o_part, sp.lse_part, splits, o, lse, batch, h_q, n_q, d, 0, st);
}

int attn_fwd_partial(const void* q, const void* k, const void* v, float* o_part, float* lse_part, int batch,
                     int h_q, int h_kv, int n_q, int n_k, int d, float scale, int causal, int dtype, void* stream) {
  int rc = check_common(batch, h_q, h_kv, n_q, n_k, d, dtype);
  if (rc) return rc;
  if (dtype != ATTN_BF16) return ATTN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o_part || !lse_part) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o_part)) return ATTN_ERR_INVALID;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  TcGeom g{};
  g.q = q;
  g.k = k;
  g.v = v;
  g.B = batch;
  g.Hq = h_q;
  g.Hkv = h_kv;
  g.Nq = n_q;
  g.Nk = n_k;
  g.D = d;
  g.causal = causal != 0;
  g.scale = scale;
  // one "split" holding every key of the block: the kernel's partial epilogue
  SplitKV sp;
  sp.num_splits = 1;
  sp.split_len = (n_k + 127) / 128 * 128;
  sp.o_part = o_part;
  sp.lse_part = lse_part;
  return launch_fwd_sm100(g, nullptr, nullptr, static_cast<cudaStream_t>(stream), &sp);
}

int attn_quantize_e4m3(const void* x, void* x8, float* scales, int batch, int n, int heads, int d, void* stream) {
  if (!x || !x8 || !scales || batch <= 0 || n <= 0 || heads <= 0) return ATTN_ERR_INVALID;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)batch * n > (1ll << 31) - 1 || batch > 65535 || heads > 65535) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(x8)) return ATTN_ERR_INVALID;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  return launch_quantize_e4m3(static_cast<const __nv_bfloat16*>(x), static_cast<uint8_t*>(x8), scales, batch, n,
                              heads, d, static_cast<cudaStream_t>(stream));
}

int attn_fwd_fp8(const void* q8, const float* q_scales, const void* k8, const float* k_scales, const void* v,
                 void* o, float* lse, int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale,
                 int causal, void* stream) {
  int rc = check_common(batch, h_q, h_kv, n_q, n_k, d, ATTN_BF16);
  if (rc) return rc;
  if (d != 128 || !(scale > 0.f)) return ATTN_ERR_UNSUPPORTED;
  if (!q8 || !q_scales || !k8 || !k_scales || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  TcGeom g{};
  g.q = q8;
  g.k = k8;
  g.v = v;
  g.B = batch;
  g.Hq = h_q;
  g.Hkv = h_kv;
  g.Nq = n_q;
  g.Nk = n_k;
  g.D = d;
  g.causal = causal != 0;
  g.scale = scale;
  return launch_fwd_fp8(g, q8, q_scales, k8, k_scales, static_cast<__nv_bfloat16*>(o), lse,
                        static_cast<cudaStream_t>(stream));
}

int attn_merge_partials(const float* o_parts, const float* lse_parts, int num_parts, void* o, float* lse, int batch,
                        int h_q, int n_q, int d, int out_dtype, void* stream) {
  if (!o_parts || !lse_parts || !o || !lse || num_parts <= 0 || batch <= 0 || h_q <= 0 || n_q <= 0)
    return ATTN_ERR_INVALID;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (out_dtype != ATTN_BF16 && out_dtype != ATTN_F32) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(o_parts) || !aligned16(o)) return ATTN_ERR_INVALID;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  return launch_merge(o_parts, lse_parts, num_parts, o, lse, batch, h_q, n_q, d, out_dtype == ATTN_F32,
                      static_cast<cudaStream_t>(stream));
}

int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                    const int* cu_seqlens_k, int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q,
                    int total_k, int h_q, int h_kv, int d, float scale, int causal, int dtype, void* stream) {
  if (num_seqs <= 0 || max_seqlen_q <= 0 || max_seqlen_k <= 0) return ATTN_ERR_INVALID;
  if (num_seqs > 65535) return ATTN_ERR_UNSUPPORTED;  // grid z runs over sequences
  int rc = check_common(1, h_q, h_kv, total_q, total_k, d, dtype);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID;
  if (max_seqlen_q > total_q || max_seqlen_k > total_k) return ATTN_ERR_INVALID;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == ATTN_F32) {
    F32Params p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.o = static_cast<float*>(o);
    p.lse = lse;
    p.cu_q = cu_seqlens_q;
    p.cu_k = cu_seqlens_k;
    p.max_nq = max_seqlen_q;
    p.max_nk = max_seqlen_k;
    p.lse_hstride = total_q;
    p.Hq = h_q;
    p.Hkv = h_kv;
    p.Nq = total_q;
    p.Nk = total_k;
    p.D = d;
    p.causal = causal != 0;
    p.scale = scale;
    return launch_fwd_f32(p, num_seqs, max_seqlen_q, st);
  }
  TcGeom g{};
  g.q = q;
  g.k = k;
  g.v = v;
  g.B = 1;
  g.Hq = h_q;
  g.Hkv = h_kv;
  g.Nq = total_q;
  g.Nk = total_k;
  g.D = d;
  g.cu_q = cu_seqlens_q;
  g.cu_k = cu_seqlens_k;
  g.num_seqs = num_seqs;
  g.max_nq = max_seqlen_q;
  g.max_nk = max_seqlen_k;
  g.causal = causal != 0;
  g.scale = scale;
  return launch_fwd_sm100(g, static_cast<__nv_bfloat16*>(o), lse, st);
}

size_t attn_naive_scratch_size(int n_q, int n_k) {
  if (n_q <= 0 || n_k <= 0) return 0;
  return align256((size_t)n_q * n_k * sizeof(float)) + align256((size_t)n_q * n_k * sizeof(__nv_bfloat16));
}

int attn_fwd_naive(const void* q, const void* k, const void* v, void* o, float* lse, void* scratch,
                   size_t scratch_bytes, int batch, int h_q, int h_kv, int n_q, int n_k, int d, float scale,
                   int causal, void* stream) {
  int rc = check_common(batch, h_q, h_kv, n_q, n_k, d, ATTN_BF16);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID;
  if (!scratch || scratch_bytes < attn_naive_scratch_size(n_q, n_k) || (reinterpret_cast<uintptr_t>(scratch) & 255u))
    return ATTN_ERR_WORKSPACE;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  TcGeom g{};
  g.q = q;
  g.k = k;
  g.v = v;
  g.B = batch;
  g.Hq = h_q;
  g.Hkv = h_kv;
  g.Nq = n_q;
  g.Nk = n_k;
  g.D = d;
  g.causal = causal != 0;
  g.scale = scale;
  float* s_scratch = static_cast<float*>(scratch);
  __nv_bfloat16* p_scratch =
      reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(scratch) + align256((size_t)n_q * n_k * sizeof(float)));
  return launch_fwd_naive(g, static_cast<__nv_bfloat16*>(o), lse, s_scratch, p_scratch,
                          static_cast<cudaStream_t>(stream));
}

const char* attn_strerror(int code) {
  switch (code) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID: return "invalid argument (null pointer, size, head grouping or alignment)";
    case ATTN_ERR_UNSUPPORTED: return "unsupported configuration (head dim, dtype, bias with packed input, or device)";
    case ATTN_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case ATTN_ERR_CUDA: return "CUDA call failed";
    case ATTN_ERR_TIMEOUT: return "a kernel abandoned a bounded wait (outputs undefined)";
    default: return "unknown error code";
  }
}

int attn_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
  int* ptr = device_status_ptr();
  if (!ptr) return ATTN_ERR_CUDA;
  int value = 0;
  const int zero = 0;
  if (cudaMemcpy(&value, ptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ATTN_ERR_CUDA;
  if (cudaMemcpy(ptr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return ATTN_ERR_CUDA;
  return value;
}

int attn_selftest_wait_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 1000 || limit_cycles > kWaitLimitCycles) return ATTN_ERR_INVALID;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  return launch_wait_selftest(limit_cycles, static_cast<cudaStream_t>(stream));
}

int attn_selftest_ex2(const float* x, float* y, long long n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return ATTN_ERR_INVALID;
  if (n == 0) return ATTN_OK;
  if (!supported_device()) return ATTN_ERR_UNSUPPORTED;
  return launch_ex2_selftest(x, y, n, static_cast<cudaStream_t>(stream));
}

int attn_set_kernel_events(int which, void* start, void* stop) {
  if (which != ATTN_KERNEL_FWD && which != ATTN_KERNEL_BWD) return ATTN_ERR_INVALID;
  if ((start == nullptr) != (stop == nullptr)) return ATTN_ERR_INVALID;
  g_kernel_events[which][0] = static_cast<cudaEvent_t>(start);
  g_kernel_events[which][1] = static_cast<cudaEvent_t>(stop);
  return ATTN_OK;
}

long long attn_launch_count(int reset) {
  const long long n = g_launches;
  if (reset) g_launches = 0;
  return n;
}

}  // extern "C"
