#include "common.cuh"
#include "kernels.h"
namespace attn {
int launch_bwd_sm100(const TcGeom&, const __nv_bfloat16*, const float*, const __nv_bfloat16*, __nv_bfloat16*,
                     __nv_bfloat16*, __nv_bfloat16*, float*, float*, cudaStream_t) {
  return ATTN_ERR_UNSUPPORTED;
}
}  // namespace attn
