// Block-sparse attention forward on tcgen05 tensor cores (placeholder until
// the kernel lands: reports the shape as unsupported).
#include "dsa_internal.cuh"

namespace dsa {

bool attn_tc_supported(const Shape&) { return false; }

cudaError_t launch_attn_tc(const Shape&, const __nv_bfloat16*, const __nv_bfloat16*,
                           const __nv_bfloat16*, const int32_t*, const int32_t*, __nv_bfloat16*,
                           float*, WsHeader*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace dsa
