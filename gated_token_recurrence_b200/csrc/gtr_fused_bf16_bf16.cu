// Fused-path kernels for bf16 inputs and bf16 outputs (one translation unit per dtype
// pair, so that the kernel instantiations compile in parallel).
#include "gtr_fused_kernel.cuh"

namespace gtr {

gtr_status_t launch_fused_bf16_bf16(const Problem& p, void* ws, cudaStream_t stream, int force_mode) {
  return launch_fused_typed<__nv_bfloat16, __nv_bfloat16>(p, ws, stream, force_mode);
}

}  // namespace gtr
