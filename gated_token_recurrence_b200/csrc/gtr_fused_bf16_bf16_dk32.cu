// Fused-path kernels for bf16 inputs, bf16 outputs and d_k = 32 (one translation unit per
// dtype pair and key width, so that the kernel instantiations compile in parallel).
#include "gtr_fused_kernel.cuh"

namespace gtr {

gtr_status_t launch_fused_bf16_bf16_dk32(const Problem& p, void* ws, cudaStream_t stream, int force_mode) {
  return launch_fused_typed<__nv_bfloat16, __nv_bfloat16, 32>(p, ws, stream, force_mode);
}

}  // namespace gtr
