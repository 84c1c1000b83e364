// Fused-path kernels for f16 inputs, f32 outputs and d_k = 64 (one translation unit per
// dtype pair and key width, so that the kernel instantiations compile in parallel).
#include "gtr_fused_kernel.cuh"

namespace gtr {

gtr_status_t launch_fused_f16_f32_dk64(const Problem& p, void* ws, cudaStream_t stream, int force_mode) {
  return launch_fused_typed<__half, float, 64>(p, ws, stream, force_mode);
}

}  // namespace gtr
