// Internal interfaces between the C ABI (gtr_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "gtr.h"

namespace gtr {

struct Problem;
struct WsHeader;

struct SplitWorkspace {
  WsHeader* hdr;
  float* U;       // [B*heads*Nc][64][64] chunk summaries
  float* S;       // [B*heads*Nc][64][64] state at the start of each chunk
  float* a_last;  // [B*heads*Nc][64]     chunk log-decays
};

struct FusedWorkspace {
  WsHeader* hdr;
  unsigned int* counters;  // per-sequence arrival counters (zero between calls)
  float* agg;              // per-segment summaries
  uint16_t* sstart;        // per-segment start states (fp16, MMA layout, their CTA's scale)
  uint16_t* qhp;           // segmented mode: per-chunk Qh' tiles (fp16, MMA layout)
  uint16_t* olc;           // segmented mode: per-chunk outputs from a zero segment start (fp16)
};

// Argument validation of the device entry points (shape, enums, dtype pairing, pointers),
// done on the host before anything is enqueued.
gtr_status_t validate_call(const void* q, const void* k, const void* v, const float* log_gamma, void* out,
                           int B, int heads, int grid_H, int grid_W, int d_k, int d_v, int direction,
                           int in_dtype, int out_dtype);

size_t split_workspace_bytes(const Problem& p);
SplitWorkspace split_workspace_carve(void* ws, const Problem& p);
gtr_status_t launch_split(const Problem& p, void* ws, cudaStream_t stream);

size_t fused_workspace_bytes(const Problem& p);
FusedWorkspace fused_workspace_carve(void* ws, const Problem& p);
int fused_launches(const Problem& p);
size_t fused_reset_bytes();  // header + counters: what a zeroed workspace must have zero
// force_mode: -1 = let the plan decide, 0 = one CTA per sequence (stream mode)
gtr_status_t launch_fused(const Problem& p, void* ws, cudaStream_t stream, int force_mode);
// one per input/output dtype pair and key width, each in its own translation unit
#define GTR_DECLARE_FUSED(tag)                                                                         \
  gtr_status_t launch_fused_##tag##_dk64(const Problem& p, void* ws, cudaStream_t stream, int force_mode); \
  gtr_status_t launch_fused_##tag##_dk32(const Problem& p, void* ws, cudaStream_t stream, int force_mode);
GTR_DECLARE_FUSED(f16_f16)
GTR_DECLARE_FUSED(f16_f32)
GTR_DECLARE_FUSED(bf16_f32)
GTR_DECLARE_FUSED(bf16_bf16)
#undef GTR_DECLARE_FUSED

}  // namespace gtr
