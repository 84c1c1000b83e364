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

size_t split_workspace_bytes(const Problem& p);
SplitWorkspace split_workspace_carve(void* ws, const Problem& p);
gtr_status_t launch_split(const Problem& p, void* ws, cudaStream_t stream);

}  // namespace gtr
