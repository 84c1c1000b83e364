// Fused path, host side: workspace layout and the dtype dispatch of the launches.
// The kernel and its launch live in gtr_fused_kernel.cuh; each input/output dtype
// pair and key width is instantiated in a translation unit of its own
// (gtr_fused_<in>_<out>_dk<d_k>.cu) so that the kernels compile in parallel.
#include "gtr_fused_kernel.cuh"

namespace gtr {

// Per-chunk tiles of the second phase (Qh' and O_local, fp16): only when sequences may
// be split over CTAs.
size_t segmented_tile_bytes(const Problem& p) {
  return seg_capacity(p) ? (size_t)p.B * p.heads * max_fused_chunks(p) * 4096 * sizeof(uint16_t) : 0;
}

size_t fused_workspace_bytes(const Problem& p) {
  const size_t segs = seg_capacity(p);
  size_t b = sizeof(WsHeader) + kCounterBytes + segs * kAggStride * sizeof(float) + segs * 4096 * sizeof(uint16_t);
  b = (b + 1023) & ~size_t(1023);  // 1 KB-aligned tiles for the bulk copies
  return b + 2 * segmented_tile_bytes(p);
}

FusedWorkspace fused_workspace_carve(void* ws, const Problem& p) {
  const size_t segs = seg_capacity(p);
  FusedWorkspace w;
  uint8_t* base = reinterpret_cast<uint8_t*>(ws);
  w.hdr = reinterpret_cast<WsHeader*>(base);
  base += sizeof(WsHeader);
  w.counters = reinterpret_cast<unsigned int*>(base);
  base += kCounterBytes;
  w.agg = reinterpret_cast<float*>(base);
  base += segs * kAggStride * sizeof(float);
  w.sstart = reinterpret_cast<uint16_t*>(base);
  base += segs * 4096 * sizeof(uint16_t);
  const size_t used = (size_t)(base - reinterpret_cast<uint8_t*>(ws));
  base = reinterpret_cast<uint8_t*>(ws) + ((used + 1023) & ~size_t(1023));
  const size_t tiles = segmented_tile_bytes(p);
  w.qhp = tiles ? reinterpret_cast<uint16_t*>(base) : nullptr;
  w.olc = tiles ? reinterpret_cast<uint16_t*>(base + tiles) : nullptr;
  return w;
}

size_t fused_reset_bytes() { return sizeof(WsHeader) + kCounterBytes; }

int fused_launches(const Problem& p) {
  (void)p;
  return 1;
}

gtr_status_t launch_fused(const Problem& p, void* ws, cudaStream_t stream, int force_mode) {
  if ((long long)p.B * p.L() >= (1ll << 31)) return GTR_ERR_UNSUPPORTED;
  const bool dk32 = p.d_k == 32;
  switch (p.in_dtype * 3 + p.out_dtype) {
    case GTR_F16 * 3 + GTR_F16:
      return dk32 ? launch_fused_f16_f16_dk32(p, ws, stream, force_mode) : launch_fused_f16_f16_dk64(p, ws, stream, force_mode);
    case GTR_F16 * 3 + GTR_F32:
      return dk32 ? launch_fused_f16_f32_dk32(p, ws, stream, force_mode) : launch_fused_f16_f32_dk64(p, ws, stream, force_mode);
    case GTR_BF16 * 3 + GTR_F32:
      return dk32 ? launch_fused_bf16_f32_dk32(p, ws, stream, force_mode)
                  : launch_fused_bf16_f32_dk64(p, ws, stream, force_mode);
    case GTR_BF16 * 3 + GTR_BF16:
      return dk32 ? launch_fused_bf16_bf16_dk32(p, ws, stream, force_mode)
                  : launch_fused_bf16_bf16_dk64(p, ws, stream, force_mode);
    default: return GTR_ERR_UNSUPPORTED;
  }
}

}  // namespace gtr
