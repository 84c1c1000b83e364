// Shared device/host definitions for the key-only GLA forward kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gtr.h"

namespace gtr {

constexpr int kChunk = 64;  // chunk length C (first GTR page, step 5 of "Method details")
constexpr int kD = 64;      // d_k = d_v supported by these kernels

// Workspace header: a device error word and a few counters, 256 bytes.
struct WsHeader {
  unsigned int error;      // first device-side failure code (gtr_status_t), 0 = none
  unsigned int error_aux;  // where it happened (kernel-specific)
  unsigned int ticket;     // dynamic work counter for ticketed kernels
  unsigned int epoch;      // call counter, bumps every fused call
  // failure injection (gtr_gla_workspace_debug; zero = off): segment dbg_skip_seg - 1 of
  // every sequence withholds its summary flag, and waits for other segments' flags give
  // up after dbg_wait_us microseconds instead of about a second
  unsigned int dbg_skip_seg;
  unsigned int dbg_wait_us;
  unsigned int pad[58];
};
static_assert(sizeof(WsHeader) == 256, "workspace header must stay 256 bytes");

// Every workspace starts with the header and a fixed 2 KB region of per-sequence
// arrival counters (used by the fused path, kept zero between calls); each path's own
// arrays start after this prefix, so calls of different paths can share a workspace.
constexpr size_t kWsCounterBytes = 2048;
constexpr size_t kWsPrefixBytes = sizeof(WsHeader) + kWsCounterBytes;
// Split path scratch per (batch, head, chunk) unit: the chunk summary U and the chunk-start
// state S (64 x 64 fp32 each) and the chunk log-decays (64 fp32).
constexpr size_t kSplitUnitBytes = (2 * kD * kD + kD) * sizeof(float);

struct Problem {
  const void* q;
  const void* k;
  const void* v;
  const float* log_gamma;
  void* out;
  int B, heads, H, W, d_k, d_v, direction, in_dtype, out_dtype;
  // Low-rank gate producer (gz != nullptr; log_gamma is then not read): log gamma of
  // token m, head h = logsigmoid(gz[b, m, :] gw2[:, h*d_k .. h*d_k+d_k-1] + gb[h*d_k ..]) / gtau,
  // gz [B, L, grank] fp32, gw2 [grank, heads * d_k] fp32, gb [heads * d_k] fp32.
  const float* gz = nullptr;
  const float* gw2 = nullptr;
  const float* gb = nullptr;
  float gtau = 1.f;
  int grank = 0;
  // RMSNorm + SiLU output gate (ogate != nullptr): out = o / sqrt(mean_j o_j^2 + oeps) *
  // onorm_w * SiLU(ogate), per token-head over d_v; ogate [B, L, heads, d_v] in the input
  // dtype, onorm_w [d_v] fp32.
  const void* ogate = nullptr;
  const float* onorm_w = nullptr;
  float oeps = 0.f;

  __host__ __device__ long long L() const { return (long long)H * (long long)W; }
  __host__ __device__ int n_chunks() const { return (int)((L() + kChunk - 1) / kChunk); }
};

// Scan position s -> token index m = y*W + x.
//   L2R rows top->bottom, x ascending    R2L rows top->bottom, x descending
//   T2B cols left->right, y ascending    B2T cols left->right, y descending
__host__ __device__ __forceinline__ long long scan_to_token(long long s, int dir, int H, int W) {
  long long x, y;
  if (dir <= GTR_R2L) {
    y = s / W;
    x = s - y * W;
    if (dir == GTR_R2L) x = W - 1 - x;
  } else {
    x = s / H;
    y = s - x * H;
    if (dir == GTR_B2T) y = H - 1 - y;
  }
  return y * W + x;
}

// Row index (token-head) of scan position s of (b, h) in the [B, L, heads, d] layout.
__host__ __device__ __forceinline__ long long token_head_row(const Problem& p, int b, int h,
                                                             long long s) {
  long long m = scan_to_token(s, p.direction, p.H, p.W);
  return ((long long)b * p.L() + m) * p.heads + h;
}

template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f32(float x) { return x; }
  static __device__ __forceinline__ float from_f32(float x) { return x; }
};
template <> struct Elem<__half> {
  static __device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }
  static __device__ __forceinline__ __half from_f32(float x) { return __float2half_rn(x); }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f32(float x) { return __float2bfloat16_rn(x); }
};

// Load 4 consecutive elements as fp32 (16-byte aligned for fp32, 8-byte for 16-bit types).
template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}
template <>
__device__ __forceinline__ float4 load4<__half>(const __half* p) {
  uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  float2 a = __half22float2(*reinterpret_cast<__half2*>(&u.x));
  float2 b = __half22float2(*reinterpret_cast<__half2*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
  uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
  float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

template <typename T>
__device__ __forceinline__ void store4(T* p, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}
template <>
__device__ __forceinline__ void store4<__half>(__half* p, float4 v) {
  __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// Record the first device-side failure in the workspace error word.
__device__ __forceinline__ void record_error(WsHeader* hdr, unsigned int code, unsigned int aux) {
  if (atomicCAS(&hdr->error, 0u, code) == 0u) hdr->error_aux = aux;
}

}  // namespace gtr
