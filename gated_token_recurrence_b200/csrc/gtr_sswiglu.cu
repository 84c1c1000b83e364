// Spatial SwiGLU stencil: z = SiLU(X W_g) * DWConv3x3(X W_v) on the H x W patch grid.
//
// GTR digest page (paper.rainbus.top), prerequisite "SwiGLU" and section "Core method":
// GTR's channel mixer is Y = SiLU(X W_g) (.) DWConv3x3(X W_v) W_o, a 3x3 depthwise
// convolution inserted in the value branch so that neighbouring patches mix (page
// 0539edu.com section 3.1, "Spatial SwiGLU").  This kernel takes the two projections
// xg = X W_g and xv = X W_v ([B, L, C], token m = y * W + x) and produces the product in
// front of W_o; the projections themselves are GEMMs outside this library.
//
// One CTA per tile of kTH x kTW tokens and one 128-byte block of channels (64 channels of
// 16-bit data, 32 of fp32).  The xv tile with a one-token halo and the xg tile come in by
// TMA; the halo box starts one row and one column before the tile, and the rows and
// columns outside the grid arrive as zeros -- the convolution's zero padding.  Each
// thread then produces one 16-byte channel piece (8 channels of 16-bit data, 4 of fp32)
// of a strip of four output tokens down one column: its nine taps in registers, the six
// halo rows the strip needs read once (each neighbour feeds every output of the strip it
// touches), plus the bias, times SiLU(xg), stored with coalesced 16-byte stores.  The
// path is bound by HBM bandwidth; the instruction count per output (shared-memory loads
// and conversions) is what keeps it below that bound.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "gtr_common.cuh"
#include "gtr_sm100.cuh"

namespace gtr {
namespace {

using namespace sm100;

constexpr int kTH = 8, kTW = 16;  // tokens per tile (rows x columns)
constexpr int kCB = 128;          // bytes of channels per tile
constexpr int kThreadsSw = 256;
constexpr int kHaloBytes = (kTH + 2) * (kTW + 2) * kCB;  // 23,040
constexpr int kXgBytes = kTH * kTW * kCB;               // 16,384
constexpr int kSmemSw = kHaloBytes + kXgBytes + 1024;    // + alignment slack

struct alignas(64) SwParams {
  CUtensorMap txv, txg;  // [B][H][W][C] views: halo box (kCB bytes, kTW+2, kTH+2), tile box
  void* out;
  const float* w;  // [C][3][3]
  const float* b;  // [C] or nullptr
  int B, H, W, C;
  int tiles_x, tiles_y, cblocks;
};

template <typename T> struct Vec8;  // 16 bytes of T <-> fp32
template <> struct Vec8<__half> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const uint4& u, float* f) {
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __half22float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  static __device__ __forceinline__ uint4 store(const float* f) {
    uint4 u;
    __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
    return u;
  }
};
template <> struct Vec8<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const uint4& u, float* f) {
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ uint4 store(const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return u;
  }
};
template <> struct Vec8<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
  static __device__ __forceinline__ uint4 store(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

template <typename T>
__global__ void __launch_bounds__(kThreadsSw) sswiglu_dwconv_kernel(const __grid_constant__ SwParams sp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* halo = smem;               // [kTH+2][kTW+2][kCB bytes]
  uint8_t* xgt = smem + kHaloBytes;   // [kTH][kTW][kCB bytes]
  __shared__ uint64_t full;
  __shared__ float wsm[kCB / sizeof(T)][9];  // this block's weights
  __shared__ float bsm[kCB / sizeof(T)];
  constexpr int kCh = kCB / (int)sizeof(T);  // channels per block
  constexpr int kN = Vec8<T>::N;             // channels per 16-byte piece

  // channel blocks vary fastest: the CTAs running at once read whole token rows
  // (C channels contiguous in memory) instead of one 128-byte piece of each token
  int t = blockIdx.x;
  const int cb = t % sp.cblocks;
  t /= sp.cblocks;
  const int tx = t % sp.tiles_x;
  t /= sp.tiles_x;
  const int ty = t % sp.tiles_y;
  const int b = t / sp.tiles_y;
  const int x0 = tx * kTW, y0 = ty * kTH, c0 = cb * kCh;
  const int tid = threadIdx.x;

  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid == 0) {
    mbar_init(&full, 1);
    fence_mbar_init();
  }
  __syncthreads();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    mbar_arrive_expect_tx(&full, (uint32_t)(kHaloBytes + kXgBytes));
    // the halo box starts one row and one column early; outside the grid it reads zeros
    tma_load_4d(halo, &sp.txv, &full, c0, x0 - 1, y0 - 1, b);
    tma_load_4d(xgt, &sp.txg, &full, c0, x0, y0, b);
  }
  for (int i = tid; i < kCh * 9; i += kThreadsSw) wsm[i / 9][i % 9] = __ldg(sp.w + (size_t)c0 * 9 + i);
  if (tid < kCh) bsm[tid] = sp.b ? __ldg(sp.b + c0 + tid) : 0.f;
  __syncthreads();
  // bounded wait for the tiles (about a second), then give up without touching them
  bool ok = mbar_wait_sleep(&full, 0, 1000000u);
  for (int it = 0; !ok && it < 1000; ++it) ok = mbar_wait_sleep(&full, 0, 1000000u);
  if (!ok) return;

  // Thread t: 16-byte channel piece j = t % 8 of column c = (t / 8) % 16 of the tile, output
  // rows 4q .. 4q + 3 (q = t / 128).  Its nine taps and bias live in registers; it walks the
  // six halo rows those outputs need once, each neighbour feeding every output it touches,
  // so a halo element is loaded and converted twice on average instead of nine times.
  constexpr int kPieces = kCB / 16;  // 8
  constexpr int kRows = kTH * kTW * kPieces / kThreadsSw;  // 4 output rows a thread
  static_assert(kTW * kPieces * (kTH / kRows) == kThreadsSw, "one column strip of kRows rows per thread");
  const int j = tid % kPieces, c = (tid / kPieces) % kTW, q = tid / (kPieces * kTW);
  float wr[9][kN], acc[kRows][kN];
#pragma unroll
  for (int e = 0; e < kN; ++e) {
#pragma unroll
    for (int tap = 0; tap < 9; ++tap) wr[tap][e] = wsm[j * kN + e][tap];
#pragma unroll
    for (int k = 0; k < kRows; ++k) acc[k][e] = bsm[j * kN + e];
  }
#pragma unroll
  for (int hr = 0; hr < kRows + 2; ++hr) {  // halo row kRows q + hr
#pragma unroll
    for (int dx = 0; dx < 3; ++dx) {
      float f[kN];
      Vec8<T>::load(*reinterpret_cast<const uint4*>(halo + ((kRows * q + hr) * (kTW + 2) + (c + dx)) * kCB + 16 * j), f);
#pragma unroll
      for (int k = 0; k < kRows; ++k) {
        const int dy = hr - k;  // output row kRows q + k takes halo rows k .. k + 2
        if (dy >= 0 && dy < 3) {
#pragma unroll
          for (int e = 0; e < kN; ++e) acc[k][e] = fmaf(wr[3 * dy + dx][e], f[e], acc[k][e]);
        }
      }
    }
  }
  const int x = x0 + c;
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int r = kRows * q + k, y = y0 + r;
    if (y >= sp.H || x >= sp.W) continue;
    float g[kN];
    Vec8<T>::load(*reinterpret_cast<const uint4*>(xgt + (r * kTW + c) * kCB + 16 * j), g);
#pragma unroll
    for (int e = 0; e < kN; ++e) acc[k][e] *= __fdividef(g[e], 1.f + __expf(-g[e]));  // SiLU(xg)
    T* o = reinterpret_cast<T*>(sp.out) + (((size_t)b * sp.H + y) * sp.W + x) * sp.C + c0 + j * kN;
    __stcs(reinterpret_cast<uint4*>(o), Vec8<T>::store(acc[k]));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 sw_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool sw_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int es, int B, int H, int W, int C, int bw,
            int bh) {
  auto enc = sw_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)C * es, (cuuint64_t)W * C * es, (cuuint64_t)H * W * C * es};
  cuuint32_t box[4] = {(cuuint32_t)(kCB / es), (cuuint32_t)bw, (cuuint32_t)bh, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T>
gtr_status_t launch_sw(const void* xg, const void* xv, const float* w, const float* bias, void* out, int B, int H,
                       int W, int C, CUtensorMapDataType dt, cudaStream_t stream) {
  SwParams sp;
  constexpr int es = (int)sizeof(T);
  if (!sw_map(&sp.txv, xv, dt, es, B, H, W, C, kTW + 2, kTH + 2) || !sw_map(&sp.txg, xg, dt, es, B, H, W, C, kTW, kTH))
    return GTR_ERR_CUDA;
  sp.out = out;
  sp.w = w;
  sp.b = bias;
  sp.B = B;
  sp.H = H;
  sp.W = W;
  sp.C = C;
  sp.tiles_x = (W + kTW - 1) / kTW;
  sp.tiles_y = (H + kTH - 1) / kTH;
  sp.cblocks = C / (kCB / es);
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(sswiglu_dwconv_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemSw);
  });
  if (attr != cudaSuccess) return GTR_ERR_CUDA;
  const long long grid = (long long)sp.tiles_x * sp.tiles_y * sp.cblocks * B;
  if (grid > 0x7fffffffll) return GTR_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreadsSw);
  cfg.dynamicSmemBytes = kSmemSw;
  cfg.stream = stream;
  cudaLaunchAttribute a[1];
  a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = a;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sswiglu_dwconv_kernel<T>, sp) == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace gtr

extern "C" gtr_status_t gtr_sswiglu_dwconv(const void* xg, const void* xv, const float* conv_w,
                                           const float* conv_b, void* out, int B, int grid_H, int grid_W, int C,
                                           int dtype, gtr_stream_t stream) {
  using namespace gtr;
  if (!xg || !xv || !conv_w || !out || B <= 0 || grid_H <= 0 || grid_W <= 0 || C <= 0) return GTR_ERR_INVALID_ARG;
  if (!aligned16(xg) || !aligned16(xv) || !aligned16(out) || (reinterpret_cast<uintptr_t>(conv_w) & 3u) ||
      (conv_b && (reinterpret_cast<uintptr_t>(conv_b) & 3u)))
    return GTR_ERR_INVALID_ARG;
  if (dtype < GTR_F32 || dtype > GTR_BF16) return GTR_ERR_INVALID_ARG;
  const int es = dtype == GTR_F32 ? 4 : 2;
  if (C % (kCB / es) != 0) return GTR_ERR_UNSUPPORTED;  // whole 128-byte channel blocks
  if ((long long)B * grid_H * grid_W * C >= (1ll << 40) || grid_H > (1 << 24) || grid_W > (1 << 24))
    return GTR_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (dtype) {
    case GTR_F16:
      return launch_sw<__half>(xg, xv, conv_w, conv_b, out, B, grid_H, grid_W, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, s);
    case GTR_BF16:
      return launch_sw<__nv_bfloat16>(xg, xv, conv_w, conv_b, out, B, grid_H, grid_W, C,
                                      CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, s);
    default:
      return launch_sw<float>(xg, xv, conv_w, conv_b, out, B, grid_H, grid_W, C, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, s);
  }
}
