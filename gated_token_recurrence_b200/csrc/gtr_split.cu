// Split path: three launches, any input dtype, fp32 FFMA arithmetic.
//
//   1. split_summary_kernel  one CTA per (chunk, head, batch): in-chunk cumulative
//                            log-gates A, chunk log-decay a_last = A[C-1] and the
//                            summary U_c = (K * exp(a_last - A))^T V.
//   2. split_scan_kernel     one thread per state entry: S_[0] = 0,
//                            S_[c+1] = Diag(exp(a_last_c)) S_[c] + U_c.
//   3. split_output_kernel   one CTA per chunk: o = d_k^{-1/2} [ (Q*exp(A)) S_[c]
//                            + masked intra-chunk term ] stored at the grid cells.
//
// These are the three stages of the chunkwise operator described on page
// 0539edu.com, section 3.3 (chunk summaries in parallel -> light boundary-state
// scan -> independent chunk outputs) and on the first GTR page, prerequisite
// "Chunkwise parallel".  Every exponent is a product of gates (<= 1): the
// intra-chunk term factorises exp(A_i - A_j) through a reference position r with
// j <= r <= i, so neither factor exceeds 1, and the 16x16 diagonal blocks use the
// direct exp(A_i - A_j).  Nothing overflows for any log_gamma <= 0.
#include <atomic>

#include "gtr_common.cuh"
#include "gtr_internal.h"

namespace gtr {
namespace {

constexpr int LD = kD + 1;  // padded smem row (floats)
constexpr int kTile = kChunk * LD;

// log gamma of channels g .. g+3 of scan position s of (b, h) from the low-rank gate
// producer: logsigmoid(z W2 + bias) / tau (the rank-r projection z of the token).
__device__ __forceinline__ float4 lowrank_log_gamma4(const Problem& p, int b, int h, long long s, int g) {
  const long long m = scan_to_token(s, p.direction, p.H, p.W);
  const float* z = p.gz + ((long long)b * p.L() + m) * p.grank;
  const int col = h * p.d_k + g, ld = p.heads * p.d_k;
  float x[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = p.gb[col + e];
  for (int i = 0; i < p.grank; ++i) {
    const float zi = z[i];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = fmaf(zi, p.gw2[(long long)i * ld + col + e], x[e]);
  }
  float r[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) r[e] = (fminf(x[e], 0.f) - log1pf(expf(-fabsf(x[e])))) / p.gtau;
  return make_float4(r[0], r[1], r[2], r[3]);
}

// Load one chunk's rows (scan positions c*64 + r) of up to four tensors into
// padded fp32 smem; rows past the sequence end are zero (log-gate 0 = no decay).  q, k
// and the log-gates have d_k channels a row (32 or 64): key channels d_k .. 63 are zero,
// so they add nothing to any product and the state rows they would feed stay zero.
template <typename Tin>
__device__ __forceinline__ void load_chunk(const Problem& p, int b, int h, int c,
                                           const Tin* q, const Tin* k, const Tin* v,
                                           float* Qs, float* Ks, float* Vs, float* Gs) {
  const long long L = p.L();
  for (int idx = threadIdx.x; idx < kChunk * (kD / 4); idx += blockDim.x) {
    const int r = idx >> 4, g = (idx & 15) * 4;
    const long long s = (long long)c * kChunk + r;
    float4 qq = make_float4(0.f, 0.f, 0.f, 0.f), kk = qq, vv = qq, gg = qq;
    if (s < L) {
      const long long th = token_head_row(p, b, h, s);
      const long long rk = th * p.d_k + g, rv = th * kD + g;
      if (g < p.d_k) {
        if (Qs) qq = load4<Tin>(q + rk);
        if (Ks) kk = load4<Tin>(k + rk);
        if (Gs) gg = p.gz ? lowrank_log_gamma4(p, b, h, s, g) : load4<float>(p.log_gamma + rk);
      }
      if (Vs) vv = load4<Tin>(v + rv);
    }
    const int o = r * LD + g;
    if (Qs) { Qs[o] = qq.x; Qs[o + 1] = qq.y; Qs[o + 2] = qq.z; Qs[o + 3] = qq.w; }
    if (Ks) { Ks[o] = kk.x; Ks[o + 1] = kk.y; Ks[o + 2] = kk.z; Ks[o + 3] = kk.w; }
    if (Vs) { Vs[o] = vv.x; Vs[o + 1] = vv.y; Vs[o + 2] = vv.z; Vs[o + 3] = vv.w; }
    if (Gs) { Gs[o] = gg.x; Gs[o + 1] = gg.y; Gs[o + 2] = gg.z; Gs[o + 3] = gg.w; }
  }
}

// In-place inclusive cumulative sum over the chunk's rows, per channel.
__device__ __forceinline__ void cumsum_rows(float* As) {
  if (threadIdx.x < kD) {
    float a = 0.f;
    for (int r = 0; r < kChunk; ++r) {
      a += As[r * LD + threadIdx.x];
      As[r * LD + threadIdx.x] = a;
    }
  }
}

template <typename Tin>
__global__ void __launch_bounds__(256) split_summary_kernel(Problem p, float* __restrict__ U,
                                                            float* __restrict__ a_last) {
  extern __shared__ float sm[];
  float* Ks = sm;
  float* Vs = Ks + kTile;
  float* As = Vs + kTile;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int Nc = p.n_chunks();

  load_chunk<Tin>(p, b, h, c, nullptr, (const Tin*)p.k, (const Tin*)p.v, nullptr, Ks, Vs, As);
  __syncthreads();
  cumsum_rows(As);
  __syncthreads();
  // K~ = K * exp(a_last - A): each factor is a product of later gates, <= 1
  for (int idx = tid; idx < kChunk * kD; idx += 256) {
    const int r = idx >> 6, ch = idx & 63;
    Ks[r * LD + ch] *= expf(As[(kChunk - 1) * LD + ch] - As[r * LD + ch]);
  }
  __syncthreads();
  // U[ch][j] = sum_r K~[r][ch] V[r][j]   (4x4 register tile per thread)
  const int ch0 = (tid >> 4) * 4, j0 = (tid & 15) * 4;
  float acc[4][4] = {};
#pragma unroll 4
  for (int r = 0; r < kChunk; ++r) {
    float a[4], bv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[e] = Ks[r * LD + ch0 + e];
      bv[e] = Vs[r * LD + j0 + e];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int f = 0; f < 4; ++f) acc[e][f] = fmaf(a[e], bv[f], acc[e][f]);
  }
  const size_t unit = ((size_t)b * p.heads + h) * Nc + c;
  float* Ub = U + unit * (kD * kD);
#pragma unroll
  for (int e = 0; e < 4; ++e)
    *reinterpret_cast<float4*>(Ub + (ch0 + e) * kD + j0) =
        make_float4(acc[e][0], acc[e][1], acc[e][2], acc[e][3]);
  if (tid < kD) a_last[unit * kD + tid] = As[(kChunk - 1) * LD + tid];
}

// One thread per state entry (ch, j) of one (batch, head); walks the chunks in order
// and writes the state at the START of every chunk.
__global__ void __launch_bounds__(256) split_scan_kernel(const float* __restrict__ U,
                                                         const float* __restrict__ a_last,
                                                         float* __restrict__ S, int Nc) {
  const size_t bh = blockIdx.x;
  const int e = blockIdx.y * 256 + threadIdx.x;
  const int ch = e >> 6;
  const float* Ub = U + bh * Nc * (kD * kD) + e;
  const float* ab = a_last + bh * Nc * kD + ch;
  float* Sb = S + bh * Nc * (kD * kD) + e;
  float st = 0.f;
#pragma unroll 8
  for (int c = 0; c < Nc; ++c) {
    Sb[(size_t)c * (kD * kD)] = st;
    st = fmaf(expf(ab[(size_t)c * kD]), st, Ub[(size_t)c * (kD * kD)]);
  }
}

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) split_output_kernel(Problem p, const float* __restrict__ S) {
  extern __shared__ float sm[];
  float* Qs = sm;
  float* Ks = Qs + kTile;
  float* Vs = Ks + kTile;
  float* As = Vs + kTile;
  float* Ss = As + kTile;
  float* Qh = Ss + kTile;
  float* Kt = Qh + kTile;
  float* Qt = Kt + kTile;  // three tiles: reference rows 15, 31, 47
  float* Ps = Qt + 3 * kTile;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int Nc = p.n_chunks();
  const long long L = p.L();
  const size_t unit = ((size_t)b * p.heads + h) * Nc + c;

  load_chunk<Tin>(p, b, h, c, (const Tin*)p.q, (const Tin*)p.k, (const Tin*)p.v, Qs, Ks, Vs, As);
  {
    const float* Sg = S + unit * (kD * kD);
    for (int idx = tid; idx < kD * (kD / 4); idx += 256) {
      const int r = idx >> 4, g = (idx & 15) * 4;
      const float4 x = *reinterpret_cast<const float4*>(Sg + r * kD + g);
      Ss[r * LD + g] = x.x; Ss[r * LD + g + 1] = x.y; Ss[r * LD + g + 2] = x.z; Ss[r * LD + g + 3] = x.w;
    }
  }
  __syncthreads();
  cumsum_rows(As);
  __syncthreads();
  // Qh = Q exp(A);  Kt[j] = K[j] exp(A[r(j)] - A[j]), r(j) = last row of j's 16-block;
  // Qt_J[i] = Q[i] exp(A[i] - A[16J+15]) for rows i past block J.  All factors <= 1.
  for (int idx = tid; idx < kChunk * kD; idx += 256) {
    const int r = idx >> 6, ch = idx & 63;
    const float a = As[r * LD + ch];
    const float qv = Qs[r * LD + ch];
    Qh[r * LD + ch] = qv * expf(a);
    Kt[r * LD + ch] = Ks[r * LD + ch] * expf(As[(r | 15) * LD + ch] - a);
#pragma unroll
    for (int J = 0; J < 3; ++J)
      if (r >= 16 * (J + 1)) Qt[J * kTile + r * LD + ch] = qv * expf(a - As[(16 * J + 15) * LD + ch]);
  }
  __syncthreads();

  const int i0 = (tid >> 4) * 4, j0 = (tid & 15) * 4;
  // intra-chunk scores P[i][j], j <= i
  {
    float P[4][4] = {};
    const int I = i0 >> 4, J = j0 >> 4;
    if (J < I) {
      const float* Qa = Qt + J * kTile;
#pragma unroll 4
      for (int k = 0; k < kD; ++k) {
        float a[4], bv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          a[e] = Qa[(i0 + e) * LD + k];
          bv[e] = Kt[(j0 + e) * LD + k];
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int f = 0; f < 4; ++f) P[e][f] = fmaf(a[e], bv[f], P[e][f]);
      }
    } else if (J == I && j0 <= i0) {
      for (int k = 0; k < kD; ++k) {
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int f = 0; f < 4; ++f)
            if (j0 + f <= i0 + e)
              P[e][f] = fmaf(Qs[(i0 + e) * LD + k] * Ks[(j0 + f) * LD + k],
                             expf(As[(i0 + e) * LD + k] - As[(j0 + f) * LD + k]), P[e][f]);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int f = 0; f < 4; ++f) Ps[(i0 + e) * LD + j0 + f] = P[e][f];
  }
  __syncthreads();

  // o[i][jv] = sum_k Qh[i][k] S[k][jv] + sum_{j<=i} P[i][j] V[j][jv]
  float acc[4][4] = {};
#pragma unroll 4
  for (int k = 0; k < kD; ++k) {
    float a[4], bv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[e] = Qh[(i0 + e) * LD + k];
      bv[e] = Ss[k * LD + j0 + e];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int f = 0; f < 4; ++f) acc[e][f] = fmaf(a[e], bv[f], acc[e][f]);
  }
  const int jmax = i0 + 4;
  for (int j = 0; j < jmax; ++j) {
    float a[4], bv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[e] = Ps[(i0 + e) * LD + j];
      bv[e] = Vs[j * LD + j0 + e];
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int f = 0; f < 4; ++f) acc[e][f] = fmaf(a[e], bv[f], acc[e][f]);
  }
  const float scale = rsqrtf((float)p.d_k);
  Tout* out = (Tout*)p.out;
#pragma unroll
  for (int e = 0; e < 4; ++e)
#pragma unroll
    for (int f = 0; f < 4; ++f) acc[e][f] *= scale;
  if (p.ogate) {
    // RMSNorm over the 64 value channels of each row (held by the 16 threads tid & 15 of
    // its row group, consecutive lanes), the norm weight and the SiLU output gate
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float ss = acc[e][0] * acc[e][0] + acc[e][1] * acc[e][1] + acc[e][2] * acc[e][2] + acc[e][3] * acc[e][3];
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float rinv = rsqrtf(ss * (1.f / kD) + p.oeps);
      const long long s = (long long)c * kChunk + i0 + e;
      if (s < L) {
        const long long row = token_head_row(p, b, h, s);
        const float4 gt = load4<Tin>(reinterpret_cast<const Tin*>(p.ogate) + row * kD + j0);
        const float gv[4] = {gt.x, gt.y, gt.z, gt.w};
#pragma unroll
        for (int f = 0; f < 4; ++f)
          acc[e][f] = acc[e][f] * rinv * p.onorm_w[j0 + f] * (gv[f] / (1.f + expf(-gv[f])));
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const long long s = (long long)c * kChunk + i0 + e;
    if (s < L) {
      const long long row = token_head_row(p, b, h, s);
      store4<Tout>(out + row * kD + j0, make_float4(acc[e][0], acc[e][1], acc[e][2], acc[e][3]));
    }
  }
}

constexpr size_t kSummarySmem = 3 * kTile * sizeof(float);
constexpr size_t kOutputSmem = 11 * kTile * sizeof(float);

template <typename Tin, typename Tout>
gtr_status_t launch_split_typed(const Problem& p, const SplitWorkspace& ws, cudaStream_t stream) {
  // dynamic smem above 48 KB needs an opt-in, once per device (kept out of later graph captures)
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GTR_ERR_CUDA;
  if (!(configured.load() & (1ull << dev))) {
    if (cudaFuncSetAttribute(split_summary_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSummarySmem) != cudaSuccess ||
        cudaFuncSetAttribute(split_output_kernel<Tin, Tout>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kOutputSmem) != cudaSuccess)
      return GTR_ERR_CUDA;
    configured.fetch_or(1ull << dev);
  }
  const int Nc = p.n_chunks();
  const dim3 grid(Nc, p.heads, p.B);
  split_summary_kernel<Tin><<<grid, 256, kSummarySmem, stream>>>(p, ws.U, ws.a_last);
  split_scan_kernel<<<dim3(p.B * p.heads, (kD * kD) / 256), 256, 0, stream>>>(ws.U, ws.a_last, ws.S, Nc);
  split_output_kernel<Tin, Tout><<<grid, 256, kOutputSmem, stream>>>(p, ws.S);
  return cudaGetLastError() == cudaSuccess ? GTR_OK : GTR_ERR_CUDA;
}

}  // namespace

size_t split_workspace_bytes(const Problem& p) {
  const size_t units = (size_t)p.B * p.heads * p.n_chunks();
  return kWsPrefixBytes + units * kSplitUnitBytes;
}

SplitWorkspace split_workspace_carve(void* ws, const Problem& p) {
  const size_t units = (size_t)p.B * p.heads * p.n_chunks();
  SplitWorkspace w;
  w.hdr = reinterpret_cast<WsHeader*>(ws);
  float* base = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kWsPrefixBytes);
  w.U = base;
  w.S = base + units * kD * kD;
  w.a_last = base + 2 * units * kD * kD;
  return w;
}

gtr_status_t launch_split(const Problem& p, void* ws, cudaStream_t stream) {
  const SplitWorkspace w = split_workspace_carve(ws, p);
  switch (p.in_dtype * 3 + p.out_dtype) {
    case GTR_F32 * 3 + GTR_F32: return launch_split_typed<float, float>(p, w, stream);
    case GTR_F16 * 3 + GTR_F16: return launch_split_typed<__half, __half>(p, w, stream);
    case GTR_F16 * 3 + GTR_F32: return launch_split_typed<__half, float>(p, w, stream);
    case GTR_BF16 * 3 + GTR_F32: return launch_split_typed<__nv_bfloat16, float>(p, w, stream);
    case GTR_BF16 * 3 + GTR_BF16: return launch_split_typed<__nv_bfloat16, __nv_bfloat16>(p, w, stream);
    default: return GTR_ERR_UNSUPPORTED;
  }
}

}  // namespace gtr
