// C ABI of libgtr.so: argument validation, workspace management, length-aware
// dispatch and the host-buffer entry.  The arithmetic lives in the kernel files.
#include <cstddef>
#include <mutex>
#include <vector>

#include "gtr_common.cuh"
#include "gtr_internal.h"

namespace gtr {
namespace {

constexpr int kMaxDevices = 64;

bool is_aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

size_t elem_size(int dt) { return dt == GTR_F32 ? 4 : 2; }

bool dtype_pair_ok(int in, int out) {
  switch (in) {
    case GTR_F32: return out == GTR_F32;
    case GTR_F16: return out == GTR_F16 || out == GTR_F32;
    case GTR_BF16: return out == GTR_F32 || out == GTR_BF16;
    default: return false;
  }
}

// Shape-only checks shared by every entry point.
gtr_status_t check_shape(int B, int heads, int H, int W, int d_k, int d_v, int direction,
                         int in_dtype, int out_dtype) {
  if (B <= 0 || heads <= 0 || H <= 0 || W <= 0 || d_k <= 0 || d_v <= 0) return GTR_ERR_INVALID_ARG;
  if (direction < GTR_L2R || direction > GTR_B2T) return GTR_ERR_INVALID_ARG;
  if (in_dtype < GTR_F32 || in_dtype > GTR_BF16 || out_dtype < GTR_F32 || out_dtype > GTR_BF16)
    return GTR_ERR_INVALID_ARG;
  if (!dtype_pair_ok(in_dtype, out_dtype)) return GTR_ERR_UNSUPPORTED;
  if ((d_k != kD && d_k != 32) || d_v != kD) return GTR_ERR_UNSUPPORTED;
  const long long L = (long long)H * W;
  if (L > (1ll << 28) || B > 65535 || heads > 65535) return GTR_ERR_UNSUPPORTED;
  if ((long long)B * L * heads * kD >= (1ll << 40)) return GTR_ERR_UNSUPPORTED;
  return GTR_OK;
}

gtr_status_t check_ptrs(const void* q, const void* k, const void* v, const float* g, void* out) {
  if (!q || !k || !v || !g || !out) return GTR_ERR_INVALID_ARG;
  if (!is_aligned(q, 16) || !is_aligned(k, 16) || !is_aligned(v, 16) || !is_aligned(g, 16) ||
      !is_aligned(out, 16))
    return GTR_ERR_INVALID_ARG;
  return GTR_OK;
}

Problem make_problem(const void* q, const void* k, const void* v, const float* g, void* out, int B,
                     int heads, int H, int W, int d_k, int d_v, int direction, int in_dtype,
                     int out_dtype) {
  Problem p;
  p.q = q; p.k = k; p.v = v; p.log_gamma = g; p.out = out;
  p.B = B; p.heads = heads; p.H = H; p.W = W; p.d_k = d_k; p.d_v = d_v;
  p.direction = direction; p.in_dtype = in_dtype; p.out_dtype = out_dtype;
  return p;
}

// Length-aware dispatch.  The fused tensor-core path takes fp16/bf16 inputs;
// fp32 inputs (exact FFMA arithmetic) and sequences shorter than one chunk take the
// split path.  For a single partial chunk the fp16 rounding of the gate-scaled
// operands is no longer averaged over many tokens (a cancelling dot product can
// dominate the output), so such sequences run on the split path even when a fused
// path is requested: every path then meets the same accuracy bound.
int choose_path(const Problem& p, int requested) {
  if (p.L() < kChunk) return GTR_PATH_SPLIT;
  if (requested != GTR_PATH_AUTO) return requested;
  if (p.in_dtype == GTR_F32) return GTR_PATH_SPLIT;
  return GTR_PATH_FUSED;
}

bool fused_ok(const Problem& p) {
  return p.in_dtype != GTR_F32 && (long long)p.B * p.L() < (1ll << 31);
}

size_t path_workspace_bytes(const Problem& p, int path) {
  switch (path) {
    case GTR_PATH_SPLIT: return split_workspace_bytes(p);
    case GTR_PATH_FUSED:
    case GTR_PATH_FUSED_SEQUENTIAL: return fused_ok(p) ? fused_workspace_bytes(p) : 0;
    default: return 0;
  }
}

int path_launches(const Problem& p, int path) {
  switch (path) {
    case GTR_PATH_SPLIT: return 3;
    case GTR_PATH_FUSED:
    case GTR_PATH_FUSED_SEQUENTIAL: return fused_launches(p);
    default: return 0;
  }
}

// ---- library-owned per-device buffers ------------------------------------------------
struct DeviceBuffer {
  void* ptr = nullptr;
  size_t bytes = 0;
};

struct DeviceCache {
  std::mutex mu;
  DeviceBuffer ws;                  // workspace for gtr_gla_fwd / typed forms
  DeviceBuffer io[5];               // q, k, v, log_gamma, out for the host-buffer entry
  unsigned int* err_host = nullptr;  // pinned word: the error word read back with the output
};

DeviceCache g_cache[kMaxDevices];

gtr_status_t current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) return GTR_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return GTR_ERR_UNSUPPORTED;
  return GTR_OK;
}

// Grow `buf` to at least `bytes`.  Refuses while `stream` is capturing.
gtr_status_t ensure(DeviceBuffer& buf, size_t bytes, cudaStream_t stream) {
  if (buf.bytes >= bytes && buf.ptr) return GTR_OK;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return GTR_ERR_CUDA;
  if (cs != cudaStreamCaptureStatusNone) return GTR_ERR_WORKSPACE;
  if (buf.ptr) {
    // earlier calls may still use the old buffer; cudaFree waits for the device
    if (cudaFree(buf.ptr) != cudaSuccess) return GTR_ERR_CUDA;
    buf.ptr = nullptr;
    buf.bytes = 0;
  }
  size_t want = bytes < 256 ? 256 : bytes;
  want = (want + 255) & ~size_t(255);
  if (cudaMalloc(&buf.ptr, want) != cudaSuccess) {
    buf.ptr = nullptr;
    cudaGetLastError();
    return GTR_ERR_CUDA;
  }
  // a zeroed workspace is a ready one (clear error word, counters and flags)
  if (cudaMemsetAsync(buf.ptr, 0, want, stream) != cudaSuccess) return GTR_ERR_CUDA;
  buf.bytes = want;
  return GTR_OK;
}

gtr_status_t run(const Problem& p, int path, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const int chosen = choose_path(p, path);
  const size_t need = path_workspace_bytes(p, chosen);
  if (need == 0) return GTR_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < need || !is_aligned(ws, 256)) return GTR_ERR_WORKSPACE;
  switch (chosen) {
    case GTR_PATH_SPLIT: return launch_split(p, ws, stream);
    case GTR_PATH_FUSED: return launch_fused(p, ws, stream, -1);
    case GTR_PATH_FUSED_SEQUENTIAL: return launch_fused(p, ws, stream, 0);
    default: return GTR_ERR_UNSUPPORTED;
  }
}

gtr_status_t fwd_internal_ws(const Problem& p, cudaStream_t stream) {
  int dev;
  gtr_status_t st = current_device(&dev);
  if (st != GTR_OK) return st;
  DeviceCache& c = g_cache[dev];
  std::lock_guard<std::mutex> lock(c.mu);
  const int path = choose_path(p, GTR_PATH_AUTO);
  const size_t need = path_workspace_bytes(p, path);
  if (need == 0) return GTR_ERR_UNSUPPORTED;
  st = ensure(c.ws, need, stream);
  if (st != GTR_OK) return st;
  return run(p, path, c.ws.ptr, c.ws.bytes, stream);
}

}  // namespace

gtr_status_t validate_call(const void* q, const void* k, const void* v, const float* log_gamma, void* out,
                           int B, int heads, int grid_H, int grid_W, int d_k, int d_v, int direction,
                           int in_dtype, int out_dtype) {
  const gtr_status_t st = check_shape(B, heads, grid_H, grid_W, d_k, d_v, direction, in_dtype, out_dtype);
  return st != GTR_OK ? st : check_ptrs(q, k, v, log_gamma, out);
}

}  // namespace gtr

using namespace gtr;

extern "C" {

gtr_status_t gtr_gla_fwd(const void* q, const void* k, const void* v, const float* log_gamma,
                         void* out, int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                         int direction, int in_dtype, int out_dtype, gtr_stream_t stream) {
  gtr_status_t st = check_shape(B, heads, grid_H, grid_W, d_k, d_v, direction, in_dtype, out_dtype);
  if (st != GTR_OK) return st;
  st = check_ptrs(q, k, v, log_gamma, out);
  if (st != GTR_OK) return st;
  const Problem p = make_problem(q, k, v, log_gamma, out, B, heads, grid_H, grid_W, d_k, d_v,
                                 direction, in_dtype, out_dtype);
  return fwd_internal_ws(p, reinterpret_cast<cudaStream_t>(stream));
}

gtr_status_t gtr_gla_fwd_f16(const void* q, const void* k, const void* v, const float* log_gamma,
                             void* out, int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                             int direction, gtr_stream_t stream) {
  return gtr_gla_fwd(q, k, v, log_gamma, out, B, heads, grid_H, grid_W, d_k, d_v, direction,
                     GTR_F16, GTR_F16, stream);
}

gtr_status_t gtr_gla_fwd_bf16(const void* q, const void* k, const void* v, const float* log_gamma,
                              void* out, int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                              int direction, gtr_stream_t stream) {
  return gtr_gla_fwd(q, k, v, log_gamma, out, B, heads, grid_H, grid_W, d_k, d_v, direction,
                     GTR_BF16, GTR_F32, stream);
}

gtr_status_t gtr_gla_fwd_f32(const void* q, const void* k, const void* v, const float* log_gamma,
                             void* out, int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                             int direction, gtr_stream_t stream) {
  return gtr_gla_fwd(q, k, v, log_gamma, out, B, heads, grid_H, grid_W, d_k, d_v, direction,
                     GTR_F32, GTR_F32, stream);
}

size_t gtr_gla_workspace_bytes(int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                               int in_dtype, int path) {
  const int out_dtype = in_dtype == GTR_F16 ? GTR_F16 : GTR_F32;
  if (check_shape(B, heads, grid_H, grid_W, d_k, d_v, GTR_L2R, in_dtype, out_dtype) != GTR_OK) return 0;
  if (path < GTR_PATH_AUTO || path > GTR_PATH_FUSED_SEQUENTIAL) return 0;
  const Problem p = make_problem(nullptr, nullptr, nullptr, nullptr, nullptr, B, heads, grid_H,
                                 grid_W, d_k, d_v, GTR_L2R, in_dtype, out_dtype);
  if (path != GTR_PATH_AUTO) return path_workspace_bytes(p, choose_path(p, path));
  size_t m = 0;
  for (int pth = GTR_PATH_SPLIT; pth <= GTR_PATH_FUSED_SEQUENTIAL; ++pth) {
    const size_t b = path_workspace_bytes(p, pth);
    if (b > m) m = b;
  }
  return m;
}

gtr_status_t gtr_gla_fwd_ex(const void* q, const void* k, const void* v, const float* log_gamma,
                            void* out, int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                            int direction, int in_dtype, int out_dtype, int path, void* workspace,
                            size_t ws_bytes, gtr_stream_t stream) {
  gtr_status_t st = check_shape(B, heads, grid_H, grid_W, d_k, d_v, direction, in_dtype, out_dtype);
  if (st != GTR_OK) return st;
  st = check_ptrs(q, k, v, log_gamma, out);
  if (st != GTR_OK) return st;
  if (path < GTR_PATH_AUTO || path > GTR_PATH_FUSED_SEQUENTIAL) return GTR_ERR_INVALID_ARG;
  const Problem p = make_problem(q, k, v, log_gamma, out, B, heads, grid_H, grid_W, d_k, d_v,
                                 direction, in_dtype, out_dtype);
  return run(p, path, workspace, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

gtr_status_t gtr_gla_block_fwd(const void* q, const void* k, const void* v, const float* log_gamma,
                               const float* gate_z, const float* gate_w2, const float* gate_b, int gate_rank,
                               float gate_tau, const void* out_gate, const float* norm_w, float norm_eps, void* out,
                               int B, int heads, int grid_H, int grid_W, int d_k, int d_v, int direction,
                               int in_dtype, int out_dtype, int path, void* workspace, size_t ws_bytes,
                               gtr_stream_t stream) {
  gtr_status_t st = check_shape(B, heads, grid_H, grid_W, d_k, d_v, direction, in_dtype, out_dtype);
  if (st != GTR_OK) return st;
  // exactly one source of the gates
  if ((log_gamma == nullptr) == (gate_z == nullptr)) return GTR_ERR_INVALID_ARG;
  const float* lg = log_gamma ? log_gamma : gate_z;  // (pointer checks below cover both)
  st = check_ptrs(q, k, v, lg, out);
  if (st != GTR_OK) return st;
  if (gate_z) {
    if (!gate_w2 || !gate_b || !is_aligned(gate_w2, 16) || !is_aligned(gate_b, 16)) return GTR_ERR_INVALID_ARG;
    if (gate_rank != 8 && gate_rank != 16) return GTR_ERR_INVALID_ARG;
    if (!(gate_tau > 0.f) || !(gate_tau < 3.0e38f)) return GTR_ERR_INVALID_ARG;
  }
  if (out_gate) {
    if (!norm_w || !is_aligned(out_gate, 16) || !is_aligned(norm_w, 16)) return GTR_ERR_INVALID_ARG;
    if (!(norm_eps >= 0.f) || !(norm_eps < 3.0e38f)) return GTR_ERR_INVALID_ARG;
  }
  if (path < GTR_PATH_AUTO || path > GTR_PATH_FUSED_SEQUENTIAL) return GTR_ERR_INVALID_ARG;
  Problem p = make_problem(q, k, v, log_gamma, out, B, heads, grid_H, grid_W, d_k, d_v, direction, in_dtype,
                           out_dtype);
  if (gate_z) {
    p.gz = gate_z;
    p.gw2 = gate_w2;
    p.gb = gate_b;
    p.grank = gate_rank;
    p.gtau = gate_tau;
  }
  if (out_gate) {
    p.ogate = out_gate;
    p.onorm_w = norm_w;
    p.oeps = norm_eps;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (workspace) return run(p, path, workspace, ws_bytes, s);
  int dev;
  st = current_device(&dev);
  if (st != GTR_OK) return st;
  DeviceCache& c = g_cache[dev];
  std::lock_guard<std::mutex> lock(c.mu);
  const size_t need = path_workspace_bytes(p, choose_path(p, path));
  if (need == 0) return GTR_ERR_UNSUPPORTED;
  st = ensure(c.ws, need, s);
  if (st != GTR_OK) return st;
  return run(p, path, c.ws.ptr, c.ws.bytes, s);
}

gtr_status_t gtr_gla_workspace_debug(void* workspace, int skip_segment, unsigned int wait_limit_us,
                                     gtr_stream_t stream) {
  if (!workspace || !is_aligned(workspace, 256)) return GTR_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return GTR_ERR_CUDA;
  const unsigned int v[2] = {skip_segment >= 0 ? (unsigned int)skip_segment + 1u : 0u,
                             skip_segment >= 0 ? wait_limit_us : 0u};
  return cudaMemcpy(reinterpret_cast<uint8_t*>(workspace) + offsetof(WsHeader, dbg_skip_seg), v, sizeof(v),
                    cudaMemcpyHostToDevice) == cudaSuccess
             ? GTR_OK
             : GTR_ERR_CUDA;
}

gtr_status_t gtr_gla_workspace_init(void* workspace, size_t ws_bytes, gtr_stream_t stream) {
  if (!workspace || !is_aligned(workspace, 256) || ws_bytes < sizeof(WsHeader)) return GTR_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, ws_bytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? GTR_OK : GTR_ERR_CUDA;
}

gtr_status_t gtr_gla_fwd_host(const void* q, const void* k, const void* v, const float* log_gamma,
                              void* out, int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                              int direction, int in_dtype, int out_dtype, gtr_stream_t stream_) {
  gtr_status_t st = check_shape(B, heads, grid_H, grid_W, d_k, d_v, direction, in_dtype, out_dtype);
  if (st != GTR_OK) return st;
  if (!q || !k || !v || !log_gamma || !out) return GTR_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  int dev;
  st = current_device(&dev);
  if (st != GTR_OK) return st;
  DeviceCache& c = g_cache[dev];
  std::lock_guard<std::mutex> lock(c.mu);

  const size_t rows = (size_t)B * grid_H * grid_W * heads;
  const size_t bytes[5] = {rows * d_k * elem_size(in_dtype), rows * d_k * elem_size(in_dtype),
                           rows * d_v * elem_size(in_dtype), rows * d_k * sizeof(float),
                           rows * d_v * elem_size(out_dtype)};
  const void* src[4] = {q, k, v, log_gamma};
  for (int i = 0; i < 5; ++i) {
    st = ensure(c.io[i], bytes[i], stream);
    if (st != GTR_OK) return st;
  }
  for (int i = 0; i < 4; ++i)
    if (cudaMemcpyAsync(c.io[i].ptr, src[i], bytes[i], cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return GTR_ERR_CUDA;
  const Problem p = make_problem(c.io[0].ptr, c.io[1].ptr, c.io[2].ptr,
                                 static_cast<const float*>(c.io[3].ptr), c.io[4].ptr, B, heads,
                                 grid_H, grid_W, d_k, d_v, direction, in_dtype, out_dtype);
  const int path = choose_path(p, GTR_PATH_AUTO);
  const size_t need = path_workspace_bytes(p, path);
  if (need == 0) return GTR_ERR_UNSUPPORTED;
  st = ensure(c.ws, need, stream);
  if (st != GTR_OK) return st;
  st = run(p, path, c.ws.ptr, c.ws.bytes, stream);
  if (st != GTR_OK) return st;
  // the output and the device error word come back in the same stream, then one synchronisation
  if (!c.err_host && cudaMallocHost(reinterpret_cast<void**>(&c.err_host), sizeof(unsigned int)) != cudaSuccess) {
    c.err_host = nullptr;
    return GTR_ERR_CUDA;
  }
  if (cudaMemcpyAsync(out, c.io[4].ptr, bytes[4], cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemcpyAsync(c.err_host, c.ws.ptr, sizeof(unsigned int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return GTR_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GTR_ERR_CUDA;
  const unsigned int err = *c.err_host;
  if (err) {
    const unsigned int zero[2] = {0u, 0u};
    if (cudaMemcpy(c.ws.ptr, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return GTR_ERR_CUDA;
  }
  return static_cast<gtr_status_t>(err);
}

gtr_status_t gtr_gla_read_error(void* workspace, gtr_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return GTR_ERR_CUDA;
  void* ws = workspace;
  if (!ws) {
    int dev;
    gtr_status_t st = current_device(&dev);
    if (st != GTR_OK) return st;
    DeviceCache& c = g_cache[dev];
    std::lock_guard<std::mutex> lock(c.mu);
    ws = c.ws.ptr;
    if (!ws) return GTR_OK;  // nothing has run on this device yet
  }
  WsHeader h;
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return GTR_ERR_CUDA;
  if (h.error) {
    const unsigned int zero[2] = {0u, 0u};
    if (cudaMemcpy(ws, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return GTR_ERR_CUDA;
    // a call that gave up on a wait may have left its arrival counters behind: clear them
    if (h.error == GTR_ERR_TIMEOUT && cudaMemset(ws, 0, fused_reset_bytes()) != cudaSuccess) return GTR_ERR_CUDA;
  }
  return static_cast<gtr_status_t>(h.error);
}

gtr_status_t gtr_gla_plan(int B, int heads, int grid_H, int grid_W, int d_k, int d_v, int in_dtype,
                          int* path, int* launches) {
  const int out_dtype = in_dtype == GTR_F16 ? GTR_F16 : GTR_F32;
  const gtr_status_t st = check_shape(B, heads, grid_H, grid_W, d_k, d_v, GTR_L2R, in_dtype, out_dtype);
  if (st != GTR_OK) return st;
  const Problem p = make_problem(nullptr, nullptr, nullptr, nullptr, nullptr, B, heads, grid_H,
                                 grid_W, d_k, d_v, GTR_L2R, in_dtype, out_dtype);
  const int chosen = choose_path(p, GTR_PATH_AUTO);
  if (path) *path = chosen;
  if (launches) *launches = path_launches(p, chosen);
  return GTR_OK;
}

const char* gtr_status_string(int status) {
  switch (status) {
    case GTR_OK: return "GTR_OK";
    case GTR_ERR_INVALID_ARG: return "GTR_ERR_INVALID_ARG";
    case GTR_ERR_UNSUPPORTED: return "GTR_ERR_UNSUPPORTED";
    case GTR_ERR_CUDA: return "GTR_ERR_CUDA";
    case GTR_ERR_TIMEOUT: return "GTR_ERR_TIMEOUT";
    case GTR_ERR_WORKSPACE: return "GTR_ERR_WORKSPACE";
    case GTR_ERR_RANGE: return "GTR_ERR_RANGE";
    default: return "GTR_ERR_UNKNOWN";
  }
}

int gtr_version(void) { return 100; }

}  // extern "C"
