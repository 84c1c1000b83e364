/*
 * gtr.h - C ABI of libgtr.so: forward pass of key-only gated linear attention
 * (GLA) over an H x W patch-token grid, for NVIDIA B200 (sm_100a).
 *
 * The operation (GTR: Gated Token Recurrence for Efficient Dense Prediction;
 * digest page paper.rainbus.top/paper/2609.26590, prerequisite "Gated linear
 * attention (GLA)" and section "Core method"; page 0539edu.com, section 3.1):
 *
 *     S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t,      S_{-1} = 0
 *     o_t = d_k^{-1/2} q_t S_t
 *
 * per (batch, head), S_t in R^{d_k x d_v}, gamma_t in (0,1]^{d_k} a per-key-
 * channel gate given as log_gamma = log(gamma) (the value side is not decayed),
 * zero initial state, forward only (the operator specialisation in step 5 of
 * that page's "Method details").  The L = grid_H * grid_W tokens are visited
 * in one of four scan orders (section "Core method": left->right,
 * right->left, top->bottom, bottom->top), read as:
 *
 *   GTR_L2R: rows top to bottom, each row x = 0 .. W-1
 *   GTR_R2L: rows top to bottom, each row x = W-1 .. 0
 *   GTR_T2B: columns left to right, each column y = 0 .. H-1
 *   GTR_B2T: columns left to right, each column y = H-1 .. 0
 *
 * as one sequence: the state carries across line ends.  The work is done
 * chunkwise (chunk C = 64): per-chunk summaries, a boundary-state scan and
 * per-chunk outputs (first page, prerequisite "Chunkwise parallel"; page
 * 0539edu.com section 3.3 "Hardware-aware chunked inference"), which reaches
 * the sequential result up to rounding.
 *
 * LAYOUT.  q, k: [B, L, heads, d_k]; v: [B, L, heads, d_v]; log_gamma (always
 * fp32): [B, L, heads, d_k]; out: [B, L, heads, d_v].  All row-major and
 * contiguous; token index m = y * grid_W + x.  out[b, m, h, :] is the output
 * of the token at grid cell m whatever the direction.
 *
 * OWNERSHIP.  The caller owns every buffer.  Device pointers must be 16-byte
 * aligned and `out` must not overlap any input.  Nothing is retained after a
 * call returns except the library's own cached workspace (below).
 *
 * ASYNCHRONY.  Device entry points enqueue work on `stream` (a cudaStream_t;
 * NULL = legacy default stream) and return without synchronising.  Numerical
 * preconditions, not checked on the device: log_gamma finite and <= 0.
 *
 * ERRORS.  Every entry point returns a gtr_status_t.  Argument problems are
 * caught on the host before anything is enqueued (GTR_ERR_INVALID_ARG,
 * GTR_ERR_UNSUPPORTED); launch failures return GTR_ERR_CUDA.  Failures found
 * on the device (a bounded wait that ran out) are recorded in an error word
 * inside the workspace and returned by gtr_gla_read_error().
 */
#ifndef GTR_H_
#define GTR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t == struct CUstream_st* */
typedef struct CUstream_st *gtr_stream_t;

typedef enum { GTR_L2R = 0, GTR_R2L = 1, GTR_T2B = 2, GTR_B2T = 3 } gtr_direction_t;

/* Element types.  log_gamma is always GTR_F32. */
typedef enum { GTR_F32 = 0, GTR_F16 = 1, GTR_BF16 = 2 } gtr_dtype_t;

typedef enum {
    GTR_OK = 0,
    GTR_ERR_INVALID_ARG = 1, /* null/misaligned pointer, non-positive size, bad enum */
    GTR_ERR_UNSUPPORTED = 2, /* valid but not implemented (d_k, d_v, dtype pairing) */
    GTR_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    GTR_ERR_TIMEOUT = 4,     /* a device-side bounded wait ran out (see gtr_gla_read_error) */
    GTR_ERR_WORKSPACE = 5,   /* workspace too small, or would have to grow during stream capture */
    GTR_ERR_RANGE = 6        /* (device error word) an input, score or state magnitude passed
                                60000, beyond the fused path's fp16 tensor-core operands; that
                                call's output is not valid - use GTR_PATH_SPLIT for such data */
} gtr_status_t;

/* Execution paths.  GTR_PATH_AUTO lets the length-aware dispatcher choose.  Sequences
 * shorter than one chunk (grid_H * grid_W < 64) always run on GTR_PATH_SPLIT, whichever
 * path is requested (the fused paths' fp16 operand rounding is not averaged over enough
 * tokens there to stay inside the accuracy bound). */
typedef enum {
    GTR_PATH_AUTO = 0,
    GTR_PATH_SPLIT = 1, /* three launches: chunk summaries -> state scan -> chunk outputs (any dtype) */
    GTR_PATH_FUSED = 2, /* single tensor-core launch (fp16/bf16 inputs); the plan splits
                           long sequences over several CTAs */
    GTR_PATH_FUSED_SEQUENTIAL = 3 /* the same kernel with one CTA per (batch, head)
                                     walking its whole sequence */
} gtr_path_t;

/*
 * Supported shapes: d_v = 64 and d_k = 64 or 32 (d_k = 32: the pages' operator shape, GTR
 * digest page, step 5 of "Method details").  dtype pairings (in -> out):
 * F32 -> F32;  F16 -> F16 or F32;  BF16 -> F32 or BF16.  A BF16 OUTPUT is an opt-in
 * outside the 1e-2 * rms accuracy bound: rounding o to bf16 alone costs up to 2^-9 max|o|
 * (about 1.5% of rms on the GTR workloads); bf16 inputs give fp32 outputs by default.
 * Limits: B*heads <= 65535 * 64, L <= 2^28, B*L*heads*64 < 2^40 elements.
 */

/*
 * Generic entry.  Uses a workspace owned by the library, cached per device
 * and grown on demand with cudaMalloc (never while `stream` is being
 * captured: that returns GTR_ERR_WORKSPACE - make one uncaptured call of the
 * same or a larger size first).  Calls sharing the cached workspace must be
 * ordered on the device (one stream, or synchronised streams); concurrent
 * calls on independent streams need their own workspaces (gtr_gla_fwd_ws).
 */
gtr_status_t gtr_gla_fwd(const void *q, const void *k, const void *v,
                         const float *log_gamma, void *out,
                         int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                         int direction, int in_dtype, int out_dtype,
                         gtr_stream_t stream);

/* Typed forms with the problem's own argument list; the output dtype is
 * F16 for F16 inputs and F32 for BF16 and F32 inputs. */
gtr_status_t gtr_gla_fwd_f16(const void *q, const void *k, const void *v,
                             const float *log_gamma, void *out, int B, int heads,
                             int grid_H, int grid_W, int d_k, int d_v, int direction,
                             gtr_stream_t stream);
gtr_status_t gtr_gla_fwd_bf16(const void *q, const void *k, const void *v,
                              const float *log_gamma, void *out, int B, int heads,
                              int grid_H, int grid_W, int d_k, int d_v, int direction,
                              gtr_stream_t stream);
gtr_status_t gtr_gla_fwd_f32(const void *q, const void *k, const void *v,
                             const float *log_gamma, void *out, int B, int heads,
                             int grid_H, int grid_W, int d_k, int d_v, int direction,
                             gtr_stream_t stream);

/* Bytes of device workspace a gtr_gla_fwd_ex call with these arguments needs
 * (for every path the dispatcher may choose, and for every direction: the fused
 * path stages some directions one grid line a chunk, which can take more chunks
 * than ceil(L / 64)).  0 for invalid arguments. */
size_t gtr_gla_workspace_bytes(int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                               int in_dtype, int path);

/*
 * Caller-managed workspace (the persistent workspace of page 0539edu.com,
 * appendix E.3.1): `workspace` is a device buffer of `ws_bytes` >=
 * gtr_gla_workspace_bytes(...), 256-byte aligned.  The library allocates
 * nothing and never synchronises, so the call can be captured in a CUDA
 * graph.  A fresh workspace must be zeroed once before its first use
 * (gtr_gla_workspace_init, or any memset to 0); after that every call leaves
 * it ready for the next, so it may be reused by the next call once this one
 * has finished on the device.  `path` is a gtr_path_t.
 */
gtr_status_t gtr_gla_fwd_ex(const void *q, const void *k, const void *v,
                            const float *log_gamma, void *out,
                            int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                            int direction, int in_dtype, int out_dtype, int path,
                            void *workspace, size_t ws_bytes, gtr_stream_t stream);

/*
 * Failure injection, for tests of the device-side failure detection (not for production
 * use; the paper has no counterpart).  Synchronises `stream`, then marks `workspace` (a
 * caller workspace of gtr_gla_fwd_ex) so that in the next fused-path calls that split a
 * sequence over several CTAs (the segmented plan), segment `skip_segment` of every
 * sequence withholds its summary, and the later segments' waits for it give up after
 * `wait_limit_us` microseconds (0 keeps the default of about a second): they record
 * GTR_ERR_TIMEOUT in the workspace's error word, skip their second phase and leave
 * cleanly, so the call ends and the GPU context stays usable; the outputs of those
 * segments are not valid.  gtr_gla_read_error() then returns GTR_ERR_TIMEOUT and clears
 * the mark together with the error.  skip_segment < 0 clears the mark.
 */
gtr_status_t gtr_gla_workspace_debug(void *workspace, int skip_segment, unsigned int wait_limit_us,
                                     gtr_stream_t stream);

/* Zero `ws_bytes` of a caller workspace on `stream` (asynchronous; capturable). */
gtr_status_t gtr_gla_workspace_init(void *workspace, size_t ws_bytes, gtr_stream_t stream);

/*
 * Host-buffer entry: q, k, v, log_gamma and out are HOST pointers (pinned
 * memory gives full copy speed; pageable works).  The library copies the
 * inputs to device buffers it caches per device, runs the forward pass on
 * `stream`, copies the result back and synchronises `stream` before
 * returning.  Not capturable.
 */
gtr_status_t gtr_gla_fwd_host(const void *q, const void *k, const void *v,
                              const float *log_gamma, void *out,
                              int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                              int direction, int in_dtype, int out_dtype,
                              gtr_stream_t stream);

/*
 * Allocation-free form of gtr_gla_fwd, for callers that may not call
 * cudaMalloc (for instance a plugin inside an inference engine that allows
 * device allocation only at build time, or a real-time loop that must not take
 * cudaMalloc's implicit device synchronisation after start-up).  The paper has
 * no counterpart: it is an interface convenience of this library.
 *
 * It runs the split path (GTR_PATH_SPLIT) with its scratch in a fixed
 * 20 MiB array compiled into the library; every GPU that loads libgtr.so
 * holds that array until the process exits.  Problems whose scratch,
 * gtr_gla_workspace_bytes(..., GTR_PATH_SPLIT), exceeds 20 MiB - more than
 * 634 chunk units B * heads * ceil(L / 64) - are refused on the host with
 * GTR_ERR_WORKSPACE before anything is enqueued (after the argument checks of
 * gtr_gla_fwd, whose codes take precedence).  The call allocates nothing (no
 * cudaMalloc, cudaFree or allocating library routine).
 *
 * The first call on each device looks up the array's device address with
 * cudaGetSymbolAddress while that device is current, and caches it; make that
 * first call before any stream capture.  All calls share the one array and it
 * keeps the last call's contents: calls that overlap on the GPU (different
 * streams or threads without ordering) race and must be serialised by the
 * caller.  Arguments, layouts and return codes are otherwise those of
 * gtr_gla_fwd.
 */
gtr_status_t gtr_gla_fwd_noalloc(const void *q, const void *k, const void *v,
                                 const float *log_gamma, void *out,
                                 int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                                 int direction, int in_dtype, int out_dtype,
                                 gtr_stream_t stream);

/*
 * The GLA token mixer of one GTR block in a single call: the key-only recurrence above
 * with two optional pieces fused into it.
 *
 * LOW-RANK GATE PRODUCER (when gate_z != NULL; log_gamma must then be NULL).  GTR digest
 * page (paper.rainbus.top), section "Core method": the retention gate is
 * gamma_t = sigmoid(x_t W1 W2 + b)^(1/tau), a rank-16 factorisation with tau = 16.  The
 * call takes z = x W1 (the rank-r projection of every token) and computes
 *     log_gamma[b, m, h, :] = logsigmoid(z[b, m, :] W2 + b)[h*d_k .. h*d_k + d_k - 1] / tau
 * on the fly instead of reading a log_gamma tensor (a quarter to a third of the bytes).
 *   gate_z  [B, L, gate_rank] fp32 (token m = y * grid_W + x, shared by the heads)
 *   gate_w2 [gate_rank, heads * d_k] fp32;  gate_b [heads * d_k] fp32
 *   gate_rank 8 or 16 (the rows of z are then whole 32-byte pieces, which the tensor-memory
 *   loads need);  gate_tau > 0 (finite)
 * When gate_z is NULL, log_gamma [B, L, heads, d_k] fp32 is read as in gtr_gla_fwd.
 *
 * RMSNORM + SILU OUTPUT GATE (when out_gate != NULL).  0539edu.com, appendix E.3.1: the
 * end-to-end implementation fuses RMSNorm and a SiLU-activated output gate into the GLA
 * kernel's output epilogue.  With o the recurrence's output row of a token-head (d_v
 * values):
 *     out[b, m, h, j] = o_j / sqrt(mean_i o_i^2 + norm_eps) * norm_w[j] * SiLU(out_gate[b, m, h, j])
 *   out_gate [B, L, heads, d_v] in in_dtype;  norm_w [d_v] fp32 (shared by the heads);
 *   norm_eps >= 0 (finite).
 * When out_gate is NULL, norm_w and norm_eps are ignored and out is o itself.
 *
 * Every other argument, layout, alignment rule and return code is that of gtr_gla_fwd_ex
 * (all pointers 16-byte aligned device pointers).  `workspace` may be NULL: the library's
 * cached workspace is then used, with the rules of gtr_gla_fwd; otherwise it is a caller
 * workspace as for gtr_gla_fwd_ex (gtr_gla_workspace_bytes gives its size: the optional
 * pieces need no extra workspace).  A bf16 OUTPUT (out_dtype GTR_BF16) is outside the
 * 1e-2 * rms accuracy bound of this library: its own rounding costs up to 2^-9 max|o|.
 */
gtr_status_t gtr_gla_block_fwd(const void *q, const void *k, const void *v, const float *log_gamma,
                               const float *gate_z, const float *gate_w2, const float *gate_b,
                               int gate_rank, float gate_tau,
                               const void *out_gate, const float *norm_w, float norm_eps,
                               void *out, int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                               int direction, int in_dtype, int out_dtype, int path,
                               void *workspace, size_t ws_bytes, gtr_stream_t stream);

/*
 * Spatial SwiGLU stencil of a GTR block: out = SiLU(xg) * DWConv3x3(xv).
 *
 * GTR digest page (paper.rainbus.top), prerequisite "SwiGLU" and section "Core method";
 * page 0539edu.com section 3.1 ("Spatial SwiGLU"): the channel mixer is
 * Y = SiLU(X W_g) (.) DWConv3x3(X W_v) W_o, a 3x3 depthwise convolution in the value branch
 * that mixes neighbouring patches.  This call takes the two projections xg = X W_g and
 * xv = X W_v and returns the product in front of W_o (the projections are GEMMs outside
 * this library):
 *     out[b, y, x, c] = SiLU(xg[b, y, x, c]) *
 *         (conv_b[c] + sum_{dy, dx in 0..2} conv_w[c, dy, dx] * xv[b, y+dy-1, x+dx-1, c])
 * with zero padding at the grid border (the cross-correlation convention of a
 * convolution layer).
 *   xg, xv, out: [B, grid_H * grid_W, C] in `dtype` (GTR_F16, GTR_BF16 or GTR_F32), token
 *                m = y * grid_W + x, 16-byte aligned device pointers; out must not overlap
 *                the inputs.
 *   conv_w: [C, 3, 3] fp32;  conv_b: [C] fp32 or NULL (no bias); device pointers.
 *   C: a multiple of 64 (16-bit data) or of 32 (fp32) -- whole 128-byte channel blocks;
 *      otherwise GTR_ERR_UNSUPPORTED.
 * Asynchronous on `stream`; no workspace; allocates nothing; capturable.  Returns
 * GTR_ERR_INVALID_ARG for null or misaligned pointers and non-positive sizes.
 */
gtr_status_t gtr_sswiglu_dwconv(const void *xg, const void *xv, const float *conv_w, const float *conv_b,
                                void *out, int B, int grid_H, int grid_W, int C, int dtype,
                                gtr_stream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device error word of
 * `workspace` (NULL = the library's cached workspace of the current device).
 * GTR_OK when no device-side failure was recorded.
 */
gtr_status_t gtr_gla_read_error(void *workspace, gtr_stream_t stream);

/*
 * The length-aware dispatcher's decision for a problem: writes the path
 * GTR_PATH_AUTO would take to *path and the number of kernel launches one
 * call enqueues to *launches (either pointer may be NULL).  Host-only.
 */
gtr_status_t gtr_gla_plan(int B, int heads, int grid_H, int grid_W, int d_k, int d_v,
                          int in_dtype, int *path, int *launches);

/* Human-readable name of a status code (static storage). */
const char *gtr_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int gtr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GTR_H_ */
