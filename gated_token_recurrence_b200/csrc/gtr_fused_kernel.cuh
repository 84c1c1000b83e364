// Fused path: one launch, tcgen05 tensor cores, fp16/bf16 inputs.
//
// The chunkwise operator of page 0539edu.com, section 3.3 (chunk summaries ->
// light boundary-state scan -> per-chunk outputs; intra-chunk causal scores
// consumed on chip) and of the first GTR page, prerequisite "Chunkwise
// parallel", built as one persistent, warp-specialised sm_100a kernel.
//
// Per chunk of C = 64 scan positions of one (batch, head), with A the in-chunk
// inclusive cumsum of log2-gates and a = A[last] (per key channel):
//   Qh = Q * 2^A   (<= |q|)     Kh = K * 2^-A / sqrt(d_k)   (bounded by the chunk's decay)
//   P  = mask_{j<=i}(Qh Kh^T)   = d_k^-1/2 sum_k q_ik k_jk 2^(A_ik - A_jk)
//   O  = Qh S + P V             (S = state at the chunk start, kept scaled by d_k^-1/2)
//   U' = Kh^T V,  S <- 2^a * (S + U')     (= Diag(d) S + K~^T V with K~ = K * 2^(a - A))
// The power of two in d_k^-1/2 (1/8 for d_k = 64; 1/4 for d_k = 32, whose remaining
// 2^-1/2 is applied to the outputs) rides on Kh, so every product below already carries
// it.  All MMA operands are fp16 (bf16 inputs convert inside the fp16 range); a CTA whose
// first chunk holds tiny inputs scales q, k, v by powers of two into that range and
// undoes it in fp32.  Accumulation and the state are fp32.  Qh and Kh overwrite the Q
// and K tiles they are built from.  A chunk whose gates decay too fast for the
// factorisation to stay inside fp16 gets its scores from the CUDA cores (2^(A_i - A_j)
// per pair), written straight into tensor memory.  Outputs that come out non-finite (an
// operand beyond the fp16 range) are reported as GTR_ERR_RANGE.
//
// Three plans.  STREAM: one CTA walks a whole sequence, carrying the exact fp32 state.
// CLUSTER: the CTAs of one thread-block cluster split a short sequence, hold their
// outputs in tensor memory and scan the segment summaries through distributed shared
// memory.  SEGMENTED: the n_s CTAs of a sequence each walk one contiguous run of its
// chunks (a segment) from a zero start state, write their partial outputs O_local and
// Qh' = Qh * 2^(A from the segment start) to the workspace and publish the segment
// summary (end state, log2 decay); segment 0's outputs are final unless the output gate
// is on.  The n_s CTAs then scan the summaries (each owns a slice of the 64x64 state
// entries), and in a second phase every CTA with partial outputs adds Qh' S_start(s) to
// O_local, one M = 128 MMA per chunk pair, spread over all four of its warpgroups.
//
// Warp roles (640 threads):
//   warps 0-7   WG_A  two warpgroups on alternating chunks: cumulative gates (from the
//               low-rank producer's z rows when given), the input scale (first chunk),
//               Qh / Kh in place, CUDA-core scores
//   warps 8-11  WG_B  score masking, fp32 state update, the next chunk-start state
//               (16-lane tensor-memory loads, so every lane of a warp does the same work)
//   warps 12-15 WG_C  epilogue (the output gate when given); SEGMENTED: summary scan
//   warp 16     producer: TMA boxes (row or column views, line chunks), or 4-row TMA
//               gathers resolving the direction remap (cp.async row copies for views of
//               2^31 rows or more); zero fill past the sequence or line end
//   warp 17     Qh' tiles of segments s > 0 (and of segment 0 under the output gate)
//   warp 18     tcgen05 MMA issuer of the scores and U' (in chunk order), tensor-memory owner
//   warp 19     tcgen05 MMA issuer of the outputs O = Qh S, O += P V (in chunk order)
//   SEGMENTED second phase: warpgroups 0-3 (warps 0-15) each take every fourth pair
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "gtr_common.cuh"
#include "gtr_internal.h"
#include "gtr_sm100.cuh"

namespace gtr {
namespace {

using namespace sm100;

constexpr int kStages = 4;          // staging depth (chunks in flight)
constexpr int kSU = 4;              // score / U' regions in tensor memory (chunks in flight)
constexpr int kThreads = 640;
constexpr int kProducerThreads = 32;  // cp.async copies (warp 16)
constexpr int kQhWarp = 17;           // Qh' tiles of segments s > 0
constexpr int kMmaWarp = 18;  // stage 1 (scores, U'); tensor-memory owner
constexpr int kOutWarp = 19;  // stages 2a / 2b (outputs)
constexpr int kWG = 128;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// shared memory (bytes); every 16-bit tile is [64][64], 128 B rows, 128 B swizzle
constexpr int kTile = 8192;
constexpr int kGTile = 16384;                        // fp32 log-gates [64][64]
constexpr int kStageBytes = 3 * kTile + kGTile;      // Q (-> Qh), K (-> Kh), V, G
// d_k = 32: the gates take the first half of the gate tile (64 rows of 32 fp32), and the
// raw q and k (dense 64-byte rows) its second half; Qh and Kh are built, zero-padded to 64
// channels, into the Q and K tiles
constexpr int kRawQ = 8192, kRawK = 12288;  // byte offsets in the gate tile
// bytes one chunk's loads bring: q, k (64 x d_k x 2 B), v (8 KB), log-gates (64 x d_k x 4 B)
template <int kDK> constexpr uint32_t chunk_load_bytes() { return 2u * 64 * kDK * 2 + kTile + 64u * kDK * 4; }

constexpr int kOffStage = 0;
constexpr int kNS = 5;                                     // chunk-start state tiles
constexpr int kOffS = kOffStage + kStages * kStageBytes;   // [kNS] chunk-start states
constexpr int kOffSst = kOffS;                             // segment start state (after the chunks: over state tile 0)
constexpr int kOffStg = kOffS + kNS * kTile;               // output staging, 4 warps x 32 rows x 128 B
constexpr int kStgBytes = 4 * 32 * 128;                    // (CLUSTER: first the segment summary, fp32)
constexpr int kOffMisc = kOffStg + kStgBytes;
constexpr int kMiscBytes = 9216;
constexpr int kSmemBytes = kOffMisc + kMiscBytes + 1024;  // + alignment slack
// second phase, pair slot q (one per warpgroup) in staging buffer q: Qh' of the pair
// (16 KB, the A operand; then the warps' fp32 output staging) and O_local (16 KB)
constexpr int kP2Olc = 16384;
static_assert(2 * kP2Olc <= kStageBytes, "a chunk pair's second-phase tiles fit one staging buffer");

// tensor memory columns
constexpr uint32_t kColSU = 0;     // [kSU] x 64: scores (lane tile 0; masked fp16 P over their first
                                   // 32 columns) and U' (lane tile 1)
constexpr int kOPairs = 4;         // output pairs in tensor memory (a ring; CLUSTER: all of a CTA's chunks)
constexpr uint32_t kColO = kColSU + 64u * kSU;  // [kOPairs] x 64 output pairs (chunk 2m lane tile 0, 2m+1 tile 1)
constexpr uint32_t kLaneTile1 = 16u << 16;
constexpr int kClusterChunks = 2 * kOPairs;  // CLUSTER: chunks per CTA (outputs held in tensor memory)
constexpr int kMaxCluster = 16;              // CLUSTER: CTAs per sequence (non-portable cluster size)
static_assert(kColO + 64 * kOPairs <= kTmemCols, "tensor memory budget");
static_assert(kClusterChunks * kTile + 3 * 16384 <= kOffS, "a CTA's Qh' tiles and three epilogue staging areas fit the idle staging buffers");
static_assert(4 * 64 <= kColO, "second-phase slots (M = 128, 64 columns each) reuse the score regions");

// Segment counters sit at a fixed place right after the workspace header, whatever
// the problem size, so that a workspace kept zero between calls stays valid across shapes.
constexpr size_t kMaxSegCtas = 256;  // CTAs of one launch in SEGMENTED mode (>= the SM count)
constexpr size_t kCounterBytes = 2 * kMaxSegCtas * sizeof(unsigned int);
constexpr int kScanBlock = 8;       // segments one WG_C thread composes in registers
// per-segment summary: U_seg [64][64] fp32, the log2 decay [64], the factor that takes a
// start state into the segment's CTA scale, padding
constexpr size_t kAggStride = 4096 + 128;
static_assert(sizeof(WsHeader) + kCounterBytes == kWsPrefixBytes, "counters fill the shared workspace prefix");

// floor(n / d) for 0 <= n < 2^31 by one wide multiply and a shift: with l = ceil(log2 d)
// and m = ceil(2^(31+l) / d) (m < 2^32), floor(n m / 2^(31+l)) = floor(n / d) for every
// such n (Granlund and Montgomery, "Division by Invariant Integers using Multiplication",
// PLDI 1994, Theorem 4.2 with N = 31).  The scan remap divides by the grid width or
// height for every staged row and every stored output row.
struct FastDiv {
  uint32_t m, sh;  // multiplier and total shift 31 + l
};
inline FastDiv make_fastdiv(uint32_t d) {
  uint32_t l = 0;
  while ((1ull << l) < d) ++l;
  return FastDiv{(uint32_t)(((1ull << (31 + l)) + d - 1) / d), 31 + l};
}
__device__ __forceinline__ uint32_t fast_div(uint32_t n, FastDiv f) {
  return (uint32_t)(((unsigned long long)n * f.m) >> f.sh);
}

struct alignas(64) FusedParams {
  // TMA tensor maps for Q, K, V (16-bit, 128-byte swizzle) and the log-gates (fp32):
  // row view [B][L][heads][64] (4-D) or column view [B][H][W][heads][64] (5-D), boxes of
  // 64 consecutive scan positions of one (batch, head)
  CUtensorMap tq, tk, tv, tg;
  CUtensorMap tz;          // low-rank gate producer: the rank-r token projections z (fp32), same views
  Problem p;
  WsHeader* hdr;
  unsigned int* counters;  // SEGMENTED: [n_seq][2] arrival counters, monotonic within a call, zero between calls
  float* agg;              // [n_seq][n_s][kAggStride] segment summaries (U_seg, log2 decay, start-state factor)
  uint16_t* sstart;        // [n_seq][n_s][64*64] segment start states, fp16, MMA layout, their CTA's scale
  uint16_t* qhp;           // [n_seq][Nc][64*64] Qh' per chunk, fp16, MMA layout
  uint16_t* olc;           // [n_seq][Nc][64][64] outputs from a zero segment start, fp16
  int n_seq, n_s, Nc, mode;  // mode 0 = STREAM, 1 = SEGMENTED, 2 = CLUSTER
  int grid;
  float max_exp2;          // largest in-chunk log2-decay the score factorisation takes
  int tma;                 // 1: one TMA box per tensor; 2: 4-row TMA gathers; 0: cp.async row copies
  int rev;                 // 1: chunks are staged in reverse scan order (right-to-left, bottom-to-top)
  FastDiv divW, divH;      // the grid width and height as invariant divisors
  int lowrank;             // 1: the log-gates come from the low-rank producer (z tiles, p.gw2, p.gb)
  float gtau_inv;          // 1 / tau of the gate producer
  int gated;               // 1: RMSNorm + SiLU output gate on the final outputs (p.ogate, p.onorm_w)
  int lines, len;          // 1: line chunks of lines `len` cells long (0: contiguous chunks)
};

// Chunk c, offset r (0..63) of its scan positions -> scan position s.  Contiguous chunks
// cover scan positions 64c .. 64c + 63; a line chunk covers grid line c (a row for the
// row directions, a column for the column ones), len < 64 cells, zero-padded past the
// line end.  False past the sequence or the line end.
__device__ __forceinline__ bool chunk_scan_pos(const FusedParams& fp, int c, int r, long long L, long long& s) {
  s = (long long)c * (fp.lines ? fp.len : kChunk) + r;
  return fp.lines ? r < fp.len : s < L;
}

// Scan position s (< L < 2^31) -> token index y*W + x: the direction remap (rows top to
// bottom, left to right or right to left; columns left to right, top to bottom or bottom
// to top), with the division by W or H done by multiplication.
__device__ __forceinline__ uint32_t scan_token(const FusedParams& fp, uint32_t s) {
  const uint32_t W = (uint32_t)fp.p.W, H = (uint32_t)fp.p.H;
  uint32_t x, y;
  if (fp.p.direction <= GTR_R2L) {
    y = fast_div(s, fp.divW);
    x = s - y * W;
    if (fp.p.direction == GTR_R2L) x = W - 1 - x;
  } else {
    x = fast_div(s, fp.divH);
    y = s - x * H;
    if (fp.p.direction == GTR_B2T) y = H - 1 - y;
  }
  return y * W + x;
}
static_assert(alignof(FusedParams) >= 64, "tensor maps need 64-byte alignment");

// Bytes one chunk's loads bring with the low-rank gate producer: the z rows (64 x rank
// fp32) instead of the log-gates.
template <int kDK>
__device__ __forceinline__ uint32_t chunk_load_bytes(const FusedParams& fp, bool lowrank) {
  return lowrank ? 2u * 64 * kDK * 2 + kTile + 64u * fp.p.grank * 4 : chunk_load_bytes<kDK>();
}

struct Misc {
  uint64_t full[kStages], empty[kStages];
  // opready is per stage: the operand builder may run up to kStages chunks ahead of the
  // MMA warp, so a two-deep ring could complete a phase twice before it is observed
  uint64_t opready[kStages];
  uint64_t su_full[kSU], su_free[kSU], pready[kSU];  // per score / U' region
  uint64_t sready[kNS];                              // per chunk-start state tile
  uint64_t qdone[kStages];                           // Qh' of the staged chunk copied out
  uint64_t o_full[kOPairs], o_free[kOPairs];         // per output pair
  uint64_t agg_pub, p2_go, mma_final[2], corr_done[kOPairs];
  uint64_t p2_full[4], p2_mma[4];  // second phase, per warpgroup: tiles landed, correction done
  uint64_t scale_ready;            // the input scale factors below are set (WG_A0, first chunk)
  uint32_t tmem_base;
  // Power-of-two input scale of this CTA, taken from its first chunk (1 unless that chunk's
  // largest |q|, |k| or |v| is tiny): q, k, v enter the fp16 operands multiplied by
  // sc_in[0..2] = 2^alpha, 2^beta, 2^gamma, so everything the CTA accumulates carries the
  // factor 2^(alpha+beta+gamma) (outputs) or 2^(beta+gamma) (the state).
  float sc_in[3];
  float sc_out;   // 2^-(alpha+beta+gamma): outputs back to the inputs' scale
  float sc_spub;  // 2^-(beta+gamma): this CTA's state back to the inputs' scale (published summaries)
  float sc_sin;   // 2^(beta+gamma): a state in the inputs' scale into this CTA's scale (start states)
  unsigned int smax[4][3];  // WG_A0: per-warp largest |q|, |k|, |v| bit patterns of the first chunk
  alignas(16) float w2s[16][64];  // low-rank gate producer: this head's W2 columns [rank][64] (zero past d_k)
  alignas(16) float bs[64];       // ... and bias (zero past d_k)
  alignas(16) float nw[64];       // output gate: RMSNorm weight
  int zrow[2][64];                // producer: z row b*L + m of each chunk row (gathers; -1 past the end)
  int abort;
  unsigned int dbg_skip, dbg_us;  // failure injection (workspace header), read once by WG_C
  int go[4][3];          // per-warpgroup wait decisions, alternating slots; [3][2]: scaled segments seen
  int fb[kStages];       // stage -> scores from the CUDA cores
  alignas(16) float dseg[64];  // CLUSTER: this segment's log2 decay per key channel (read by the cluster)
  alignas(16) float red[2][2][4][32];  // WG_A cumsum: per warpgroup, channel half and warp, channel totals
  alignas(16) float eseg[64];          // Qh' warp: 2^(decay from the segment start) per channel
  int rowoff[2][64];              // producer, per chunk row: the row of the gather view (past the end: a row past the view) or, for row copies, grid cell b*L + m (-1 past the end)
};
// The in-chunk log2 decay per channel (a) of a staged chunk is kept in row 0 of its
// gate tile once the gates are consumed, the factor 2^(decay from the segment start)
// in row 1; the summary scan exchanges its block transfers through the segment-start-
// state tile, which is idle at that point.
static_assert(sizeof(Misc) <= kMiscBytes, "misc area too small");
static_assert(sizeof(Misc::red) >= kStages * 64 * sizeof(float), "the in-place Qh' factors fit the cumsum exchange");
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// 2^x on the special-function unit.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log2(x) on the special-function unit.
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log(sigmoid(x)) = min(x, 0) - log(1 + e^-|x|): neither term overflows; the log of
// 1 + e^-|x| is taken in base 2 on the special-function unit.
__device__ __forceinline__ float log_sigmoid_fast(float x) {
  return fminf(x, 0.f) - 0.69314718055994531f * lg2(1.f + ex2(-fabsf(x) * 1.4426950408889634f));
}

// SiLU(x) = x * sigmoid(x) = x / (1 + e^-x).
// (the approximate divide: a few ulp, and 0 once 1 + e^-x passes 2^126, the limit of
// x / (1 + e^-x) for very negative x)
__device__ __forceinline__ float silu_fast(float x) {
  return __fdividef(x, 1.f + ex2(-x * 1.4426950408889634f));
}

// Bounded mbarrier wait: the thread sleeps in hardware until the phase completes; only
// after about a second without completion does the CTA record a timeout and abort.
// kOut: the loop after the first attempt is a call (out of line), so that a chunk loop full
// of waits keeps only their fast paths (the segmented kernel, measured faster so).
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, Misc* ms, WsHeader* hdr, uint32_t where);
template <bool kOut = false>
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Misc* ms, WsHeader* hdr, uint32_t where) {
  if (mbar_wait_sleep(bar, parity, 1000000u)) return true;
  if constexpr (kOut) return wait_bar_slow(bar, parity, ms, hdr, where);
  const uint64_t t0 = globaltimer();
  while (true) {
    if (*(volatile int*)&ms->abort) return false;
    if (mbar_wait_sleep(bar, parity, 1000000u)) return true;
    if (globaltimer() - t0 > 1000000000ull) {
      record_error(hdr, GTR_ERR_TIMEOUT, where);
      *(volatile int*)&ms->abort = 1;
      return false;
    }
  }
}

// Bounded wait by polling (no suspension), for the MMA-issuing threads: they react to a
// completed phase at once.
__device__ __noinline__ bool wait_spin_slow(uint64_t* bar, uint32_t parity, Misc* ms, WsHeader* hdr, uint32_t where);
template <bool kOut = false>
__device__ __forceinline__ bool wait_spin(uint64_t* bar, uint32_t parity, Misc* ms, WsHeader* hdr, uint32_t where) {
  for (int i = 0; i < 64; ++i)
    if (mbar_test(bar, parity)) return true;
  if constexpr (kOut) return wait_spin_slow(bar, parity, ms, hdr, where);
  const uint64_t t0 = globaltimer();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_test(bar, parity)) return true;
    if (*(volatile int*)&ms->abort) return false;
    if (globaltimer() - t0 > 1000000000ull) {
      record_error(hdr, GTR_ERR_TIMEOUT, where);
      *(volatile int*)&ms->abort = 1;
      return false;
    }
  }
}

__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, Misc* ms, WsHeader* hdr, uint32_t where) {
  return wait_bar<false>(bar, parity, ms, hdr, where);
}
__device__ __noinline__ bool wait_spin_slow(uint64_t* bar, uint32_t parity, Misc* ms, WsHeader* hdr, uint32_t where) {
  return wait_spin<false>(bar, parity, ms, hdr, where);
}

// Bounded wait until a global counter reaches `target` (`limit_ns`: about a second, or the
// workspace's failure-injection limit).
// Arrivals count in the low 16 bits; the high 16 bits carry a side count (returned in
// *high on success).
__device__ bool wait_counter(const unsigned int* ctr, unsigned int target, Misc* ms, WsHeader* hdr,
                             uint32_t where, uint64_t limit_ns = 1000000000ull, unsigned int* high = nullptr) {
  const uint64_t t0 = globaltimer();
  while (true) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if ((v & 0xffffu) >= target) {
      if (high) *high = v >> 16;
      return true;
    }
    if (*(volatile int*)&ms->abort) return false;
    if (globaltimer() - t0 > limit_ns) {
      record_error(hdr, GTR_ERR_TIMEOUT, where);
      *(volatile int*)&ms->abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void red_release_add(unsigned int* ctr, unsigned int v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(ctr), "r"(v) : "memory");
}


// Named barrier of one 128-thread warpgroup (ids 1..3).
__device__ __forceinline__ void wg_sync(int wg) { asm volatile("bar.sync %0, 128;" ::"r"(wg + 1) : "memory"); }

// Warpgroup wait: its first thread does the bounded wait, then every thread of the
// group takes the same decision (no thread is left alone at a named barrier) and
// observes the completed phase itself.
template <bool kOut = false>
__device__ __forceinline__ bool wg_wait(int wg, int wtid, uint64_t* bar, uint32_t parity, Misc* ms, WsHeader* hdr,
                                        uint32_t where, int& slot, bool spin = false) {
  if (wtid == 0) {
    const bool ok = spin ? wait_spin<kOut>(bar, parity, ms, hdr, where) : wait_bar<kOut>(bar, parity, ms, hdr, where);
    ms->go[wg][slot] = ok && !*(volatile int*)&ms->abort;
  }
  wg_sync(wg);
  const bool go = *(volatile int*)&ms->go[wg][slot] != 0;
  slot ^= 1;
  if (go) (void)mbar_try_wait(bar, parity);
  return go;
}

// AND of a predicate over the 128 threads of warpgroup wg (named barrier wg + 1).
__device__ __forceinline__ bool wg_all(int wg, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(wg + 1)
      : "memory");
  return r != 0;
}

__device__ bool wg_agree(int wg, int wtid, bool ok0, Misc* ms, int& slot) {
  if (wtid == 0) ms->go[wg][slot] = ok0 && !*(volatile int*)&ms->abort;
  wg_sync(wg);
  const bool go = *(volatile int*)&ms->go[wg][slot] != 0;
  slot ^= 1;
  return go;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t pack_h2(float a, float b) { return h2_bits(__floats2half2_rn(a, b)); }

// Two 16-bit input values -> fp32.
template <typename T> struct In2;
template <> struct In2<__half> {
  static __device__ __forceinline__ float2 unpack(uint32_t u) { return __half22float2(bits_h2(u)); }
};
template <> struct In2<__nv_bfloat16> {
  static __device__ __forceinline__ float2 unpack(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  }
};

// Two fp32 values -> two 16-bit values of type T (round to nearest even).
template <typename T> struct Pack2;
template <> struct Pack2<__half> {
  static __device__ __forceinline__ uint32_t pack(float a, float b) { return pack_h2(a, b); }
};
template <> struct Pack2<__nv_bfloat16> {
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

__device__ __forceinline__ void sts32(uint8_t* p, uint32_t v) { *reinterpret_cast<uint32_t*>(p) = v; }

// 16-byte chunk j of staged row R (rows of kRowB bytes) sits at R*kRowB + 16*(j ^ sw(R)),
// so the row-per-lane writes and the row-per-group reads both spread over all banks.
template <int kRowB>
__device__ __forceinline__ int stage_chunk(int R, int j) {
  constexpr int kLanesPerRow = kRowB / 16;
  const int swz = (kLanesPerRow == 8) ? (R & 7) : ((R >> 1) & 3);
  return R * kRowB + 16 * (j ^ swz);
}

// One half (32 columns) of the 32 rows of one warp -> memory as Tout: `v` holds this
// lane's row.  Each lane writes its row into a per-warp staging tile in shared memory;
// after __syncwarp the warp copies the tile out with whole rows per 8 (fp32) or 4 (16-bit)
// lanes, so every 16-byte global store covers 4 or 8 full row segments.  `rowdst` is this
// lane's destination row (nullptr: not stored).  `nf` collects x * 0 over the values: it
// turns NaN once any is not finite.
template <typename Tout>
__device__ __forceinline__ void stage_store_half(const float (&v)[32], uint8_t* rowdst, uint8_t* wstage, int lane,
                                                 int half, float& nf) {
  constexpr int kRowB = 32 * (int)sizeof(Tout);  // staged bytes per row and half
  constexpr int kLanesPerRow = kRowB / 16;       // 8 (fp32) or 4 (16-bit)
  constexpr int kRowsPerOp = 32 / kLanesPerRow;
  const unsigned long long myrow = reinterpret_cast<unsigned long long>(rowdst);
  uint8_t* buf = wstage;  // one 32-row tile, reused by both halves
  if constexpr (sizeof(Tout) == 4) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      nf = fmaf(v[4 * j], 0.f, nf);
      nf = fmaf(v[4 * j + 1], 0.f, nf);
      nf = fmaf(v[4 * j + 2], 0.f, nf);
      nf = fmaf(v[4 * j + 3], 0.f, nf);
      *reinterpret_cast<float4*>(buf + stage_chunk<kRowB>(lane, j)) =
          make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    }
  } else {
    __half2 acc = __float2half2_rn(0.f);
    const __half2 zero = __float2half2_rn(0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t pk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float x0 = v[8 * j + 2 * u], x1 = v[8 * j + 2 * u + 1];
        if constexpr (std::is_same<Tout, __half>::value) {
          pk[u] = pack_h2(x0, x1);
          acc = __hfma2(bits_h2(pk[u]), zero, acc);
        } else {
          __nv_bfloat162 hb = __floats2bfloat162_rn(x0, x1);
          pk[u] = *reinterpret_cast<uint32_t*>(&hb);
          nf = fmaf(x0, 0.f, nf);
          nf = fmaf(x1, 0.f, nf);
        }
      }
      *reinterpret_cast<uint4*>(buf + stage_chunk<kRowB>(lane, j)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    if constexpr (std::is_same<Tout, __half>::value) {
      const float2 a = __half22float2(acc);
      nf += a.x + a.y;
    }
  }
  __syncwarp();
  const int jj = lane % kLanesPerRow;
#pragma unroll
  for (int it = 0; it < kLanesPerRow; ++it) {
    const int R = it * kRowsPerOp + lane / kLanesPerRow;
    const unsigned long long dr = __shfl_sync(0xffffffffu, myrow, R);
    const uint4 x = *reinterpret_cast<const uint4*>(buf + stage_chunk<kRowB>(R, jj));
    if (dr) __stcs(reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(dr) + kRowB * half + 16 * jj), x);
  }
  __syncwarp();  // the staging tile is free again
}

// The 32 rows of one warp (its lanes of a tensor-memory region, 64 fp32 columns) ->
// memory as Tout, 32 columns at a time, every value multiplied by `osc` (a power of two:
// the CTA's input scale undone; times 2^-1/2 when d_k = 32).
template <typename Tout>
__device__ __forceinline__ void epilogue_rows(uint32_t taddr, uint8_t* rowdst, uint8_t* wstage, int lane,
                                              float& nf, float osc) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float v[32];
    tmem_ld32(taddr + 32u * half, v);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= osc;
    stage_store_half<Tout>(v, rowdst, wstage, lane, half, nf);
  }
}

// The same rows through the GLA output epilogue (0539edu.com appendix E.3.1: RMSNorm and a
// SiLU-activated output gate fused into the kernel): with o = osc * (tensor memory row
// [+ the row's partial output olc, fp16, SEGMENTED second phase]),
//   y_j = o_j / sqrt(mean_i o_i^2 + eps) * nw_j * SiLU(gate_j),
// the lane's gate row `grow` (Tin, 64 values; nullptr for rows that are not stored).  Two
// passes over tensor memory: the row's sum of squares, then the values.  The gate row (128
// bytes) is requested first, in 16-byte loads that stay ahead of the tensor-memory loads, so
// its latency overlaps the norm pass instead of following each use; the partial output is
// read 16 bytes at a time.  Out of line.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
template <typename Tout, typename Tin>
__device__ __noinline__ void gated_rows(uint32_t taddr, const uint8_t* olc, uint8_t* rowdst, const Tin* grow,
                                        const float* nw, float eps, uint8_t* wstage, int lane, float& nf, float osc) {
  uint4 gq[8];  // the gate row, 8 x 16 bytes (values 8c .. 8c + 7 in gq[c])
#pragma unroll
  for (int c = 0; c < 8; ++c) gq[c] = grow ? ld_nc_v4(reinterpret_cast<const uint4*>(grow) + c) : make_uint4(0, 0, 0, 0);
  float ss = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float v[32];
    tmem_ld32(taddr + 32u * half, v);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 o4 = make_uint4(0, 0, 0, 0);
      if (olc) o4 = *reinterpret_cast<const uint4*>(olc + 64 * half + 16 * c);
      const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 o = __half22float2(bits_h2(ow[u]));
        const float x0 = (v[8 * c + 2 * u] + o.x) * osc, x1 = (v[8 * c + 2 * u + 1] + o.y) * osc;
        ss = fmaf(x0, x0, fmaf(x1, x1, ss));
      }
    }
  }
  const float rinv = rsqrtf(ss * (1.f / 64.f) + eps);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float v[32];
    tmem_ld32(taddr + 32u * half, v);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 o4 = make_uint4(0, 0, 0, 0);
      if (olc) o4 = *reinterpret_cast<const uint4*>(olc + 64 * half + 16 * c);
      const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
      const uint4 g4 = gq[4 * half + c];
      const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = 8 * c + 2 * u;  // value 32 half + j of the row
        const float2 o = __half22float2(bits_h2(ow[u]));
        const float2 g = In2<Tin>::unpack(gw[u]);
        v[j] = (v[j] + o.x) * osc * rinv * nw[32 * half + j] * silu_fast(g.x);
        v[j + 1] = (v[j + 1] + o.y) * osc * rinv * nw[32 * half + j + 1] * silu_fast(g.y);
      }
    }
    stage_store_half<Tout>(v, rowdst, wstage, lane, half, nf);
  }
}

// Grid-cell destination of output row s of (b, h), or nullptr when not `valid`.
template <typename Tout>
__device__ __forceinline__ uint8_t* out_row(const FusedParams& fp, int b, int h, bool valid, long long s) {
  if (!valid) return nullptr;
  const long long m = ((long long)b * fp.p.L() + scan_token(fp, (uint32_t)s)) * fp.p.heads + h;
  return reinterpret_cast<uint8_t*>(reinterpret_cast<Tout*>(fp.p.out) + m * 64);
}

// Output-gate row (64 values of the input dtype) of output row s of (b, h), or nullptr.
template <typename Tin>
__device__ __forceinline__ const Tin* gate_row(const FusedParams& fp, int b, int h, bool valid, long long s) {
  if (!valid) return nullptr;
  const long long m = ((long long)b * fp.p.L() + scan_token(fp, (uint32_t)s)) * fp.p.heads + h;
  return reinterpret_cast<const Tin*>(fp.p.ogate) + m * 64;
}

// Low-rank gate producer (GTR digest page, "Core method": gamma = sigmoid(x W1 W2 + b)^(1/tau),
// rank 16): ln gamma of this thread's rows row0 .. row0+3 and channels 32p + 4cc .. +3
// (p < d_k / 32) from the chunk's z rows (dense [64][rank] fp32 at zt) and this head's W2
// columns and bias (shared memory), into lr[p][row][channel].  Out of line.
template <int kDK>
__device__ __noinline__ void lowrank_gate_values(const float* zt, const Misc* ms, int rank, float tinv, int row0,
                                                 int cc, float (*lr)[4][4]) {
  for (int ps = 0; ps < kDK / 32; ++ps) {
    const int ch0 = 32 * ps + 4 * cc;
    const float4 b4 = *reinterpret_cast<const float4*>(ms->bs + ch0);
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = b4.x, acc[i][1] = b4.y, acc[i][2] = b4.z, acc[i][3] = b4.w;
    for (int j = 0; j < rank; j += 4) {
      float4 zr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) zr[i] = *reinterpret_cast<const float4*>(zt + (row0 + i) * rank + j);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float4 w4 = *reinterpret_cast<const float4*>(&ms->w2s[j + jj][ch0]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float zv = jj == 0 ? zr[i].x : jj == 1 ? zr[i].y : jj == 2 ? zr[i].z : zr[i].w;
          acc[i][0] = fmaf(zv, w4.x, acc[i][0]);
          acc[i][1] = fmaf(zv, w4.y, acc[i][1]);
          acc[i][2] = fmaf(zv, w4.z, acc[i][2]);
          acc[i][3] = fmaf(zv, w4.w, acc[i][3]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) lr[ps][i][e] = log_sigmoid_fast(acc[i][e]) * tinv;
  }
}

// Segmented mode, second phase: the 32 rows of one warp hold the correction Qh' S_start
// (fp32, tensor memory); the row's partial output O_local (fp16, row-major 128 B rows at
// `olc_rows` in shared memory) is added on the way out and the sum, times `osc`, stored
// as Tout.
template <typename Tout>
__device__ __forceinline__ void epilogue_rows_add(uint32_t taddr, uint8_t* rowdst, const uint8_t* olc_rows,
                                                  uint8_t* wstage, int lane, float& nf, float osc) {
  constexpr int kRowB = 128;  // fp32 staging, 32 columns per half
  const unsigned long long myrow = reinterpret_cast<unsigned long long>(rowdst);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float v[32];
    tmem_ld32(taddr + 32u * half, v);
    tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(wstage + stage_chunk<kRowB>(lane, j)) =
          make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    __syncwarp();
    const int jj = lane & 7;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int R = it * 4 + (lane >> 3);
      const unsigned long long dr = __shfl_sync(0xffffffffu, myrow, R);
      const float4 c = *reinterpret_cast<const float4*>(wstage + stage_chunk<kRowB>(R, jj));
      const uint2 ol = *reinterpret_cast<const uint2*>(olc_rows + R * 128 + (32 * half + 4 * jj) * 2);
      const float2 o01 = __half22float2(bits_h2(ol.x)), o23 = __half22float2(bits_h2(ol.y));
      const float y0 = (c.x + o01.x) * osc, y1 = (c.y + o01.y) * osc, y2 = (c.z + o23.x) * osc,
                  y3 = (c.w + o23.y) * osc;
      if (dr) {  // (rows past the sequence end hold stale partials: neither checked nor stored)
        nf = fmaf(y0, 0.f, nf);
        nf = fmaf(y1, 0.f, nf);
        nf = fmaf(y2, 0.f, nf);
        nf = fmaf(y3, 0.f, nf);
        uint8_t* d = reinterpret_cast<uint8_t*>(dr) + (32 * half + 4 * jj) * (int)sizeof(Tout);
        if constexpr (sizeof(Tout) == 4) {
          __stcs(reinterpret_cast<float4*>(d), make_float4(y0, y1, y2, y3));
        } else if constexpr (std::is_same<Tout, __half>::value) {
          __stcs(reinterpret_cast<uint2*>(d), make_uint2(pack_h2(y0, y1), pack_h2(y2, y3)));
        } else {
          __nv_bfloat162 b0 = __floats2bfloat162_rn(y0, y1), b1 = __floats2bfloat162_rn(y2, y3);
          __stcs(reinterpret_cast<uint2*>(d),
                 make_uint2(*reinterpret_cast<uint32_t*>(&b0), *reinterpret_cast<uint32_t*>(&b1)));
        }
      }
    }
    __syncwarp();
  }
}

struct Span {
  int c0, c1;
};

// Chunk run of segment s: one contiguous, balanced run per segment (STREAM: the whole
// sequence).  With n_s <= Nc every segment holds at least one chunk.
__device__ __forceinline__ Span seg_span(const FusedParams& fp, int s) {
  if (fp.mode == 0) return Span{0, fp.Nc};  // (SEGMENTED and CLUSTER: balanced runs)
  return Span{(int)((long long)s * fp.Nc / fp.n_s), (int)((long long)(s + 1) * fp.Nc / fp.n_s)};
}

// Phase parity for the n-th use of a barrier of a ring `depth` deep, and for waiting on
// the release of use n - depth (passes at once for n < depth on a fresh barrier).
template <int depth>
__device__ __forceinline__ uint32_t ph_use(int n) { return (uint32_t)(n / depth) & 1u; }
template <int depth>
__device__ __forceinline__ uint32_t ph_rel(int n) { return ((uint32_t)(n / depth) & 1u) ^ 1u; }

// Second phase of a segment s > 0, run by warpgroup q (named barrier q + 1) once the
// segment start state S_start is in shared memory: for chunk pairs m = q, q+4, ...
//   out = O_local + Qh' S_start,
// Qh' and O_local of the pair (two chunks each, consecutive in the workspace) come back
// by bulk copy into staging buffer q; one M = 128 MMA puts chunk 2m's rows in lanes
// 0-63 and chunk 2m+1's in lanes 64-127 of tensor-memory slot q; warp wq of the group
// takes lanes 32wq .. 32wq+31 (chunk 2m + wq/2, rows 32(wq%2) ..).
// Byte offset of the 8 bytes holding channels ch0 .. ch0+3 (ch0 a multiple of 4) of row
// `row` in a 128-byte-swizzled 16-bit tile.
__device__ __forceinline__ uint32_t sw_off8(int row, int ch0) {
  return row * 128u + ((((uint32_t)ch0 >> 3) ^ ((uint32_t)row & 7u)) << 4) + ((ch0 >> 2) & 1) * 8;
}

// Byte offset of channels ch0 .. ch0+3 of row `row` in the raw q / k tiles as loaded:
// 128-byte-swizzled 64-channel rows (d_k = 64), dense 64-byte rows (d_k = 32).
template <int kDK>
__device__ __forceinline__ uint32_t raw_off8(int row, int ch0) {
  return kDK == 64 ? sw_off8(row, ch0) : (uint32_t)(row * 64 + 2 * ch0);
}

// Largest |x| over `bytes` bytes of 16-bit values as a bit pattern with the sign dropped
// (for non-negative fp16 and bf16 values the integer order of the patterns is their
// numeric order), reduced over the calling warp; a warpgroup's 128 threads cover the tile.
__device__ __forceinline__ uint32_t absmax_bits(const uint8_t* t, int bytes, int wtid) {
  uint32_t m = 0;
  for (int i = wtid; i < bytes / 16; i += kWG) {
    const uint4 x = *reinterpret_cast<const uint4*>(t + 16 * i);
    m = __vmaxu2(__vmaxu2(m, x.x & 0x7fff7fffu), x.y & 0x7fff7fffu);
    m = __vmaxu2(__vmaxu2(m, x.z & 0x7fff7fffu), x.w & 0x7fff7fffu);
  }
  return __reduce_max_sync(0xffffffffu, max(m & 0xffffu, m >> 16));
}

template <typename T> __device__ __forceinline__ float bits16_to_float(unsigned int b);
template <> __device__ __forceinline__ float bits16_to_float<__half>(unsigned int b) {
  return __half2float(__ushort_as_half((unsigned short)b));
}
template <> __device__ __forceinline__ float bits16_to_float<__nv_bfloat16>(unsigned int b) {
  return __uint_as_float(b << 16);
}
// Exponent e >= 0 of the power of two that brings a tile maximum m into [1, 2), applied
// only when 0 < m < 2^-6 (inputs that small would lose their precision, or vanish, in the
// fp16 operands).  At most 40 for bf16 inputs, so that the undoing factors stay normal
// fp32 numbers; at most 15 for fp16 inputs, whose factors are applied inside fp16 numbers
// (2^15 already brings the smallest fp16 subnormal, 2^-24, up to 2^-9).
template <typename Tin>
__device__ __forceinline__ int input_scale_exp(float m) {
  if (!(m > 0.f) || m >= 0.015625f) return 0;
  int ex;
  (void)frexpf(m, &ex);  // m = f * 2^ex, f in [0.5, 1)
  return min(1 - ex, std::is_same<Tin, __half>::value ? 15 : 40);
}
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }  // |e| <= 126

// Scores of a chunk whose gates decay too fast for the factorisation, on the CUDA cores:
// d_k^-1/2 sum_k q_ik k_jk 2^(A_ik - A_jk) over scan(j) <= scan(i), from the raw q / k
// tiles and the full A in the gate tile, into the 16 rows of warp w4 of the chunk's score
// region (16x256b shape: register 4c+q is row r0 + 8(q>>1), column 8c + cq + (q&1)).
// Out of line: the chunk loops stay small for the instruction cache.
// d_k = 64: the raw q and k tiles are the 128-byte-swizzled Q and K tiles; d_k = 32: dense
// 64-byte rows at `qraw` / `kraw` (the upper half of the gate tile), the gate tile rows 32
// floats apart.
template <typename Tin, bool kRev, int kDK>
__device__ __noinline__ void cuda_core_scores(const uint8_t* sb, const float* G, uint32_t taddr, int w4, int lane,
                                              float ssc, float sq, float sk) {
  const uint8_t* qraw = kDK == 64 ? sb : reinterpret_cast<const uint8_t*>(G) + kRawQ;
  const uint8_t* kraw = kDK == 64 ? sb + kTile : reinterpret_cast<const uint8_t*>(G) + kRawK;
  const int r0 = 16 * w4 + (lane >> 2), cq = 2 * (lane & 3);
  for (int ps = 0; ps < 2; ++ps) {
    float sv[16];
    for (int x = 0; x < 16; ++x) {
      const int i = r0 + 8 * ((x & 3) >> 1);
      const int j = 32 * ps + 8 * (x >> 2) + cq + (x & 1);
      float acc = 0.f;
      if (kRev ? j >= i : j <= i) {  // scan(j) <= scan(i)
        for (int k = 0; k < kDK; k += 2) {
          const uint32_t oi = kDK == 64 ? sw128_offset(i, k) : (uint32_t)(i * 64 + 2 * k);
          const uint32_t oj = kDK == 64 ? sw128_offset(j, k) : (uint32_t)(j * 64 + 2 * k);
          float2 qv = In2<Tin>::unpack(*reinterpret_cast<const uint32_t*>(qraw + oi));
          float2 kv = In2<Tin>::unpack(*reinterpret_cast<const uint32_t*>(kraw + oj));
          qv.x *= sq, qv.y *= sq, kv.x *= sk, kv.y *= sk;  // the CTA's input factors (exact)
          acc = fmaf(qv.x * kv.x, ex2(G[i * kDK + k] - G[j * kDK + k]), acc);
          acc = fmaf(qv.y * kv.y, ex2(G[i * kDK + k + 1] - G[j * kDK + k + 1]), acc);
        }
      }
      sv[x] = acc * ssc;  // with qv sq, kv sk: the powers of two that Qh and Kh carry
    }
    tmem_st16x256_x4(taddr + 32u * ps, sv);
  }
}

// The other operand warpgroup's wait for the CTA's input scale (its first chunk): the
// factors sq, sk, sv, and w = 1 when the wait succeeded.  The caller flips its slot.  Out
// of line, like the CUDA-core chunk below: both run rarely, and code that stays in the
// chunk loop costs instruction-cache misses even when it is skipped.
__device__ __noinline__ float4 take_input_scale(int wg, int wtid, Misc* ms, WsHeader* hdr, int slot) {
  if (!wg_wait(wg, wtid, &ms->scale_ready, 0u, ms, hdr, 0x305, slot, true)) return make_float4(1.f, 1.f, 1.f, 0.f);
  return make_float4(ms->sc_in[0], ms->sc_in[1], ms->sc_in[2], 1.f);
}

// A chunk whose gates decay too fast for the factorisation: the full A (the thread's rows
// plus the offsets o0 / o1 of its two passes) into the gate tile, then, once the score
// region is free, the CUDA-core scores straight into tensor memory.  False: the wait gave
// up.  The caller flips its slot.
// Scores of a chunk whose gates allow the factorisation, in fp32 on the CUDA cores:
// d_k^-1/2 sum_k (q_ik 2^A_ik)(k_jk 2^-A_jk) over scan(j) <= scan(i) -- the tensor-core
// factorisation without its fp16 rounding.  The operand warpgroup first writes
// Kf = k 2^-A (times sk) transposed ([k][j], fp32) into `kft` (16 KB), then each thread
// forms its 32 scores (the 16x256b tensor-memory layout of cuda_core_scores: rows r0 and
// r0 + 8 of warp w4, 16 columns a pass) from its rows' q 2^A and the shared Kf.  Used for
// a sequence's first chunk under the output gate, whose first rows sum few terms.
template <typename Tin, bool kRev, int kDK>
__device__ __noinline__ void factored_scores(const uint8_t* sb, const float* G, float* kft, uint32_t taddr, int w4,
                                             int lane, int wg, int row0, int cc, float ssc, float sq, float sk) {
  const uint8_t* qraw = kDK == 64 ? sb : reinterpret_cast<const uint8_t*>(G) + kRawQ;
  const uint8_t* kraw = kDK == 64 ? sb + kTile : reinterpret_cast<const uint8_t*>(G) + kRawK;
  // Kf, transposed: this thread's rows row0 .. row0+3, channels 32p + 4cc .. +3
  for (int ps = 0; ps < kDK / 32; ++ps)
    for (int i = 0; i < 4; ++i) {
      const int j = row0 + i, k0 = 32 * ps + 4 * cc;
      for (int e = 0; e < 4; e += 2) {
        const uint32_t oj = kDK == 64 ? sw128_offset(j, k0 + e) : (uint32_t)(j * 64 + 2 * (k0 + e));
        const float2 kv = In2<Tin>::unpack(*reinterpret_cast<const uint32_t*>(kraw + oj));
        kft[(k0 + e) * 64 + j] = kv.x * sk * ex2(-G[j * kDK + k0 + e]);
        kft[(k0 + e + 1) * 64 + j] = kv.y * sk * ex2(-G[j * kDK + k0 + e + 1]);
      }
    }
  wg_sync(wg);
  const int r0 = 16 * w4 + (lane >> 2), cq = 2 * (lane & 3);
  for (int ps = 0; ps < 2; ++ps) {
    float acc[2][8];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[r][t] = 0.f;
    for (int k = 0; k < kDK; k += 2) {
      float2 qf[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = r0 + 8 * r;
        const uint32_t oi = kDK == 64 ? sw128_offset(i, k) : (uint32_t)(i * 64 + 2 * k);
        const float2 qv = In2<Tin>::unpack(*reinterpret_cast<const uint32_t*>(qraw + oi));
        qf[r] = make_float2(qv.x * sq * ex2(G[i * kDK + k]), qv.y * sq * ex2(G[i * kDK + k + 1]));
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 kf = *reinterpret_cast<const float2*>(kft + (k + kk) * 64 + 32 * ps + 8 * c + cq);
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const float q1 = kk ? qf[r].y : qf[r].x;
            acc[r][2 * c] = fmaf(q1, kf.x, acc[r][2 * c]);
            acc[r][2 * c + 1] = fmaf(q1, kf.y, acc[r][2 * c + 1]);
          }
        }
    }
    float sv[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const int r = (x & 3) >> 1, c = x >> 2, b = x & 1;
      const int i = r0 + 8 * r, j = 32 * ps + 8 * c + cq + b;
      sv[x] = (kRev ? j >= i : j <= i) ? acc[r][2 * c + b] * ssc : 0.f;  // scan(j) <= scan(i)
    }
    tmem_st16x256_x4(taddr + 32u * ps, sv);
  }
}

template <typename Tin, bool kRev, int kDK>
__device__ __noinline__ bool cuda_core_chunk(float* G, float4 o0, float4 o1, int row0, int cc, Misc* ms,
                                             WsHeader* hdr, int wg, int wtid, int slot, int n, const uint8_t* sb,
                                             uint32_t taddr, int w4, int lane, float ssc, float sq, float sk,
                                             float* kft) {
  for (int ps = 0; ps < kDK / 32; ++ps) {
    const float4 o = ps ? o1 : o0;
    for (int i = 0; i < 4; ++i) {
      float4* gp = reinterpret_cast<float4*>(G + (row0 + i) * kDK + 32 * ps + 4 * cc);
      const float4 a4 = *gp;
      *gp = make_float4(a4.x + o.x, a4.y + o.y, a4.z + o.z, a4.w + o.w);
    }
  }
  if (!wg_wait(wg, wtid, &ms->su_free[n % kSU], ph_rel<kSU>(n), ms, hdr, 0x302, slot)) return false;
  tc_fence_after();  // (the wait's barrier also publishes the full A)
  if (kft)  // gates that allow the factorisation: fp32 factored scores
    factored_scores<Tin, kRev, kDK>(sb, G, kft, taddr, w4, lane, wg, row0, cc, ssc, sq, sk);
  else
    cuda_core_scores<Tin, kRev, kDK>(sb, G, taddr, w4, lane, ssc, sq, sk);
  tmem_wait_st();
  tc_fence_before();
  wg_sync(wg);  // raw q / k reads done before the overwrite
  return true;
}

// Bulk copies of pair m2's Qh' and O_local tiles into staging buffer q (second phase).
__device__ __forceinline__ void p2_load(const FusedParams& fp, Misc* ms, uint8_t* smem, int seq, Span sp, int q, int m2) {
  const int c = sp.c0 + 2 * m2, nb = min(2, sp.c1 - c);
  const size_t t0 = ((size_t)seq * fp.Nc + c) * 4096;
  uint8_t* sbuf = smem + kOffStage + q * kStageBytes;
  mbar_arrive_expect_tx(&ms->p2_full[q], (uint32_t)(2 * nb * kTile));
  bulk_load(sbuf, fp.qhp + t0, (uint32_t)(nb * kTile), &ms->p2_full[q]);
  bulk_load(sbuf + kP2Olc, fp.olc + t0, (uint32_t)(nb * kTile), &ms->p2_full[q]);
}

template <typename Tin, typename Tout, int kDK, bool kBlock>
__device__ __forceinline__ void second_phase_body(const FusedParams& fp, Misc* ms, WsHeader* hdr, uint8_t* smem,
                                                  uint32_t tmem, int q, int wtid, int lane, int seq, int b, int h,
                                                  Span sp, int& slot, float& nf) {
  const int wq = (wtid >> 5) & 3;
  if (!wg_wait(q, wtid, &ms->p2_go, 0u, ms, hdr, 0x700u + q, slot)) return;
  const long long L = fp.p.L();
  const int cnt = sp.c1 - sp.c0, npairs = (cnt + 1) / 2;
  uint8_t* sbuf = smem + kOffStage + q * kStageBytes;
  const uint32_t s_base = smem_u32(smem);
  const uint32_t a0 = s_base + kOffStage + q * kStageBytes;
  const uint32_t id_128 = idesc_f16(0, 128, 64, 0, 1);  // A K-major, B MN-major
  const uint32_t dq = tmem + 64u * (uint32_t)q;
  int u = 0;
  for (int m2 = q; m2 < npairs; m2 += 4, ++u) {
    if (wtid == 0 && u > 0) p2_load(fp, ms, smem, seq, sp, q, m2);  // (the first pair's load is issued early)
    if (!wg_wait(q, wtid, &ms->p2_full[q], (uint32_t)u & 1u, ms, hdr, 0x710u + q, slot)) return;
    if (wtid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < kDK / 16; ++k)
        mma_f16(dq, sw128_desc(a0 + 32 * k), sw128_desc(s_base + kOffSst + 2048 * k), id_128, k > 0);
      mma_commit(&ms->p2_mma[q]);
    }
    if (!wg_wait(q, wtid, &ms->p2_mma[q], (uint32_t)u & 1u, ms, hdr, 0x720u + q, slot)) return;
    tc_fence_after();
    const int ci = 2 * m2 + (wq >> 1), row = 32 * (wq & 1) + lane;
    long long s = 0;
    const bool valid = ci < cnt && chunk_scan_pos(fp, sp.c0 + ci, fp.rev ? 63 - row : row, L, s);
    const uint8_t* olc_rows = sbuf + kP2Olc + (wq >> 1) * kTile + 32 * (wq & 1) * 128;
    // fp32 staging over the pair's Qh' (its MMA has completed)
    if (kBlock && fp.gated)
      gated_rows<Tout, Tin>(dq + ((uint32_t)(32 * wq) << 16), olc_rows + lane * 128, out_row<Tout>(fp, b, h, valid, s),
                            gate_row<Tin>(fp, b, h, valid, s), ms->nw, fp.p.oeps, sbuf + wq * 4096, lane, nf,
                            ms->sc_out);
    else
      epilogue_rows_add<Tout>(dq + ((uint32_t)(32 * wq) << 16), out_row<Tout>(fp, b, h, valid, s), olc_rows,
                              sbuf + wq * 4096, lane, nf, ms->sc_out);
    tc_fence_before();
    fence_proxy_async_smem();  // generic accesses of the buffer before the next pair's copies
    wg_sync(q);
  }
}

// How the second phase joins the kernel, per output type, by the measured time of segmented
// launches: fp16 outputs inline, bf16 outputs as the compiler decides, fp32 outputs (twice
// the staging traffic and registers) as a call, which keeps the kernel's own register
// allocation from spilling.
template <typename Tin, typename Tout, int kDK, bool kBlock>
__device__ __noinline__ void second_phase_call(const FusedParams& fp, Misc* ms, WsHeader* hdr, uint8_t* smem,
                                               uint32_t tmem, int q, int wtid, int lane, int seq, int b, int h,
                                               Span sp, int& slot, float& nf) {
  second_phase_body<Tin, Tout, kDK, kBlock>(fp, ms, hdr, smem, tmem, q, wtid, lane, seq, b, h, sp, slot, nf);
}
template <typename Tin, typename Tout, int kDK, bool kBlock>
__device__ void second_phase_auto(const FusedParams& fp, Misc* ms, WsHeader* hdr, uint8_t* smem, uint32_t tmem,
                                  int q, int wtid, int lane, int seq, int b, int h, Span sp, int& slot, float& nf) {
  second_phase_body<Tin, Tout, kDK, kBlock>(fp, ms, hdr, smem, tmem, q, wtid, lane, seq, b, h, sp, slot, nf);
}
template <typename Tin, typename Tout, int kDK, bool kBlock>
__device__ __forceinline__ void second_phase(const FusedParams& fp, Misc* ms, WsHeader* hdr, uint8_t* smem,
                                             uint32_t tmem, int q, int wtid, int lane, int seq, int b, int h, Span sp,
                                             int& slot, float& nf) {
  if constexpr (sizeof(Tout) == 4)
    second_phase_call<Tin, Tout, kDK, kBlock>(fp, ms, hdr, smem, tmem, q, wtid, lane, seq, b, h, sp, slot, nf);
  else if constexpr (std::is_same<Tout, __half>::value)
    second_phase_body<Tin, Tout, kDK, kBlock>(fp, ms, hdr, smem, tmem, q, wtid, lane, seq, b, h, sp, slot, nf);
  else
    second_phase_auto<Tin, Tout, kDK, kBlock>(fp, ms, hdr, smem, tmem, q, wtid, lane, seq, b, h, sp, slot, nf);
}

// kBlock: the kernel also carries the optional pieces of the GTR block (low-rank gate
// producer, RMSNorm + SiLU output gate), switched on at run time by fp.lowrank / fp.gated;
// the kernels without them keep none of their code.
template <typename Tin, typename Tout, bool kRev, bool kBox, int kMode, int kDK, bool kBlock>
__global__ void __launch_bounds__(kThreads, 1)
    fused_gla_kernel(const __grid_constant__ FusedParams fp) {
  constexpr bool kOL = kMode == 1;  // out-of-line slow paths of the waits
  const bool lowrank = kBlock && fp.lowrank != 0;
  const bool gated = kBlock && fp.gated != 0;
  static_assert(kDK == 64 || kDK == 32, "key widths 64 and 32");
  // the power of two of d_k^-1/2 that Kh carries; d_k = 32 applies the remaining 2^-1/2 to
  // the outputs (sc_out)
  constexpr float kKf = kDK == 64 ? 0.125f : 0.25f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc* ms = reinterpret_cast<Misc*>(smem + kOffMisc);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const Problem& p = fp.p;
  WsHeader* hdr = fp.hdr;

  // kMode: the plan's mode (0 STREAM, 1 SEGMENTED, 2 CLUSTER) fixed at compile time, or -1:
  // read at run time (the kernel with the GTR block pieces).  Each mode's own kernel holds
  // only that mode's code: the segmented one spills a little more than the run-time one
  // but misses the instruction cache less, and was measured faster (2048^2: 59.1 -> 57.3 us).
  const bool segm = kMode < 0 ? fp.mode == 1 : kMode == 1;  // the CTAs of a sequence exchange segment summaries
  const bool clus = kMode < 0 ? fp.mode == 2 : kMode == 2;  // ... through distributed shared memory
  const int seq = (segm || clus) ? (int)blockIdx.x / fp.n_s : (int)blockIdx.x;
  const int seg = (segm || clus) ? (int)blockIdx.x % fp.n_s : 0;
  // outputs completed in the second phase: segments s > 0, and with the output gate segment 0
  // too (its start state is zero), so that its gated epilogues run on all four warpgroups in
  // the second phase instead of holding up every segment at the summary barrier
  const bool partial = segm && (seg > 0 || gated);
  const int b = seq / p.heads, h = seq % p.heads;
  const long long L = p.L();
  const Span sp = seg_span(fp, seg);
  const int cnt = sp.c1 - sp.c0;           // chunks of this CTA
  // CLUSTER with at most kStages chunks a CTA: the staging buffers are never refilled, so
  // each chunk's Qh stays in its own and becomes Qh' in place at the end
  const bool inplace = clus && cnt <= kStages;
  const bool qhw = partial || (clus && seg > 0 && !inplace);  // Qh' tiles go to the workspace (the Qh' warp)
  float nonfinite = 0.f;
  bool cwaited = false;                    // CLUSTER: this thread has passed the start barrier

  // The next launch may start its prologue now (programmatic dependent launch): it waits
  // for this grid to complete before it touches global memory.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  static_assert(kStages <= 8 && kSU <= 8 && kNS <= 8 && kOPairs <= 8, "barrier arrays fit lanes 0-7");
  if (warp == 0) {  // lane i initialises entry i of every barrier array (a few inits a lane)
    const int i = lane;
    if (i < kStages) {
      mbar_init(&ms->full[i], fp.tma ? 1 : kProducerThreads);
      mbar_init(&ms->empty[i], 1);
      mbar_init(&ms->opready[i], 4);  // every warp of the WG_A warpgroup that builds the chunk
      mbar_init(&ms->qdone[i], 1);
      ms->fb[i] = 0;
    }
    if (i < kSU) {
      mbar_init(&ms->su_full[i], 1);
      mbar_init(&ms->su_free[i], 1);
      mbar_init(&ms->pready[i], 4);  // every WG_B warp
    }
    if (i < kNS) mbar_init(&ms->sready[i], 4);  // every WG_B warp
    if (i < kOPairs) {
      mbar_init(&ms->o_full[i], 1);
      mbar_init(&ms->o_free[i], 1);
      mbar_init(&ms->corr_done[i], 1);
    }
    if (i < 4) {
      mbar_init(&ms->p2_full[i], 1);
      mbar_init(&ms->p2_mma[i], 1);
      ms->go[i][0] = ms->go[i][1] = 0;
    }
    if (i == 8) mbar_init(&ms->agg_pub, qhw ? 2 : 1);  // WG_B (summary); the Qh' warp when it runs
    if (i == 10) mbar_init(&ms->mma_final[0], 1);
    if (i == 11) mbar_init(&ms->mma_final[1], 1);
    if (i == 9) mbar_init(&ms->p2_go, 1);
    if (i == 12) ms->abort = 0;
    if (i == 13) mbar_init(&ms->scale_ready, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ms->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ms->tmem_base;
  // every global access of this grid comes after the previous grid in the stream has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // CLUSTER: a CTA's shared memory is written by the others only once every CTA of the
  // cluster has started (the matching wait comes before the first remote access)
  if (clus) cluster_arrive_relaxed();

  if (warp == 16) {
    // ===================================================================== producer
    // Staged chunk row r holds scan position c*64 + r, or c*64 + 63 - r for the reversed
    // directions (right-to-left, bottom-to-top), where a chunk is stored in memory order.
    // A staging buffer is refilled once the P V of its previous chunk has completed and,
    // in a segment s > 0, that chunk's Qh' has been copied out.
    auto stage_free = [&](int n, int st) -> bool {
      if (!wait_bar<kOL>(&ms->empty[st], ph_rel<kStages>(n), ms, hdr, 0x100)) return false;
      return !qhw || wait_bar<kOL>(&ms->qdone[st], ph_rel<kStages>(n), ms, hdr, 0x101);
    };
    if constexpr (kBox) {
      // One thread issues four TMA boxes per chunk (Q, K, V with the 128-byte swizzle, G
      // plain); rows past the sequence end arrive zero-filled.
      if (lane == 0) {
        for (int c = sp.c0, n = 0; c < sp.c1; ++c, ++n) {
          const int st = n % kStages;
          if (!stage_free(n, st)) break;
          uint8_t* sb = smem + kOffStage + st * kStageBytes;
          uint8_t* qd = kDK == 64 ? sb : sb + 3 * kTile + kRawQ;  // raw q and k (d_k = 32: dense, in the gate tile)
          uint8_t* kd = kDK == 64 ? sb + kTile : sb + 3 * kTile + kRawK;
          mbar_arrive_expect_tx(&ms->full[st], chunk_load_bytes<kDK>(fp, lowrank));
          const long long s0 = (long long)c * kChunk;
          if (fp.lines) {
            // line chunk: the 64 cells of grid line c from o0 (memory order along the line);
            // cells past either end of the line read as zeros (k = v = 0 and log gamma = 0
            // there: the state passes such rows unchanged)
            const int o0 = kRev ? fp.len - kChunk : 0;
            const int cx = p.direction <= GTR_R2L ? o0 : c, cy = p.direction <= GTR_R2L ? c : o0;
            tma_load_5d(qd, &fp.tq, &ms->full[st], 0, h, cx, cy, b);
            tma_load_5d(kd, &fp.tk, &ms->full[st], 0, h, cx, cy, b);
            tma_load_5d(sb + 2 * kTile, &fp.tv, &ms->full[st], 0, h, cx, cy, b);
            tma_load_5d(sb + 3 * kTile, &fp.tg, &ms->full[st], 0, h, cx, cy, b);
          } else if (p.direction <= GTR_R2L) {
            // row view: 64 consecutive grid cells m (right-to-left: one image row)
            long long m0 = s0;
            if (p.direction == GTR_R2L) {
              const long long y = s0 / p.W;
              m0 = y * p.W + (p.W - 64 - (s0 - y * p.W));
            }
            tma_load_4d(qd, &fp.tq, &ms->full[st], 0, h, (int)m0, b);
            tma_load_4d(kd, &fp.tk, &ms->full[st], 0, h, (int)m0, b);
            tma_load_4d(sb + 2 * kTile, &fp.tv, &ms->full[st], 0, h, (int)m0, b);
            if (lowrank)  // the token's z row (per-token tensor: heads coordinate 0)
              tma_load_4d(sb + 3 * kTile, &fp.tz, &ms->full[st], 0, 0, (int)m0, b);
            else
              tma_load_4d(sb + 3 * kTile, &fp.tg, &ms->full[st], 0, h, (int)m0, b);
          } else {
            // column view: 64 consecutive y of one column x
            const int x = (int)(s0 / p.H);
            int y0 = (int)(s0 - (long long)x * p.H);
            if (p.direction == GTR_B2T) y0 = p.H - 64 - y0;
            tma_load_5d(qd, &fp.tq, &ms->full[st], 0, h, x, y0, b);
            tma_load_5d(kd, &fp.tk, &ms->full[st], 0, h, x, y0, b);
            tma_load_5d(sb + 2 * kTile, &fp.tv, &ms->full[st], 0, h, x, y0, b);
            if (lowrank)
              tma_load_5d(sb + 3 * kTile, &fp.tz, &ms->full[st], 0, 0, x, y0, b);
            else
              tma_load_5d(sb + 3 * kTile, &fp.tg, &ms->full[st], 0, h, x, y0, b);
          }
        }
      }
    } else if (fp.tma == 2) {
      // Chunks that are not one box (right-to-left rows or columns not a multiple of 64
      // long): lane t resolves the rows of scan positions c*64 + t and c*64 + 32 + t (the
      // direction remap) in the 2-D row views [B*L*heads][64] into a shared table; then
      // each lane issues two 4-row TMA gathers (lanes 8i .. 8i+7: tensor i of Q, K, V, G),
      // which land in the same tile layouts as the boxes.  Rows past the sequence end point
      // past the view and arrive zero-filled.
      const int oob = (int)((long long)p.B * L * p.heads);  // first row past the views
      const int rbase = (int)((long long)b * L * p.heads + h);
      const int t = lane >> 3, g0 = 2 * (lane & 7);
      const void* tmap = t == 0 ? (const void*)&fp.tq : t == 1 ? (const void*)&fp.tk
                         : t == 2 ? (const void*)&fp.tv : lowrank ? (const void*)&fp.tz : (const void*)&fp.tg;
      // low-rank gate producer: z rows of a per-token [B*L][rank] view
      const int zoob = (int)((long long)p.B * L), zbase = (int)((long long)b * L);
      for (int c = sp.c0, n = 0; c < sp.c1; ++c, ++n) {
        const int st = n % kStages;
        int* rows = ms->rowoff[n & 1];
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          const int pt = lane + 32 * hlf;
          const long long s = (long long)c * kChunk + pt;
          const int tok = s < L ? (int)scan_token(fp, (uint32_t)s) : -1;
          rows[kRev ? 63 - pt : pt] = tok >= 0 ? rbase + tok * p.heads : oob;
          ms->zrow[n & 1][kRev ? 63 - pt : pt] = tok >= 0 ? zbase + tok : zoob;
        }
        int ok = 0;
        if (lane == 0) {
          ok = stage_free(n, st) ? 1 : 0;
          if (ok) mbar_arrive_expect_tx(&ms->full[st], chunk_load_bytes<kDK>(fp, lowrank));  // the arrival comes first
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        __syncwarp();  // (the row table is complete)
        uint8_t* sb = smem + kOffStage + st * kStageBytes;
        // q, k: 64-channel swizzled tiles, or (d_k = 32) dense 64-byte rows in the gate tile
        uint8_t* tile = t == 2 ? sb + 2 * kTile
                        : t == 3 ? sb + 3 * kTile
                        : kDK == 64 ? sb + t * kTile : sb + 3 * kTile + (t == 0 ? kRawQ : kRawK);
        const bool zt = t == 3 && lowrank;
        const int rowb = t == 2 ? 128 : t == 3 ? (zt ? 4 * p.grank : 4 * kDK) : 2 * kDK;
        const int* rr = zt ? ms->zrow[n & 1] : rows;
#pragma unroll
        for (int gi = g0; gi < g0 + 2; ++gi)
          tma_gather4(tile + gi * 4 * rowb, tmap, &ms->full[st], 0, rr[4 * gi], rr[4 * gi + 1], rr[4 * gi + 2],
                      rr[4 * gi + 3]);
      }
    } else {
      // Per chunk, lane t first resolves the grid cells of scan positions c*64 + t and
      // c*64 + 32 + t (the direction remap) into a shared table; then the warp copies the
      // tiles with whole 128-byte rows per group of 8 lanes (Q, K, V: placed in the
      // 128-byte-swizzle layout) and 256-byte gate rows per group of 16, so each copy
      // instruction touches only 4 (2) full lines.  Rows past the sequence end are
      // zero-filled (source size 0).
      const uint8_t* gq = reinterpret_cast<const uint8_t*>(p.q);
      const uint8_t* gk = reinterpret_cast<const uint8_t*>(p.k);
      const uint8_t* gv = reinterpret_cast<const uint8_t*>(p.v);
      const uint8_t* gg = reinterpret_cast<const uint8_t*>(p.log_gamma);
      const int j8 = lane & 7, rq = lane >> 3;     // 16-byte column, row within a group of 4
      const int j16 = lane & 15, rg = lane >> 4;   // gate rows: 16-byte column, row within 2
      for (int c = sp.c0, n = 0; c < sp.c1; ++c, ++n) {
        const int st = n % kStages;
        int* rows = ms->rowoff[n & 1];
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          const int pt = lane + 32 * hlf;
          const long long s = (long long)c * kChunk + pt;
          rows[kRev ? 63 - pt : pt] = s < L ? (int)((long long)b * L + scan_token(fp, (uint32_t)s)) : -1;
        }
        __syncwarp();
        int ok = 0;
        if (lane == 0) ok = stage_free(n, st) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;  // (the row table is complete, too)
        const uint32_t sb = smem_u32(smem + kOffStage + st * kStageBytes);
        if constexpr (kDK == 64) {
#pragma unroll 4
          for (int it = 0; it < 16; ++it) {
            const int row = 4 * it + rq;
            const int cell = rows[row];
            const uint32_t nb = cell >= 0 ? 16u : 0u;
            const long long src = ((long long)(cell >= 0 ? cell : 0) * p.heads + h) * 128 + 16 * j8;
            const uint32_t dst = sb + row * 128 + (uint32_t)((j8 ^ (row & 7)) << 4);
            cp_async16(dst, gq + src, nb);
            cp_async16(dst + kTile, gk + src, nb);
            cp_async16(dst + 2 * kTile, gv + src, nb);
          }
#pragma unroll 4
          for (int it = 0; it < 32 && !lowrank; ++it) {
            const int row = 2 * it + rg;
            const int cell = rows[row];
            const uint32_t nb = cell >= 0 ? 16u : 0u;
            cp_async16(sb + 3 * kTile + row * 256 + 16 * j16,
                       gg + ((long long)(cell >= 0 ? cell : 0) * p.heads + h) * 256 + 16 * j16, nb);
          }
        } else {
          // d_k = 32: q and k 64-byte rows (groups of 4 lanes) dense into the gate tile's
          // upper half; v 128-byte rows (swizzled) and gate 128-byte rows per group of 8
          const int j4 = lane & 3, r8 = lane >> 2;
#pragma unroll 4
          for (int it = 0; it < 8; ++it) {
            const int row = 8 * it + r8;
            const int cell = rows[row];
            const uint32_t nb = cell >= 0 ? 16u : 0u;
            const long long src = ((long long)(cell >= 0 ? cell : 0) * p.heads + h) * 64 + 16 * j4;
            cp_async16(sb + 3 * kTile + kRawQ + row * 64 + 16 * j4, gq + src, nb);
            cp_async16(sb + 3 * kTile + kRawK + row * 64 + 16 * j4, gk + src, nb);
          }
#pragma unroll 4
          for (int it = 0; it < 16; ++it) {
            const int row = 4 * it + rq;
            const int cell = rows[row];
            const uint32_t nb = cell >= 0 ? 16u : 0u;
            const long long src = ((long long)(cell >= 0 ? cell : 0) * p.heads + h) * 128 + 16 * j8;
            cp_async16(sb + 2 * kTile + row * 128 + (uint32_t)((j8 ^ (row & 7)) << 4), gv + src, nb);
            if (!lowrank) cp_async16(sb + 3 * kTile + row * 128 + 16 * j8, gg + src, nb);
          }
        }
        if (lowrank) {
          // z rows (rank / 4 pieces of 16 bytes a row) dense at the start of the gate tile
          const int P = p.grank / 4;
          const uint8_t* gz = reinterpret_cast<const uint8_t*>(p.gz);
          for (int idx = lane; idx < 64 * P; idx += 32) {
            const int row = idx / P, pc = idx - row * P;
            const int cell = rows[row];
            cp_async16(sb + 3 * kTile + row * 16 * P + 16 * pc,
                       gz + (long long)(cell >= 0 ? cell : 0) * 16 * P + 16 * pc, cell >= 0 ? 16u : 0u);
          }
        }
        cp_async_arrive_noinc(&ms->full[st]);
      }
      // copies already issued must land before this CTA's shared memory is released
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
  } else if (warp == kQhWarp) {
    // ===================================================================== Qh' tiles
    // Segment s > 0: per chunk, Qh' = Qh 2^(A from the segment start) -> the chunk's
    // workspace tile, fp16 in the staged 128-byte-swizzle layout (the A operand of the
    // second phase).  Lane l keeps the decay from the segment start of channels 2l, 2l+1
    // (the sum of the earlier chunks' decays, row 0 of their gate tiles) and takes the
    // 16-byte pieces l, l+32, ... of the tile, so every store instruction writes 512
    // contiguous bytes.
    if (qhw) {
      bool ok = true;
      float a2s0 = 0.f, a2s1 = 0.f;
      const float* eseg = ms->eseg;
      for (int c = sp.c0, n = 0; c < sp.c1; ++c, ++n) {
        const int st = n % kStages;
        if (!wait_bar<kOL>(&ms->opready[st], ph_use<kStages>(n), ms, hdr, 0x110)) { ok = false; break; }
        const uint8_t* qt = smem + kOffStage + st * kStageBytes;  // Qh, built in place
        {
          *reinterpret_cast<float2*>(&ms->eseg[2 * lane]) = make_float2(ex2(a2s0), ex2(a2s1));
          const float2 a2 = *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(qt + 3 * kTile) + 2 * lane);
          a2s0 += a2.x;
          a2s1 += a2.y;
          __syncwarp();
        }
        uint8_t* dst = reinterpret_cast<uint8_t*>(fp.qhp + ((size_t)seq * fp.Nc + c) * 4096);
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int idx = lane + 32 * i, r = idx >> 3, jp = idx & 7, jl = jp ^ (r & 7);
          uint4 v = *reinterpret_cast<const uint4*>(qt + r * 128 + 16 * jp);  // channels 8 jl .. 8 jl + 7
          const float4 e0 = *reinterpret_cast<const float4*>(eseg + 8 * jl);
          const float4 e1 = *reinterpret_cast<const float4*>(eseg + 8 * jl + 4);
          v.x = h2_bits(__hmul2(bits_h2(v.x), __floats2half2_rn(e0.x, e0.y)));
          v.y = h2_bits(__hmul2(bits_h2(v.y), __floats2half2_rn(e0.z, e0.w)));
          v.z = h2_bits(__hmul2(bits_h2(v.z), __floats2half2_rn(e1.x, e1.y)));
          v.w = h2_bits(__hmul2(bits_h2(v.w), __floats2half2_rn(e1.z, e1.w)));
          *reinterpret_cast<uint4*>(dst + r * 128 + 16 * jp) = v;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms->qdone[st]);  // the staged chunk is released
      }
      // the tiles are read back by bulk copy (async proxy)
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&ms->agg_pub);
    }
  } else if (warp == kMmaWarp) {
    // ===================================================================== MMA issuer, stage 1
    // Scores = Qh Kh^T (tensor-core chunks) and U' = Kh^T V, in chunk order, up to kSU
    // chunks ahead of the outputs.
    if (lane == 0) {
      const uint32_t id_qk = idesc_f16(0, 64, 64, 0, 0);  // A K-major, B K-major
      const uint32_t id_kv = idesc_f16(0, 64, 64, 1, 1);  // A MN-major, B MN-major
      const uint32_t s_base = smem_u32(smem);
      for (int n = 0; n < cnt; ++n) {
        const int st = n % kStages;
        if (!wait_spin<kOL>(&ms->opready[st], ph_use<kStages>(n), ms, hdr, 0x200)) break;
        if (!wait_spin<kOL>(&ms->su_free[n % kSU], ph_rel<kSU>(n), ms, hdr, 0x201)) break;
        const uint32_t a_q = s_base + kOffStage + st * kStageBytes;  // Qh (built in place)
        const uint32_t a_k = a_q + kTile;                            // Kh
        const uint32_t a_v = a_q + 2 * kTile;
        tc_fence_after();
        const uint32_t su = tmem + kColSU + 64u * (uint32_t)(n % kSU);
        if (!*(volatile int*)&ms->fb[st]) {  // (K = d_k: channels past d_k are zero)
          for (int k = 0; k < kDK / 16; ++k)
            mma_f16(su, sw128_desc(a_q + 32 * k), sw128_desc(a_k + 32 * k), id_qk, k > 0);
        }
        for (int k = 0; k < 4; ++k)
          mma_f16(su + kLaneTile1, sw128_desc(a_k + 2048 * k), sw128_desc(a_v + 2048 * k), id_kv, k > 0);
        mma_commit(&ms->su_full[n % kSU]);
      }
      // every MMA issued here has completed before tensor memory is freed
      mma_commit(&ms->mma_final[0]);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&ms->mma_final[0], 0) && globaltimer() - t0 < 1000000000ull) {
      }
    }
  } else if (warp == kOutWarp) {
    // ===================================================================== MMA issuer, stage 2
    // Per chunk m in order: O = Qh S (2a, once Qh is built, the chunk-start state is
    // written and, for the first chunk of a pair, the pair's output region is free), then
    // O += P V (2b, with P in tensor memory), which frees the chunk's staging buffer and
    // score region.
    if (lane == 0) {
      const uint32_t id_qs = idesc_f16(0, 64, 64, 0, 1);  // A K-major, B MN-major
      const uint32_t s_base = smem_u32(smem);
      for (int m = 0; m < cnt; ++m) {
        const int st = m % kStages, su = m % kSU;
        // output region of chunk m: pair (m/2) % 2, lane tile m % 2
        const uint32_t d_o = tmem + kColO + 64u * (uint32_t)((m >> 1) % kOPairs) + ((m & 1) ? kLaneTile1 : 0u);
        // Qh built (the stage-1 issuer waits on the same phase; neither can lap it, as the
        // stage is refilled only after this chunk's P V), chunk-start state written
        if (!wait_spin<kOL>(&ms->opready[st], ph_use<kStages>(m), ms, hdr, 0x205)) break;
        if (!wait_spin<kOL>(&ms->sready[m % kNS], ph_use<kNS>(m), ms, hdr, 0x202)) break;
        if (!(m & 1) && !wait_spin<kOL>(&ms->o_free[(m >> 1) % kOPairs], ph_rel<kOPairs>(m >> 1), ms, hdr, 0x203)) break;
        const uint32_t a_q = s_base + kOffStage + st * kStageBytes;
        const uint32_t a_s = s_base + kOffS + (m % kNS) * kTile;
        tc_fence_after();
        for (int k = 0; k < kDK / 16; ++k)
          mma_f16(d_o, sw128_desc(a_q + 32 * k), sw128_desc(a_s + 2048 * k), id_qs, k > 0);
        if (!wait_spin<kOL>(&ms->pready[su], ph_use<kSU>(m), ms, hdr, 0x204)) break;
        // P sits in the lane tile of the chunk's output (A and D rows share lanes)
        const uint32_t a_v = a_q + 2 * kTile;
        const uint32_t a_p = tmem + kColSU + 64u * su + ((m & 1) ? kLaneTile1 : 0u);
        tc_fence_after();
        for (int k = 0; k < 4; ++k)
          mma_f16_ta(d_o, a_p + 8 * k, sw128_desc(a_v + 2048 * k), id_qs, 1);
        mma_commit(&ms->su_free[su]);
        mma_commit(&ms->empty[st]);
        if ((m & 1) || m + 1 == cnt) mma_commit(&ms->o_full[(m >> 1) % kOPairs]);
      }
      mma_commit(&ms->mma_final[1]);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&ms->mma_final[1], 0) && globaltimer() - t0 < 1000000000ull) {
      }
    }
  } else if (warp < 8) {
    // ===================================================================== WG_A: operand tiles
    // The two warpgroups take alternate chunks (warpgroup hh: chunks n = hh, hh+2, ...),
    // each in d_k / 32 passes over the key channels (two halves when d_k = 64): its warp w4
    // takes rows 16w4 .. 16w4+15, a thread 4 rows x 4 channels per pass.  d_k = 32: the
    // raw q and k sit in the upper half of the gate tile and Qh, Kh are built into the Q
    // and K tiles with channels 32 .. 63 zero.
    constexpr int kPasses = kDK / 32;
    const int hh = warp >> 2, w4 = warp & 3;
    const int wg = hh, wtid = tid - kWG * hh;
    const int cc = lane & 7;                     // channels 32p + 4cc .. 32p + 4cc + 3 in pass p
    const int row0 = 16 * w4 + 4 * (lane >> 3);  // rows row0 .. row0+3
    constexpr bool rev = kRev;
    int slot = 0;
    bool alive = true;
    float sq = 1.f, sk = 1.f, sv = 1.f;  // this CTA's input scale factors (set at the first chunk)
    if (lowrank) {
      // both warpgroups: this head's gate-producer columns and bias (zero past d_k) into
      // shared memory, then a barrier of the two (named barrier 5, 256 threads)
      const int ld = p.heads * kDK, t2 = tid;  // tid < 256 here
      for (int i = t2; i < 16 * 64; i += 2 * kWG) {
        const int j = i >> 6, c = i & 63;
        ms->w2s[j][c] = (j < p.grank && c < kDK) ? __ldg(p.gw2 + (long long)j * ld + h * kDK + c) : 0.f;
      }
      if (t2 < 64) ms->bs[t2] = t2 < kDK ? __ldg(p.gb + h * kDK + t2) : 0.f;
      asm volatile("bar.sync 5, 256;" ::: "memory");
    }
    for (int n = hh; n < cnt; n += 2) {
      const int st = n % kStages;
      if (!wg_wait<kOL>(wg, wtid, &ms->full[st], ph_use<kStages>(n), ms, hdr, 0x301, slot)) {
        alive = false;
        break;
      }
      uint8_t* sb = smem + kOffStage + st * kStageBytes;
      float* G = reinterpret_cast<float*>(sb + 3 * kTile);
      uint8_t* qr = kDK == 64 ? sb : sb + 3 * kTile + kRawQ;  // raw q, k
      uint8_t* kr = kDK == 64 ? sb + kTile : sb + 3 * kTile + kRawK;
      if (n == 0) {
        // the CTA's first chunk: its largest |q|, |k|, |v| per warp (published by the
        // barrier after the gate sums, before any tile is overwritten)
        const uint32_t m0 = absmax_bits(qr, 128 * kDK, wtid), m1 = absmax_bits(kr, 128 * kDK, wtid);
        const uint32_t m2 = absmax_bits(sb + 2 * kTile, kTile, wtid);
        if (lane == 0) ms->smax[w4][0] = m0, ms->smax[w4][1] = m1, ms->smax[w4][2] = m2;
      }
      // ---- in-chunk cumulative log2-gates in scan order: my 4 rows (written back over
      // the gates, still without the offset of the rows before them), a scan over the
      // warp's 4 row blocks, then over the 4 warps through shared memory (staged rows run
      // backwards in scan order when the chunk is reversed)
      float run[2][4], incl[2][4];
      float lr[2][4][4];  // low-rank producer: this thread's ln gamma values
      if (lowrank) {
        // the gates come from the chunk's z rows (where the gate tile starts); every thread
        // has read its z rows before any thread writes the gate tile
        lowrank_gate_values<kDK>(G, ms, p.grank, fp.gtau_inv, row0, cc, lr);
        wg_sync(wg);
      }
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
        const int ch0 = 32 * ps + 4 * cc;
        float gv[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (lowrank) {
            gv[i][0] = lr[ps][i][0]; gv[i][1] = lr[ps][i][1]; gv[i][2] = lr[ps][i][2]; gv[i][3] = lr[ps][i][3];
          } else {
            const float4 g4 = *reinterpret_cast<const float4*>(G + (row0 + i) * kDK + ch0);
            gv[i][0] = g4.x; gv[i][1] = g4.y; gv[i][2] = g4.z; gv[i][3] = g4.w;
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) run[ps][e] = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = rev ? 3 - k : k;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            run[ps][e] = fmaf(gv[i][e], kLog2e, run[ps][e]);
            gv[i][e] = run[ps][e];
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<float4*>(G + (row0 + i) * kDK + ch0) = make_float4(gv[i][0], gv[i][1], gv[i][2], gv[i][3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = run[ps][e];
          if (!rev) {
            float x = __shfl_up_sync(0xffffffffu, v, 8);
            if (lane >= 8) v += x;
            x = __shfl_up_sync(0xffffffffu, v, 16);
            if (lane >= 16) v += x;
          } else {
            float x = __shfl_down_sync(0xffffffffu, v, 8);
            if (lane < 24) v += x;
            x = __shfl_down_sync(0xffffffffu, v, 16);
            if (lane < 16) v += x;
          }
          incl[ps][e] = v;
        }
        if (rev ? lane < 8 : lane >= 24)
          *reinterpret_cast<float4*>(&ms->red[hh][ps][w4][4 * cc]) =
              make_float4(incl[ps][0], incl[ps][1], incl[ps][2], incl[ps][3]);
      }
      wg_sync(wg);
      if (n == 0) {
        // the CTA's input scale: powers of two that bring a tiny first-chunk maximum into
        // [1, 2), so that scaling and undoing it are exact; every thread derives it from the
        // four warps' maxima, thread 0 publishes it for the other warpgroups
        int e[3];
#pragma unroll
        for (int t = 0; t < 3; ++t) {
          const unsigned int m = max(max(ms->smax[0][t], ms->smax[1][t]), max(ms->smax[2][t], ms->smax[3][t]));
          e[t] = input_scale_exp<Tin>(bits16_to_float<Tin>(m));
        }
        sq = pow2f(e[0]);
        sk = pow2f(e[1]);
        sv = pow2f(e[2]);
        if (wtid == 0) {
          ms->sc_in[0] = sq;
          ms->sc_in[1] = sk;
          ms->sc_in[2] = sv;
          ms->sc_out = pow2f(-(e[0] + e[1] + e[2])) * (kDK == 64 ? 1.f : 0.70710678118654752f);
          ms->sc_spub = pow2f(-(e[1] + e[2]));
          ms->sc_sin = pow2f(e[1] + e[2]);
          mbar_arrive(&ms->scale_ready);
        }
      } else if (n == hh) {
        // the other operand warpgroup's first chunk: the scale WG_A0 derived
        const float4 f = take_input_scale(wg, wtid, ms, hdr, slot);
        slot ^= 1;
        if (f.w == 0.f) {
          alive = false;
          break;
        }
        sq = f.x;
        sk = f.y;
        sv = f.z;
      }
      // fp16 inputs: V enters the MMAs as it is, and its factor sv rides on Kh instead
      // (2^ev on Kh's exponent; the factorisation limit shrinks by ev, so that Kh keeps its
      // range); bf16 inputs: V is converted to fp16 anyway, times sv
      constexpr bool kHalfIn = std::is_same<Tin, __half>::value;
      const float eq = __log2f(sq), evk = kHalfIn ? __log2f(sv) : 0.f;  // (exact: powers of two)
      const float max_exp2 = fp.max_exp2 - evk;
      // offsets of my rows (the rows of earlier lanes and warps) and the chunk decay a
      float off[2][4], last[2][4];
      bool exp_unsafe = false;
#pragma unroll
      for (int ps = 0; ps < kPasses; ++ps) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          off[ps][e] = incl[ps][e] - run[ps][e];
          last[ps][e] = 0.f;
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float4 t4 = *reinterpret_cast<const float4*>(&ms->red[hh][ps][w][4 * cc]);
          const float t[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (rev ? w > w4 : w < w4) off[ps][e] += t[e];
            last[ps][e] += t[e];
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (-last[ps][e] > max_exp2) exp_unsafe = true;
      }
      // CUDA-core decision: the lanes of every warp hold the decays of all d_k channels.  With
      // the output gate, the sequence's first chunk also takes the exact CUDA-core scores: its
      // first tokens' outputs sum few terms, and the RMSNorm scales each row to unit size, so
      // the fp16 rounding of the factorised operands would no longer be averaged away.
      const bool unsafe = __any_sync(0xffffffffu, exp_unsafe);
      const bool fbx = unsafe || (gated && sp.c0 + n == 0);
      if (fbx) {
        // ---- CUDA-core scores, straight into tensor memory (lane tile 0 of the chunk's
        // score region): d_k^-1/2 sum_k q_ik k_jk 2^(A_ik - A_jk) over scan(j) <= scan(i),
        // times the CTA's factors (Kh's: kKf sk, and sv for fp16 inputs).  The full A goes to
        // the gate tile so that every thread can read every row and channel.
        const bool ok = cuda_core_chunk<Tin, rev, kDK>(
            G, make_float4(off[0][0], off[0][1], off[0][2], off[0][3]),
            make_float4(off[kPasses - 1][0], off[kPasses - 1][1], off[kPasses - 1][2], off[kPasses - 1][3]), row0, cc,
            ms, hdr, wg, wtid, slot, n, sb, tmem + ((uint32_t)(32 * w4) << 16) + kColSU + 64u * (uint32_t)(n % kSU), w4,
            lane, kHalfIn ? kKf * sv : kKf, sq, sk,
            unsafe ? nullptr : reinterpret_cast<float*>(smem + kOffStg));  // (the staging area is idle until the first epilogue)
        slot ^= 1;
        if (!ok) {
          alive = false;
          break;
        }
#pragma unroll
        for (int ps = 0; ps < kPasses; ++ps)
#pragma unroll
          for (int e = 0; e < 4; ++e) off[ps][e] = 0.f;  // the gate tile holds the full A now
      }
      // ---- Qh = q 2^(A + eq), Kh = k 2^(evk - A) kKf sk (k 2^(a - A + evk) kKf sk for
      // CUDA-core chunks), kKf = 1/8 (d_k = 64: in place) or 1/4 (d_k = 32, the remaining
      // 2^-1/2 of d_k^-1/2 is applied to the outputs).  The factors ride on the offsets that
      // are added anyway: A + eq is the row's gate sum plus (offset + eq), and Kh's exponent
      // is (decay or 0) + eq + evk minus that, so they cost no instruction per element.
      const float kfs = kKf * sk;
      const __half2 kfh = __float2half2_rn(kfs);
#pragma unroll 1
      for (int ps = 0; ps < kPasses; ++ps) {  // (rolled: the loop body stays small for the instruction cache)
        const int ch0 = 32 * ps + 4 * cc;
        float offp[4], kx[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          offp[e] = (ps ? off[1][e] : off[0][e]) + eq;
          kx[e] = (fbx ? (ps ? last[1][e] : last[0][e]) : 0.f) + eq + evk;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = row0 + i;
          const float4 a4 = *reinterpret_cast<const float4*>(G + row * kDK + ch0);
          const float Ar[4] = {a4.x + offp[0], a4.y + offp[1], a4.z + offp[2], a4.w + offp[3]};
          // channels ch0 .. ch0+3: 8 bytes at 16-byte chunk ch0/8, half (ch0/4) & 1
          const uint32_t off8 = sw_off8(row, ch0);
          const uint32_t roff = raw_off8<kDK>(row, ch0);
          uint2 qraw = *reinterpret_cast<const uint2*>(qr + roff);
          uint2 kraw = *reinterpret_cast<const uint2*>(kr + roff);
          uint32_t* qw = reinterpret_cast<uint32_t*>(&qraw);
          uint32_t* kw = reinterpret_cast<uint32_t*>(&kraw);
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const float A0 = Ar[2 * e2], A1 = Ar[2 * e2 + 1];  // A + eq
            const float xk0 = kx[2 * e2] - A0, xk1 = kx[2 * e2 + 1] - A1;
            __half2 qh, kh;
            if constexpr (kHalfIn) {  // (2^(A + eq) <= 2^15, kfs <= 2^12, 2^xk0 <= 2^max(11.5, ev))
              qh = __hmul2(bits_h2(qw[e2]), bits_h2(pack_h2(ex2(A0), ex2(A1))));
              kh = __hmul2(__hmul2(bits_h2(kw[e2]), kfh), bits_h2(pack_h2(ex2(xk0), ex2(xk1))));
            } else {
              const float2 qv = In2<Tin>::unpack(qw[e2]), kv = In2<Tin>::unpack(kw[e2]);
              qh = __floats2half2_rn(qv.x * ex2(A0), qv.y * ex2(A1));
              kh = __floats2half2_rn(kv.x * kfs * ex2(xk0), kv.y * kfs * ex2(xk1));
            }
            qw[e2] = h2_bits(qh);
            kw[e2] = h2_bits(kh);
          }
          *reinterpret_cast<uint2*>(sb + off8) = qraw;
          *reinterpret_cast<uint2*>(sb + kTile + off8) = kraw;
          if constexpr (kDK == 32) {  // channels 32 .. 63 of Qh and Kh are zero
            const uint32_t offz = sw_off8(row, 32 + ch0);
            *reinterpret_cast<uint2*>(sb + offz) = make_uint2(0u, 0u);
            *reinterpret_cast<uint2*>(sb + kTile + offz) = make_uint2(0u, 0u);
          }
        }
      }
      if constexpr (!kHalfIn) {
        // bf16 inputs: the V tile becomes fp16 in place, times the CTA's v factor (exact
        // inside the fp16 range)
        uint4* vt = reinterpret_cast<uint4*>(sb + 2 * kTile);
#pragma unroll
        for (int i = wtid; i < kTile / 16; i += kWG) {
          uint4 x = vt[i];
          uint32_t* w = reinterpret_cast<uint32_t*>(&x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = In2<Tin>::unpack(w[e]);
            w[e] = pack_h2(f.x * sv, f.y * sv);
          }
          vt[i] = x;
        }
      }
      if (w4 == 0 && lane < 8) {
        // the first 64 floats of the gate tile (rows read by these lanes only, above) now
        // hold the chunk's decay a per key channel (0 for channels d_k .. 63)
#pragma unroll
        for (int ps = 0; ps < 2; ++ps)
          *reinterpret_cast<float4*>(G + 32 * ps + 4 * cc) =
              ps < kPasses ? make_float4(last[ps][0], last[ps][1], last[ps][2], last[ps][3])
                           : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (wtid == 0) ms->fb[st] = fbx ? 1 : 0;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->opready[st]);  // every warp, once its writes are done
    }
    if (partial && alive)
      second_phase<Tin, Tout, kDK, kBlock>(fp, ms, hdr, smem, tmem, wg, wtid, lane, seq, b, h, sp, slot, nonfinite);
  } else if (warp < 12) {
    // ===================================================================== WG_B: masking, state
    // Tensor-memory rows through the 16-lane shape: register 4c+q of this thread is row
    // r0 + 8(q>>1), column 8c + cq + (q&1) of the warp's 16-row slice.  No named barrier
    // inside the chunk loop: every thread waits on the mbarriers itself (bounded), every
    // warp arrives on the ones it feeds.
    const int wg = 2, wtid = tid - 2 * kWG, wq = warp & 3;
    const int r0 = 16 * wq + (lane >> 2), r1 = r0 + 8, cq = 2 * (lane & 3);
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);  // this warp's lane quarter
    constexpr bool rev = kRev;
    float Ls[32];                  // fp32 state entries (rows r0 / r1 = key channels)
    float a2r0 = 0.f, a2r1 = 0.f;  // log2 segment decay of rows r0 / r1
    int slot = 0;
    bool alive = true;
#pragma unroll
    for (int e = 0; e < 32; ++e) Ls[e] = 0.f;
    {  // zero start state of the segment's first chunk (state tile 0, first use)
      const uint4 z = make_uint4(0, 0, 0, 0);
      uint4* sz = reinterpret_cast<uint4*>(smem + kOffS);
      for (int i = wtid; i < kTile / 16; i += kWG) sz[i] = z;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->sready[0]);
    }
    for (int n = 0; n < cnt; ++n) {
      const int st = n % kStages, su = n % kSU;
      if (!wait_bar<kOL>(&ms->su_full[su], ph_use<kSU>(n), ms, hdr, 0x400)) { alive = false; break; }
      tc_fence_after();
      const bool fbk = ms->fb[st] != 0;
      const float* alast = reinterpret_cast<const float*>(smem + kOffStage + st * kStageBytes + 3 * kTile);
      const float l0 = alast[r0], l1 = alast[r1];
      const float dl0 = ex2(l0), dl1 = ex2(l1);
      const uint32_t sreg = tl + kColSU + 64u * (uint32_t)su;
      {
        float u[32];
        tmem_ld16x256_x8(sreg + kLaneTile1, u);
        tmem_wait_ld();
        // state rows r0 / r1: S <- 2^a (S + U')   (CUDA-core chunks: S <- 2^a S + U)
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const float d = (x & 2) ? dl1 : dl0;
          Ls[x] = fbk ? fmaf(d, Ls[x], u[x]) : d * (Ls[x] + u[x]);
        }
      }
      a2r0 += l0;
      a2r1 += l1;
      // masked scores -> fp16 P over the first 32 columns of the chunk's score region,
      // the A operand of P V.  A rows are read from the lanes of the output rows, so P
      // goes to the lane tile of the chunk's output region (tile 1: over U', already
      // loaded).  Register 2c+q of the 16x128b shape is row r0 + 8q, column 4c + lane%4,
      // i.e. the score pair (8c + cq, 8c + cq + 1) of that row.
      const uint32_t pdst = sreg + ((n & 1) ? kLaneTile1 : 0u);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {  // score columns 32hf .. 32hf+31 -> P columns 16hf .. 16hf+15
        float sc[16];
        tmem_ld16x256_x4(sreg + 32u * hf, sc);
        tmem_wait_ld();
        uint32_t pw[8];
#pragma unroll
        for (int cl = 0; cl < 4; ++cl) {
          const int cb = 4 * hf + cl;
          float x0 = sc[4 * cl], x1 = sc[4 * cl + 1], x2 = sc[4 * cl + 2], x3 = sc[4 * cl + 3];
          if (rev ? cb < 2 * wq : cb > 2 * wq + 1) {
            x0 = x1 = x2 = x3 = 0.f;  // scan(j) > scan(i) for the whole block
          } else if (cb >= 2 * wq && cb <= 2 * wq + 1) {
            const int j = 8 * cb + cq;
            if (!rev) {
              x0 = (j <= r0) ? x0 : 0.f;
              x1 = (j + 1 <= r0) ? x1 : 0.f;
              x2 = (j <= r1) ? x2 : 0.f;
              x3 = (j + 1 <= r1) ? x3 : 0.f;
            } else {
              x0 = (j >= r0) ? x0 : 0.f;
              x1 = (j + 1 >= r0) ? x1 : 0.f;
              x2 = (j >= r1) ? x2 : 0.f;
              x3 = (j + 1 >= r1) ? x3 : 0.f;
            }
          }
          pw[2 * cl] = pack_h2(x0, x1);
          pw[2 * cl + 1] = pack_h2(x2, x3);
        }
        tmem_st16x128_x4(pdst + 16u * hf, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms->pready[su]);
      if (n + 1 < cnt) {
        // the next chunk's start state, into state tile (n+1) % kNS.  Its last reader,
        // O = Qh S of chunk n+1-kNS, has completed: the P V of that chunk, issued after
        // it by the same thread, released the score region chunk n's scores went to.
        uint8_t* srow0 = smem + kOffS + ((n + 1) % kNS) * kTile + r0 * 128;
        uint8_t* srow1 = srow0 + 8 * 128;
#pragma unroll
        for (int cb = 0; cb < 8; ++cb) {
          const uint32_t o = (((uint32_t)cb ^ ((uint32_t)r0 & 7u)) << 4) + cq * 2;
          sts32(srow0 + o, pack_h2(Ls[4 * cb], Ls[4 * cb + 1]));
          sts32(srow1 + o, pack_h2(Ls[4 * cb + 2], Ls[4 * cb + 3]));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ms->sready[(n + 1) % kNS]);
      }
    }
    // every thread leaves the loop (the waits are bounded): agree on the outcome, and that
    // the input scale is known (the summaries go back to the inputs' scale; the scale was
    // set before chunk 0's operands, so this spin finds it complete)
    if ((segm || clus) && alive) alive = wait_spin<kOL>(&ms->scale_ready, 0u, ms, hdr, 0x405);
    alive = wg_all(wg, alive);
    if (clus && alive) {
      // segment summary for the cluster's scan, read by the other CTAs after the cluster
      // barrier: U_seg (fp32, row-major) over the output staging area (idle: the outputs
      // are held), the log2 decay per key channel in the misc area
      float* U = reinterpret_cast<float*>(smem + kOffStg);
      const float f = ms->sc_spub;  // in the inputs' scale
#pragma unroll
      for (int cb = 0; cb < 8; ++cb) {
        *reinterpret_cast<float2*>(U + r0 * 64 + 8 * cb + cq) = make_float2(Ls[4 * cb] * f, Ls[4 * cb + 1] * f);
        *reinterpret_cast<float2*>(U + r1 * 64 + 8 * cb + cq) = make_float2(Ls[4 * cb + 2] * f, Ls[4 * cb + 3] * f);
      }
      if ((lane & 3) == 0) {
        ms->dseg[r0] = a2r0;
        ms->dseg[r1] = a2r1;
      }
      wg_sync(wg);
      if (wtid == 0) mbar_arrive(&ms->agg_pub);
    }
    if (segm && alive) {
      // segment summary: U_seg = local end state (in the inputs' scale), its log2 decay, and
      // the factor that takes a start state into this CTA's scale
      float* mine = fp.agg + ((size_t)seq * fp.n_s + seg) * kAggStride;
      const float f = ms->sc_spub;
#pragma unroll
      for (int cb = 0; cb < 8; ++cb) {
        __stcg(reinterpret_cast<float2*>(mine + r0 * 64 + 8 * cb + cq), make_float2(Ls[4 * cb] * f, Ls[4 * cb + 1] * f));
        __stcg(reinterpret_cast<float2*>(mine + r1 * 64 + 8 * cb + cq),
               make_float2(Ls[4 * cb + 2] * f, Ls[4 * cb + 3] * f));
      }
      if ((lane & 3) == 0) {
        mine[4096 + r0] = a2r0;
        mine[4096 + r1] = a2r1;
      }
      if (wtid == 0) mine[4096 + 64] = ms->sc_sin;
      __threadfence();
      wg_sync(wg);
      if (wtid == 0) mbar_arrive(&ms->agg_pub);
      if (partial)
        second_phase<Tin, Tout, kDK, kBlock>(fp, ms, hdr, smem, tmem, wg, wtid, lane, seq, b, h, sp, slot, nonfinite);
    }
  } else if (warp < 16) {
    // ===================================================================== WG_C: epilogue, scan
    const int wg = 3, wtid = tid - 3 * kWG, wq = warp & 3;
    const int trow = wq * 16 + (lane & 15);
    const int tsel = lane >> 4;  // lane tile: chunk 2m (0) or 2m+1 (1) of an output pair
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    uint8_t* wstage = smem + kOffStg + wq * 32 * 128;  // this warp's output staging tile
    int slot = 0;
    // the output gate's norm weight (read by this warpgroup's epilogues, and by the others'
    // after barriers that follow this warpgroup's)
    if (gated && wtid < 64) ms->nw[wtid] = __ldg(p.onorm_w + wtid);
    if (segm && wtid == 0) {  // failure injection marks of the workspace (zero: off), read by this warpgroup
      ms->dbg_skip = *(volatile unsigned int*)&hdr->dbg_skip_seg;
      ms->dbg_us = *(volatile unsigned int*)&hdr->dbg_wait_us;
    }
    // the CTA's input scale (WG_A0 derives it from the first chunk; the outputs go back to
    // the inputs' scale); the wait's barrier also publishes the marks above
    bool alive = wg_wait<kOL>(wg, wtid, &ms->scale_ready, 0u, ms, hdr, 0x506, slot);
    if (clus) {
      // the outputs stay in tensor memory until the start state is known: wait for their
      // last MMAs; then (segments s > 0) the chunks' Qh' tiles start loading into the idle
      // staging buffers
      for (int pr = 0; pr < (cnt + 1) / 2 && alive; ++pr)
        alive = wg_wait<kOL>(wg, wtid, &ms->o_full[pr], 0u, ms, hdr, 0x520, slot);
      if (alive && qhw && wg_wait<kOL>(wg, wtid, &ms->agg_pub, 0u, ms, hdr, 0x521, slot) && wtid == 0) {
        mbar_arrive_expect_tx(&ms->p2_full[0], (uint32_t)(cnt * kTile));
        for (int g = 0; g < cnt; g += 2) {
          const int nb = min(2, cnt - g);
          bulk_load(smem + kOffStage + g * kTile, fp.qhp + ((size_t)seq * fp.Nc + sp.c0 + g) * 4096,
                    (uint32_t)(nb * kTile), &ms->p2_full[0]);
        }
      }
    } else {
      // this CTA's chunks; in a segment s > 0 the outputs are partial: fp16 rows of the
      // workspace, completed in the second phase
      const int pairs = alive ? (cnt + 1) / 2 : 0;
      const float osc = ms->sc_out;
      for (int pr = 0; pr < pairs; ++pr) {
        if (!wg_wait<kOL>(wg, wtid, &ms->o_full[pr % kOPairs], ph_use<kOPairs>(pr), ms, hdr, 0x500, slot)) { alive = false; break; }
        tc_fence_after();
        const int ci = 2 * pr + tsel;
        long long s = 0;
        const bool valid = ci < cnt && chunk_scan_pos(fp, sp.c0 + ci, kRev ? 63 - trow : trow, L, s);
        const uint32_t src = tl + kColO + 64u * (uint32_t)(pr % kOPairs);
        if (partial) {
          uint8_t* od = valid ? reinterpret_cast<uint8_t*>(fp.olc + ((size_t)seq * fp.Nc + sp.c0 + ci) * 4096) + trow * 128
                              : nullptr;
          epilogue_rows<__half>(src, od, wstage, lane, nonfinite, 1.f);  // (kept in this CTA's scale)
        } else if (gated) {
          gated_rows<Tout, Tin>(src, nullptr, out_row<Tout>(fp, b, h, valid, s), gate_row<Tin>(fp, b, h, valid, s),
                                ms->nw, fp.p.oeps, wstage, lane, nonfinite, osc);
        } else {
          epilogue_rows<Tout>(src, out_row<Tout>(fp, b, h, valid, s), wstage, lane, nonfinite, osc);
        }
        tc_fence_before();
        wg_sync(wg);
        if (wtid == 0) mbar_arrive(&ms->o_free[pr % kOPairs]);
      }
      // the O_local rows written above are read back by bulk copy (async proxy)
      if (partial) asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    if (segm && alive) {
      // Scan of the segment summaries.  This CTA owns state entries [4 f0, 4 f1) (float4
      // units f, F of them).  Threads split into nB blocks of bs consecutive segments x FP
      // float4 columns (nB * FP <= 128): a thread loads its block's summaries for its f
      // all at once (consecutive threads read consecutive float4s), composes them
      // sequentially, and the block compositions are exchanged through shared memory;
      // each thread then walks its segments again from its block's carry-in, writing
      // each segment's start state (fp16, MMA layout, in that segment's CTA scale).
      const int ns = fp.n_s;
      const int f0 = (int)((long long)seg * 1024 / ns), f1 = (int)((long long)(seg + 1) * 1024 / ns);
      const int F = f1 - f0;
      int nB = kWG / (F > 0 ? F : 1);
      nB = nB < 1 ? 1 : (nB > ns ? ns : nB);
      if ((ns + nB - 1) / nB > kScanBlock) nB = (ns + kScanBlock - 1) / kScanBlock;
      const int bs = (ns + nB - 1) / nB;
      const int FP = kWG / nB;
      const int bi = wtid / FP, fi = wtid % FP;
      const int s_lo = bi * bs, s_hi = min(ns, s_lo + bs);
      unsigned int* ctr = fp.counters + (size_t)seq * 2;
      const float* aggs = fp.agg + (size_t)seq * ns * kAggStride;
      uint16_t* sst = fp.sstart + (size_t)seq * ns * 4096;
      float* xD = reinterpret_cast<float*>(smem + kOffSst);              // [128] block decays
      float4* xU = reinterpret_cast<float4*>(smem + kOffSst + 4 * kWG);  // [128] block summaries
      float* segfac = reinterpret_cast<float*>(smem + kOffSst + 4096);   // [ns] start-state factors
      // a CTA whose inputs were scaled says so in the high half of its arrival; only then
      // are the segments' start-state factors fetched
      const unsigned int arrival = 1u + (ms->sc_sin != 1.f ? 0x10000u : 0u);
      unsigned int scaled = 0;
      const unsigned int target = (unsigned int)ns;
      // failure injection: a segment withholds its arrival, and the waits give up early
      const unsigned int dbg_us = ms->dbg_us;
      const uint64_t limit = dbg_us ? 1000ull * dbg_us : 1000000000ull;
      const int loads = partial ? min(4, (cnt + 1) / 2) : 0;
      bool ok0 = wg_wait<kOL>(wg, wtid, &ms->agg_pub, 0u, ms, hdr, 0x600, slot);
      int issued = 0;
      if (ok0) {
        if (wtid == 0) {
          // the second phase's first four pairs start loading now (every MMA of this
          // CTA has completed, so all staging buffers are free; the Qh' and O_local
          // tiles are written and fenced)
          for (int q = 0; q < loads; ++q) p2_load(fp, ms, smem, seq, sp, q, q);
          issued = loads;
          if (ms->dbg_skip != (unsigned int)seg + 1u) red_release_add(ctr, arrival);
          ok0 = wait_counter(ctr, target, ms, hdr, 0x601, limit, &scaled);
          ms->go[wg][2] = (int)scaled;
        }
        ok0 = wg_agree(wg, wtid, ok0, ms, slot);
      }
      if (ok0) {
        scaled = (unsigned int)*(volatile int*)&ms->go[wg][2];
        if (scaled) {
          for (int sg = wtid; sg < ns; sg += kWG) segfac[sg] = __ldcg(aggs + (size_t)sg * kAggStride + 4096 + 64);
          wg_sync(wg);
        }
        for (int base = f0; base < f1; base += FP) {
          const int f = base + fi;
          const bool act = bi < nB && f < f1;
          const int kk = f >> 4;
          float4 u[kScanBlock];
          float dd[kScanBlock];
          float4 X = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int j = 0; j < kScanBlock; ++j) {
            const int sg = s_lo + j;
            const bool on = act && sg < s_hi;
            const float* a2p = aggs + (size_t)(on ? sg : 0) * kAggStride;
            u[j] = on ? __ldcg(reinterpret_cast<const float4*>(a2p) + f) : make_float4(0.f, 0.f, 0.f, 0.f);
            dd[j] = on ? __ldcg(a2p + 4096 + kk) : 0.f;
          }
          // this block's transfer: state_after = D * state_before + U
          float D = 1.f;
          float4 U = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int j = 0; j < kScanBlock; ++j) {
            dd[j] = ex2(dd[j]);  // inactive entries: 2^0 = 1 with a zero summary
            U = make_float4(fmaf(dd[j], U.x, u[j].x), fmaf(dd[j], U.y, u[j].y), fmaf(dd[j], U.z, u[j].z),
                            fmaf(dd[j], U.w, u[j].w));
            D *= dd[j];
          }
          if (nB > 1) {
            if (bi < nB) {
              xD[bi * FP + fi] = D;
              xU[bi * FP + fi] = U;
            }
            wg_sync(wg);
            for (int b2 = 0; b2 < bi && b2 < nB; ++b2) {
              const float d2 = xD[b2 * FP + fi];
              const float4 u2 = xU[b2 * FP + fi];
              X = make_float4(fmaf(d2, X.x, u2.x), fmaf(d2, X.y, u2.y), fmaf(d2, X.z, u2.z), fmaf(d2, X.w, u2.w));
            }
          }
          if (act) {
            const int v0 = 4 * (f & 15);
            const uint32_t so = (uint32_t)kk * 128u + ((((uint32_t)v0 >> 3) ^ ((uint32_t)kk & 7u)) << 4) + (v0 & 7) * 2;
#pragma unroll
            for (int j = 0; j < kScanBlock; ++j) {
              const int sg = s_lo + j;
              if (sg < s_hi) {  // segment sg's start state: fp16 in its CTA's scale, MMA layout
                const float fs = scaled ? segfac[sg] : 1.f;
                __stcg(reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(sst + (size_t)sg * 4096) + so),
                       make_uint2(pack_h2(X.x * fs, X.y * fs), pack_h2(X.z * fs, X.w * fs)));
                X = make_float4(fmaf(dd[j], X.x, u[j].x), fmaf(dd[j], X.y, u[j].y), fmaf(dd[j], X.z, u[j].z),
                                fmaf(dd[j], X.w, u[j].w));
              }
            }
          }
          if (nB > 1) wg_sync(wg);  // the exchange slots are reused by the next column pass
        }
        __threadfence();
        wg_sync(wg);
        if (wtid == 0) {
          red_release_add(ctr + 1, 1u);
          ok0 = wait_counter(ctr + 1, target, ms, hdr, 0x602, limit);
        }
        ok0 = wg_agree(wg, wtid, ok0, ms, slot);
      }
      if (ok0 && partial) {
        // this segment's start state (already in this CTA's scale and the MMA layout) ->
        // shared memory, then the second phase on all four warpgroups
        const uint4* src = reinterpret_cast<const uint4*>(sst + (size_t)seg * 4096);
        uint4* dst = reinterpret_cast<uint4*>(smem + kOffSst);
        for (int i = wtid; i < 512; i += kWG) dst[i] = __ldcg(src + i);
        fence_proxy_async_smem();
        wg_sync(wg);
        if (wtid == 0) mbar_arrive(&ms->p2_go);
        second_phase<Tin, Tout, kDK, kBlock>(fp, ms, hdr, smem, tmem, wg, wtid, lane, seq, b, h, sp, slot, nonfinite);
      } else if (wtid == 0) {
        // giving up: this CTA's own bulk copies land before it leaves (they read the
        // workspace only, so they complete on their own; the wait is bounded all the same)
        for (int q = 0; q < issued; ++q)
          for (int it = 0; it < 1000 && !mbar_wait_sleep(&ms->p2_full[q], 0u, 1000000u); ++it) {
          }
      }
    }
  }

  if (clus) {
    // ===================================================================== CLUSTER combine
    // The n_s CTAs of a sequence form one cluster.  Every thread of every CTA meets at the
    // cluster barrier (all waits before it are bounded): the summaries are delivered and
    // every MMA of the cluster has completed.  CTA rank r then composes its units over the
    // n_s segments from its receive area and writes each segment's start state (fp16, MMA
    // layout) into that segment's CTA; after a second barrier every CTA holds its own.
    if (!cwaited) cluster_wait();
    __syncwarp();
    cluster_sync_all();
    if (tid < 4 * kWG) {
      const int ns = fp.n_s;
      const int u0 = seg * 2048 / ns, u1 = (seg + 1) * 2048 / ns;
      for (int u = u0 + tid; u < u1; u += 4 * kWG) {  // (more than one unit a thread below 4 CTAs)
        const int kk = u >> 5, v0 = 2 * (u & 31);  // key channel, value pair
        const uint32_t a_u = smem_u32(smem + kOffStg) + (uint32_t)(kk * 64 + v0) * 4u;
        const uint32_t a_d = smem_u32(&ms->dseg[kk]);
        const uint32_t a_f = smem_u32(&ms->sc_sin);
        const uint32_t a_s = smem_u32(smem + kOffSst) + (uint32_t)kk * 128u +
                             ((((uint32_t)v0 >> 3) ^ ((uint32_t)kk & 7u)) << 4) + (uint32_t)(v0 & 7) * 2u;
        // every segment's summary entries first (the remote loads overlap), then the
        // sequential composition
        float2 uj[kMaxCluster];
        float dj[kMaxCluster], fj[kMaxCluster];  // fj: a start state into CTA j's scale
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j) {
          if (j < ns) {
            uj[j] = ld_cluster_f32x2(cluster_map(a_u, (uint32_t)j));
            dj[j] = ld_cluster_f32(cluster_map(a_d, (uint32_t)j));
            fj[j] = ld_cluster_f32(cluster_map(a_f, (uint32_t)j));
          }
        }
        float2 X = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < kMaxCluster; ++j) {
          if (j < ns) {
            st_cluster_u32(cluster_map(a_s, (uint32_t)j), pack_h2(X.x * fj[j], X.y * fj[j]));
            const float d = ex2(dj[j]);
            X = make_float2(fmaf(d, X.x, uj[j].x), fmaf(d, X.y, uj[j].y));
          }
        }
      }
    }
    if (inplace && seg > 0 && tid < 4 * kWG) {
      // Qh' = Qh 2^(decay from the segment start) in place: per chunk and channel the factor
      // sums row 0 (the decay a) of the earlier chunks' gate tiles, then every 16-byte piece
      // of the tiles is scaled
      float* fac = &ms->red[0][0][0][0];  // [cnt][64] (the cumsum exchange is idle now)
      if (tid < cnt * 64) {
        const int g = tid >> 6, ch = tid & 63;
        float a2 = 0.f;
        for (int j = 0; j < g; ++j)
          a2 += reinterpret_cast<const float*>(smem + kOffStage + j * kStageBytes + 3 * kTile)[ch];
        fac[tid] = ex2(a2);
      }
      asm volatile("bar.sync 7, 512;" ::: "memory");
      for (int i = tid; i < cnt * 512; i += 4 * kWG) {
        const int g = i >> 9, pi = i & 511, r = pi >> 3, jp = pi & 7, jl = jp ^ (r & 7);
        uint4* ptr = reinterpret_cast<uint4*>(smem + kOffStage + g * kStageBytes + r * 128 + 16 * jp);
        const float4 f0 = *reinterpret_cast<const float4*>(fac + g * 64 + 8 * jl);
        const float4 f1 = *reinterpret_cast<const float4*>(fac + g * 64 + 8 * jl + 4);
        uint4 v = *ptr;
        v.x = h2_bits(__hmul2(bits_h2(v.x), __floats2half2_rn(f0.x, f0.y)));
        v.y = h2_bits(__hmul2(bits_h2(v.y), __floats2half2_rn(f0.z, f0.w)));
        v.z = h2_bits(__hmul2(bits_h2(v.z), __floats2half2_rn(f1.x, f1.y)));
        v.w = h2_bits(__hmul2(bits_h2(v.w), __floats2half2_rn(f1.z, f1.w)));
        *ptr = v;
      }
    }
    // the start states and the in-place Qh' are read by the MMA (async proxy)
    asm volatile("fence.proxy.async;" ::: "memory");
    __syncwarp();
    cluster_sync_all();
    if (tid < 4 * kWG) {
      // outputs += Qh' S_start (segments s > 0; issued by one thread, one commit per pair),
      // then the epilogue of the held pairs: warpgroup q (warps 4q .. 4q+3) takes pair q
      const int q = warp >> 2, wtid = tid - kWG * q, wq = warp & 3;
      const int trow = wq * 16 + (lane & 15), tsel = lane >> 4;
      const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
      // staging: warpgroup 3 over the summary area (read out), the others past the Qh' tiles
      // (in place: over the K and V tiles of stages 0-2)
      uint8_t* wstage = (q == 3 ? smem + kOffStg
                                : (inplace ? smem + kOffStage + q * kStageBytes + kTile
                                           : smem + kOffStage + kClusterChunks * kTile + q * 4 * 32 * 128)) +
                        wq * 32 * 128;
      const int npairs = (cnt + 1) / 2;
      int slot = 0;
      if (seg > 0 && q == 3 && wtid == 0 && (inplace || wait_bar<kOL>(&ms->p2_full[0], 0u, ms, hdr, 0x530))) {
        const uint32_t id_qs = idesc_f16(0, 64, 64, 0, 1);
        const uint32_t s_base = smem_u32(smem);
        tc_fence_after();
        for (int g = 0; g < cnt; ++g) {
          const uint32_t d_o = tmem + kColO + 64u * (uint32_t)(g >> 1) + ((g & 1) ? kLaneTile1 : 0u);
          const uint32_t a_q = s_base + kOffStage + g * (inplace ? kStageBytes : kTile);  // the chunk's Qh'
          for (int k = 0; k < kDK / 16; ++k)
            mma_f16(d_o, sw128_desc(a_q + 32 * k), sw128_desc(s_base + kOffSst + 2048 * k), id_qs, 1);
          if ((g & 1) || g + 1 == cnt) mma_commit(&ms->corr_done[g >> 1]);
        }
      }
      for (int pr = q; pr < npairs; pr += 4) {
        if (seg > 0 && !wg_wait<kOL>(q, wtid, &ms->corr_done[pr], 0u, ms, hdr, 0x531, slot)) break;
        tc_fence_after();
        const int ci = 2 * pr + tsel;
        long long s = 0;
        const bool valid = ci < cnt && chunk_scan_pos(fp, sp.c0 + ci, kRev ? 63 - trow : trow, L, s);
        if (gated)
          gated_rows<Tout, Tin>(tl + kColO + 64u * (uint32_t)pr, nullptr, out_row<Tout>(fp, b, h, valid, s),
                                gate_row<Tin>(fp, b, h, valid, s), ms->nw, fp.p.oeps, wstage, lane, nonfinite,
                                ms->sc_out);
        else
          epilogue_rows<Tout>(tl + kColO + 64u * (uint32_t)pr, out_row<Tout>(fp, b, h, valid, s), wstage, lane,
                              nonfinite, ms->sc_out);
      }
    }
  }

  if (__any_sync(0xffffffffu, nonfinite != nonfinite) && lane == 0) record_error(hdr, GTR_ERR_RANGE, 0x500u + warp);

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
  // last CTA out resets this call's counters: the workspace is ready for the next call
  if (segm && tid == 0) {
    __threadfence();
    const unsigned int done = atomicAdd(&hdr->ticket, 1u);
    if (done == (unsigned int)fp.grid - 1) {
      for (int i = 0; i < 2 * fp.n_seq; ++i) fp.counters[i] = 0u;
      __threadfence();
      hdr->ticket = 0u;
    }
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// Tensor map over a [B][H][W][nh][d] tensor (row-major grid cells m = y*W + x) whose box
// is 64 consecutive scan positions of one (batch, head): the row view [B][L][nh][d] with a
// box of 64 cells m, or the column view with a box of 64 rows y of one column x.  nh is the
// heads dimension (1 for a per-token tensor), d the channels (d * esize a multiple of 16).
// rowline: the row-line view [B][H][W][nh][d] with a box of 64 consecutive x of one row y
// (line chunks of the row directions: cells past the row's ends read as zeros).
bool make_chunk_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, const Problem& p,
                    bool column, bool swizzle, int d, int nh, bool rowline = false) {
  auto enc = get_encode();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15u)) return false;
  const cuuint64_t e = (cuuint64_t)esize, hd = (cuuint64_t)nh, dd = (cuuint64_t)d;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapSwizzle sw = swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r;
  if (rowline) {
    cuuint64_t dims[5] = {dd, hd, (cuuint64_t)p.W, (cuuint64_t)p.H, (cuuint64_t)p.B};
    cuuint64_t strides[4] = {dd * e, hd * dd * e, (cuuint64_t)p.W * hd * dd * e,
                             (cuuint64_t)p.H * p.W * hd * dd * e};
    cuuint32_t box[5] = {(cuuint32_t)d, 1, 64, 1, 1};
    r = enc(m, dt, 5, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else if (!column) {
    cuuint64_t dims[4] = {dd, hd, (cuuint64_t)p.L(), (cuuint64_t)p.B};
    cuuint64_t strides[3] = {dd * e, hd * dd * e, (cuuint64_t)p.L() * hd * dd * e};
    cuuint32_t box[4] = {(cuuint32_t)d, 1, 64, 1};
    r = enc(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    cuuint64_t dims[5] = {dd, hd, (cuuint64_t)p.W, (cuuint64_t)p.H, (cuuint64_t)p.B};
    cuuint64_t strides[4] = {dd * e, hd * dd * e, (cuuint64_t)p.W * hd * dd * e,
                             (cuuint64_t)p.H * p.W * hd * dd * e};
    cuuint32_t box[5] = {(cuuint32_t)d, 1, 1, 64, 1};
    r = enc(m, dt, 5, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS;
}

// Tensor map over a [rows][d] view (one token-head a row) whose box is one row: the source
// of 4-row TMA gathers.
bool make_row_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, long long rows,
                  bool swizzle, int d) {
  auto enc = get_encode();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 15u) || rows >= (1ll << 31)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * esize};
  cuuint32_t box[2] = {(cuuint32_t)d, 1};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct Plan {
  int mode, n_seq, n_s, grid;
};

// Line chunks for directions whose 64 consecutive scan positions are not one box (right-
// to-left rows, or columns, not a multiple of 64 long): one grid line a chunk, zero-padded
// past the line end, each one TMA box per tensor, instead of contiguous chunks staged by 64
// single-row gathers.  Taken for lines of 39 to 63 cells (the padding keeps at least 60%
// of the staged rows) and at most 64 lines, where a sequence's few chunks leave the
// gathers' issue time on the critical path (a 40 x 40 grid: 40 line chunks beat 25
// gathered ones).  More chunks were measured slower than the gathers, which then overlap
// with the work of the chunks before them (the 48-cell columns of a 48 x 80 grid: 80
// chunks instead of 60; its 80-cell rows, two chunks a line: 96).  Not with the low-rank
// gate producer: a zero z row would not give a gate of 1.
bool use_lines(const Problem& p) {
  if (p.gz != nullptr || p.direction == GTR_L2R) return false;
  const bool column = p.direction >= GTR_T2B;
  const int len = column ? p.H : p.W, lines = column ? p.W : p.H;
  return len >= 39 && len < 64 && lines <= 64;
}
// Chunks of one sequence on the fused path, for the problem's direction.
int fused_chunks(const Problem& p) {
  if (!use_lines(p)) return p.n_chunks();
  return p.direction >= GTR_T2B ? p.W : p.H;
}
// The most chunks of one sequence over the four directions (the workspace query takes no
// direction).
int max_fused_chunks(const Problem& p) {
  int m = p.n_chunks();
  for (int d = GTR_L2R; d <= GTR_B2T; ++d) {
    Problem q = p;
    q.direction = d;
    q.gz = nullptr;
    const int c = fused_chunks(q);
    if (c > m) m = c;
  }
  return m;
}

// Length-aware plan: many sequences -> one CTA each (STREAM); few sequences -> each is
// split into n_s segments, one CTA each, so that the launch fills the SMs (SEGMENTED).
Plan make_plan(const Problem& p, int Nc, int sms) {
  Plan pl;
  pl.n_seq = p.B * p.heads;
  const int cap = sms < (int)kMaxSegCtas ? sms : (int)kMaxSegCtas;
  if (pl.n_seq * 2 > cap || Nc <= 1) {
    pl.mode = 0;
    pl.n_s = 1;
    pl.grid = pl.n_seq;
  } else {
    pl.mode = 1;
    pl.n_s = cap / pl.n_seq;
    if (pl.n_s > Nc) pl.n_s = Nc;
    // the longest segment sets the time: with k = ceil(Nc / n_s) chunks in it, take the
    // fewest segments that still hold at most k each (less contention, a shorter scan).
    // Runs of one or two chunks keep every CTA: most segments are then a single chunk.
    const int k = (Nc + pl.n_s - 1) / pl.n_s;
    if (k >= 3) pl.n_s = (Nc + k - 1) / k;
    pl.grid = pl.n_seq * pl.n_s;
  }
  return pl;
}

int device_sms() {
  static int sms[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!sms[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    sms[dev] = v > 0 ? v : 148;
  }
  return sms[dev];
}

// Segment summaries and start states the workspace holds room for (0: STREAM only).
size_t seg_capacity(const Problem& p) {
  const size_t n_seq = (size_t)p.B * p.heads;
  return n_seq * 2 <= kMaxSegCtas ? n_seq * (kMaxSegCtas / n_seq) : 0;
}

// Clusters of `cs` CTAs of this kernel the device can hold at once (cached per device,
// kernel kind and size).
template <typename K>
int max_active_clusters(K kern, int dev, int kind, int cs) {
  static int cache[64][4][kMaxCluster + 1];
  static std::once_flag once;
  static std::mutex mu;
  std::call_once(once, [] {
    for (auto& a : cache)
      for (auto& b : a)
        for (int& c : b) c = -1;
  });
  std::lock_guard<std::mutex> lock(mu);
  int& c = cache[dev][kind][cs];
  if (c < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    c = cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess ? n : 0;
    (void)cudaGetLastError();  // a refused size only means no cluster mode
  }
  return c;
}

template <typename Tin, typename Tout, int kMode, int kDK, bool kBlock = false>
void (*pick_kernel(bool rev, bool box))(FusedParams) {
  return rev ? (box ? fused_gla_kernel<Tin, Tout, true, true, kMode, kDK, kBlock>
                    : fused_gla_kernel<Tin, Tout, true, false, kMode, kDK, kBlock>)
             : (box ? fused_gla_kernel<Tin, Tout, false, true, kMode, kDK, kBlock>
                    : fused_gla_kernel<Tin, Tout, false, false, kMode, kDK, kBlock>);
}

template <typename Tin, typename Tout, int kDK>
gtr_status_t launch_fused_typed(const Problem& p, void* ws, cudaStream_t stream, int force_mode) {
  const bool rev = p.direction == GTR_R2L || p.direction == GTR_B2T;
  FusedParams fp;
  fp.p = p;
  // chunks are staged in reverse scan order for the reversed directions; a chunk is one
  // TMA box per tensor when its 64 scan positions are consecutive cells of one row view
  // (left-to-right always; right-to-left when rows hold whole chunks) or of one column
  // (top-to-bottom / bottom-to-top when columns hold whole chunks)
  fp.rev = (p.direction == GTR_R2L || p.direction == GTR_B2T) ? 1 : 0;
  const bool column = p.direction >= GTR_T2B;
  const bool lines = use_lines(p);
  fp.lines = lines ? 1 : 0;
  fp.len = column ? p.H : p.W;
  const bool one_box = lines || p.direction == GTR_L2R || (p.direction == GTR_R2L && p.W % 64 == 0) ||
                       (column && p.H % 64 == 0);
  const bool rowline = lines && !column;  // (line chunks of the column directions use the column view)
  const CUtensorMapDataType dt16 =
      std::is_same<Tin, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // optional pieces of the GTR block: the low-rank gate producer (z tiles instead of the
  // log-gates) and the RMSNorm + SiLU output gate
  fp.lowrank = p.gz != nullptr ? 1 : 0;
  fp.gtau_inv = fp.lowrank ? 1.f / p.gtau : 1.f;
  fp.gated = p.ogate != nullptr ? 1 : 0;
  // q, k: 128-byte swizzle (d_k = 64; built in place), or dense rows (d_k = 32)
  const bool swqk = kDK == 64;
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  fp.tma = one_box && make_chunk_map(&fp.tq, p.q, dt16, 2, p, column, swqk, kDK, p.heads, rowline) &&
                   make_chunk_map(&fp.tk, p.k, dt16, 2, p, column, swqk, kDK, p.heads, rowline) &&
                   make_chunk_map(&fp.tv, p.v, dt16, 2, p, column, true, 64, p.heads, rowline) &&
                   (fp.lowrank ? make_chunk_map(&fp.tz, p.gz, f32, 4, p, column, false, p.grank, 1)
                               : make_chunk_map(&fp.tg, p.log_gamma, f32, 4, p, column, false, kDK, p.heads, rowline))
               ? 1
               : 0;
  if (!fp.tma) fp.lines = 0;  // (no box view: contiguous chunks by gathers)
  const int Nc = fp.lines ? fused_chunks(p) : p.n_chunks();
  fp.divW = make_fastdiv((uint32_t)p.W);
  fp.divH = make_fastdiv((uint32_t)p.H);
  if (!fp.tma) {  // other chunks: 4-row gathers from [B*L*heads][d] row views
    const long long rows = (long long)p.B * p.L() * p.heads;
    fp.tma = make_row_map(&fp.tq, p.q, dt16, 2, rows, swqk, kDK) && make_row_map(&fp.tk, p.k, dt16, 2, rows, swqk, kDK) &&
                     make_row_map(&fp.tv, p.v, dt16, 2, rows, true, 64) &&
                     (fp.lowrank ? make_row_map(&fp.tz, p.gz, f32, 4, (long long)p.B * p.L(), false, p.grank)
                                 : make_row_map(&fp.tg, p.log_gamma, f32, 4, rows, false, kDK))
                 ? 2
                 : 0;
  }

  // one kernel per direction kind, producer and mode: each carries only the code its
  // plan runs (the one-box producer's kernels none of the row-table code)
  const bool box = fp.tma == 1;
  const int kind = (rev ? 2 : 0) + (box ? 1 : 0);
  using Kern = void (*)(FusedParams);
  // with the optional block pieces: one kernel that reads the plan mode at run time
  const bool blk = fp.lowrank || fp.gated;
  const Kern kb = pick_kernel<Tin, Tout, -1, kDK, true>(rev, box);
  const Kern kerns[3] = {blk ? kb : pick_kernel<Tin, Tout, 0, kDK>(rev, box),
                         blk ? kb : pick_kernel<Tin, Tout, 1, kDK>(rev, box),
                         blk ? kb : pick_kernel<Tin, Tout, 2, kDK>(rev, box)};
  static std::atomic<unsigned long long> configured[8];
  const int ckind = kind + (blk ? 4 : 0);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GTR_ERR_CUDA;
  if (!(configured[ckind].load() & (1ull << dev))) {
    for (Kern k : kerns)
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess ||
          cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
        return GTR_ERR_CUDA;
    configured[ckind].fetch_or(1ull << dev);
  }
  Plan pl = make_plan(p, Nc, device_sms());
  if (pl.mode == 1 && force_mode < 0) {
    // short sequences: one cluster per sequence (the largest size the device holds for
    // every sequence at once), at most kClusterChunks chunks per CTA; then the fewest
    // CTAs that keep the longest run
    int best_k = kClusterChunks + 1;
    for (int cs = kMaxCluster; cs >= 2; --cs) {
      if (max_active_clusters(kerns[2], dev, kind, cs) < pl.n_seq) continue;
      const int k = (Nc + cs - 1) / cs;
      if (k < best_k) best_k = k;
    }
    if (best_k <= kClusterChunks) {
      const int cs = (Nc + best_k - 1) / best_k;
      if (cs >= 2 && max_active_clusters(kerns[2], dev, kind, cs) >= pl.n_seq) {
        pl.mode = 2;
        pl.n_s = cs;
        pl.grid = pl.n_seq * cs;
      }
    }
  }
  if (force_mode == 0) {
    pl.mode = 0;
    pl.n_s = 1;
    pl.grid = pl.n_seq;
  }
  const FusedWorkspace w = fused_workspace_carve(ws, p);
  fp.hdr = w.hdr;
  fp.counters = w.counters;
  fp.agg = w.agg;
  fp.sstart = w.sstart;
  fp.qhp = w.qhp;
  fp.olc = w.olc;
  fp.n_seq = pl.n_seq;
  fp.n_s = pl.n_s;
  fp.Nc = Nc;
  fp.mode = pl.mode;
  fp.grid = pl.grid;
  // the score factor 2^-A of a chunk stays below 2^11.5 (about e^8): Kh and the
  // fp16 rounding of the small Qh values keep their precision
  fp.max_exp2 = 11.5f;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pl.mode == 2) {  // one cluster per sequence
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = pl.n_s;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pl.mode == 1) {  // the CTAs of a sequence wait on one another (measured faster than
    // a normal launch with programmatic dependent launch: 2048^2 58.5 against 62.9 us)
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na].val.cooperative = 1;
    ++na;
  } else {  // the prologue may overlap the previous launch's tail
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  if (cudaLaunchKernelEx(&cfg, kerns[pl.mode], fp) != cudaSuccess) return GTR_ERR_CUDA;
  return GTR_OK;
}


}  // namespace
}  // namespace gtr
