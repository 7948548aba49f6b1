// Internal declarations shared by the kernels and the host orchestrator of the
// B200 DeepSeekMoE layer library. Not part of the public ABI (include/ktmoe.h).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "ktmoe.h"

namespace ktmoe {

// ---------------------------------------------------------------------------
// Tiling constants
// ---------------------------------------------------------------------------
constexpr int kPermChunk = 32;      // tokens per gate-select / scatter CTA
constexpr int kChunkRowsF8 = 224;  // MXFP8 layers: two 224-column accumulators + scales in TMEM
constexpr int kChunkRows = 256;     // token rows per GEMM chunk (MMA N <= 256)
// Schedule tuning (compile-time; -D overrides are for tuning sweeps).
#ifndef KT_TILE_BLOCK
#define KT_TILE_BLOCK 8
#endif
#ifndef KT_HEAVY_ROWS
#define KT_HEAVY_ROWS 192
#endif
#ifndef KT_L2_HINTS
#define KT_L2_HINTS 2
#endif
constexpr int kTileBlock = KT_TILE_BLOCK;   // chunks per schedule block (feature-tile-major inside)
constexpr int kHeavyRows = KT_HEAVY_ROWS;   // experts with at least this many rows are compute-bound
constexpr int kMaxExperts = 512;
constexpr int kMaxGroups = 32;
constexpr int kMaxTopk = 32;
constexpr int kMaxShared = 8;
constexpr int kSmallTokens = 64;    // up to this many tokens the gate logits are split over K
constexpr int kGateSplitK = 16;     // ... into this many partial sums

// Words at the start of the workspace that every call zeroes first: [0] the
// device error word, [1] its detail, [kGateDoneWord, +16) the split-K logits'
// per-expert-block completion counters.
constexpr int kGateDoneWord = 8;
constexpr int kCallWords = kGateDoneWord + kMaxExperts / 32;

// Device error word codes (workspace offset 0). The second int holds a detail.
constexpr int kDevErrTimeout = 1;
constexpr int kDevErrBounds = 2;   // checked build only: an index check failed

// ---------------------------------------------------------------------------
// Config with every automatic choice resolved
// ---------------------------------------------------------------------------
struct Resolved {
  int E, G, TG, k, S, d, I, gs;
  float route_scale;
  int score_func;   // KT_SCORE_*
  int norm;         // 0/1
  int group_score;  // KT_GROUP_AMAX / KT_GROUP_TOP2SUM (G == 1: unused)
  int dtype;        // KT_DTYPE_*
  int act_bf16;     // tokens, gate weights and output in bf16 (KT_DTYPE_BF16 / MXFP8)
  int fp8;          // block-scaled expert weights (MXFP8 or MXFP4): tokens and hidden rows in MXFP8
  int w4;           // expert weights in MXFP4 (E2M1 codes, two per byte)
  int chunk_rows;   // token rows per GEMM chunk: kChunkRows, or kChunkRowsF8 for MXFP8
  int n_local;      // routed experts computed here (all: E); their weights are the first
                    // n_local slots of w1/w3/w2 (placed by a SlotTable), the shared ones follow
  int sb, se;       // tokens the shared experts run on here: [sb, se) (all: [0, T))
  int num_sms;      // SMs of the device (set by the forward before its launches)
  int add_residual;
  int y_fp32;       // y in fp32 (else in dtype)
  int has_bias;
};

// One token chunk of one expert group, as scheduled on the grouped GEMMs.
// Rows live in the "hidden-row" space: routed rows 0..T*k-1 sorted by expert,
// then shared expert s at T*k + s*T + t.
struct Chunk {
  int32_t group;    // weight slot: 0..ee-eb-1 routed expert eb + slot, then the shared ones
  int32_t row0;     // first hidden row of the chunk
  int32_t nrows;    // rows in the chunk (<= chunk size)
  int32_t src_row0; // first activation row: permuted-x row (routed) or token (shared)
};

// Weight slots of a launch: the routed experts computed here, then the shared ones.
inline int routed_slots(const Resolved& r) { return r.n_local; }
inline int weight_slots(const Resolved& r) { return r.n_local + r.S; }

// Routed expert -> weight slot of this launch, -1 for an expert computed
// elsewhere (passed by value to the permutation kernels). The plain forward
// uses the identity; the expert-parallel forms a range or any placement.
struct SlotTable {
  int16_t slot[kMaxExperts];
};

// Byte offsets of the workspace's internal buffers.
struct Layout {
  size_t err;          // int32[kCallWords], zeroed by every call (256 bytes)
  size_t meta;         // int32[16]: [0] chunks, [1] up tiles, [2] down tiles,
                       // [3] / [4] up / down GEMM tile counters
  size_t logits;       // fp32 [splits][T, E]; the first slot ends as the logits
  size_t idx;          // int32 [T, k] (when the caller gives no output buffer)
  size_t w;            // fp32 [T, k]
  size_t chunk_counts; // int32 [nperm, E]
  size_t chunk_base;   // int32 [nperm, E]
  size_t counts;       // int32 [E+S]
  size_t offsets;      // int32 [E+S+1]
  size_t row_of;       // int32 [T*k]
  size_t tok_of;       // int32 [T*k]
  size_t row_weight;   // fp32 [T*k]
  size_t chunks;       // Chunk [max_chunks]
  size_t tiles_up;     // int2 (chunk, feature tile) [max_chunks * ceil(I/128)]
  size_t tiles_down;   // int2 [max_chunks * ceil(d/256)]
  size_t xperm;        // [T*k, d]: bf16 (bf16 layers) or E4M3 codes (MXFP8 layers)
  size_t hidden;       // [T*(k+S), I]: dtype, or E4M3 codes (MXFP8)
  // MXFP8 layers only (else empty):
  size_t xq;           // E4M3 codes of x [T, d]
  size_t xs;           // their scale bytes [T, d/32] (row-major)
  size_t tok_sf;       // token scales per GEMM chunk and 128-wide K slab: [chunks][d/128][1 KB]
  size_t hid_sf;       // hidden-row scales, same form: [chunks][I/128][1 KB]
  size_t gchunk0;      // int32 [E+S]: index of each group's first GEMM chunk
  size_t expert_out;   // fp32 [T*(k+S), d]
  size_t total;
  int64_t nperm, max_chunks;
};

int resolve(const kt_moe_config* cfg, int64_t T, int has_bias, Resolved* r);
Layout make_layout(const Resolved& r, int64_t T);

// ---------------------------------------------------------------------------
// Kernel launchers (each returns the cudaError_t of its launch)
// ---------------------------------------------------------------------------
// Number of [T, E] slots the logits region holds (1, or kGateSplitK split-K
// partial sums for calls of at most kSmallTokens tokens; after the logits
// kernel the first slot holds the logits in either case).
int gate_logit_splits(const Resolved& r, int64_t T);
cudaError_t launch_gate_logits(const Resolved& r, int64_t T, const void* x, const void* w_gate,
                               float* logits, int* err, int num_sms, cudaStream_t st);
// bf16 logits on the tensor cores (the grouped GEMM with one group); E % 4 == 0.
cudaError_t launch_gate_logits_tc(const Resolved& r, int64_t T, const void* x, const void* w_gate,
                                  float* logits, int* err, int num_sms, cudaStream_t st);
cudaError_t launch_gate_select(const Resolved& r, int64_t T, const float* logits,
                               const float* scores_in, const float* bias, int32_t* idx,
                               float* w, int32_t* chunk_counts, int* err, cudaStream_t st);
// Scores s [T, E] fp32 from the logits region (gate step 1's score function).
cudaError_t launch_gate_scores(const Resolved& r, int64_t T, const float* logits, float* scores,
                               cudaStream_t st);
// Load statistics (balance.cu).
cudaError_t launch_bias_update(const Resolved& r, int64_t T, const int32_t* idx, float* bias,
                               float gamma, int32_t* load_out, cudaStream_t st);
// Token chunks of the balance statistics and the scratch bytes they need.
int balance_chunks(int64_t T, int* tokens_per_chunk);
size_t balance_scratch_bytes(const Resolved& r, int64_t T);
cudaError_t launch_balance_stats(const Resolved& r, int64_t T, const float* scores,
                                 const int32_t* idx, float alpha, float* f, float* P, float* loss,
                                 void* scratch, cudaStream_t st);
cudaError_t launch_permute(const Resolved& r, const SlotTable& tab, int64_t T, const Layout& L,
                           char* ws, const int32_t* idx, const float* w, const void* x,
                           cudaStream_t st);
// up = true: the gate/up GEMM (wa = W1, wb = W3); up = false: the down GEMM
// (wa = W2, wb unused).
cudaError_t launch_experts_bf16(const Resolved& r, int64_t T, const Layout& L, char* ws,
                                const void* x, const void* wa, const void* wb, int num_sms,
                                cudaStream_t st, bool up);
// Host-side setup of the grouped GEMM (shared-memory limits, the tensor-map
// encoder), done before a stream capture so that the capture holds only
// stream work.
cudaError_t prepare_grouped_gemm();
// One bounded wait on a barrier that never completes (limit_ns), recording the
// timeout in the error word like the GEMM kernels' waits.
cudaError_t launch_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t st);
cudaError_t launch_experts_f32(const Resolved& r, int64_t T, const Layout& L, char* ws,
                               const void* x, const void* w1, const void* w3, const void* w2,
                               int num_sms, cudaStream_t st, bool up);
cudaError_t launch_combine(const Resolved& r, int64_t T, const Layout& L, char* ws,
                           const void* x, void* y, cudaStream_t st);
// Expert-parallel forms: this launch's experts summed per token in fp32 (no
// residual), and the finish after the sum over ranks.
cudaError_t launch_combine_partial(const Resolved& r, int64_t T, const Layout& L, char* ws,
                                   float* y_part, cudaStream_t st);
cudaError_t launch_ep_finish(const Resolved& r, int64_t T, const float* y_sum, const void* x,
                             void* y, int num_sms, cudaStream_t st);

// MXFP8 (mxfp8.cu).
cudaError_t launch_mx_quantize(const void* src, int64_t rows, int64_t K, uint8_t* codes,
                               uint8_t* scales, cudaStream_t st);
// MXFP4: packed E2M1 codes [rows, K/2] (element 2i in the low nibble of byte i).
cudaError_t launch_mx4_quantize(const void* src, int64_t rows, int64_t K, uint8_t* codes,
                                uint8_t* scales, cudaStream_t st);
size_t mx_packed_bytes(const Resolved& r, bool down);
cudaError_t launch_mx_pack(const Resolved& r, const void* w1, const void* w3, const void* w2,
                           uint8_t* w1q, uint8_t* w3q, uint8_t* w2q, uint8_t* sf_up,
                           uint8_t* sf_down, cudaStream_t st);
// The grouped GEMMs with MXFP8 weights (up: wa/wb = W1/W3 codes, sf = packed
// gate/up scales; down: wa = W2 codes, sf = packed down scales).
cudaError_t launch_experts_mxfp8(const Resolved& r, int64_t T, const Layout& L, char* ws,
                                 const void* wa, const void* wb, const uint8_t* sf, int num_sms,
                                 cudaStream_t st, bool up);

// MX block scale of a block with absolute maximum amax (>= 0): the smallest e
// with amax <= 448 * 2^e, from the fp32 bits (amax = 1.m * 2^E: e = E - 8 +
// (1.m > 1.75)); zero or subnormal amax gives -127; clamped to [-127, 127].
__device__ __forceinline__ int mx_scale_exp(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ef = (int)((b >> 23) & 0xFF);
  if (ef == 0) return -127;
  const int e = ef - 127 - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}
// 2^-e as an fp32 (e <= 126 for every finite amax).
__device__ __forceinline__ float mx_inv_scale(int e) {
  return e >= 127 ? 0x1p-127f : __uint_as_float((uint32_t)(127 - e) << 23);
}
// E4M3 code of v * inv, round to nearest even (|v * inv| <= 448 by the scale rule).
__device__ __forceinline__ uint8_t mx_code(float v, float inv) {
  return (uint8_t)__nv_cvt_float_to_fp8(__fmul_rn(v, inv), __NV_SATFINITE, __NV_E4M3);
}
// MXFP4 scale exponent: the smallest e with amax <= 6 * 2^e (amax = m * 2^E,
// m in [1, 2): e = E - 2 + (m > 1.5)); 0 or subnormal amax gives -127.
__device__ __forceinline__ int mx4_scale_exp(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ef = (int)((b >> 23) & 0xFF);
  if (ef == 0) return -127;
  const int e = ef - 127 - 2 + ((b & 0x7FFFFFu) > 0x400000u ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}
// E2M1 code (0..15, sign in bit 3) of v: round to nearest of the magnitudes
// 0, 0.5, 1, 1.5, 2, 3, 4, 6, ties to the even code (mantissa bit 0), values
// above 6 to 6. The code is the number of decision points at or below |v|;
// each tie point counts toward the even neighbour (a strict or a non-strict
// comparison).
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  const float a = fabsf(v);
  const uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                     (a >= 3.5f) + (a > 5.0f);
  return c | ((__float_as_uint(v) >> 28) & 8u);
}

// Byte offset of the scale of (row m of a GEMM chunk, K block b) in the chunk
// scale blocks [chunk][K / 128][1 KB]: two 512-byte halves of 128 rows, each in
// the order the tensor cores read block scales (16 * (m % 32) + 4 * (m / 32 % 4)
// + b % 4).
__device__ __forceinline__ int64_t chunk_scale_offset(int64_t chunk, int nslab, int m, int b) {
  return (chunk * nslab + b / 4) * 1024 + (m / 128) * 512 + 16 * (m % 32) + 4 * ((m / 32) % 4) +
         (b % 4);
}

// Device-side helpers used by several kernels.
__device__ __forceinline__ void set_error(int* err, int code, int detail) {
  if (atomicCAS(err, 0, code) == 0) err[1] = detail;
}

// Index checks of the checked build (compiled with -DKT_CHECKED into
// libktmoe_checked.so). Every index one kernel takes from another kernel's
// output (expert ids, row maps, GEMM chunk and tile lists, token ids, chunk
// counts) is range-checked where it is used: a failed check records
// kDevErrBounds and the site in the error word and the access is skipped, so
// kt_moe_check reports KT_ERR_BOUNDS instead of the kernel touching memory it
// does not own. In release builds in_range is constant true and the checks
// compile away.
#ifdef KT_CHECKED
constexpr bool kChecked = true;
#else
constexpr bool kChecked = false;
#endif
__device__ __forceinline__ bool in_range(int64_t v, int64_t lo, int64_t hi, int* err, int site) {
  if (!kChecked || (v >= lo && v < hi)) return true;
  set_error(err, kDevErrBounds, site);
  return false;
}
// A GEMM chunk: weight slot in [0, n_groups), 1..max_rows rows inside the
// n_rows hidden rows, a non-negative first activation row.
__device__ __forceinline__ bool chunk_in_range(const Chunk& c, int n_groups, int64_t n_rows,
                                               int max_rows, int* err, int site) {
  return in_range(c.group, 0, n_groups, err, site) &&
         in_range(c.nrows, 1, max_rows + 1, err, site + 1) &&
         in_range(c.row0, 0, n_rows - c.nrows + 1, err, site + 2) &&
         in_range(c.src_row0, 0, INT32_MAX, err, site + 3);
}

// Programmatic dependent launch: the forward's kernels are launched so that the
// next one is scheduled as soon as every CTA of the previous one has exited,
// without waiting for the previous grid's completion to be processed first.
// pdl_wait() blocks until the previous kernel of the stream has completed and
// its writes are visible, so every such kernel calls it before its first global
// memory access. (No kernel signals its dependents early: measured on the V3
// shapes, an early signal gained nothing over this and cost up to 2% at
// prefill.) A no-op for a kernel launched without the attribute.
#ifndef KT_PDL
#define KT_PDL 1
#endif
__device__ __forceinline__ void pdl_wait() {
#if KT_PDL
  asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
}

// Launch with the programmatic-stream-serialisation attribute (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = KT_PDL;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace ktmoe
