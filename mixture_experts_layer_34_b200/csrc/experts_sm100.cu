// Routed + shared expert SwiGLU FFNs (and the bf16 gate logits) on the sm_100a
// tensor cores.
//
// The expert FFN of the total-output equation in the "DeepSeekMoE 三改进"
// passage of the DeepSeek-V3 model.py notes (73biji.xyz/llm_pp_dsv3),
//     FFN_e(u) = W2_e (silu(W1_e u) * W3_e u),
// runs as two grouped GEMMs over the expert-sorted token rows:
//   up   : hidden[r, f]     = silu(<W1_e[f], u_r>) * <W3_e[f], u_r>      (bf16)
//   down : expert_out[r, o] = w_r * <W2_e[o], hidden[r]>                 (fp32)
// with w_r the routing weight of row r (1 for shared-expert rows), as in the
// "y[idx] += expert(x[idx]) * w" loop of "MoE 前向四步". The same kernel with a
// plain epilogue computes the gate logits W_g u (one group).
//
// Design: persistent CTA pairs (a 2-CTA cluster per pair of SMs), 192 threads
// per CTA, tcgen05 with cta_group::2.
//   - Operands are swapped relative to the math (D^T = W X^T): weights are the
//     M = 256 operand (128 rows in each CTA of the pair) and the tokens of one
//     chunk are N (a multiple of 32, at most 256; each CTA loads N/2 rows). An
//     expert with 37 tokens runs an N = 64 MMA instead of a 128-row tile of
//     padding, and decode streams weights at N = 32.
//   - Gate/up: each CTA's 128 weight rows are [64 rows of W1 | the same 64 rows
//     of W3] (two TMA boxes), so TMEM lanes 0-63 hold gate and 64-127 hold up of
//     the same 64 features; the "up" epilogue warps hand their values to the
//     "gate" warps through a double-buffered shared-memory exchange. One pair
//     tile covers 128 features; down and logits tiles cover 256 rows.
//   - Few, large TMA boxes per stage (TMA cost grows with the box count): the
//     weight tile in one or two boxes, the token rows in one 128-row box for a
//     full chunk, else in 32-row boxes.
//   - warp 0: TMA producer (3-stage ring of 64 KB per CTA, each stage two K
//     slabs of 64 so one wait and one commit serve 8 MMAs); warp 1: TMEM owner,
//     and in the even CTA the single thread issuing tcgen05.mma for the pair;
//     warps 2-5: epilogue (tcgen05.ld, SwiGLU / routing weight / none, staging
//     through shared memory for 16-byte row stores).
//   - Both CTAs' TMA loads signal the even CTA's "full" barrier; the MMA thread
//     commits to the "empty" and "accumulator full" barriers of both CTAs; both
//     epilogues arrive on the even CTA's "accumulator empty" barrier. Two TMEM
//     accumulator buffers of 256 columns overlap the epilogue with the next tile.
//   - The tile list (chunk, feature tile) is built on the device: within an
//     expert, blocks of 8 token chunks run feature-tile-major, so that tiles
//     reading one weight tile are neighbours in the list. Pairs take tiles from
//     a device counter (the even CTA's producer claims the next tile halfway
//     through the current one and publishes it to both CTAs through a 4-slot
//     ring of mbarrier-guarded slots), so tiles start in list order and
//     neighbours run together and share the weight tile through L2, however
//     long earlier tiles took.
//   - Launched with programmatic dependent launch: the barrier and TMEM setup
//     overlaps the previous kernel's tail; global memory is touched only after
//     griddepcontrol.wait.
// No TMA multicast is used.
//
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the
// kernel records KT_ERR_TIMEOUT in the workspace error word, drains what it
// issued, frees TMEM and returns.
#include <cuda.h>
#include <atomic>
#include <cstring>
#include <cuda_bf16.h>

#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

// A pipeline stage holds kSlabs K-slabs of 64 (each [weight tile | token tile]),
// so the MMA thread's per-stage wait and commit are shared by 4 * kSlabs MMAs.
#ifndef KT_SLABS
#define KT_SLABS 2
#endif
#ifndef KT_STAGES
#define KT_STAGES (6 / KT_SLABS)
#endif
constexpr int kSlabs = KT_SLABS;
constexpr int kStages = KT_STAGES;
constexpr int kBK = 64;                          // K elements per stage (128 B of bf16)
constexpr int kARowsCta = 128;                   // weight rows per CTA (MMA M = 256 per pair)
constexpr int kATileBytes = kARowsCta * kBK * 2;   // 16 KB
constexpr int kBHalfMax = kChunkRows / 2;        // token rows per CTA
constexpr int kBTileBytes = kBHalfMax * kBK * 2;   // 16 KB
constexpr int kSlabBytes = kATileBytes + kBTileBytes;   // 32 KB
constexpr int kStageBytes = kSlabs * kSlabBytes;
constexpr int kBoxRows = 32;                     // token-row TMA box for partial chunks
constexpr int kBoxBytes = kBoxRows * kBK * 2;    // 4 KB
constexpr int kThreads = 192;
constexpr int kStagingBytes = 4 * 16 * 32 * 4;   // 4 epilogue warps x [16 tokens][32 x 4 B]
constexpr int kXchgBytes = 2 * 2 * 16 * 32 * 4;  // up -> gate: 2 warp pairs x 2 buffers
constexpr int kCtrlBytes = 512;                  // mbarriers, TMEM address, schedule slots
// Stage layout: [weight tiles of the stage's K slabs | token tiles of the same
// slabs], each slab's weight tile 128 rows x 64 (16 KB) and its token tile
// hb x 32 rows x 64, hb = ceil(token rows per CTA / 32). A tile with hb = 1 (a
// pair N of at most 64) carries three K slabs per stage, others two.
constexpr int kSlabsLight = 3;
static_assert(kSlabsLight * (kATileBytes + kBoxBytes) <= kStageBytes, "3-slab stage layout");
static_assert(kSlabs * (kATileBytes + kBTileBytes) <= kStageBytes, "2-slab stage layout");
__device__ __forceinline__ int stage_slabs(int hb) { return hb == 1 ? kSlabsLight : kSlabs; }
// MXFP8 kinds: the block scales of each stage's slabs (per slab: 512 B for the
// CTA's 128 weight rows, 1 KB for the pair tile's up to 256 token rows).
constexpr int kSfaSlabBytes = 512, kSfbSlabBytes = 1024;
constexpr int kScaleStageBytes = kSlabsLight * (kSfaSlabBytes + kSfbSlabBytes);
constexpr int kSmemBase = kStages * kStageBytes + kStagingBytes + kXchgBytes + kCtrlBytes + 1024;
constexpr int kAccColsF8 = kChunkRowsF8;         // MXFP8 accumulator buffers (2 x 224 columns)
constexpr int kSfaCol = 2 * kAccColsF8;          // TMEM columns of the A scales (4)
constexpr int kSfbCol = kSfaCol + 4;             // and of the B scales (8)
static_assert(kSfbCol + 8 <= 512, "MXFP8 TMEM budget");
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr int kSched = 4;                        // tile schedule ring slots
// Consumers of a schedule slot: the MMA thread and 4 epilogue warps of the even
// CTA, the producer and 4 epilogue warps of the odd CTA.
constexpr int kSchedConsumers = 10;

// Epilogue kinds.
constexpr int kKindUp = 0;      // hidden = silu(W1 u) * W3 u            (bf16 out)
constexpr int kKindDown = 1;    // expert_out = w_r * W2 h               (fp32 out)
constexpr int kKindLogits = 2;  // logits = W_g u, implicit token chunks (fp32 out)
constexpr int kKindUpF8 = 3;    // MXFP8 weights and tokens: hidden as MXFP8 codes + scales
constexpr int kKindDownF8 = 4;  // MXFP8 weights and hidden rows: expert_out (fp32 out)

template <int kKind>
struct Kind {
  static constexpr bool kF8 = kKind == kKindUpF8 || kKind == kKindDownF8;
  static constexpr bool kUp = kKind == kKindUp || kKind == kKindUpF8;
  static constexpr int kOutBytes = kKind == kKindUpF8 ? 1 : (kUp ? 2 : 4);
  static constexpr int kRowsPerPair = kUp ? 128 : 256;   // output features per pair tile
  static constexpr int kSlabK = kF8 ? 128 : kBK;         // K elements per 128-byte slab
  static constexpr int kAccCols = kF8 ? kAccColsF8 : 256;  // TMEM columns per accumulator
  static constexpr int kSmem = kSmemBase + (kF8 ? kStages * kScaleStageBytes : 0);
};

struct GemmArgs {
  const Chunk* chunks;
  const int2* tiles;         // (chunk index, feature tile) in schedule order
  const int32_t* n_tiles;    // device count of tiles
  int* counter;              // device tile counter (zeroed before the launch), or null:
                             // then pair p takes tiles p, p + pairs, ...
  int implicit_rows;         // > 0: logits; chunks of implicit_chunk over this many token rows
  int implicit_chunk;        // logits: token rows per chunk (a multiple of 32, <= kChunkRows)
  int n_ftiles;              // feature tiles per group
  int rows_per_group;        // weight rows per group (I for up, d for down, E for logits)
  int K;                     // reduction length
  int E;                     // routed experts (up: groups >= E read x directly)
  int out_cols;              // valid output columns
  int ldo;                   // output row stride in elements
  void* out;
  const float* row_weight;   // down: weight of routed rows
  int n_routed_rows;         // T * k
  int* err;
  // Bounds of the chunk and tile lists (the checked build verifies each tile):
  int n_groups;              // weight slots
  int64_t n_rows;            // hidden rows T * (k + S)
  int max_chunks;            // chunk list capacity
  int max_chunk_rows;        // rows per chunk at most
  int a_fp4;                 // MXFP8 kinds: weights as packed E2M1 codes (MXFP4), else E4M3
  int tma3d;                 // 1: one box per stage from the 3-D/4-D maps (K % 64 == 0)
  int gate_hi;               // up, 3-D maps: W3 precedes W1 in memory, so the upper 64
                             // rows of each CTA's weight tile are W1 (gate)
  // MXFP8 kinds:
  int n_kslabs;              // K / 128
  int n_ftiles_sf;           // feature tiles per group in the packed weight scales
  uint8_t* hid_sf;           // up: hidden-row scale blocks [chunk][I / 128][1 KB]
};

// Tensor maps of one launch (bf16, 128-byte swizzle). Token-row sources: up: 0
// the permuted rows, 1 x (shared experts); down: the hidden rows; logits: x.
//   2-D maps (K a multiple of 8): one K slab per box.
//   3-D/4-D maps (K a multiple of 64): K split as [K / 64][64], so one box
//   covers all K slabs of a stage; the gate/up weight map has a fourth
//   dimension that steps from one of W1, W3 to the other, so one box yields
//   [64 rows of one | the same 64 rows of the other] for every slab.
struct TmaMaps {
  CUtensorMap a2[2];      // weights, one slab: W1 | W2 | W_g, and W3 (up)
  CUtensorMap b2[2][2];   // [source][32-row box, 128-row box], one slab
  CUtensorMap a3[2];      // weights of a [2-slab, 3-slab] stage
  CUtensorMap b3[2][5];   // [source][2-slab stage of 32/64/96/128 rows, 3-slab stage of 32]
  // MXFP8 kinds: the packed weight scales and the token chunks' scales, as
  // rows of 256 bytes; boxes of [2-slab, 3-slab] stages.
  CUtensorMap sfa[2];
  CUtensorMap sfb[2];
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Arrive on a barrier given by its shared::cluster address (own or peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr)
               : "memory");
}
// The same arrive without release semantics: it does not wait until this
// thread's earlier memory operations are visible across the cluster.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t caddr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr)
               : "memory");
}
// Arrive on this CTA's barrier, ordering this thread's earlier writes to its
// own shared memory before the arrive (CTA scope).
__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// Arrive on a barrier at a shared::cluster address and raise its expected
// transaction bytes by `bytes` (completed by st.async below).
__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t caddr, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.relaxed.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(
                   caddr),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait. Returns false (after recording the timeout) if the phase did not
// complete within kWaitLimitNs, or if another CTA already recorded an error.
// Slow path of mbar_wait, out of line so the issuing loops stay short.
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, int* err, int where,
                                            uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile int*>(err) != 0) return false;
      if (globaltimer() - t0 > limit_ns) {
        set_error(err, kDevErrTimeout, where);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, int where) {
  return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, err, where);
}
// 2-D tiled TMA load into this CTA's shared memory, completing on the barrier
// at shared::cluster address `bar` (the even CTA's, for the pair), with an L2
// eviction-priority policy.
__device__ __forceinline__ void tma_load_pair(void* dst, const CUtensorMap* map, uint32_t bar, int c0,
                                              int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_load3_pair(void* dst, const CUtensorMap* map, uint32_t bar,
                                               int c0, int c1, int c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_load4_pair(void* dst, const CUtensorMap* map, uint32_t bar,
                                               int c0, int c1, int c2, int c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "l"(policy)
      : "memory");
}
// L2 policies: data read once soon (evict first) and data re-read later (evict last).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 B, 8-row groups 1024 B apart (SBO), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;             // LBO (unused for swizzled K-major)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;     // SBO
  d |= static_cast<uint64_t>(1u) << 46;             // version
  d |= static_cast<uint64_t>(2u) << 61;             // SWIZZLE_128B
  return d;
}
// Instruction descriptor, kind::f16: bf16 A and B (K-major), fp32 D, M x N.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
// MXFP8: E4M3 A and B, E8M0 block scales (one per 32 along K) read from TMEM;
// the scale byte used by this K = 32 MMA is selected by sf_id (bits 29-30 for A,
// 4-5 for B). a_fmt (bits 7-9) is A's element format: 0 E4M3, 5 E2M1 (MXFP4
// weights; B stays E4M3). Accumulation is fp32.
constexpr uint32_t kFmtE4M3 = 0, kFmtE2M1 = 5;
__device__ __forceinline__ uint32_t idesc_mxf8(int M, int N, int sf_id, uint32_t a_fmt) {
  return (static_cast<uint32_t>(sf_id) << 4) | (a_fmt << 7) |
         (static_cast<uint32_t>(N >> 3) << 17) | (1u << 23) |
         (static_cast<uint32_t>(M >> 4) << 24) | (static_cast<uint32_t>(sf_id) << 29);
}
__device__ __forceinline__ void mma_pair_mxf8(uint32_t d_tmem, uint64_t a, uint64_t b,
                                              uint32_t idesc, uint32_t sfa_tmem,
                                              uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// Shared-memory descriptor of a block of 32 rows x 16 bytes (no swizzle,
// K-major, 8-row core matrices 128 bytes apart), the source of a scale copy.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;      // LBO
  d |= static_cast<uint64_t>(128u >> 4) << 32;      // SBO
  d |= static_cast<uint64_t>(1u) << 46;             // version
  return d;
}
// 512 bytes of block scales (128 rows x 4 K blocks) into 4 TMEM columns of all
// 128 lanes of both CTAs of the pair, each from its own shared memory.
__device__ __forceinline__ void sf_copy_pair(uint32_t tmem_col, uint32_t saddr) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(tmem_col),
               "l"(sf_desc(saddr))
               : "memory");
}
__device__ __forceinline__ void mma_pair_bf16(uint32_t d_tmem, uint64_t a, uint64_t b,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at shared::cluster address `bar` when every MMA
// this thread issued so far has completed.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// The same arrival on the barrier at this shared::cta offset in both CTAs of
// the pair (CTA mask 0b11).
__device__ __forceinline__ void mma_commit_both(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// silu(g) = g / (1 + e^-g) with the fast reciprocal division (within 2 ulp;
// the result is rounded to bf16 or quantised to E4M3 right after). For very
// negative g the denominator overflows and the result is 0 (silu -> 0 there).
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Asynchronous stores into a peer CTA's shared memory, each completing its
// bytes on the peer's barrier `bar` (shared::cluster addresses; 16- and 8-byte
// aligned).
__device__ __forceinline__ void st_async_v4(uint32_t caddr, int a, int b, int c, int d,
                                            uint32_t bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.s32 [%0], {%1, %2, %3, %4}, [%5];" ::
          "r"(caddr),
      "r"(a), "r"(b), "r"(c), "r"(d), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t caddr, int a, int b, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.s32 [%0], {%1, %2}, [%3];" ::
                   "r"(caddr),
               "r"(a), "r"(b), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void read_slot(const int* slot, Chunk& ch, int& ft, int& ci) {
  const volatile int* v = slot;
  ch = Chunk{v[0], v[1], v[2], v[3]};
  ft = v[4];
  ci = v[5];
}

// True iff `v` holds on every thread that continues together: the warp, or the
// 64 threads of an up-epilogue warp pair (named barrier `bar_id`).
template <bool kPair>
__device__ __forceinline__ bool uniform_ok(bool v, int bar_id) {
  if (kPair) {
    uint32_t all_ok;
    asm volatile(
        "{\n\t.reg .pred p, r;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred r, %2, 64, p;\n\t"
        "selp.u32 %0, 1, 0, r;\n\t}"
        : "=r"(all_ok)
        : "r"(v ? 1u : 0u), "r"(bar_id)
        : "memory");
    return all_ok != 0;
  }
  return __all_sync(0xffffffffu, v);
}

__device__ __forceinline__ void get_tile(const GemmArgs& a, int t, Chunk& ch, int& ft, int& ci) {
  if (a.implicit_rows > 0) {
    const int c = a.implicit_chunk;
    ci = t / a.n_ftiles;
    ft = t % a.n_ftiles;
    ch = Chunk{0, ci * c, min(c, a.implicit_rows - ci * c), ci * c};
  } else {
    const int2 e = a.tiles[t];
    ci = e.x;
    ft = e.y;
    // (Checked build) a tile naming a chunk, feature tile, weight slot or rows
    // outside the lists ends this pair's schedule like the end marker.
    if (!in_range(e.x, 0, a.max_chunks, a.err, 131) || !in_range(e.y, 0, a.n_ftiles, a.err, 132)) {
      ch = Chunk{-1, 0, 0, 0};
      return;
    }
    ch = a.chunks[e.x];
    if (!chunk_in_range(ch, a.n_groups, a.n_rows, a.max_chunk_rows, a.err, 133)) ch = Chunk{-1, 0, 0, 0};
  }
}

// Token columns of a chunk rounded up so that each CTA of the pair gets a
// multiple of 16 rows (the MMA N is then a multiple of 32).
__device__ __forceinline__ int pair_cols(int nrows) { return (nrows + 31) & ~31; }

// ---------------------------------------------------------------------------
// The grouped GEMM kernel
// ---------------------------------------------------------------------------
template <int kKind>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ TmaMaps maps, const GemmArgs args) {
  using KD = Kind<kKind>;
  constexpr bool kUp = KD::kUp;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stage_base = smem;
  uint8_t* staging = smem + kStages * kStageBytes;
  float* xchg = reinterpret_cast<float*>(smem + kStages * kStageBytes + kStagingBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kStagingBytes +
                                               kXchgBytes);
  uint64_t* full_bar = bars;                        // [kStages]  (even CTA's are used)
  uint64_t* empty_bar = bars + kStages;             // [kStages]
  uint64_t* tfull_bar = bars + 2 * kStages;         // [2]
  uint64_t* tempty_bar = bars + 2 * kStages + 2;    // [2]        (even CTA's are used)
  uint64_t* drain_bar = bars + 2 * kStages + 4;     // [1]
  uint64_t* sched_full = bars + 2 * kStages + 5;    // [kSched] tile published (each CTA)
  uint64_t* sched_empty = sched_full + kSched;      // [kSched] slot consumed (even CTA's)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sched_empty + kSched);
  // MXFP8: per stage [A scales of up to 3 slabs | B scales of up to 3 slabs].
  uint8_t* sf_base = smem + kSmemBase - 1024;
  // Schedule slots: {group, row0, nrows, src_row0, feature tile, -, -, -}; group
  // -1 ends the schedule.
  int* sched_info = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(bars) + 256);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();             // 0: even (MMA-issuing) CTA, 1: odd
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 8);     // 4 epilogue warps x 2 CTAs
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < kSched; ++i) {
      mbar_init(&sched_full[i], 1);     // one arrival: the even CTA's producer (on the
                                        // odd CTA, plus the slot's 24 bytes as transactions)
      mbar_init(&sched_empty[i], kSchedConsumers);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (KD::kF8)
      for (int i = 0; i < 2; ++i) {
        prefetch_tmap(&maps.sfa[i]);
        prefetch_tmap(&maps.sfb[i]);
      }
    if (args.tma3d) {
      for (int i = 0; i < 2; ++i) prefetch_tmap(&maps.a3[i]);
      for (int i = 0; i < (kUp ? 2 : 1); ++i)
        for (int j = 0; j < 5; ++j) prefetch_tmap(&maps.b3[i][j]);
    } else {
      for (int i = 0; i < (kUp ? 2 : 1); ++i) {
        prefetch_tmap(&maps.a2[i]);
        prefetch_tmap(&maps.b2[i][0]);
        prefetch_tmap(&maps.b2[i][1]);
      }
    }
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, 512);
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touches only this CTA pair's shared memory, TMEM and the
  // kernel parameters; the previous kernel's outputs are read after this.
  pdl_wait();

  const int n_tiles =
      args.implicit_rows > 0
          ? ((args.implicit_rows + args.implicit_chunk - 1) / args.implicit_chunk) * args.n_ftiles
          : *args.n_tiles;
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;   // static schedule only
  // K slabs per tile (the last may run past K: TMA fills those columns with zeros).
  const int n_slabs = (args.K + KD::kSlabK - 1) / KD::kSlabK;
  int* err = args.err;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      // The even CTA's producer also schedules: it takes the pair's next tile and
      // publishes it to both CTAs' schedule slots; the odd CTA's producer reads it.
      // The next tile is claimed halfway through the current tile's stages and
      // read after its last stage is issued, so the claim (a global atomic) and
      // the reads of the tile list overlap the copies in flight instead of
      // stalling the pipeline between tiles.
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      int sslot = 0, iter = 0;
      uint32_t sphase = 0;
      const uint64_t p_first = policy_evict_first(), p_normal = policy_evict_normal(),
                     p_last = policy_evict_last();
      int t_next = 0;
      Chunk c_next{-1, 0, 0, 0};
      int f_next = 0, ci_next = 0;
      auto claim = [&]() {
        t_next = args.counter ? atomicAdd(args.counter, 1) : pair + iter * n_pairs;
        ++iter;
      };
      auto fetch = [&]() {
        c_next = Chunk{-1, 0, 0, 0};
        f_next = 0;
        ci_next = 0;
        if (t_next < n_tiles) get_tile(args, t_next, c_next, f_next, ci_next);
      };
      if (leader) {
        claim();
        fetch();
      }
      for (;;) {
        if (leader) {
          if (!mbar_wait(&sched_empty[sslot], sphase ^ 1u, err, 5 + 8 * kKind)) {
            ok = false;
            break;
          }
          const Chunk c = c_next;
          const int f = f_next, cidx = ci_next;
          int* slot = sched_info + 8 * sslot;
          slot[0] = c.group;
          slot[1] = c.row0;
          slot[2] = c.nrows;
          slot[3] = c.src_row0;
          slot[4] = f;
          slot[5] = cidx;
          const uint32_t peer_slot = map_to_cta(smem_u32(slot), 1);
          // The odd CTA's copy travels by st.async and completes its 24 bytes
          // on that CTA's barrier, so no release (which would wait for this
          // thread's copies and remote stores in flight) sits between the last
          // stage of one tile and the first copies of the next.
          const uint32_t peer_full = map_to_cta(smem_u32(&sched_full[sslot]), 1);
          st_async_v4(peer_slot, c.group, c.row0, c.nrows, c.src_row0, peer_full);
          st_async_v2(peer_slot + 16, f, cidx, peer_full);
          mbar_arrive_expect_tx_cluster(peer_full, 24u);
          mbar_arrive_local(&sched_full[sslot]);
        } else {
          if (!mbar_wait(&sched_full[sslot], sphase, err, 6 + 8 * kKind)) {
            ok = false;
            break;
          }
        }
        Chunk ch;
        int ft, ci;
        read_slot(sched_info + 8 * sslot, ch, ft, ci);
        const uint32_t empty_leader = map_to_cta(smem_u32(&sched_empty[sslot]), 0);
        if (!leader && ch.group < 0) mbar_arrive_cluster(empty_leader);
        if (++sslot == kSched) {
          sslot = 0;
          sphase ^= 1u;
        }
        if (ch.group < 0) break;
        const int half = pair_cols(ch.nrows) / 2;
        // First weight row of this CTA's half of the pair tile.
        const int a_row = ch.group * args.rows_per_group + ft * KD::kRowsPerPair +
                          (kUp ? 64 : 128) * (int)rank;
        // L2 priorities (KT_L2_HINTS): 0 none; 1 weights evict-first, token rows
        // evict-last; 2 as 1 for partial chunks, while a full chunk's weights
        // (re-read by the expert's other chunks) stay normal; 3 as 2 with
        // normal token rows. The gate logits re-read W_g for every chunk.
        uint64_t pol_a = p_normal, pol_b = p_normal;
        if (KT_L2_HINTS != 0) {
          const bool full = ch.nrows == (KD::kF8 ? kChunkRowsF8 : kChunkRows);
          if (kKind == kKindLogits) {
            pol_a = p_last;
            pol_b = p_first;
          } else if (KT_L2_HINTS == 1) {
            pol_a = p_first;
            pol_b = p_last;
          } else {
            pol_a = full ? p_normal : p_first;
            pol_b = (KT_L2_HINTS == 2 && full) ? p_last : p_normal;
          }
        }
        const int src = (kUp && ch.group >= args.E) ? 1 : 0;
        int b_row = (kUp ? ch.src_row0 : ch.row0) + half * (int)rank;
        // Token rows in 32-row blocks (the last may run up to 16 rows past the
        // chunk; those columns are unused).
        const int hb = (half + kBoxRows - 1) / kBoxRows;
        const int slabs = stage_slabs(hb);
        const int nk = (n_slabs + slabs - 1) / slabs;
        const uint32_t b_slab = hb * kBoxBytes;   // token-tile bytes of one slab
        // Maps of this tile's stage shape: 3-slab stages for one 32-row token
        // block per CTA (hb == 1), else 2-slab stages of hb blocks.
        const CUtensorMap* a3 = &maps.a3[hb == 1 ? 1 : 0];
        const CUtensorMap* b3 = &maps.b3[src][hb == 1 ? 4 : hb - 1];
        for (int kb = 0; kb < nk; ++kb) {
          const int s0 = kb * slabs;
          const int valid = min(slabs, n_slabs - s0);
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, err, 1 + 8 * kKind)) {
            ok = false;
            break;
          }
          const uint32_t fbar = map_to_cta(smem_u32(&full_bar[stage]), 0);
          uint8_t* sA = stage_base + stage * kStageBytes;
          uint8_t* sB = sA + slabs * kATileBytes;
          if (args.tma3d) {
            // Two boxes for the whole stage; slabs past K are filled with zeros
            // and counted in the transaction bytes. Packed 4-bit weight codes
            // count their global bytes, half the weight tile's shared bytes.
            const uint32_t sf_bytes = KD::kF8 ? slabs * (kSfaSlabBytes + kSfbSlabBytes) : 0;
            const uint32_t a_tx = (KD::kF8 && args.a_fp4) ? kATileBytes / 2 : kATileBytes;
            if (leader)
              mbar_arrive_expect_tx(&full_bar[stage], 2u * (slabs * (a_tx + b_slab) + sf_bytes));
            if (kUp)
              tma_load4_pair(sA, a3, fbar, 0, a_row, 0, s0, pol_a);
            else
              tma_load3_pair(sA, a3, fbar, 0, a_row, s0, pol_a);
            tma_load3_pair(sB, b3, fbar, 0, b_row, s0, pol_b);
            if (KD::kF8) {
              // Scales: this CTA's 128 weight rows (packed, 512 B per slab) and all
              // token rows of the pair tile (1 KB per slab of the chunk's blocks),
              // as rows of 256 bytes.
              uint8_t* sS = sf_base + stage * kScaleStageBytes;
              const int li = hb == 1 ? 1 : 0;
              const int64_t ablk =
                  ((int64_t)(ch.group * args.n_ftiles_sf + ft) * 2 + rank) * args.n_kslabs + s0;
              tma_load_pair(sS, &maps.sfa[li], fbar, 0, (int)(2 * ablk), pol_a);
              tma_load_pair(sS + kSlabsLight * kSfaSlabBytes, &maps.sfb[li], fbar, 0,
                            (int)(((int64_t)ci * args.n_kslabs + s0) * 4), pol_b);
            }
          } else {
            if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * valid * (kATileBytes + b_slab));
            for (int j = 0; j < valid; ++j) {
              const int kc = (s0 + j) * KD::kSlabK;
              uint8_t* a = sA + j * kATileBytes;
              uint8_t* b = sB + j * b_slab;
              if (kUp) {
                // [64 rows of W1 | the same 64 rows of W3]
                tma_load_pair(a, &maps.a2[0], fbar, kc, a_row, pol_a);
                tma_load_pair(a + 64 * 128, &maps.a2[1], fbar, kc, a_row, pol_a);
              } else {
                tma_load_pair(a, &maps.a2[0], fbar, kc, a_row, pol_a);
              }
              if (half == kBHalfMax) {
                tma_load_pair(b, &maps.b2[src][1], fbar, kc, b_row, pol_b);
              } else {
                for (int i = 0; i < hb; ++i)
                  tma_load_pair(b + i * kBoxBytes, &maps.b2[src][0], fbar, kc,
                                b_row + i * kBoxRows, pol_b);
              }
            }
          }
          issued = issued < kStages ? issued + 1 : kStages;
          if (leader) {
            if (kb == nk / 2) claim();
            if (kb == nk - 1) fetch();
          }
          // The slot's values are in the copies just issued (their coordinates
          // needed the loads), so the slot is free: a relaxed arrive, which
          // does not wait for the copies themselves.
          if (!leader && kb == 0) mbar_arrive_cluster_relaxed(empty_leader);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (!ok && leader) {
        // Let the copies already in flight land before the CTA can exit.
        int s = stage;
        uint32_t ph = phase;
        for (int i = 0; i < issued; ++i) {
          if (--s < 0) {
            s = kStages - 1;
            ph ^= 1u;
          }
          const uint64_t t0 = globaltimer();
          while (!mbar_try_wait(&full_bar[s], ph) && globaltimer() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer (even CTA, for the pair) ----------------
      const uint64_t desc_a0 = sw128_desc(smem_u32(stage_base));
      const uint32_t a_fmt = args.a_fp4 ? kFmtE2M1 : kFmtE4M3;
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      bool ok = true;
      bool issued_any = false;
      int sslot = 0;
      uint32_t sphase = 0;
      for (;;) {
        if (!mbar_wait(&sched_full[sslot], sphase, err, 7 + 8 * kKind)) break;
        Chunk ch;
        int ft, ci;
        read_slot(sched_info + 8 * sslot, ch, ft, ci);
        const uint32_t empty_own = smem_u32(&sched_empty[sslot]);
        if (ch.group < 0) mbar_arrive_cluster(empty_own);
        if (++sslot == kSched) {
          sslot = 0;
          sphase ^= 1u;
        }
        if (ch.group < 0) break;
        const int n = pair_cols(ch.nrows);
        if (!mbar_wait(&tempty_bar[buf], bphase ^ 1u, err, 2 + 8 * kKind)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(256, n);
        const uint32_t d0 = tmem_base + buf * KD::kAccCols;
        const int hb = (n / 2 + kBoxRows - 1) / kBoxRows;
        const int slabs = stage_slabs(hb);
        const int nk = (n_slabs + slabs - 1) / slabs;
        const uint32_t b_off = slabs * kATileBytes, b_slab = hb * kBoxBytes;
        for (int kb = 0; kb < nk; ++kb) {
          const int valid = min(slabs, n_slabs - kb * slabs);
          if (!mbar_wait(&full_bar[stage], phase, err, 3 + 8 * kKind)) {
            ok = false;
            break;
          }
          // Descriptors of this stage: the start-address field counts 16-byte
          // units, so the 32-byte step between K sub-blocks adds 2.
#pragma unroll
          for (int j = 0; j < kSlabsLight; ++j) {
            if (j >= valid) break;
            const uint64_t da = desc_a0 + (uint64_t)((stage * kStageBytes + j * kATileBytes) >> 4);
            const uint64_t db =
                desc_a0 + (uint64_t)((stage * kStageBytes + b_off + j * b_slab) >> 4);
            if (KD::kF8) {
              // This slab's block scales into TMEM (in issue order with the MMAs
              // that read them and with the previous slab's MMAs), then four
              // K = 32 MMAs, each reading its K block's scale byte.
              const uint32_t sS = smem_u32(sf_base + stage * kScaleStageBytes);
              const uint32_t sB = sS + kSlabsLight * kSfaSlabBytes + j * kSfbSlabBytes;
              // Token rows 128 and up (second half of the slab's token scales)
              // exist only in tiles of more than 128 columns.
              const uint32_t sfa = tmem_base + kSfaCol, sfb = tmem_base + kSfbCol;
              sf_copy_pair(sfa, sS + j * kSfaSlabBytes);
              sf_copy_pair(sfb, sB);
              if (n > 128) sf_copy_pair(sfb + 4, sB + kSfbSlabBytes / 2);
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_pair_mxf8(d0, da + 2 * ks, db + 2 * ks, idesc_mxf8(256, n, ks, a_fmt), sfa,
                              sfb, (kb | j | ks) != 0);
            } else {
#pragma unroll
              for (int ks = 0; ks < kBK / 16; ++ks)
                mma_pair_bf16(d0, da + 2 * ks, db + 2 * ks, idesc, (kb | j | ks) != 0);
            }
          }
          mma_commit_both(smem_u32(&empty_bar[stage]));
          issued_any = true;
          // The slot's values are in the MMAs just issued: relaxed arrive (a
          // release would wait for the MMAs in flight).
          if (kb == 0) mbar_arrive_cluster_relaxed(empty_own);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_both(smem_u32(&tfull_bar[buf]));
        if (++buf == 2) {
          buf = 0;
          bphase ^= 1u;
        }
      }
      // Wait (bounded) until every MMA issued has completed, so TMEM and shared
      // memory can be released.
      if (issued_any) {
        mma_commit_pair(smem_u32(drain_bar));
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(drain_bar, 0) && globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ---------------- Epilogue (warps 2..5, both CTAs) ----------------
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    uint8_t* stg = staging + (warp - 2) * 16 * 32 * 4;
    // Gate/up: quarters 0,1 hold gate of features 0-31 / 32-63, quarters 2,3
    // hold up of the same features; warp pair p = q & 1 meets on named barrier
    // 1 + p (64 threads).
    const int pr = q & 1;
    const bool gate_warp = (q < 2) != (args.gate_hi != 0);
    const uint32_t tempty_leader0 = map_to_cta(smem_u32(&tempty_bar[0]), 0);
    const uint32_t tempty_leader1 = map_to_cta(smem_u32(&tempty_bar[1]), 0);
    int buf = 0;
    uint32_t bphase = 0;
    int xb = 0;                          // exchange buffer in use (up pairs)
    int sslot = 0;
    uint32_t sphase = 0;
    const uint32_t sched_empty_leader = map_to_cta(smem_u32(&sched_empty[0]), 0);
    for (;;) {
      // Wait outcomes must be uniform over the threads that go on together:
      // tcgen05.ld is .sync.aligned, and up pairs meet on named barriers.
      const bool got = mbar_wait(&sched_full[sslot], sphase, err, 8 + 8 * kKind);
      if (!uniform_ok<kUp>(got, 1 + pr)) break;
      Chunk ch;
      int ft, ci;
      read_slot(sched_info + 8 * sslot, ch, ft, ci);
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(sched_empty_leader + sslot * 8);
      if (++sslot == kSched) {
        sslot = 0;
        sphase ^= 1u;
      }
      if (ch.group < 0) break;
      const int n = pair_cols(ch.nrows);
      // Down: the routing weights of the tile's rows (lane l holds rows l + 32 i;
      // shared-expert rows weigh 1), loaded before the accumulator wait so their
      // latency overlaps it instead of stalling every 16-column block.
      constexpr bool kDown = kKind == kKindDown || kKind == kKindDownF8;
      float rw[kDown ? 8 : 1];
      if (kDown) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = lane + 32 * i, row = ch.row0 + r;
          rw[i] = (r < ch.nrows && row < args.n_routed_rows) ? args.row_weight[row] : 1.0f;
        }
      }
      const bool ready = mbar_wait(&tfull_bar[buf], bphase, err, 4 + 8 * kKind);
      if (!uniform_ok<kUp>(ready, 1 + pr)) break;
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * KD::kAccCols;
      // First output column of this warp.
      const int col0 = kUp ? ft * 128 + 64 * (int)rank + 32 * pr
                           : ft * 256 + 128 * (int)rank + 32 * q;
      for (int c0 = 0; c0 < n; c0 += 16) {
        float v[16];
        tmem_ld16(tbase + c0, v);
        tmem_ld_wait();
        if (KD::kF8 && kUp) {
          // MXFP8 hidden rows. The two warps of a pair split the 16 columns: each
          // sends the other the 8 values it lacks (gate or up), then computes,
          // quantises and stores its own 8 token rows. The warp's 32 features of
          // one token are one block: its scale is the rule's exponent of the
          // block's absolute maximum (one integer warp reduction over |h| bits),
          // written into the down GEMM's scale blocks of this chunk.
          float* xc = xchg + (pr * 2 + xb) * 16 * 32;
          const int mine0 = gate_warp ? 0 : 8, other0 = 8 - mine0;
#pragma unroll
          for (int i = 0; i < 8; ++i) xc[(other0 + i) * 32 + lane] = gate_warp ? v[8 + i] : v[i];
          asm volatile("bar.sync %0, 64;" ::"r"(1 + pr) : "memory");
          xb ^= 1;
          uint8_t* s8 = stg;
          uint8_t my_scale = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            // (static indices into v: the selects keep it in registers)
            const float mv = gate_warp ? v[i] : v[8 + i], ov = xc[(mine0 + i) * 32 + lane];
            const float h = gate_warp ? silu(mv) * ov : silu(ov) * mv;
            const uint32_t amax =
                __reduce_max_sync(0xffffffffu, __float_as_uint(h) & 0x7fffffffu);
            const int e = mx_scale_exp(__uint_as_float(amax));
            s8[i * 32 + lane] = mx_code(h, mx_inv_scale(e));
            if (lane == i) my_scale = (uint8_t)(e + 127);
          }
          const int cr = c0 + mine0;
          if (lane < 8 && cr + lane < ch.nrows)
            args.hid_sf[chunk_scale_offset(ci, args.out_cols / 128, cr + lane, col0 / 32)] =
                my_scale;
          __syncwarp();
          // 8 token rows x 32 code bytes: 16 chunks of 16 bytes.
          if (lane < 16) {
            const int rr = lane / 2, part = lane % 2;
            if (cr + rr < ch.nrows)
              *reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                        (int64_t)(ch.row0 + cr + rr) * args.ldo + col0 +
                                        part * 16) =
                  *reinterpret_cast<const uint4*>(s8 + rr * 32 + part * 16);
          }
          __syncwarp();
          continue;
        }
        if (kUp) {
          float* xc = xchg + (pr * 2 + xb) * 16 * 32;
          if (!gate_warp) {
#pragma unroll
            for (int i = 0; i < 16; ++i) xc[i * 32 + lane] = v[i];
          }
          asm volatile("bar.sync %0, 64;" ::"r"(1 + pr) : "memory");
          xb ^= 1;
          if (gate_warp) {
            __nv_bfloat16* sb = reinterpret_cast<__nv_bfloat16*>(stg);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              sb[i * 32 + lane] = __float2bfloat16_rn(silu(v[i]) * xc[i * 32 + lane]);
          }
        } else {
          if (kDown) {
            // Column c0 + i is row c0 + i of the tile: lane (c0 + i) % 32 holds
            // its weight in rw[0] (c0 is a multiple of 16; rw moves down one
            // register after every 32 columns, so all indices stay static).
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= __shfl_sync(0xffffffffu, rw[0], (c0 & 16) + i);
            if (c0 & 16) {
#pragma unroll
              for (int k = 0; k + 1 < (kDown ? 8 : 1); ++k) rw[k] = rw[k + 1];
            }
          }
          float* sf = reinterpret_cast<float*>(stg);
#pragma unroll
          for (int i = 0; i < 16; ++i) sf[i * 32 + lane] = v[i];
        }
        if (!kUp || gate_warp) {
          __syncwarp();
          // 16 token rows of this warp's 32 output columns in 16-byte chunks:
          // 32 B per row (MXFP8 hidden codes), 64 B (bf16 hidden) or 128 B (fp32).
          constexpr int kRowBytes = 32 * KD::kOutBytes;
          constexpr int kChunksPerRow = kRowBytes / 16;
          constexpr int kElemsPerChunk = 16 / KD::kOutBytes;
#pragma unroll
          for (int it = 0; it < 16 * kChunksPerRow / 32; ++it) {
            const int idx = lane + it * 32;
            const int rr = idx / kChunksPerRow, part = idx % kChunksPerRow;
            const int c = c0 + rr;
            const int col = col0 + part * kElemsPerChunk;
            if (c < ch.nrows && col < args.out_cols) {
              const uint4 val = *reinterpret_cast<const uint4*>(stg + rr * kRowBytes + part * 16);
              *reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                        ((int64_t)(ch.row0 + c) * args.ldo + col) *
                                            KD::kOutBytes) = val;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1u;
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launches
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix; box = box_rows x 64.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 3-D view [cols / slab][rows][slab] of a row-major [rows, cols] matrix of bf16
// (slab 64) or one-byte E4M3 codes (u8: slab 128) with cols a multiple of the
// slab; box = box_slabs x box_rows x slab (128 bytes wide), landing slab-major.
// Element kinds of the K-slab maps: bf16 (64 per 128-byte slab), bytes (E4M3
// codes, 128 per slab), and packed E2M1 codes (128 per slab: 64 bytes in
// global memory, which the copy spreads to 128 bytes in shared memory, each 8
// bytes of codes followed by an 8-byte gap, the layout the block-scaled MMA
// reads 4-bit operands in; its transaction count is the 64 global bytes).
enum { kElemBf16 = 0, kElemU8 = 1, kElemFp4 = 2 };

CUtensorMapDataType elem_type(int elem) {
  return elem == kElemFp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B
                          : (elem == kElemU8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                             : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

bool make_map3(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
               uint32_t box_slabs, int elem = kElemBf16) {
  EncodeTiledFn enc = get_encode_fn();
  // Elements per slab and global bytes per slab row.
  const uint64_t slab = elem == kElemBf16 ? 64 : 128, slab_bytes = elem == kElemFp4 ? 64 : 128;
  if (!enc || cols % slab != 0) return false;
  const cuuint64_t dims[3] = {slab, rows, cols / slab};
  const cuuint64_t strides[2] = {cols / slab * slab_bytes, slab_bytes};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(slab), box_rows, box_slabs};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, elem_type(elem), 3,
             const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 4-D view [cols / 64][2][rows][64] of two equally shaped row-major bf16
// matrices p and q (cols a multiple of 64): the second index steps from the one
// at the lower address to the other. box = box_slabs x 2 x box_rows x 64, i.e.
// per slab [box_rows rows of the first | the same rows of the second].
// *q_first tells whether q is the first.
bool make_map4_pair(CUtensorMap* m, const void* p, const void* q, uint64_t rows, uint64_t cols,
                    uint32_t box_rows, uint32_t box_slabs, bool* q_first, int elem = kElemBf16) {
  EncodeTiledFn enc = get_encode_fn();
  const uint64_t up = reinterpret_cast<uint64_t>(p), uq = reinterpret_cast<uint64_t>(q);
  const uint64_t lo = up < uq ? up : uq, hi = up < uq ? uq : up;
  const uint64_t slab = elem == kElemBf16 ? 64 : 128, slab_bytes = elem == kElemFp4 ? 64 : 128;
  const uint64_t align = elem == kElemFp4 ? 32 : 16;   // packed 4-bit maps: 32-byte strides
  *q_first = uq < up;
  if (!enc || cols % slab != 0 || hi == lo || (hi - lo) % align != 0 || (hi - lo) >= (1ull << 40))
    return false;
  const cuuint64_t dims[4] = {slab, rows, 2, cols / slab};
  const cuuint64_t strides[3] = {cols / slab * slab_bytes, hi - lo, slab_bytes};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(slab), box_rows, 2, box_slabs};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, elem_type(elem), 4,
             reinterpret_cast<void*>(lo), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Token-row maps of one source: 2-D boxes of 32 and 128 rows; 3-D boxes of
// 2-slab stages (32, 64, 96, 128 rows) and of 3-slab stages (32 rows).
// Rows of 256 bytes over a byte array of n_rows * 256 bytes (block scales);
// box = 256 bytes x box_rows, no swizzle.
bool make_map_rows256(CUtensorMap* m, const void* base, uint64_t n_rows, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {256, n_rows};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// E4M3 token-row maps of one source (3-D only).
bool make_token_maps_u8(TmaMaps* M, int src, const void* base, uint64_t rows, uint64_t cols) {
  for (int hb = 1; hb <= 4; ++hb)
    if (!make_map3(&M->b3[src][hb - 1], base, rows, cols, hb * kBoxRows, kSlabs, kElemU8))
      return false;
  return make_map3(&M->b3[src][4], base, rows, cols, kBoxRows, kSlabsLight, kElemU8);
}

bool make_token_maps(TmaMaps* M, int src, const void* base, uint64_t rows, uint64_t cols,
                     bool three_d) {
  if (!make_map(&M->b2[src][0], base, rows, cols, kBoxRows) ||
      !make_map(&M->b2[src][1], base, rows, cols, kBHalfMax))
    return false;
  if (!three_d) return true;
  for (int hb = 1; hb <= 4; ++hb)
    if (!make_map3(&M->b3[src][hb - 1], base, rows, cols, hb * kBoxRows, kSlabs)) return false;
  return make_map3(&M->b3[src][4], base, rows, cols, kBoxRows, kSlabsLight);
}

// The dynamic shared-memory limit of each kernel kind, raised once per device
// (a plain host call, kept out of stream capture after the first time).
template <int kKind>
cudaError_t ensure_smem_attr() {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? 1ull << dev : 0;
  if (bit && (done.load() & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<kKind>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           Kind<kKind>::kSmem);
  if (e == cudaSuccess && bit) done.fetch_or(bit);
  return e;
}

template <int kKind>
cudaError_t launch(const TmaMaps& maps, const GemmArgs& args, int grid, cudaStream_t st) {
  cudaError_t e = ensure_smem_attr<kKind>();
  if (e != cudaSuccess) return e;
  return launch_pdl(grouped_gemm_kernel<kKind>, dim3(grid), dim3(kThreads), Kind<kKind>::kSmem, st,
                    maps, args);
}

// Grid of whole CTA pairs: at most one pair per two SMs, at most max_pairs.
int pair_grid(int num_sms, int max_pairs) {
  int pairs = num_sms / 2;
  if (max_pairs > 0 && max_pairs < pairs) pairs = max_pairs;
  return 2 * (pairs > 0 ? pairs : 1);
}

// Diagnostic of the bounded wait: one thread waits, through the same slow path
// as the GEMM kernels, on a barrier that nothing ever arrives on.
__global__ void wait_selftest_kernel(int* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  mbar_wait_slow(&bar, 0, err, 99, limit_ns);
}

}  // namespace

cudaError_t launch_wait_selftest(int* err, uint64_t limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

cudaError_t prepare_grouped_gemm() {
  cudaError_t e = ensure_smem_attr<kKindUp>();
  if (e == cudaSuccess) e = ensure_smem_attr<kKindDown>();
  if (e == cudaSuccess) e = ensure_smem_attr<kKindLogits>();
  if (e == cudaSuccess) e = ensure_smem_attr<kKindUpF8>();
  if (e == cudaSuccess) e = ensure_smem_attr<kKindDownF8>();
  if (e == cudaSuccess && !get_encode_fn()) e = cudaErrorNotSupported;
  return e;
}

cudaError_t launch_experts_bf16(const Resolved& r, int64_t T, const Layout& L, char* ws,
                                const void* x, const void* wa, const void* wb, int num_sms,
                                cudaStream_t st, bool up) {
  const int NG = weight_slots(r);
  const int64_t R = T * (r.k + r.S);     // hidden rows
  const int64_t Rr = T * r.k;            // routed rows
  const int32_t* meta = reinterpret_cast<const int32_t*>(ws + L.meta);
  GemmArgs a{};
  a.chunks = reinterpret_cast<const Chunk*>(ws + L.chunks);
  a.implicit_rows = 0;
  a.n_routed_rows = (int)Rr;
  a.err = reinterpret_cast<int*>(ws + L.err);
  a.E = routed_slots(r);
  a.n_groups = NG;
  a.n_rows = R;
  a.max_chunks = (int)L.max_chunks;
  a.max_chunk_rows = kChunkRows;
  const int grid = pair_grid(num_sms, 0);
  TmaMaps M;
  memset(&M, 0, sizeof(M));
  if (up) {
    const uint64_t rows = (uint64_t)NG * r.I;
    if (!make_map(&M.a2[0], wa, rows, r.d, 64) || !make_map(&M.a2[1], wb, rows, r.d, 64) ||
        !make_token_maps(&M, 0, ws + L.xperm, Rr, r.d, false) ||
        !make_token_maps(&M, 1, x, T, r.d, false))
      return cudaErrorInvalidValue;
    bool w3_first = false;
    a.tma3d = make_map4_pair(&M.a3[0], wa, wb, rows, r.d, 64, kSlabs, &w3_first) &&
              make_map4_pair(&M.a3[1], wa, wb, rows, r.d, 64, kSlabsLight, &w3_first) &&
              make_token_maps(&M, 0, ws + L.xperm, Rr, r.d, true) &&
              make_token_maps(&M, 1, x, T, r.d, true);
    a.gate_hi = a.tma3d && w3_first;
    a.tiles = reinterpret_cast<const int2*>(ws + L.tiles_up);
    a.n_tiles = meta + 1;
    a.counter = const_cast<int32_t*>(meta) + 3;
    a.n_ftiles = (r.I + 127) / 128;
    a.rows_per_group = r.I;
    a.K = r.d;
    a.out_cols = r.I;
    a.ldo = r.I;
    a.out = ws + L.hidden;
    a.row_weight = nullptr;
    return launch<kKindUp>(M, a, grid, st);
  }
  const uint64_t rows = (uint64_t)NG * r.d;
  if (!make_map(&M.a2[0], wa, rows, r.I, kARowsCta) ||
      !make_token_maps(&M, 0, ws + L.hidden, R, r.I, false))
    return cudaErrorInvalidValue;
  a.tma3d = make_map3(&M.a3[0], wa, rows, r.I, kARowsCta, kSlabs) &&
            make_map3(&M.a3[1], wa, rows, r.I, kARowsCta, kSlabsLight) &&
            make_token_maps(&M, 0, ws + L.hidden, R, r.I, true);
  a.gate_hi = 0;
  a.tiles = reinterpret_cast<const int2*>(ws + L.tiles_down);
  a.n_tiles = meta + 2;
  a.counter = const_cast<int32_t*>(meta) + 4;
  a.n_ftiles = (r.d + 255) / 256;
  a.rows_per_group = r.d;
  a.K = r.I;
  a.out_cols = r.d;
  a.ldo = r.d;
  a.out = ws + L.expert_out;
  a.row_weight = reinterpret_cast<const float*>(ws + L.row_weight);
  return launch<kKindDown>(M, a, grid, st);
}

cudaError_t launch_experts_mxfp8(const Resolved& r, int64_t T, const Layout& L, char* ws,
                                 const void* wa, const void* wb, const uint8_t* sf, int num_sms,
                                 cudaStream_t st, bool up) {
  const int NG = weight_slots(r);
  const int64_t R = T * (r.k + r.S);     // hidden rows
  const int64_t Rr = T * r.k;            // routed rows
  const int32_t* meta = reinterpret_cast<const int32_t*>(ws + L.meta);
  GemmArgs a{};
  a.chunks = reinterpret_cast<const Chunk*>(ws + L.chunks);
  a.implicit_rows = 0;
  a.n_routed_rows = (int)Rr;
  a.err = reinterpret_cast<int*>(ws + L.err);
  a.E = routed_slots(r);
  a.n_groups = NG;
  a.n_rows = R;
  a.max_chunks = (int)L.max_chunks;
  a.max_chunk_rows = kChunkRowsF8;
  a.tma3d = 1;
  a.a_fp4 = r.w4;
  const int welem = r.w4 ? kElemFp4 : kElemU8;   // weight codes: E2M1 pairs or E4M3 bytes
  const int grid = pair_grid(num_sms, 0);
  TmaMaps M;
  memset(&M, 0, sizeof(M));
  if (up) {
    const uint64_t rows = (uint64_t)NG * r.I;
    const uint64_t sfb_rows = (uint64_t)L.max_chunks * (r.d / 128) * 4;
    bool w3_first = false;
    if (!make_map4_pair(&M.a3[0], wa, wb, rows, r.d, 64, kSlabs, &w3_first, welem) ||
        !make_map4_pair(&M.a3[1], wa, wb, rows, r.d, 64, kSlabsLight, &w3_first, welem) ||
        !make_token_maps_u8(&M, 0, ws + L.xperm, Rr, r.d) ||
        !make_token_maps_u8(&M, 1, ws + L.xq, T, r.d) ||
        !make_map_rows256(&M.sfa[0], sf, mx_packed_bytes(r, false) / 256, 2 * kSlabs) ||
        !make_map_rows256(&M.sfa[1], sf, mx_packed_bytes(r, false) / 256, 2 * kSlabsLight) ||
        !make_map_rows256(&M.sfb[0], ws + L.tok_sf, sfb_rows, 4 * kSlabs) ||
        !make_map_rows256(&M.sfb[1], ws + L.tok_sf, sfb_rows, 4 * kSlabsLight))
      return cudaErrorInvalidValue;
    if (w3_first) return cudaErrorInvalidValue;   // the packed scales list W1 first
    a.gate_hi = 0;
    a.n_kslabs = r.d / 128;
    a.n_ftiles_sf = r.I / 128;
    a.hid_sf = reinterpret_cast<uint8_t*>(ws + L.hid_sf);
    a.tiles = reinterpret_cast<const int2*>(ws + L.tiles_up);
    a.n_tiles = meta + 1;
    a.counter = const_cast<int32_t*>(meta) + 3;
    a.n_ftiles = r.I / 128;
    a.rows_per_group = r.I;
    a.K = r.d;
    a.out_cols = r.I;
    a.ldo = r.I;
    a.out = ws + L.hidden;
    a.row_weight = nullptr;
    return launch<kKindUpF8>(M, a, grid, st);
  }
  const uint64_t rows = (uint64_t)NG * r.d;
  const uint64_t sfb_rows = (uint64_t)L.max_chunks * (r.I / 128) * 4;
  if (!make_map3(&M.a3[0], wa, rows, r.I, kARowsCta, kSlabs, welem) ||
      !make_map3(&M.a3[1], wa, rows, r.I, kARowsCta, kSlabsLight, welem) ||
      !make_token_maps_u8(&M, 0, ws + L.hidden, R, r.I) ||
      !make_map_rows256(&M.sfa[0], sf, mx_packed_bytes(r, true) / 256, 2 * kSlabs) ||
      !make_map_rows256(&M.sfa[1], sf, mx_packed_bytes(r, true) / 256, 2 * kSlabsLight) ||
      !make_map_rows256(&M.sfb[0], ws + L.hid_sf, sfb_rows, 4 * kSlabs) ||
      !make_map_rows256(&M.sfb[1], ws + L.hid_sf, sfb_rows, 4 * kSlabsLight))
    return cudaErrorInvalidValue;
  a.gate_hi = 0;
  a.n_kslabs = r.I / 128;
  a.n_ftiles_sf = (r.d + 255) / 256;
  a.hid_sf = nullptr;
  a.tiles = reinterpret_cast<const int2*>(ws + L.tiles_down);
  a.n_tiles = meta + 2;
  a.counter = const_cast<int32_t*>(meta) + 4;
  a.n_ftiles = (r.d + 255) / 256;
  a.rows_per_group = r.d;
  a.K = r.I;
  a.out_cols = r.d;
  a.ldo = r.d;
  a.out = ws + L.expert_out;
  a.row_weight = reinterpret_cast<const float*>(ws + L.row_weight);
  return launch<kKindDownF8>(M, a, grid, st);
}

cudaError_t launch_gate_logits_tc(const Resolved& r, int64_t T, const void* x, const void* w_gate,
                                  float* logits, int* err, int num_sms, cudaStream_t st) {
  TmaMaps M;
  memset(&M, 0, sizeof(M));
  if (!make_map(&M.a2[0], w_gate, (uint64_t)r.E, r.d, kARowsCta) ||
      !make_token_maps(&M, 0, x, T, r.d, false))
    return cudaErrorInvalidValue;
  GemmArgs a{};
  a.tma3d = make_map3(&M.a3[0], w_gate, (uint64_t)r.E, r.d, kARowsCta, kSlabs) &&
            make_map3(&M.a3[1], w_gate, (uint64_t)r.E, r.d, kARowsCta, kSlabsLight) &&
            make_token_maps(&M, 0, x, T, r.d, true);
  a.gate_hi = 0;
  a.chunks = nullptr;
  a.tiles = nullptr;
  a.n_tiles = nullptr;
  a.counter = nullptr;
  a.implicit_rows = (int)T;
  a.n_ftiles = (r.E + 255) / 256;
  a.rows_per_group = r.E;
  a.K = r.d;
  a.E = 1;                  // every chunk reads its token rows from source 0
  a.out_cols = r.E;
  a.ldo = r.E;
  a.out = logits;
  a.row_weight = nullptr;
  a.n_routed_rows = 0;
  a.err = err;
  // Token chunks of 256 rows, halved (down to 64) while twice the tiles still
  // fit in one wave of CTA pairs: W_g is small and stays in L2, so narrower
  // tiles cost little more traffic and spread the logits over more of the GPU.
  const int64_t n_pairs = num_sms / 2;
  int chunk = kChunkRows;
  while (chunk > 64 && 2 * ((T + chunk - 1) / chunk) * a.n_ftiles <= n_pairs) chunk /= 2;
  a.implicit_chunk = chunk;
  const int tiles = (int)((T + chunk - 1) / chunk) * a.n_ftiles;
  return launch<kKindLogits>(M, a, pair_grid(num_sms, tiles), st);
}

}  // namespace ktmoe
