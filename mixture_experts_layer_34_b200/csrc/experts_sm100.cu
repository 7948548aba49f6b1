// Routed + shared expert SwiGLU FFNs on the sm_100a tensor cores.
//
// The expert FFN of the total-output equation in the "DeepSeekMoE 三改进"
// passage of the DeepSeek-V3 model.py notes (73biji.xyz/llm_pp_dsv3),
//     FFN_e(u) = W2_e (silu(W1_e u) * W3_e u),
// runs as two grouped GEMMs over the expert-sorted token rows:
//   up   : hidden[r, f]     = silu(<W1_e[f], u_r>) * <W3_e[f], u_r>
//   down : expert_out[r, o] = w_r * <W2_e[o], hidden[r]>   (fp32, so the
//          combine sums unrounded terms)
// with w_r the routing weight of row r (1 for shared-expert rows), as in the
// "y[idx] += expert(x[idx]) * w" loop of "MoE 前向四步".
//
// Design (one persistent CTA per SM, 192 threads):
//   warp 0     TMA producer: weight tile (128 rows x 64 K) and the token-row
//              tile (N rows x 64 K, in 16-row boxes) into a 4-stage ring;
//   warp 1     allocates 512 TMEM columns; lane 0 issues tcgen05.mma
//              (kind::f16, bf16 in, fp32 accumulate) and tcgen05.commit;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator, SwiGLU (up) or the
//              routing weight (down), store through a shared staging tile.
// Operands are swapped relative to the math (D^T = W X^T): the weight tile is
// the M = 128 operand and the tokens of the chunk are N (a multiple of 16 up to
// 128 for up, 256 for down), so an expert with few tokens costs an MMA of
// matching width instead of a 128-row tile of padding. Two accumulators (gate
// and up) per tile for the up GEMM; two TMEM buffers so the epilogue of one tile
// overlaps the main loop of the next.
//
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the
// kernel records KT_ERR_TIMEOUT in the workspace error word, drains what it
// issued, frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

constexpr int kStages = 4;
constexpr int kBK = 64;                      // K elements per stage (128 B of bf16)
constexpr int kATileBytes = kWRows * kBK * 2;  // 16 KB
constexpr int kBoxRows = 16;                 // token rows per TMA box
constexpr int kThreads = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Epilogue kinds of the grouped GEMM.
constexpr int kKindUp = 0;      // hidden = silu(W1 u) * W3 u          (bf16 out)
constexpr int kKindDown = 1;    // expert_out = w_r * W2 h             (fp32 out)
constexpr int kKindLogits = 2;  // logits = W_g u, one group, implicit token chunks (fp32 out)

template <int kKind>
struct Cfg {
  static constexpr bool kUp = kKind == kKindUp;
  static constexpr int kNumA = kUp ? 2 : 1;
  static constexpr int kMaxN = kKind == kKindDown ? kDownChunk : kUpChunk;
  static constexpr int kBBytes = kMaxN * kBK * 2;
  static constexpr int kStageBytes = kNumA * kATileBytes + kBBytes;
  static constexpr int kAccCols = 256;       // TMEM columns per accumulator buffer
  static constexpr int kOutBytes = kUp ? 2 : 4;   // bf16 hidden rows / fp32 expert outputs
  static constexpr int kStagingBytes = 4 * 16 * 32 * 4;
  static constexpr int kSmemBytes = kStages * kStageBytes + kStagingBytes + 256 + 1024;
};

struct GemmArgs {
  const Chunk* chunks;
  const int32_t* n_chunks;   // device: number of chunks
  int implicit_rows;         // > 0: no chunk list; chunks of kMaxN rows over this many rows of group 0
  int n_ftiles;              // weight-row tiles per group
  int rows_per_group;        // weight rows per expert (I for up, d for down)
  int K;                     // reduction length (d for up, I for down)
  int E;                     // routed experts (up: groups >= E read x directly)
  int out_cols;              // valid output columns (I or d)
  int ldo;                   // output row stride in elements
  void* out;                 // up: bf16 hidden rows; down: fp32 weighted expert outputs
  const float* row_weight;   // down: weight of routed rows
  int n_routed_rows;         // T * k
  int* err;
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait. Returns false (after recording the timeout) if the phase did not
// complete within kWaitLimitNs, or if another CTA already recorded an error.
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* err, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*reinterpret_cast<volatile int*>(err) != 0) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        set_error(err, kDevErrTimeout, where);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
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
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
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
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
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

__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

template <int kKind>
__device__ __forceinline__ Chunk get_chunk(const GemmArgs& a, int ci) {
  if (a.implicit_rows > 0) {
    constexpr int n = Cfg<kKind>::kMaxN;
    return Chunk{0, ci * n, min(n, a.implicit_rows - ci * n), ci * n};
  }
  return a.chunks[ci];
}

// ---------------------------------------------------------------------------
// The grouped GEMM kernel
// ---------------------------------------------------------------------------
template <int kKind>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA0,   // W1 (up) or W2 (down)
                    const __grid_constant__ CUtensorMap tmA1,   // W3 (up)
                    const __grid_constant__ CUtensorMap tmB0,   // permuted x (up) or hidden (down)
                    const __grid_constant__ CUtensorMap tmB1,   // x (up, shared experts)
                    const GemmArgs args) {
  using C = Cfg<kKind>;
  constexpr bool kUp = C::kUp;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stage_base = smem;
  uint8_t* staging = smem + kStages * C::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * C::kStageBytes + C::kStagingBytes);
  uint64_t* full_bar = bars;                    // [kStages]
  uint64_t* empty_bar = bars + kStages;         // [kStages]
  uint64_t* tfull_bar = bars + 2 * kStages;     // [2]
  uint64_t* tempty_bar = bars + 2 * kStages + 2;  // [2]
  uint64_t* drain_bar = bars + 2 * kStages + 4;   // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 4);
    }
    mbar_init(drain_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tmA0);
    prefetch_tmap(&tmB0);
    if (kUp) {
      prefetch_tmap(&tmA1);
      prefetch_tmap(&tmB1);
    }
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int n_chunks = args.implicit_rows > 0 ? (args.implicit_rows + C::kMaxN - 1) / C::kMaxN
                                              : *args.n_chunks;
  const int n_tiles = n_chunks * args.n_ftiles;
  const int nk = (args.K + kBK - 1) / kBK;
  int* err = args.err;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;   // loads issued and not yet known complete (drained on error)
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const Chunk ch = get_chunk<kKind>(args, tile / args.n_ftiles);
        const int ft = tile % args.n_ftiles;
        const int nb = (ch.nrows + kBoxRows - 1) & ~(kBoxRows - 1);
        const int a_row = ch.group * args.rows_per_group + ft * kWRows;
        const CUtensorMap* bmap = &tmB0;
        int b_row = ch.row0;
        if (kUp) {
          b_row = ch.src_row0;
          if (ch.group >= args.E) bmap = &tmB1;
        }
        const uint32_t tx = C::kNumA * kATileBytes + nb * kBK * 2;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u, err, 1 + 8 * kKind)) {
            ok = false;
            break;
          }
          uint8_t* sb = stage_base + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full_bar[stage], tx);
          tma_load_2d(sb, &tmA0, &full_bar[stage], kb * kBK, a_row);
          if (kUp) tma_load_2d(sb + kATileBytes, &tmA1, &full_bar[stage], kb * kBK, a_row);
          uint8_t* sB = sb + C::kNumA * kATileBytes;
          for (int rr = 0; rr < nb; rr += kBoxRows)
            tma_load_2d(sB + rr * kBK * 2, bmap, &full_bar[stage], kb * kBK, b_row + rr);
          issued = issued < kStages ? issued + 1 : kStages;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA can exit: wait
        // (bounded) on the full barrier of each of the last `issued` stages.
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
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t bphase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const Chunk ch = get_chunk<kKind>(args, tile / args.n_ftiles);
        const int nb = (ch.nrows + kBoxRows - 1) & ~(kBoxRows - 1);
        if (!mbar_wait(&tempty_bar[buf], bphase ^ 1u, err, 2 + 8 * kKind)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(kWRows, nb);
        const uint32_t d0 = tmem_base + buf * C::kAccCols;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full_bar[stage], phase, err, 3 + 8 * kKind)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(stage_base + stage * C::kStageBytes);
          const uint32_t sB = sb + C::kNumA * kATileBytes;
#pragma unroll
          for (int ks = 0; ks < kBK / 16; ++ks) {
            const uint64_t bdesc = sw128_desc(sB + ks * 32);
            const uint32_t acc = (kb | ks) != 0;
            mma_bf16(d0, sw128_desc(sb + ks * 32), bdesc, idesc, acc);
            if (kUp) mma_bf16(d0 + 128, sw128_desc(sb + kATileBytes + ks * 32), bdesc, idesc, acc);
          }
          mma_commit(&empty_bar[stage]);
          issued_any = true;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&tfull_bar[buf]);
        if (++buf == 2) {
          buf = 0;
          bphase ^= 1u;
        }
      }
      // Wait (bounded) until every MMA this thread issued has completed, so TMEM
      // and shared memory can be released.
      if (issued_any) {
        mma_commit(drain_bar);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(drain_bar, 0) && globaltimer() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ---------------- Epilogue (warps 2..5) ----------------
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    uint8_t* stg = staging + (warp - 2) * 16 * 32 * 4;
    int buf = 0;
    uint32_t bphase = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const Chunk ch = get_chunk<kKind>(args, tile / args.n_ftiles);
      const int ft = tile % args.n_ftiles;
      const int nb = (ch.nrows + kBoxRows - 1) & ~(kBoxRows - 1);
      // The outcome must be warp-uniform: tcgen05.ld below is .sync.aligned.
      const bool ready = mbar_wait(&tfull_bar[buf], bphase, err, 4 + 8 * kKind);
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * C::kAccCols;
      const int col0 = ft * kWRows + q * 32;   // first output column of this warp
      for (int c0 = 0; c0 < nb; c0 += 16) {
        float h[16];
        if (kUp) {
          float g[16], u[16];
          tmem_ld16(tbase + c0, g);
          tmem_ld16(tbase + 128 + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) h[i] = silu(g[i]) * u[i];
        } else {
          tmem_ld16(tbase + c0, h);
          tmem_ld_wait();
          if (kKind == kKindDown) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int row = ch.row0 + c0 + i;
              const float wr = row < args.n_routed_rows ? args.row_weight[row] : 1.0f;
              h[i] *= wr;
            }
          }
        }
        // Transpose through shared memory: stg[token][feature], then 16-byte
        // stores along each output row (32 features = 64 B bf16 / 128 B fp32).
        if (kUp) {
          __nv_bfloat16* sb = reinterpret_cast<__nv_bfloat16*>(stg);
#pragma unroll
          for (int i = 0; i < 16; ++i) sb[i * 32 + lane] = __float2bfloat16_rn(h[i]);
        } else {
          float* sf = reinterpret_cast<float*>(stg);
#pragma unroll
          for (int i = 0; i < 16; ++i) sf[i * 32 + lane] = h[i];
        }
        __syncwarp();
        constexpr int kChunksPerRow = 32 * C::kOutBytes / 16;
        constexpr int kElemsPerChunk = 16 / C::kOutBytes;
#pragma unroll
        for (int it = 0; it < 16 * kChunksPerRow / 32; ++it) {
          const int idx = lane + it * 32;
          const int rr = idx / kChunksPerRow, part = idx % kChunksPerRow;
          const int c = c0 + rr;
          const int col = col0 + part * kElemsPerChunk;
          if (c < ch.nrows && col < args.out_cols) {
            const uint4 v = *reinterpret_cast<const uint4*>(stg + rr * 32 * C::kOutBytes + part * 16);
            *reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                      ((int64_t)(ch.row0 + c) * args.ldo + col) * C::kOutBytes) = v;
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[buf]);
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, 512);
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

template <int kKind>
cudaError_t set_smem_attr() {
  return cudaFuncSetAttribute(grouped_gemm_kernel<kKind>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<kKind>::kSmemBytes);
}

}  // namespace

cudaError_t launch_experts_bf16(const Resolved& r, int64_t T, const Layout& L, char* ws,
                                const void* x, const void* wa, const void* wb, int num_sms,
                                cudaStream_t st, bool up) {
  const int NG = r.E + r.S;
  const int64_t R = T * (r.k + r.S);     // hidden rows
  const int64_t Rr = T * r.k;            // routed rows
  int32_t* meta = reinterpret_cast<int32_t*>(ws + L.meta);
  int* err = reinterpret_cast<int*>(ws + L.err);
  GemmArgs a{};
  a.n_routed_rows = (int)Rr;
  a.err = err;
  a.E = r.E;
  if (up) {
    CUtensorMap mW1, mW3, mXp, mX;
    if (!make_map(&mW1, wa, (uint64_t)NG * r.I, r.d, kWRows) ||
        !make_map(&mW3, wb, (uint64_t)NG * r.I, r.d, kWRows) ||
        !make_map(&mXp, ws + L.xperm, Rr, r.d, kBoxRows) || !make_map(&mX, x, T, r.d, kBoxRows))
      return cudaErrorInvalidValue;
    cudaError_t e = set_smem_attr<kKindUp>();
    if (e != cudaSuccess) return e;
    a.chunks = reinterpret_cast<const Chunk*>(ws + L.up_chunks);
    a.n_chunks = meta + 0;
    a.n_ftiles = (r.I + kWRows - 1) / kWRows;
    a.rows_per_group = r.I;
    a.K = r.d;
    a.out_cols = r.I;
    a.ldo = r.I;
    a.out = ws + L.hidden;
    a.row_weight = nullptr;
    grouped_gemm_kernel<kKindUp><<<num_sms, kThreads, Cfg<kKindUp>::kSmemBytes, st>>>(mW1, mW3, mXp, mX, a);
  } else {
    CUtensorMap mW2, mH;
    if (!make_map(&mW2, wa, (uint64_t)NG * r.d, r.I, kWRows) ||
        !make_map(&mH, ws + L.hidden, R, r.I, kBoxRows))
      return cudaErrorInvalidValue;
    cudaError_t e = set_smem_attr<kKindDown>();
    if (e != cudaSuccess) return e;
    a.chunks = reinterpret_cast<const Chunk*>(ws + L.down_chunks);
    a.n_chunks = meta + 1;
    a.n_ftiles = (r.d + kWRows - 1) / kWRows;
    a.rows_per_group = r.d;
    a.K = r.I;
    a.out_cols = r.d;
    a.ldo = r.d;
    a.out = ws + L.expert_out;
    a.row_weight = reinterpret_cast<const float*>(ws + L.row_weight);
    grouped_gemm_kernel<kKindDown><<<num_sms, kThreads, Cfg<kKindDown>::kSmemBytes, st>>>(mW2, mW2, mH, mH, a);
  }
  return cudaGetLastError();
}

cudaError_t launch_gate_logits_tc(const Resolved& r, int64_t T, const void* x, const void* w_gate,
                                  float* logits, int* err, int num_sms, cudaStream_t st) {
  CUtensorMap mWg, mX;
  if (!make_map(&mWg, w_gate, (uint64_t)r.E, r.d, kWRows) || !make_map(&mX, x, T, r.d, kBoxRows))
    return cudaErrorInvalidValue;
  cudaError_t e = set_smem_attr<kKindLogits>();
  if (e != cudaSuccess) return e;
  GemmArgs a{};
  a.chunks = nullptr;
  a.n_chunks = nullptr;
  a.implicit_rows = (int)T;
  a.n_ftiles = (r.E + kWRows - 1) / kWRows;
  a.rows_per_group = r.E;
  a.K = r.d;
  a.E = 1;                  // every chunk reads its token rows from the first B map
  a.out_cols = r.E;
  a.ldo = r.E;
  a.out = logits;
  a.row_weight = nullptr;
  a.n_routed_rows = 0;
  a.err = err;
  const int tiles = (int)((T + kUpChunk - 1) / kUpChunk) * a.n_ftiles;
  const int grid = tiles < num_sms ? tiles : num_sms;
  grouped_gemm_kernel<kKindLogits><<<grid, kThreads, Cfg<kKindLogits>::kSmemBytes, st>>>(
      mWg, mWg, mX, mX, a);
  return cudaGetLastError();
}

}  // namespace ktmoe
