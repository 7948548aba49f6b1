// Gate of the DeepSeekMoE layer: logits, score function and the group-limited
// top-k selection. Follows "Gate 选专家流程（model.py，五步）" of the DeepSeek-V3
// model.py notes (73biji.xyz/llm_pp_dsv3) and the bias rule of its
// "V3 改进①：无辅助损失负载均衡" section.
//
//   logits             : l = u W_g^T with fp32 accumulation. bf16 layers with
//                        more than 64 tokens use the tcgen05 grouped GEMM
//                        (experts_sm100.cu); otherwise gate_logits_small_kernel
//                        (one warp per expert, for few tokens) or the
//                        register-tiled gate_logits_kernel (fp32 layers).
//   gate_select_kernel : one warp per token; scores, keys s + b, group scores,
//                        top topk_groups groups, top-k experts, weights. Each
//                        CTA covers one 32-token chunk and also writes that
//                        chunk's per-expert counts for the token permutation.
#include <cuda_bf16.h>

#include <cmath>

#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

// ---------------------------------------------------------------------------
// Logits: CTA tile 64 tokens x 128 experts, 128 threads, 8x8 outputs per
// thread (rows ty*4+{0..3} and 32+ty*4+{0..3}; experts tx*4+{0..3} and
// 64+tx*4+{0..3}), K slab of 32 staged in shared memory k-major.
// ---------------------------------------------------------------------------
constexpr int kLT = 64, kLE = 128, kLK = 32, kLThreads = 128;

template <typename T>
struct Vec16;  // 16-byte chunk of T
template <>
struct Vec16<float> {
  static constexpr int n = 4;
  __device__ static void load(const float* p, float* out) {
    float4 v = *reinterpret_cast<const float4*>(p);
    out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void load(const __nv_bfloat16* p, float* out) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      out[2 * i] = __uint_as_float(w[i] << 16);
      out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

// Load a [rows x kLK] slab (row-major source, leading dim ld) into s[k][row]
// (k-major), zero-filling rows >= nrows and columns >= ncols.
template <typename T, int ROWS>
__device__ __forceinline__ void load_slab(const T* src, int64_t ld, int nrows, int ncols, int k0,
                                          float (*s)[ROWS + 4]) {
  constexpr int VN = Vec16<T>::n;
  constexpr int chunks_per_row = kLK / VN;
  constexpr int total = ROWS * chunks_per_row;
  for (int c = threadIdx.x; c < total; c += kLThreads) {
    const int row = c / chunks_per_row;
    const int kk = (c % chunks_per_row) * VN;
    float v[VN];
    if (row < nrows && k0 + kk < ncols) {
      Vec16<T>::load(src + (int64_t)row * ld + k0 + kk, v);
    } else {
#pragma unroll
      for (int i = 0; i < VN; ++i) v[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < VN; ++i) s[kk + i][row] = v[i];
  }
}

template <typename T>
__global__ void __launch_bounds__(kLThreads)
gate_logits_kernel(const T* __restrict__ x, const T* __restrict__ wg, float* __restrict__ logits,
                   int T_, int E, int d) {
  pdl_wait();
  __shared__ float xs[kLK][kLT + 4];
  __shared__ float ws[kLK][kLE + 4];
  const int e0 = blockIdx.x * kLE;
  const int t0 = blockIdx.y * kLT;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const T* xb = x + (int64_t)t0 * d;
  const T* wb = wg + (int64_t)e0 * d;
  for (int k0 = 0; k0 < d; k0 += kLK) {
    load_slab<T, kLT>(xb, d, T_ - t0, d, k0, xs);
    load_slab<T, kLE>(wb, d, E - e0, d, k0, ws);
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kLK; ++kk) {
      float a[8], b[8];
      *reinterpret_cast<float4*>(a) = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      *reinterpret_cast<float4*>(a + 4) = *reinterpret_cast<const float4*>(&xs[kk][32 + ty * 4]);
      *reinterpret_cast<float4*>(b) = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
      *reinterpret_cast<float4*>(b + 4) = *reinterpret_cast<const float4*>(&ws[kk][64 + tx * 4]);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + (i < 4 ? ty * 4 + i : 32 + ty * 4 + (i - 4));
    if (t >= T_) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = e0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (e < E) logits[(int64_t)t * E + e] = acc[i][j];
    }
  }
}

// ---------------------------------------------------------------------------
// Logits for few tokens (T <= 64), split over K: CTA (eb, ks) computes the
// partial dot products of 32 experts over the ks-th K range for all tokens
// (one warp per 4 experts computed together, 16-byte loads along K split over
// the lanes, 8 tokens at a time) and writes them to part[ks][t][e]. The last of
// an expert block's kSplitK CTAs to finish (a counter in the workspace, zeroed
// at the start of every call) adds the partials in ks order and writes the sum
// over part[0]: the result does not depend on scheduling, and the selection
// reads one value per logit.
// ---------------------------------------------------------------------------
constexpr int kSmallWarps = 8, kSmallTok = 8, kSplitK = kGateSplitK;

template <typename T>
__global__ void __launch_bounds__(kSmallWarps * 32)
gate_logits_splitk_kernel(const T* __restrict__ x, const T* __restrict__ wg,
                          float* __restrict__ part, int T_, int E, int d, int kc,
                          int* __restrict__ block_done) {
  pdl_wait();
  constexpr int VN = Vec16<T>::n, EW = 4;  // experts per warp, computed together
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ks = blockIdx.y;
  const int k0 = ks * kc, k1 = min(d, k0 + kc);
  const int nc = k1 > k0 ? (k1 - k0) / VN : 0;
  const int e0 = blockIdx.x * 32 + warp * EW;
  for (int t0 = 0; e0 < E && t0 < T_; t0 += kSmallTok) {
    float acc[EW][kSmallTok];
#pragma unroll
    for (int ei = 0; ei < EW; ++ei)
#pragma unroll
      for (int j = 0; j < kSmallTok; ++j) acc[ei][j] = 0.f;
    for (int c = lane; c < nc; c += 32) {
      float wv[EW][VN];
#pragma unroll
      for (int ei = 0; ei < EW; ++ei) {
        if (e0 + ei < E) {
          Vec16<T>::load(wg + (int64_t)(e0 + ei) * d + k0 + c * VN, wv[ei]);
        } else {
#pragma unroll
          for (int i = 0; i < VN; ++i) wv[ei][i] = 0.f;
        }
      }
#pragma unroll
      for (int j = 0; j < kSmallTok; ++j) {
        if (t0 + j < T_) {
          float xv[VN];
          Vec16<T>::load(x + (int64_t)(t0 + j) * d + k0 + c * VN, xv);
#pragma unroll
          for (int ei = 0; ei < EW; ++ei)
#pragma unroll
            for (int i = 0; i < VN; ++i) acc[ei][j] = fmaf(wv[ei][i], xv[i], acc[ei][j]);
        }
      }
    }
#pragma unroll
    for (int ei = 0; ei < EW; ++ei)
#pragma unroll
      for (int j = 0; j < kSmallTok; ++j) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          acc[ei][j] += __shfl_xor_sync(0xffffffffu, acc[ei][j], off);
        if (lane == 0 && t0 + j < T_ && e0 + ei < E)
          part[((int64_t)ks * T_ + t0 + j) * E + e0 + ei] = acc[ei][j];
      }
  }
  // The last CTA of this expert block sums the partials.
  __shared__ int last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&block_done[blockIdx.x], 1) == (int)gridDim.y - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  const int eb0 = blockIdx.x * 32;
  for (int i = threadIdx.x; i < T_ * 32; i += blockDim.x) {
    const int t = i / 32, e = eb0 + i % 32;
    if (e >= E) continue;
    float sum = __ldcg(&part[(int64_t)t * E + e]);
    for (int q = 1; q < (int)gridDim.y; ++q) sum += __ldcg(&part[((int64_t)q * T_ + t) * E + e]);
    part[(int64_t)t * E + e] = sum;
  }
}

// ---------------------------------------------------------------------------
// Selection: 8 warps per CTA, 4 tokens per warp, 32 tokens per CTA.
// Lane l holds experts e = i*32 + l, i < ceil(E/32) (at most 16).
// ---------------------------------------------------------------------------
constexpr int kSelWarps = 8;
constexpr unsigned kFull = 0xffffffffu;

// Keys as order-preserving unsigned integers, so that a warp's maximum is one
// redux.sync: ord(a) < ord(b) iff a < b for non-NaN fp32 a, b (-0 and +0 map
// to the same value, as they compare equal). 0 lies below every key and marks
// "no candidate" (an expert already taken).
__device__ __forceinline__ uint32_t ord_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) == 0) b = 0;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_of(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
// Warp argmax over one (key, index) candidate per lane: the largest key, and
// among equal keys the lowest index (the tie rule of both top-k's). Returns the
// index; `best` gets the key.
__device__ __forceinline__ int warp_argmax(uint32_t u, int idx, uint32_t& best) {
  best = __reduce_max_sync(kFull, u);
  return (int)__reduce_min_sync(kFull, u == best ? (unsigned)idx : 0xffffffffu);
}

// Gate step 1 and the score function for token t, one warp: lane l gets the
// scores of experts i * 32 + l in s[i], from the logits (or, if `scores_in` is
// given, those scores as they are). Lanes past E hold -inf (scores_in), 0
// (sigmoid of -inf) or 0 (softmax).
template <int NP>
__device__ __forceinline__ void token_scores(const Resolved& r, const float* __restrict__ logits,
                                             const float* __restrict__ scores_in, int t, int lane,
                                             float (&s)[NP]) {
  const int E = r.E;
  const float NEG_INF = -INFINITY;
  const float* row = (scores_in ? scores_in : logits) + (int64_t)t * E;
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const int e = i * 32 + lane;
    s[i] = e < E ? row[e] : NEG_INF;
  }
  if (!scores_in) {
    if (r.score_func == KT_SCORE_SIGMOID) {
#pragma unroll
      for (int i = 0; i < NP; ++i)
        s[i] = 1.0f / (1.0f + expf(-s[i]));
    } else {
      float m = NEG_INF;
#pragma unroll
      for (int i = 0; i < NP; ++i)
        m = fmaxf(m, s[i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
      float z = 0.f;
#pragma unroll
      for (int i = 0; i < NP; ++i)
        {
          s[i] = (i * 32 + lane < E) ? expf(s[i] - m) : 0.f;
          z += s[i];
        }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(kFull, z, off);
#pragma unroll
      for (int i = 0; i < NP; ++i)
        s[i] = __fdiv_rn(s[i], z);
    }
  }
}

// NP = experts per lane (E <= 32 * NP), a compile-time bound so the per-lane
// arrays stay in registers.
template <int NP>
__global__ void __launch_bounds__(kSelWarps * 32)
gate_select_kernel(Resolved r, int T_, const float* __restrict__ logits,
                   const float* __restrict__ scores_in, const float* __restrict__ bias,
                   int32_t* __restrict__ out_idx, float* __restrict__ out_w,
                   int32_t* __restrict__ chunk_counts, int* __restrict__ err) {
  pdl_wait();
  __shared__ int scount[kMaxExperts];
  __shared__ float skey[kSelWarps][kMaxExperts];
  const int E = r.E, k = r.k, G = r.G, gs = r.gs;
  for (int e = threadIdx.x; e < E; e += blockDim.x) scount[e] = 0;
  __syncthreads();

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const float NEG_INF = -INFINITY;
  // Tokens interleave over the warps, so a chunk of fewer than 32 tokens (a
  // decode step) still keeps every warp busy.
  for (int tt = 0; tt < kPermChunk / kSelWarps; ++tt) {
    const int t = blockIdx.x * kPermChunk + tt * kSelWarps + warp;
    if (t >= T_) break;
    // Step 1: scores (kept raw for step 5).
    float s[NP];
    token_scores<NP>(r, logits, scores_in, t, lane, s);
    // Step 2a: selection keys s + b (the bias takes part in the selection only),
    // as ordered integers (NaN keys count as -inf: indices stay valid).
    const uint32_t kNegInf = ord_key(NEG_INF);
    uint32_t ku[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int e = i * 32 + lane;
      if (e < E) {
        const float kv = r.has_bias ? __fadd_rn(s[i], bias[e]) : s[i];
        ku[i] = kv != kv ? kNegInf : ord_key(kv);
      } else {
        ku[i] = 0;
      }
    }
    // Steps 2b-3: group scores, keep topk_groups groups, mask the rest.
    if (G > 1) {
      // Group score of group g in lane g: the group max (no bias) or the sum
      // of its two largest keys, larger first (bias).
      float gsc = NEG_INF;
      const bool top2 = r.group_score == KT_GROUP_TOP2SUM;
      if (gs == 32) {
        // Group g is slot g of every lane: warp reductions.
#pragma unroll
        for (int g = 0; g < NP; ++g) {
          if (g >= G) break;
          const uint32_t m1 = __reduce_max_sync(kFull, ku[g]);
          float v = key_of(m1);
          if (top2) {
            const bool dup = __popc(__ballot_sync(kFull, ku[g] == m1)) > 1;
            const uint32_t m2 = dup ? m1 : __reduce_max_sync(kFull, ku[g] == m1 ? 0u : ku[g]);
            v = __fadd_rn(v, key_of(m2));
          }
          if (lane == g) gsc = v;
        }
      } else {
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          const int e = i * 32 + lane;
          if (e < E) skey[warp][e] = key_of(ku[i]);
        }
        __syncwarp();
        if (lane < G) {
          const float* kg = &skey[warp][lane * gs];
          if (top2) {
            float b1 = NEG_INF, b2 = NEG_INF;
            for (int i = 0; i < gs; ++i) {
              const float v = kg[i];
              if (v > b1) {
                b2 = b1;
                b1 = v;
              } else if (v > b2) {
                b2 = v;
              }
            }
            gsc = __fadd_rn(b1, b2);
          } else {
            for (int i = 0; i < gs; ++i) gsc = fmaxf(gsc, kg[i]);
          }
        }
        __syncwarp();
      }
      unsigned kept = 0;
      uint32_t gu = lane < G ? ord_key(gsc != gsc ? NEG_INF : gsc) : 0u;
      for (int rr = 0; rr < r.TG; ++rr) {
        uint32_t best;
        const int g = warp_argmax(gu, lane, best);
        kept |= 1u << g;
        if (lane == g) gu = 0;
      }
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        const int e = i * 32 + lane;
        if (e < E && !((kept >> (e / gs)) & 1u)) ku[i] = kNegInf;
      }
    }
    // Step 4: global top-k over the masked keys; lane j keeps slot j.
    int my_e = 0;
    float my_s = 0.f;
    for (int j = 0; j < k; ++j) {
      // this lane's best key (strict > keeps the lowest index among equals)
      uint32_t lu = 0;
      int li = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < NP; ++i)
        if (ku[i] > lu) {
          lu = ku[i];
          li = i * 32 + lane;
        }
      uint32_t best;
      const int b = warp_argmax(lu, li, best);
      float won_s = 0.f;
      if (lane == (b & 31)) {
#pragma unroll
        for (int i = 0; i < NP; ++i)
          if (i == (b >> 5)) {
            won_s = s[i];
            ku[i] = 0;                  // taken: never wins again
          }
      }
      won_s = __shfl_sync(kFull, won_s, b & 31);
      if (lane == j) {
        my_e = b;
        my_s = won_s;
      }
    }
    // Step 5: gather raw scores, renormalise (slot order), times route_scale.
    float sum = 0.f;
    for (int j = 0; j < k; ++j) sum = __fadd_rn(sum, __shfl_sync(kFull, my_s, j));
    if (lane < k) {
      float wv = r.norm ? __fdiv_rn(my_s, sum) : my_s;
      wv = __fmul_rn(wv, r.route_scale);
      out_idx[(int64_t)t * k + lane] = my_e;
      out_w[(int64_t)t * k + lane] = wv;
      if (in_range(my_e, 0, E, err, 161)) atomicAdd(&scount[my_e], 1);
    }
  }
  __syncthreads();
  if (chunk_counts)
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      chunk_counts[(int64_t)blockIdx.x * E + e] = scount[e];
}

// Scores alone: s [T, E] fp32, the score function of the logits, computed by
// the same token_scores as the selection (so selecting from these scores gives
// the selection's result bit for bit). Same token-to-warp mapping.
template <int NP>
__global__ void __launch_bounds__(kSelWarps * 32)
gate_scores_kernel(Resolved r, int T_, const float* __restrict__ logits,
                   float* __restrict__ out) {
  pdl_wait();
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int tt = 0; tt < kPermChunk / kSelWarps; ++tt) {
    const int t = blockIdx.x * kPermChunk + tt * kSelWarps + warp;
    if (t >= T_) break;
    float s[NP];
    token_scores<NP>(r, logits, nullptr, t, lane, s);
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int e = i * 32 + lane;
      if (e < r.E) out[(int64_t)t * r.E + e] = s[i];
    }
  }
}

}  // namespace

int gate_logit_splits(const Resolved& r, int64_t T) { return T <= kSmallTokens ? kSplitK : 1; }

cudaError_t launch_gate_logits(const Resolved& r, int64_t T, const void* x, const void* w_gate,
                               float* logits, int* err, int num_sms, cudaStream_t st) {
  const bool bf16 = r.act_bf16 != 0;
  if (T <= kSmallTokens) {
    const int vn = bf16 ? 8 : 4;
    const int kc = ((r.d + kSplitK - 1) / kSplitK + vn - 1) / vn * vn;
    const dim3 grid((unsigned)((r.E + 31) / 32), kSplitK);
    const dim3 block(kSmallWarps * 32);
    int* done = err + kGateDoneWord;   // per expert block, zeroed with the error word
    if (bf16)
      (void)launch_pdl(gate_logits_splitk_kernel<__nv_bfloat16>, grid, block, 0, st,
                       (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_gate, logits, (int)T,
                       r.E, r.d, kc, done);
    else
      (void)launch_pdl(gate_logits_splitk_kernel<float>, grid, block, 0, st, (const float*)x,
                       (const float*)w_gate, logits, (int)T, r.E, r.d, kc, done);
    return cudaGetLastError();
  }
  // Tensor-core logits write 16-byte chunks of fp32 rows of E entries.
  if (bf16 && r.E % 4 == 0) return launch_gate_logits_tc(r, T, x, w_gate, logits, err, num_sms, st);
  dim3 grid((r.E + kLE - 1) / kLE, (unsigned)((T + kLT - 1) / kLT));
  if (bf16)
    (void)launch_pdl(gate_logits_kernel<__nv_bfloat16>, grid, dim3(kLThreads), 0, st,
                     (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_gate, logits, (int)T, r.E,
                     r.d);
  else
    (void)launch_pdl(gate_logits_kernel<float>, grid, dim3(kLThreads), 0, st, (const float*)x,
                     (const float*)w_gate, logits, (int)T, r.E, r.d);
  return cudaGetLastError();
}

cudaError_t launch_gate_select(const Resolved& r, int64_t T, const float* logits,
                               const float* scores_in, const float* bias, int32_t* idx, float* w,
                               int32_t* chunk_counts, int* err, cudaStream_t st) {
  const unsigned grid = (unsigned)((T + kPermChunk - 1) / kPermChunk);
  const int np = (r.E + 31) / 32;
#define KT_SELECT(NPV)                                                                         \
  (void)launch_pdl(gate_select_kernel<NPV>, dim3(grid), dim3(kSelWarps * 32), 0, st, r, (int)T, \
                   logits, scores_in, bias, idx, w, chunk_counts, err)
  if (np <= 1) KT_SELECT(1);
  else if (np <= 2) KT_SELECT(2);
  else if (np <= 4) KT_SELECT(4);
  else if (np <= 8) KT_SELECT(8);
  else KT_SELECT(16);
#undef KT_SELECT
  return cudaGetLastError();
}

}  // namespace ktmoe

namespace ktmoe {

cudaError_t launch_gate_scores(const Resolved& r, int64_t T, const float* logits, float* scores,
                               cudaStream_t st) {
  const unsigned grid = (unsigned)((T + kPermChunk - 1) / kPermChunk);
  const int np = (r.E + 31) / 32;
#define KT_SCORES(NPV) \
  (void)launch_pdl(gate_scores_kernel<NPV>, dim3(grid), dim3(kSelWarps * 32), 0, st, r, (int)T, \
                   logits, scores)
  if (np <= 1) KT_SCORES(1);
  else if (np <= 2) KT_SCORES(2);
  else if (np <= 4) KT_SCORES(4);
  else if (np <= 8) KT_SCORES(8);
  else KT_SCORES(16);
#undef KT_SCORES
  return cudaGetLastError();
}

}  // namespace ktmoe
