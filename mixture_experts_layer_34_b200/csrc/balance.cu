// Load statistics of the routing: the aux-loss-free bias update and the
// sequence-wise balance statistics of the DeepSeek-V3 model.py notes
// (73biji.xyz/llm_pp_dsv3):
//   - "V3 改进①：无辅助损失负载均衡": the selection bias b_i follows expert i's
//     load at a speed gamma; an overloaded expert's bias goes down, an
//     underloaded one's up. Load = picks of expert i among the T*k (token,
//     slot) pairs; the mean is T*k/E; an expert exactly at the mean keeps its
//     bias.
//   - "V3 改进②：序列级平衡损失": L_Bal = alpha * sum_i f_i P_i with
//     f_i = load_i / T (top-k activation frequency) and
//     P_i = (1/T) sum_t s_{i,t} / sum_j s_{j,t} (time mean of the normalised
//     affinity).
//
//   bias_update_kernel    : one CTA; shared-memory histogram (integer atomics,
//                           exact), then one fp32 addition per expert.
//   balance_partial_kernel: per chunk of tokens, one warp per token (interleaved
//                           over 8 warps) adds s / sum(s) per expert in
//                           registers; the chunk's warps are added in warp
//                           order and its picks counted.
//   balance_final_kernel  : one CTA adds the chunk partials in chunk order, then
//                           f, P and the loss (double accumulation over the
//                           experts). The result does not depend on scheduling.
#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

constexpr int kBalWarps = 8;
constexpr int kBalMaxChunks = 512;
constexpr unsigned kFullMask = 0xffffffffu;

__global__ void __launch_bounds__(1024)
bias_update_kernel(int E, int64_t n, const int32_t* __restrict__ idx, float* __restrict__ bias,
                   float gamma, int32_t* __restrict__ load_out) {
  __shared__ int load[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) load[e] = 0;
  __syncthreads();
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
    const int e = idx[i];
    if (e >= 0 && e < E) atomicAdd(&load[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    // load_e > n / E, decided in integers.
    const int64_t scaled = (int64_t)load[e] * E;
    float b = bias[e];
    if (scaled > n)
      b = __fsub_rn(b, gamma);
    else if (scaled < n)
      b = __fadd_rn(b, gamma);
    bias[e] = b;
    if (load_out) load_out[e] = load[e];
  }
}

template <int NP>
__global__ void __launch_bounds__(kBalWarps * 32)
balance_partial_kernel(int E, int T_, int k, int tpc, const float* __restrict__ scores,
                       const int32_t* __restrict__ idx, float* __restrict__ part_p,
                       int32_t* __restrict__ part_c) {
  __shared__ float acc[kBalWarps][kMaxExperts];
  __shared__ int cnt[kMaxExperts];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  float a[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) a[i] = 0.f;
  const int t0 = blockIdx.x * tpc;
  for (int tt = warp; tt < tpc; tt += kBalWarps) {
    const int t = t0 + tt;
    if (t >= T_) break;
    float s[NP];
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int e = i * 32 + lane;
      s[i] = e < E ? scores[(int64_t)t * E + e] : 0.f;
      z += s[i];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(kFullMask, z, off);
#pragma unroll
    for (int i = 0; i < NP; ++i)
      if (i * 32 + lane < E) a[i] += __fdiv_rn(s[i], z);
    for (int j = lane; j < k; j += 32) {
      const int e = idx[(int64_t)t * k + j];
      if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    }
  }
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const int e = i * 32 + lane;
    if (e < E) acc[warp][e] = a[i];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float p = 0.f;
    for (int w = 0; w < kBalWarps; ++w) p += acc[w][e];
    part_p[(int64_t)blockIdx.x * E + e] = p;
    part_c[(int64_t)blockIdx.x * E + e] = cnt[e];
  }
}

__global__ void __launch_bounds__(512)
balance_final_kernel(int E, int T_, int nchunks, float alpha, const float* __restrict__ part_p,
                     const int32_t* __restrict__ part_c, float* __restrict__ f,
                     float* __restrict__ P, float* __restrict__ loss) {
  __shared__ double prod[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float p = 0.f;
    int c = 0;
    for (int b = 0; b < nchunks; ++b) {
      p += part_p[(int64_t)b * E + e];
      c += part_c[(int64_t)b * E + e];
    }
    const float fe = __fdiv_rn((float)c, (float)T_);
    const float pe = __fdiv_rn(p, (float)T_);
    f[e] = fe;
    P[e] = pe;
    prod[e] = (double)fe * (double)pe;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double l = 0.0;
    for (int e = 0; e < E; ++e) l += prod[e];
    *loss = (float)((double)alpha * l);
  }
}

}  // namespace

cudaError_t launch_bias_update(const Resolved& r, int64_t T, const int32_t* idx, float* bias,
                               float gamma, int32_t* load_out, cudaStream_t st) {
  bias_update_kernel<<<1, 1024, 0, st>>>(r.E, T * r.k, idx, bias, gamma, load_out);
  return cudaGetLastError();
}

// Chunks of a multiple of 32 tokens, at most kBalMaxChunks of them.
int balance_chunks(int64_t T, int* tokens_per_chunk) {
  const int64_t per = (T + kBalMaxChunks - 1) / kBalMaxChunks;
  const int tpc = (int)(((per + 31) / 32) * 32);
  *tokens_per_chunk = tpc;
  return (int)((T + tpc - 1) / tpc);
}

size_t balance_scratch_bytes(const Resolved& r, int64_t T) {
  int tpc = 0;
  const int n = balance_chunks(T, &tpc);
  const size_t half = ((size_t)n * r.E * 4 + 255) / 256 * 256;
  return 2 * half;
}

cudaError_t launch_balance_stats(const Resolved& r, int64_t T, const float* scores,
                                 const int32_t* idx, float alpha, float* f, float* P, float* loss,
                                 void* scratch, cudaStream_t st) {
  int tpc = 0;
  const int n = balance_chunks(T, &tpc);
  const size_t half = balance_scratch_bytes(r, T) / 2;
  float* part_p = static_cast<float*>(scratch);
  int32_t* part_c = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) + half);
  const int np = (r.E + 31) / 32;
#define KT_BAL(NPV)                                                                      \
  balance_partial_kernel<NPV><<<n, kBalWarps * 32, 0, st>>>(r.E, (int)T, r.k, tpc, scores, \
                                                             idx, part_p, part_c)
  if (np <= 1) KT_BAL(1);
  else if (np <= 2) KT_BAL(2);
  else if (np <= 4) KT_BAL(4);
  else if (np <= 8) KT_BAL(8);
  else KT_BAL(16);
#undef KT_BAL
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  balance_final_kernel<<<1, 512, 0, st>>>(r.E, (int)T, n, alpha, part_p, part_c, f, P, loss);
  return cudaGetLastError();
}

}  // namespace ktmoe
