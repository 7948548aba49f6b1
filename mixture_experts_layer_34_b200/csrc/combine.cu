// Unpermute and combine: the sum of the total-output equation of the
// "DeepSeekMoE 三改进" passage (DeepSeek-V3 model.py notes,
// 73biji.xyz/llm_pp_dsv3) and the "加共享专家 z" step of "MoE 前向四步":
//     y_t = sum_s out[shared row of (s, t)] + sum_j out[row_of[t, j]]  (+ u_t)
// The weighted expert outputs (fp32) were written per row by the down GEMM. The sum
// runs in fp32 in a fixed order (shared experts, then the routed slots in key
// order, then the residual), so the result does not depend on scheduling.
// One CTA per token; 16-byte loads along the hidden dimension.
#include <cuda_bf16.h>

#include <algorithm>

#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

// 8 (bf16 input) or 4 (fp32) elements per thread per iteration; y in bf16 or
// fp32 (kF32Out).
template <bool kBF16, bool kF32Out>
__global__ void __launch_bounds__(128)
combine_kernel(int T_, int k, int S, int d, int add_residual, const int32_t* __restrict__ row_of,
               const float* __restrict__ expert_out, const void* __restrict__ x,
               void* __restrict__ y, int* __restrict__ err) {
  pdl_wait();
  constexpr int V = kBF16 ? 8 : 4;
  __shared__ int rows[kMaxShared + kMaxTopk];
  const int t = blockIdx.x;
  if (threadIdx.x < S) rows[threadIdx.x] = T_ * k + threadIdx.x * T_ + t;
  if (threadIdx.x < k) {
    const int row = row_of[(int64_t)t * k + threadIdx.x];
    rows[S + threadIdx.x] = in_range(row, 0, (int64_t)T_ * k, err, 121) ? row : -1;
  }
  __syncthreads();
  const int nrow = S + k;
  const int nq = d / V;
  // blockIdx.y: a slice of the columns (few tokens: several CTAs per token).
  const int per = (nq + gridDim.y - 1) / gridDim.y;
  const int q1 = min(nq, (int)(blockIdx.y + 1) * per);
  for (int q = blockIdx.y * per + threadIdx.x; q < q1; q += blockDim.x) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;
    for (int j = 0; j < nrow; ++j) {
      if (kChecked && rows[j] < 0) continue;
      const float4* src = reinterpret_cast<const float4*>(expert_out + (int64_t)rows[j] * d) + q * (V / 4);
#pragma unroll
      for (int h = 0; h < V / 4; ++h) {
        const float4 v = src[h];
        acc[4 * h] += v.x;
        acc[4 * h + 1] += v.y;
        acc[4 * h + 2] += v.z;
        acc[4 * h + 3] += v.w;
      }
    }
    if (kBF16) {
      if (add_residual) {
        const uint4 v = static_cast<const uint4*>(x)[(int64_t)t * nq + q];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += __uint_as_float(w[i] << 16);
          acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
        }
      }
      if (kF32Out) {
        float4* yo = static_cast<float4*>(y) + ((int64_t)t * nq + q) * 2;
        yo[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        yo[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
      } else {
        uint4 o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
          ow[i] = *reinterpret_cast<const uint32_t*>(&p);
        }
        static_cast<uint4*>(y)[(int64_t)t * nq + q] = o;
      }
    } else {
      if (add_residual) {
        const float4 v = static_cast<const float4*>(x)[(int64_t)t * nq + q];
        acc[0] += v.x;
        acc[1] += v.y;
        acc[2] += v.z;
        acc[3] += v.w;
      }
      static_cast<float4*>(y)[(int64_t)t * nq + q] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
  }
}

// Expert-parallel partial sum (the local expert loop of "MoE 前向四步"): per
// token, the shared experts if the token is in [sb, se), then the routed slots
// whose expert is computed here (row_of >= 0), in fp32; no residual.
__global__ void __launch_bounds__(128)
combine_partial_kernel(int T_, int k, int S, int d, int sb, int se,
                       const int32_t* __restrict__ row_of, const float* __restrict__ expert_out,
                       float4* __restrict__ y, int* __restrict__ err) {
  pdl_wait();
  __shared__ int rows[kMaxShared + kMaxTopk];
  __shared__ int nrow;
  const int t = blockIdx.x;
  if (threadIdx.x == 0) {
    int n = 0;
    if (t >= sb && t < se)
      for (int s = 0; s < S; ++s) rows[n++] = T_ * k + s * T_ + t;
    for (int j = 0; j < k; ++j) {
      const int row = row_of[(int64_t)t * k + j];
      if (row >= 0 && in_range(row, 0, (int64_t)T_ * k, err, 122)) rows[n++] = row;
    }
    nrow = n;
  }
  __syncthreads();
  const int nq = d / 4;
  const int per = (nq + gridDim.y - 1) / gridDim.y;
  const int q1 = min(nq, (int)(blockIdx.y + 1) * per);
  for (int q = blockIdx.y * per + threadIdx.x; q < q1; q += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < nrow; ++j) {
      const float4 v = reinterpret_cast<const float4*>(expert_out + (int64_t)rows[j] * d)[q];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    y[(int64_t)t * nq + q] = acc;
  }
}

// After the sum over ranks ("all_reduce(y)" of "MoE 前向四步", the shared
// experts' z already inside it): y = y_sum (+ u), in y's type.
template <bool kBF16X, bool kF32Out>
__global__ void __launch_bounds__(256)
ep_finish_kernel(int64_t n4, int add_residual, const float4* __restrict__ y_sum,
                 const void* __restrict__ x, void* __restrict__ y) {
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (int64_t)gridDim.x * blockDim.x) {
    float4 v = y_sum[i];
    if (add_residual) {
      if (kBF16X) {
        const uint2 u = static_cast<const uint2*>(x)[i];
        v.x += __uint_as_float(u.x << 16);
        v.y += __uint_as_float(u.x & 0xffff0000u);
        v.z += __uint_as_float(u.y << 16);
        v.w += __uint_as_float(u.y & 0xffff0000u);
      } else {
        const float4 u = static_cast<const float4*>(x)[i];
        v.x += u.x;
        v.y += u.y;
        v.z += u.z;
        v.w += u.w;
      }
    }
    if (kF32Out) {
      static_cast<float4*>(y)[i] = v;
    } else {
      const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
      static_cast<uint2*>(y)[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                                             *reinterpret_cast<const uint32_t*>(&hi));
    }
  }
}

}  // namespace

// Column slices per token: one CTA per token when there are many, several when
// few (a decode step), each slice at least 128 columns of 16-byte vectors.
dim3 combine_grid(int64_t T, int d, int num_sms) {
  const int64_t most = std::max<int64_t>(1, d / (128 * 8));
  const int64_t target = 2 * (num_sms > 0 ? num_sms : 148);
  return dim3((unsigned)T, (unsigned)std::max<int64_t>(1, std::min<int64_t>(most, target / T)));
}

cudaError_t launch_combine_partial(const Resolved& r, int64_t T, const Layout& L, char* ws,
                                   float* y_part, cudaStream_t st) {
  (void)launch_pdl(combine_partial_kernel, combine_grid(T, r.d, r.num_sms), dim3(128), 0, st,
      (int)T, r.k, r.S, r.d, r.sb, r.se, reinterpret_cast<const int32_t*>(ws + L.row_of),
      reinterpret_cast<const float*>(ws + L.expert_out), reinterpret_cast<float4*>(y_part),
      reinterpret_cast<int*>(ws + L.err));
  return cudaGetLastError();
}

cudaError_t launch_ep_finish(const Resolved& r, int64_t T, const float* y_sum, const void* x,
                             void* y, int num_sms, cudaStream_t st) {
  const int64_t n4 = T * r.d / 4;
  const unsigned grid = (unsigned)std::min<int64_t>((n4 + 255) / 256, (int64_t)num_sms * 8);
  const float4* ys = reinterpret_cast<const float4*>(y_sum);
  if (r.act_bf16 && !r.y_fp32)
    (void)launch_pdl(ep_finish_kernel<true, false>, dim3(grid), dim3(256), 0, st, n4,
                     r.add_residual, ys, x, y);
  else if (r.act_bf16)
    (void)launch_pdl(ep_finish_kernel<true, true>, dim3(grid), dim3(256), 0, st, n4,
                     r.add_residual, ys, x, y);
  else
    (void)launch_pdl(ep_finish_kernel<false, true>, dim3(grid), dim3(256), 0, st, n4,
                     r.add_residual, ys, x, y);
  return cudaGetLastError();
}

cudaError_t launch_combine(const Resolved& r, int64_t T, const Layout& L, char* ws, const void* x,
                           void* y, cudaStream_t st) {
  const int32_t* row_of = reinterpret_cast<const int32_t*>(ws + L.row_of);
  const float* eo = reinterpret_cast<const float*>(ws + L.expert_out);
  const dim3 grid = combine_grid(T, r.d, r.num_sms);
  int* err = reinterpret_cast<int*>(ws + L.err);
  if (r.act_bf16 && !r.y_fp32)
    (void)launch_pdl(combine_kernel<true, false>, grid, dim3(128), 0, st, (int)T, r.k, r.S, r.d,
                     r.add_residual, row_of, eo, x, y, err);
  else if (r.act_bf16)
    (void)launch_pdl(combine_kernel<true, true>, grid, dim3(128), 0, st, (int)T, r.k, r.S, r.d,
                     r.add_residual, row_of, eo, x, y, err);
  else
    (void)launch_pdl(combine_kernel<false, true>, grid, dim3(128), 0, st, (int)T, r.k, r.S, r.d,
                     r.add_residual, row_of, eo, x, y, err);
  return cudaGetLastError();
}

}  // namespace ktmoe
