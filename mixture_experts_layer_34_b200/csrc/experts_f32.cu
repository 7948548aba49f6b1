// Expert SwiGLU FFNs for fp32 layers, on the SIMT FMA pipes.
//
// Same two grouped steps as the tensor-core path (up: silu(W1 u) * W3 u; down:
// w_r * W2 h, see "DeepSeekMoE 三改进" / "MoE 前向四步" of the DeepSeek-V3 model.py
// notes), in fp32 FMA arithmetic: TF32 tensor cores would not meet a 1e-4
// relative tolerance. Tiles of 32 rows x 32 output columns, K slabs of 32 in
// shared memory; token rows are gathered from x through tok_of (routed) or
// taken in order (shared experts), so no permuted copy of x is needed. Chunks
// name weight slots; slots below E (the routed-slot count passed in) are routed.
#include <cmath>

#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

constexpr int kTB = 32;   // rows and columns per tile
constexpr int kTK = 32;   // K slab

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + expf(-g)); }

__global__ void __launch_bounds__(256)
up_f32_kernel(const Chunk* __restrict__ chunks, const int32_t* __restrict__ n_chunks_p, int E,
              int d, int I, const float* __restrict__ x, const float* __restrict__ w1,
              const float* __restrict__ w3, const int32_t* __restrict__ tok_of,
              float* __restrict__ hidden, int T_, int n_routed_rows, int n_groups,
              int64_t n_rows, int max_chunks, int* __restrict__ err) {
  pdl_wait();
  __shared__ float xs[kTB][kTK + 1];
  __shared__ float as[kTB][kTK + 1];
  __shared__ float bs[kTB][kTK + 1];
  __shared__ int tok[kTB];
  int n_chunks = *n_chunks_p;
  if (!in_range(n_chunks, 0, max_chunks + 1, err, 141)) n_chunks = 0;
  const int rblocks = kChunkRows / kTB;
  const int fblocks = (I + kTB - 1) / kTB;
  const int ntiles = n_chunks * rblocks * fblocks;
  const int ty = threadIdx.x / 8, tx = threadIdx.x % 8;   // row ty, columns tx*4..+3
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int ci = tile / (rblocks * fblocks);
    const int rb = (tile / fblocks) % rblocks;
    const int fb = tile % fblocks;
    const Chunk ch = chunks[ci];
    if (!chunk_in_range(ch, n_groups, n_rows, kChunkRows, err, 142)) continue;
    const int r0 = rb * kTB;
    if (r0 >= ch.nrows) continue;   // uniform across the CTA
    const int f0 = fb * kTB;
    const float* wa = w1 + ((int64_t)ch.group * I + f0) * d;
    const float* wb = w3 + ((int64_t)ch.group * I + f0) * d;
    __syncthreads();
    if (threadIdx.x < kTB) {
      const int rr = r0 + threadIdx.x;
      int t = -1;
      if (rr < ch.nrows) {
        if (ch.group >= E) {
          t = ch.src_row0 + rr;
        } else {
          const int sr = ch.src_row0 + rr;
          t = in_range(sr, 0, n_routed_rows, err, 146) ? tok_of[sr] : -1;
        }
        if (t >= 0 && !in_range(t, 0, T_, err, 147)) t = -1;
      }
      tok[threadIdx.x] = t;
    }
    float g[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < d; k0 += kTK) {
      __syncthreads();
      for (int q = threadIdx.x; q < kTB * kTK; q += blockDim.x) {
        const int rr = q / kTK, kk = q % kTK;
        const int kg = k0 + kk;
        const int t = tok[rr];
        xs[rr][kk] = (t >= 0 && kg < d) ? x[(int64_t)t * d + kg] : 0.f;
        const bool fo = (f0 + rr < I) && kg < d;
        as[rr][kk] = fo ? wa[(int64_t)rr * d + kg] : 0.f;
        bs[rr][kk] = fo ? wb[(int64_t)rr * d + kg] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kTK; ++kk) {
        const float xv = xs[ty][kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          g[j] = fmaf(xv, as[tx * 4 + j][kk], g[j]);
          u[j] = fmaf(xv, bs[tx * 4 + j][kk], u[j]);
        }
      }
    }
    const int rr = r0 + ty;
    if (rr < ch.nrows)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int f = f0 + tx * 4 + j;
        if (f < I) hidden[(int64_t)(ch.row0 + rr) * I + f] = silu_f32(g[j]) * u[j];
      }
  }
}

__global__ void __launch_bounds__(256)
down_f32_kernel(const Chunk* __restrict__ chunks, const int32_t* __restrict__ n_chunks_p, int d,
                int I, int n_routed_rows, const float* __restrict__ hidden,
                const float* __restrict__ w2, const float* __restrict__ row_weight,
                float* __restrict__ out, int n_groups, int64_t n_rows, int max_chunks,
                int* __restrict__ err) {
  pdl_wait();
  __shared__ float hs[kTB][kTK + 1];
  __shared__ float ws[kTB][kTK + 1];
  int n_chunks = *n_chunks_p;
  if (!in_range(n_chunks, 0, max_chunks + 1, err, 151)) n_chunks = 0;
  const int rblocks = kChunkRows / kTB;
  const int oblocks = (d + kTB - 1) / kTB;
  const int ntiles = n_chunks * rblocks * oblocks;
  const int ty = threadIdx.x / 8, tx = threadIdx.x % 8;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int ci = tile / (rblocks * oblocks);
    const int rb = (tile / oblocks) % rblocks;
    const int ob = tile % oblocks;
    const Chunk ch = chunks[ci];
    if (!chunk_in_range(ch, n_groups, n_rows, kChunkRows, err, 152)) continue;
    const int r0 = rb * kTB;
    if (r0 >= ch.nrows) continue;
    const int o0 = ob * kTB;
    const float* wa = w2 + ((int64_t)ch.group * d + o0) * I;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < I; k0 += kTK) {
      __syncthreads();
      for (int q = threadIdx.x; q < kTB * kTK; q += blockDim.x) {
        const int rr = q / kTK, kk = q % kTK;
        const int kg = k0 + kk;
        hs[rr][kk] = (r0 + rr < ch.nrows && kg < I) ? hidden[(int64_t)(ch.row0 + r0 + rr) * I + kg] : 0.f;
        ws[rr][kk] = (o0 + rr < d && kg < I) ? wa[(int64_t)rr * I + kg] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kTK; ++kk) {
        const float hv = hs[ty][kk];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = fmaf(hv, ws[tx * 4 + j][kk], acc[j]);
      }
    }
    const int rr = r0 + ty;
    if (rr < ch.nrows) {
      const int row = ch.row0 + rr;
      const float wr = row < n_routed_rows ? row_weight[row] : 1.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int o = o0 + tx * 4 + j;
        if (o < d) out[(int64_t)row * d + o] = acc[j] * wr;
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_experts_f32(const Resolved& r, int64_t T, const Layout& L, char* ws,
                               const void* x, const void* w1, const void* w3, const void* w2,
                               int num_sms, cudaStream_t st, bool up) {
  const int32_t* meta = reinterpret_cast<const int32_t*>(ws + L.meta);
  const int grid = num_sms * 4;
  const int64_t n_rows = T * (r.k + r.S);
  int* err = reinterpret_cast<int*>(ws + L.err);
  if (up) {
    (void)launch_pdl(up_f32_kernel, dim3(grid), dim3(256), 0, st,
        reinterpret_cast<const Chunk*>(ws + L.chunks), meta + 0, routed_slots(r), r.d, r.I,
        static_cast<const float*>(x), static_cast<const float*>(w1), static_cast<const float*>(w3),
        reinterpret_cast<const int32_t*>(ws + L.tok_of), reinterpret_cast<float*>(ws + L.hidden),
        (int)T, (int)(T * r.k), weight_slots(r), n_rows, (int)L.max_chunks, err);
    return cudaGetLastError();
  }
  (void)launch_pdl(down_f32_kernel, dim3(grid), dim3(256), 0, st,
      reinterpret_cast<const Chunk*>(ws + L.chunks), meta + 0, r.d, r.I, (int)(T * r.k),
      reinterpret_cast<const float*>(ws + L.hidden), static_cast<const float*>(w2),
      reinterpret_cast<const float*>(ws + L.row_weight),
      reinterpret_cast<float*>(ws + L.expert_out), weight_slots(r), n_rows, (int)L.max_chunks,
      err);
  return cudaGetLastError();
}

}  // namespace ktmoe
