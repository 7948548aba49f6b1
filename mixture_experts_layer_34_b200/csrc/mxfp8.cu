// MXFP8 quantisation for the FP8-expert form of the layer: E4M3 elements, one
// power-of-two scale per 32 consecutive elements along K, stored as a biased
// exponent byte (e + 127).
//
// The pages name the format family (the DeepSeek-V3 notes' FP8 mixed
// precision, the KTransformers page's native MXFP4 routed experts) but no
// rule; the rule here: e is the smallest integer with amax <= 448 * 2^e (no
// element saturates) and each element is the E4M3 round-to-nearest-even of
// v * 2^-e (mx_scale_exp and mx_code in ktmoe_internal.cuh).
//
//   mx_quantize_kernel : row-major [rows, K] bf16 -> codes [rows, K] and
//                        scale bytes [rows, K/32] (one thread per 32 elements)
//   mx_pack_kernel     : expert weights -> codes in place of the bf16 layout
//                        and the packed scale blocks the grouped GEMM loads
//                        (mx_packed_offset_*: the layout kt_moe_mxfp8_pack
//                        documents).
//
// MXFP4 (kW4 = true; the 4-bit form): the same blocks with E2M1 elements and
// the rule e = the smallest integer with amax <= 6 * 2^e (mx4_scale_exp,
// e2m1_code); 32 codes pack into 16 bytes, element 2i in the low nibble of
// byte i. The scale layout is the same.
#include <cuda_bf16.h>

#include "ktmoe_internal.cuh"

namespace ktmoe {
namespace {

// 32 bf16 values (64 bytes) to 32 codes (32 bytes); returns the scale byte.
__device__ __forceinline__ uint8_t mx_block_bf16(const uint4* __restrict__ src,
                                                 uint4* __restrict__ dst) {
  float v[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = src[q];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = mx_scale_exp(amax);
  const float inv = mx_inv_scale(e);
  uint32_t packed[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t p = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) p |= (uint32_t)mx_code(v[4 * q + i], inv) << (8 * i);
    packed[q] = p;
  }
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  return (uint8_t)(e + 127);
}

// 32 bf16 values (64 bytes) to 32 E2M1 codes (16 bytes); returns the scale byte.
__device__ __forceinline__ uint8_t mx4_block_bf16(const uint4* __restrict__ src,
                                                  uint4* __restrict__ dst) {
  float v[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = src[q];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[8 * q + 2 * i] = __uint_as_float(w[i] << 16);
      v[8 * q + 2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = mx4_scale_exp(amax);
  const float inv = mx_inv_scale(e);
  uint32_t packed[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t p = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) p |= e2m1_code(__fmul_rn(v[8 * q + i], inv)) << (4 * i);
    packed[q] = p;
  }
  dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  return (uint8_t)(e + 127);
}

template <bool kW4>
__global__ void __launch_bounds__(256)
mx_quantize_kernel(const uint4* __restrict__ src, int64_t nblocks, uint4* __restrict__ codes,
                   uint8_t* __restrict__ scales) {
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  scales[i] =
      kW4 ? mx4_block_bf16(src + i * 4, codes + i) : mx_block_bf16(src + i * 4, codes + i * 2);
}

// Packed scale offsets (bytes). Gate/up: a 512-byte block per (group, feature
// tile of 128, CTA half, K slab of 128); tile row m < 64 is W1 row
// 128 ft + 64 h + m, m >= 64 the same row of W3. Down: a block per (group,
// feature tile of 256 output rows, half, K slab); tile row m is W2 row
// 256 ft + 128 h + m. Inside a block: 16 * (m % 32) + 4 * (m / 32) + k1.
__device__ __forceinline__ int64_t mx_packed_offset_up(int64_t g, int f, int which, int b, int I,
                                                       int d) {
  const int ft = f / 128, h = (f % 128) / 64, m = (f % 64) + 64 * which;
  const int64_t blk = ((g * (I / 128) + ft) * 2 + h) * (d / 128) + b / 4;
  return blk * 512 + 16 * (m % 32) + 4 * (m / 32) + (b % 4);
}
__device__ __forceinline__ int64_t mx_packed_offset_down(int64_t g, int o, int b, int I, int d) {
  const int nft = (d + 255) / 256;
  const int ft = o / 256, h = (o % 256) / 128, m = o % 128;
  const int64_t blk = ((g * nft + ft) * 2 + h) * (I / 128) + b / 4;
  return blk * 512 + 16 * (m % 32) + 4 * (m / 32) + (b % 4);
}

// which: 0 W1, 1 W3 (rows NG*I, K = d), 2 W2 (rows NG*d, K = I).
template <bool kW4>
__global__ void __launch_bounds__(256)
mx_pack_kernel(const uint4* __restrict__ src, int64_t nblocks, int which, int d, int I,
               uint4* __restrict__ codes, uint8_t* __restrict__ sf) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nblocks) return;
  const uint8_t s =
      kW4 ? mx4_block_bf16(src + i * 4, codes + i) : mx_block_bf16(src + i * 4, codes + i * 2);
  const int K = which == 2 ? I : d;
  const int64_t row = i / (K / 32);
  const int b = (int)(i % (K / 32));
  if (which == 2)
    sf[mx_packed_offset_down(row / d, (int)(row % d), b, I, d)] = s;
  else
    sf[mx_packed_offset_up(row / I, (int)(row % I), which, b, I, d)] = s;
}

}  // namespace

cudaError_t launch_mx_quantize(const void* src, int64_t rows, int64_t K, uint8_t* codes,
                               uint8_t* scales, cudaStream_t st) {
  const int64_t nb = rows * (K / 32);
  if (nb == 0) return cudaSuccess;
  (void)launch_pdl(mx_quantize_kernel<false>, dim3((unsigned)((nb + 255) / 256)), dim3(256), 0, st,
      static_cast<const uint4*>(src), nb, reinterpret_cast<uint4*>(codes), scales);
  return cudaGetLastError();
}

cudaError_t launch_mx4_quantize(const void* src, int64_t rows, int64_t K, uint8_t* codes,
                                uint8_t* scales, cudaStream_t st) {
  const int64_t nb = rows * (K / 32);
  if (nb == 0) return cudaSuccess;
  (void)launch_pdl(mx_quantize_kernel<true>, dim3((unsigned)((nb + 255) / 256)), dim3(256), 0, st,
      static_cast<const uint4*>(src), nb, reinterpret_cast<uint4*>(codes), scales);
  return cudaGetLastError();
}

size_t mx_packed_bytes(const Resolved& r, bool down) {
  const size_t NG = (size_t)weight_slots(r);
  if (down) return NG * ((r.d + 255) / 256) * 2 * (r.I / 128) * 512;
  return NG * (r.I / 128) * 2 * (r.d / 128) * 512;
}

cudaError_t launch_mx_pack(const Resolved& r, const void* w1, const void* w3, const void* w2,
                           uint8_t* w1q, uint8_t* w3q, uint8_t* w2q, uint8_t* sf_up,
                           uint8_t* sf_down, cudaStream_t st) {
  const int64_t NG = weight_slots(r);
  // Blocks of packed rows past d (a last down feature tile of 128 rows) stay 0.
  cudaError_t e = cudaMemsetAsync(sf_down, 0, mx_packed_bytes(r, true), st);
  if (e != cudaSuccess) return e;
  const int64_t nb_up = NG * r.I * (r.d / 32), nb_dn = NG * r.d * (r.I / 32);
  const unsigned gu = (unsigned)((nb_up + 255) / 256), gd = (unsigned)((nb_dn + 255) / 256);
  auto pack = r.w4 ? mx_pack_kernel<true> : mx_pack_kernel<false>;
  pack<<<gu, 256, 0, st>>>(static_cast<const uint4*>(w1), nb_up, 0, r.d, r.I,
                           reinterpret_cast<uint4*>(w1q), sf_up);
  pack<<<gu, 256, 0, st>>>(static_cast<const uint4*>(w3), nb_up, 1, r.d, r.I,
                           reinterpret_cast<uint4*>(w3q), sf_up);
  pack<<<gd, 256, 0, st>>>(static_cast<const uint4*>(w2), nb_dn, 2, r.d, r.I,
                           reinterpret_cast<uint4*>(w2q), sf_down);
  return cudaGetLastError();
}

}  // namespace ktmoe
