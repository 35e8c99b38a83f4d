// Per-tensor absmax quantisation of bf16 to FP8-E4M3 (the input side of the FP8 attention
// variant).
//
// The AMD ROCm summary page (xDiT on Radeon AI PRO R9700S) names an FP8 attention backend
// and notes that FP8 runs natively and changes outputs relative to BF16.  The pages fix no
// scaling scheme; this library uses one scale per tensor:
//     amax = max |x|,  descale = amax / 448 (1 if amax = 0),  code = e4m3_rn_satfinite(x / descale)
// with an IEEE fp32 division, so that the codes are reproducible bit for bit.
//
// Two launches, both HBM-bound: (1) per-block partial maxima into a small workspace,
// (2) every block reduces the partials (a few KB, L2-resident), then quantises its share
// with 16-byte loads and 8-byte stores.  Block 0 also writes descale.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dit {

constexpr int kQuantThreads = 256;
constexpr int kQuantMaxBlocks = 1184;          // 8 per SM on 148 SMs

__host__ __device__ inline int quant_blocks(long long n) {
  long long g = (n + 8191) / 8192;
  if (g < 1) g = 1;
  if (g > kQuantMaxBlocks) g = kQuantMaxBlocks;
  return static_cast<int>(g);
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (threadIdx.x < blockDim.x / 32) ? red[threadIdx.x] : 0.0f;
  if (w == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (l == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

__global__ void __launch_bounds__(kQuantThreads) absmax_partial_kernel(const uint16_t* __restrict__ x, long long n,
                                                                       float* __restrict__ partials) {
  __shared__ float red[kQuantThreads / 32];
  float m = 0.0f;
  const long long nvec = n / 8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < nvec; i += stride) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(x) + i);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      m = fmaxf(m, fabsf(bf16_bits_to_float(w[k] & 0xFFFFu)));
      m = fmaxf(m, fabsf(bf16_bits_to_float(w[k] >> 16)));
    }
  }
  if (blockIdx.x == 0)
    for (long long i = nvec * 8 + threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, fabsf(bf16_bits_to_float(x[i])));
  m = block_max(m, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = m;
}

__global__ void __launch_bounds__(kQuantThreads) quant_e4m3_kernel(const uint16_t* __restrict__ x, long long n,
                                                                   const float* __restrict__ partials, int n_partials,
                                                                   uint8_t* __restrict__ x8, float* __restrict__ descale_out) {
  __shared__ float red[kQuantThreads / 32];
  float m = 0.0f;
  for (int i = threadIdx.x; i < n_partials; i += blockDim.x) m = fmaxf(m, partials[i]);
  const float amax = block_max(m, red);
  const float descale = (amax > 0.0f) ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *descale_out = descale;

  const long long nvec = n / 8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < nvec; i += stride) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(x) + i);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
    uint32_t packed[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float v0 = __fdiv_rn(bf16_bits_to_float(w[2 * k] & 0xFFFFu), descale);
      const float v1 = __fdiv_rn(bf16_bits_to_float(w[2 * k] >> 16), descale);
      const float v2 = __fdiv_rn(bf16_bits_to_float(w[2 * k + 1] & 0xFFFFu), descale);
      const float v3 = __fdiv_rn(bf16_bits_to_float(w[2 * k + 1] >> 16), descale);
      packed[k] = pack_e4m3x4(v0, v1, v2, v3);
    }
    reinterpret_cast<uint2*>(x8)[i] = make_uint2(packed[0], packed[1]);
  }
  if (blockIdx.x == 0) {
    for (long long i = nvec * 8 + threadIdx.x; i < n; i += blockDim.x) {
      const float v = __fdiv_rn(bf16_bits_to_float(x[i]), descale);
      x8[i] = static_cast<uint8_t>(pack_e4m3x4(v, 0.f, 0.f, 0.f) & 0xFFu);
    }
  }
}

}  // namespace dit
