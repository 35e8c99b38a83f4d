// Absmax quantisation of bf16 to FP8-E4M3 (the input side of the FP8 attention variant).
//
// The AMD ROCm summary page (xDiT on Radeon AI PRO R9700S) names an FP8 attention backend
// and notes that FP8 runs natively and changes outputs relative to BF16.  The pages fix no
// scaling scheme; this library uses one scale per tensor (and, as a finer variant, one per
// 128-row block of a head):
//     amax = max |x|,  descale = amax / 448 (1 if amax = 0),  code = e4m3_rn_satfinite(x / descale)
// with the codes of an IEEE fp32 division, reproducible bit for bit (see quot_e4m3).
//
// Per tensor: two launches, both HBM-bound: (1) per-block partial maxima into a small
// workspace, (2) every block reduces the partials (a few KB, L2-resident), then quantises its
// share with 16-byte loads and 8-byte stores.  Block 0 also writes descale.
// Per block: one launch, one CTA per block (quant_e4m3_rows_kernel below).
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dit {

constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;                // 16-byte loads in flight per thread
constexpr int kQuantMaxBlocks = 1184;          // 8 per SM on 148 SMs

__host__ __device__ inline int quant_blocks(long long n) {
  long long g = (n + 8 * kQuantThreads * kQuantUnroll - 1) / (8 * kQuantThreads * kQuantUnroll);
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

// The quotient x / d as far as its E4M3 code is concerned, without a division per element.
// r = 1/d correctly rounded; x * r differs from x / d by at most 2^-23 relative (two roundings
// of 2^-24), i.e. under 2.5 fp32 ulps from the IEEE quotient.  Both give the same E4M3 code
// unless an E4M3 rounding midpoint lies between them.  Above 2^-6 (the E4M3 normal range,
// 3 mantissa bits) the midpoints are the fp32 values whose low 20 mantissa bits are
// 0x80000, so a product more than 8 ulps away from that pattern keeps its code; anything
// else (near a midpoint, E4M3 subnormal range, zero, NaN) takes the IEEE division.
__device__ __forceinline__ float quot_e4m3(float x, float d, float r) {
  const float q = x * r;
  const uint32_t low = __float_as_uint(q) & 0xFFFFFu;
  if (fabsf(q) >= 0.015625f && (low - 0x7FFF8u) > 0x10u) return q;
  return __fdiv_rn(x, d);
}

__global__ void __launch_bounds__(kQuantThreads) absmax_partial_kernel(const uint16_t* __restrict__ x, long long n,
                                                                       float* __restrict__ partials) {
  __shared__ float red[kQuantThreads / 32];
  float m = 0.0f;
  const long long nvec = n / 8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x * kQuantUnroll;
  // kQuantUnroll independent 16-byte loads per thread before any is used
  for (long long i0 = blockIdx.x * static_cast<long long>(blockDim.x) * kQuantUnroll + threadIdx.x; i0 < nvec;
       i0 += stride) {
    uint4 a[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const long long i = i0 + static_cast<long long>(u) * blockDim.x;
      a[u] = i < nvec ? __ldg(reinterpret_cast<const uint4*>(x) + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const uint32_t w[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        m = fmaxf(m, fabsf(bf16_bits_to_float(w[k] & 0xFFFFu)));
        m = fmaxf(m, fabsf(bf16_bits_to_float(w[k] >> 16)));
      }
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
  const float rcp = __frcp_rn(descale);
  if (blockIdx.x == 0 && threadIdx.x == 0) *descale_out = descale;

  const long long nvec = n / 8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x * kQuantUnroll;
  for (long long i0 = blockIdx.x * static_cast<long long>(blockDim.x) * kQuantUnroll + threadIdx.x; i0 < nvec;
       i0 += stride) {
    uint4 a[kQuantUnroll];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const long long i = i0 + static_cast<long long>(u) * blockDim.x;
      a[u] = i < nvec ? __ldg(reinterpret_cast<const uint4*>(x) + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const long long i = i0 + static_cast<long long>(u) * blockDim.x;
      if (i >= nvec) break;
      const uint32_t w[4] = {a[u].x, a[u].y, a[u].z, a[u].w};
      uint32_t packed[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float v0 = quot_e4m3(bf16_bits_to_float(w[2 * k] & 0xFFFFu), descale, rcp);
        const float v1 = quot_e4m3(bf16_bits_to_float(w[2 * k] >> 16), descale, rcp);
        const float v2 = quot_e4m3(bf16_bits_to_float(w[2 * k + 1] & 0xFFFFu), descale, rcp);
        const float v3 = quot_e4m3(bf16_bits_to_float(w[2 * k + 1] >> 16), descale, rcp);
        packed[k] = pack_e4m3x4(v0, v1, v2, v3);
      }
      reinterpret_cast<uint2*>(x8)[i] = make_uint2(packed[0], packed[1]);
    }
  }
  if (blockIdx.x == 0) {
    for (long long i = nvec * 8 + threadIdx.x; i < n; i += blockDim.x) {
      const float v = __fdiv_rn(bf16_bits_to_float(x[i]), descale);
      x8[i] = static_cast<uint8_t>(pack_e4m3x4(v, 0.f, 0.f, 0.f) & 0xFFu);
    }
  }
}

// Per-block scales: one CTA per block of 128 consecutive rows of one (b, h) of a [B,H,S,D]
// tensor (the last block of a head may be shorter).  The block is contiguous in memory (at
// most 128 x 128 bf16 = 32 KB): one bulk copy brings it into shared memory, the CTA reduces
// its absolute maximum there and writes the codes: one HBM read and one write per element,
// with several CTAs' copies in flight per SM.  An all-zero block gets descale 0 (it holds only
// zero codes; a consumer can tell it apart from a block whose maximum is 448) and codes of
// x / 1, the per-tensor rule for an all-zero tensor.
constexpr int kQuantBlockRows = 128;
constexpr int kQuantRowThreads = 256;
constexpr int kQuantRowVecs = kQuantBlockRows * 128 / 8;     // 16-byte vectors of a full D = 128 block

__global__ void __launch_bounds__(kQuantRowThreads) quant_e4m3_rows_kernel(const uint16_t* __restrict__ x, int S,
                                                                           int D, int nblk, uint8_t* __restrict__ x8,
                                                                           float* __restrict__ descales,
                                                                           unsigned long long timeout_ns) {
  __shared__ __align__(128) uint4 buf[kQuantRowVecs];
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  __shared__ float red[kQuantRowThreads / 32];
  const long long bh = blockIdx.x / nblk;
  const int i = static_cast<int>(blockIdx.x - bh * nblk);
  const int r0 = i * kQuantBlockRows;
  const int rows = min(kQuantBlockRows, S - r0);
  const long long base = (bh * S + r0) * static_cast<long long>(D);      // first element
  const int nvec = rows * D / 8;                                         // D % 8 == 0
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(nvec) * 16u);
    bulk_load(buf, x + base, static_cast<uint32_t>(nvec) * 16u, &bar);
  }
  const bool ok = mbar_wait(&bar, 0, &abort_flag, timeout_ns, 0xB0);
  if (!__syncthreads_and(ok)) {
    // the copy this CTA issued must land before its shared memory goes away
    if (threadIdx.x == 0) mbar_wait_drain(&bar, 0, timeout_ns);
    return;
  }
  float m = 0.0f;
  for (int idx = threadIdx.x; idx < nvec; idx += kQuantRowThreads) {
    const uint4 a = buf[idx];
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      m = fmaxf(m, fabsf(bf16_bits_to_float(w[e] & 0xFFFFu)));
      m = fmaxf(m, fabsf(bf16_bits_to_float(w[e] >> 16)));
    }
  }
  const float amax = block_max(m, red);
  const float descale = (amax > 0.0f) ? __fdiv_rn(amax, 448.0f) : 1.0f;
  const float rcp = __frcp_rn(descale);
  if (threadIdx.x == 0) descales[blockIdx.x] = (amax > 0.0f) ? descale : 0.0f;
  for (int idx = threadIdx.x; idx < nvec; idx += kQuantRowThreads) {
    const uint4 a = buf[idx];
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
    uint32_t packed[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      packed[h] = pack_e4m3x4(quot_e4m3(bf16_bits_to_float(w[2 * h] & 0xFFFFu), descale, rcp),
                              quot_e4m3(bf16_bits_to_float(w[2 * h] >> 16), descale, rcp),
                              quot_e4m3(bf16_bits_to_float(w[2 * h + 1] & 0xFFFFu), descale, rcp),
                              quot_e4m3(bf16_bits_to_float(w[2 * h + 1] >> 16), descale, rcp));
    reinterpret_cast<uint2*>(x8 + base)[idx] = make_uint2(packed[0], packed[1]);
  }
}

}  // namespace dit
