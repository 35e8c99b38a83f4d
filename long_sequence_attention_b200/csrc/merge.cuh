// Exact log-sum-exp merge of attention partials computed over disjoint KV chunks.
//
// This is the combine step of the USP "Ring" dimension (xDiT overview page, section 3.2.2:
// the sequence is split into blocks that travel around a ring, so each rank holds partial
// attention results over one block of keys at a time).  The pages do not print the combine;
// the exact one is, per query row,
//     M = max_c lse_c,  w_c = exp(lse_c - M),  L = sum_c w_c,
//     lse = M + log L,  out = sum_c (w_c / L) out_c,
// with every lse_c = -inf (all chunks empty) giving out = 0, lse = -inf.
//
// HBM-bound: each thread owns 8 consecutive elements of one row (one or two 16-byte loads
// per chunk, all coalesced); the handful of lse values per row are re-read by the row's
// threads from L1.  Arithmetic in fp32.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dit {

constexpr int kMaxMergeChunks = 16;

struct MergeParams {
  const void* outs[kMaxMergeChunks];
  const float* lses[kMaxMergeChunks];
  int n;
  void* out;
  float* lse;
  long long rows;     // B * H * S
  int D;
  int in_fp32;
  int out_fp32;
};

__device__ __forceinline__ void load8(const void* base, long long elem, bool fp32, float (&v)[8]) {
  if (fp32) {
    const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem);
    const float4 a = __ldg(src), b = __ldg(src + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + elem));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

__global__ void __launch_bounds__(256) lse_merge_kernel(const MergeParams p) {
  const int tpr = p.D / 8;                                     // threads per row
  const long long units = p.rows * tpr;
  for (long long u = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = u / tpr;
    const int col = static_cast<int>(u - row * tpr) * 8;
    const long long e = row * p.D + col;
    float M = -INFINITY;
    for (int c = 0; c < p.n; ++c) M = fmaxf(M, __ldg(p.lses[c] + row));
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float L = 0.0f;
    if (M != -INFINITY) {
      // Four chunks at a time: all their loads are issued before any is used, so each thread
      // keeps up to 4 x 32 bytes in flight.  An empty chunk (lse = -inf) has weight exactly 0
      // and its values are discarded by a select, whatever its buffer holds.
      for (int c0 = 0; c0 < p.n; c0 += 4) {
        float v[4][8];
        float w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = c0 + k;
          w[k] = 0.0f;
          if (c < p.n) {
            w[k] = __expf(__ldg(p.lses[c] + row) - M);
            load8(p.outs[c], e, p.in_fp32 != 0, v[k]);
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (c0 + k < p.n) {
            L += w[k];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = (w[k] != 0.0f) ? fmaf(w[k], v[k][i], acc[i]) : acc[i];
          }
        }
      }
      const float inv = 1.0f / L;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= inv;
    }
    if (p.out_fp32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + e);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint4 w;
      w.x = pack_bf16x2(acc[0], acc[1]);
      w.y = pack_bf16x2(acc[2], acc[3]);
      w.z = pack_bf16x2(acc[4], acc[5]);
      w.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + e) = w;
    }
    if (col == 0 && p.lse != nullptr) p.lse[row] = (M == -INFINITY) ? -INFINITY : M + logf(L);
  }
}

}  // namespace dit
