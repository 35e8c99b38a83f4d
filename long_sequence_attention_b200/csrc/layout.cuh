// Chunk transpose for the Ulysses re-partition (xDiT overview page, section 3.2.2: the
// sequence-parallel dimension that exchanges heads for sequence with an all-to-all).
//
// dst[i1][i0] = src[i0][i1] for chunks of chunk_vecs 16-byte vectors.  An all-to-all sends
// one contiguous piece per peer; with a batch dimension B > 1 the piece for peer p of a
// [B, H, S_loc, D] tensor is strided ([B][P][H/P * S_loc * D] -> [P][B][...]), so this
// copy makes it contiguous before the exchange and undoes it after the return exchange.
// HBM-bound: each byte read once and written once, 16-byte loads and stores, consecutive
// threads on consecutive vectors of one chunk.
#pragma once

#include <cstdint>

namespace dit {

__global__ void __launch_bounds__(256) swap01_chunks_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                            long long d0, long long d1, long long chunk_vecs) {
  const long long total = d0 * d1 * chunk_vecs;
  for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < total;
       v += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long c = v / chunk_vecs;
    const long long off = v - c * chunk_vecs;
    const long long i0 = c / d1, i1 = c - i0 * d1;
    dst[(i1 * d0 + i0) * chunk_vecs + off] = __ldg(src + v);
  }
}

}  // namespace dit
