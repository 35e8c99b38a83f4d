// C-ABI boundary of the DiT attention library: argument validation, TMA descriptor
// construction, kernel launches and status codes.  See include/dit_attn.h for the contract.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/dit_attn.h"
#include "attn_fwd.cuh"
#include "merge.cuh"
#include "quant.cuh"
#include "layout.cuh"

namespace {

using namespace dit;

std::atomic<unsigned long long> g_timeout_ns{1000000000ull};
std::atomic<int> g_sm_reserve{0};   // SMs the persistent attention grid leaves free

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry-point lookup, so the library does
// not link libcuda directly (it loads on machines without a GPU driver).
EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

typedef CUresult (*MemGetAddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);

// cuMemGetAddressRange through the same entry-point lookup (the allocation holding a pointer,
// needed to export a pointer that lies inside a larger allocation).
MemGetAddressRangeFn addr_range_fn() {
  static std::once_flag once;
  static MemGetAddressRangeFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<MemGetAddressRangeFn>(p);
  });
  return fn;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (a == nullptr || b == nullptr || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// 3-D tiled map over a [B*H, S, D] tensor: box = (128 bytes of D, 128 rows, 1 head),
// 128-byte swizzle, zero fill out of bounds (rows past S read as zeros, per head).
// 4-D map (D, seg, BH, S / seg) of a tensor whose rows are stored in sequence segments:
// row r of head bh at ((r / seg) * BH + bh) * seg + r % seg.  seg = S is the plain
// [BH, S, D] layout.  Box: 128 bytes x 128 rows, 128-byte swizzle; rows past a segment or
// past the last segment read as zero.
int make_map(CUtensorMap* m, const void* ptr, bool fp8, int D, int S, int BH, int seg) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return DIT_ERR_CUDA;
  const cuuint64_t elem = fp8 ? 1 : 2;
  const cuuint64_t n_seg = static_cast<cuuint64_t>(S / seg);
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(seg), static_cast<cuuint64_t>(BH), n_seg};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * elem, static_cast<cuuint64_t>(seg) * D * elem,
                           static_cast<cuuint64_t>(BH) * seg * D * elem};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / elem), 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                         const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DIT_OK : DIT_ERR_CUDA;
}

// 5-D map (D, X, Y, T, BH) of a bf16 [BH, T*Y*X, D] tensor on a T x Y x X token grid for
// the neighborhood-attention kernel.  Box: 128 bytes x a bx x by x bt (x, y, t) brick of
// tokens (bx * by * bt = 128 rows), 128-byte swizzle; tokens past the grid read as zero.
int make_map_na(CUtensorMap* m, const void* ptr, int D, int T, int Y, int X, int BH, int bt, int by, int bx) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return DIT_ERR_CUDA;
  const cuuint64_t e = 2;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(X), static_cast<cuuint64_t>(Y),
                        static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(D) * e, static_cast<cuuint64_t>(X) * D * e,
                           static_cast<cuuint64_t>(Y) * X * D * e, static_cast<cuuint64_t>(T) * Y * X * D * e};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(128 / e), static_cast<cuuint32_t>(bx), static_cast<cuuint32_t>(by),
                       static_cast<cuuint32_t>(bt), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DIT_OK : DIT_ERR_CUDA;
}

// Q brick and pairing axis of the neighborhood kernel for a grid and window.  Each Q brick
// (t, y, x extents, powers of two with product 128) visits the KV bricks that cover the union
// of its rows' windows, and a unit (two Q bricks side by side along axis pax) takes as many
// KV steps as the longer of its two lists.  The choice minimises the steps of a head plus
// kNaUnitCost steps for every unit (the epilogue and the next Q load of a unit boundary).
// The step count factorises over the dimensions: a brick's list length is the product of
// its per-dimension brick counts, and the two bricks of a unit differ along pax only.
constexpr long long kNaUnitCost = 2;

int na_host_wstart(int i, int K, int L) { return std::min(std::max(i - K / 2, 0), L - K); }

// KV bricks of extent b covering the windows of the queries [a, min(a + ext, L)); 0 if a >= L.
long long na_host_count(int a, int ext, int K, int L, int b) {
  if (a >= L) return 0;
  const int last = std::min(a + ext, L) - 1;
  const int first = na_host_wstart(a, K, L);
  return (na_host_wstart(last, K, L) + K - first + b - 1) / b;
}

struct NaChoice {
  int qb[3];          // Q brick extents (t, y, x)
  int pax;            // axis of the unit's brick pair
  int nu[3];          // units along t, y, x
  long long steps;    // KV steps of one head
};

NaChoice na_choose(const int L[3], const int K[3]) {
  static const int kb[3] = {kNaBt, kNaBy, kNaBx};
  NaChoice best{{kNaBt, kNaBy, kNaBx}, 1, {0, 0, 0}, 0};
  long long best_cost = -1;
  for (int lt = 0; lt <= 7; ++lt)
    for (int ly = 0; lt + ly <= 7; ++ly) {
      const int qb[3] = {1 << lt, 1 << ly, 1 << (7 - lt - ly)};
      for (int pax = 0; pax < 3; ++pax) {
        long long steps = 1, units = 1;
        int nu[3];
        for (int d = 0; d < 3; ++d) {
          const int e = qb[d] * (d == pax ? 2 : 1);
          nu[d] = (L[d] + e - 1) / e;
          long long sd = 0;
          for (int i = 0; i < nu[d]; ++i) {
            const int o = i * e;
            long long c = na_host_count(o, qb[d], K[d], L[d], kb[d]);
            if (d == pax) c = std::max(c, na_host_count(o + qb[d], qb[d], K[d], L[d], kb[d]));
            sd += c;
          }
          steps *= sd;
          units *= nu[d];
        }
        const long long cost = steps + kNaUnitCost * units;
        if (best_cost < 0 || cost < best_cost) {
          best_cost = cost;
          best = NaChoice{{qb[0], qb[1], qb[2]}, pax, {nu[0], nu[1], nu[2]}, steps};
        }
      }
    }
  return best;
}

// Number of SMs of the current device (cached per device).
int sm_count(int* out) {
  static std::atomic<int> cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_CUDA;
  if (dev >= 0 && dev < 64 && cache[dev].load() > 0) {
    *out = cache[dev].load();
    return DIT_OK;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return DIT_ERR_CUDA;
  if (dev >= 0 && dev < 64) cache[dev].store(n);
  *out = n;
  return DIT_OK;
}

// Raise the dynamic shared-memory limit of a kernel once per device.
template <typename K>
int ensure_smem_attr(K kernel, int bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  if (done_mask.load() & bit) return DIT_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return DIT_ERR_CUDA;
  done_mask.fetch_or(bit);
  return DIT_OK;
}

// The forward kernel re-splits registers between warpgroups with setmaxnreg; the increase
// only completes if the block was launched with at least the registers the split adds up to.
// Refuse to launch a build where that does not hold (it would wait forever).
template <int D, bool FP8, bool NA, bool PARTS>
int check_register_split() {
  using C = AttnCfg<D, FP8>;
  static std::atomic<int> split_state{0};   // 0 unknown, 1 ok, 2 bad
  int v = split_state.load();
  if (v == 0) {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, attn_fwd_kernel<D, FP8, NA, PARTS>) != cudaSuccess) return DIT_ERR_CUDA;
    const long long launched = static_cast<long long>(attr.numRegs) * C::kThreads;
    const long long wanted = 2LL * 128 * C::kRegsSoftmax + 128LL * C::kRegsCtl;
    v = (attr.numRegs == C::kRegsLaunch && launched >= wanted) ? 1 : 2;
    split_state.store(v);
  }
  return v == 1 ? DIT_OK : DIT_ERR_UNSUPPORTED;
}

// Parts launch: per part p a 4-D map (D, part_rows, H, B) over heads [h0, h0 + H) of the
// part's [B, part_H, part_rows, D] tensor (the address may belong to a peer GPU).
int make_map_part(CUtensorMap* m, const void* ptr, int D, int part_rows, int H, int B, int part_H, int h0) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return DIT_ERR_CUDA;
  const cuuint64_t e = 2;
  const char* base = static_cast<const char*>(ptr) + static_cast<size_t>(h0) * part_rows * D * e;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(part_rows), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * e, static_cast<cuuint64_t>(part_rows) * D * e,
                           static_cast<cuuint64_t>(part_H) * part_rows * D * e};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / e), 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<char*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DIT_OK : DIT_ERR_CUDA;
}

// Q/K/V pointers of a launch: one tensor each, or one per part.
struct QKV {
  const void* q[kMaxParts];
  const void* k[kMaxParts];
  const void* v[kMaxParts];
};

template <int D, bool FP8, bool NA = false, bool PARTS = false>
int launch_attn(const QKV& in, const AttnParams& prm, cudaStream_t st) {
  using C = AttnCfg<D, FP8>;
  static std::atomic<uint64_t> attr_done{0};
  int rc = check_register_split<D, FP8, NA, PARTS>();
  if (rc != DIT_OK) return rc;
  constexpr int kSmem = AttnSmem<D, FP8, NA>::kBytes;
  rc = ensure_smem_attr(attn_fwd_kernel<D, FP8, NA, PARTS>, kSmem, attr_done);
  if (rc != DIT_OK) return rc;
  MapSet<PARTS ? kMaxParts : 1> maps;
  std::memset(&maps, 0, sizeof(maps));
  CUtensorMap& tq = maps.q[0];
  CUtensorMap& tk = maps.k[0];
  CUtensorMap& tv = maps.v[0];
  const void* q = in.q[0];
  const void* k = in.k[0];
  const void* v = in.v[0];
  const int BH = prm.B * prm.H;
  AttnParams pr = prm;
  if constexpr (PARTS) {
    for (int pt = 0; pt < prm.n_q_parts; ++pt)
      if ((rc = make_map_part(&maps.q[pt], in.q[pt], D, prm.part_rows, prm.H, prm.B, prm.part_H, prm.part_h0)) != DIT_OK)
        return rc;
    for (int pt = 0; pt < prm.n_kv_parts; ++pt) {
      if ((rc = make_map_part(&maps.k[pt], in.k[pt], D, prm.part_rows, prm.H, prm.B, prm.part_H, prm.part_h0)) != DIT_OK)
        return rc;
      if ((rc = make_map_part(&maps.v[pt], in.v[pt], D, prm.part_rows, prm.H, prm.B, prm.part_H, prm.part_h0)) != DIT_OK)
        return rc;
    }
    pr.n_qblk = (prm.S_q + 2 * C::kBM - 1) / (2 * C::kBM);
    const long long units = static_cast<long long>(pr.n_qblk) * prm.H * prm.B;
    if (units > 0x7FFFFFFFLL) return DIT_ERR_INVALID_ARG;
    pr.n_units = static_cast<int>(units);
  } else if constexpr (NA) {
    const int L[3] = {prm.na_T, prm.na_Y, prm.na_X}, K[3] = {prm.na_Kt, prm.na_Ky, prm.na_Kx};
    const NaChoice ch = na_choose(L, K);
    if ((rc = make_map_na(&tq, q, D, prm.na_T, prm.na_Y, prm.na_X, BH, ch.qb[0], ch.qb[1], ch.qb[2])) != DIT_OK)
      return rc;
    if ((rc = make_map_na(&tk, k, D, prm.na_T, prm.na_Y, prm.na_X, BH, kNaBt, kNaBy, kNaBx)) != DIT_OK) return rc;
    if ((rc = make_map_na(&tv, v, D, prm.na_T, prm.na_Y, prm.na_X, BH, kNaBt, kNaBy, kNaBx)) != DIT_OK) return rc;
    pr.na_qbt = ch.qb[0]; pr.na_qby = ch.qb[1]; pr.na_qbx = ch.qb[2]; pr.na_pax = ch.pax;
    pr.na_nut = ch.nu[0]; pr.na_nuy = ch.nu[1]; pr.na_nux = ch.nu[2];
    const long long units = static_cast<long long>(BH) * ch.nu[0] * ch.nu[1] * ch.nu[2];
    if (units > 0x7FFFFFFFLL) return DIT_ERR_INVALID_ARG;
    pr.n_qblk = 0;
    pr.n_units = static_cast<int>(units);
  } else {
    if ((rc = make_map(&tq, q, FP8, D, prm.S_q, BH, prm.seg_q)) != DIT_OK) return rc;
    if ((rc = make_map(&tk, k, FP8, D, prm.S_kv, BH, prm.seg_kv)) != DIT_OK) return rc;
    if ((rc = make_map(&tv, v, FP8, D, prm.S_kv, BH, prm.seg_kv)) != DIT_OK) return rc;
    pr.n_qblk = (prm.S_q + 2 * C::kBM - 1) / (2 * C::kBM);
    const long long units = static_cast<long long>(pr.n_qblk) * prm.H * prm.B;
    if (units > 0x7FFFFFFFLL) return DIT_ERR_INVALID_ARG;
    pr.n_units = static_cast<int>(units);
  }
  int sms = 0;
  if ((rc = sm_count(&sms)) != DIT_OK) return rc;
  // persistent: at most one CTA per SM, minus the SMs reserved for concurrent kernels
  const int reserve = g_sm_reserve.load();
  const int slots = sms - reserve > 1 ? sms - reserve : 1;
  const int grid = pr.n_units < slots ? pr.n_units : slots;
  attn_fwd_kernel<D, FP8, NA, PARTS><<<grid, C::kThreads, kSmem, st>>>(maps, pr);
  return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

int grid_for(long long units, int threads, int max_blocks) {
  long long g = (units + threads - 1) / threads;
  if (g < 1) g = 1;
  if (g > max_blocks) g = max_blocks;
  return static_cast<int>(g);
}

__global__ void selftest_wait_kernel(unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, timeout_ns, 0xEE);  // nothing arrives
}

}  // namespace

// ---------------------------------------------------------------------------------------
// Scratch of dit_quant_fp8_noalloc: one partial absolute maximum per block of the first
// quantisation pass.  It is part of the loaded module, so every GPU that loads this library
// holds these 4736 bytes until the process exits; no call allocates anything.  Host code must
// not hand this name to a kernel (on the host it is only a stand-in for the symbol): the
// device address is looked up once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------------------
constexpr int kNoAllocScratchFloats = dit::kQuantMaxBlocks;
static __device__ __align__(256) float g_quant_noalloc_scratch[kNoAllocScratchFloats];
static_assert(dit::kQuantMaxBlocks <= kNoAllocScratchFloats, "scratch must hold every partial maximum");

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_scratch_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry-point lookup (no libcuda link).
CtxGetCurrentFn ctx_current_fn() {
  static std::once_flag once;
  static CtxGetCurrentFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of the static scratch on the current device.  Set-up happens on the first
// call per device, and again if the device's context has changed since (a cudaDeviceReset
// reloads the module, which may move the array): the cached address belongs to the context
// it was looked up in.
int noalloc_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DIT_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DIT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext ctx = nullptr;
  CtxGetCurrentFn cur = ctx_current_fn();
  if (g_noalloc_scratch_ptr[dev] != nullptr) {
    // the runtime has made the device's context current by now (cudaGetDevice does not, so
    // ask the driver only when there is a cached address to validate)
    if (cur == nullptr || cur(&ctx) != CUDA_SUCCESS) return DIT_ERR_CUDA;
  }
  if (g_noalloc_scratch_ptr[dev] == nullptr || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_quant_noalloc_scratch) != cudaSuccess || p == nullptr) return DIT_ERR_CUDA;
    if (cur == nullptr || cur(&ctx) != CUDA_SUCCESS) return DIT_ERR_CUDA;
    g_noalloc_scratch_ptr[dev] = static_cast<float*>(p);
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_scratch_ptr[dev];
  return DIT_OK;
}

}  // namespace

namespace {

// Per-block e4m3 descales (all three null for per-tensor scales).
struct BlockScales {
  const float* dq = nullptr;
  const float* dk = nullptr;
  const float* dv = nullptr;
};

int attn_chunk_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H, int S_q,
                    int S_kv, int D, int k0, int k1, float scale, int dtype, int out_dtype,
                    const float* descale_qkv, void* stream, bool accumulate, const BlockScales& bs = BlockScales(),
                    int seg = 0) {
  const bool blocks = bs.dq != nullptr || bs.dk != nullptr || bs.dv != nullptr;
  // seg > 0: q, k, v, out and lse in sequence segments of seg rows (S_q == S_kv, k0 = 0)
  if (seg < 0) return DIT_ERR_INVALID_ARG;
  if (seg > 0) {
    if (S_q != S_kv || k0 != 0 || k1 != S_kv || S_q % seg != 0) return DIT_ERR_INVALID_ARG;
    if (seg != S_q && seg % 128 != 0) return DIT_ERR_UNSUPPORTED;   // tiles must not straddle segments
  }
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || S_q < 1 || S_kv < 1 || B > 65535 || H > 65535) return DIT_ERR_INVALID_ARG;
  if (k0 < 0 || k1 < k0 || k1 > S_kv) return DIT_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return DIT_ERR_INVALID_ARG;
  if (dtype != DIT_BF16 && dtype != DIT_FP8_E4M3) return DIT_ERR_INVALID_ARG;
  if (out_dtype != DIT_BF16 && out_dtype != DIT_FP32) return DIT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DIT_ERR_UNSUPPORTED;
  const bool fp8 = dtype == DIT_FP8_E4M3;
  if (fp8 && D != 128) return DIT_ERR_UNSUPPORTED;
  if (fp8 && !blocks && descale_qkv == nullptr) return DIT_ERR_INVALID_ARG;
  if (blocks) {
    if (!fp8 || bs.dq == nullptr || bs.dk == nullptr || bs.dv == nullptr) return DIT_ERR_INVALID_ARG;
    if (!aligned(bs.dq, 4) || !aligned(bs.dk, 4) || !aligned(bs.dv, 4)) return DIT_ERR_MISALIGNED;
    if (k0 % 128 != 0) return DIT_ERR_UNSUPPORTED;   // KV tiles must coincide with scale blocks
  }
  if (static_cast<long long>(B) * H > 0x7FFFFFFFLL) return DIT_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return DIT_ERR_MISALIGNED;
  if (lse != nullptr && !aligned(lse, 4)) return DIT_ERR_MISALIGNED;
  if (descale_qkv != nullptr && !aligned(descale_qkv, 4)) return DIT_ERR_MISALIGNED;
  const size_t in_elem = fp8 ? 1 : 2, out_elem = out_dtype == DIT_FP32 ? 4 : 2;
  const size_t rows_q = static_cast<size_t>(B) * H * S_q, rows_kv = static_cast<size_t>(B) * H * S_kv;
  const size_t out_bytes = rows_q * D * out_elem;
  if (overlaps(out, out_bytes, q, rows_q * D * in_elem) || overlaps(out, out_bytes, k, rows_kv * D * in_elem) ||
      overlaps(out, out_bytes, v, rows_kv * D * in_elem))
    return DIT_ERR_INVALID_ARG;
  if (lse != nullptr && (overlaps(lse, rows_q * 4, out, out_bytes) || overlaps(lse, rows_q * 4, q, rows_q * D * in_elem) ||
                         overlaps(lse, rows_q * 4, k, rows_kv * D * in_elem) ||
                         overlaps(lse, rows_q * 4, v, rows_kv * D * in_elem)))
    return DIT_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  if (accumulate && k0 == k1) return DIT_OK;   // merging an empty range changes nothing
  if (k0 == k1) {
    const long long rows = static_cast<long long>(rows_q);
    attn_fill_empty_kernel<<<grid_for(rows * D, 256, 148 * 16), 256, 0, st>>>(out, lse, rows, D,
                                                                               out_dtype == DIT_FP32);
    return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
  }

  AttnParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.B = B; prm.H = H; prm.S_q = S_q; prm.S_kv = S_kv; prm.k0 = k0; prm.k1 = k1;
  prm.scale = scale;
  prm.descale = fp8 ? descale_qkv : nullptr;
  prm.out = out;
  prm.lse = lse;
  prm.out_fp32 = out_dtype == DIT_FP32;
  prm.accumulate = accumulate ? 1 : 0;
  prm.dq_blk = blocks ? bs.dq : nullptr;
  prm.dk_blk = blocks ? bs.dk : nullptr;
  prm.dv_blk = blocks ? bs.dv : nullptr;
  prm.nb_q = (S_q + 127) / 128;
  prm.nb_kv = (S_kv + 127) / 128;
  prm.seg_q = seg > 0 ? seg : S_q;
  prm.seg_kv = seg > 0 ? seg : S_kv;
  prm.timeout_ns = g_timeout_ns.load();
  QKV in;
  in.q[0] = q;
  in.k[0] = k;
  in.v[0] = v;
  if (fp8) return launch_attn<128, true>(in, prm, st);
  if (D == 64) return launch_attn<64, false>(in, prm, st);
  return launch_attn<128, false>(in, prm, st);
}

}  // namespace

extern "C" {

int dit_attn_fwd_chunk(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
                       int S_q, int S_kv, int D, int k0, int k1, float scale, int dtype, int out_dtype,
                       const float* descale_qkv, void* stream) {
  return attn_chunk_impl(q, k, v, out, lse, B, H, S_q, S_kv, D, k0, k1, scale, dtype, out_dtype, descale_qkv,
                         stream, false);
}

int dit_attn_fwd_chunk_acc(const void* q, const void* k, const void* v, float* acc_out, float* acc_lse, int B,
                           int H, int S_q, int S_kv, int D, int k0, int k1, float scale, int dtype,
                           const float* descale_qkv, void* stream) {
  if (acc_out == nullptr || acc_lse == nullptr) return DIT_ERR_INVALID_ARG;
  return attn_chunk_impl(q, k, v, acc_out, acc_lse, B, H, S_q, S_kv, D, k0, k1, scale, dtype, DIT_FP32,
                         descale_qkv, stream, true);
}

int dit_attn_fwd_fp8_blocks(const void* q8, const void* k8, const void* v8, const float* dq_blk, const float* dk_blk,
                            const float* dv_blk, void* out, float* lse, int B, int H, int S_q, int S_kv, int D,
                            int k0, int k1, float scale, int out_dtype, void* stream) {
  if (dq_blk == nullptr || dk_blk == nullptr || dv_blk == nullptr) return DIT_ERR_INVALID_ARG;
  BlockScales bs;
  bs.dq = dq_blk;
  bs.dk = dk_blk;
  bs.dv = dv_blk;
  return attn_chunk_impl(q8, k8, v8, out, lse, B, H, S_q, S_kv, D, k0, k1, scale, DIT_FP8_E4M3, out_dtype, nullptr,
                         stream, false, bs);
}

int dit_attn_fwd_seg(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H, int S,
                     int D, int seg, float scale, int dtype, int out_dtype, const float* descale_qkv,
                     void* stream) {
  if (seg < 1) return DIT_ERR_INVALID_ARG;
  return attn_chunk_impl(q, k, v, out, lse, B, H, S, S, D, 0, S, scale, dtype, out_dtype, descale_qkv, stream,
                         false, BlockScales(), seg);
}

int dit_na3d_plan(int T, int Y, int X, int Kt, int Ky, int Kx, int* q_brick, long long* units_per_head,
                  long long* steps_per_head) {
  if (q_brick == nullptr || units_per_head == nullptr || steps_per_head == nullptr) return DIT_ERR_INVALID_ARG;
  if (T < 1 || Y < 1 || X < 1 || static_cast<long long>(T) * Y * X > 0x7FFFFFFFLL) return DIT_ERR_INVALID_ARG;
  if (Kt < 1 || Ky < 1 || Kx < 1 || Kt % 2 == 0 || Ky % 2 == 0 || Kx % 2 == 0 || Kt > T || Ky > Y || Kx > X)
    return DIT_ERR_INVALID_ARG;
  const int L[3] = {T, Y, X}, K[3] = {Kt, Ky, Kx};
  const NaChoice ch = na_choose(L, K);
  for (int d = 0; d < 3; ++d) q_brick[d] = ch.qb[d];
  q_brick[3] = ch.pax;
  *units_per_head = static_cast<long long>(ch.nu[0]) * ch.nu[1] * ch.nu[2];
  *steps_per_head = ch.steps;
  return DIT_OK;
}

int dit_na3d_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H, int T, int Y,
                 int X, int D, int Kt, int Ky, int Kx, float scale, void* stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || T < 1 || Y < 1 || X < 1 || B > 65535 || H > 65535) return DIT_ERR_INVALID_ARG;
  if (Kt < 1 || Ky < 1 || Kx < 1 || Kt % 2 == 0 || Ky % 2 == 0 || Kx % 2 == 0 || Kt > T || Ky > Y || Kx > X)
    return DIT_ERR_INVALID_ARG;
  // (keys outside a query's window get a score penalty of -2^100, which must dominate
  // scale * log2(e) times any score difference)
  if (!(scale >= 1e-20f) || !std::isfinite(scale)) return DIT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DIT_ERR_UNSUPPORTED;
  const long long S = static_cast<long long>(T) * Y * X;
  if (S > 0x7FFFFFFFLL || static_cast<long long>(B) * H * S > (1LL << 40)) return DIT_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return DIT_ERR_MISALIGNED;
  if (lse != nullptr && !aligned(lse, 4)) return DIT_ERR_MISALIGNED;
  const size_t rows = static_cast<size_t>(B) * H * S, bytes = rows * D * 2;
  if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) || overlaps(out, bytes, v, bytes))
    return DIT_ERR_INVALID_ARG;
  if (lse != nullptr && (overlaps(lse, rows * 4, out, bytes) || overlaps(lse, rows * 4, q, bytes) ||
                         overlaps(lse, rows * 4, k, bytes) || overlaps(lse, rows * 4, v, bytes)))
    return DIT_ERR_INVALID_ARG;
  AttnParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.B = B; prm.H = H; prm.S_q = static_cast<int>(S); prm.S_kv = static_cast<int>(S);
  prm.k0 = 0; prm.k1 = static_cast<int>(S);
  prm.scale = scale;
  prm.out = out;
  prm.lse = lse;
  prm.seg_q = prm.S_q;
  prm.seg_kv = prm.S_kv;
  prm.na_T = T; prm.na_Y = Y; prm.na_X = X;
  prm.na_Kt = Kt; prm.na_Ky = Ky; prm.na_Kx = Kx;
  prm.timeout_ns = g_timeout_ns.load();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  QKV in;
  in.q[0] = q;
  in.k[0] = k;
  in.v[0] = v;
  if (D == 64) return launch_attn<64, false, true>(in, prm, st);
  return launch_attn<128, false, true>(in, prm, st);
}

int dit_attn_fwd_parts(const void* const* q_parts, int n_q_parts, const void* const* k_parts,
                       const void* const* v_parts, int n_kv_parts, void* const* out_parts, float* const* lse_parts,
                       int B, int part_H, int h0, int H, int part_rows, int D, float scale, void* stream) {
  if (q_parts == nullptr || k_parts == nullptr || v_parts == nullptr || out_parts == nullptr)
    return DIT_ERR_INVALID_ARG;
  if (n_q_parts < 1 || n_q_parts > kMaxParts || n_kv_parts < 1 || n_kv_parts > kMaxParts) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || part_rows < 1 || h0 < 0 || h0 + H > part_H || B > 65535 || part_H > 65535)
    return DIT_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return DIT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DIT_ERR_UNSUPPORTED;
  if ((n_q_parts > 1 || n_kv_parts > 1) && part_rows % 128 != 0) return DIT_ERR_UNSUPPORTED;   // no straddling
  const long long S_q = static_cast<long long>(n_q_parts) * part_rows;
  const long long S_kv = static_cast<long long>(n_kv_parts) * part_rows;
  if (S_q > 0x7FFFFFFFLL || S_kv > 0x7FFFFFFFLL) return DIT_ERR_INVALID_ARG;
  const size_t part_bytes = static_cast<size_t>(B) * part_H * part_rows * D * 2;
  for (int i = 0; i < n_kv_parts; ++i) {
    if (k_parts[i] == nullptr || v_parts[i] == nullptr) return DIT_ERR_INVALID_ARG;
    if (!aligned(k_parts[i], 16) || !aligned(v_parts[i], 16)) return DIT_ERR_MISALIGNED;
  }
  for (int i = 0; i < n_q_parts; ++i) {
    if (q_parts[i] == nullptr || out_parts[i] == nullptr) return DIT_ERR_INVALID_ARG;
    if (!aligned(q_parts[i], 16) || !aligned(out_parts[i], 16)) return DIT_ERR_MISALIGNED;
    if (lse_parts != nullptr && (lse_parts[i] == nullptr || !aligned(lse_parts[i], 4))) return DIT_ERR_INVALID_ARG;
    for (int j = 0; j < n_q_parts; ++j)
      if (overlaps(out_parts[i], part_bytes, q_parts[j], part_bytes) ||
          (i != j && overlaps(out_parts[i], part_bytes, out_parts[j], part_bytes)))
        return DIT_ERR_INVALID_ARG;
    for (int j = 0; j < n_kv_parts; ++j)
      if (overlaps(out_parts[i], part_bytes, k_parts[j], part_bytes) ||
          overlaps(out_parts[i], part_bytes, v_parts[j], part_bytes))
        return DIT_ERR_INVALID_ARG;
  }
  // An LSE block must not overlap any input or output block, nor another LSE block: the
  // kernel's LSE stores would otherwise race with TMA loads of the same bytes.
  const size_t lse_bytes = static_cast<size_t>(B) * part_H * part_rows * 4;
  if (lse_parts != nullptr) {
    for (int i = 0; i < n_q_parts; ++i) {
      const void* l = lse_parts[i];
      for (int j = 0; j < n_q_parts; ++j)
        if (overlaps(l, lse_bytes, q_parts[j], part_bytes) || overlaps(l, lse_bytes, out_parts[j], part_bytes) ||
            (i != j && overlaps(l, lse_bytes, lse_parts[j], lse_bytes)))
          return DIT_ERR_INVALID_ARG;
      for (int j = 0; j < n_kv_parts; ++j)
        if (overlaps(l, lse_bytes, k_parts[j], part_bytes) || overlaps(l, lse_bytes, v_parts[j], part_bytes))
          return DIT_ERR_INVALID_ARG;
    }
  }
  AttnParams prm;
  std::memset(&prm, 0, sizeof(prm));
  prm.B = B; prm.H = H; prm.S_q = static_cast<int>(S_q); prm.S_kv = static_cast<int>(S_kv);
  prm.k0 = 0; prm.k1 = static_cast<int>(S_kv);
  prm.scale = scale;
  prm.n_q_parts = n_q_parts; prm.n_kv_parts = n_kv_parts;
  prm.part_rows = part_rows; prm.part_H = part_H; prm.part_h0 = h0;
  QKV in;
  std::memset(&in, 0, sizeof(in));
  for (int i = 0; i < n_kv_parts; ++i) {
    in.k[i] = k_parts[i];
    in.v[i] = v_parts[i];
  }
  for (int i = 0; i < n_q_parts; ++i) {
    in.q[i] = q_parts[i];
    prm.out_parts[i] = out_parts[i];
    prm.lse_parts[i] = lse_parts != nullptr ? lse_parts[i] : nullptr;
  }
  prm.seg_q = prm.S_q;
  prm.seg_kv = prm.S_kv;
  prm.timeout_ns = g_timeout_ns.load();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 64) return launch_attn<64, false, false, true>(in, prm, st);
  return launch_attn<128, false, false, true>(in, prm, st);
}

int dit_ipc_export(const void* ptr, void* handle, long long* offset) {
  if (ptr == nullptr || handle == nullptr || offset == nullptr) return DIT_ERR_INVALID_ARG;
  MemGetAddressRangeFn range = addr_range_fn();
  if (range == nullptr) return DIT_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return DIT_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return DIT_ERR_CUDA;
  std::memcpy(handle, &h, sizeof(h));
  *offset = static_cast<long long>(reinterpret_cast<uintptr_t>(ptr) - static_cast<uintptr_t>(base));
  return DIT_OK;
}

int dit_ipc_import(const void* handle, long long offset, void** ptr, void** base) {
  if (handle == nullptr || ptr == nullptr || base == nullptr || offset < 0) return DIT_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* b = nullptr;
  if (cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return DIT_ERR_CUDA;
  *base = b;
  *ptr = static_cast<char*>(b) + offset;
  return DIT_OK;
}

int dit_ipc_close(void* base) {
  if (base == nullptr) return DIT_ERR_INVALID_ARG;
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

int dit_swap01_chunks(const void* src, void* dst, long long d0, long long d1, long long chunk_bytes,
                      void* stream) {
  if (src == nullptr || dst == nullptr || d0 < 1 || d1 < 1 || chunk_bytes < 16) return DIT_ERR_INVALID_ARG;
  if (chunk_bytes % 16 != 0) return DIT_ERR_UNSUPPORTED;
  if (!aligned(src, 16) || !aligned(dst, 16)) return DIT_ERR_MISALIGNED;
  if (d0 > (1LL << 40) / d1 || d0 * d1 > (1LL << 48) / chunk_bytes) return DIT_ERR_INVALID_ARG;
  const long long bytes = d0 * d1 * chunk_bytes;
  if (overlaps(dst, static_cast<size_t>(bytes), src, static_cast<size_t>(bytes))) return DIT_ERR_INVALID_ARG;
  const long long vecs = bytes / 16;
  swap01_chunks_kernel<<<grid_for(vecs, 256, 148 * 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), d0, d1, chunk_bytes / 16);
  return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

int dit_quant_fp8_blocks(const void* x_bf16, void* x_fp8, float* descales, int B, int H, int S, int D,
                         void* stream) {
  if (x_bf16 == nullptr || x_fp8 == nullptr || descales == nullptr) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || S < 1 || D < 8) return DIT_ERR_INVALID_ARG;
  if (D % 8 != 0 || D > 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned(x_bf16, 16) || !aligned(x_fp8, 8) || !aligned(descales, 4)) return DIT_ERR_MISALIGNED;
  const long long nblk = (S + 127) / 128;
  const long long grid = static_cast<long long>(B) * H * nblk;
  if (grid > 0x7FFFFFFFLL) return DIT_ERR_INVALID_ARG;
  const size_t n = static_cast<size_t>(B) * H * S * D;
  if (overlaps(x_fp8, n, x_bf16, 2 * n) || overlaps(descales, static_cast<size_t>(grid) * 4, x_bf16, 2 * n) ||
      overlaps(descales, static_cast<size_t>(grid) * 4, x_fp8, n))
    return DIT_ERR_INVALID_ARG;
  quant_e4m3_rows_kernel<<<static_cast<unsigned>(grid), kQuantRowThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(x_bf16), S, D, static_cast<int>(nblk), static_cast<uint8_t*>(x_fp8), descales,
      g_timeout_ns.load());
  return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

int dit_attn_acc_init(float* acc_out, float* acc_lse, int B, int H, int S, int D, void* stream) {
  if (acc_out == nullptr || acc_lse == nullptr || B < 1 || H < 1 || S < 1) return DIT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DIT_ERR_UNSUPPORTED;
  if (!aligned(acc_out, 16) || !aligned(acc_lse, 4)) return DIT_ERR_MISALIGNED;
  const long long rows = static_cast<long long>(B) * H * S;
  if (overlaps(acc_out, static_cast<size_t>(rows) * D * 4, acc_lse, static_cast<size_t>(rows) * 4))
    return DIT_ERR_INVALID_ARG;
  attn_fill_empty_kernel<<<grid_for(rows * D, 256, 148 * 16), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      acc_out, acc_lse, rows, D, 1);
  return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

int dit_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H, int S,
                 int D, float scale, int dtype, const float* descale_qkv, void* stream) {
  return dit_attn_fwd_chunk(q, k, v, out, lse, B, H, S, S, D, 0, S, scale, dtype, DIT_BF16, descale_qkv, stream);
}

int dit_attn_merge(const void* const* outs, const float* const* lses, int n_chunks, void* out, float* lse,
                   int B, int H, int S, int D, int in_dtype, int out_dtype, void* stream) {
  if (outs == nullptr || lses == nullptr || out == nullptr) return DIT_ERR_INVALID_ARG;
  if (n_chunks < 1 || n_chunks > kMaxMergeChunks) return DIT_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || S < 1) return DIT_ERR_INVALID_ARG;
  if (in_dtype != DIT_BF16 && in_dtype != DIT_FP32) return DIT_ERR_INVALID_ARG;
  if (out_dtype != DIT_BF16 && out_dtype != DIT_FP32) return DIT_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return DIT_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(B) * H * S;
  const size_t in_bytes = static_cast<size_t>(rows) * D * (in_dtype == DIT_FP32 ? 4 : 2);
  const size_t out_bytes = static_cast<size_t>(rows) * D * (out_dtype == DIT_FP32 ? 4 : 2);
  if (!aligned(out, 16) || (lse != nullptr && !aligned(lse, 4))) return DIT_ERR_MISALIGNED;
  MergeParams prm;
  std::memset(&prm, 0, sizeof(prm));
  for (int c = 0; c < n_chunks; ++c) {
    if (outs[c] == nullptr || lses[c] == nullptr) return DIT_ERR_INVALID_ARG;
    if (!aligned(outs[c], 16) || !aligned(lses[c], 4)) return DIT_ERR_MISALIGNED;
    if (overlaps(out, out_bytes, outs[c], in_bytes) || overlaps(out, out_bytes, lses[c], rows * 4))
      return DIT_ERR_INVALID_ARG;
    if (lse != nullptr && (overlaps(lse, rows * 4, outs[c], in_bytes) || overlaps(lse, rows * 4, lses[c], rows * 4)))
      return DIT_ERR_INVALID_ARG;
    prm.outs[c] = outs[c];
    prm.lses[c] = lses[c];
  }
  if (lse != nullptr && overlaps(lse, rows * 4, out, out_bytes)) return DIT_ERR_INVALID_ARG;
  prm.n = n_chunks;
  prm.out = out;
  prm.lse = lse;
  prm.rows = rows;
  prm.D = D;
  prm.in_fp32 = in_dtype == DIT_FP32;
  prm.out_fp32 = out_dtype == DIT_FP32;
  const long long units = rows * (D / 8);
  lse_merge_kernel<<<grid_for(units, 256, 148 * 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(prm);
  return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

size_t dit_quant_fp8_workspace_bytes(long long n) {
  return static_cast<size_t>(quant_blocks(n)) * sizeof(float);
}

int dit_quant_fp8(const void* x_bf16, void* x_fp8, float* descale, long long n, void* workspace,
                  size_t workspace_bytes, void* stream) {
  if (x_bf16 == nullptr || x_fp8 == nullptr || descale == nullptr || workspace == nullptr) return DIT_ERR_INVALID_ARG;
  if (n < 1) return DIT_ERR_INVALID_ARG;
  if (workspace_bytes < dit_quant_fp8_workspace_bytes(n)) return DIT_ERR_INVALID_ARG;
  if (!aligned(x_bf16, 16) || !aligned(x_fp8, 16) || !aligned(descale, 4) || !aligned(workspace, 4))
    return DIT_ERR_MISALIGNED;
  if (overlaps(x_fp8, n, x_bf16, n * 2) || overlaps(workspace, workspace_bytes, x_bf16, n * 2) ||
      overlaps(workspace, workspace_bytes, x_fp8, n) || overlaps(descale, 4, x_bf16, n * 2) ||
      overlaps(descale, 4, x_fp8, n) || overlaps(descale, 4, workspace, workspace_bytes))
    return DIT_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int g = quant_blocks(n);
  float* partials = static_cast<float*>(workspace);
  absmax_partial_kernel<<<g, kQuantThreads, 0, st>>>(static_cast<const uint16_t*>(x_bf16), n, partials);
  if (cudaGetLastError() != cudaSuccess) return DIT_ERR_CUDA;
  quant_e4m3_kernel<<<g, kQuantThreads, 0, st>>>(static_cast<const uint16_t*>(x_bf16), n, partials, g,
                                                  static_cast<uint8_t*>(x_fp8), descale);
  return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

int dit_quant_fp8_noalloc(const void* x_bf16, void* x_fp8, float* descale, long long n, void* stream) {
  if (x_bf16 == nullptr || x_fp8 == nullptr || descale == nullptr) return DIT_ERR_INVALID_ARG;
  if (n < 1) return DIT_ERR_INVALID_ARG;
  if (!aligned(x_bf16, 16) || !aligned(x_fp8, 16) || !aligned(descale, 4)) return DIT_ERR_MISALIGNED;
  if (overlaps(x_fp8, n, x_bf16, n * 2) || overlaps(descale, 4, x_bf16, n * 2) || overlaps(descale, 4, x_fp8, n))
    return DIT_ERR_INVALID_ARG;
  const int g = quant_blocks(n);
  if (g > kNoAllocScratchFloats) return DIT_ERR_UNSUPPORTED;  // more partials than the static scratch holds
  float* scratch = nullptr;
  const int rc = noalloc_scratch(&scratch);
  if (rc != DIT_OK) return rc;
  // Pass 1 writes every slot 0..g-1 before pass 2 reads them, so nothing needs clearing.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  absmax_partial_kernel<<<g, kQuantThreads, 0, st>>>(static_cast<const uint16_t*>(x_bf16), n, scratch);
  if (cudaGetLastError() != cudaSuccess) return DIT_ERR_CUDA;
  quant_e4m3_kernel<<<g, kQuantThreads, 0, st>>>(static_cast<const uint16_t*>(x_bf16), n, scratch, g,
                                                  static_cast<uint8_t*>(x_fp8), descale);
  return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

int dit_device_status(int* status, int clear) {
  if (status == nullptr) return DIT_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return DIT_ERR_CUDA;
  unsigned int w = 0;
  if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return DIT_ERR_CUDA;
  *status = static_cast<int>(w);
  if (clear) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return DIT_ERR_CUDA;
  }
  return DIT_OK;
}

int dit_set_wait_timeout_us(unsigned long long timeout_us) {
  g_timeout_ns.store(timeout_us == 0 ? 1000000000ull : timeout_us * 1000ull);
  return DIT_OK;
}

int dit_set_sm_reserve(int n_sms) {
  if (n_sms < 0 || n_sms > 1024) return DIT_ERR_INVALID_ARG;
  g_sm_reserve.store(n_sms);
  return DIT_OK;
}

int dit_selftest_wait_timeout(unsigned long long timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 10000000ull) return DIT_ERR_INVALID_ARG;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

const char* dit_status_str(int status) {
  switch (status & 0xFF) {
    case DIT_OK: return "DIT_OK";
    case DIT_ERR_INVALID_ARG: return "DIT_ERR_INVALID_ARG";
    case DIT_ERR_UNSUPPORTED: return "DIT_ERR_UNSUPPORTED";
    case DIT_ERR_MISALIGNED: return "DIT_ERR_MISALIGNED";
    case DIT_ERR_CUDA: return "DIT_ERR_CUDA";
    case DIT_ERR_TIMEOUT: return "DIT_ERR_TIMEOUT";
    default: return "DIT_ERR_UNKNOWN";
  }
}

int dit_version(void) { return 100; }

}  // extern "C"
