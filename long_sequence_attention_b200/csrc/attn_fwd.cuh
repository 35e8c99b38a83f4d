// Flash-style forward attention for sm_100a: TMA-staged Q/K/V tiles, tcgen05 MMAs with
// S = Q K^T and O += P V accumulated in TMEM, online softmax in registers.
//
// What it computes (joint image+text self-attention of a DiT block; the xDiT overview page,
// section 2.1, describes DiT inference as prefill-like and compute-bound, with every token
// attending to every token and no KV cache): for each (b, h) and query row i, over the keys
// k0 <= j < k1,
//     out_i = sum_j softmax_j(scale * q_i . k_j) v_j,   lse_i = log sum_j exp(scale * q_i . k_j).
// The KV-range form is the per-block step of the USP "Ring" dimension (xDiT overview,
// section 3.2.2): a ring step attends the local queries to one block of keys and the partial
// results are combined afterwards by the log-sum-exp merge (merge.cuh).
//
// Work unit: (b, h, 256 query rows) = two 128-row Q tiles that ping-pong, so the
// exponentials of one tile overlap the tensor-core work of the other.  The kernel is
// persistent: a grid of at most one CTA per SM walks the units u = blockIdx.x + k*gridDim.x
// (query block fastest, so the CTAs running at the same time share a head's K/V in L2).
// Barrier phases and ring stages follow a per-CTA running count g of KV steps (every role
// adds each unit's step count, which varies per unit only in the neighborhood form, where
// each Q tile also has its own K / V ring slots), so the next unit's Q load, its first S MMAs
// and this unit's epilogue overlap.
//
// Instantiations (template <D, FP8, NA, PARTS>): the dense form (bf16 D = 64 / 128, e4m3
// D = 128, per-tensor or per-block scales, plain or sequence-segmented layouts, optional
// running (O, LSE) accumulator); NA, 3-D neighborhood attention, where a tile is a brick of
// tokens, each Q brick visits only the KV bricks of its own rows' windows, and the keys of a
// brick outside a row's window get a score penalty from one more step of the S MMA; PARTS,
// where the query and key rows lie in blocks held by several ranks
// (possibly other GPUs) and every tile is loaded from the block that holds it.
//
// Warp roles (384 threads = 3 warpgroups):
//   warps 0-3  softmax warpgroup for Q tile 0 (thread = one query row = one TMEM lane)
//   warps 4-7  softmax warpgroup for Q tile 1
//   warp  8    MMA issuer (one thread issues every tcgen05.mma and commit; NA: each tile's
//              next P.V + S in whichever order the two tiles become ready)
//   warp  9    TMA producer (Q once, then a ring of K stages and a ring of V stages)
//   warp  10   NA only: TMA producer of Q tile 1's K and V tiles (warp 9 then loads tile 0's)
//   warps 10-11 otherwise idle (they complete the third warpgroup)
// The block launches with 168 registers per thread; the third warpgroup then gives
// registers back (setmaxnreg.dec to kRegsCtl) and the softmax warpgroups take them
// (setmaxnreg.inc to kRegsSoftmax): 2*128*216 + 128*72 = 64512 = 384*168, so the increase
// never waits on registers that do not exist.  The host checks the compiled register count
// against that sum before the first launch.
//
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).  P (bf16 or
// e4m3) is written over the first columns of S and read from TMEM by the P.V MMA.
//
// Ordering facts the pipeline relies on:
//   * MMAs issued by one thread execute in order, and tcgen05.commit fires only when every
//     earlier MMA of that thread is done.  The MMA thread issues  PV_t(j-1)  before  S_t(j)
//     for each tile t, so when the softmax warpgroup sees S_t(j) ready, PV_t(j-1) has also
//     finished: O_t is quiescent and the warpgroup may rescale it in place before it
//     publishes P_t(j).  It also means S_t(j) never overwrites P_t(j-1) while it is read.
//   * Max tracking is lazy: a row keeps its running max m_use until a new tile raises the
//     max by more than kRescaleLog2 (in log2 units); until then p = 2^(c(x - m_use)) may
//     exceed 1 but stays <= 2^kRescaleLog2, which bf16 / fp32 hold exactly enough.  The final
//     normalisation uses the same m_use for l and O, so the result is exact up to rounding.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ptx.cuh"

namespace dit {

struct AttnParams {
  int B, H, S_q, S_kv;
  int n_qblk;              // ceil(S_q / 256) query blocks per head
  int n_units;             // n_qblk * H * B
  int k0, k1;
  float scale;             // softmax scale applied to q.k
  const float* descale;    // e4m3 path: device pointer to {descale_q, descale_k, descale_v}
  void* out;               // [B,H,S_q,D] bf16 or fp32
  float* lse;              // [B,H,S_q] natural-log LSE, may be null
  int out_fp32;
  int accumulate;          // 1: out (fp32) and lse hold a running (O, LSE); merge this range into them
  // e4m3 with per-block scales (else null): descales of 128-row blocks per (b, h),
  // dq_blk [B*H, nb_q], dk_blk / dv_blk [B*H, nb_kv]; k0 is then a multiple of 128
  const float* dq_blk;
  const float* dk_blk;
  const float* dv_blk;
  int nb_q, nb_kv;
  // Sequence segments: row r of head bh lives at ((r / seg) * B*H + bh) * seg + r % seg (the
  // layout [S/seg, B*H, seg, D] that an all-to-all over the sequence leaves behind).
  // seg = S is the plain [B, H, S, D] layout.
  int seg_q, seg_kv;
  // Neighborhood attention (the NA instantiation only): T x Y x X token grid, odd window
  // sizes, the Q brick (t, y, x extents, product 128), the axis along which the two Q bricks
  // of a unit lie next to each other (0 = t, 1 = y, 2 = x), and the unit grid.
  int na_T, na_Y, na_X;
  int na_Kt, na_Ky, na_Kx;
  int na_qbt, na_qby, na_qbx, na_pax;
  int na_nut, na_nuy, na_nux;
  // Parts (the PARTS instantiation only): the keys are n_kv_parts blocks and the queries
  // n_q_parts blocks of part_rows rows each, block p held by tensors [B, part_H, part_rows, D]
  // at (possibly a peer GPU's) addresses; this launch computes heads [part_h0, part_h0 + H)
  // and writes the rows of query block p into out_parts[p] / lse_parts[p] (same layout).
  int n_q_parts, n_kv_parts, part_rows, part_H, part_h0;
  void* out_parts[8];
  float* lse_parts[8];
  unsigned long long timeout_ns;
};

constexpr int kMaxParts = 8;

// Tensor maps of one launch: one each for Q, K, V, or one per part.
template <int NM>
struct MapSet {
  CUtensorMap q[NM];
  CUtensorMap k[NM];
  CUtensorMap v[NM];
};

// ---------------------------------------------------------------------------------------
// Neighborhood attention geometry (the operation NATTEN calls na3d; the LTX notes page,
// section 5, reports it as the decoder's hot spot).  The neighborhood of a query at
// position i along a dimension of length L is the K positions starting at
// clamp(i - K/2, 0, L - K); the 3-D neighborhood is the product over (t, y, x).
// A 128-row Q tile is a brick of qbt x qby x qbx tokens and a KV tile a brick of
// kNaBt x kNaBy x kNaBx tokens, each loaded by one 5-D TMA box (x fastest), so tile row c is
// token (c / (by * bx), (c / bx) % by, c % bx) of its brick.  A unit is two Q bricks side by
// side along one axis (the two ping-pong tiles); each Q brick has its own list of KV bricks,
// laid from the origin of the union of its rows' windows (TMA boxes may start at any token;
// only the innermost D coordinate has an alignment rule), and each row masks the keys outside
// its own window.  A unit takes as many KV steps as the longer of its two lists; the other
// tile's extra steps are empty (no exponentials, P = 0).
// ---------------------------------------------------------------------------------------
constexpr int kNaBt = 4, kNaBy = 4, kNaBx = 8;

__device__ __forceinline__ int na_wstart(int i, int K, int L) { return min(max(i - K / 2, 0), L - K); }

struct NaTile {
  int qt, qy, qx;        // token origin of the Q brick
  int ut, uy, ux;        // token origin of the union of its rows' windows
  int nt, ny, nx;        // KV bricks along t, y, x (all 0 for a Q brick past the grid)
  __device__ __forceinline__ int n() const { return nt * ny * nx; }
  // token origin of KV tile j (x fastest, then y, then t)
  __device__ __forceinline__ void kv_origin(int j, int& t, int& y, int& x) const {
    const int jx = j % nx, jy = (j / nx) % ny, jt = j / (nx * ny);
    t = ut + jt * kNaBt;
    y = uy + jy * kNaBy;
    x = ux + jx * kNaBx;
  }
};

// Union [first, first + len) of the windows of the queries [a, min(a + ext, L)) along one
// dimension (window starts never decrease with the position), covered by `count` bricks of b;
// no queries (a >= L) gives count 0.
__device__ __forceinline__ void na_span(int a, int ext, int K, int L, int b, int& first, int& count) {
  if (a >= L) {
    first = 0;
    count = 0;
    return;
  }
  const int last = min(a + ext, L) - 1;
  first = na_wstart(a, K, L);
  count = (na_wstart(last, K, L) + K - first + b - 1) / b;
}

// Head index of unit u and Q tile t (0 or 1) of it.
__device__ __forceinline__ int na_unit_bh(const AttnParams& p, int u) {
  return u / (p.na_nut * p.na_nuy * p.na_nux);
}
__device__ __forceinline__ NaTile na_tile(const AttnParams& p, int u, int t) {
  NaTile w;
  const int per_bh = p.na_nut * p.na_nuy * p.na_nux;
  const int r = u % per_bh;
  const int ix = r % p.na_nux, iy = (r / p.na_nux) % p.na_nuy, it = r / (p.na_nux * p.na_nuy);
  const int et = p.na_qbt * (p.na_pax == 0 ? 2 : 1);
  const int ey = p.na_qby * (p.na_pax == 1 ? 2 : 1);
  const int ex = p.na_qbx * (p.na_pax == 2 ? 2 : 1);
  w.qt = it * et + (p.na_pax == 0 ? t * p.na_qbt : 0);
  w.qy = iy * ey + (p.na_pax == 1 ? t * p.na_qby : 0);
  w.qx = ix * ex + (p.na_pax == 2 ? t * p.na_qbx : 0);
  na_span(w.qt, p.na_qbt, p.na_Kt, p.na_T, kNaBt, w.ut, w.nt);
  na_span(w.qy, p.na_qby, p.na_Ky, p.na_Y, kNaBy, w.uy, w.ny);
  na_span(w.qx, p.na_qbx, p.na_Kx, p.na_X, kNaBx, w.ux, w.nx);
  if (w.nt == 0 || w.ny == 0 || w.nx == 0) w.nt = w.ny = w.nx = 0;
  return w;
}

// KV steps of unit u: the longer of its two tiles' lists (tile 0 always lies in the grid).
__device__ __forceinline__ int na_steps(const AttnParams& p, int u) {
  return max(na_tile(p, u, 0).n(), na_tile(p, u, 1).n());
}

// Window penalties.  Every S tile of the NA form gets one more K = 16 MMA step: a 16-feature
// row per query (A operand) times a 16-feature row per key (B operand).  Key c of a KV brick
// carries one-hot features of its brick position: feature ct = c / 32 (t), 4 + cy with
// cy = (c / 8) % 4 (y), 8 + cx with cx = c % 8 (x).  A query row carries, for the brick being
// visited, -kNaPen at each position whose coordinate lies outside its window along that axis
// and 0 elsewhere, so the extra step adds 0 to every key in the row's window (exact) and at
// most -3 kNaPen to the others, whose exponentials then vanish.  Both operands are K-major
// without swizzle: row r's 32 bytes at (r / 8) * 256 + (r % 8) * 16, features 8-15 128 bytes
// further on.
constexpr uint32_t kNaPenBits = 0xF180u;   // bf16 -2^100
constexpr uint32_t kNaOneBits = 0x3F80u;   // bf16 1.0
constexpr int kNaXBytes = 128 * 32;        // one 128-row feature block

// Write the penalty features of one query row (window starts wt, wy, wx) for the KV brick at
// token origin (ot, oy, ox) into block sX.
__device__ __forceinline__ void na_write_pen(uint8_t* sX, int row, int wt, int wy, int wx, int Kt, int Ky, int Kx,
                                             int ot, int oy, int ox) {
  auto pen = [](int v, int lo, int K) -> uint32_t { return (v >= lo && v < lo + K) ? 0u : kNaPenBits; };
  uint32_t h[8];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    h[i] = pen(ot + 2 * i, wt, Kt) | (pen(ot + 2 * i + 1, wt, Kt) << 16);
    h[2 + i] = pen(oy + 2 * i, wy, Ky) | (pen(oy + 2 * i + 1, wy, Ky) << 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) h[4 + i] = pen(ox + 2 * i, wx, Kx) | (pen(ox + 2 * i + 1, wx, Kx) << 16);
  uint8_t* base = sX + (row >> 3) * 256 + (row & 7) * 16;
  *reinterpret_cast<uint4*>(base) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(base + 128) = make_uint4(h[4], h[5], h[6], h[7]);
}

// Write the one-hot position features of key c of a KV brick into block sX.
__device__ __forceinline__ void na_write_keyfeat(uint8_t* sX, int c) {
  const int ft = c >> 5, fy = 4 + ((c >> 3) & 3), fx = 8 + (c & 7);
  uint32_t h[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int f0 = 2 * i, f1 = 2 * i + 1;
    h[i] = ((f0 == ft || f0 == fy || f0 == fx) ? kNaOneBits : 0u) |
           (((f1 == ft || f1 == fy || f1 == fx) ? kNaOneBits : 0u) << 16);
  }
  uint8_t* base = sX + (c >> 3) * 256 + (c & 7) * 16;
  *reinterpret_cast<uint4*>(base) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4*>(base + 128) = make_uint4(h[4], h[5], h[6], h[7]);
}

// Token of row `row` of Q brick w and the starts of its window.
__device__ __forceinline__ void na_row_geo(const AttnParams& p, const NaTile& w, int row, int& qt, int& qy, int& qx,
                                           int& wt, int& wy, int& wx) {
  qt = w.qt + row / (p.na_qby * p.na_qbx);
  qy = w.qy + (row / p.na_qbx) % p.na_qby;
  qx = w.qx + row % p.na_qbx;
  wt = na_wstart(qt, p.na_Kt, p.na_T);
  wy = na_wstart(qy, p.na_Ky, p.na_Y);
  wx = na_wstart(qx, p.na_Kx, p.na_X);
}

// exp2 on the FMA pipe, two values at once with packed fp32x2 instructions: x = n + f with
// n = rint(x), f in [-1/2, 1/2]; 2^f by a degree-3 polynomial (minimax in relative error,
// max 7.5e-5; coefficients from fit_exp2_poly.py); 2^n by adding n to the exponent field.
// x is clamped to [-125, 126] so the exponent field neither underflows nor runs into the
// sign bit: 2^-125 stands in for 0 (it only ever multiplies V values), and any x above 126
// gives about 2^126, far above every row-sum bound, so a speculative tile whose scores rose
// that far is always redone exactly.  Adding 1.5 * 2^23 rounds x to an integer whose low
// bits (two's complement) are n; shifting them into the exponent field adds n.
__device__ __forceinline__ void exp2_fma2(float x0, float x1, float& e0, float& e1) {
  const uint64_t x = f2_pack(fminf(fmaxf(x0, -125.0f), 126.0f), fminf(fmaxf(x1, -125.0f), 126.0f));
  const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);
  const uint64_t t = f2_add(x, magic);
  const uint64_t f = f2_sub(x, f2_sub(t, magic));
  uint64_t p = f2_fma(f2_pack(0.0551716685295105f, 0.0551716685295105f), f,
                      f2_pack(0.2426111251115799f, 0.2426111251115799f));
  p = f2_fma(p, f, f2_pack(0.6932609677314758f, 0.6932609677314758f));
  p = f2_fma(p, f, f2_pack(0.9999280571937561f, 0.9999280571937561f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  e0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  e1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

template <int D, bool FP8>
struct AttnCfg {
  static constexpr int kBM = 128;                       // query rows per tile
  static constexpr int kBN = 128;                       // keys per KV tile
  static constexpr int kElem = FP8 ? 1 : 2;             // bytes per element
  static constexpr int kRowBytes = D * kElem;           // bytes of one row
  static constexpr int kBlkBytes = 128 * 128;           // one 128-row x 128-byte swizzle block
  static constexpr int kNBlk = kRowBytes / 128;         // 128-byte column blocks per row
  static constexpr int kTileBytes = 128 * kRowBytes;
  static constexpr int kBoxInner = 128 / kElem;         // TMA box width in elements
  static constexpr int kKStages = (kTileBytes >= 32768) ? 2 : 4;
  static constexpr int kVStages = kKStages;
  static constexpr int kUmmaK = 32 / kElem;             // K per MMA instruction (32 bytes)
  static constexpr int kQKSteps = kRowBytes / 32;       // MMAs per S tile
  static constexpr int kPVSteps = kBN / kUmmaK;         // MMAs per P.V
  static constexpr int kThreads = 384;
  static constexpr int kRegsLaunch = 168;      // per thread at launch (__launch_bounds__(384, 1))
  static constexpr int kRegsSoftmax = 216;     // softmax warpgroups after setmaxnreg.inc
  static constexpr int kRegsCtl = 72;          // MMA / TMA warpgroup after setmaxnreg.dec
  static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsCtl <= kThreads * kRegsLaunch, "register split");
  static constexpr int kMmaWarp = 8;
  static constexpr int kTmaWarp = 9;
  static constexpr int kTmemCols = 512;
  static constexpr int kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
  // P is kept <= 2^(kRescaleLog2 + kPShift); for e4m3 (max 448) it is shifted up so that
  // most probabilities are normal numbers rather than subnormals.
  static constexpr float kRescaleLog2 = FP8 ? 4.0f : 8.0f;
  static constexpr float kPShift = FP8 ? 4.0f : 0.0f;
  static constexpr float kSumBound = 256.0f;           // = 2^(kRescaleLog2 + kPShift)
  static constexpr int kPWordsHalf = FP8 ? 16 : 32;     // 32-bit P words per half row
  // exp2 split: bit i set = column pair i of every 8 uses the FMA-pipe polynomial instead of
  // the MUFU (measured best: none at bf16 D=128; pairs 3 and 7 at bf16 D=64 and for e4m3,
  // spread out so the polynomial's FMA work falls between MUFU instructions)
  static constexpr int kEmuMask = (FP8 || D == 64) ? 0x88 : 0x00;
  // bf16: exponentiate with the running max first and redo a tile exactly only when its row
  // sum exceeds kSumBound.  e4m3 P is shifted up by 2^kPShift, so its sums sit near the bound
  // and it always takes the max first.
  static constexpr bool kSpeculative = !FP8;

  // shared memory layout (offsets from a 1024-byte aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kKStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kVStages * kTileBytes;
  static constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 1 + 2;
  static constexpr int kOffMisc = kOffBar + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-byte alignment
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(!FP8 || D == 128, "e4m3 path is built for D = 128");
};

// Shared memory of one launch.  The NA form adds the window-penalty features after the
// barriers: one 4 KB block per Q tile and one for the keys.
template <int D, bool FP8, bool NA>
struct AttnSmem {
  using C = AttnCfg<D, FP8>;
  static constexpr int kOffX = ((C::kOffMisc + 16 + 1023) / 1024) * 1024;
  static constexpr int kBytes = NA ? kOffX + 3 * kNaXBytes + 1024 : C::kSmemBytes;
  static_assert(kBytes <= 227 * 1024, "shared memory budget");
};

// Columns c >= valid of a 128-column score row become -inf (keys past the range).
__device__ __forceinline__ void mask_tail(uint32_t (&s)[128], int valid) {
#pragma unroll
  for (int c = 0; c < 128; ++c)
    if (c >= valid) s[c] = 0xFF800000u;
}

// Row max of 128 scores: 8 independent chains of 3-input max.
__device__ __forceinline__ float row_max128(const uint32_t (&s)[128]) {
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    mx[i] = fmax3(__uint_as_float(s[i]), __uint_as_float(s[i + 8]), __uint_as_float(s[i + 16]));
#pragma unroll
  for (int c = 24; c < 120; c += 16)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      mx[i] = fmax3(mx[i], __uint_as_float(s[c + i]), __uint_as_float(s[c + 8 + i]));
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = fmaxf(mx[i], __uint_as_float(s[120 + i]));
  return fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// p = 2^(cl*s - mc) for the 128 scores of a row, two lanes per instruction; column pair c
// uses the FMA-pipe polynomial when bit c % 8 of kEmuMask is set, the MUFU ex2 otherwise.
// Writes the P words (bf16 pairs: 64 words, or e4m3 quads: 32 words) and the row sum.
template <bool FP8, int kEmuMask>
__device__ __forceinline__ void exp_pass(const uint32_t (&s)[128], float cl, float mc, uint32_t* pw, float& sum) {
  const uint64_t cl2 = f2_pack(cl, cl), nmc2 = f2_pack(-mc, -mc);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c2 = 0; c2 < 64; ++c2) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(s[2 * c2]), __uint_as_float(s[2 * c2 + 1])), cl2, nmc2);
    float x0, x1, e0, e1;
    f2_unpack(x, x0, x1);
    if ((kEmuMask >> (c2 & 7)) & 1) {
      exp2_fma2(x0, x1, e0, e1);
    } else {
      e0 = ex2_approx(x0);
      e1 = ex2_approx(x1);
    }
    acc[c2 & 3] = f2_add(acc[c2 & 3], f2_pack(e0, e1));
    if constexpr (!FP8) {
      pw[c2] = pack_bf16x2(e0, e1);
    } else {
      // four e4m3 per TMEM column: pair 2q in bytes 0-1, pair 2q+1 in bytes 2-3
      const uint32_t h = pack_e4m3x2(e0, e1);
      if (c2 & 1) pw[c2 >> 1] |= h << 16;
      else pw[c2 >> 1] = h;
    }
  }
  const uint64_t a01 = f2_add(acc[0], acc[1]), a23 = f2_add(acc[2], acc[3]);
  float lo, hi;
  f2_unpack(f2_add(a01, a23), lo, hi);
  sum = lo + hi;
}

template <int D, bool FP8, bool NA = false, bool PARTS = false>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_kernel(const __grid_constant__ MapSet<PARTS ? kMaxParts : 1> maps, const AttnParams p) {
  const CUtensorMap& tm_q = maps.q[0];
  const CUtensorMap& tm_k = maps.k[0];
  const CUtensorMap& tm_v = maps.v[0];
  using C = AttnCfg<D, FP8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* bar_q_full = bars;
  uint64_t* bar_k_full = bars + 1;
  uint64_t* bar_k_empty = bar_k_full + C::kKStages;
  uint64_t* bar_v_full = bar_k_empty + C::kKStages;
  uint64_t* bar_v_empty = bar_v_full + C::kVStages;
  uint64_t* bar_s_full = bar_v_empty + C::kVStages;   // [2]
  uint64_t* bar_p_full = bar_s_full + 2;              // [2]
  uint64_t* bar_o_final = bar_p_full + 2;             // [2]
  uint64_t* bar_drain = bar_o_final + 2;              // [1]
  uint64_t* bar_q_empty = bar_drain + 1;              // [1]
  uint64_t* bar_x0 = bar_q_empty + 1;                 // [2] NA: first penalty features written
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_kv = (p.k1 - p.k0 + C::kBN - 1) / C::kBN;   // >= 1 (empty ranges never launch)
  // unit -> (head index b*H + h, first query row); query block fastest
  auto unit_bh = [&](int u) { return u / p.n_qblk; };
  auto unit_q0 = [&](int u) { return (u % p.n_qblk) * (2 * C::kBM); };
  const uint64_t tmo = p.timeout_ns;

  if (threadIdx.x == C::kTmaWarp * 32) {
    mbar_init(bar_q_full, 1);
    for (int s = 0; s < C::kKStages; ++s) { mbar_init(bar_k_full + s, 1); mbar_init(bar_k_empty + s, 1); }
    for (int s = 0; s < C::kVStages; ++s) { mbar_init(bar_v_full + s, 1); mbar_init(bar_v_empty + s, 1); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s_full + t, 1);
      mbar_init(bar_p_full + t, 4);
      mbar_init(bar_o_final + t, 1);
    }
    mbar_init(bar_drain, 1);
    mbar_init(bar_q_empty, 1);
    mbar_init(bar_x0, 4);
    mbar_init(bar_x0 + 1, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;

  if (warp >= 8) {
    regs_dec<C::kRegsCtl>();
  if (warp == C::kTmaWarp || (NA && warp == C::kTmaWarp + 1)) {
    // ------------------------------------------------------------------ TMA producer
    // (NA: warp 9 loads Q and the K / V tiles of Q tile 0, warp 10 those of Q tile 1)
    if (lane == 0) {
      if constexpr (PARTS) {
        for (int pt = 0; pt < p.n_q_parts; ++pt) tma_prefetch_desc(&maps.q[pt]);
        for (int pt = 0; pt < p.n_kv_parts; ++pt) {
          tma_prefetch_desc(&maps.k[pt]);
          tma_prefetch_desc(&maps.v[pt]);
        }
      } else {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      int k_issued = 0, v_issued = 0, q_issued = 0;   // running counts over all units
      bool ok = true;
      const int lt = warp - C::kTmaWarp;               // NA: the Q tile whose K / V this thread loads
      if constexpr (NA) {
        // Each Q tile has its own ring of K slots (lt, lt + 2, ...) and of V slots; K(j + 1)
        // reuses the slot of K(j + 1 - kKPer), freed when that tile's S MMA is done, and
        // V(j + 1) the slot freed by its P.V.
        constexpr int kKPer = C::kKStages / 2, kVPer = C::kVStages / 2;
        int G = 0;                                     // running KV step count at unit start
        for (int it = 0, u = blockIdx.x; ok && u < p.n_units; ++it, u += gridDim.x) {
          const int bh = na_unit_bh(p, u);
          const NaTile w0 = na_tile(p, u, 0), w1 = na_tile(p, u, 1);
          const int n = max(w0.n(), w1.n());
          if (lt == 0) {
            // Q of this unit may overwrite the previous unit's only after its last S MMA.
            if (it > 0 && !(ok = mbar_wait(bar_q_empty, (it - 1) & 1, abort_flag, tmo, 0))) break;
            mbar_arrive_expect_tx(bar_q_full, 2 * C::kTileBytes);
            for (int b = 0; b < C::kNBlk; ++b) {
              tma_load_5d(sQ + b * C::kBlkBytes, &tm_q, bar_q_full, b * C::kBoxInner, w0.qx, w0.qy, w0.qt, bh);
              tma_load_5d(sQ + C::kTileBytes + b * C::kBlkBytes, &tm_q, bar_q_full, b * C::kBoxInner, w1.qx, w1.qy,
                          w1.qt, bh);
            }
            q_issued = it + 1;
          }
          // a step past the tile's own list (its P is 0) reloads one of its bricks (or, for a
          // Q brick past the grid, one of tile 0's) so that the MMA reads finite data
          const NaTile& w = (lt ? w1 : w0).n() > 0 ? (lt ? w1 : w0) : w0;
          for (int j = 0; j < n; ++j) {
            int ot, oy, ox;
            w.kv_origin(min(j, w.n() - 1), ot, oy, ox);
            const int i = G + j;
            const int ks = lt + 2 * (i % kKPer);
            if (i >= kKPer && !(ok = mbar_wait(bar_k_empty + ks, ((i / kKPer) + 1) & 1, abort_flag, tmo, 1))) break;
            mbar_arrive_expect_tx(bar_k_full + ks, C::kTileBytes);
            for (int b = 0; b < C::kNBlk; ++b)
              tma_load_5d(sK + ks * C::kTileBytes + b * C::kBlkBytes, &tm_k, bar_k_full + ks, b * C::kBoxInner, ox,
                          oy, ot, bh);
            k_issued = i + 1;
            const int vs = lt + 2 * (i % kVPer);
            if (i >= kVPer && !(ok = mbar_wait(bar_v_empty + vs, ((i / kVPer) + 1) & 1, abort_flag, tmo, 2))) break;
            mbar_arrive_expect_tx(bar_v_full + vs, C::kTileBytes);
            for (int b = 0; b < C::kNBlk; ++b)
              tma_load_5d(sV + vs * C::kTileBytes + b * C::kBlkBytes, &tm_v, bar_v_full + vs, b * C::kBoxInner, ox,
                          oy, ot, bh);
            v_issued = i + 1;
          }
          G += n;
        }
      } else {
      int g0 = 0;                                      // running KV tile count at unit start
      for (int it = 0, u = blockIdx.x; ok && u < p.n_units; ++it, u += gridDim.x) {
        const int bh = unit_bh(u), q0 = unit_q0(u), nkv = n_kv;
        // Q of this unit may overwrite the previous unit's only after its last S MMA.
        if (it > 0 && !(ok = mbar_wait(bar_q_empty, (it - 1) & 1, abort_flag, tmo, 0))) break;
        mbar_arrive_expect_tx(bar_q_full, 2 * C::kTileBytes);
        for (int t = 0; t < 2; ++t)
          for (int b = 0; b < C::kNBlk; ++b) {
            if constexpr (PARTS) {
              // row -> (part, row in part); rows past the last part read as zero (past its end)
              const int row = q0 + t * C::kBM;
              const int pt = min(row / p.part_rows, p.n_q_parts - 1);
              tma_load_4d(sQ + t * C::kTileBytes + b * C::kBlkBytes, &maps.q[pt], bar_q_full, b * C::kBoxInner,
                          row - pt * p.part_rows, bh % p.H, bh / p.H);
            } else
              tma_load_4d(sQ + t * C::kTileBytes + b * C::kBlkBytes, &tm_q, bar_q_full, b * C::kBoxInner,
                          (q0 + t * C::kBM) % p.seg_q, bh, (q0 + t * C::kBM) / p.seg_q);
          }
        q_issued = it + 1;
        for (int j = 0; j < nkv; ++j) {
          const int g = g0 + j;
          const int kv_row = p.k0 + j * C::kBN;
          const int ks = g % C::kKStages;
          if (g >= C::kKStages &&
              !(ok = mbar_wait(bar_k_empty + ks, ((g / C::kKStages) + 1) & 1, abort_flag, tmo, 1)))
            break;
          mbar_arrive_expect_tx(bar_k_full + ks, C::kTileBytes);
          for (int b = 0; b < C::kNBlk; ++b) {
            if constexpr (PARTS) {
              const int pt = min(kv_row / p.part_rows, p.n_kv_parts - 1);
              tma_load_4d(sK + ks * C::kTileBytes + b * C::kBlkBytes, &maps.k[pt], bar_k_full + ks,
                          b * C::kBoxInner, kv_row - pt * p.part_rows, bh % p.H, bh / p.H);
            } else
              tma_load_4d(sK + ks * C::kTileBytes + b * C::kBlkBytes, &tm_k, bar_k_full + ks,
                          b * C::kBoxInner, kv_row % p.seg_kv, bh, kv_row / p.seg_kv);
          }
          k_issued = g + 1;
          const int vs = g % C::kVStages;
          if (g >= C::kVStages &&
              !(ok = mbar_wait(bar_v_empty + vs, ((g / C::kVStages) + 1) & 1, abort_flag, tmo, 2)))
            break;
          mbar_arrive_expect_tx(bar_v_full + vs, C::kTileBytes);
          for (int b = 0; b < C::kNBlk; ++b) {
            if constexpr (PARTS) {
              const int pt = min(kv_row / p.part_rows, p.n_kv_parts - 1);
              tma_load_4d(sV + vs * C::kTileBytes + b * C::kBlkBytes, &maps.v[pt], bar_v_full + vs,
                          b * C::kBoxInner, kv_row - pt * p.part_rows, bh % p.H, bh / p.H);
            } else
              tma_load_4d(sV + vs * C::kTileBytes + b * C::kBlkBytes, &tm_v, bar_v_full + vs,
                          b * C::kBoxInner, kv_row % p.seg_kv, bh, kv_row / p.seg_kv);
          }
          v_issued = g + 1;
        }
        g0 += nkv;
      }
      }
      // Drain: the last load armed on every stage must land before the CTA may exit
      // (a no-op in a healthy run, where the consumers already waited for all of them).
      // (NA: this thread's ring is the slots lt + 2 r, with per-tile counts)
      constexpr int kKRing = NA ? C::kKStages / 2 : C::kKStages, kVRing = NA ? C::kVStages / 2 : C::kVStages;
      const int slot_step = NA ? 2 : 1, slot0 = NA ? lt : 0;
      if (q_issued > 0) mbar_wait_drain(bar_q_full, (q_issued - 1) & 1, tmo);
      for (int r = 0; r < kKRing; ++r) {
        const int last = r + ((k_issued - 1 - r) / kKRing) * kKRing;
        if (k_issued > r) mbar_wait_drain(bar_k_full + slot0 + slot_step * r, (last / kKRing) & 1, tmo);
      }
      for (int r = 0; r < kVRing; ++r) {
        const int last = r + ((v_issued - 1 - r) / kVRing) * kVRing;
        if (v_issued > r) mbar_wait_drain(bar_v_full + slot0 + slot_step * r, (last / kVRing) & 1, tmo);
      }
    }
  } else if (warp == C::kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t fmt = FP8 ? 0u : 1u;
      constexpr uint32_t id_s = instr_desc(fmt, false, 128, C::kBN);
      constexpr uint32_t id_o = instr_desc(fmt, true, 128, D);

      // Descriptors differ only in their start-address field (bits 0..13 of the low word,
      // address >> 4; shared-memory addresses stay below 2^18), so every K step is the low
      // word of a base descriptor plus (offset >> 4), with one high word for all of them.
      const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = smem_desc_sw128(smem_u32(sV), C::kBlkBytes, 1024);
      const uint32_t qk_hi = static_cast<uint32_t>(dq >> 32), v_hi = static_cast<uint32_t>(dv >> 32);
      const uint32_t q_lo = static_cast<uint32_t>(dq), k_lo = static_cast<uint32_t>(dk),
                     v_lo = static_cast<uint32_t>(dv);
      // NA: window-penalty features (query rows of tile t, keys), no swizzle, K-major
      uint8_t* sX = smem + AttnSmem<D, FP8, NA>::kOffX;
      const uint64_t dx = smem_desc_noswz(smem_u32(sX), 128, 256);
      const uint32_t x_lo = static_cast<uint32_t>(dx), x_hi = static_cast<uint32_t>(dx >> 32);
      auto issue_s = [&](int t, int ks) {
        const uint32_t a0 = q_lo + ((t * C::kTileBytes) >> 4);
        const uint32_t b0 = k_lo + ((ks * C::kTileBytes) >> 4);
        const uint32_t d = tmem_base + (t ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < C::kQKSteps; ++kk) {
          const uint32_t off = ((kk * 32 / 128) * C::kBlkBytes + (kk * 32) % 128) >> 4;
          mma_ss_lohi(FP8, d, a0 + off, qk_hi, b0 + off, qk_hi, id_s, kk > 0 ? 1u : 0u);
        }
        if constexpr (NA)
          mma_ss_lohi(false, d, x_lo + ((t * kNaXBytes) >> 4), x_hi, x_lo + ((2 * kNaXBytes) >> 4), x_hi, id_s, 1u);
      };
      auto issue_pv = [&](int t, int vs, bool acc) {
        const uint32_t b0 = v_lo + ((vs * C::kTileBytes) >> 4);
        const uint32_t a_tm = tmem_base + (t ? C::kColS1 : C::kColS0);
        const uint32_t d = tmem_base + (t ? C::kColO1 : C::kColO0);
#pragma unroll
        for (int kk = 0; kk < C::kPVSteps; ++kk) {
          // V tile is [kv rows][D] with D contiguous: MN-major B operand.  One MMA covers
          // kUmmaK kv rows (groups of 8 rows 1024 bytes apart) and all of D (64-element,
          // 128-byte atoms kBlkBytes apart).
          const uint32_t off = (kk * C::kUmmaK * 128) >> 4;
          mma_ts_lohi(FP8, d, a_tm + kk * 8, b0 + off, v_hi, id_o, (acc || kk > 0) ? 1u : 0u);
        }
      };

      bool ok = true;
      if constexpr (NA) {
        // The two Q tiles have their own K and V tiles and their own ring slots (tile t uses
        // slots t, t + 2, ...), so they are independent pipelines: this thread issues a
        // tile's next P.V + S as soon as that tile's P and K / V tiles are ready, in whatever
        // order the two tiles get there, and never holds one tile back behind the other.
        constexpr int kKPer = C::kKStages / 2, kVPer = C::kVStages / 2;
        int G = 0;                                     // running KV step count at unit start
        PollGuard guard;
        // steps of the next unit, computed while this thread waits anyway (at a unit boundary
        // the softmax warpgroups' epilogue stores make every instruction here slow)
        int n_next = blockIdx.x < p.n_units ? na_steps(p, blockIdx.x) : 0;
        // the softmax warpgroups have written the key features and each tile's first
        // penalty features (later ones are written before the P that precedes their S)
        if (blockIdx.x < p.n_units)
          ok = mbar_wait(bar_x0, 0, abort_flag, tmo, 3) && mbar_wait(bar_x0 + 1, 0, abort_flag, tmo, 3);
        for (int it = 0, u = blockIdx.x; ok && u < p.n_units; ++it, u += gridDim.x) {
          const int n = n_next;
          if (!(ok = mbar_wait(bar_q_full, it & 1, abort_flag, tmo, 3))) break;
          n_next = u + static_cast<int>(gridDim.x) < p.n_units ? na_steps(p, u + gridDim.x) : 0;
          tc_fence_after();
          // js[t] = j: the tile's next action issues P.V(j - 1) (j > 0) and S(j) (j < n)
          int js[2] = {0, 0};
          bool q_released = false;
          while (ok && (js[0] <= n || js[1] <= n)) {
            bool progress = false;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int j = js[t];
              if (j > n) continue;
              const int ik = G + j, iv = G + j - 1;
              const int ks = t + 2 * (ik % kKPer), vs = t + 2 * ((iv + kVPer) % kVPer);
              if (j < n && !mbar_test(bar_k_full + ks, (ik / kKPer) & 1)) continue;
              if (j > 0 && !(mbar_test(bar_v_full + vs, (iv / kVPer) & 1) && mbar_test(bar_p_full + t, iv & 1)))
                continue;
              tc_fence_after();
              if (j > 0) {
                issue_pv(t, vs, j > 1);
                if (j == n) tc_commit(bar_o_final + t);
                tc_commit(bar_v_empty + vs);
              }
              if (j < n) {
                issue_s(t, ks);
                tc_commit(bar_s_full + t);
                tc_commit(bar_k_empty + ks);
              }
              js[t] = j + 1;
              progress = true;
            }
            if (!q_released && js[0] >= n && js[1] >= n) {
              tc_commit(bar_q_empty);                  // every S MMA of this unit is issued
              q_released = true;
            }
            if (progress) {
              guard.progress();
            } else {
              ok = guard.idle(abort_flag, tmo, 4);
              __nanosleep(20);                         // leave the issue slots to the softmax warps
            }
          }
          G += n;
        }
      } else {
      int g0 = 0;                                      // running KV tile count at unit start
      for (int it = 0, u = blockIdx.x; ok && u < p.n_units; ++it, u += gridDim.x) {
        const int nkv = n_kv;
        if (!(ok = mbar_wait(bar_q_full, it & 1, abort_flag, tmo, 3))) break;
        tc_fence_after();
        for (int j = 0; ok && j < nkv; ++j) {
          const int g = g0 + j;
          const int ks = g % C::kKStages;
          if (!(ok = mbar_wait(bar_k_full + ks, (g / C::kKStages) & 1, abort_flag, tmo, 4))) break;
          tc_fence_after();
          const int gp = g - 1, vs = (g - 1) % C::kVStages;
          if (j > 0) {
            if (!(ok = mbar_wait(bar_v_full + vs, (gp / C::kVStages) & 1, abort_flag, tmo, 5))) break;
            if (!(ok = mbar_wait(bar_p_full + 0, gp & 1, abort_flag, tmo, 6))) break;
            tc_fence_after();
            issue_pv(0, vs, j - 1 > 0);
          }
          issue_s(0, ks);
          tc_commit(bar_s_full + 0);
          if (j > 0) {
            if (!(ok = mbar_wait(bar_p_full + 1, gp & 1, abort_flag, tmo, 7))) break;
            tc_fence_after();
            issue_pv(1, vs, j - 1 > 0);
            tc_commit(bar_v_empty + vs);
          }
          issue_s(1, ks);
          tc_commit(bar_s_full + 1);
          tc_commit(bar_k_empty + ks);
        }
        if (!ok) break;
        tc_commit(bar_q_empty);                    // every S MMA of this unit is issued
        const int gl = g0 + nkv - 1, vs = gl % C::kVStages;
        ok = mbar_wait(bar_v_full + vs, (gl / C::kVStages) & 1, abort_flag, tmo, 8);
        if (ok) ok = mbar_wait(bar_p_full + 0, gl & 1, abort_flag, tmo, 9);
        if (ok) {
          tc_fence_after();
          issue_pv(0, vs, nkv > 1);
          tc_commit(bar_o_final + 0);
          ok = mbar_wait(bar_p_full + 1, gl & 1, abort_flag, tmo, 10);
        }
        if (ok) {
          tc_fence_after();
          issue_pv(1, vs, nkv > 1);
          tc_commit(bar_o_final + 1);
          tc_commit(bar_v_empty + vs);
        }
        g0 += nkv;
      }
      }
      // Every MMA this thread issued must finish before TMEM is released.
      tc_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, tmo);
    }
  }  // warp 11 (and warp 10 outside NA) has no role
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    regs_inc<C::kRegsSoftmax>();
    const int t = warp >> 2;                // Q tile of this warpgroup
    const int quad = warp & 3;              // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;       // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + (t ? C::kColS1 : C::kColS0);
    const uint32_t tO = tmem_base + lane_off + (t ? C::kColO1 : C::kColO0);

    // Scales.  bf16: scores in raw units, cl = scale * log2(e) turns them into log2 units.
    // e4m3: the running max is kept in log2 units, and every KV tile j has its own
    //   cl_j = scale * descale_q(tile) * descale_k(j) * log2(e)
    // (one value for all tiles with per-tensor scales).  With per-block V scales, tile j's
    // P is stored as p * r_j, r_j = descale_v(j) / dv_out (dv_out = the largest V descale of
    // the range, so r_j <= 1 and P stays in range), which puts descale_v(j) / dv_out into
    // the P.V products; the epilogue multiplies by dv_out.  The row sum uses p itself: the
    // sum of the stored values divided by r_j.
    float dq = 1.0f, dk = 1.0f, dv = 1.0f;
    const bool blk = FP8 && p.dk_blk != nullptr;
    if constexpr (FP8) {
      if (!blk) { dq = p.descale[0]; dk = p.descale[1]; dv = p.descale[2]; }
    }
    const float scale_eff = p.scale * dq * dk;                 // natural-log units per raw score
    const float cl = scale_eff * 1.4426950408889634f;          // log2 units per raw score
    bool ok = true;

    int g0 = 0;                                                // running KV tile count at unit start
    uint8_t* sX = smem + AttnSmem<D, FP8, NA>::kOffX;          // NA: window-penalty features
    if constexpr (NA) {
      // the keys' position features (static), and each tile's features for its first step
      if (blockIdx.x < p.n_units) {
        if (t == 0) na_write_keyfeat(sX + 2 * kNaXBytes, row);
        const NaTile w0 = na_tile(p, blockIdx.x, t);
        if (w0.n() > 0) {
          int a, b, c, wt0, wy0, wx0, ot, oy, ox;
          na_row_geo(p, w0, row, a, b, c, wt0, wy0, wx0);
          w0.kv_origin(0, ot, oy, ox);
          na_write_pen(sX + t * kNaXBytes, row, wt0, wy0, wx0, p.na_Kt, p.na_Ky, p.na_Kx, ot, oy, ox);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_x0 + t);
      }
    }
    for (int it = 0, u = blockIdx.x; ok && u < p.n_units; ++it, u += gridDim.x) {
    NaTile w;
    int bh, q_start, nkv, n_own = 0;     // NA: n_own = KV bricks of this tile's own list
    int qt = 0, qy = 0, qx = 0, wt = 0, wy = 0, wx = 0;       // NA: this row's token and window starts
    if constexpr (NA) {
      w = na_tile(p, u, t);
      n_own = w.n();
      bh = na_unit_bh(p, u); q_start = 0; nkv = max(n_own, na_tile(p, u, t ^ 1).n());
      na_row_geo(p, w, row, qt, qy, qx, wt, wy, wx);
    } else {
      bh = unit_bh(u); q_start = unit_q0(u); nkv = n_kv;
    }
    float m_use = -INFINITY;             // running (lazy) max: raw units (bf16), log2 units (e4m3)
    float l = 0.0f;
    float cl_q = cl, dv_out = dv;        // per unit and Q tile (e4m3 per-block scales)
    float dk_nxt = dk, dv_nxt = dv;      // descales of the next KV tile, loaded one tile ahead
    if constexpr (FP8) {
      if (blk) {
        const int bq = min((q_start + t * C::kBM) / C::kBM, p.nb_q - 1);
        cl_q = p.scale * __ldg(p.dq_blk + static_cast<size_t>(bh) * p.nb_q + bq) * 1.4426950408889634f;
        const float* dvr = p.dv_blk + static_cast<size_t>(bh) * p.nb_kv;
        const int kt0 = p.k0 / C::kBN, kt1 = (p.k1 + C::kBN - 1) / C::kBN;
        float mx = 0.0f;
        for (int kt = kt0; kt < kt1; ++kt) mx = fmaxf(mx, __ldg(dvr + kt));
        dv_out = mx;
        dk_nxt = __ldg(p.dk_blk + static_cast<size_t>(bh) * p.nb_kv + kt0);
        dv_nxt = __ldg(dvr + kt0);
      }
    }
    for (int j = 0; j < nkv; ++j) {
      const int g = g0 + j;
      // e4m3: this tile's cl_j and V ratio; prefetch the next tile's descales
      float clj = cl, lrj = 0.0f, inv_rj = 1.0f;
      if constexpr (FP8) {
        if (blk) {
          const float dkj = dk_nxt, dvj = dv_nxt;
          if (j + 1 < nkv) {
            const size_t nx = static_cast<size_t>(bh) * p.nb_kv + p.k0 / C::kBN + j + 1;
            dk_nxt = __ldg(p.dk_blk + nx);
            dv_nxt = __ldg(p.dv_blk + nx);
          }
          clj = cl_q * dkj;
          if (dvj > 0.0f) {                  // an all-zero V block (descale 0) keeps r_j = 1
            lrj = __log2f(dvj / dv_out);
            inv_rj = dv_out / dvj;
          }
        }
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full + t, g & 1, abort_flag, tmo, 11 + t));
      if (!ok) break;
      tc_fence_after();
      uint32_t pw[2 * C::kPWordsHalf];
      float sum = 0.0f;
      float alpha = 1.0f;
      bool need = false;
      if (NA && j >= n_own) {
        // a step past this tile's own KV list (the other tile's list is longer): no keys, P = 0
#pragma unroll
        for (int i = 0; i < 2 * C::kPWordsHalf; ++i) pw[i] = 0u;
      } else {
      uint32_t s[128];
      tmem_ld128_sync(tS, s);
      const int valid = p.k1 - (p.k0 + j * C::kBN);
      // (NA: keys outside the row's window already carry the penalty from the S MMA)
      if constexpr (!NA) {
        if (valid < C::kBN) mask_tail(s, valid);
      }
      // Speculative pass (bf16): exponentiate with the running max m_use and keep the result
      // when the row sum shows that no p exceeds the lazy-rescale bound (every p <= sum <=
      // kSumBound), the usual case after the first tile.  Otherwise (first tile, a row max
      // that rose a lot, or the e4m3 path) the warp takes the exact route: (re)load S (still
      // intact in TMEM, P is not written yet), exact row max, rescale, exponentiate.
      // (NA: a row whose window has missed every tile so far has no max yet: exact route)
      bool slow = (j == 0) || !C::kSpeculative || (NA && __any_sync(0xffffffffu, m_use == -INFINITY));
      if (!slow) {
        exp_pass<FP8, C::kEmuMask>(s, cl, m_use * cl - C::kPShift, pw, sum);
        slow = __any_sync(0xffffffffu, !(sum <= C::kSumBound));
      }
      if (slow) {
        if (j > 0 && C::kSpeculative) {
          tmem_ld128_sync(tS, s);
          if constexpr (!NA) {
            if (valid < C::kBN) mask_tail(s, valid);
          }
        }
        if constexpr (FP8) {
          const float m_new = fmaxf(m_use, clj * row_max128(s));
          need = m_new - m_use > C::kRescaleLog2;            // true on the first tile
          if (need) {
            alpha = ex2_approx(m_use - m_new);               // 0 when m_use = -inf
            m_use = m_new;
          }
          exp_pass<FP8, C::kEmuMask>(s, clj, m_use - C::kPShift - lrj, pw, sum);
          sum *= inv_rj;
        } else {
          float rm = row_max128(s);
          // NA: a row max at the penalty's scale means no key of this tile lies in the row's
          // window; the row keeps no max (as with -inf keys), so its exponentials stay 0
          if constexpr (NA) {
            if (rm < -1.0e27f) rm = -INFINITY;
          }
          const float m_new = fmaxf(m_use, rm);
          need = (m_new - m_use) * cl > C::kRescaleLog2;     // true on the first tile
          if (need) {
            alpha = ex2_approx((m_use - m_new) * cl);        // 0 when m_use = -inf
            m_use = m_new;
          }
          // (a row with no key in its window yet keeps m_use = -inf: exponents of -inf, p = 0)
          const float mc = (NA && m_use == -INFINITY) ? 0.0f : m_use * cl;
          exp_pass<FP8, C::kEmuMask>(s, cl, mc - C::kPShift, pw, sum);
        }
      }
      }
      tmem_st32(tS, *reinterpret_cast<uint32_t(*)[32]>(&pw[0]));
      if constexpr (!FP8) tmem_st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pw[32]));
      tmem_st_wait();
      // O_t is quiescent here (PV_t(j-1) completed before S_t(j) was signalled).
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32_sync(tO + cc * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + cc * 32, o);
        }
        tmem_st_wait();
      }
      l = fmaf(l, alpha, sum);
      if constexpr (NA) {
        // penalty features of this tile's next step, written before P(j) lets the MMA thread
        // issue that step's S (S(j) is complete, so the block is free): the next brick of this
        // unit, or the first brick of this tile in the CTA's next unit
        if (j + 1 < n_own) {
          int ot, oy, ox;
          w.kv_origin(j + 1, ot, oy, ox);
          na_write_pen(sX + t * kNaXBytes, row, wt, wy, wx, p.na_Kt, p.na_Ky, p.na_Kx, ot, oy, ox);
        } else if (j + 1 == nkv && u + static_cast<int>(gridDim.x) < p.n_units) {
          const NaTile w2 = na_tile(p, u + gridDim.x, t);
          if (w2.n() > 0) {
            int a, b, c, wt2, wy2, wx2, ot, oy, ox;
            na_row_geo(p, w2, row, a, b, c, wt2, wy2, wx2);
            w2.kv_origin(0, ot, oy, ox);
            na_write_pen(sX + t * kNaXBytes, row, wt2, wy2, wx2, p.na_Kt, p.na_Ky, p.na_Kx, ot, oy, ox);
          }
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p_full + t);
    }

    g0 += nkv;

    // ---------------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_o_final + t, it & 1, abort_flag, tmo, 13 + t));
    if (ok) {
      tc_fence_after();
      const int grow = q_start + t * C::kBM + row;
      bool store;
      size_t row_idx;
      void* out_base = p.out;
      float* lse_base = p.lse;
      if constexpr (NA) {
        store = qt < p.na_T && qy < p.na_Y && qx < p.na_X;
        row_idx = static_cast<size_t>(bh) * p.S_q + (static_cast<size_t>(qt) * p.na_Y + qy) * p.na_X + qx;
      } else if constexpr (PARTS) {
        // the row goes to the part that holds it, at its head in the part's full-head layout
        store = grow < p.S_q;
        const int pt = min(grow / p.part_rows, p.n_q_parts - 1);
        out_base = p.out_parts[pt];
        lse_base = p.lse_parts[pt];
        row_idx = (static_cast<size_t>(bh / p.H) * p.part_H + p.part_h0 + bh % p.H) * p.part_rows +
                  (grow - pt * p.part_rows);
      } else {
        store = grow < p.S_q;
        row_idx = (static_cast<size_t>(grow / p.seg_q) * p.B * p.H + bh) * p.seg_q + grow % p.seg_q;
      }
      const size_t row_elem = row_idx * D;
      const float lse_c = (FP8 ? m_use * 0.6931471805599453f : scale_eff * m_use) + logf(l) -
                          C::kPShift * 0.6931471805599453f;
      // Accumulate mode (one ring step): (O, LSE) <- exact LSE merge of the running pair and
      // this range's partial, w = exp(lse - M) / L with M the larger LSE and L the weight sum.
      float w_old = 0.0f, w_new = 1.0f, lse_out = lse_c;
      if (p.accumulate && store) {
        const float la = lse_base[row_idx];
        const float M = fmaxf(la, lse_c);
        const float ea = __expf(la - M);                     // 0 for an empty accumulator
        const float ec = __expf(lse_c - M);
        const float L = ea + ec;
        w_old = ea / L;
        w_new = ec / L;
        lse_out = M + logf(L);
      }
      const float inv_l = dv_out / l * w_new;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32_sync(tO + cc * 32, o);
        if (store) {
          if (p.accumulate && w_old != 0.0f) {
            // (an empty accumulator, w_old = 0, is overwritten below without being read, so
            // whatever its buffer holds cannot leak in)
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out_base) + row_elem + cc * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 a = dst[i];
              dst[i] = make_float4(fmaf(a.x, w_old, __uint_as_float(o[4 * i]) * inv_l),
                                   fmaf(a.y, w_old, __uint_as_float(o[4 * i + 1]) * inv_l),
                                   fmaf(a.z, w_old, __uint_as_float(o[4 * i + 2]) * inv_l),
                                   fmaf(a.w, w_old, __uint_as_float(o[4 * i + 3]) * inv_l));
            }
          } else if (p.out_fp32 || p.accumulate) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out_base) + row_elem + cc * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                   __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
          } else {
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out_base) + row_elem + cc * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
      if (store && lse_base != nullptr) lse_base[row_idx] = lse_out;
      // The O reads above end with tcgen05.wait::ld; the next unit's first P.V (which
      // overwrites O_t) is issued only after this warpgroup publishes that unit's P_t.
    }
    }  // units
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Empty KV range: out = 0, lse = -inf.
__global__ void attn_fill_empty_kernel(void* out, float* lse, long long rows, int D, int out_fp32) {
  const long long n = rows * D;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    if (out_fp32) static_cast<float*>(out)[i] = 0.0f;
    else static_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16(0.0f);
    if (lse != nullptr && i < rows) lse[i] = -INFINITY;
  }
}

}  // namespace dit
