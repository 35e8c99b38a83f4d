/*
 * dit_attn.h - C ABI of a B200 (sm_100a) library for DiT joint self-attention.
 *
 * What the library computes
 * -------------------------
 * The attention at the heart of a diffusion-transformer (DiT) block: image or video patch
 * tokens concatenated with text tokens, every token attending to every token (no causal
 * mask, no padding mask, no KV cache).  The source pages describe DiT inference as
 * prefill-like and compute-bound from start to finish, with sequences of many thousands of
 * tokens (xDiT overview page, sections 1 and 2.1-2.2).  For each batch b, head h and query
 * row i, over the keys j of a range [k0, k1):
 *
 *     out_i = sum_j softmax_j(scale * q_i . k_j) v_j
 *     lse_i = log sum_j exp(scale * q_i . k_j)          (natural log)
 *
 * Partial results over disjoint key ranges are combined exactly by dit_attn_merge, the
 * combine step that the USP "Ring" dimension relies on (xDiT overview page, section 3.2.2:
 * the sequence is split into blocks passed around a ring; the xDiT docs page exposes it as
 * --ring_degree).  An FP8-E4M3 input variant follows the FP8 attention backend named on the
 * AMD ROCm summary page (--attention_backend aiter_flydsl_fp8; "FP8 may change outputs").
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are dense row-major [B, H, S, D] (D innermost, stride 1); LSE arrays are fp32
 *    [B, H, S].  D must be 64 or 128.
 *  - Every tensor pointer is a DEVICE pointer on the current CUDA device, 16-byte aligned
 *    (LSE pointers 4-byte aligned).  The caller owns all buffers; the library never
 *    allocates, frees or keeps device memory, and never synchronises the stream.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is enqueued on it
 *    and the call returns immediately; the calls are therefore usable inside CUDA-graph
 *    capture.
 *  - Return value: DIT_OK or a DIT_ERR_* code.  Argument errors are detected on the host
 *    before anything is enqueued.  A failed launch returns DIT_ERR_CUDA.  Errors that can
 *    only arise on the device (a bounded wait that ran out, DIT_ERR_TIMEOUT) are recorded
 *    in a device status word read by dit_device_status().
 *  - Outputs must not overlap inputs.
 *  - Thread-safe: calls on different streams or host threads may run concurrently.
 */
#ifndef DIT_ATTN_H
#define DIT_ATTN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types */
#define DIT_BF16 0     /* bfloat16 */
#define DIT_FP8_E4M3 1 /* FP8 E4M3 ("fn": no infinities, max 448) with a per-tensor descale */
#define DIT_FP32 2     /* float32 (outputs only) */

/* status codes */
#define DIT_OK 0
#define DIT_ERR_INVALID_ARG 1 /* null pointer, bad size, bad range, overlapping buffers */
#define DIT_ERR_UNSUPPORTED 2 /* valid but not built: D not in {64,128}, FP8 with D != 128 */
#define DIT_ERR_MISALIGNED 3  /* a pointer breaks the alignment rule above */
#define DIT_ERR_CUDA 4        /* a CUDA runtime/driver call or a launch failed */
#define DIT_ERR_TIMEOUT 5     /* device side: a bounded wait inside a kernel ran out */

/*
 * dit_attn_fwd - full attention forward over all S keys.
 *
 *   q, k, v   [B,H,S,D] inputs, bf16 (dtype = DIT_BF16) or E4M3 codes (DIT_FP8_E4M3).
 *   out       [B,H,S,D] bf16 output.
 *   lse       [B,H,S] fp32 natural-log LSE, or NULL to skip it.
 *   scale     softmax scale (finite, > 0), usually 1/sqrt(D).
 *   descale_qkv  DIT_FP8_E4M3 only: device pointer to 3 floats {descale_q, descale_k,
 *             descale_v}; the real input is code * descale (see dit_quant_fp8).  NULL for bf16.
 *
 * Same as dit_attn_fwd_chunk(q,k,v,out,lse,B,H,S,S,D,0,S,scale,dtype,DIT_BF16,descale,stream).
 */
int dit_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
                 int S, int D, float scale, int dtype, const float* descale_qkv, void* stream);

/*
 * dit_attn_fwd_chunk - attention of S_q queries against the keys k0 <= j < k1 of a
 * [B,H,S_kv,D] K/V pair: one ring step of the USP Ring dimension, all on one GPU.
 *
 *   q         [B,H,S_q,D];  k, v  [B,H,S_kv,D] (full tensors; the range selects rows).
 *   out       [B,H,S_q,D], out_dtype DIT_BF16 or DIT_FP32 (fp32 keeps partials exact
 *             enough for a later merge).
 *   lse       [B,H,S_q] fp32, or NULL.
 *   0 <= k0 <= k1 <= S_kv.  k0 == k1 (an empty range) writes out = 0 and lse = -inf.
 */
int dit_attn_fwd_chunk(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                       int H, int S_q, int S_kv, int D, int k0, int k1, float scale, int dtype,
                       int out_dtype, const float* descale_qkv, void* stream);

/*
 * dit_attn_fwd_chunk_acc - one ring step fused into the forward: attention of the S_q queries
 * against the keys k0 <= j < k1, merged in the epilogue into a running accumulator
 *     lse' = log(exp(acc_lse) + exp(lse_c)),
 *     acc_out' = (exp(acc_lse - lse') acc_out + exp(lse_c - lse') out_c)
 * (the same exact combination as dit_attn_merge, applied pairwise), so a ring of chunks needs
 * no stored partials and no separate merge launch.  This is the per-block step of the USP
 * Ring dimension (xDiT overview page, section 3.2.2), on one GPU.
 *
 *   acc_out   [B,H,S_q,D] fp32, read and written (16-byte aligned).
 *   acc_lse   [B,H,S_q] fp32, read and written.  An accumulator with acc_lse = -inf (and any
 *             acc_out) is empty: see dit_attn_acc_init.  The first chunk may also be written
 *             by dit_attn_fwd_chunk with out_dtype = DIT_FP32.
 *   Other arguments as for dit_attn_fwd_chunk.  k0 == k1 leaves the accumulator unchanged.
 *   Calls that update the same accumulator must be ordered (same stream, or events).
 *   The final bf16 output can be produced with dit_attn_merge(n_chunks = 1).
 */
int dit_attn_fwd_chunk_acc(const void* q, const void* k, const void* v, float* acc_out, float* acc_lse,
                           int B, int H, int S_q, int S_kv, int D, int k0, int k1, float scale,
                           int dtype, const float* descale_qkv, void* stream);

/*
 * dit_attn_fwd_seg - dit_attn_fwd_chunk over all S keys (S_q = S_kv = S) for tensors stored in
 * sequence segments: row r of head (b, h) at index ((r / seg) * B*H + b*H + h) * seg + r % seg,
 * i.e. [S/seg, B, H, seg, D] (lse: [S/seg, B, H, seg]).  This is the layout in which the
 * sequence-to-head all-to-all of the USP Ulysses dimension (xDiT overview page, section
 * 3.2.2) delivers Q, K and V (segment p = the rows that came from rank p), and the layout
 * its return all-to-all sends from, so neither side needs a re-layout copy.
 *
 *   seg       rows per segment; S % seg == 0; seg % 128 == 0 unless seg == S (seg == S is
 *             the plain [B,H,S,D] layout), else DIT_ERR_UNSUPPORTED.
 *   Other arguments as for dit_attn_fwd_chunk (out_dtype DIT_BF16 or DIT_FP32; E4M3 inputs
 *   with per-tensor descales).
 */
int dit_attn_fwd_seg(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
                     int S, int D, int seg, float scale, int dtype, int out_dtype,
                     const float* descale_qkv, void* stream);

/*
 * dit_na3d_fwd - 3-D neighborhood attention on a T x Y x X token grid (the operation NATTEN
 * calls na3d; the LTX notes page, section 5, reports it as the hot spot of a video decoder).
 * Token s = (t * Y + y) * X + x of each (b, h) attends only to the keys of its neighborhood:
 * along each dimension of length L with odd window K, the K positions starting at
 * clamp(i - K/2, 0, L - K) (fixed size, shifted inward at the borders; dilation 1,
 * non-causal); the neighborhood is the product of the three windows.
 *     out_s = sum_{j in N(s)} softmax_j(scale * q_s . k_j) v_j,
 *     lse_s = log sum_{j in N(s)} exp(scale * q_s . k_j).
 *
 *   q, k, v   [B,H,T*Y*X,D] bf16;  out [B,H,T*Y*X,D] bf16;  lse [B,H,T*Y*X] fp32 or NULL.
 *   Kt, Ky, Kx odd, 1 <= K <= the grid dimension, else DIT_ERR_INVALID_ARG.  D = 64 or 128.
 *   scale >= 1e-20 (else DIT_ERR_INVALID_ARG); scores |q . k| below 1e27.
 *   Each 128-query brick of the grid (its shape chosen per call from the grid and window)
 *   visits only the 128-key bricks (4 x 4 x 8 in t, y, x) that cover its queries' windows; the
 *   keys of a brick outside a query's window get a score penalty of -2^100 (an extra step of
 *   the score MMA), so their weights are exactly 0.
 */
int dit_na3d_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
                 int T, int Y, int X, int D, int Kt, int Ky, int Kx, float scale, void* stream);

/*
 * dit_na3d_plan - the tiling dit_na3d_fwd uses for a grid and window (host only, no GPU):
 * q_brick[0..2] = the Q brick's t, y, x extents (product 128), q_brick[3] = the axis (0 = t,
 * 1 = y, 2 = x) along which the two Q bricks of a unit lie side by side; *units_per_head =
 * units of one (b, h); *steps_per_head = KV steps of one (b, h) (each step: one 128-key brick
 * per Q brick of the unit).  Executed MMA work of a call = 4 * B*H * steps * 256 * 128 * D
 * FLOPs, plus the window-penalty step (K = 16) of every S tile.
 *   q_brick int[4], units_per_head, steps_per_head: host pointers, written on success.
 *   Returns DIT_ERR_INVALID_ARG for the grid / window errors dit_na3d_fwd rejects.
 */
int dit_na3d_plan(int T, int Y, int X, int Kt, int Ky, int Kx, int* q_brick, long long* units_per_head,
                  long long* steps_per_head);

/*
 * dit_attn_fwd_parts - attention whose inputs lie in blocks held by several ranks (possibly on
 * other GPUs, through peer addresses over NVLink), one kernel, no exchange.  The keys are
 * n_kv_parts blocks and the queries n_q_parts blocks of part_rows rows each; block p is held
 * by tensors [B, part_H, part_rows, D].  The call computes, for heads [h0, h0 + H), full
 * attention of all n_q_parts * part_rows query rows over all n_kv_parts * part_rows keys:
 * Q/K/V tiles are loaded by TMA straight from the block that holds them, and every output row
 * (and LSE) is written into the query block it belongs to, out_parts[p][b, h0 + h, row, :].
 * Loads are plain TMA loads into the loading CTA's shared memory; stores are plain global stores.
 *  - Ulysses step of USP (xDiT overview page, section 3.2.2): n_q_parts = n_kv_parts = P, one
 *    launch per rank with h0 = rank * H (H = part_H / P): replaces both all-to-alls and the
 *    re-layout copies around them.
 *  - Ring step of USP without the ring: n_q_parts = 1 (this rank's rows), n_kv_parts = P,
 *    h0 = 0, H = part_H: every rank reads the other ranks' K/V in place.
 *
 *   q_parts, out_parts  HOST arrays of n_q_parts device pointers; k_parts, v_parts: HOST arrays
 *             of n_kv_parts device pointers (bf16, 16-byte aligned); lse_parts: host array of
 *             n_q_parts fp32 device pointers, or NULL.  The arrays are read during the call only.
 *   1 <= n_q_parts, n_kv_parts <= 8; part_rows % 128 == 0 unless both are 1 (else
 *   DIT_ERR_UNSUPPORTED); 0 <= h0, h0 + H <= part_H; D = 64 or 128.
 *   Ordering across GPUs is the caller's: every block must be written before any launch that
 *   reads it starts, and the outputs are complete when every launch that writes them has
 *   finished (e.g. a barrier before and after).
 */
int dit_attn_fwd_parts(const void* const* q_parts, int n_q_parts, const void* const* k_parts,
                       const void* const* v_parts, int n_kv_parts, void* const* out_parts,
                       float* const* lse_parts, int B, int part_H, int h0, int H, int part_rows,
                       int D, float scale, void* stream);

/*
 * dit_ipc_export / dit_ipc_import / dit_ipc_close - share device buffers between the processes
 * of one node (one per GPU), for dit_attn_fwd_parts on peer memory.
 *   dit_ipc_export: the CUDA IPC handle (64 bytes, written to `handle`) of the allocation that
 *     holds `ptr`, and ptr's byte offset inside it.
 *   dit_ipc_import: opens a handle exported by another process (peer access enabled lazily)
 *     and returns the mapped allocation (`base`) and base + offset (`ptr`).
 *   dit_ipc_close: unmaps an imported allocation (`base` from dit_ipc_import).
 * A handle cannot be imported by the process that exported it.  DIT_ERR_CUDA on failure.
 */
int dit_ipc_export(const void* ptr, void* handle, long long* offset);
int dit_ipc_import(const void* handle, long long offset, void** ptr, void** base);
int dit_ipc_close(void* base);

/*
 * dit_swap01_chunks - dst[i1][i0] = src[i0][i1] for a [d0][d1] grid of chunks of chunk_bytes
 * bytes each (the batch/peer transpose around a Ulysses all-to-all when B > 1).
 *   src, dst  device buffers of d0 * d1 * chunk_bytes bytes, 16-byte aligned, not overlapping.
 *   chunk_bytes a multiple of 16 (else DIT_ERR_UNSUPPORTED).
 */
int dit_swap01_chunks(const void* src, void* dst, long long d0, long long d1, long long chunk_bytes,
                      void* stream);

/*
 * dit_attn_acc_init - empty accumulator: acc_out = 0, acc_lse = -inf ([B,H,S,D] / [B,H,S] fp32).
 */
int dit_attn_acc_init(float* acc_out, float* acc_lse, int B, int H, int S, int D, void* stream);

/*
 * dit_attn_merge - exact log-sum-exp combination of n_chunks partials (out_c, lse_c):
 *     M = max_c lse_c, w_c = exp(lse_c - M), L = sum_c w_c,
 *     lse = M + log L, out = sum_c (w_c / L) out_c;  all lse_c = -inf -> out = 0, lse = -inf.
 *
 *   outs      HOST array of n_chunks DEVICE pointers, each [B,H,S,D] of in_dtype
 *             (DIT_BF16 or DIT_FP32).
 *   lses      HOST array of n_chunks DEVICE pointers, each [B,H,S] fp32.
 *   n_chunks  1..16.
 *   out       [B,H,S,D] of out_dtype (DIT_BF16 or DIT_FP32);  lse [B,H,S] fp32 or NULL.
 *   The host arrays are read during the call only.
 */
int dit_attn_merge(const void* const* outs, const float* const* lses, int n_chunks, void* out,
                   float* lse, int B, int H, int S, int D, int in_dtype, int out_dtype,
                   void* stream);

/*
 * dit_quant_fp8 - per-tensor absmax quantisation of n bf16 values to E4M3:
 *     amax = max|x|, descale = amax / 448 (1 if amax = 0), x_fp8 = rn_satfinite(x / descale)
 * with IEEE fp32 division.  The FP8 scaling scheme is not given by the pages; this is the
 * plain per-tensor reading of their FP8 backend.
 *
 *   x_bf16    n bf16 values (16-byte aligned);  x_fp8  n bytes (16-byte aligned).
 *   descale   device pointer to 1 float (written).
 *   workspace device scratch of at least dit_quant_fp8_workspace_bytes(n) bytes, 4-byte
 *             aligned, owned by the caller; its contents on entry do not matter.
 */
size_t dit_quant_fp8_workspace_bytes(long long n);
int dit_quant_fp8(const void* x_bf16, void* x_fp8, float* descale, long long n, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * dit_quant_fp8_blocks - per-block E4M3 quantisation: every run of 128 consecutive rows
 * (tokens) of one (b, h) of a [B,H,S,D] bf16 tensor is quantised as a tensor of its own
 * (the rule of dit_quant_fp8), the last run of a head ragged when S % 128 != 0.  A finer
 * variant of the per-tensor scheme for inputs whose magnitude varies along the sequence; the
 * pages fix no FP8 scaling scheme.  An all-zero block records descale 0 and zero codes.
 *
 *   x_bf16    [B,H,S,D] bf16 (16-byte aligned);  x_fp8  [B,H,S,D] E4M3 codes (8-byte aligned).
 *   descales  [B,H,ceil(S/128)] fp32, written.  8 <= D <= 128, D % 8 == 0.
 *   One kernel launch; each element is read and written once.
 */
int dit_quant_fp8_blocks(const void* x_bf16, void* x_fp8, float* descales, int B, int H, int S, int D,
                         void* stream);

/*
 * dit_attn_fwd_fp8_blocks - dit_attn_fwd_chunk on E4M3 inputs quantised per block by
 * dit_quant_fp8_blocks: q_ij = code * dq_blk[b,h,i/128], likewise k and v.
 *
 *   q8, k8, v8  [B,H,S_q,D] / [B,H,S_kv,D] E4M3 codes.
 *   dq_blk      [B,H,ceil(S_q/128)] fp32;  dk_blk, dv_blk  [B,H,ceil(S_kv/128)] fp32.
 *   D = 128.  k0 must be a multiple of 128 (each 128-key tile has one scale), else
 *   DIT_ERR_UNSUPPORTED.  Other arguments and results as for dit_attn_fwd_chunk.
 *   In the kernel, Q and K scales enter the softmax scale of each tile pair; V scales enter
 *   P as ratios descale_v(j) / max_j descale_v(j) <= 1 and the maximum is applied to O.
 */
int dit_attn_fwd_fp8_blocks(const void* q8, const void* k8, const void* v8, const float* dq_blk,
                            const float* dk_blk, const float* dv_blk, void* out, float* lse, int B,
                            int H, int S_q, int S_kv, int D, int k0, int k1, float scale,
                            int out_dtype, void* stream);

/*
 * dit_quant_fp8_noalloc - the same quantisation as dit_quant_fp8, for callers that cannot
 * allocate device memory: code that runs where cudaMalloc is off limits (for example while
 * a stream is being captured into a CUDA graph, or inside a framework whose allocator owns
 * all device memory and forbids raw allocations), and so has no way to provide the
 * workspace.  The pages have no counterpart to this call; it exists for such callers only.
 *
 *   x_bf16, x_fp8, descale, n: as for dit_quant_fp8; the caller still provides these.
 *   Scratch: a 4736-byte array of partial maxima (1184 floats) that lives in the library's
 *   own device data, so every GPU that loads the library keeps it until the process exits.
 *   The call allocates and frees nothing.  Every n >= 1 fits: the first pass uses at most
 *   1184 blocks, one scratch slot each; a block count above the array's size would be
 *   rejected with DIT_ERR_UNSUPPORTED.
 *   Set-up: the first call on each device (with that device current) looks up the array's
 *   device address with cudaGetSymbolAddress; make that first call before any stream
 *   capture.  Later calls reuse the address while the device keeps the same context; after
 *   a cudaDeviceReset the next call repeats the set-up (the reset reloads the module), so
 *   that call, too, should come before any capture.
 *   Sharing: all calls on a device share the one array and it keeps the last call's
 *   contents.  Nothing in it needs to start at zero (each call writes every slot it reads
 *   before reading it), but calls whose kernels overlap on the GPU (different streams, no
 *   ordering between them) race on the array and give wrong results; order them.
 */
int dit_quant_fp8_noalloc(const void* x_bf16, void* x_fp8, float* descale, long long n,
                          void* stream);

/*
 * dit_device_status - synchronises the current device, then reads the device status word
 * into *status: DIT_OK, or DIT_ERR_TIMEOUT | (site << 8) when a bounded wait inside a
 * kernel ran out (the kernel then wound down without hanging; its outputs are invalid).
 * clear != 0 resets the word to DIT_OK afterwards.  Returns DIT_ERR_CUDA if the device
 * cannot be synchronised or read.
 */
int dit_device_status(int* status, int clear);

/*
 * dit_set_wait_timeout_us - process-wide limit for every bounded wait inside the kernels
 * (default 1,000,000 us).  A healthy kernel waits microseconds; the limit only matters
 * if the pipeline is broken.  0 restores the default.
 */
int dit_set_wait_timeout_us(unsigned long long timeout_us);

/*
 * dit_set_sm_reserve - process-wide number of SMs that the attention kernels leave free
 * (default 0).  The attention forward is a persistent kernel with one CTA per SM that fills
 * each SM's shared memory and registers, so no other kernel can run beside it; a KV ring
 * whose NCCL send/recv kernels should overlap the attention of the current block reserves
 * a few SMs for them.  The grid is max(1, SMs - n_sms) CTAs at most; results do not depend
 * on it.  0 <= n_sms <= 1024, else DIT_ERR_INVALID_ARG.
 */
int dit_set_sm_reserve(int n_sms);

/*
 * dit_selftest_wait_timeout - enqueues a one-thread kernel that waits on a barrier nothing
 * ever arrives at, with the given limit, so the caller can check that the bounded wait
 * gives up and that dit_device_status() then reports DIT_ERR_TIMEOUT.
 */
int dit_selftest_wait_timeout(unsigned long long timeout_us, void* stream);

/* Human-readable name of a status code (static string). */
const char* dit_status_str(int status);

/* ABI version: major * 10000 + minor * 100 + patch. */
int dit_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DIT_ATTN_H */
