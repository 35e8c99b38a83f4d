"""KV ring across ranks: the Ring dimension of USP (xDiT overview page, section 3.2.2).

The sequence is split into blocks, one per rank.  Each rank keeps its own query rows and
passes key/value blocks around a ring (rank r sends to r+1 and receives from r-1), so after
P steps every rank has seen every block.  Each step's block is folded into a running fp32
(O, LSE) accumulator by ``dit_attn_fwd_chunk_acc``, the fused ring step, so the ring keeps
no partials and needs no final merge over P buffers.  The xDiT docs page exposes this
dimension as ``--ring_degree``.

Overlap: the send/recv of step t is posted before the attention of step t is enqueued, so
the transfer of the next block runs beside the attention of the current one (over NVLink /
NVSwitch with NCCL).  The attention kernel is persistent and fills every SM it runs on,
so the ring asks the library to leave ``sm_reserve`` SMs free for NCCL's kernels
(``dit_set_sm_reserve``) while it runs, and sets the reserve back to 0 when it returns.

Block lengths may differ between ranks (an S that does not divide by P): lengths are
exchanged once on the host and every receive is posted with the sender's exact size.

``ring_attention_peers`` computes the same result without moving blocks at all: one launch
per rank reads every rank's K/V in place over peer memory (dit_attn_fwd_parts), the buffers
shared through CUDA IPC handles.

This module is plumbing around the C entry points: buffers, streams and the send/recv
schedule.  All arithmetic runs in the library's kernels (or, in the CPU tests of this
schedule, in the step functions those tests pass in).
"""

from __future__ import annotations

from typing import Optional, Sequence


class CudaRingOps:
    """The three calls one ring needs, on the library's kernels."""

    def __init__(self, scale: float, dtype: int, out_dtype=None, stream=None):
        self.scale, self.dtype, self.out_dtype, self.stream = scale, dtype, out_dtype, stream

    def init(self, acc, lse):
        from . import dit_attn_acc_init
        B, H, S, D = (int(x) for x in acc.shape)
        dit_attn_acc_init(acc, lse, B, H, S, D, self.stream)

    def step(self, q, k_blk, v_blk, s_kv: int, acc, lse, descale):
        from . import dit_attn_fwd_chunk_acc
        B, H, S_q, D = (int(x) for x in q.shape)
        if s_kv == 0:
            return
        dit_attn_fwd_chunk_acc(q, k_blk, v_blk, acc, lse, B, H, S_q, s_kv, D, 0, s_kv, self.scale,
                               self.dtype, descale, self.stream)

    def finish(self, acc, lse):
        import torch
        if self.out_dtype is None or self.out_dtype == torch.float32:
            return acc, lse
        from . import merge
        return merge([acc], [lse], out_dtype=self.out_dtype, stream=self.stream)


def _peer(group, idx: int) -> int:
    import torch.distributed as dist
    return idx if group is None else dist.get_global_rank(group, idx)


def ring_attention_dist(q, k, v, scale: Optional[float] = None, *, group=None, descale_qkv=None,
                        out_dtype=None, sm_reserve: int = 8, ops=None, block_lens: Optional[Sequence[int]] = None):
    """Attention of this rank's queries over the keys/values of every rank in ``group``.

    q          [B,H,S_q,D] this rank's query rows (bf16, or E4M3 codes as uint8).
    k, v       [B,H,S_r,D] this rank's key/value block (same dtype as q); S_r may differ
               between ranks; ranks hold blocks in rank order.
    descale_qkv  E4M3 only: this rank's 3-float device tensor {descale_q, descale_k,
               descale_v}; the k/v descales travel around the ring with their block.
    out_dtype  None or torch.float32: return the fp32 accumulator; torch.bfloat16: a final
               bf16 output (one dit_attn_merge over the single accumulator).
    ops        the step functions (default: the library's kernels, CudaRingOps).
    block_lens optional list of every rank's S_r (else exchanged on the host).

    Returns (out [B,H,S_q,D], lse [B,H,S_q] fp32).  Collective: every rank of the group must
    call it with the same B, H, D and dtype.
    """
    import torch
    import torch.distributed as dist

    B, H, S_q, D = (int(x) for x in q.shape)
    if tuple(k.shape[:2]) != (B, H) or int(k.shape[3]) != D or k.shape != v.shape:
        raise ValueError("k and v must be [B,H,S_r,D] with q's B, H and D")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k and v must be contiguous")
    fp8 = q.dtype == torch.uint8
    if fp8 and descale_qkv is None:
        raise ValueError("E4M3 inputs need descale_qkv")
    scale = (1.0 / D ** 0.5) if scale is None else float(scale)
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    if block_lens is None:
        lens = [None] * P
        dist.all_gather_object(lens, int(k.shape[2]), group=group)
    else:
        lens = [int(x) for x in block_lens]
    if len(lens) != P or lens[r] != int(k.shape[2]):
        raise ValueError("block_lens must list every rank's S_r")
    if ops is None:
        from . import DIT_BF16, DIT_FP8_E4M3
        ops = CudaRingOps(scale, DIT_FP8_E4M3 if fp8 else DIT_BF16, out_dtype)
    nxt, prv = _peer(group, (r + 1) % P), _peer(group, (r - 1) % P)

    acc = torch.empty((B, H, S_q, D), dtype=torch.float32, device=q.device)
    lse = torch.empty((B, H, S_q), dtype=torch.float32, device=q.device)
    ops.init(acc, lse)

    # Two spare (k, v, descale) slots: the block of step t+1 is received into the slot the
    # attention of step t-1 read, never into the one being sent or read now.
    s_max = max(lens)
    row = B * H * D
    spare = [(torch.empty(row * s_max, dtype=k.dtype, device=k.device),
              torch.empty(row * s_max, dtype=v.dtype, device=v.device),
              None if not fp8 else descale_qkv.clone()) for _ in range(2 if P > 2 else P - 1)]

    def view(slot, n):
        kb, vb, ds = slot
        return kb[: row * n].view(B, H, n, D), vb[: row * n].view(B, H, n, D), ds

    cur = (k, v, descale_qkv)
    lib_reserve = None
    if isinstance(ops, CudaRingOps) and P > 1:
        from . import dit_set_sm_reserve
        dit_set_sm_reserve(sm_reserve)
        lib_reserve = True
    try:
        for t in range(P):
            owner = (r - t) % P
            reqs = []
            if t + 1 < P:
                # send the block of `owner` on, receive the block of the next owner; a block
                # of length 0 is skipped by both of its ends alike
                nxt_len = lens[(r - t - 1) % P]
                slot = view(spare[t % len(spare)], nxt_len)
                p2p = []
                if lens[owner] > 0:
                    p2p += [dist.P2POp(dist.isend, cur[0].reshape(-1), nxt, group),
                            dist.P2POp(dist.isend, cur[1].reshape(-1), nxt, group)]
                if nxt_len > 0:
                    p2p += [dist.P2POp(dist.irecv, slot[0].reshape(-1), prv, group),
                            dist.P2POp(dist.irecv, slot[1].reshape(-1), prv, group)]
                if fp8:
                    p2p += [dist.P2POp(dist.isend, cur[2][1:3], nxt, group),
                            dist.P2POp(dist.irecv, slot[2][1:3], prv, group)]
                if p2p:
                    reqs = dist.batch_isend_irecv(p2p)
            ops.step(q, cur[0], cur[1], lens[owner], acc, lse, cur[2])
            for w in reqs:
                w.wait()
            if t + 1 < P:
                cur = slot
    finally:
        if lib_reserve:
            from . import dit_set_sm_reserve
            dit_set_sm_reserve(0)
    return ops.finish(acc, lse)


def ring_attention_peers(q, k, v, scale: Optional[float] = None, *, group=None, ops=None, out=None, lse=None):
    """The Ring dimension without a ring: one launch per rank reads every rank's K/V block in
    place over peer memory (dit_attn_fwd_parts with this rank's queries as the only query
    block), so no block travels and no partials are merged.

    q, k, v    [B,H,S_loc,D] bf16: this rank's rows (ranks hold consecutive rows, equal S_loc,
               a multiple of 128 when there is more than one rank).
    Buffers are shared with CUDA IPC through `ops` (ulysses.CudaPeerOps; pass the same one
    across calls to keep the peers' mappings open).  Barrier, launch, barrier.
    Returns (out [B,H,S_loc,D] bf16, lse [B,H,S_loc] fp32).  Collective over `group`.
    """
    import torch
    import torch.distributed as dist
    from .ulysses import CudaPeerOps

    B, H, S_loc, D = (int(x) for x in q.shape)
    if tuple(k.shape) != (B, H, S_loc, D) or k.shape != v.shape:
        raise ValueError("q, k and v must all be [B,H,S_loc,D]")
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    if P > 8:
        raise ValueError("at most 8 ranks")
    if P > 1 and S_loc % 128 != 0:
        raise ValueError(f"S_loc = {S_loc} rows per rank must be a multiple of 128")
    scale = (1.0 / D ** 0.5) if scale is None else float(scale)
    ops = CudaPeerOps() if ops is None else ops
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S_loc), dtype=torch.float32, device=q.device)
    everyone = [None] * P
    dist.all_gather_object(everyone, (S_loc, [ops.export(k), ops.export(v)]), group=group)
    if any(e[0] != S_loc for e in everyone):
        raise ValueError("every rank must hold the same number of rows")
    ks, vs = [], []
    for p_, (_, handles) in enumerate(everyone):
        if p_ == r:
            ks.append(k.data_ptr())
            vs.append(v.data_ptr())
        else:
            ks.append(ops.import_(p_, *handles[0]))
            vs.append(ops.import_(p_, *handles[1]))
    ops.sync()
    dist.barrier(group=group)                     # every rank's k, v are written
    ops.launch([q.data_ptr()], ks, vs, [out.data_ptr()], [lse.data_ptr()], B, H, 0, H, S_loc, D, scale)
    ops.sync()
    dist.barrier(group=group)                     # no rank overwrites its k, v while others read them
    return out, lse
