"""Ulysses re-partition across ranks: the other sequence-parallel dimension of USP (xDiT
overview page, section 3.2.2; ``--ulysses_degree`` on the xDiT docs page).

Each of the P ranks holds S/P rows (tokens) of every head.  One all-to-all per tensor turns
that into all S rows of H/P heads, each rank computes full attention for its heads, and one
all-to-all on the output turns it back.  The attention needs no exchange of its own.

No re-layout copies at B = 1: the all-to-all over a [1, H, S/P, D] tensor sends head group p
(contiguous) to rank p, and delivers segment q of the sequence (the rows rank q held) as the
q-th contiguous piece, i.e. in the layout [P, H/P, S/P, D].  ``dit_attn_fwd_seg`` reads Q, K,
V in exactly that layout (a 4-D TMA map) and writes O in it, which is what the return
all-to-all sends: piece q goes back to rank q, which receives head group p as its p-th
piece, [P, H/P, S/P, D] = [H, S/P, D].  With B > 1 the piece for one peer is strided
([B][P][...]); ``dit_swap01_chunks`` makes it contiguous before the exchange and restores
[B][P][...] after the return.

Requirements: H divisible by P; every rank holds the same S/P rows, a multiple of 128 (the
kernel's tiles must not straddle two segments) unless P = 1; bf16 inputs.

``ulysses_attention_peers`` does the same step with no all-to-all at all: one launch per rank
reads its head group of every rank's Q/K/V straight from the peers' memory (plain TMA
loads into the reading CTA) and stores each output row into the rank it belongs to (dit_attn_fwd_parts), the
buffers shared through CUDA IPC handles.

This module is plumbing: buffers and collectives.  The attention and the copies run in the
library's kernels (or, in the CPU tests of this schedule, in the functions those tests pass
in).
"""

from __future__ import annotations

from typing import Optional


class CudaUlyssesOps:
    """The two device operations the re-partition needs, on the library's kernels."""

    def __init__(self, scale: float, out_dtype=None, stream=None):
        self.scale, self.out_dtype, self.stream = scale, out_dtype, stream

    def swap01(self, src, dst, d0: int, d1: int, chunk_elems: int):
        from . import dit_swap01_chunks
        dit_swap01_chunks(src, dst, d0, d1, chunk_elems * src.element_size(), self.stream)

    def attention_seg(self, q, k, v, out, lse, B: int, H: int, S: int, D: int, seg: int):
        import torch
        from . import DIT_BF16, DIT_FP32, dit_attn_fwd_seg
        dit_attn_fwd_seg(q, k, v, out, lse, B, H, S, D, seg, self.scale, DIT_BF16,
                         DIT_FP32 if out.dtype == torch.float32 else DIT_BF16, None, self.stream)


def ulysses_attention_dist(q, k, v, scale: Optional[float] = None, *, group=None, out_dtype=None,
                           with_lse: bool = True, ops=None):
    """Attention over the whole sequence for a sequence split across the ranks of ``group``.

    q, k, v    [B,H,S_loc,D] this rank's rows of every head (bf16, contiguous); the full
               sequence is the ranks' rows in rank order.
    out_dtype  torch.bfloat16 (default) or torch.float32.
    Returns (out [B,H,S_loc,D], lse [B,H,S_loc] fp32 or None) for this rank's rows.
    Collective: every rank of the group calls it with the same shapes.
    """
    import torch
    import torch.distributed as dist

    B, H, S_loc, D = (int(x) for x in q.shape)
    if tuple(k.shape) != (B, H, S_loc, D) or k.shape != v.shape:
        raise ValueError("q, k and v must all be [B,H,S_loc,D]")
    if not (q.is_contiguous() and k.is_contiguous() and v.is_contiguous()):
        raise ValueError("q, k and v must be contiguous")
    P = dist.get_world_size(group)
    if H % P != 0:
        raise ValueError(f"H = {H} heads do not divide over {P} ranks")
    if P > 1 and S_loc % 128 != 0:
        raise ValueError(f"S_loc = {S_loc} rows per rank must be a multiple of 128")
    lens = [None] * P
    dist.all_gather_object(lens, S_loc, group=group)
    if any(n != S_loc for n in lens):
        raise ValueError(f"every rank must hold the same number of rows, got {lens}")
    Hp, S = H // P, P * S_loc
    scale = (1.0 / D ** 0.5) if scale is None else float(scale)
    odt = torch.bfloat16 if out_dtype is None else out_dtype
    if ops is None:
        ops = CudaUlyssesOps(scale, odt)
    piece = Hp * S_loc * D                         # elements one rank sends one peer, per batch

    def to_peers(x):
        """[B][P][piece] -> contiguous [P][B][piece] (a view when B = 1 or P = 1)."""
        if B == 1 or P == 1:
            return x.reshape(-1)
        buf = torch.empty(x.numel(), dtype=x.dtype, device=x.device)
        ops.swap01(x.reshape(-1), buf, B, P, piece)
        return buf

    recv = []
    for x in (q, k, v):
        r = torch.empty(x.numel(), dtype=x.dtype, device=x.device)
        dist.all_to_all_single(r, to_peers(x), group=group)
        recv.append(r)
    # received: [P(source rank = sequence segment)][B][Hp][S_loc][D], the segmented layout
    out_seg = torch.empty(P * B * Hp * S_loc * D, dtype=odt, device=q.device)
    lse_seg = torch.empty(P * B * Hp * S_loc, dtype=torch.float32, device=q.device) if with_lse else None
    ops.attention_seg(recv[0], recv[1], recv[2], out_seg, lse_seg, B, Hp, S, D, S_loc)
    del recv

    def back(seg_buf, per_row):
        """Return exchange of a [P][B][Hp][S_loc](*per_row) buffer -> [B][H][S_loc](*per_row)."""
        r = torch.empty_like(seg_buf)
        dist.all_to_all_single(r, seg_buf, group=group)
        if B == 1 or P == 1:
            return r
        out = torch.empty_like(r)
        ops.swap01(r, out, P, B, Hp * S_loc * per_row)
        return out

    out = back(out_seg, D).view(B, H, S_loc, D)
    lse = back(lse_seg, 1).view(B, H, S_loc) if with_lse else None
    return out, lse


class CudaPeerOps:
    """Buffer sharing and the fused launch for ulysses_attention_peers, on the library."""

    def __init__(self):
        self._opened = {}                 # (rank, handle) -> (base of the mapped allocation)

    def export(self, t):
        from . import dit_ipc_export
        return dit_ipc_export(t)

    def import_(self, rank: int, handle: bytes, offset: int) -> int:
        from . import dit_ipc_import
        key = (rank, handle)
        if key not in self._opened:
            _, base = dit_ipc_import(handle, 0)
            self._opened[key] = base
        return self._opened[key] + offset

    def close(self):
        from . import dit_ipc_close
        for base in self._opened.values():
            dit_ipc_close(base)
        self._opened.clear()

    def sync(self):
        import torch
        torch.cuda.synchronize()

    def launch(self, qs, ks, vs, outs, lses, B, H, h0, Hp, rows, D, scale):
        from . import dit_attn_fwd_parts
        dit_attn_fwd_parts(qs, ks, vs, outs, lses, B, H, h0, Hp, rows, D, scale)


def ulysses_attention_peers(q, k, v, scale: Optional[float] = None, *, group=None, ops=None, out=None, lse=None):
    """The Ulysses step as one kernel over peer memory (dit_attn_fwd_parts): no all-to-all.

    q, k, v    [B,H,S_loc,D] bf16, this rank's rows of every head (ranks hold consecutive rows).
    out, lse   optional output buffers [B,H,S_loc,D] bf16 / [B,H,S_loc] fp32 (allocated if None).
    Every rank exports its q, k, v, out and lse through CUDA IPC, opens the others' (kept
    open by `ops` across calls: pass the same CudaPeerOps to reuse them), and after a barrier
    runs one launch for its head group [rank*H/P, (rank+1)*H/P): its tiles are loaded by TMA
    from the ranks that hold the rows, and its output rows are stored into the ranks they
    belong to.  A second barrier makes every rank's out complete before it returns.
    Returns (out, lse) for this rank's rows.  Collective over `group`.
    """
    import torch
    import torch.distributed as dist

    B, H, S_loc, D = (int(x) for x in q.shape)
    if tuple(k.shape) != (B, H, S_loc, D) or k.shape != v.shape:
        raise ValueError("q, k and v must all be [B,H,S_loc,D]")
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    if H % P != 0:
        raise ValueError(f"H = {H} heads do not divide over {P} ranks")
    if P > 1 and S_loc % 128 != 0:
        raise ValueError(f"S_loc = {S_loc} rows per rank must be a multiple of 128")
    if P > 8:
        raise ValueError("at most 8 ranks")
    scale = (1.0 / D ** 0.5) if scale is None else float(scale)
    ops = CudaPeerOps() if ops is None else ops
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, S_loc), dtype=torch.float32, device=q.device)
    mine = [q, k, v, out, lse]
    exported = [ops.export(t) for t in mine]
    everyone = [None] * P
    dist.all_gather_object(everyone, (S_loc, exported), group=group)
    if any(e[0] != S_loc for e in everyone):
        raise ValueError("every rank must hold the same number of rows")
    ptrs = []                                     # ptrs[p] = (q, k, v, out, lse) addresses of rank p
    for p_, (_, handles) in enumerate(everyone):
        if p_ == r:
            ptrs.append([t.data_ptr() for t in mine])
        else:
            ptrs.append([ops.import_(p_, h, off) for h, off in handles])
    Hp = H // P
    ops.sync()
    dist.barrier(group=group)                     # every rank's q, k, v are written
    ops.launch([x[0] for x in ptrs], [x[1] for x in ptrs], [x[2] for x in ptrs], [x[3] for x in ptrs],
               [x[4] for x in ptrs], B, H, r * Hp, Hp, S_loc, D, scale)
    ops.sync()
    dist.barrier(group=group)                     # every rank's rows of out are written
    return out, lse
