"""fp64 oracle: 3-D neighborhood attention on a token grid.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never imports this
module.

What the pages fix, and what is a reading
-----------------------------------------
The LTX notes page (section 5, on choosing a kernel that matches the operation) reports that
the diffusion decoder of the high-resolution pass spent most of its time in neighborhood
attention run through a general flex-attention implementation, and that NATTEN's prebuilt
3-D neighborhood attention kernel ("na3d") cut that decode from 293 s to 18.3 s and halved
its peak memory.  The page names the operation, not its parameters.  Readings:

* Tokens lie on a T x Y x X grid (frames, rows, columns), flattened frame-major:
  s = (t * Y + y) * X + x, the same [B, H, S, D] layout as the joint attention.
* The neighborhood of query (t, y, x) along a dimension of length L with odd kernel size
  K <= L is the K consecutive positions starting at clamp(i - K // 2, 0, L - K): a window
  of fixed size, centred on the query where it fits and shifted inward at the borders, so
  every query sees exactly K positions per dimension (NATTEN's definition, dilation 1,
  non-causal).  The 3-D neighborhood is the product of the three windows.
* out_i = sum_{j in N(i)} softmax_j(scale * q_i . k_j) v_j and
  lse_i = log sum_{j in N(i)} exp(scale * q_i . k_j), as for the joint attention.
"""

from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np


def window_start(i: int, K: int, L: int) -> int:
    """First position of the K-wide window of position i on a line of L positions."""
    if not (K % 2 == 1 and 1 <= K <= L):
        raise ValueError(f"kernel size {K} must be odd and at most {L}")
    return min(max(i - K // 2, 0), L - K)


def neighbor_index(grid: Sequence[int], kernel: Sequence[int], s: int) -> np.ndarray:
    """Flattened key indices of the neighborhood of token s (frame-major order)."""
    T, Y, X = grid
    Kt, Ky, Kx = kernel
    t, rem = divmod(int(s), Y * X)
    y, x = divmod(rem, X)
    ts = np.arange(window_start(t, Kt, T), window_start(t, Kt, T) + Kt)
    ys = np.arange(window_start(y, Ky, Y), window_start(y, Ky, Y) + Ky)
    xs = np.arange(window_start(x, Kx, X), window_start(x, Kx, X) + Kx)
    return ((ts[:, None, None] * Y + ys[None, :, None]) * X + xs[None, None, :]).reshape(-1)


def neighborhood_attention_3d(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: Sequence[int],
                              kernel: Sequence[int], scale: float,
                              rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Neighborhood attention in fp64.

    q, k, v: [B, H, S, D] with S = T * Y * X; grid = (T, Y, X); kernel = (Kt, Ky, Kx), odd,
    each at most its grid dimension.  rows: optional subset of query tokens.
    Returns (out [B, H, R, D], lse [B, H, R]) with an explicit softmax over each query's
    Kt * Ky * Kx neighbours.
    """
    B, H, S, D = q.shape
    if S != int(np.prod(grid)):
        raise ValueError(f"S = {S} is not T * Y * X = {int(np.prod(grid))}")
    row_idx = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    nbr = np.stack([neighbor_index(grid, kernel, s) for s in row_idx])       # [R, Kvol]
    out = np.zeros((B, H, len(row_idx), v.shape[3]), dtype=np.float64)
    lse = np.zeros((B, H, len(row_idx)), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            qq = np.asarray(q[b, h], dtype=np.float64)
            kk = np.asarray(k[b, h], dtype=np.float64)
            vv = np.asarray(v[b, h], dtype=np.float64)
            for r0 in range(0, len(row_idx), 64):
                sel = slice(r0, r0 + 64)
                kn = kk[nbr[sel]]                                            # [r, Kvol, D]
                x = float(scale) * np.einsum("rd,rkd->rk", qq[row_idx[sel]], kn)
                m = x.max(axis=1, keepdims=True)
                e = np.exp(x - m)
                den = e.sum(axis=1, keepdims=True)
                out[b, h, sel] = np.einsum("rk,rkd->rd", e / den, vv[nbr[sel]])
                lse[b, h, sel] = (m + np.log(den))[:, 0]
    return out, lse
