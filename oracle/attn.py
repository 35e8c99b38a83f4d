"""fp64 oracle: joint self-attention and the LSE merge of KV-chunk partials.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this module.

What the source pages fix, and what is a reading
------------------------------------------------
* DiT inference is prefill-like from start to finish: no decode phase, no KV cache,
  every token of the sequence is processed at once (xDiT overview, section 2.1
  "computation pattern comparison").  Image/video patch tokens are joined with text
  tokens and all of them attend to all of them, so attention is non-causal with no
  padding mask.  The pages never print the formula; the plain reading used here is
  out_i = sum_j softmax_j(s * q_i . k_j) v_j.
* The Ring dimension of USP splits the sequence into blocks and passes them around a
  ring (xDiT overview, section 3.2.2 "USP hybrid design", Ring dimension; xDiT docs,
  ``--ring_degree``).  The pages do not print how per-block partial results are
  combined; the exact combination is the log-sum-exp merge in ``merge`` below.
* LSE is the natural log of sum_j exp(s * q_i . k_j) over the keys of the range.
* An empty KV range gives out = 0 and lse = -inf (a reading: the empty sum).

Every quantity is computed in float64 from inputs that are exactly representable
(bf16 values, or E4M3 codes times a float32 descale), so the only rounding is fp64's.
"""

from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

NEG_INF = -np.inf
_ROW_BLOCK = 256  # query rows per block: the S x S score matrix is never held whole


def _as_f64(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def softmax_rows(q_rows: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """Explicit softmax rows P_ij = exp(x_ij - m_i) / sum_j exp(x_ij - m_i), with
    x_ij = scale * q_i . k_j, for one (b, h): q_rows [R, D], k [N, D] -> P [R, N].
    """
    x = float(scale) * (_as_f64(q_rows) @ _as_f64(k).T)
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=1, keepdims=True)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
              k0: int = 0, k1: Optional[int] = None,
              rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Non-causal multi-head attention over the keys k0 <= j < k1, in fp64.

    q: [B, H, S_q, D]; k, v: [B, H, S_kv, D] (any real dtype; converted to fp64).
    rows: optional query-row subset (same for every b, h).
    Returns (out [B, H, R, D] fp64, lse [B, H, R] fp64), R = S_q or len(rows).

    For each (b, h) and query row i:
        x_ij = scale * sum_d q_id k_jd
        m_i = max_j x_ij
        P_ij = exp(x_ij - m_i) / sum_j exp(x_ij - m_i)     (full row, not online)
        out_i = sum_j P_ij v_j
        lse_i = m_i + log sum_j exp(x_ij - m_i)
    """
    B, H, S_q, D = q.shape
    S_kv = k.shape[2]
    if k1 is None:
        k1 = S_kv
    if not (0 <= k0 <= k1 <= S_kv):
        raise ValueError(f"bad KV range [{k0}, {k1}) for S_kv={S_kv}")
    row_idx = np.arange(S_q) if rows is None else np.asarray(rows, dtype=np.int64)
    R = len(row_idx)
    out = np.zeros((B, H, R, v.shape[3]), dtype=np.float64)
    lse = np.full((B, H, R), NEG_INF, dtype=np.float64)
    if k1 == k0:
        return out, lse
    for b in range(B):
        for h in range(H):
            kk = _as_f64(k[b, h, k0:k1])
            vv = _as_f64(v[b, h, k0:k1])
            for r0 in range(0, R, _ROW_BLOCK):
                sel = row_idx[r0:r0 + _ROW_BLOCK]
                o_blk, l_blk = _row_block(_as_f64(q[b, h, sel]), kk, vv, float(scale))
                out[b, h, r0:r0 + len(sel)] = o_blk
                lse[b, h, r0:r0 + len(sel)] = l_blk
    return out, lse


def _row_block(qb: np.ndarray, kk: np.ndarray, vv: np.ndarray,
               scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """One block of query rows against the whole KV range: (out [R, D], lse [R])."""
    x = scale * (qb @ kk.T)
    m = x.max(axis=1, keepdims=True)
    e = np.exp(x - m)
    den = e.sum(axis=1, keepdims=True)
    p = e / den
    return p @ vv, (m + np.log(den))[:, 0]


def merge(outs: Sequence[np.ndarray], lses: Sequence[np.ndarray]) -> Tuple[np.ndarray, np.ndarray]:
    """Exact combination of per-chunk partials (out_c, lse_c), c = 0..n-1, in fp64.

    M = max_c lse_c;  w_c = exp(lse_c - M);  L = sum_c w_c;
    lse = M + log L;  out = sum_c (w_c / L) out_c.
    Rows whose lse_c are all -inf (every chunk empty) give out = 0, lse = -inf.

    outs: n arrays [..., D]; lses: n arrays [...] (same leading shape).
    """
    if len(outs) != len(lses) or len(outs) == 0:
        raise ValueError("need n >= 1 matching partials")
    L_stack = np.stack([_as_f64(l) for l in lses])           # [n, ...]
    O_stack = np.stack([_as_f64(o) for o in outs])           # [n, ..., D]
    M = L_stack.max(axis=0)                                   # [...]
    empty = np.isneginf(M)
    M_safe = np.where(empty, 0.0, M)
    w = np.where(np.isneginf(L_stack), 0.0, np.exp(L_stack - M_safe))  # [n, ...]
    Lsum = w.sum(axis=0)
    Lsum_safe = np.where(empty, 1.0, Lsum)
    out = (w[..., None] * O_stack).sum(axis=0) / Lsum_safe[..., None]
    out = np.where(empty[..., None], 0.0, out)
    lse = np.where(empty, NEG_INF, M_safe + np.log(Lsum_safe))
    return out, lse
