"""Seeded synthetic workloads for DiT joint attention.

This module is shared by the fp64 oracle tests and by the CUDA path's tests and
benchmark.  It holds no attention arithmetic: it only draws seeded N(0,1) numbers,
rounds them to bf16, and describes the workload shapes.

Workload shapes follow the DiT models the source pages name (xDiT docs page,
"Supported models": Flux.1 and Stable Diffusion 3; the Chinese xDiT overview,
section 2.2, "sequence length reaches millions of pixels/frames"; the AMD ROCm
summary, FP8 attention backend).  Joint attention concatenates image (or video)
patch tokens with text tokens, image first; with i.i.d. inputs the order does not
matter, so a workload is described by its total length S.

Seeds: Q uses seed 0, K seed 1, V seed 2 and the outlier-channel pick seed 3, each a
numpy PCG64 generator (``numpy.random.default_rng``).  Values are drawn as float32
N(0,1) and rounded once to bf16 with round-to-nearest-even.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

SEED_Q, SEED_K, SEED_V, SEED_OUTLIER = 0, 1, 2, 3


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    scale: float
    outlier_frac: float = 0.0      # fraction of the H*D key channels scaled x8
    n_chunks: int = 1              # KV chunks for the chunk + merge emulation (1 = none)
    fp8: bool = False              # also run as an FP8-E4M3 variant
    note: str = ""

    @property
    def flops(self) -> float:
        """4*B*H*S^2*D: the two GEMMs of attention, softmax not counted."""
        return 4.0 * self.B * self.H * self.S * self.S * self.D

    def describe(self) -> Dict[str, object]:
        return {"workload": self.name, "B": self.B, "H": self.H, "S": self.S,
                "D": self.D, "scale": self.scale}


WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("tiny", 1, 2, 256, 64, 1.0 / 8.0, n_chunks=2,
                 note="16x16 patch grid, no text; also 2 KV chunks of 128 merged"),
        Workload("sd3_1024", 2, 24, 4429, 64, 1.0 / math.sqrt(64.0),
                 note="SD3-medium 1024px: 4096 image + 333 text tokens, B=2 = CFG "
                      "cond/uncond stacked; ragged tail of 77 rows"),
        Workload("flux_1024", 1, 24, 4608, 128, 1.0 / math.sqrt(128.0), outlier_frac=0.01,
                 note="FLUX 1024px: 4096 image + 512 text tokens; 1% of K channels x8"),
        Workload("flux_2048", 1, 24, 16896, 128, 1.0 / math.sqrt(128.0), n_chunks=4,
                 note="FLUX 2048px: 16384 image + 512 text tokens; full and 4 KV chunks "
                      "of 4224 merged (single-GPU ring-step emulation)"),
        Workload("video", 1, 40, 32760, 128, 1.0 / math.sqrt(128.0), fp8=True,
                 note="video DiT: 21 latent frames x 30x52 patches; ragged tail of 120 "
                      "rows; plus an FP8-E4M3 variant with per-tensor absmax scales"),
    ]
}


def bf16_round(x: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Round float32 values to bf16 (round-to-nearest-even).

    Returns (values as float32, raw bf16 bit patterns as uint16).  Inputs must be
    finite (the generators only produce finite normals).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bits = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
            >> np.uint32(16)).astype(np.uint16)
    vals = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return vals, bits


def normal_bf16(shape: Sequence[int], seed: int, mean: float = 0.0,
                std: float = 1.0) -> Tuple[np.ndarray, np.ndarray]:
    """Seeded N(mean, std^2) float32 draw rounded to bf16: (float32 values, uint16 bits)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(size=tuple(shape), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if mean != 0.0:
        x += np.float32(mean)
    return bf16_round(x)


def outlier_channels(H: int, D: int, frac: float, seed: int = SEED_OUTLIER) -> np.ndarray:
    """The (h, d) key channels scaled x8: round(frac*H*D) of them, seeded permutation.

    Returns an int array of shape [n, 2] holding (h, d) pairs.
    """
    n = int(round(frac * H * D))
    if n == 0:
        return np.zeros((0, 2), dtype=np.int64)
    idx = np.random.default_rng(seed).permutation(H * D)[:n]
    return np.stack([idx // D, idx % D], axis=1)


def make_qkv(w: Workload, seed_offset: int = 0) -> Dict[str, np.ndarray]:
    """Q, K, V of a workload, [B,H,S,D].

    Keys ``q, k, v`` hold float32 arrays whose values are exactly bf16; ``q_bits,
    k_bits, v_bits`` hold the same values as uint16 bf16 bit patterns (what goes to
    the GPU).  ``seed_offset`` shifts all three seeds (used for extra test cases).
    """
    shape = (w.B, w.H, w.S, w.D)
    out: Dict[str, np.ndarray] = {}
    for name, seed in (("q", SEED_Q), ("k", SEED_K), ("v", SEED_V)):
        vals, bits = normal_bf16(shape, seed + seed_offset)
        out[name], out[name + "_bits"] = vals, bits
    if w.outlier_frac > 0.0:
        ch = outlier_channels(w.H, w.D, w.outlier_frac)
        k = out["k"]
        for h, d in ch:
            k[:, h, :, d] *= np.float32(8.0)   # power of two: stays exactly bf16
        out["k"], out["k_bits"] = bf16_round(k)
    return out


def make_tensor(shape: Sequence[int], seed: int, std: float = 1.0) -> np.ndarray:
    """A seeded bf16-valued float32 tensor of any shape (test helper)."""
    return normal_bf16(shape, seed, std=std)[0]


def to_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of a float32 array that already holds bf16 values."""
    vals, bits = bf16_round(x)
    if not np.array_equal(vals, np.asarray(x, dtype=np.float32)):
        raise ValueError("array does not hold bf16-representable values")
    return bits


def chunk_bounds(S: int, n: int) -> List[Tuple[int, int]]:
    """Half-open KV ranges [k0, k1) of n chunks: floor(S/n) keys each, the remainder
    in the last chunk."""
    if n < 1:
        raise ValueError("n must be >= 1")
    step = S // n
    bounds = [(i * step, (i + 1) * step) for i in range(n - 1)]
    bounds.append(((n - 1) * step, S))
    return bounds


def sample_rows(S: int, n_rows: int, seed: int = 7, include_tail: bool = True) -> np.ndarray:
    """Sorted seeded subset of query rows of one head, always including the first and
    the last row (the ragged tail) when ``include_tail``."""
    rng = np.random.default_rng(seed)
    n_rows = min(n_rows, S)
    rows = set(rng.choice(S, size=n_rows, replace=False).tolist())
    if include_tail:
        rows.update({0, S - 1})
    return np.array(sorted(rows), dtype=np.int64)
