"""Helpers shared by the GPU parity tests: uploading seeded bf16 inputs, error metrics and
the tolerances the parity bar is stated in."""

import numpy as np

# Parity bar (per output tensor, against the fp64 oracle on the same inputs):
BF16_REL_L2 = 5e-3     # || gpu - ref ||_2 / || ref ||_2
BF16_MAX_ABS = 2e-2    # max_i | gpu_i - ref_i |
LSE_MAX_ABS = 1e-3     # max_i | lse_gpu_i - lse_ref_i |
FP8_REL_L2 = 5e-2      # FP8-E4M3 inputs: vs the oracle on the dequantised inputs


def to_dev_bf16(bits_u16: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).view(torch.bfloat16).to(device)


def to_dev_u8(codes: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes)).to(device)


def host_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def metrics(out_gpu: np.ndarray, out_ref: np.ndarray, lse_gpu=None, lse_ref=None):
    diff = out_gpu - out_ref
    m = {
        "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(out_ref), 1e-300)),
        "max_abs": float(np.max(np.abs(diff))) if diff.size else 0.0,
    }
    if lse_gpu is not None:
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lse_gpu), fin), "lse finiteness differs"
        assert np.array_equal(lse_gpu[~fin], lse_ref[~fin]), "non-finite lse values differ"
        m["lse_max_abs"] = float(np.max(np.abs(lse_gpu[fin] - lse_ref[fin]))) if fin.any() else 0.0
    return m


def assert_fp8_parity(m, what=""):
    """FP8-E4M3 inputs: rel-L2 against the oracle on the dequantised inputs, and the same LSE
    bar as bf16 (the row sums are formed in fp32 before P is rounded to E4M3, so the LSE
    carries no FP8 rounding)."""
    assert m["rel_l2"] <= FP8_REL_L2, (what, m)
    assert "lse_max_abs" in m, (what, "FP8 parity needs the LSE compared too")
    assert m["lse_max_abs"] <= LSE_MAX_ABS, (what, m)


def assert_bf16_parity(m, what=""):
    assert m["rel_l2"] <= BF16_REL_L2, (what, m)
    assert m["max_abs"] <= BF16_MAX_ABS, (what, m)
    if "lse_max_abs" in m:
        assert m["lse_max_abs"] <= LSE_MAX_ABS, (what, m)
