"""GPU parity of the attention forward (full and KV-chunk) against the fp64 oracle.

Small and medium shapes are compared element by element; the full-size FLUX-2048 and video
workloads (in the same launch configuration the benchmark times) are compared on seeded
samples of query rows, which the oracle computes row by row.
"""

import numpy as np
import pytest

import oracle
from gpu_util import assert_bf16_parity, host_f64, metrics, to_dev_bf16
from workloads import WORKLOADS, chunk_bounds, make_qkv, normal_bf16, sample_rows

pytestmark = pytest.mark.gpu


def _case(B, H, Sq, Skv, D, seed, std=1.0):
    q, qb = normal_bf16((B, H, Sq, D), seed, std=std)
    k, kb = normal_bf16((B, H, Skv, D), seed + 1, std=std)
    v, vb = normal_bf16((B, H, Skv, D), seed + 2)
    return (q, k, v), (to_dev_bf16(qb), to_dev_bf16(kb), to_dev_bf16(vb))


def _check_full(lsa, host, dev, scale, what):
    import torch
    out, lse = lsa.attention(*dev, scale)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, scale)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, what)
    return out, lse


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("S", [1, 2, 77, 127, 128, 129, 255, 256, 257, 300, 513])
def test_full_edge_lengths(cuda_lib, S, D):
    host, dev = _case(2, 3, S, S, D, seed=10 * S + D)
    _check_full(cuda_lib, host, dev, 1.0 / np.sqrt(D), f"S={S} D={D}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Sq,Skv", [(300, 1000), (1000, 77), (129, 4096), (1, 640)])
def test_q_and_kv_lengths_differ(cuda_lib, Sq, Skv, D):
    import torch
    host, dev = _case(1, 2, Sq, Skv, D, seed=Sq + Skv + D)
    scale = 1.0 / np.sqrt(D)
    out, lse = cuda_lib.attention_chunk(*dev, 0, Skv, scale)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, scale)
    assert_bf16_parity(metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl), (Sq, Skv, D))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("k0,k1", [(0, 700), (0, 1), (13, 141), (128, 256), (650, 700), (699, 700),
                                   (1, 699), (300, 300), (0, 0), (700, 700)])
@pytest.mark.parametrize("out_fp32", [True, False])
def test_chunk_ranges(cuda_lib, k0, k1, D, out_fp32):
    import torch
    S = 700
    host, dev = _case(1, 2, S, S, D, seed=k0 * 7 + k1 + D)
    scale = 1.0 / np.sqrt(D)
    od = torch.float32 if out_fp32 else torch.bfloat16
    out, lse = cuda_lib.attention_chunk(*dev, k0, k1, scale, out_dtype=od)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, scale, k0, k1)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    if k0 == k1:
        assert m["max_abs"] == 0.0 and np.all(np.isneginf(lse.cpu().numpy()))
    else:
        assert_bf16_parity(m, (k0, k1, D, out_fp32))


@pytest.mark.parametrize("D", [64, 128])
def test_rising_scores_force_rescaling(cuda_lib, D):
    """Key norms grow along the sequence, so every KV tile raises the row max by far more
    than the lazy-rescale threshold: exercises the in-place O correction on every tile."""
    S = 1024
    q, _ = normal_bf16((1, 2, S, D), 31)
    k, _ = normal_bf16((1, 2, S, D), 32)
    v, _ = normal_bf16((1, 2, S, D), 33)
    growth = np.repeat(np.linspace(1.0, 12.0, S // 128), 128).astype(np.float32)
    from workloads import bf16_round
    k, kb = bf16_round(k * growth[None, None, :, None])
    q, qb = bf16_round(q * np.float32(2.0))
    v, vb = bf16_round(v)
    host = (q, k, v)
    dev = (to_dev_bf16(qb), to_dev_bf16(kb), to_dev_bf16(vb))
    _check_full(cuda_lib, host, dev, 1.0 / np.sqrt(D), "rising scores")


@pytest.mark.parametrize("D", [64, 128])
def test_dominant_key_far_above_running_max(cuda_lib, D):
    """A key in a later KV tile whose score beats the running max of the earlier tiles by
    about 180 log2 units, in the columns the FMA-pipe exp2 serves at D = 64 (tile 1 column 0,
    tile 2 column 16).  The speculative softmax must notice the rise and redo the tile
    exactly; the oracle's result is that key's V row for the aligned query rows."""
    from workloads import bf16_round
    S, H = 512, 2
    scale = 1.0 / np.sqrt(D)
    q, _ = normal_bf16((1, H, S, D), 41)
    k, _ = normal_bf16((1, H, S, D), 42)
    v, vb = normal_bf16((1, H, S, D), 43)
    u, _ = normal_bf16((D,), 44)
    gap_raw = 180.0 / (scale * np.log2(np.e))             # 180 log2 units above ~0
    alpha = np.float32(gap_raw / np.linalg.norm(u.astype(np.float64)))
    q[:, :, 0:256] = u                                     # both Q tiles of the first unit
    k[:, 0, 128] = alpha * u / np.linalg.norm(u)           # head 0: tile 1, column 0
    k[:, 1, 272] = alpha * u / np.linalg.norm(u)           # head 1: tile 2, column 16
    q, qb = bf16_round(q)
    k, kb = bf16_round(k)
    host = (q, k, v)
    dev = (to_dev_bf16(qb), to_dev_bf16(kb), to_dev_bf16(vb))
    out, _ = _check_full(cuda_lib, host, dev, scale, f"dominant key D={D}")
    o = host_f64(out)
    assert np.max(np.abs(o[0, 0, :256] - v[0, 0, 128].astype(np.float64))) <= 2e-2
    assert np.max(np.abs(o[0, 1, :256] - v[0, 1, 272].astype(np.float64))) <= 2e-2


@pytest.mark.parametrize("scale", [1e-3, 0.05, 0.5])
def test_scale_range(cuda_lib, scale):
    host, dev = _case(1, 2, 520, 520, 128, seed=int(scale * 1000) + 5, std=2.0)
    _check_full(cuda_lib, host, dev, scale, f"scale={scale}")


def test_deterministic(cuda_lib):
    import torch
    host, dev = _case(1, 4, 1000, 1000, 128, seed=77)
    o1, l1 = cuda_lib.attention(*dev, 0.1)
    o2, l2 = cuda_lib.attention(*dev, 0.1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert cuda_lib.dit_device_status(clear=True) == 0


def test_tiny_workload_full_and_two_chunks(cuda_lib):
    import torch
    w = WORKLOADS["tiny"]
    d = make_qkv(w)
    host = (d["q"], d["k"], d["v"])
    dev = tuple(to_dev_bf16(d[n + "_bits"]) for n in "qkv")
    _check_full(cuda_lib, host, dev, w.scale, "tiny")
    parts = [cuda_lib.attention_chunk(*dev, a, b, w.scale) for a, b in chunk_bounds(w.S, w.n_chunks)]
    mo, ml = cuda_lib.merge([p[0] for p in parts], [p[1] for p in parts])
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, w.scale)
    assert_bf16_parity(metrics(host_f64(mo), ro, ml.cpu().numpy().astype(np.float64), rl), "tiny merged")
    for (a, b), (po, pl) in zip(chunk_bounds(w.S, w.n_chunks), parts):
        co, cl = oracle.attention(*host, w.scale, a, b)
        assert_bf16_parity(metrics(host_f64(po), co, pl.cpu().numpy().astype(np.float64), cl), ("tiny chunk", a, b))


@pytest.mark.parametrize("name", ["sd3_1024", "flux_1024"])
def test_medium_workloads_elementwise(cuda_lib, name):
    w = WORKLOADS[name]
    d = make_qkv(w)
    host = (d["q"], d["k"], d["v"])
    dev = tuple(to_dev_bf16(d[n + "_bits"]) for n in "qkv")
    _check_full(cuda_lib, host, dev, w.scale, name)


@pytest.fixture(scope="module")
def flux2k():
    w = WORKLOADS["flux_2048"]
    d = make_qkv(w)
    return w, d, tuple(to_dev_bf16(d[n + "_bits"]) for n in "qkv")


def test_flux2048_full_sampled_rows(cuda_lib, flux2k):
    import torch
    w, d, dev = flux2k
    out, lse = cuda_lib.attention(*dev, w.scale)
    torch.cuda.synchronize()
    rows = sample_rows(w.S, 192, seed=11).tolist()
    ro, rl = oracle.attention(d["q"], d["k"], d["v"], w.scale, rows=rows)
    m = metrics(host_f64(out[:, :, rows]), ro, lse[:, :, rows].cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, "flux_2048 full")
    assert torch.isfinite(out).all()


def test_flux2048_four_chunks_merged_sampled_rows(cuda_lib, flux2k):
    import torch
    w, d, dev = flux2k
    parts = [cuda_lib.attention_chunk(*dev, a, b, w.scale) for a, b in chunk_bounds(w.S, w.n_chunks)]
    mo, ml = cuda_lib.merge([p[0] for p in parts], [p[1] for p in parts])
    torch.cuda.synchronize()
    rows = sample_rows(w.S, 192, seed=12).tolist()
    ro, rl = oracle.attention(d["q"], d["k"], d["v"], w.scale, rows=rows)
    m = metrics(host_f64(mo[:, :, rows]), ro, ml[:, :, rows].cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, "flux_2048 4-chunk merge")
    for (a, b), (po, pl) in zip(chunk_bounds(w.S, w.n_chunks), parts):
        co, cl = oracle.attention(d["q"], d["k"], d["v"], w.scale, a, b, rows=rows[:48])
        m = metrics(host_f64(po[:, :, rows[:48]]), co, pl[:, :, rows[:48]].cpu().numpy().astype(np.float64), cl)
        assert_bf16_parity(m, ("flux_2048 chunk", a, b))


def test_video_full_sampled_rows(cuda_lib):
    import torch
    w = WORKLOADS["video"]
    d = make_qkv(w)
    dev = tuple(to_dev_bf16(d[n + "_bits"]) for n in "qkv")
    out, lse = cuda_lib.attention(*dev, w.scale)
    torch.cuda.synchronize()
    rows = sample_rows(w.S, 96, seed=13).tolist()
    ro, rl = oracle.attention(d["q"], d["k"], d["v"], w.scale, rows=rows)
    m = metrics(host_f64(out[:, :, rows]), ro, lse[:, :, rows].cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, "video bf16")
    assert torch.isfinite(out).all()
