"""GPU parity of 3-D neighborhood attention (dit_na3d_fwd) against the fp64 oracle: grids
that are and are not multiples of the kernel's 4 x 4 x 8 bricks, windows from 1 to the whole
grid, D = 64 and 128, and the video grid at full size on sampled rows."""

import numpy as np
import pytest

import oracle
from oracle import neighborhood as onb
from gpu_util import assert_bf16_parity, host_f64, metrics, to_dev_bf16
from workloads import WORKLOADS, make_qkv, normal_bf16, sample_rows

pytestmark = pytest.mark.gpu


def _case(B, H, grid, D, seed):
    S = int(np.prod(grid))
    host, dev = [], []
    for i in range(3):
        x, bits = normal_bf16((B, H, S, D), seed + i)
        host.append(x)
        dev.append(to_dev_bf16(bits))
    return host, dev


@pytest.mark.parametrize("grid,kernel", [((3, 10, 20), (3, 5, 7)), ((1, 12, 16), (1, 5, 5)), ((5, 6, 9), (5, 5, 9)),
                                         ((4, 8, 8), (1, 1, 1)), ((1, 3, 5), (1, 3, 3)), ((6, 9, 17), (3, 7, 3)),
                                         ((8, 4, 16), (7, 3, 15))])
@pytest.mark.parametrize("D", [64, 128])
def test_na3d_matches_oracle(cuda_lib, grid, kernel, D):
    import torch
    host, dev = _case(1, 2, grid, D, seed=sum(grid) + D)
    scale = 1.0 / np.sqrt(D)
    out, lse = cuda_lib.neighborhood_attention(*dev, grid, kernel, scale)
    torch.cuda.synchronize()
    assert cuda_lib.dit_device_status() == 0
    ro, rl = onb.neighborhood_attention_3d(*host, grid, kernel, scale)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, (grid, kernel, D))


def test_na3d_whole_grid_window_is_dense_attention(cuda_lib):
    import torch
    grid = (3, 7, 9)
    host, dev = _case(2, 2, grid, 128, seed=5)
    out, lse = cuda_lib.neighborhood_attention(*dev, grid, grid, 0.1)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, 0.1)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, "whole grid")


def test_na3d_video_grid_sampled_rows(cuda_lib):
    import torch
    w = WORKLOADS["video"]
    grid, kernel = (21, 30, 52), (7, 7, 7)
    assert int(np.prod(grid)) == w.S
    d = make_qkv(w)
    dev = [to_dev_bf16(d[n + "_bits"]) for n in "qkv"]
    out, lse = cuda_lib.neighborhood_attention(*dev, grid, kernel, w.scale)
    torch.cuda.synchronize()
    assert cuda_lib.dit_device_status() == 0
    heads = [0, 13, 39]
    rows = sorted(set(sample_rows(w.S, 48, seed=9).tolist()) | {0, w.S - 1, 52 * 30 - 1, 52 * 29})
    ro, rl = onb.neighborhood_attention_3d(d["q"][:, heads], d["k"][:, heads], d["v"][:, heads], grid, kernel,
                                           w.scale, rows=rows)
    og = host_f64(out[:, heads][:, :, rows])
    lg = lse[:, heads][:, :, rows].cpu().numpy().astype(np.float64)
    m = metrics(og, ro, lg, rl)
    assert_bf16_parity(m, "video na3d")


@pytest.mark.parametrize("kernel", [(2, 3, 3), (3, 3, 4), (5, 3, 3), (1, 0, 1)])
def test_na3d_rejects_bad_windows(cuda_lib, kernel):
    import torch
    x = torch.zeros((1, 1, 3 * 4 * 5, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cuda_lib.DitError) as e:
        cuda_lib.neighborhood_attention(x, x.clone(), x.clone(), (3, 4, 5), kernel, 0.1)
    assert e.value.status == cuda_lib.DIT_ERR_INVALID_ARG


@pytest.mark.parametrize("gain,scale", [(8.0, None), (1.0, 1e-6)])
def test_na3d_score_extremes(cuda_lib, gain, scale):
    """Keys outside a window carry a -2^100 score penalty: scores 64x the usual size (inputs x8,
    exact in bf16) and a tiny softmax scale must still give exactly the windowed softmax."""
    import torch
    grid, kernel, D = (6, 9, 17), (3, 7, 3), 128
    S = int(np.prod(grid))
    host, dev = [], []
    for i in range(3):
        x, bits = normal_bf16((1, 2, S, D), 40 + i)
        t = to_dev_bf16(bits)
        if i < 2:
            t = t * gain
            x = x * gain
        host.append(x)
        dev.append(t.contiguous())
    scale = (1.0 / np.sqrt(D)) if scale is None else scale
    out, lse = cuda_lib.neighborhood_attention(*dev, grid, kernel, scale)
    torch.cuda.synchronize()
    assert cuda_lib.dit_device_status() == 0
    ro, rl = onb.neighborhood_attention_3d(*host, grid, kernel, scale)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, ("extremes", gain, scale))


def test_na3d_video_grid_d64_sampled_rows(cuda_lib):
    """D = 64 on the full video grid (many units per CTA, each Q tile's two-slot K / V rings
    wrap many times), 4 heads, sampled rows against the oracle."""
    import torch
    grid, kernel, D, H = (21, 30, 52), (7, 7, 7), 64, 4
    S = int(np.prod(grid))
    host, dev = _case(1, H, grid, D, seed=77)
    out, lse = cuda_lib.neighborhood_attention(*dev, grid, kernel, 1.0 / np.sqrt(D))
    torch.cuda.synchronize()
    assert cuda_lib.dit_device_status() == 0
    rows = sorted(set(sample_rows(S, 48, seed=11).tolist()) | {52 * 30 * 20, 52 * 30 - 1})
    heads = [0, 3]
    ro, rl = onb.neighborhood_attention_3d(host[0][:, heads], host[1][:, heads], host[2][:, heads], grid, kernel,
                                           1.0 / np.sqrt(D), rows=rows)
    m = metrics(host_f64(out[:, heads][:, :, rows]), ro, lse[:, heads][:, :, rows].cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, "video na3d D=64")
