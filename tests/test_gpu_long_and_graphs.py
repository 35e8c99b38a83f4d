"""Long sequences (up to 2^20 tokens of one head) against the oracle on sampled rows, and the
library's calls captured in a CUDA graph (they allocate nothing and never synchronise)."""

import numpy as np
import pytest

import oracle
from gpu_util import assert_bf16_parity, host_f64, metrics, to_dev_bf16
from workloads import chunk_bounds, normal_bf16, sample_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,H,D", [(131072, 2, 128), (1 << 20, 1, 128), (262144 + 77, 1, 64)])
def test_long_sequence_sampled_rows(cuda_lib, S, H, D):
    """A single head at 128k and 1M tokens (and a ragged 256k + 77 at D = 64): thousands of KV
    tiles per unit, long runs of the lazy-max path, row indices far past 2^16."""
    import torch
    host, dev = [], []
    for i in range(3):
        x, bits = normal_bf16((1, H, S, D), 500 + i + S % 97)
        host.append(x)
        dev.append(to_dev_bf16(bits))
    out, lse = cuda_lib.attention(*dev, 1.0 / np.sqrt(D))
    torch.cuda.synchronize()
    assert cuda_lib.dit_device_status() == 0
    rows = sorted(set(sample_rows(S, 24, seed=S % 1000).tolist()) | {0, S - 1, S - 129})
    ro, rl = oracle.attention(*host, 1.0 / np.sqrt(D), rows=rows)
    m = metrics(host_f64(out[:, :, rows]), ro, lse[:, :, rows].cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, ("long", S, H, D))


def test_step_captured_in_cuda_graph(cuda_lib):
    """Full forward + 3 chunks + merge captured once and replayed on new inputs: the graph's
    results equal eager calls bit for bit."""
    import torch
    B, H, S, D = 1, 3, 1000, 128
    bounds = chunk_bounds(S, 3)
    q, k, v = (torch.empty((B, H, S, D), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    parts = [(torch.empty((B, H, S, D), dtype=torch.float32, device="cuda"),
              torch.empty((B, H, S), dtype=torch.float32, device="cuda")) for _ in bounds]
    mout = torch.empty_like(q)
    mlse = torch.empty_like(lse)

    def step(st):
        cuda_lib.dit_attn_fwd(q, k, v, out, lse, B, H, S, D, 0.09, cuda_lib.DIT_BF16, None, st)
        for (a, b), (po, pl) in zip(bounds, parts):
            cuda_lib.dit_attn_fwd_chunk(q, k, v, po, pl, B, H, S, S, D, a, b, 0.09, cuda_lib.DIT_BF16,
                                        cuda_lib.DIT_FP32, None, st)
        cuda_lib.dit_attn_merge([p[0] for p in parts], [p[1] for p in parts], mout, mlse, B, H, S, D,
                                cuda_lib.DIT_FP32, cuda_lib.DIT_BF16, st)

    def fill(seed):
        for i, t in enumerate((q, k, v)):
            _, bits = normal_bf16((B, H, S, D), seed + i)
            t.copy_(to_dev_bf16(bits))

    s = torch.cuda.Stream()
    fill(1)
    with torch.cuda.stream(s):
        step(s)                                   # warm-up outside capture (kernel attributes, maps)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(s)
    for seed in (10, 20):
        fill(seed)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (out, lse, mout, mlse)]
        with torch.cuda.stream(s):
            step(s)
        s.synchronize()
        for a, b in zip(got, (out, lse, mout, mlse)):
            assert torch.equal(a, b)
    assert cuda_lib.dit_device_status() == 0
