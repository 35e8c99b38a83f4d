"""dit_quant_fp8_noalloc against dit_quant_fp8.

Some callers cannot allocate device memory at the point where they quantise (for example
while capturing a CUDA graph, or under a framework allocator that forbids raw cudaMalloc),
so they cannot provide the workspace dit_quant_fp8 needs.  dit_quant_fp8_noalloc keeps its
scratch in a static array inside the library instead.  This test calls it through the C ABI
twice in a row, on inputs of different sizes and ranges (so stale scratch from the first call
would show up in the second), and checks both results against the workspace entry point and
against the oracle's own quantiser (so a fault shared by both CUDA quantisers cannot pass):
E4M3 codes and descale are byte work, so the tolerance is exact equality.

The file is named to be collected last: it must pass on its own in a fresh process (where its
first call does the per-device set-up) and after every other test.
"""

import ctypes

import numpy as np
import pytest

from gpu_util import to_dev_bf16
from oracle import fp8 as ofp8
from workloads import normal_bf16

pytestmark = pytest.mark.gpu


def _with_workspace(lsa, x, n):
    import torch
    codes = torch.empty((n,), dtype=torch.uint8, device="cuda")
    descale = torch.empty((1,), dtype=torch.float32, device="cuda")
    ws_bytes = lsa.dit_quant_fp8_workspace_bytes(n)
    ws = torch.empty((ws_bytes // 4,), dtype=torch.float32, device="cuda")
    lsa.dit_quant_fp8(x, codes, descale, n, ws, ws_bytes)
    return codes, descale


def _no_alloc_via_c_abi(lsa, x, n):
    import torch
    codes = torch.full((n,), 0xAB, dtype=torch.uint8, device="cuda")
    descale = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = lsa.lib.dit_quant_fp8_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(codes.data_ptr()),
                                       ctypes.c_void_p(descale.data_ptr()), ctypes.c_longlong(n),
                                       ctypes.c_void_p(stream))
    assert rc == 0, lsa.status_str(rc)
    return codes, descale


def test_no_alloc_quant_matches_workspace_entry_point_on_two_calls(cuda_lib):
    import torch
    # call 1: many blocks and a large range; call 2: fewer blocks and a small range
    cases = [((1 << 22) + 5, 4.0, 301), ((1 << 16) + 3, 0.25, 302)]
    for n, std, seed in cases:
        host, bits = normal_bf16((n,), seed, std=std)
        x = to_dev_bf16(bits)
        ref_codes, ref_descale = _with_workspace(cuda_lib, x, n)
        codes, descale = _no_alloc_via_c_abi(cuda_lib, x, n)
        torch.cuda.synchronize()
        assert torch.equal(descale, ref_descale), (n, descale.item(), ref_descale.item())
        assert torch.equal(codes, ref_codes), n
        oracle_codes, oracle_descale = ofp8.quantize_per_tensor(host)
        assert np.float32(descale.item()) == oracle_descale, (n, descale.item(), oracle_descale)
        assert np.array_equal(codes.cpu().numpy(), oracle_codes), n
    assert cuda_lib.dit_device_status(clear=True) == 0


def test_no_alloc_rejects_bad_arguments(cuda_lib):
    import torch
    x = torch.zeros((64,), dtype=torch.bfloat16, device="cuda")
    c = torch.zeros((64,), dtype=torch.uint8, device="cuda")
    d = torch.zeros((1,), dtype=torch.float32, device="cuda")
    f = cuda_lib.lib.dit_quant_fp8_noalloc
    assert f(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(d.data_ptr()),
             ctypes.c_longlong(0), None) == cuda_lib.DIT_ERR_INVALID_ARG
    assert f(None, ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(d.data_ptr()), ctypes.c_longlong(64),
             None) == cuda_lib.DIT_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(x.data_ptr() + 2), ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(d.data_ptr()),
             ctypes.c_longlong(32), None) == cuda_lib.DIT_ERR_MISALIGNED
