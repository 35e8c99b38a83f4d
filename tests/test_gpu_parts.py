"""GPU parity of the fused Ulysses step (dit_attn_fwd_parts) with virtual ranks on one GPU.

Each virtual rank p holds its own [B, H, S_loc, D] Q, K, V and output buffers (separate
allocations, as they would be on separate GPUs).  Launch r reads heads [r*H/P, (r+1)*H/P) of
every rank's Q/K/V through per-part tensor maps and writes each output row into the rank
that holds it.  After the P launches every rank's output must equal the oracle's attention
over the concatenated sequence.  The launches never wait on one another: they only read the
inputs and write disjoint rows, so running them one after another on one GPU is the same
computation as running them on P GPUs at once."""

import numpy as np
import pytest

import oracle
from gpu_util import assert_bf16_parity, host_f64, metrics, to_dev_bf16
from workloads import normal_bf16

pytestmark = pytest.mark.gpu


def _ranks(P, B, H, S_loc, D, seed):
    full = [normal_bf16((B, H, P * S_loc, D), seed + i) for i in range(3)]
    dev = []
    for r in range(P):
        rows = slice(r * S_loc, (r + 1) * S_loc)
        dev.append([to_dev_bf16(np.ascontiguousarray(bits[:, :, rows])) for _, bits in full])
    return [x for x, _ in full], dev


@pytest.mark.parametrize("P,B,H,S_loc,D", [(1, 1, 4, 333, 128), (2, 1, 4, 256, 128), (4, 1, 8, 128, 128),
                                           (2, 2, 6, 384, 64), (3, 1, 3, 256, 128), (8, 1, 8, 128, 64)])
def test_parts_equal_full_attention(cuda_lib, P, B, H, S_loc, D):
    import torch
    host, dev = _ranks(P, B, H, S_loc, D, seed=P * 10 + D)
    outs = [torch.empty((B, H, S_loc, D), dtype=torch.bfloat16, device="cuda") for _ in range(P)]
    lses = [torch.empty((B, H, S_loc), dtype=torch.float32, device="cuda") for _ in range(P)]
    Hp = H // P
    scale = 1.0 / np.sqrt(D)
    for r in range(P):
        cuda_lib.dit_attn_fwd_parts([d[0] for d in dev], [d[1] for d in dev], [d[2] for d in dev], outs, lses,
                                    B, H, r * Hp, Hp, S_loc, D, scale)
    torch.cuda.synchronize()
    assert cuda_lib.dit_device_status() == 0
    ro, rl = oracle.attention(*host, scale)
    for r in range(P):
        rows = slice(r * S_loc, (r + 1) * S_loc)
        m = metrics(host_f64(outs[r]), ro[:, :, rows], lses[r].cpu().numpy().astype(np.float64), rl[:, :, rows])
        assert_bf16_parity(m, (P, B, H, S_loc, D, r))


def test_parts_matches_plain_call_bit_for_bit(cuda_lib):
    """With one part the call is the plain forward on the same tensor."""
    import torch
    host, dev = _ranks(1, 1, 2, 700, 128, seed=3)
    out = torch.empty((1, 2, 700, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 2, 700), dtype=torch.float32, device="cuda")
    cuda_lib.dit_attn_fwd_parts([dev[0][0]], [dev[0][1]], [dev[0][2]], [out], [lse], 1, 2, 0, 2, 700, 128, 0.1)
    o2, l2 = cuda_lib.attention(*dev[0], 0.1)
    torch.cuda.synchronize()
    assert torch.equal(out, o2) and torch.equal(lse, l2)


def test_parts_argument_checks(cuda_lib):
    import torch
    x = [torch.zeros((1, 4, 192, 128), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    o = [torch.empty_like(t) for t in x]
    with pytest.raises(cuda_lib.DitError) as e:      # 192 rows per part: tiles would straddle parts
        cuda_lib.dit_attn_fwd_parts(x, x, x, o, None, 1, 4, 0, 2, 192, 128, 0.1)
    assert e.value.status == cuda_lib.DIT_ERR_UNSUPPORTED
    with pytest.raises(cuda_lib.DitError) as e:      # heads past part_H
        cuda_lib.dit_attn_fwd_parts(x, x, x, o, None, 1, 4, 3, 2, 192, 128, 0.1)
    assert e.value.status == cuda_lib.DIT_ERR_INVALID_ARG


def test_peer_driver_single_rank_nccl(cuda_lib):
    """ulysses_attention_peers on a one-rank NCCL group: its own buffers, no IPC import (the
    exchange across ranks is covered by the shared-memory emulation on CPU)."""
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    from long_sequence_attention_b200.ulysses import ulysses_attention_peers
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    host, dev = _ranks(1, 2, 4, 300, 128, seed=17)
    try:
        out, lse = ulysses_attention_peers(*dev[0], 0.1)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ro, rl = oracle.attention(*host, 0.1)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, "peer driver, one rank")


def test_ipc_export_reports_offset_inside_allocation(cuda_lib):
    """The exported offset of a pointer inside a larger allocation is its distance from the
    allocation's start (importing needs another process, so only the export side runs here)."""
    import torch
    big = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    h0, off0 = cuda_lib.dit_ipc_export(big)
    h1, off1 = cuda_lib.dit_ipc_export(big[4096:])
    assert len(h0) == 64 and h0 == h1 and off1 - off0 == 4096


@pytest.mark.parametrize("P,B,H,S_loc,D", [(2, 1, 3, 256, 128), (4, 2, 2, 128, 64), (1, 1, 2, 300, 128)])
def test_ring_without_ring_equals_full_attention(cuda_lib, P, B, H, S_loc, D):
    """Each virtual rank: its own rows as the only query block, every rank's K/V as key blocks."""
    import torch
    host, dev = _ranks(P, B, H, S_loc, D, seed=P + 50)
    scale = 1.0 / np.sqrt(D)
    outs, lses = [], []
    for r in range(P):
        o = torch.empty((B, H, S_loc, D), dtype=torch.bfloat16, device="cuda")
        l = torch.empty((B, H, S_loc), dtype=torch.float32, device="cuda")
        cuda_lib.dit_attn_fwd_parts([dev[r][0]], [d[1] for d in dev], [d[2] for d in dev], [o], [l],
                                    B, H, 0, H, S_loc, D, scale)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    assert cuda_lib.dit_device_status() == 0
    ro, rl = oracle.attention(*host, scale)
    for r in range(P):
        rows = slice(r * S_loc, (r + 1) * S_loc)
        m = metrics(host_f64(outs[r]), ro[:, :, rows], lses[r].cpu().numpy().astype(np.float64), rl[:, :, rows])
        assert_bf16_parity(m, (P, r))
