"""GPU parity of the Ulysses pieces: attention on the segmented layout an all-to-all over the
sequence leaves behind (dit_attn_fwd_seg), the batch/peer chunk transpose, and the driver on
a one-rank NCCL group.  The exchange schedule across ranks is covered by the gloo tests."""

import numpy as np
import pytest

import oracle
from gpu_util import assert_bf16_parity, host_f64, metrics
from workloads import normal_bf16

pytestmark = pytest.mark.gpu


def _seg(x, seg):
    """[B,H,S,D] -> [S/seg, B, H, seg, D] (row r of head bh at ((r//seg)*BH + bh)*seg + r%seg)."""
    B, H, S, D = x.shape
    return np.ascontiguousarray(x.reshape(B * H, S // seg, seg, D).transpose(1, 0, 2, 3))


def _unseg(y, B, H, S, D, seg):
    return y.reshape(S // seg, B * H, seg, D).transpose(1, 0, 2, 3).reshape(B, H, S, D)


@pytest.mark.parametrize("B,H,S,seg,D", [(1, 2, 512, 128, 128), (2, 3, 384, 128, 64), (1, 4, 1024, 256, 128),
                                         (2, 2, 333, 333, 128), (1, 1, 128, 128, 64)])
@pytest.mark.parametrize("fp32_out", [False, True])
def test_seg_layout_matches_oracle(cuda_lib, B, H, S, seg, D, fp32_out):
    import torch
    host = []
    dev = []
    for i in range(3):
        x, bits = normal_bf16((B, H, S, D), 300 + S + i)
        host.append(x)
        dev.append(torch.from_numpy(_seg(bits.view(np.int16), seg)).cuda().view(torch.bfloat16))
    out = torch.empty((S // seg, B, H, seg, D), dtype=torch.float32 if fp32_out else torch.bfloat16, device="cuda")
    lse = torch.empty((S // seg, B, H, seg), dtype=torch.float32, device="cuda")
    scale = 1.0 / np.sqrt(D)
    cuda_lib.dit_attn_fwd_seg(*dev, out, lse, B, H, S, D, seg, scale, 0, 2 if fp32_out else 0)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, scale)
    og = _unseg(host_f64(out), B, H, S, D, seg)
    lg = _unseg(lse.cpu().numpy().astype(np.float64)[..., None], B, H, S, 1, seg)[..., 0]
    m = metrics(og, ro, lg, rl)
    assert_bf16_parity(m, (B, H, S, seg, D))


def test_seg_equal_to_plain_layout_when_one_segment(cuda_lib):
    """seg == S is the plain layout: bit-identical to dit_attn_fwd."""
    import torch
    _, bits = normal_bf16((3, 1, 3, 700, 128), 9)
    q, k, v = [torch.from_numpy(b.view(np.int16)).cuda().view(torch.bfloat16) for b in bits]
    o1, l1 = cuda_lib.attention(q, k, v, 0.09)
    o2 = torch.empty_like(o1)
    l2 = torch.empty_like(l1)
    cuda_lib.dit_attn_fwd_seg(q, k, v, o2, l2, 1, 3, 700, 128, 700, 0.09)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_seg_rejects_straddling_segments(cuda_lib):
    import torch
    x = torch.zeros((2, 1, 1, 192, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(x)
    l = torch.empty((2, 1, 1, 192), dtype=torch.float32, device="cuda")
    with pytest.raises(cuda_lib.DitError) as e:
        cuda_lib.dit_attn_fwd_seg(x, x.clone(), x.clone(), o, l, 1, 1, 384, 128, 192, 0.1)
    assert e.value.status == cuda_lib.DIT_ERR_UNSUPPORTED


@pytest.mark.parametrize("d0,d1,chunk", [(2, 4, 16), (3, 5, 4096), (1, 7, 48), (8, 1, 160)])
def test_swap01_bit_exact(cuda_lib, d0, d1, chunk):
    import torch
    a = np.random.default_rng(d0 * d1).integers(0, 256, size=(d0, d1, chunk), dtype=np.uint8)
    src = torch.from_numpy(a.reshape(-1)).cuda()
    dst = torch.empty_like(src)
    cuda_lib.dit_swap01_chunks(src, dst, d0, d1, chunk)
    torch.cuda.synchronize()
    assert np.array_equal(dst.cpu().numpy(), a.transpose(1, 0, 2).reshape(-1))


@pytest.mark.parametrize("B", [1, 2])
def test_ulysses_driver_single_rank_nccl(cuda_lib, B):
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    from long_sequence_attention_b200.ulysses import ulysses_attention_dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    host, dev = [], []
    for i in range(3):
        x, bits = normal_bf16((B, 4, 300, 128), 40 + i)
        host.append(x)
        dev.append(torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16))
    try:
        out, lse = ulysses_attention_dist(*dev, 0.1)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ro, rl = oracle.attention(*host, 0.1)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, B)
