"""GPU parity of the fused ring step (dit_attn_fwd_chunk_acc): a KV range's attention merged
into a running (O, LSE) accumulator in the kernel epilogue, against the fp64 oracle."""

import numpy as np
import pytest

import oracle
from oracle import fp8 as ofp8
from gpu_util import assert_fp8_parity, assert_bf16_parity, host_f64, metrics, to_dev_bf16
from workloads import WORKLOADS, chunk_bounds, make_qkv, normal_bf16, sample_rows

pytestmark = pytest.mark.gpu


def _case(B, H, Sq, Skv, D, seed):
    q, qb = normal_bf16((B, H, Sq, D), seed)
    k, kb = normal_bf16((B, H, Skv, D), seed + 1)
    v, vb = normal_bf16((B, H, Skv, D), seed + 2)
    return (q, k, v), (to_dev_bf16(qb), to_dev_bf16(kb), to_dev_bf16(vb))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bounds", [[(0, 700)], [(0, 350), (350, 700)], [(0, 129), (129, 130), (130, 700)],
                                    [(500, 700), (0, 0), (0, 500)], [(0, 128), (128, 256), (256, 384), (384, 700)],
                                    [(600, 700), (300, 600), (0, 300)]])
def test_ring_accumulate_equals_full_attention(cuda_lib, bounds, D):
    import torch
    host, dev = _case(1, 3, 300, 700, D, seed=D + len(bounds))
    scale = 1.0 / np.sqrt(D)
    out, lse = cuda_lib.ring_attention(*dev, bounds, scale)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, scale)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, (bounds, D))


def test_first_step_from_fwd_chunk_and_bf16_finish(cuda_lib):
    """First chunk written by dit_attn_fwd_chunk (fp32), later ones fused; final bf16 through
    dit_attn_merge with one input."""
    import torch
    host, dev = _case(2, 2, 257, 1000, 128, seed=9)
    scale = 0.1
    acc, acc_lse = cuda_lib.attention_chunk(*dev, 0, 400, scale)           # fp32 partial
    B, H, S_q, D = 2, 2, 257, 128
    for k0, k1 in [(400, 401), (401, 1000)]:
        cuda_lib.dit_attn_fwd_chunk_acc(*dev, acc, acc_lse, B, H, S_q, 1000, D, k0, k1, scale)
    ob, lb = cuda_lib.merge([acc], [acc_lse])                               # bf16 out
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, scale)
    assert_bf16_parity(metrics(host_f64(ob), ro, lb.cpu().numpy().astype(np.float64), rl), "bf16 finish")


def test_fp8_ring_accumulate(cuda_lib):
    import torch
    D, S = 128, 900
    host, bits = zip(*[normal_bf16((1, 2, S, D), 120 + i) for i in range(3)])
    codes, descales, deq = [], [], []
    for x, b in zip(host, bits):
        c, d = cuda_lib.quantize_fp8(to_dev_bf16(b))
        codes.append(c)
        descales.append(d)
        rc, rd = ofp8.quantize_per_tensor(x)
        deq.append(ofp8.dequantize(rc, rd))
    ds = torch.cat(descales)
    scale = 1.0 / np.sqrt(D)
    out, lse = cuda_lib.ring_attention(*codes, [(0, 300), (300, 600), (600, 900)], scale, descale_qkv=ds)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*deq, scale)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_fp8_parity(m)


def test_flux2048_four_fused_ring_steps_sampled_rows(cuda_lib):
    import torch
    w = WORKLOADS["flux_2048"]
    d = make_qkv(w)
    dev = tuple(to_dev_bf16(d[n + "_bits"]) for n in "qkv")
    out, lse = cuda_lib.ring_attention(*dev, chunk_bounds(w.S, w.n_chunks), w.scale)
    torch.cuda.synchronize()
    rows = sample_rows(w.S, 128, seed=31).tolist()
    ro, rl = oracle.attention(d["q"], d["k"], d["v"], w.scale, rows=rows)
    m = metrics(host_f64(out[:, :, rows]), ro, lse[:, :, rows].cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, "flux_2048 fused ring")


def test_empty_accumulator_ignores_garbage(cuda_lib):
    import torch
    host, dev = _case(1, 2, 130, 300, 128, seed=41)
    B, H, S_q, D = 1, 2, 130, 128
    acc = torch.full((B, H, S_q, D), float("nan"), device="cuda")
    acc_lse = torch.full((B, H, S_q), float("-inf"), device="cuda")
    for k0, k1 in [(0, 200), (200, 300)]:
        cuda_lib.dit_attn_fwd_chunk_acc(*dev, acc, acc_lse, B, H, S_q, 300, D, k0, k1, 0.1)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*host, 0.1)
    assert torch.isfinite(acc).all()
    assert_bf16_parity(metrics(host_f64(acc), ro, acc_lse.cpu().numpy().astype(np.float64), rl), "garbage acc")


def test_acc_argument_validation(cuda_lib):
    import torch
    x = torch.zeros((1, 1, 64, 64), dtype=torch.bfloat16, device="cuda")
    a = torch.zeros((1, 1, 64, 64), dtype=torch.float32, device="cuda")
    l = torch.zeros((1, 1, 64), dtype=torch.float32, device="cuda")
    f = cuda_lib.lib.dit_attn_fwd_chunk_acc
    assert f(x.data_ptr(), x.data_ptr(), x.data_ptr(), None, l.data_ptr(), 1, 1, 64, 64, 64, 0, 64, 0.1, 0, None, None) == 1
    assert f(x.data_ptr(), x.data_ptr(), x.data_ptr(), a.data_ptr(), l.data_ptr(), 1, 1, 64, 64, 64, 10, 5, 0.1, 0,
             None, None) == 1
    assert cuda_lib.lib.dit_attn_acc_init(a.data_ptr(), l.data_ptr(), 1, 1, 64, 96, None) == 2


def test_sm_reserve_leaves_results_bit_identical(cuda_lib):
    """A smaller persistent grid (SMs reserved for concurrent kernels) processes the same work
    units in another order per CTA; every unit's arithmetic is unchanged."""
    import torch
    host, dev = _case(2, 3, 900, 900, 128, seed=5)
    ref_o, ref_l = cuda_lib.attention(*dev, 0.09)
    try:
        cuda_lib.dit_set_sm_reserve(140)
        o, l = cuda_lib.attention(*dev, 0.09)
        torch.cuda.synchronize()
    finally:
        cuda_lib.dit_set_sm_reserve(0)
    assert torch.equal(o, ref_o) and torch.equal(l, ref_l)
    with pytest.raises(cuda_lib.DitError):
        cuda_lib.dit_set_sm_reserve(-1)


@pytest.mark.parametrize("out_bf16", [False, True])
def test_ring_driver_single_rank_nccl(cuda_lib, out_bf16):
    """The multi-rank ring driver on a one-rank NCCL group: one fused step over the local
    block (the send/recv schedule itself is covered by the gloo tests on CPU)."""
    import datetime
    import socket
    import torch
    import torch.distributed as dist
    from long_sequence_attention_b200.ring import ring_attention_dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=30))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        host, dev = _case(1, 4, 333, 333, 128, seed=8)
        out, lse = ring_attention_dist(*dev, 0.1, out_dtype=torch.bfloat16 if out_bf16 else None)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert out.dtype == (torch.bfloat16 if out_bf16 else torch.float32)
    ro, rl = oracle.attention(*host, 0.1)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, out_bf16)
