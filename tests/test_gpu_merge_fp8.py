"""GPU parity of the LSE merge and of the FP8-E4M3 path (quantiser bit for bit; attention on
E4M3 inputs within the FP8 tolerance), plus the bounded-wait self-test."""

import numpy as np
import pytest

import oracle
from oracle import fp8 as ofp8
from gpu_util import assert_fp8_parity, assert_bf16_parity, host_f64, metrics, to_dev_bf16, to_dev_u8
from workloads import WORKLOADS, make_qkv, normal_bf16, sample_rows

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------------ merge
@pytest.mark.parametrize("n", [1, 2, 3, 4, 7, 16])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("in_fp32,out_fp32", [(True, False), (False, False), (True, True), (False, True)])
def test_merge_random_partials(cuda_lib, n, D, in_fp32, out_fp32):
    import torch
    B, H, S = 2, 3, 333
    rng = np.random.default_rng(n * 100 + D)
    outs_h, lses_h = [], []
    for c in range(n):
        o, _ = normal_bf16((B, H, S, D), 1000 + c)
        l = rng.normal(0.0, 4.0, size=(B, H, S)).astype(np.float32)
        if c % 3 == 1:
            l[:, :, ::5] = -np.inf                      # empty chunk on some rows
        outs_h.append(o)
        lses_h.append(l)
    if n >= 2:
        for c in range(n):
            lses_h[c][0, 0, 7] = -np.inf                # a row with every chunk empty
    dt = torch.float32 if in_fp32 else torch.bfloat16
    outs = [torch.from_numpy(o).to("cuda").to(dt) for o in outs_h]
    lses = [torch.from_numpy(l).to("cuda") for l in lses_h]
    mo, ml = cuda_lib.merge(outs, lses, out_dtype=torch.float32 if out_fp32 else torch.bfloat16)
    torch.cuda.synchronize()
    ro, rl = oracle.merge(outs_h, lses_h)
    m = metrics(host_f64(mo), ro, ml.cpu().numpy().astype(np.float64), rl)
    assert_bf16_parity(m, (n, D, in_fp32, out_fp32))
    if n >= 2:
        assert np.all(host_f64(mo)[0, 0, 7] == 0.0) and np.isneginf(ml[0, 0, 7].item())
    if out_fp32:
        assert m["max_abs"] < 1e-5 and m["lse_max_abs"] < 1e-5


def test_merge_of_empty_and_full_chunk_is_identity(cuda_lib):
    import torch
    host_o, _ = normal_bf16((1, 2, 129, 64), 5)
    o = torch.from_numpy(host_o).cuda()
    l = torch.randn(1, 2, 129, device="cuda")
    z = torch.zeros_like(o)
    ninf = torch.full_like(l, float("-inf"))
    mo, ml = cuda_lib.merge([z, o, z], [ninf, l, ninf], out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(mo, o) and torch.allclose(ml, l, atol=1e-6, rtol=0)


@pytest.mark.parametrize("n", [2, 5])
def test_merge_ignores_garbage_in_empty_chunks(cuda_lib, n):
    """An empty chunk (lse = -inf) has weight 0: whatever its out buffer holds (NaN, inf)
    must not reach the result."""
    import torch
    B, H, S, D = 1, 2, 130, 128
    good_o, _ = normal_bf16((B, H, S, D), 77)
    good_l = np.random.default_rng(1).normal(size=(B, H, S)).astype(np.float32)
    outs_h = [good_o] + [np.full((B, H, S, D), np.nan, dtype=np.float32) for _ in range(n - 1)]
    outs_h[-1][..., ::2] = np.inf
    lses_h = [good_l] + [np.full((B, H, S), -np.inf, dtype=np.float32) for _ in range(n - 1)]
    outs = [torch.from_numpy(o).cuda() for o in outs_h]
    lses = [torch.from_numpy(l).cuda() for l in lses_h]
    mo, ml = cuda_lib.merge(outs, lses, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.isfinite(mo).all()
    assert torch.equal(mo.cpu(), torch.from_numpy(good_o))
    assert torch.allclose(ml.cpu(), torch.from_numpy(good_l), atol=1e-6, rtol=0)


# ------------------------------------------------------------------------------ E4M3 quantiser
def _quant_dev(lsa, x_bits):
    import torch
    x = to_dev_bf16(x_bits)
    codes, descale = lsa.quantize_fp8(x)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), np.float32(descale.item())


def test_quant_bit_exact_on_ties_and_subnormals(cuda_lib):
    """448 is in the tensor, so descale = 1 and the codes are the plain encodings of every
    E4M3 value, every midpoint between neighbours (ties go to the even code), values just
    off the midpoints, the subnormal range, signed zero and values past 448 (saturate)."""
    from workloads import bf16_round
    pos = ofp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2
    vals = np.concatenate([pos, mids, mids * (1 + 2 ** -7), mids * (1 - 2 ** -7), [2.0 ** -10, 2.0 ** -11, 0.0]])
    vals = np.concatenate([vals, -vals, [-0.0, 448.0]])
    x, bits = bf16_round(vals.astype(np.float32))
    assert np.max(np.abs(x)) == 448.0
    codes, descale = _quant_dev(cuda_lib, bits)
    ref_codes, ref_descale = ofp8.quantize_per_tensor(x)
    assert descale == ref_descale == np.float32(1.0)
    assert np.array_equal(codes, ref_codes)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 4096 + 3, 1 << 20, (1 << 24) + 5])
def test_quant_bit_exact_random(cuda_lib, n):
    """(At 2^24 elements about 250 quotients fall within 8 fp32 ulps of an E4M3 rounding
    midpoint, where the quantiser leaves its reciprocal product for the IEEE division.)"""
    x, bits = normal_bf16((n,), 50 + n, std=3.0)
    codes, descale = _quant_dev(cuda_lib, bits)
    ref_codes, ref_descale = ofp8.quantize_per_tensor(x)
    assert descale == ref_descale
    assert np.array_equal(codes, ref_codes)


def test_quant_all_zero(cuda_lib):
    codes, descale = _quant_dev(cuda_lib, np.zeros(1000, dtype=np.uint16))
    assert descale == np.float32(1.0) and np.all(codes == 0)


# ------------------------------------------------------------------------------ FP8 attention
def _fp8_case(lsa, qkv_host, qkv_bits):
    import torch
    codes, descales, deq = [], [], []
    for x, b in zip(qkv_host, qkv_bits):
        c = lsa.quantize_fp8(to_dev_bf16(b))
        codes.append(c[0])
        descales.append(c[1])
    torch.cuda.synchronize()
    ds = torch.cat(descales)
    for x, c, d in zip(qkv_host, codes, descales):
        # oracle side: its own quantisation of the same bf16 values (bit-identical codes)
        rc, rd = ofp8.quantize_per_tensor(x)
        assert np.float32(d.item()) == rd
        deq.append(ofp8.dequantize(rc, rd))
    return codes, ds, deq


@pytest.mark.parametrize("S", [1, 129, 700, 2048])
def test_fp8_attention_small(cuda_lib, S):
    import torch
    D = 128
    host, bits = zip(*[normal_bf16((1, 3, S, D), 60 + S + i) for i in range(3)])
    codes, ds, deq = _fp8_case(cuda_lib, host, bits)
    for c, h in zip(codes, host):
        assert np.array_equal(c.cpu().numpy(), ofp8.quantize_per_tensor(h)[0])
    scale = 1.0 / np.sqrt(D)
    out, lse = cuda_lib.attention(*codes, scale, descale_qkv=ds)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*deq, scale)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_fp8_parity(m)


def test_fp8_chunk_and_merge(cuda_lib):
    import torch
    D, S = 128, 1000
    host, bits = zip(*[normal_bf16((1, 2, S, D), 90 + i) for i in range(3)])
    codes, ds, deq = _fp8_case(cuda_lib, host, bits)
    scale = 1.0 / np.sqrt(D)
    parts = [cuda_lib.attention_chunk(*codes, a, b, scale, descale_qkv=ds) for a, b in [(0, 333), (333, 1000)]]
    mo, ml = cuda_lib.merge([p[0] for p in parts], [p[1] for p in parts])
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*deq, scale)
    m = metrics(host_f64(mo), ro, ml.cpu().numpy().astype(np.float64), rl)
    assert_fp8_parity(m)


def test_fp8_video_sampled_rows(cuda_lib):
    import torch
    w = WORKLOADS["video"]
    d = make_qkv(w)
    host = (d["q"], d["k"], d["v"])
    bits = (d["q_bits"], d["k_bits"], d["v_bits"])
    codes = []
    descales = []
    for b in bits:
        c, s = cuda_lib.quantize_fp8(to_dev_bf16(b))
        codes.append(c)
        descales.append(s)
    torch.cuda.synchronize()
    ds = torch.cat(descales)
    out, lse = cuda_lib.attention(*codes, w.scale, descale_qkv=ds)
    torch.cuda.synchronize()
    rows = sample_rows(w.S, 64, seed=21).tolist()
    heads = [0, 17, 39]
    deq = []
    for x, c, s in zip(host, codes, descales):
        rd = ofp8.absmax_descale(x)
        assert np.float32(s.item()) == rd
        # codes of the sampled heads, bit for bit, from the oracle's own quantiser
        sub = x[:, heads]
        rc = ofp8.e4m3_encode((sub / rd).astype(np.float32))
        assert np.array_equal(c[:, heads].cpu().numpy(), rc)
        deq.append(ofp8.dequantize(rc, rd))
    ro, rl = oracle.attention(deq[0], deq[1], deq[2], w.scale, rows=rows)
    og = host_f64(out[:, heads][:, :, rows])
    lg = lse[:, heads][:, :, rows].cpu().numpy().astype(np.float64)
    m = metrics(og, ro, lg, rl)
    assert_fp8_parity(m)
    # for context: error against the bf16-input oracle
    rb, _ = oracle.attention(d["q"][:, heads], d["k"][:, heads], d["v"][:, heads], w.scale, rows=rows)
    print("fp8 video vs dequantised oracle", m, "vs bf16 oracle rel_l2",
          float(np.linalg.norm(og - rb) / np.linalg.norm(rb)))


# ------------------------------------------------------------------------------ bounded waits
def test_bounded_wait_gives_up_and_reports_timeout(cuda_lib):
    assert cuda_lib.dit_device_status(clear=True) == 0
    cuda_lib.dit_selftest_wait_timeout(20000)          # 20 ms on a barrier nothing arrives at
    st = cuda_lib.dit_device_status(clear=True)
    assert st & 0xFF == cuda_lib.DIT_ERR_TIMEOUT and (st >> 8) & 0xFF == 0xEE
    assert cuda_lib.dit_device_status(clear=True) == 0
