"""GPU parity of the per-block E4M3 path: the 128-row block quantiser bit for bit against the
oracle's, and attention on per-block-scaled inputs against the fp64 oracle on the same
dequantised values (FP8 tolerance)."""

import numpy as np
import pytest

import oracle
from oracle import fp8 as ofp8
from gpu_util import assert_fp8_parity, host_f64, metrics, to_dev_bf16
from workloads import WORKLOADS, make_qkv, normal_bf16, sample_rows

pytestmark = pytest.mark.gpu


def _quant(lsa, bits):
    import torch
    codes, ds = lsa.quantize_fp8_blocks(to_dev_bf16(bits))
    torch.cuda.synchronize()
    return codes, ds


@pytest.mark.parametrize("shape", [(1, 2, 300, 128), (2, 3, 129, 64), (1, 1, 128, 8), (1, 1, 1, 16), (3, 1, 513, 128)])
def test_block_quant_bit_exact(cuda_lib, shape):
    x, bits = normal_bf16(shape, 7 + shape[2], std=2.0)
    x = x.copy()
    bits = bits.copy()
    if shape[2] > 128:                                     # an outlier run and an all-zero block
        x[0, 0, 130:140] *= 300.0
        from workloads import bf16_round
        x, bits = bf16_round(x)
        x = x.copy()
        bits = bits.copy()
        bits[-1, -1, 128:256] = 0
        x[-1, -1, 128:256] = 0.0
    codes, ds = _quant(cuda_lib, bits)
    rc, rd = ofp8.quantize_per_block(x)
    assert np.array_equal(ds.cpu().numpy(), rd)
    assert np.array_equal(codes.cpu().numpy(), rc)


def _blocks_case(lsa, B, H, Sq, Skv, seed, head_gain=None):
    from workloads import bf16_round
    host, dev, descs, deq = [], [], [], []
    for i, S in enumerate((Sq, Skv, Skv)):
        x, _ = normal_bf16((B, H, S, 128), seed + i)
        if head_gain is not None:
            x = x * head_gain[None, :, None, None]
        x, bits = bf16_round(x.astype(np.float32))
        c, d = _quant(lsa, bits)
        rc, rd = ofp8.quantize_per_block(x)
        assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(d.cpu().numpy(), rd)
        host.append(x)
        dev.append(c)
        descs.append(d)
        deq.append(ofp8.dequantize_per_block(rc, rd))
    return host, dev, descs, deq


@pytest.mark.parametrize("Sq,Skv", [(1, 1), (129, 129), (700, 700), (300, 2048), (2048, 513)])
def test_block_fp8_attention_matches_oracle(cuda_lib, Sq, Skv):
    import torch
    _, dev, ds, deq = _blocks_case(cuda_lib, 1, 3, Sq, Skv, seed=Sq + Skv)
    scale = 1.0 / np.sqrt(128)
    out, lse = cuda_lib.attention_fp8_blocks(*dev, *ds, scale)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*deq, scale)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_fp8_parity(m)


@pytest.mark.parametrize("k0,k1", [(0, 700), (256, 700), (128, 129), (640, 700)])
def test_block_fp8_chunk_fp32(cuda_lib, k0, k1):
    import torch
    _, dev, ds, deq = _blocks_case(cuda_lib, 2, 2, 333, 700, seed=k0 + 3)
    scale = 0.1
    out, lse = cuda_lib.attention_fp8_blocks(*dev, *ds, scale, k0=k0, k1=k1, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(deq[0], deq[1][:, :, k0:k1], deq[2][:, :, k0:k1], scale)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_fp8_parity(m)


def test_block_fp8_all_zero_v_block(cuda_lib):
    """A V block of zeros has descale 0; its tile keeps r = 1 and contributes only to the row
    sums, as the oracle's zero values do."""
    import torch
    from workloads import bf16_round
    _, dev, ds, deq = _blocks_case(cuda_lib, 1, 2, 300, 500, seed=40)
    v = deq[2].copy()
    v[:, :, 128:256] = 0.0
    x, bits = bf16_round(v.astype(np.float32))
    codes, dv = _quant(cuda_lib, bits)
    assert np.all(dv.cpu().numpy()[:, :, 1] == 0.0)
    out, lse = cuda_lib.attention_fp8_blocks(dev[0], dev[1], codes, ds[0], ds[1], dv, 0.1, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rc, rd = ofp8.quantize_per_block(x)
    ro, rl = oracle.attention(deq[0], deq[1], ofp8.dequantize_per_block(rc, rd), 0.1)
    m = metrics(host_f64(out), ro, lse.cpu().numpy().astype(np.float64), rl)
    assert_fp8_parity(m)


def test_block_scales_beat_per_tensor_on_uneven_heads(cuda_lib):
    """Heads of very different magnitude (one 2^16 times louder): one per-tensor scale pushes
    the quiet heads' codes into the subnormal range, per-block scales do not.  Error against
    the bf16-input oracle (which includes E4M3's own rounding, a few percent)."""
    import torch
    gain = np.array([1.0, 1.0, 65536.0, 1.0], dtype=np.float32)
    host, dev, ds, deq = _blocks_case(cuda_lib, 1, 4, 512, 512, seed=77, head_gain=gain)
    scale = 1.0 / np.sqrt(128)
    ob, _ = cuda_lib.attention_fp8_blocks(*dev, *ds, scale, out_dtype=torch.float32)
    # the same inputs through the per-tensor path
    from workloads import bf16_round
    codes, descs = [], []
    for x in host:
        c, d = cuda_lib.quantize_fp8(to_dev_bf16(bf16_round(x)[1]))
        codes.append(c)
        descs.append(d)
    ot, _ = cuda_lib.attention(*codes, scale, descale_qkv=torch.cat(descs))
    torch.cuda.synchronize()
    ref, _ = oracle.attention(*host, scale)
    quiet = [0, 1, 3]
    eb = np.linalg.norm(host_f64(ob)[:, quiet] - ref[:, quiet]) / np.linalg.norm(ref[:, quiet])
    et = np.linalg.norm(host_f64(ot)[:, quiet] - ref[:, quiet]) / np.linalg.norm(ref[:, quiet])
    print("quiet heads rel-L2 vs bf16 oracle: per-block", eb, "per-tensor", et)
    assert eb < 0.1 and eb < 0.5 * et


def test_block_fp8_video_sampled_rows(cuda_lib):
    import torch
    w = WORKLOADS["video"]
    d = make_qkv(w)
    heads = [0, 21, 39]
    rows = sample_rows(w.S, 48, seed=5).tolist()
    codes, descs, deq = [], [], []
    for n in "qkv":
        c, s = cuda_lib.quantize_fp8_blocks(to_dev_bf16(d[n + "_bits"]))
        torch.cuda.synchronize()
        sub = d[n][:, heads]
        rc, rd = ofp8.quantize_per_block(sub)
        assert np.array_equal(s[:, heads].cpu().numpy(), rd)
        assert np.array_equal(c[:, heads].cpu().numpy(), rc)
        codes.append(c)
        descs.append(s)
        deq.append(ofp8.dequantize_per_block(rc, rd))
    out, lse = cuda_lib.attention_fp8_blocks(*codes, *descs, w.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.attention(*deq, w.scale, rows=rows)
    og = host_f64(out[:, heads][:, :, rows])
    lg = lse[:, heads][:, :, rows].cpu().numpy().astype(np.float64)
    m = metrics(og, ro, lg, rl)
    assert_fp8_parity(m)


def test_block_fp8_argument_checks(cuda_lib):
    import torch
    _, dev, ds, _ = _blocks_case(cuda_lib, 1, 1, 256, 256, seed=1)
    with pytest.raises(cuda_lib.DitError) as e:
        cuda_lib.attention_fp8_blocks(*dev, *ds, 0.1, k0=64, k1=256)
    assert e.value.status == cuda_lib.DIT_ERR_UNSUPPORTED
    out = torch.empty((1, 1, 256, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 1, 256), dtype=torch.float32, device="cuda")
    rc = cuda_lib.lib.dit_attn_fwd_fp8_blocks(dev[0].data_ptr(), dev[1].data_ptr(), dev[2].data_ptr(),
                                              ds[0].data_ptr(), None, ds[2].data_ptr(), out.data_ptr(),
                                              lse.data_ptr(), 1, 1, 256, 256, 128, 0, 256, 0.1, 0, None)
    assert rc == cuda_lib.DIT_ERR_INVALID_ARG
