"""E4M3 attention on key tensors with outlier channels: the FLUX-1024 workload, where 31 of
the 3072 (head, channel) key channels are scaled x8 (1% of K channels, the same channels for
every token).

The AMD ROCm summary page ("What is new", "Tuning guide") warns that the FP8 attention
backend changes outputs and that results must be compared on fixed seeds.  This study runs
the seeded FLUX-1024 tensors through both E4M3 granularities of the library, per tensor
(dit_quant_fp8 + dit_attn_fwd) and per 128-row block (dit_quant_fp8_blocks +
dit_attn_fwd_fp8_blocks), and reports two errors for each:

* the parity gate: against the fp64 oracle on the dequantised inputs the GPU actually saw
  (rel-L2 <= 5e-2, LSE <= 1e-3);
* the accuracy cost: against the fp64 oracle on the bf16 inputs, for the heads that hold an
  outlier channel and for the clean heads separately.

What the numbers show (and the last assertions hold): the heads with an outlier channel lose
about twice as much accuracy as the clean heads, and per-block scales barely change that.
Scales along tokens cannot isolate a channel; and since E4M3 keeps the same relative
precision over its whole normal range (under 0.1% of these K codes are subnormal), a
per-channel K scale, or moving a channel's scale into Q, would not help either: every
product q_d * k_d, and so the score error, stays the same.
"""

import numpy as np
import pytest

import oracle
from gpu_util import assert_fp8_parity, host_f64, metrics, to_dev_bf16
from oracle import fp8 as ofp8
from workloads import WORKLOADS, make_qkv, outlier_channels

pytestmark = pytest.mark.gpu


def _rel(a, b, heads):
    return float(np.linalg.norm(a[:, heads] - b[:, heads]) / np.linalg.norm(b[:, heads]))


def test_fp8_outlier_channels_flux_1024(cuda_lib):
    import torch
    w = WORKLOADS["flux_1024"]
    d = make_qkv(w)
    host = (d["q"], d["k"], d["v"])
    dev = [to_dev_bf16(d[n + "_bits"]) for n in "qkv"]
    loud = sorted({int(h) for h, _ in outlier_channels(w.H, w.D, w.outlier_frac)})
    clean = [h for h in range(w.H) if h not in loud]
    assert 0 < len(loud) < w.H

    # per tensor
    pt = [cuda_lib.quantize_fp8(x) for x in dev]
    o_t, l_t = cuda_lib.attention(*[c for c, _ in pt], w.scale, descale_qkv=torch.cat([s for _, s in pt]))
    # per 128-row block
    pb = [cuda_lib.quantize_fp8_blocks(x) for x in dev]
    o_b, l_b = cuda_lib.attention_fp8_blocks(*[c for c, _ in pb], *[s for _, s in pb], w.scale)
    torch.cuda.synchronize()

    deq_t, deq_b = [], []
    for x, (c, s), (cb, sb) in zip(host, pt, pb):
        rc, rd = ofp8.quantize_per_tensor(x)
        assert np.array_equal(c.cpu().numpy(), rc) and np.float32(s.item()) == rd
        deq_t.append(ofp8.dequantize(rc, rd))
        rcb, rdb = ofp8.quantize_per_block(x)
        assert np.array_equal(cb.cpu().numpy(), rcb) and np.array_equal(sb.cpu().numpy(), rdb)
        deq_b.append(ofp8.dequantize_per_block(rcb, rdb))

    ref_bf16, _ = oracle.attention(*host, w.scale)
    report = {}
    for name, o, l, deq in (("per_tensor", o_t, l_t, deq_t), ("per_block", o_b, l_b, deq_b)):
        ro, rl = oracle.attention(*deq, w.scale)
        og = host_f64(o)
        m = metrics(og, ro, l.cpu().numpy().astype(np.float64), rl)
        assert_fp8_parity(m, name)
        report[name] = {"gate_rel_l2": m["rel_l2"], "gate_lse": m["lse_max_abs"],
                        "vs_bf16_loud_heads": _rel(og, ref_bf16, loud),
                        "vs_bf16_clean_heads": _rel(og, ref_bf16, clean),
                        "input_quant_only_loud": _rel(ro, ref_bf16, loud),
                        "input_quant_only_clean": _rel(ro, ref_bf16, clean)}
    print("fp8 outlier-channel study (flux_1024):", report)
    for name, r in report.items():
        # the loud heads pay about twice the clean heads' accuracy cost ...
        assert r["vs_bf16_loud_heads"] > 1.5 * r["vs_bf16_clean_heads"], (name, r)
    # ... and scales along tokens recover little of it
    assert report["per_block"]["vs_bf16_loud_heads"] > 0.7 * report["per_tensor"]["vs_bf16_loud_heads"], report
