"""Run one kernel of the library on seeded synthetic device inputs, a given number of times.

    python -m long_sequence_attention_b200.cases <case> [--reps N] [--shape B,H,S,D]
        [--grid T,Y,X --window Kt,Ky,Kx]

For profiling (a profiler can capture the n-th launch of a known kernel without the rest of a
benchmark) and quick timing: prints the average time per call from CUDA events.  Cases:

    attn          dit_attn_fwd, bf16
    chunk         dit_attn_fwd_chunk over the second quarter of the keys, fp32 out
    merge         dit_attn_merge of 4 fp32 partials
    quant         dit_quant_fp8 (per tensor) of one tensor
    quant_blocks  dit_quant_fp8_blocks of one tensor
    fp8           dit_attn_fwd on E4M3 codes (per-tensor descales)
    seg           dit_attn_fwd_seg with 4 segments
    parts         dit_attn_fwd_parts: 4 ranks' blocks in separate buffers, one launch per rank
                  (each for a quarter of the heads; on one GPU the launches run one after another)
    na3d          dit_na3d_fwd on a T x Y x X grid

Inputs are N(0,1) drawn on the device (torch), rounded to bf16: this is a timing and
profiling driver, not a parity check (the tests compare every call with the oracle).
"""

from __future__ import annotations

import argparse


def main(argv=None) -> None:
    import torch
    import long_sequence_attention_b200 as lsa

    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["attn", "chunk", "merge", "quant", "quant_blocks", "fp8", "seg", "parts",
                                     "na3d"])
    ap.add_argument("--reps", type=int, default=2)
    ap.add_argument("--shape", default="1,24,16896,128", help="B,H,S,D")
    ap.add_argument("--grid", default="21,30,52", help="T,Y,X (na3d; S = T*Y*X)")
    ap.add_argument("--window", default="7,7,7", help="Kt,Ky,Kx (na3d)")
    a = ap.parse_args(argv)
    B, H, S, D = (int(x) for x in a.shape.split(","))
    grid = tuple(int(x) for x in a.grid.split(","))
    window = tuple(int(x) for x in a.window.split(","))
    if a.case == "na3d":
        S = grid[0] * grid[1] * grid[2]
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(0)

    def rnd():
        return torch.randn((B, H, S, D), generator=g, device=dev).to(torch.bfloat16)

    scale = D ** -0.5
    st = torch.cuda.current_stream().cuda_stream
    if a.case in ("attn", "chunk", "fp8", "seg", "na3d"):
        q, k, v = rnd(), rnd(), rnd()
    if a.case == "attn":
        out, lse = torch.empty_like(q), torch.empty((B, H, S), device=dev)
        call = lambda: lsa.dit_attn_fwd(q, k, v, out, lse, B, H, S, D, scale, lsa.DIT_BF16, None, st)
    elif a.case == "chunk":
        out, lse = torch.empty((B, H, S, D), device=dev), torch.empty((B, H, S), device=dev)
        call = lambda: lsa.dit_attn_fwd_chunk(q, k, v, out, lse, B, H, S, S, D, S // 4, S // 2, scale, lsa.DIT_BF16,
                                              lsa.DIT_FP32, None, st)
    elif a.case == "merge":
        parts = [torch.randn((B, H, S, D), generator=g, device=dev) for _ in range(4)]
        lses = [torch.randn((B, H, S), generator=g, device=dev) for _ in range(4)]
        out, lse = torch.empty((B, H, S, D), dtype=torch.bfloat16, device=dev), torch.empty((B, H, S), device=dev)
        call = lambda: lsa.dit_attn_merge(parts, lses, out, lse, B, H, S, D, lsa.DIT_FP32, lsa.DIT_BF16, st)
    elif a.case in ("quant", "quant_blocks"):
        x = rnd()
        codes = torch.empty(x.shape, dtype=torch.uint8, device=dev)
        if a.case == "quant":
            n = x.numel()
            ds = torch.empty(1, device=dev)
            wsb = lsa.dit_quant_fp8_workspace_bytes(n)
            ws = torch.empty(wsb // 4 + 1, device=dev)
            call = lambda: lsa.dit_quant_fp8(x, codes, ds, n, ws, wsb, st)
        else:
            ds = torch.empty((B, H, (S + 127) // 128), device=dev)
            call = lambda: lsa.dit_quant_fp8_blocks(x, codes, ds, B, H, S, D, st)
    elif a.case == "fp8":
        qs = [lsa.quantize_fp8(t) for t in (q, k, v)]
        codes = [c for c, _ in qs]
        ds = torch.cat([d for _, d in qs])
        out, lse = torch.empty_like(q), torch.empty((B, H, S), device=dev)
        call = lambda: lsa.dit_attn_fwd(*codes, out, lse, B, H, S, D, scale, lsa.DIT_FP8_E4M3, ds, st)
    elif a.case == "seg":
        P = 4
        seg = S // P
        out, lse = torch.empty_like(q), torch.empty((B, H, S), device=dev)
        call = lambda: lsa.dit_attn_fwd_seg(q, k, v, out, lse, B, H, S, D, seg, scale, lsa.DIT_BF16, lsa.DIT_BF16,
                                            None, st)
    elif a.case == "parts":
        P = 4
        rows = S // P
        blocks = [[torch.randn((B, H, rows, D), generator=g, device=dev).to(torch.bfloat16) for _ in range(3)]
                  for _ in range(P)]
        outs = [torch.empty((B, H, rows, D), dtype=torch.bfloat16, device=dev) for _ in range(P)]
        lses = [torch.empty((B, H, rows), device=dev) for _ in range(P)]

        def call():
            for r in range(P):
                lsa.dit_attn_fwd_parts([b[0] for b in blocks], [b[1] for b in blocks], [b[2] for b in blocks], outs,
                                       lses, B, H, r * (H // P), H // P, rows, D, scale, st)
    else:
        out, lse = torch.empty_like(q), torch.empty((B, H, S), device=dev)
        call = lambda: lsa.dit_na3d_fwd(q, k, v, out, lse, B, H, *grid, D, *window, scale, st)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.reps):
        call()
    e1.record()
    torch.cuda.synchronize()
    status = lsa.dit_device_status()
    print(f"{a.case}: {e0.elapsed_time(e1) / a.reps:.4f} ms per call over {a.reps} calls, device status {status}")
    if status != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
